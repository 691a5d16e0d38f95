// CUDA-core split-K GEMV for the decode linear at small M (sm_100a).
//
//   y[m, n] = sum_k x[m, k] * deq(W)[n, k]      m < MM <= 4
//
// The weight stream is the whole cost of a decode step (gpt-fast write-up,
// m.greenbasetech.com article 46368139_1106049486, paragraph on the memory
// bandwidth bound: every generated token reads every weight once).  The kernel
// reads each packed byte exactly once and hides dequantization under the stream:
//
//  * A CTA owns a block of R output rows over its share of K.  When R would not
//    fill one stage (small N), a thread-block cluster splits K and its CTAs sum
//    the cluster's partials through distributed shared memory, each finishing a
//    slice of the rows (no scratch, a fixed order: the result is deterministic).
//  * K is cut into chunks of 32 lanes x LANE_K weights.  A stage of the
//    shared-memory ring holds one chunk of kJ rows per consumer warp plus, for
//    a chunk's first stage, that chunk of x, and (int4, when a row of scales is
//    a multiple of 16 bytes) the scales and zeros of the stage's rows.  A
//    producer warp (or, without one, the last consumer warp out of the stage)
//    fills the ring with 2-D tensor copies of 8-row boxes and bulk copies of x,
//    completing on the stage's mbarrier, ahead of the consumers.
//  * With a producer, a converter warp takes the stages in order as they land,
//    converts each chunk of x once per CTA, in place, to the packed fp32 pairs
//    the consumer lanes multiply with (int4: pre-scaled, plus each lane's sum),
//    and releases the stage on a second mbarrier; the consumers copy them into
//    registers, where they stay for the whole chunk.  Without a producer
//    (M >= 3) every consumer warp converts x itself.
//  * Each consumer lane reads its 16 bytes (FP6: 16 + 8) of a row from shared
//    memory, decodes them in registers (explicit LOP3 / funnel-shift / PRMT PTX,
//    decode.cuh) and multiplies with the packed fp32 FMA.  Lane partials
//    accumulate in shared memory across stages (M <= 2) or are reduced with
//    shuffles per stage (M >= 3); the sums are scaled and rounded to bf16 once.
//
// Dequantization arithmetic (fp32 accumulation):
//  * int4: decoded value q * 2^(p - 8) against activations scaled by 2^(8 - p)
//    (p the nibble's bit position, decode.cuh): exact products q x; per lane
//    and group s * sum(x q) + z * sum(x)  =  sum(x (q s + z)).
//  * FP6: decoded value v * 2^-124 (bf16 pair widened to fp32, subnormal for
//    e = 0); y = 2^124 s_n sum.
//  * int8: fp32 q; y = s_n sum.   bf16: plain products.
#include "wq_internal.h"
#include "wq_kernels.cuh"
#include "decode.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace wq {

template <int FMT>
struct GemvFmt;
template <>
struct GemvFmt<WQ_INT4> {
  static constexpr int kLaneK = 32;        // weights per lane per row-chunk
  static constexpr int kRowBytes = 512;    // packed bytes of one row-chunk
};
template <>
struct GemvFmt<WQ_FP6_E3M2> {
  static constexpr int kLaneK = 32;
  static constexpr int kRowBytes = 768;    // 4-bit plane (512) then 2-bit plane (256)
};
template <>
struct GemvFmt<WQ_INT8> {
  static constexpr int kLaneK = 16;
  static constexpr int kRowBytes = 512;
};
template <>
struct GemvFmt<WQ_BF16> {
  static constexpr int kLaneK = 8;
  static constexpr int kRowBytes = 512;
};

constexpr int kJ = 4;  // rows of a stage each consumer warp takes
// Launch shape per format and M (measured on B200):
//  * M = 1, int4 / int8 / bf16: two CTAs per SM, each with eight consumer warps,
//    a producer warp that keeps the ring full and a converter warp; the next
//    layer's CTAs can start while the last CTAs of this one drain (programmatic
//    dependent launch);
//  * M = 1, FP6 (decode-bound): one CTA per SM with sixteen consumer warps, a
//    producer and a converter, so every SM carries the same share;
//  * M = 2: one CTA per SM, eight consumer warps, a producer and a converter;
//  * M >= 3: one CTA per SM, eight consumer warps and no producer, so each thread
//    may hold up to 255 registers (the activations of a chunk need them); the
//    last warp to finish a stage refills its slot.
// A stage holds kJ rows per consumer warp.
__host__ __device__ constexpr bool gemv_has_producer(int, int mm) { return mm <= 2; }
// int4 with a producer: a converter warp prepares x once per CTA (its per-lane
// conversion, with the pre-scaling and the lane sums, is the costliest); the
// other formats convert their few values per lane in the consumers (measured
// 1-2 % faster than with a converter)
__host__ __device__ constexpr bool gemv_has_converter(int fmt, int mm) {
  return gemv_has_producer(fmt, mm) && fmt == WQ_INT4;
}
__host__ __device__ constexpr int gemv_cw(int fmt, int mm) { return (mm == 1 && fmt == WQ_FP6_E3M2) ? 16 : 8; }
__host__ __device__ constexpr int gemv_rb(int fmt, int mm) { return kJ * gemv_cw(fmt, mm); }
__host__ __device__ constexpr int gemv_ctas_per_sm(int fmt, int mm) { return (mm == 1 && fmt != WQ_FP6_E3M2) ? 2 : 1; }
// warps: the producer, the converter, then the consumers
__host__ __device__ constexpr int gemv_threads(int fmt, int mm) {
  return 32 * (gemv_cw(fmt, mm) + (gemv_has_producer(fmt, mm) ? 1 : 0) + (gemv_has_converter(fmt, mm) ? 1 : 0));
}
__host__ __device__ constexpr bool gemv_lane_partials(int mm) { return mm <= 2; }

// One ring slot: the weights of a stage's kRB rows, then per activation row
// the chunk's activations, then (int4 with staged scales) the scales and zeros
// of the stage's rows.  The activation area holds the lane registers' values
// in the order the consumers load them (pairs of packed fp32 pairs, lane after
// lane, so that a warp's 16-byte loads are conflict-free), then the lane sums;
// the raw bf16 chunk lands in the tail of the same area and the producer
// converts it in place.
template <int FMT, int MM>
struct GemvLayout {
  static constexpr int kLaneK = GemvFmt<FMT>::kLaneK;
  static constexpr int kChunkK = 32 * kLaneK;
  static constexpr int kXBytes = kChunkK * 2;   // one chunk of one activation row, bf16
  static constexpr int kRB = gemv_rb(FMT, MM);  // rows per stage
  static constexpr int kWBytes = kRB * GemvFmt<FMT>::kRowBytes;
  static constexpr int kPairs = kLaneK / 2;     // packed fp32 pairs per lane and activation row
  static constexpr int kCxBytes = gemv_has_converter(FMT, MM) ? 32 * kPairs * 8 + 32 * 4 : kXBytes;
  static constexpr int kRawOff = kCxBytes - kXBytes;
  static constexpr int kXOff = kWBytes;
  static constexpr int kSzOff = (kXOff + MM * kCxBytes + 127) / 128 * 128;
  static_assert(kRawOff % 16 == 0 && kCxBytes % 16 == 0 && kXOff % 128 == 0, "bulk copies need 16-byte offsets");
  // scales then zeros of the stage's rows, gpc groups each (int4)
  static constexpr int stage_bytes(int gpc, bool sz) {
    return (kSzOff + (sz ? 2 * kRB * gpc * 2 : 0) + 127) / 128 * 128;
  }
};

__device__ __forceinline__ float fp16_bits_to_float(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// Packed bytes of `kc` weights of one row for the format.
template <int FMT>
__host__ __device__ __forceinline__ uint32_t row_chunk_bytes(int kc) {
  if (FMT == WQ_INT4) return uint32_t(kc) / 2;
  if (FMT == WQ_FP6_E3M2) return uint32_t(kc) / 2 + uint32_t(kc) / 4;
  if (FMT == WQ_INT8) return uint32_t(kc);
  return uint32_t(kc) * 2;
}

// Per-lane activation registers of one chunk, for MM rows of x, as packed fp32
// pairs matching the weight pairs the decoder produces:
//  * int4: pair 8 w + n = (k_a, k_a + 8) with k_a = 16 w + 2 (n & 3) + (n >> 2)
//    (nibble n of words 2w and 2w + 1), scaled by 2^(8 - p(n)) (decode.cuh);
//  * other formats: pair i = (2 i, 2 i + 1).
// All conversions and scalings are exact (powers of two).
template <int FMT, int MM>
struct XRegs {
  uint64_t v2[MM][GemvFmt<FMT>::kLaneK / 2];
  float xsum[MM];  // int4: sum of the lane's 32 activations (unscaled)
};

__host__ __device__ constexpr float pow2f(int e) {
  return e >= 0 ? float(1u << e) : 1.0f / float(1u << -e);
}

// Lanes past the end of K (last chunk) get zeros: their weights are the tensor
// copy's zero fill, so every product is zero without a per-lane branch.
// `xs` is the raw chunk of activation row 0; row m is m * L::kCxBytes further.
template <int FMT, int MM>
__device__ __forceinline__ void load_x_smem(XRegs<FMT, MM>& xr, const uint8_t* xs, int lane, bool valid) {
  using L = GemvLayout<FMT, MM>;
  constexpr int LK = GemvFmt<FMT>::kLaneK;
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    const uint8_t* base = xs + m * L::kCxBytes + lane * LK * 2;
    float xf[LK];
#pragma unroll
    for (int q = 0; q < LK / 8; ++q) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (valid) v = *reinterpret_cast<const uint4*>(base + 16 * q);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        xf[8 * q + 2 * i] = bf16_lo_f(w[i]);
        xf[8 * q + 2 * i + 1] = bf16_hi_f(w[i]);
      }
    }
    if constexpr (FMT == WQ_INT4) {
#pragma unroll
      for (int wp = 0; wp < 2; ++wp)
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          const int ka = 16 * wp + 2 * (n & 3) + (n >> 2);
          constexpr float kScale[8] = {pow2f(int4_x_scale_exp(0)), pow2f(int4_x_scale_exp(1)),
                                       pow2f(int4_x_scale_exp(2)), pow2f(int4_x_scale_exp(3)),
                                       pow2f(int4_x_scale_exp(4)), pow2f(int4_x_scale_exp(5)),
                                       pow2f(int4_x_scale_exp(6)), pow2f(int4_x_scale_exp(7))};
          xr.v2[m][8 * wp + n] = pack2(xf[ka] * kScale[n], xf[ka + 8] * kScale[n]);
        }
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int i = 0; i < LK; i += 2) {
        s0 += xf[i];
        s1 += xf[i + 1];
      }
      xr.xsum[m] = s0 + s1;
    } else {
#pragma unroll
      for (int i = 0; i < LK / 2; ++i) xr.v2[m][i] = pack2(xf[2 * i], xf[2 * i + 1]);
    }
  }
}

// Producer warp: converts the raw chunk at the tail of the activation area
// `cx` into the lane-register layout, in place (every lane has read its raw
// values before any lane writes).  The fence orders these generic writes before
// the tensor copies that later refill the slot.
template <int FMT, int MM>
__device__ __forceinline__ void convert_x(uint8_t* cx, int lane, bool valid) {
  using L = GemvLayout<FMT, MM>;
  XRegs<FMT, MM> xr;
  load_x_smem<FMT, MM>(xr, cx + L::kRawOff, lane, valid);
  __syncwarp();
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    uint8_t* row = cx + m * L::kCxBytes;
#pragma unroll
    for (int q = 0; q < L::kPairs / 2; ++q)
      *reinterpret_cast<ulonglong2*>(row + (q * 32 + lane) * 16) =
          make_ulonglong2(xr.v2[m][2 * q], xr.v2[m][2 * q + 1]);
    if constexpr (FMT == WQ_INT4) *reinterpret_cast<float*>(row + L::kPairs * 256 + lane * 4) = xr.xsum[m];
  }
  fence_proxy_async_shared();
}

// Consumer: the lane's activation registers of a chunk converted by the producer.
template <int FMT, int MM>
__device__ __forceinline__ void load_cx(XRegs<FMT, MM>& xr, const uint8_t* cx, int lane) {
  using L = GemvLayout<FMT, MM>;
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    const uint8_t* row = cx + m * L::kCxBytes;
#pragma unroll
    for (int q = 0; q < L::kPairs / 2; ++q) {
      const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(row + (q * 32 + lane) * 16);
      xr.v2[m][2 * q] = v.x;
      xr.v2[m][2 * q + 1] = v.y;
    }
    if constexpr (FMT == WQ_INT4) xr.xsum[m] = *reinterpret_cast<const float*>(row + L::kPairs * 256 + lane * 4);
  }
}

template <int FMT>
struct DecodeConsts {
  Int4PairConsts i4;
  uint64_t i8;
};
template <int FMT>
__device__ __forceinline__ DecodeConsts<FMT> make_decode_consts() {
  DecodeConsts<FMT> d{};
  if constexpr (FMT == WQ_INT4) d.i4 = int4_pair_consts();
  if constexpr (FMT == WQ_INT8) d.i8 = int8_f32_bias();
  return d;
}

// Lane partial of one row-chunk for every activation row.  `w` points at the
// lane's row in shared memory (FP6: `w2p` at its 2-bit plane).  Decoded values
// are exact fp32 pairs and accumulate with the packed fp32 FMA (one pair of
// accumulators per activation row).
template <int FMT, int MM>
__device__ __forceinline__ void lane_dot(const uint8_t* w, const uint8_t* w2p, int lane, const XRegs<FMT, MM>& xr,
                                         const DecodeConsts<FMT>& dc, float acc[MM]) {
  uint64_t ac[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) ac[m] = 0ull;
  if constexpr (FMT == WQ_INT4) {
    const uint4 wv = *reinterpret_cast<const uint4*>(w + lane * 16);
    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int wp = 0; wp < 2; ++wp) {
      const uint32_t wa = words[2 * wp], wb = words[2 * wp + 1];
      const uint32_t sa = wa >> 12, sb = wb >> 12;
      const uint64_t v[8] = {int4_pair<0>(wa, wb, dc.i4), int4_pair<1>(wa, wb, dc.i4), int4_pair<2>(wa, wb, dc.i4),
                             int4_pair<3>(wa, wb, dc.i4), int4_pair<4>(wa, wb, dc.i4), int4_pair<5>(sa, sb, dc.i4),
                             int4_pair<6>(sa, sb, dc.i4), int4_pair<7>(sa, sb, dc.i4)};
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int m = 0; m < MM; ++m) ffma2p(ac[m], v[n], xr.v2[m][8 * wp + n]);
    }
  } else if constexpr (FMT == WQ_FP6_E3M2) {
    const uint4 w4 = *reinterpret_cast<const uint4*>(w + lane * 16);
    const uint2 w2 = *reinterpret_cast<const uint2*>(w2p + lane * 8);
    const uint32_t a4[4] = {w4.x, w4.y, w4.z, w4.w};
    const uint32_t a2[2] = {w2.x, w2.y};
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      uint32_t p[8];
      decode_fp6_words(a2[v], a4[2 * v], a4[2 * v + 1], p);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint64_t pw = pack2(bf16_lo_f(p[j]), bf16_hi_f(p[j]));
#pragma unroll
        for (int m = 0; m < MM; ++m) ffma2p(ac[m], pw, xr.v2[m][8 * v + j]);
      }
    }
  } else if constexpr (FMT == WQ_INT8) {
    const uint4 wv = *reinterpret_cast<const uint4*>(w + lane * 16);
    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t wq = words[q];
      const uint64_t p0 = fadd2p(__uint_as_float(__byte_perm(wq, 0x4B000000u, 0x7540)),
                                 __uint_as_float(__byte_perm(wq, 0x4B000000u, 0x7541)), dc.i8);
      const uint64_t p1 = fadd2p(__uint_as_float(__byte_perm(wq, 0x4B000000u, 0x7542)),
                                 __uint_as_float(__byte_perm(wq, 0x4B000000u, 0x7543)), dc.i8);
#pragma unroll
      for (int m = 0; m < MM; ++m) {
        ffma2p(ac[m], p0, xr.v2[m][2 * q]);
        ffma2p(ac[m], p1, xr.v2[m][2 * q + 1]);
      }
    }
  } else {
    const uint4 wv = *reinterpret_cast<const uint4*>(w + lane * 16);
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint64_t pw = pack2(bf16_lo_f(ww[i]), bf16_hi_f(ww[i]));
#pragma unroll
      for (int m = 0; m < MM; ++m) ffma2p(ac[m], pw, xr.v2[m][i]);
    }
  }
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    float lo, hi;
    unpack2(ac[m], lo, hi);
    acc[m] = lo + hi;
  }
}

// Position of a stage in the CTA's sequence: ring slot and phase parity, row
// block and (rotated) chunk.  Stages run chunk-major over the row blocks.
struct StagePos {
  int slot;
  uint32_t phase;
  int rb;
  int c;
};
// chunks cycle through [clo, chi), the CTA's share of K
__device__ __forceinline__ void advance(StagePos& p, int NS, int NRB, int clo, int chi) {
  if (++p.rb == NRB) {
    p.rb = 0;
    p.c = (p.c + 1 == chi) ? clo : p.c + 1;
  }
  if (++p.slot == NS) {
    p.slot = 0;
    p.phase ^= 1u;
  }
}

// SZ (int4 only): the scales and zeros of each stage's rows travel with its
// weights by tensor copies; otherwise each consumer lane loads its own one
// stage ahead.
template <int FMT, int MM, bool SZ>
__global__ void __launch_bounds__(gemv_threads(FMT, MM), gemv_ctas_per_sm(FMT, MM)) gemv_kernel(const __grid_constant__ GemvParams a) {
  using F = GemvFmt<FMT>;
  using L = GemvLayout<FMT, MM>;
  constexpr int kChunkK = L::kChunkK;
  constexpr bool kProducer = gemv_has_producer(FMT, MM);
  constexpr bool kConv = gemv_has_converter(FMT, MM);
  constexpr int CWN = gemv_cw(FMT, MM);
  constexpr int kRB = L::kRB;
  extern __shared__ __align__(1024) uint8_t smem[];

  static_assert(!SZ || FMT == WQ_INT4, "staged scales are an int4 layout");
  const int NS = a.stages;
  const int SB = a.stage_bytes;
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(NS) * SB);
  uint64_t* empty = full + NS;                          // [NS] warps finished reading the slot's stage
  uint64_t* xready = empty + NS;                        // [NS] converter: the stage was handed over (x converted)
  int* done_cnt = reinterpret_cast<int*>(xready + NS);  // [NS] arrivals counted, to elect the refilling warp
  int* last_issued = done_cnt + NS;                    // [NS] stage last issued into the slot
  // partial sums.  Lane partials (M <= 2): [R][MM][32 lanes], each (row, lane)
  // entry owned by one thread, so stages add into it with no cross-lane step and
  // the lanes are summed once in the epilogue.  Otherwise [C][R][MM]: one value
  // per chunk after a shuffle reduction.
  constexpr bool kLanePart = gemv_lane_partials(MM);
  float* part = reinterpret_cast<float*>(last_issued + NS + (NS & 1));
  const int C = (a.K + kChunkK - 1) / kChunkK;
  // split K: the S CTAs of a cluster share a row block, rank q taking chunks
  // [CLO, CHI); at the end rank q sums the cluster's partials of its slice of
  // the rows
  const int S = a.ksplit;
  const int rank = blockIdx.x % S;
  const int n0 = (blockIdx.x / S) * a.rows_per_cta;
  const int R = min(a.rows_per_cta, a.N - n0);
  const int NRB = (R + kRB - 1) / kRB;
  const int CLO = rank * a.chunks_per_split;
  const int CHI = min(C, CLO + a.chunks_per_split);
  const int T = (CHI - CLO) * NRB;
  // each CTA starts at a different chunk so that concurrent CTAs fetch
  // different parts of x
  const int c_rot = CLO + (blockIdx.x / S) % (CHI - CLO);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t policy = l2_policy_evict_first();
  // int4: log2 of the group size, groups per chunk
  const int gshift = (FMT == WQ_INT4) ? __ffs(a.groupsize) - 1 : 0;
  const int gpc = kChunkK >> gshift;

  // Issue the tensor copies of one stage into its slot (one thread): the weight
  // boxes and, with SZ, the scale and zero boxes of the same rows.  The x of a
  // chunk travels with the chunk's first stage only (issue_x).
  auto issue_w = [&](const StagePos& p) {
    const int rows = min(kRB, R - p.rb * kRB);
    const int nbox = (rows + a.box_rows - 1) / a.box_rows;
    const int kc = min(kChunkK, a.K - p.c * kChunkK);
    uint32_t bytes = uint32_t(nbox * a.box_rows * F::kRowBytes) + (p.rb == 0 ? MM * uint32_t(kc) * 2 : 0u);
    if constexpr (SZ) bytes += uint32_t(nbox * a.box_rows * gpc * 4);
    mbar_arrive_expect_tx(&full[p.slot], bytes);
    uint8_t* st = ring + size_t(p.slot) * SB;
    const int row0 = n0 + p.rb * kRB;
    for (int b = 0; b < nbox; ++b) {
      const int row = row0 + b * a.box_rows;
      if constexpr (FMT == WQ_FP6_E3M2) {
        tma_load_2d(st + b * a.box_rows * 512, &a.tm_w, p.c * (512 / 4), row, &full[p.slot], policy);
        tma_load_2d(st + kRB * 512 + b * a.box_rows * 256, &a.tm_w2, p.c * (256 / 4), row, &full[p.slot], policy);
      } else {
        tma_load_2d(st + b * a.box_rows * F::kRowBytes, &a.tm_w, p.c * (F::kRowBytes / 4), row, &full[p.slot], policy);
      }
      if constexpr (SZ) {
        uint8_t* sz = st + L::kSzOff + b * a.box_rows * gpc * 2;
        tma_load_2d(sz, &a.tm_s, p.c * gpc, row, &full[p.slot], policy);
        tma_load_2d(sz + kRB * gpc * 2, &a.tm_z, p.c * gpc, row, &full[p.slot], policy);
      }
    }
  };
  auto issue_x = [&](const StagePos& p) {
    if (p.rb != 0) return;
    const int kc = min(kChunkK, a.K - p.c * kChunkK);
    for (int m = 0; m < MM; ++m)
      bulk_g2s(ring + size_t(p.slot) * SB + L::kXOff + m * L::kCxBytes + L::kRawOff,
               a.x + size_t(m) * a.K + size_t(p.c) * kChunkK, uint32_t(kc) * 2, &full[p.slot]);
  };

  if (a.pdl) pdl_launch_dependents();
  const int T0 = min(T, NS);
  if constexpr (kLanePart)
    for (int i = threadIdx.x; i < R * MM * 32; i += blockDim.x) part[i] = 0.f;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CWN);
      mbar_init(&xready[s], 32);
      done_cnt[s] = 0;
      last_issued[s] = -1;
    }
    fence_mbar_init();
    prefetch_tmap(&a.tm_w);
    if (FMT == WQ_FP6_E3M2) prefetch_tmap(&a.tm_w2);
    if (SZ) {
      prefetch_tmap(&a.tm_s);
      prefetch_tmap(&a.tm_z);
    }
    if constexpr (!kProducer) {
      // first ring fill: weights at once; x after the previous kernel (which may
      // write it) has finished, under programmatic dependent launch
      StagePos q = {0, 0u, 0, c_rot};
      for (int t = 0; t < T0; ++t) {
        issue_w(q);
        last_issued[q.slot] = t;
        advance(q, NS, NRB, CLO, CHI);
      }
      if (a.pdl) pdl_wait();
      q = {0, 0u, 0, c_rot};
      for (int t = 0; t < T0; ++t) {
        issue_x(q);
        advance(q, NS, NRB, CLO, CHI);
      }
    }
  }
  __syncthreads();

  bool failed = false;
  if (kProducer && warp == 0) {
    // ------------------------------------------------------------ producer (M <= 2)
    if (lane == 0) {
      StagePos p = {0, 0u, 0, c_rot};
      for (int t = 0; t < T; ++t) {
        if (!mbar_wait(&empty[p.slot], p.phase ^ 1u)) {
          failed = true;
          break;
        }
        issue_w(p);
        last_issued[p.slot] = t;
        if (t >= T0 || !a.pdl) issue_x(p);
        if (t == T0 - 1 && a.pdl) {
          // weights of the first ring fill are in flight; x may be written by
          // the previous kernel, so wait for it before fetching x
          pdl_wait();
          StagePos q = {0, 0u, 0, c_rot};
          for (int t2 = 0; t2 < T0; ++t2) {
            issue_x(q);
            advance(q, NS, NRB, CLO, CHI);
          }
        }
        advance(p, NS, NRB, CLO, CHI);
      }
      if (failed && a.pdl) pdl_wait();
    }
    __syncwarp();
  } else if (kConv && warp == 1) {
    // ------------------------------------------------------------ converter (int4, M <= 2)
    // Takes the stages in order as they land: converts the activations of a
    // chunk's first stage and releases every stage to the consumers on its
    // xready barrier.  Consumers wait for xready at every stage, so a slot is
    // never refilled before the converter has passed it.
    if constexpr (kConv) {
      StagePos u = {0, 0u, 0, c_rot};
      for (int t = 0; t < T; ++t) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[u.slot], u.phase))) {
          failed = true;
          break;
        }
        if (u.rb == 0)
          convert_x<FMT, MM>(ring + size_t(u.slot) * SB + L::kXOff, lane, u.c * kChunkK + lane * F::kLaneK < a.K);
        mbar_arrive(&xready[u.slot]);
        advance(u, NS, NRB, CLO, CHI);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int cw = warp - (kProducer ? 1 : 0) - (kConv ? 1 : 0);
    if (a.pdl) pdl_wait();
    int cur_c = -1;
    XRegs<FMT, MM> xr;
    const DecodeConsts<FMT> dc = make_decode_consts<FMT>();
    constexpr int J = kJ;
    const int G = (FMT == WQ_INT4) ? (a.K >> gshift) : 0;
    // int4 without staged scales: raw 16-bit scale and zero of this warp's rows
    // at the lane's group, fetched one stage ahead into the other of two register
    // sets; the load zero-extends, so no instruction touches them before the fold
    // a stage later (rows past N are skipped: only the last CTA has them)
    const int G8 = G * CWN;
    // int4 with staged scales: the lane's group in the stage's [kRB][gpc] arrays
    const int sz_lane = (FMT == WQ_INT4) ? (cw * gpc + ((lane * F::kLaneK) >> gshift)) * 2 : 0;
    const int sz_row = CWN * gpc * 2;
    const int sz_zero = kRB * gpc * 2;
    auto fetch_sz = [&](const StagePos& p, uint32_t (&ds)[J], uint32_t (&dz)[J]) {
      if constexpr (FMT == WQ_INT4 && !SZ) {
        const int k0 = p.c * kChunkK + lane * F::kLaneK;
        const int row = n0 + p.rb * kRB + cw;
        const int off = row * G + (k0 >> gshift);
        const uint16_t* sp = a.scales + off;
        const uint16_t* zp = a.zeros + off;
#pragma unroll
        for (int j = 0; j < J; ++j) {
          if (k0 < a.K && row + j * CWN < a.N) {
            ds[j] = ld_nc_u16_u32(sp + j * G8);
            dz[j] = ld_nc_u16_u32(zp + j * G8);
          }
        }
      }
    };
    // one stage: prefetch the next stage's scales, wait for this stage's tiles,
    // dot products of the warp's rows, hand the slot back (the last warp out
    // refills it with stage t + NS), reduce across lanes
    auto stage = [&](int t, StagePos& p, StagePos& pr, bool has_next, const uint32_t (&ss)[J],
                     const uint32_t (&zz)[J], uint32_t (&ss_next)[J], uint32_t (&zz_next)[J]) -> bool {
      StagePos nx = p;
      advance(nx, NS, NRB, CLO, CHI);
      if (!SZ && has_next) fetch_sz(nx, ss_next, zz_next);
      if (!mbar_wait(&full[p.slot], p.phase)) return false;
      if (kConv && !mbar_wait(&xready[p.slot], p.phase)) return false;
      const int rows = min(kRB, R - p.rb * kRB);
      const uint8_t* st = ring + p.slot * SB;
      if (p.c != cur_c) {
        // a chunk's first stage (rb == 0) carries its activations
        if constexpr (kConv) {
          load_cx<FMT, MM>(xr, st + L::kXOff, lane);
        } else {
          load_x_smem<FMT, MM>(xr, st + L::kXOff + L::kRawOff, lane, p.c * kChunkK + lane * F::kLaneK < a.K);
        }
        cur_c = p.c;
      }
      // all J rows of this warp at once: independent chains interleave.  A full
      // stage runs every row without a test; in a partial stage (the last rows
      // of a CTA) rows past its end are skipped, the test uniform across the
      // warp, and their partials are zero and never stored.
      float acc[J][MM];
      auto row_dot = [&](int j) {
        const int i = cw + j * CWN;
        if constexpr (FMT == WQ_FP6_E3M2)
          lane_dot<FMT, MM>(st + i * 512, st + kRB * 512 + i * 256, lane, xr, dc, acc[j]);
        else
          lane_dot<FMT, MM>(st + i * F::kRowBytes, nullptr, lane, xr, dc, acc[j]);
        if constexpr (FMT == WQ_INT4) {
          // sum over the lane's 32 k (one group): s * sum(q x) + z * sum(x)
          uint32_t sb = ss[j], zb = zz[j];
          if constexpr (SZ) {
            const uint8_t* szp = st + L::kSzOff + sz_lane + j * sz_row;
            sb = *reinterpret_cast<const uint16_t*>(szp);
            zb = *reinterpret_cast<const uint16_t*>(szp + sz_zero);
          }
          const float sc = __uint_as_float(sb << 16);
          const float zc = __uint_as_float(zb << 16);
#pragma unroll
          for (int m = 0; m < MM; ++m) acc[j][m] = fmaf(sc, acc[j][m], zc * xr.xsum[m]);
        }
      };
      if (rows == kRB) {
#pragma unroll
        for (int j = 0; j < J; ++j) row_dot(j);
      } else {
#pragma unroll
        for (int j = 0; j < J; ++j) {
          if (cw + j * CWN < rows) {
            row_dot(j);
          } else {
#pragma unroll
            for (int m = 0; m < MM; ++m) acc[j][m] = 0.f;
          }
        }
      }
      // every lane's shared-memory reads of the stage are done: release them on
      // the slot's empty barrier
      __syncwarp();
      bool ok = true;
      if (lane == 0) {
        mbar_arrive(&empty[p.slot]);
        if constexpr (!kProducer) {
          // the counter elects the last warp, which waits for the barrier
          // (acquiring every warp's reads) and refills the slot with stage t + NS
          if (atomicAdd(&done_cnt[p.slot], 1) == CWN - 1) {
            done_cnt[p.slot] = 0;
            ok = mbar_wait(&empty[p.slot], p.phase);
            if (ok && t + NS < T) {
              fence_proxy_async_shared();
              issue_w(pr);
              issue_x(pr);
              last_issued[pr.slot] = t + NS;
            }
          }
        }
      }
      if (!kProducer && !__shfl_sync(0xFFFFFFFFu, int(ok), 0)) return false;
      if constexpr (kLanePart) {
        // add the lane partials of the warp's rows (rows past R belong to the
        // next CTA or hold stale data: skipped, uniformly across the warp)
#pragma unroll
        for (int j = 0; j < J; ++j) {
          const int row = p.rb * kRB + cw + j * CWN;
          if (row < R) {
            float* dst = part + row * (MM * 32) + lane;
#pragma unroll
            for (int m = 0; m < MM; ++m) dst[m * 32] += acc[j][m];
          }
        }
      } else {
        // transposed butterfly: 6 shuffles reduce the 4 rows; lane 8j holds row j
        static_assert(J == 4, "reduction below assumes 4 rows per warp and stage");
#pragma unroll
        for (int m = 0; m < MM; ++m) {
          const bool hi16 = lane & 16;
          float k0v = hi16 ? acc[2][m] : acc[0][m];
          float k1v = hi16 ? acc[3][m] : acc[1][m];
          k0v += __shfl_xor_sync(0xFFFFFFFFu, hi16 ? acc[0][m] : acc[2][m], 16);
          k1v += __shfl_xor_sync(0xFFFFFFFFu, hi16 ? acc[1][m] : acc[3][m], 16);
          const bool hi8 = lane & 8;
          float kv = hi8 ? k1v : k0v;
          kv += __shfl_xor_sync(0xFFFFFFFFu, hi8 ? k0v : k1v, 8);
          kv += __shfl_xor_sync(0xFFFFFFFFu, kv, 4);
          kv += __shfl_xor_sync(0xFFFFFFFFu, kv, 2);
          kv += __shfl_xor_sync(0xFFFFFFFFu, kv, 1);
          if ((lane & 7) == 0) {
            const int j = lane >> 3;  // 2 * (bit 4) + (bit 3)
            const int i = cw + j * CWN;
            if (i < rows) part[((p.c * R) + p.rb * kRB + i) * MM + m] = kv;
          }
        }
      }
      p = nx;
      advance(pr, NS, NRB, CLO, CHI);
      return true;
    };
    uint32_t sA[J], zA[J], sB[J], zB[J];
#pragma unroll
    for (int j = 0; j < J; ++j) sA[j] = zA[j] = sB[j] = zB[j] = 0u;
    StagePos p = {0, 0u, 0, c_rot};
    StagePos pr = p;  // position of stage t + NS
    for (int i = 0; i < NS; ++i) advance(pr, NS, NRB, CLO, CHI);
    fetch_sz(p, sA, zA);
    for (int t = 0; t < T; t += 2) {
      if (!stage(t, p, pr, t + 1 < T, sA, zA, sB, zB)) {
        failed = true;
        break;
      }
      if (t + 1 < T && !stage(t + 1, p, pr, t + 2 < T, sB, zB, sA, zA)) {
        failed = true;
        break;
      }
    }
  }

  // ---------------------------------------------------------------- epilogue
  const bool any_failed = __syncthreads_or(failed);
  if (any_failed) {
    // wait (bounded) until every copy issued into the ring has landed
    if (threadIdx.x == 0) {
      for (int s = 0; s < NS; ++s) {
        const int u = last_issued[s];
        if (u >= 0) mbar_wait(&full[s], (u / NS) & 1);
      }
    }
  }
  // scale of a finished sum, rounding to bf16 and the store
  auto store_y = [&](int r, int m, float v) {
    const int n = n0 + r;
    if constexpr (FMT == WQ_INT8) {
      v *= fp16_bits_to_float(a.scales[n]);
    } else if constexpr (FMT == WQ_FP6_E3M2) {
      v = (v * 0x1p124f) * fp16_bits_to_float(a.scales[n]);
    }
    a.y[size_t(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  };
  // sum of a warp's 32 lane values by a fixed shuffle tree (every lane ends with
  // the same, deterministic total)
  auto warp_sum = [](float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
  };
  const int nwarps = int(blockDim.x) >> 5;
  if constexpr (kLanePart) {
    if (S > 1) {
      // every CTA of the cluster reaches both cluster barriers, failed or not
      cluster_sync_all();  // all lane partials of the cluster are final
      if (!any_failed) {
        // rank q finishes its slice of the rows, one warp per (row, activation
        // row): lane l adds the S CTAs' partials of lane l in rank order (the
        // loads are issued together), then the shuffle tree sums the lanes
        const int RS = (R + S - 1) / S;
        const int lo = rank * RS * MM, hi = min(R, (rank + 1) * RS) * MM;
        for (int idx = lo + warp; idx < hi; idx += nwarps) {
          const uint32_t base = smem_u32(part + idx * 32 + lane);
          float pv[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (q < S) pv[q] = ld_cluster_f32(map_to_rank(base, uint32_t(q)));
          float v = 0.f;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (q < S) v += pv[q];
          v = warp_sum(v);
          if (lane == 0) store_y(idx / MM, idx % MM, v);
        }
      }
      cluster_sync_all();  // keep every CTA's shared memory until all ranks have read it
      return;
    }
  }
  if (any_failed) return;
  if constexpr (kLanePart) {
    // one thread per (row, activation row): its 32 lane partials in a fixed
    // order, starting at a rotating lane so that neighbouring threads read
    // different banks (a warp per row with a shuffle tree measured slower here:
    // with many rows per CTA its dependent shuffles serialise)
    for (int idx = threadIdx.x; idx < R * MM; idx += blockDim.x) {
      const float* src = part + idx * 32;
      float v = 0.f;
      for (int l = 0; l < 32; ++l) v += src[(l + idx) & 31];
      store_y(idx / MM, idx % MM, v);
    }
  } else {
    // the per-chunk values in chunk order
    for (int idx = threadIdx.x; idx < R * MM; idx += blockDim.x) {
      const int m = idx / R;
      const int r = idx - m * R;
      float v = 0.f;
      for (int c = 0; c < C; ++c) v += part[(c * R + r) * MM + m];
      store_y(r, m, v);
    }
  }
}

// ----------------------------------------------------------------- launcher
constexpr size_t kGemvSmemPerSm = 220 * 1024;

constexpr int kBoxRows = 8;

template <int FMT, int MM, bool SZ>
static cudaError_t launch_gemv_t(const GemvParams& p0, cudaStream_t stream, int sm_count) {
  using L = GemvLayout<FMT, MM>;
  using F = GemvFmt<FMT>;
  GemvParams p = p0;
  const int C = (p.K + L::kChunkK - 1) / L::kChunkK;
  const int target = sm_count * gemv_ctas_per_sm(FMT, MM);
  const size_t kGemvSmemBudget = kGemvSmemPerSm / gemv_ctas_per_sm(FMT, MM);
  // rows per CTA: a multiple of the box height, about N / target
  int R = (p.N + target * kBoxRows - 1) / (target * kBoxRows) * kBoxRows;
  // keep the partial-sum area within half (lane partials) or a quarter of the budget
  const size_t part_row = gemv_lane_partials(MM) ? size_t(32) * MM * 4 : size_t(C) * MM * 4;
  const int max_r = int((gemv_lane_partials(MM) ? kGemvSmemBudget / 2 : kGemvSmemBudget / 4) / part_row) / kBoxRows * kBoxRows;
  if (R > max_r) R = max_r;
  if (R < kBoxRows) R = kBoxRows;
  // split K over a cluster when the rows per CTA would not fill one stage (small
  // N): each CTA then takes one full stage of rows and a share of the chunks
  int S = 1, CPS = C;
  if (gemv_lane_partials(MM) && R < L::kRB) {
    const int nblk = (p.N + L::kRB - 1) / L::kRB;
    int s = target / nblk;
    s = s > 8 ? 8 : s;
    s = s > C ? C : s;
    if (s >= 2) {
      CPS = (C + s - 1) / s;
      S = (C + CPS - 1) / CPS;
      R = L::kRB;
    }
  }
  p.ksplit = S;
  p.chunks_per_split = CPS;
  p.rows_per_cta = R;
  p.box_rows = kBoxRows;
  const int gpc = FMT == WQ_INT4 ? L::kChunkK / p.groupsize : 0;
  p.sz_tma = SZ ? 1 : 0;
  p.stage_bytes = L::stage_bytes(gpc, SZ);
  // barriers and counters: full, empty, xready (8 bytes each), done_cnt, last_issued (4 each) per slot
  const size_t fixed = 8 * 32 + 16 + size_t(R) * part_row;
  if (fixed + 2 * size_t(p.stage_bytes) > 200 * 1024) return cudaErrorInvalidValue;
  int stages = fixed < kGemvSmemBudget ? int((kGemvSmemBudget - fixed) / p.stage_bytes) : 2;
  if (stages > 8) stages = 8;
  if (stages < 2) stages = 2;
  p.stages = stages;
  const size_t smem = size_t(stages) * p.stage_bytes + size_t(stages) * 32 + 16 + size_t(R) * part_row;

  // tensor maps: rows of packed bytes viewed as 32-bit elements, one chunk per box
  cudaError_t e;
  if constexpr (FMT == WQ_FP6_E3M2) {
    const uint8_t* p2 = static_cast<const uint8_t*>(p.packed);
    const uint8_t* p4 = p2 + size_t(p.N) * (p.K / 4);
    e = make_tmap_u32_2d(&p.tm_w, p4, uint64_t(p.K) / 8, uint64_t(p.N), uint64_t(p.K) / 2, 512 / 4, kBoxRows);
    if (e == cudaSuccess)
      e = make_tmap_u32_2d(&p.tm_w2, p2, uint64_t(p.K) / 16, uint64_t(p.N), uint64_t(p.K) / 4, 256 / 4, kBoxRows);
  } else {
    const uint64_t rowb = row_chunk_bytes<FMT>(p.K);
    e = make_tmap_u32_2d(&p.tm_w, p.packed, rowb / 4, uint64_t(p.N), rowb, F::kRowBytes / 4, kBoxRows);
  }
  if (e != cudaSuccess) return e;
  if constexpr (SZ) {
    // scales / zeros [N, G] bf16: boxes of one chunk's gpc groups x 8 rows (the
    // row pitch 2 G is a multiple of 16 bytes, checked by the caller)
    const uint64_t G = uint64_t(p.K / p.groupsize);
    e = make_tmap_2d(&p.tm_s, p.scales, 2, G, uint64_t(p.N), G * 2, uint32_t(gpc), kBoxRows, 0);
    if (e == cudaSuccess) e = make_tmap_2d(&p.tm_z, p.zeros, 2, G, uint64_t(p.N), G * 2, uint32_t(gpc), kBoxRows, 0);
    if (e != cudaSuccess) return e;
  }
  auto kernel = gemv_kernel<FMT, MM, SZ>;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int grid = (p.N + R - 1) / R * S;
  if (S > 1) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(gemv_threads(FMT, MM));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (S > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = S;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (p.pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// int4 stages its scales and zeros by tensor copies when a row of them (K / g
// bf16) is a multiple of 16 bytes (the arrays are 16-byte aligned by contract)
template <int FMT, int MM>
static cudaError_t launch_gemv_sz(const GemvParams& p, cudaStream_t s, int sm_count) {
  if constexpr (FMT == WQ_INT4) {
    if ((p.K / p.groupsize) % 8 == 0) return launch_gemv_t<FMT, MM, true>(p, s, sm_count);
  }
  return launch_gemv_t<FMT, MM, false>(p, s, sm_count);
}

template <int FMT>
static cudaError_t launch_gemv_fmt(const GemvParams& p, cudaStream_t s, int sm_count) {
  switch (p.M) {
    case 1: return launch_gemv_sz<FMT, 1>(p, s, sm_count);
    case 2: return launch_gemv_sz<FMT, 2>(p, s, sm_count);
    case 3: return launch_gemv_sz<FMT, 3>(p, s, sm_count);
    default: return launch_gemv_sz<FMT, 4>(p, s, sm_count);
  }
}

cudaError_t launch_gemv(const GemvParams& p, cudaStream_t s, int sm_count) {
  switch (p.fmt) {
    case WQ_INT4: return launch_gemv_fmt<WQ_INT4>(p, s, sm_count);
    case WQ_FP6_E3M2: return launch_gemv_fmt<WQ_FP6_E3M2>(p, s, sm_count);
    case WQ_INT8: return launch_gemv_fmt<WQ_INT8>(p, s, sm_count);
    default: return launch_gemv_fmt<WQ_BF16>(p, s, sm_count);
  }
}

cudaError_t gemv_take_status(uint32_t* status) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(status, g_device_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(uint32_t));
}

}  // namespace wq
