// CUDA-core split-K GEMV for the decode linear at small M (sm_100a).
//
//   y[m, n] = sum_k x[m, k] * deq(W)[n, k]      m < MM <= 4
//
// The weight stream is the whole cost of a decode step (gpt-fast write-up,
// m.greenbasetech.com article 46368139_1106049486, paragraph on the memory
// bandwidth bound: every generated token reads every weight once).  The kernel
// reads each packed byte exactly once and hides dequantization under the stream:
//
//  * A CTA owns a contiguous block of R output rows over all of K (one
//    contiguous region of the row-major packed matrix, so no cross-CTA
//    reduction and a deterministic result).
//  * K is cut into chunks of 32 lanes x LANE_K weights.  A stage of the
//    shared-memory ring holds one chunk of up to 32 rows plus that chunk of x;
//    warp 0 fills the ring with bulk asynchronous copies (TMA engine), one row
//    per lane, completing on the stage's mbarrier, far ahead of the consumers.
//  * Eight consumer warps take the rows of a stage; every lane reads its 16
//    bytes (FP6: 16 + 8) of the row from shared memory, decodes them in
//    registers (bit-parallel unpack, see decode.cuh) and multiplies with its
//    activations held in registers for the whole chunk.  A shuffle butterfly
//    reduces each (row, chunk); partials are summed in chunk order in shared
//    memory, scaled and rounded to bf16.
//
// Dequantization arithmetic (fp32 accumulation):
//  * int4: decoded value 128 + q (bf16); per lane and group
//    s * sum(x (128 + q)) + (z - 128 s) * sum(x)  =  sum(x (q s + z)).
//  * FP6: decoded value v * 2^-124 (bf16, subnormal for e = 0); y = 2^124 s_n sum.
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
  static constexpr int kLaneK = 8;
  static constexpr int kRowBytes = 256;
};
template <>
struct GemvFmt<WQ_BF16> {
  static constexpr int kLaneK = 8;
  static constexpr int kRowBytes = 512;
};

constexpr int kRB = 32;                 // rows per stage (one per producer lane)
constexpr int kConsumerWarps = 8;
constexpr int kGemvThreads = 32 * (1 + kConsumerWarps);
// Two CTAs per SM while the activations of one chunk fit the register budget, one beyond.
__host__ __device__ constexpr int gemv_ctas_per_sm(int mm) { return mm <= 2 ? 2 : 1; }

template <int FMT, int MM>
struct GemvLayout {
  static constexpr int kChunkK = 32 * GemvFmt<FMT>::kLaneK;
  static constexpr int kXBytes = kChunkK * 2;  // one chunk of one activation row
  static constexpr int kStageBytes = (kRB * GemvFmt<FMT>::kRowBytes + MM * kXBytes + 127) / 128 * 128;
};

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
__device__ __forceinline__ float fp16_bits_to_float(uint16_t b) { return __half2float(__ushort_as_half(b)); }
__device__ __forceinline__ uint16_t ld_u16(const uint16_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// Packed bytes of `kc` weights of one row for the format.
template <int FMT>
__host__ __device__ __forceinline__ uint32_t row_chunk_bytes(int kc) {
  if (FMT == WQ_INT4) return uint32_t(kc) / 2;
  if (FMT == WQ_FP6_E3M2) return uint32_t(kc) / 2 + uint32_t(kc) / 4;
  if (FMT == WQ_INT8) return uint32_t(kc);
  return uint32_t(kc) * 2;
}

// Per-lane activation registers of one chunk, for MM rows of x, as fp32 (exact).
template <int FMT, int MM>
struct XRegs {
  float v[MM][GemvFmt<FMT>::kLaneK];
  float xsum[MM];  // int4: sum of the lane's 32 activations
};

template <int FMT, int MM>
__device__ __forceinline__ void load_x_smem(XRegs<FMT, MM>& xr, const uint8_t* xs, int lane) {
  using L = GemvLayout<FMT, MM>;
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    const uint8_t* base = xs + m * L::kXBytes + lane * GemvFmt<FMT>::kLaneK * 2;
#pragma unroll
    for (int q = 0; q < GemvFmt<FMT>::kLaneK / 8; ++q) {
      const uint4 v = *reinterpret_cast<const uint4*>(base + 16 * q);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        xr.v[m][8 * q + 2 * i] = bf16_lo_f(w[i]);
        xr.v[m][8 * q + 2 * i + 1] = bf16_hi_f(w[i]);
      }
    }
    if constexpr (FMT == WQ_INT4) {
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int i = 0; i < GemvFmt<FMT>::kLaneK; i += 2) {
        s0 += xr.v[m][i];
        s1 += xr.v[m][i + 1];
      }
      xr.xsum[m] = s0 + s1;
    }
  }
}

// Lane partial of one row-chunk for every activation row.  `w` points at the
// lane's row in shared memory (FP6: `w2p` at its 2-bit plane).  Decoded bf16
// pairs are widened to fp32 exactly (a shift and a mask) and accumulated with the
// packed fp32 FMA; the two halves of each pair use separate accumulators.
template <int FMT, int MM>
__device__ __forceinline__ void lane_dot(const uint8_t* w, const uint8_t* w2p, int lane, const XRegs<FMT, MM>& xr,
                                         float acc[MM]) {
  float a0[MM], a1[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) a0[m] = a1[m] = 0.f;
  if constexpr (FMT == WQ_INT4) {
    const uint4 wv = *reinterpret_cast<const uint4*>(w + lane * 16);
    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t p[4];
      decode_int4_word(words[q], p);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float lo = bf16_lo_f(p[r]), hi = bf16_hi_f(p[r]);
#pragma unroll
        for (int m = 0; m < MM; ++m) ffma2(a0[m], a1[m], lo, hi, xr.v[m][8 * q + 2 * r], xr.v[m][8 * q + 2 * r + 1]);
      }
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
        const float lo = bf16_lo_f(p[j]), hi = bf16_hi_f(p[j]);
#pragma unroll
        for (int m = 0; m < MM; ++m) ffma2(a0[m], a1[m], lo, hi, xr.v[m][16 * v + 2 * j], xr.v[m][16 * v + 2 * j + 1]);
      }
    }
  } else if constexpr (FMT == WQ_INT8) {
    const uint2 wv = *reinterpret_cast<const uint2*>(w + lane * 8);
    float v[8];
    decode_int8_word(wv.x, v);
    decode_int8_word(wv.y, v + 4);
#pragma unroll
    for (int i = 0; i < 8; i += 2)
#pragma unroll
      for (int m = 0; m < MM; ++m) ffma2(a0[m], a1[m], v[i], v[i + 1], xr.v[m][i], xr.v[m][i + 1]);
  } else {
    const uint4 wv = *reinterpret_cast<const uint4*>(w + lane * 16);
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = bf16_lo_f(ww[i]), hi = bf16_hi_f(ww[i]);
#pragma unroll
      for (int m = 0; m < MM; ++m) ffma2(a0[m], a1[m], lo, hi, xr.v[m][2 * i], xr.v[m][2 * i + 1]);
    }
  }
#pragma unroll
  for (int m = 0; m < MM; ++m) acc[m] = a0[m] + a1[m];
}


template <int FMT, int MM>
__global__ void __launch_bounds__(kGemvThreads, gemv_ctas_per_sm(MM)) gemv_kernel(const __grid_constant__ GemvParams a) {
  using F = GemvFmt<FMT>;
  using L = GemvLayout<FMT, MM>;
  constexpr int kChunkK = L::kChunkK;
  extern __shared__ __align__(1024) uint8_t smem[];

  const int NS = a.stages;
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(NS) * L::kStageBytes);
  uint64_t* empty = full + NS;
  int* drain_info = reinterpret_cast<int*>(empty + NS);  // [0] stages issued
  float* part = reinterpret_cast<float*>(drain_info + 4);  // [C][R][MM]
  const int C = (a.K + kChunkK - 1) / kChunkK;
  const int n0 = blockIdx.x * a.rows_per_cta;
  const int R = min(a.rows_per_cta, a.N - n0);
  const int NRB = (R + kRB - 1) / kRB;
  const int T = C * NRB;
  // stages run chunk-major over the CTA's row blocks; each CTA starts at a
  // different chunk so that concurrent CTAs fetch different parts of x
  const int c_rot = blockIdx.x % C;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (a.pdl) pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    drain_info[0] = 0;
    fence_mbar_init();
  }
  __syncthreads();

  bool failed = false;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t policy = l2_policy_evict_first();
    const int T0 = min(T, NS);
    const int BH = a.box_rows;
    if (lane == 0) {
      prefetch_tmap(&a.tm_w);
      if (FMT == WQ_FP6_E3M2) prefetch_tmap(&a.tm_w2);
    }
    auto issue_x = [&](int t) {
      const int s = t % NS;
      if (t % NRB != 0) return;  // x of a chunk travels with the chunk's first stage only
      int c = t / NRB + c_rot;
      c = c >= C ? c - C : c;
      const int kc = min(kChunkK, a.K - c * kChunkK);
      if (lane < MM)
        bulk_g2s(ring + size_t(s) * L::kStageBytes + kRB * F::kRowBytes + lane * L::kXBytes,
                 a.x + size_t(lane) * a.K + size_t(c) * kChunkK, uint32_t(kc) * 2, &full[s]);
    };
    int t = 0;
    for (; t < T; ++t) {
      const int s = t % NS;
      if (!mbar_wait(&empty[s], ((t / NS) & 1) ^ 1)) {
        failed = true;
        break;
      }
      const int ci = t / NRB;
      const int rb = t - ci * NRB;
      const int c = ci + c_rot >= C ? ci + c_rot - C : ci + c_rot;
      const int rows = min(kRB, R - rb * kRB);
      const int nbox = (rows + BH - 1) / BH;
      const int kc = min(kChunkK, a.K - c * kChunkK);
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], uint32_t(nbox * BH * F::kRowBytes) + (rb == 0 ? MM * uint32_t(kc) * 2 : 0u));
        uint8_t* st = ring + size_t(s) * L::kStageBytes;
        for (int b = 0; b < nbox; ++b) {
          const int row = n0 + rb * kRB + b * BH;
          if constexpr (FMT == WQ_FP6_E3M2) {
            tma_load_2d(st + b * BH * 512, &a.tm_w, c * (512 / 4), row, &full[s], policy);
            tma_load_2d(st + kRB * 512 + b * BH * 256, &a.tm_w2, c * (256 / 4), row, &full[s], policy);
          } else {
            tma_load_2d(st + b * BH * F::kRowBytes, &a.tm_w, c * (F::kRowBytes / 4), row, &full[s], policy);
          }
        }
      }
      __syncwarp();
      if (t >= T0 || !a.pdl) issue_x(t);
      if (t == T0 - 1 && a.pdl) {
        // weights of the first ring fill are in flight; x may be written by
        // the previous kernel, so wait for it before fetching x
        pdl_wait();
        for (int t2 = 0; t2 < T0; ++t2) issue_x(t2);
      }
    }
    if (lane == 0) drain_info[0] = t;
    if (failed && a.pdl && t < T0) pdl_wait();
  } else {
    // ------------------------------------------------------------ consumers
    const int cw = warp - 1;
    const int ctid = threadIdx.x - 32;
    if (a.pdl) pdl_wait();
    int cur_c = -1;
    XRegs<FMT, MM> xr;
    constexpr int J = kRB / kConsumerWarps;  // rows of a stage this warp takes (4)
    // int4 scales / zeros of this warp's rows, fetched kPf stages ahead (a small
    // register ring), so their global latency hides behind the ring
    constexpr int kPf = (FMT == WQ_INT4) ? 3 : 1;
    uint32_t szq[kPf][J];
    auto fetch_sz = [&](int t, uint32_t* dst) {
      if constexpr (FMT == WQ_INT4) {
        if (t >= T) return;
        const int ci = t / NRB;
        const int rb = t - ci * NRB;
        const int c = ci + c_rot >= C ? ci + c_rot - C : ci + c_rot;
        const int rows = min(kRB, R - rb * kRB);
        const int k0 = c * kChunkK + lane * F::kLaneK;
        if (k0 >= a.K) return;
        const int G = a.K / a.groupsize;
#pragma unroll
        for (int j = 0; j < J; ++j) {
          const int i = cw + j * kConsumerWarps;
          if (i < rows) {
            const size_t gi = size_t(n0 + rb * kRB + i) * G + k0 / a.groupsize;
            dst[j] = uint32_t(ld_u16(a.scales + gi)) | (uint32_t(ld_u16(a.zeros + gi)) << 16);
          }
        }
      }
    };
    if constexpr (FMT == WQ_INT4) {
#pragma unroll
      for (int d = 0; d < kPf; ++d) fetch_sz(d, szq[d]);
    }
    for (int t = 0; t < T; ++t) {
      const int s = t % NS;
      uint32_t sz_cur[J];
      if constexpr (FMT == WQ_INT4) {
        // rotate the register ring: slot 0 is this stage
#pragma unroll
        for (int j = 0; j < J; ++j) sz_cur[j] = szq[0][j];
#pragma unroll
        for (int d = 0; d + 1 < kPf; ++d)
#pragma unroll
          for (int j = 0; j < J; ++j) szq[d][j] = szq[d + 1][j];
        fetch_sz(t + kPf, szq[kPf - 1]);
      }
      if (!mbar_wait(&full[s], (t / NS) & 1)) {
        failed = true;
        break;
      }
      const int ci = t / NRB;
      const int rb = t - ci * NRB;
      const int c = ci + c_rot >= C ? ci + c_rot - C : ci + c_rot;
      const int rows = min(kRB, R - rb * kRB);
      const int k0 = c * kChunkK + lane * F::kLaneK;
      const bool active = k0 < a.K;
      const uint8_t* st = ring + size_t(s) * L::kStageBytes;
      if (c != cur_c) {
        if (active) {
          load_x_smem<FMT, MM>(xr, st + kRB * F::kRowBytes, lane);
        }
        cur_c = c;
      }
      // all J rows of this warp at once: independent chains interleave
      float acc[J][MM];
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int i = cw + j * kConsumerWarps;
        if (active && i < rows) {
          if constexpr (FMT == WQ_FP6_E3M2)
            lane_dot<FMT, MM>(st + i * 512, st + kRB * 512 + i * 256, lane, xr, acc[j]);
          else
            lane_dot<FMT, MM>(st + i * F::kRowBytes, nullptr, lane, xr, acc[j]);
          if constexpr (FMT == WQ_INT4) {
            const float sc = bf16_bits_to_float(uint16_t(sz_cur[j] & 0xFFFFu));
            const float zc = fmaf(-128.f, sc, bf16_bits_to_float(uint16_t(sz_cur[j] >> 16)));
#pragma unroll
            for (int m = 0; m < MM; ++m) acc[j][m] = fmaf(sc, acc[j][m], zc * xr.xsum[m]);
          }
        } else {
#pragma unroll
          for (int m = 0; m < MM; ++m) acc[j][m] = 0.f;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // shared memory of the stage no longer read
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
          const int i = cw + j * kConsumerWarps;
          if (i < rows) part[(size_t(c) * R + rb * kRB + i) * MM + m] = kv;
        }
      }
    }
  }

  // ---------------------------------------------------------------- epilogue
  __syncthreads();
  const bool any_failed = __syncthreads_or(failed);
  if (any_failed) {
    // wait (bounded) until every copy issued into the ring has landed, then leave
    if (threadIdx.x == 0) {
      const int issued = drain_info[0];
      for (int t = max(0, issued - NS); t < issued; ++t) mbar_wait(&full[t % NS], (t / NS) & 1);
    }
    return;
  }
  for (int idx = threadIdx.x; idx < R * MM; idx += blockDim.x) {
    const int m = idx / R;
    const int r = idx - m * R;
    float v = 0.f;
    for (int c = 0; c < C; ++c) v += part[(size_t(c) * R + r) * MM + m];
    const int n = n0 + r;
    if constexpr (FMT == WQ_INT8) {
      v *= fp16_bits_to_float(a.scales[n]);
    } else if constexpr (FMT == WQ_FP6_E3M2) {
      v = (v * 0x1p124f) * fp16_bits_to_float(a.scales[n]);
    }
    a.y[size_t(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

// ----------------------------------------------------------------- launcher
constexpr size_t kGemvSmemPerSm = 220 * 1024;

constexpr int kBoxRows = 8;

template <int FMT, int MM>
static cudaError_t launch_gemv_t(const GemvParams& p0, cudaStream_t stream, int sm_count) {
  using L = GemvLayout<FMT, MM>;
  using F = GemvFmt<FMT>;
  GemvParams p = p0;
  const int C = (p.K + L::kChunkK - 1) / L::kChunkK;
  const int target = sm_count * gemv_ctas_per_sm(MM);
  const size_t kGemvSmemBudget = kGemvSmemPerSm / gemv_ctas_per_sm(MM);
  // rows per CTA: a multiple of the box height, about N / target
  int R = (p.N + target * kBoxRows - 1) / (target * kBoxRows) * kBoxRows;
  // keep the partial-sum area within a quarter of the budget
  const int max_r = int((kGemvSmemBudget / 4) / (size_t(C) * MM * 4)) / kBoxRows * kBoxRows;
  if (R > max_r) R = max_r;
  if (R < kBoxRows) R = kBoxRows;
  p.rows_per_cta = R;
  p.box_rows = kBoxRows;
  const size_t fixed = 16 * 8 + 16 + size_t(C) * R * MM * 4;
  if (fixed + 2 * size_t(L::kStageBytes) > 200 * 1024) return cudaErrorInvalidValue;
  int stages = fixed < kGemvSmemBudget ? int((kGemvSmemBudget - fixed) / L::kStageBytes) : 2;
  if (stages > 8) stages = 8;
  if (stages < 2) stages = 2;
  p.stages = stages;
  const size_t smem = size_t(stages) * L::kStageBytes + size_t(stages) * 16 + 16 + size_t(C) * R * MM * 4;

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
  e = cudaFuncSetAttribute(gemv_kernel<FMT, MM>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int grid = (p.N + R - 1) / R;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<FMT, MM>, p);
}

template <int FMT>
static cudaError_t launch_gemv_fmt(const GemvParams& p, cudaStream_t s, int sm_count) {
  switch (p.M) {
    case 1: return launch_gemv_t<FMT, 1>(p, s, sm_count);
    case 2: return launch_gemv_t<FMT, 2>(p, s, sm_count);
    case 3: return launch_gemv_t<FMT, 3>(p, s, sm_count);
    default: return launch_gemv_t<FMT, 4>(p, s, sm_count);
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
