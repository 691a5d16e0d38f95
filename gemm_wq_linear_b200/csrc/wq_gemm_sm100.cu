// Swap-AB weight-only-quantized GEMM on the sm_100a tensor cores (tcgen05),
// for the decode linear at 5 <= M <= 32.
//
//   D[n, m] = sum_k deq(W)[n, k] * x[m, k]     (the weight tile is the MMA's M = 128,
//                                               the activation rows its N = MPAD)
//
// The pages' kernel design (FP6-LLM / TC-FPx article, m.zhengruan.com news
// 124379, section "重新设计内核方案") dequantizes the weights in registers with
// SIMT bit operations and feeds them to the tensor cores as 16-bit operands,
// with a software pipeline overlapping dequantization and MMA.  Here that is
// laid out for B200:
//
//  * warp 0 streams packed weight tiles (128 rows x 128 k) and the matching
//    activation tile with 2-D tensor copies into an mbarrier ring;
//  * warps 2-5 (one thread per weight row) decode their row in registers and
//    write exact bf16 code values into an A tile in the canonical K-major
//    128-byte-swizzle layout (int4 as 128 + q, FP6 as its e3m2 value, int8 as q);
//  * one thread of warp 1 issues tcgen05.mma (kind::f16, 128 x MPAD x 16) with
//    A and B from shared memory and the fp32 accumulator in tensor memory;
//  * the same four warps read the accumulator with tcgen05.ld and apply the
//    scales in fp32: per output channel at the end (int8, FP6), or per group as
//    each group's partial product completes (int4: y += s_g D_g + (z_g - 128 s_g) X_g,
//    X_g the sum of x over the group);
//  * K is split over the CTAs of a thread-block cluster; the partial results are
//    summed in rank order through distributed shared memory (no global scratch).
//
// Activations and decoded weights are exact in bf16, so every product is exact
// and only the fp32 accumulation rounds.
#include "wq_internal.h"
#include "wq_kernels.cuh"
#include "decode.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace wq {

namespace gemm {

constexpr int kBM = 128;   // weight rows per tile (MMA M)
constexpr int kBK = 128;   // k per pipeline stage
constexpr int kThreads = 192;
constexpr int kATileBytes = kBM * kBK * 2;  // 32 KB: two 64-column swizzle atoms
constexpr int kNumA = 2;

template <int FMT>
struct Fmt;
template <>
struct Fmt<WQ_INT4> {
  static constexpr int kWBytes = kBM * 64;  // packed bytes of a 128 x 128 tile
};
template <>
struct Fmt<WQ_FP6_E3M2> {
  static constexpr int kWBytes = kBM * 64 + kBM * 32;  // 4-bit plane tile, then 2-bit plane tile
};
template <>
struct Fmt<WQ_INT8> {
  static constexpr int kWBytes = kBM * 128;
};
template <>
struct Fmt<WQ_BF16> {
  static constexpr int kWBytes = kBM * 256;  // the A operand itself (two swizzle atoms)
};

template <int FMT, int MPAD>
struct Layout {
  static constexpr int kXBytes = MPAD * 256;                    // two atoms of MPAD x 128 B
  static constexpr int kStage = Fmt<FMT>::kWBytes + kXBytes;   // multiple of 1024
  static constexpr int kNumW = (FMT == WQ_BF16) ? 5 : ((FMT == WQ_INT4) ? 6 : 4);
  static constexpr int kRingBytes = kNumW * kStage;
  static constexpr int kABytes = (FMT == WQ_BF16) ? 0 : kNumA * kATileBytes;
  static_assert(kStage % 1024 == 0, "stages must keep 1024-byte alignment");
};

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
__device__ __forceinline__ float fp16f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// Byte offset of 16-byte chunk c of row r in a tile whose rows are `row_bytes`
// long, written by a tensor copy with the matching swizzle (32/64/128 bytes).
template <int ROW_BYTES>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  if constexpr (ROW_BYTES == 32) return r * 32 + 16 * (c ^ ((r >> 2) & 1));
  else if constexpr (ROW_BYTES == 64) return r * 64 + 16 * (c ^ ((r >> 1) & 3));
  else return r * 128 + 16 * (c ^ (r & 7));
}

// Store 8 bf16 (one 16-byte chunk, k = 8 ac .. 8 ac + 7 within a 64-column atom)
// of row r into the A tile.
__device__ __forceinline__ void st_a_chunk(uint8_t* A, int r, int k0, uint4 v) {
  const int atom = k0 >> 6;
  const int ac = (k0 & 63) >> 3;
  *reinterpret_cast<uint4*>(A + atom * (kBM * 128) + swz<128>(r, ac)) = v;
}

// Decode row r of the packed stage tile into bf16 code values in A.
template <int FMT>
__device__ __forceinline__ void dequant_row(const uint8_t* W, uint8_t* A, int r) {
  if constexpr (FMT == WQ_INT4) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 w = *reinterpret_cast<const uint4*>(W + swz<64>(r, c));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        uint32_t p[4];
        decode_int4_word(ws[t], p);
        st_a_chunk(A, r, 32 * c + 8 * t, make_uint4(p[0], p[1], p[2], p[3]));
      }
    }
  } else if constexpr (FMT == WQ_FP6_E3M2) {
    const uint8_t* W2 = W + kBM * 64;
    uint32_t p4[16], p2[8];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 w = *reinterpret_cast<const uint4*>(W + swz<64>(r, c));
      p4[4 * c + 0] = w.x;
      p4[4 * c + 1] = w.y;
      p4[4 * c + 2] = w.z;
      p4[4 * c + 3] = w.w;
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint4 w = *reinterpret_cast<const uint4*>(W2 + swz<32>(r, c));
      p2[4 * c + 0] = w.x;
      p2[4 * c + 1] = w.y;
      p2[4 * c + 2] = w.z;
      p2[4 * c + 3] = w.w;
    }
    constexpr uint32_t kRebias = 0x7D807D80u;  // bf16 2^124 in both halves
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      uint32_t p[8];
      decode_fp6_words(p2[v], p4[2 * v], p4[2 * v + 1], p);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // value * 2^-124 (subnormal for e = 0) -> exact normal bf16 value
        asm("mul.rn.bf16x2 %0, %0, %1;" : "+r"(p[j]) : "r"(kRebias));
      }
      st_a_chunk(A, r, 16 * v, make_uint4(p[0], p[1], p[2], p[3]));
      st_a_chunk(A, r, 16 * v + 8, make_uint4(p[4], p[5], p[6], p[7]));
    }
  } else if constexpr (FMT == WQ_INT8) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 w = *reinterpret_cast<const uint4*>(W + swz<128>(r, c));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      uint32_t q[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float f[4];
        decode_int8_word(ws[t], f);
        q[2 * t] = pack_bf16x2_rn(f[0], f[1]);
        q[2 * t + 1] = pack_bf16x2_rn(f[2], f[3]);
      }
      st_a_chunk(A, r, 16 * c, make_uint4(q[0], q[1], q[2], q[3]));
      st_a_chunk(A, r, 16 * c + 8, make_uint4(q[4], q[5], q[6], q[7]));
    }
  }
}

__device__ __forceinline__ void dq_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

template <int FMT, int MPAD>
__global__ void __launch_bounds__(kThreads, 1) wq_gemm_kernel(const __grid_constant__ GemmParams a) {
  using L = Layout<FMT, MPAD>;
  constexpr int NW = L::kNumW;
  constexpr bool kInt4 = FMT == WQ_INT4;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment of the tiles (swizzle atoms and descriptors need it)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* atile = ring + L::kRingBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(atile + L::kABytes);
  uint64_t* full_w = bars;             // [NW]  tensor copies landed
  uint64_t* empty_w = full_w + NW;     // [NW]  MMA finished with the stage
  uint64_t* afull = empty_w + NW;      // [2]   A tile written
  uint64_t* aempty = afull + kNumA;    // [2]   MMA finished with the A tile
  uint64_t* dfull = aempty + kNumA;    // [8]   accumulator buffer complete
  uint64_t* dempty = dfull + 8;        // [8]   accumulator buffer drained
  uint64_t* done = dempty + 8;         // [1]   every MMA of the CTA completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* issued_slot = reinterpret_cast<int*>(tmem_slot + 1);
  float* xsum = reinterpret_cast<float*>(tmem_slot + 4);  // int4: [groups][MPAD]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = a.splits;
  const int tile = blockIdx.x / S;
  const int split = blockIdx.x % S;
  const int n0 = tile * kBM;
  const int KB = (a.K + kBK - 1) / kBK;
  const int kb0 = split * a.kb_per_split;
  const int nkb = max(0, min(a.kb_per_split, KB - kb0));
  const int g = kInt4 ? a.groupsize : kBK;
  const int gpb = kBK / g;                                  // groups per k-block (int4)
  const int kbeg = kb0 * kBK;
  const int kend = min(a.K, (kb0 + nkb) * kBK);
  const int ngroups = kInt4 ? (kend - kbeg) / g : 0;      // groups of this CTA
  const int nd = kInt4 ? 2 * gpb : 1;                      // accumulator buffers
  const uint32_t tmem_cols = a.tmem_cols;

  if (a.pdl) pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < NW; ++i) {
      mbar_init(&full_w[i], 1);
      mbar_init(&empty_w[i], 1);
    }
    for (int i = 0; i < kNumA; ++i) {
      mbar_init(&afull[i], 4);
      mbar_init(&aempty[i], 1);
    }
    for (int i = 0; i < 8; ++i) {
      mbar_init(&dfull[i], 1);
      mbar_init(&dempty[i], 4);
    }
    mbar_init(done, 1);
    *issued_slot = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool failed = false;
  float acc[MPAD];
#pragma unroll
  for (int m = 0; m < MPAD; ++m) acc[m] = 0.f;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      prefetch_tmap(&a.tm_w);
      prefetch_tmap(&a.tm_x);
      if (FMT == WQ_FP6_E3M2) prefetch_tmap(&a.tm_w2);
      const int T0 = min(nkb, NW);
      auto issue_x = [&](int j) {
        uint8_t* st = ring + size_t(j % NW) * L::kStage;
        const int kx = (kb0 + j) * kBK;
        tma_load_2d_nohint(st + Fmt<FMT>::kWBytes, &a.tm_x, kx, 0, &full_w[j % NW]);
        tma_load_2d_nohint(st + Fmt<FMT>::kWBytes + MPAD * 128, &a.tm_x, kx + 64, 0, &full_w[j % NW]);
      };
      int j = 0;
      for (; j < nkb; ++j) {
        const int s = j % NW;
        if (!mbar_wait(&empty_w[s], ((j / NW) & 1) ^ 1)) {
          failed = true;
          break;
        }
        mbar_arrive_expect_tx(&full_w[s], uint32_t(L::kStage));
        uint8_t* st = ring + size_t(s) * L::kStage;
        const int kb = kb0 + j;
        if constexpr (FMT == WQ_INT4) {
          tma_load_2d(st, &a.tm_w, kb * 16, n0, &full_w[s], policy);
        } else if constexpr (FMT == WQ_FP6_E3M2) {
          tma_load_2d(st, &a.tm_w, kb * 16, n0, &full_w[s], policy);
          tma_load_2d(st + kBM * 64, &a.tm_w2, kb * 8, n0, &full_w[s], policy);
        } else if constexpr (FMT == WQ_INT8) {
          tma_load_2d(st, &a.tm_w, kb * 32, n0, &full_w[s], policy);
        } else {
          tma_load_2d(st, &a.tm_w, kb * kBK, n0, &full_w[s], policy);
          tma_load_2d(st + kBM * 128, &a.tm_w, kb * kBK + 64, n0, &full_w[s], policy);
        }
        if (j >= T0 || !a.pdl) issue_x(j);
        if (j == T0 - 1 && a.pdl) {
          pdl_wait();  // x may come from the previous kernel
          for (int j2 = 0; j2 < T0; ++j2) issue_x(j2);
        }
      }
      *issued_slot = j;
      if (failed && a.pdl && j < T0) pdl_wait();
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, MPAD);
      int dcount = 0;  // int4: accumulator buffers used so far
      for (int j = 0; j < nkb && !failed; ++j) {
        const int s = j % NW;
        const int ai = j % kNumA;
        uint8_t* A;
        if constexpr (FMT == WQ_BF16) {
          if (!mbar_wait(&full_w[s], (j / NW) & 1)) { failed = true; break; }
          A = ring + size_t(s) * L::kStage;
        } else {
          if (!mbar_wait(&afull[ai], (j / kNumA) & 1)) { failed = true; break; }
          A = atile + size_t(ai) * kATileBytes;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(A);
        const uint32_t b_base = smem_u32(ring + size_t(s) * L::kStage + Fmt<FMT>::kWBytes);
        if constexpr (kInt4) {
          const int kvalid = min(kBK, a.K - (kb0 + j) * kBK);
          for (int gi = 0; gi < gpb && gi * g < kvalid; ++gi, ++dcount) {
            const int b = dcount % nd;
            if (!mbar_wait(&dempty[b], ((dcount / nd) & 1) ^ 1)) { failed = true; break; }
            tc_fence_after();
            for (int kk = gi * (g / 16); kk < (gi + 1) * (g / 16); ++kk) {
              const uint32_t ao = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
              const uint32_t bo = (kk >> 2) * (MPAD * 128) + (kk & 3) * 32;
              mma_bf16(tmem + b * MPAD, smem_desc_sw128(a_base + ao), smem_desc_sw128(b_base + bo), idesc,
                       kk != gi * (g / 16));
            }
            mma_commit(&dfull[b]);
          }
        } else {
#pragma unroll 1
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t ao = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
            const uint32_t bo = (kk >> 2) * (MPAD * 128) + (kk & 3) * 32;
            mma_bf16(tmem, smem_desc_sw128(a_base + ao), smem_desc_sw128(b_base + bo), idesc, (j | kk) != 0);
          }
        }
        if constexpr (FMT != WQ_BF16) mma_commit(&aempty[ai]);
        mma_commit(&empty_w[s]);
      }
      if (!kInt4) mma_commit(&dfull[0]);  // accumulator complete
      mma_commit(done);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequant + epilogue
    const int r = 32 * (warp & 3) + lane;  // TMEM lane quadrant of this warp
    const int n = n0 + r;
    const uint32_t taddr_row = tmem + (uint32_t(32 * (warp & 3)) << 16);
    if (a.pdl) pdl_wait();
    if constexpr (kInt4) {
      // sums of x over every group of this CTA's k range
      for (int idx = threadIdx.x - 64; idx < ngroups * MPAD; idx += 128) {
        const int gl = idx / MPAD;
        const int m = idx - gl * MPAD;
        float sacc = 0.f;
        if (m < a.M) {
          const uint4* xp = reinterpret_cast<const uint4*>(a.x + size_t(m) * a.K + kbeg + gl * g);
          for (int q = 0; q < g / 8; ++q) {
            const uint4 v = __ldg(xp + q);
            sacc += (bf16_lo_f(v.x) + bf16_hi_f(v.x)) + (bf16_lo_f(v.y) + bf16_hi_f(v.y)) +
                    (bf16_lo_f(v.z) + bf16_hi_f(v.z)) + (bf16_lo_f(v.w) + bf16_hi_f(v.w));
          }
        }
        xsum[idx] = sacc;
      }
      dq_sync();
    }
    int gdone = 0;  // int4: groups folded into acc so far
    // int4: fold the accumulator buffers of groups [gdone, upto) into acc
    auto fold_groups = [&](int upto) {
      if constexpr (kInt4) {
        const int G = a.K / g;
        for (; gdone < upto && !failed; ++gdone) {
          const int b = gdone % nd;
          if (!mbar_wait(&dfull[b], (gdone / nd) & 1)) { failed = true; break; }
          tc_fence_after();
          uint32_t d[MPAD];
          tmem_ld_32x32b<MPAD>(taddr_row + b * MPAD, d);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dempty[b]);
          if (n < a.N) {
            const size_t gi = size_t(n) * G + (kbeg / g) + gdone;
            const float sc = bf16f(a.scales[gi]);
            const float zc = fmaf(-128.f, sc, bf16f(a.zeros[gi]));
            const float* xs = xsum + gdone * MPAD;
#pragma unroll
            for (int m = 0; m < MPAD; ++m) acc[m] = fmaf(sc, __uint_as_float(d[m]), fmaf(zc, xs[m], acc[m]));
          }
        }
      }
    };
    if constexpr (FMT != WQ_BF16) {
      for (int j = 0; j < nkb && !failed; ++j) {
        const int s = j % NW;
        const int ai = j % kNumA;
        if (!mbar_wait(&full_w[s], (j / NW) & 1)) { failed = true; break; }
        if (!mbar_wait(&aempty[ai], ((j / kNumA) & 1) ^ 1)) { failed = true; break; }
        dequant_row<FMT>(ring + size_t(s) * L::kStage, atile + size_t(ai) * kATileBytes, r);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[ai]);
        // fold the groups of the previous k-block while the MMA runs on this one
        if constexpr (kInt4) fold_groups(min(ngroups, j * gpb));
      }
    }
    if constexpr (kInt4) {
      fold_groups(ngroups);
    } else if (!failed) {
      if (mbar_wait(&dfull[0], 0)) {
        tc_fence_after();
        uint32_t d[MPAD];
        tmem_ld_32x32b<MPAD>(taddr_row, d);
        tmem_ld_wait();
        float sc = 1.f;
        if (n < a.N) {
          if constexpr (FMT == WQ_INT8 || FMT == WQ_FP6_E3M2) sc = fp16f(a.scales[n]);
        }
#pragma unroll
        for (int m = 0; m < MPAD; ++m) acc[m] = __uint_as_float(d[m]) * sc;
      } else {
        failed = true;
      }
    }
  }

  // ---------------------------------------------------------------- reduction + output
  tc_fence_before();
  const bool any_failed = __syncthreads_or(failed);
  if (any_failed) {
    if (threadIdx.x == 0) {
      // let every issued copy land and every issued MMA finish before leaving
      const int issued = *issued_slot;
      for (int j = max(0, issued - NW); j < issued; ++j) mbar_wait(&full_w[j % NW], (j / NW) & 1);
      mbar_wait(done, 0);
    }
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, tmem_cols);

  const bool epi = warp >= 2;
  const int r = 32 * (warp & 3) + lane;
  const int n = n0 + r;
  if (S == 1) {
    if (epi && !any_failed && n < a.N) {
#pragma unroll
      for (int m = 0; m < MPAD; ++m)
        if (m < a.M) a.y[size_t(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[m]));
    }
    return;
  }
  // split-K over the cluster: partials through distributed shared memory
  float* red = reinterpret_cast<float*>(ring);  // [128][MPAD], the ring is idle now
  if (epi) {
#pragma unroll
    for (int m = 0; m < MPAD; m += 4)
      *reinterpret_cast<float4*>(red + r * MPAD + m) = make_float4(acc[m], acc[m + 1], acc[m + 2], acc[m + 3]);
  }
  cluster_sync_all();
  if (cluster_ctarank() == 0 && epi && !any_failed && n < a.N) {
    const uint32_t base = smem_u32(red + r * MPAD);
    for (int q = 1; q < S; ++q) {
      const uint32_t rb = map_to_rank(base, uint32_t(q));
#pragma unroll
      for (int m = 0; m < MPAD; m += 4) {
        const float4 v = ld_cluster_f4(rb + m * 4);
        acc[m] += v.x;
        acc[m + 1] += v.y;
        acc[m + 2] += v.z;
        acc[m + 3] += v.w;
      }
    }
#pragma unroll
    for (int m = 0; m < MPAD; ++m)
      if (m < a.M) a.y[size_t(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[m]));
  }
  cluster_sync_all();  // keep every CTA's shared memory alive until rank 0 has read it
}

}  // namespace gemm

// ----------------------------------------------------------------- launcher
template <int FMT, int MPAD>
static cudaError_t launch_gemm_t(const GemmParams& p0, cudaStream_t stream, int sm_count) {
  using L = gemm::Layout<FMT, MPAD>;
  GemmParams p = p0;
  const int tiles = (p.N + gemm::kBM - 1) / gemm::kBM;
  const int KB = (p.K + gemm::kBK - 1) / gemm::kBK;
  // split K over a cluster so that about one CTA per SM is busy; int4 keeps each
  // CTA's k range at most 4096 (the per-group x sums live in shared memory)
  int S = (sm_count + tiles / 2) / tiles;
  if (FMT == WQ_INT4) S = S < (p.K + 4095) / 4096 ? (p.K + 4095) / 4096 : S;
  if (S > 8) S = 8;
  if (S > KB) S = KB;
  if (S < 1) S = 1;
  int kbps = (KB + S - 1) / S;
  S = (KB + kbps - 1) / kbps;
  if (FMT == WQ_INT4 && kbps * gemm::kBK > 4096) return cudaErrorInvalidValue;  // K > 32768 for int4
  p.splits = S;
  p.kb_per_split = kbps;
  const int g = FMT == WQ_INT4 ? p.groupsize : gemm::kBK;
  const int nd = FMT == WQ_INT4 ? 2 * (gemm::kBK / g) : 1;
  uint32_t cols = 32;
  while (cols < uint32_t(nd * MPAD)) cols <<= 1;
  p.tmem_cols = cols;
  const size_t xsum_bytes = FMT == WQ_INT4 ? size_t(kbps * gemm::kBK / g) * MPAD * 4 : 0;
  const size_t smem = 1024 + L::kRingBytes + L::kABytes + 64 * 8 + 64 + xsum_bytes;

  cudaError_t e;
  const uint8_t* w = static_cast<const uint8_t*>(p.packed);
  if constexpr (FMT == WQ_INT4) {
    e = make_tmap_2d(&p.tm_w, w, 4, uint64_t(p.K) / 8, p.N, uint64_t(p.K) / 2, 16, gemm::kBM, 64);
  } else if constexpr (FMT == WQ_FP6_E3M2) {
    e = make_tmap_2d(&p.tm_w, w + size_t(p.N) * (p.K / 4), 4, uint64_t(p.K) / 8, p.N, uint64_t(p.K) / 2, 16, gemm::kBM,
                     64);
    if (e == cudaSuccess) e = make_tmap_2d(&p.tm_w2, w, 4, uint64_t(p.K) / 16, p.N, uint64_t(p.K) / 4, 8, gemm::kBM, 32);
  } else if constexpr (FMT == WQ_INT8) {
    e = make_tmap_2d(&p.tm_w, w, 4, uint64_t(p.K) / 4, p.N, uint64_t(p.K), 32, gemm::kBM, 128);
  } else {
    e = make_tmap_2d(&p.tm_w, w, 2, uint64_t(p.K), p.N, uint64_t(p.K) * 2, 64, gemm::kBM, 128);
  }
  if (e == cudaSuccess) e = make_tmap_2d(&p.tm_x, p.x, 2, uint64_t(p.K), p.M, uint64_t(p.K) * 2, 64, MPAD, 128);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gemm::wq_gemm_kernel<FMT, MPAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  if (S > 1) {
    e = cudaFuncSetAttribute(gemm::wq_gemm_kernel<FMT, MPAD>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * S);
  cfg.blockDim = dim3(gemm::kThreads);
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
  return cudaLaunchKernelEx(&cfg, gemm::wq_gemm_kernel<FMT, MPAD>, p);
}

template <int FMT>
static cudaError_t launch_gemm_fmt(const GemmParams& p, cudaStream_t s, int sms) {
  if (p.M <= 8) return launch_gemm_t<FMT, 8>(p, s, sms);
  if (p.M <= 16) return launch_gemm_t<FMT, 16>(p, s, sms);
  return launch_gemm_t<FMT, 32>(p, s, sms);
}

cudaError_t launch_gemm(const GemmParams& p, cudaStream_t s, int sms) {
  switch (p.fmt) {
    case WQ_INT4: return launch_gemm_fmt<WQ_INT4>(p, s, sms);
    case WQ_FP6_E3M2: return launch_gemm_fmt<WQ_FP6_E3M2>(p, s, sms);
    case WQ_INT8: return launch_gemm_fmt<WQ_INT8>(p, s, sms);
    default: return launch_gemm_fmt<WQ_BF16>(p, s, sms);
  }
}

cudaError_t gemm_take_status(uint32_t* status) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(status, g_device_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(uint32_t));
}

}  // namespace wq
