// CUDA-core split-K GEMV for the decode linear at small M (sm_100a).
//
//   y[m, n] = sum_k x[m, k] * deq(W)[n, k]      m < MM <= 4
//
// The weight stream is the whole cost of a decode step (gpt-fast write-up,
// m.greenbasetech.com article 46368139_1106049486, paragraph on the memory
// bandwidth bound: each generated token reads every weight once).  The kernel
// therefore reads each packed byte exactly once with 128-bit non-allocating
// loads and hides the dequantization under the stream:
//
//  * A CTA owns a contiguous block of R output rows over all of K, so its bytes
//    are one contiguous region of the row-major packed matrix.
//  * K is cut into chunks of 32 lanes x LANE_K weights; the pair (row, chunk) is
//    one warp item: every lane loads 16 bytes (FP6: 16 + 8) of the row, decodes
//    them in registers and multiplies with its activations, which it holds in
//    registers for the whole chunk (permuted once so that decoded weight pairs
//    line up with activation pairs).
//  * A butterfly of warp shuffles reduces each item; per-(row, chunk) partials go
//    to shared memory and are summed in chunk order (deterministic), scaled and
//    rounded to bf16.
//
// Dequantization arithmetic (exact, fp32 accumulation):
//  * int4: decoded value 128 + q (bf16); per lane and group
//    s * sum(x (128 + q)) + (z - 128 s) * sum(x)  =  sum(x (q s + z)).
//  * FP6: decoded value v * 2^-124 (bf16, subnormal for e = 0); y = 2^124 s_n sum.
//  * int8: fp32 q; y = s_n sum.   bf16: plain products.
#include "wq_internal.h"
#include "wq_kernels.cuh"
#include "decode.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace wq {

template <int FMT>
struct GemvFmt;
template <>
struct GemvFmt<WQ_INT4> {
  static constexpr int kLaneK = 32, kBatch = 4;
};
template <>
struct GemvFmt<WQ_FP6_E3M2> {
  static constexpr int kLaneK = 32, kBatch = 4;
};
template <>
struct GemvFmt<WQ_INT8> {
  static constexpr int kLaneK = 8, kBatch = 8;
};
template <>
struct GemvFmt<WQ_BF16> {
  static constexpr int kLaneK = 8, kBatch = 4;
};

constexpr int kGemvThreads = 256;
// CTAs per SM the register budget is sized for (64 / 85 / 128 registers a thread).
__host__ __device__ constexpr int gemv_min_blocks(int mm) { return mm == 1 ? 4 : (mm == 2 ? 3 : 2); }

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint16_t ld_u16(const uint16_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
__device__ __forceinline__ float fp16_bits_to_float(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// Per-lane weight registers of one item.
template <int FMT>
struct WRegs;
template <>
struct WRegs<WQ_INT4> {
  uint4 w;
  uint16_t s, z;
};
template <>
struct WRegs<WQ_FP6_E3M2> {
  uint4 w4;
  uint2 w2;
};
template <>
struct WRegs<WQ_INT8> {
  uint2 w;
};
template <>
struct WRegs<WQ_BF16> {
  uint4 w;
};

// Per-lane activation registers of one chunk, for MM rows of x.
template <int FMT, int MM>
struct XRegs;
template <int MM>
struct XRegs<WQ_INT4, MM> {
  uint32_t p[MM][16];
  float sum[MM];
};
template <int MM>
struct XRegs<WQ_FP6_E3M2, MM> {
  uint32_t p[MM][16];
};
template <int MM>
struct XRegs<WQ_INT8, MM> {
  float v[MM][8];
};
template <int MM>
struct XRegs<WQ_BF16, MM> {
  uint32_t p[MM][4];
};

// Load the lane's activations of chunk-lane position k0 (permuted as needed).
template <int FMT, int MM>
__device__ __forceinline__ void load_x(XRegs<FMT, MM>& xr, const uint16_t* __restrict__ x, int K, int k0) {
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    const uint16_t* xm = x + size_t(m) * K + k0;
    if constexpr (FMT == WQ_INT4 || FMT == WQ_FP6_E3M2) {
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(xm) + q);
        xr.p[m][4 * q + 0] = pair_lo(v.x, v.z);
        xr.p[m][4 * q + 1] = pair_hi(v.x, v.z);
        xr.p[m][4 * q + 2] = pair_lo(v.y, v.w);
        xr.p[m][4 * q + 3] = pair_hi(v.y, v.w);
        if constexpr (FMT == WQ_INT4) {
          s += (bf16_lo_f(v.x) + bf16_hi_f(v.x)) + (bf16_lo_f(v.y) + bf16_hi_f(v.y)) +
               (bf16_lo_f(v.z) + bf16_hi_f(v.z)) + (bf16_lo_f(v.w) + bf16_hi_f(v.w));
        }
      }
      if constexpr (FMT == WQ_INT4) xr.sum[m] = s;
    } else if constexpr (FMT == WQ_INT8) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(xm));
      xr.v[m][0] = bf16_lo_f(v.x);
      xr.v[m][1] = bf16_hi_f(v.x);
      xr.v[m][2] = bf16_lo_f(v.y);
      xr.v[m][3] = bf16_hi_f(v.y);
      xr.v[m][4] = bf16_lo_f(v.z);
      xr.v[m][5] = bf16_hi_f(v.z);
      xr.v[m][6] = bf16_lo_f(v.w);
      xr.v[m][7] = bf16_hi_f(v.w);
    } else {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(xm));
      xr.p[m][0] = v.x;
      xr.p[m][1] = v.y;
      xr.p[m][2] = v.z;
      xr.p[m][3] = v.w;
    }
  }
}

template <int FMT>
__device__ __forceinline__ void load_w(WRegs<FMT>& wr, const GemvParams& a, int n, int k0) {
  if constexpr (FMT == WQ_INT4) {
    const uint8_t* base = static_cast<const uint8_t*>(a.packed) + size_t(n) * (a.K / 2) + k0 / 2;
    wr.w = ld_stream16(base);
    const size_t gidx = size_t(n) * (a.K / a.groupsize) + k0 / a.groupsize;
    wr.s = ld_u16(a.scales + gidx);
    wr.z = ld_u16(a.zeros + gidx);
  } else if constexpr (FMT == WQ_FP6_E3M2) {
    const uint8_t* p2 = static_cast<const uint8_t*>(a.packed);
    const uint8_t* p4 = p2 + size_t(a.N) * (a.K / 4);
    wr.w4 = ld_stream16(p4 + size_t(n) * (a.K / 2) + k0 / 2);
    wr.w2 = ld_stream8(p2 + size_t(n) * (a.K / 4) + k0 / 4);
  } else if constexpr (FMT == WQ_INT8) {
    wr.w = ld_stream8(static_cast<const uint8_t*>(a.packed) + size_t(n) * a.K + k0);
  } else {
    wr.w = ld_stream16(static_cast<const uint8_t*>(a.packed) + size_t(n) * a.K * 2 + size_t(k0) * 2);
  }
}

// Lane partial of one item for every activation row.
template <int FMT, int MM>
__device__ __forceinline__ void item_dot(const WRegs<FMT>& wr, const XRegs<FMT, MM>& xr, float acc[MM]) {
#pragma unroll
  for (int m = 0; m < MM; ++m) acc[m] = 0.f;
  if constexpr (FMT == WQ_INT4) {
    const uint32_t words[4] = {wr.w.x, wr.w.y, wr.w.z, wr.w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t p[4];
      decode_int4_word(words[q], p);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int m = 0; m < MM; ++m) fma_bf16x2(acc[m], p[r], xr.p[m][4 * q + r]);
    }
    const float s = bf16_bits_to_float(wr.s);
    const float zc = fmaf(-128.f, s, bf16_bits_to_float(wr.z));
#pragma unroll
    for (int m = 0; m < MM; ++m) acc[m] = fmaf(s, acc[m], zc * xr.sum[m]);
  } else if constexpr (FMT == WQ_FP6_E3M2) {
    const uint32_t w4[4] = {wr.w4.x, wr.w4.y, wr.w4.z, wr.w4.w};
    const uint32_t w2[2] = {wr.w2.x, wr.w2.y};
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      uint32_t p[8];
      decode_fp6_words(w2[v], w4[2 * v], w4[2 * v + 1], p);
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int m = 0; m < MM; ++m) fma_bf16x2(acc[m], p[j], xr.p[m][8 * v + j]);
    }
  } else if constexpr (FMT == WQ_INT8) {
    float v[8];
    decode_int8_word(wr.w.x, v);
    decode_int8_word(wr.w.y, v + 4);
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int m = 0; m < MM; ++m) acc[m] = fmaf(xr.v[m][i], v[i], acc[m]);
  } else {
    const uint32_t w[4] = {wr.w.x, wr.w.y, wr.w.z, wr.w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < MM; ++m) fma_bf16x2(acc[m], w[i], xr.p[m][i]);
  }
}

template <int FMT, int MM>
__global__ void __launch_bounds__(kGemvThreads, gemv_min_blocks(MM)) gemv_kernel(const GemvParams a) {
  using F = GemvFmt<FMT>;
  constexpr int kChunkK = 32 * F::kLaneK;
  constexpr int U = F::kBatch;
  extern __shared__ float part[];  // [C][R][MM]

  if (a.pdl) pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int n0 = blockIdx.x * a.rows_per_cta;
  const int R = min(a.rows_per_cta, a.N - n0);
  const int C = (a.K + kChunkK - 1) / kChunkK;
  const int I = R * C;
  const int i_beg = int((long long)warp * I / nwarps);
  const int i_end = int((long long)(warp + 1) * I / nwarps);

  bool waited = !a.pdl;
  int cur_c = -1;
  XRegs<FMT, MM> xr;

  for (int i = i_beg; i < i_end;) {
    const int c = i / R;
    const int r0 = i - c * R;
    const int nb = min(U, min(i_end - i, R - r0));
    const int k0 = c * kChunkK + lane * F::kLaneK;
    const bool active = k0 < a.K;

    WRegs<FMT> wr[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (u < nb && active) load_w<FMT>(wr[u], a, n0 + r0 + u, k0);

    if (!waited) {
      pdl_wait();
      waited = true;
    }
    if (c != cur_c) {
      if (active) load_x<FMT, MM>(xr, a.x, a.K, k0);
      cur_c = c;
    }

#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (u < nb) {
        float acc[MM];
        if (active) {
          item_dot<FMT, MM>(wr[u], xr, acc);
        } else {
#pragma unroll
          for (int m = 0; m < MM; ++m) acc[m] = 0.f;
        }
#pragma unroll
        for (int m = 0; m < MM; ++m) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xFFFFFFFFu, acc[m], o);
        }
        if (lane == 0) {
#pragma unroll
          for (int m = 0; m < MM; ++m) part[(size_t(c) * R + r0 + u) * MM + m] = acc[m];
        }
      }
    }
    i += nb;
  }
  if (!waited) pdl_wait();
  __syncthreads();

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
static int gemv_smem_rows(int N, int C, int MM, int sm_count) {
  const int target_ctas = sm_count * gemv_min_blocks(MM);
  int R = (N + target_ctas - 1) / target_ctas;
  const int max_r = 48 * 1024 / (C * MM * 4);
  if (R > max_r) R = max_r;
  return R < 1 ? 1 : R;
}

template <int FMT, int MM>
static cudaError_t launch_gemv_t(const GemvParams& p0, cudaStream_t stream, int sm_count) {
  constexpr int kChunkK = 32 * GemvFmt<FMT>::kLaneK;
  GemvParams p = p0;
  const int C = (p.K + kChunkK - 1) / kChunkK;
  p.rows_per_cta = gemv_smem_rows(p.N, C, MM, sm_count);
  const int grid = (p.N + p.rows_per_cta - 1) / p.rows_per_cta;
  const size_t smem = size_t(C) * p.rows_per_cta * MM * sizeof(float);
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

}  // namespace wq
