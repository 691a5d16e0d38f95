// Launch parameters and launchers of the wq device kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace wq {

struct GemvParams {
  const uint16_t* x;       // bf16 [M, K]
  const void* packed;      // packed weights of `fmt`
  const uint16_t* scales;  // fp16 [N] (int8, FP6) or bf16 [N, K/g] (int4)
  const uint16_t* zeros;   // bf16 [N, K/g] (int4)
  uint16_t* y;             // bf16 [M, N]
  int M, N, K, groupsize, fmt;
  int rows_per_cta;        // set by the launcher
  int pdl;                 // programmatic dependent launch enabled
};

// CUDA-core GEMV, 1 <= M <= 4.
cudaError_t launch_gemv(const GemvParams& p, cudaStream_t s, int sm_count);

// Decode-only kernel: code values as bf16 [N, K].
cudaError_t launch_unpack_debug(const void* packed, int fmt, int N, int K, uint16_t* out, cudaStream_t s);

}  // namespace wq
