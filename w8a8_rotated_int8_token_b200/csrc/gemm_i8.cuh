// Launch interface of the tcgen05 int8 GEMM (+ epilogue).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace convrot {

enum GemmEpilogue : int {
  kEpiDequantBf16 = 0,  // Y = bf16_rne(float(acc) * (x_scale[m] * w_scale) + bias[n])
  kEpiRawS32 = 1,       // acc as int32
};

struct GemmParams {
  int M, N, K;
  const float* x_scale;   // [M]   (dequant epilogue)
  const float* w_scale;   // [1]   (dequant epilogue)
  const uint16_t* bias;   // [N] bf16 bits or null
  int* status;            // status word: a timed-out wait ORs 5 into it
  uint64_t timeout_ns;    // bound of every device-side wait
  int group_m;            // M-blocks per raster group (0 = default)
  int num_m_blocks, num_n_blocks, num_k_blocks;  // filled by the launcher
};

// A = Xq [M,K] int8, B = Wq [N,K] int8, out = Y [M,N] bf16 or acc [M,N] int32.
cudaError_t launch_gemm_i8(int epi, const int8_t* A, const int8_t* B, void* out, GemmParams p,
                           cudaStream_t stream);

// One CTA waits on a barrier that nothing completes, for at most timeout_ns,
// then ORs 5 into *status.
cudaError_t launch_wait_timeout(int* status, uint64_t timeout_ns, cudaStream_t stream);

}  // namespace convrot
