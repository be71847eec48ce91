// Launch interface of the rotation + int8 quantisation kernels.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace convrot {

enum RotQuantMode : int {
  kRqActivation = 0,    // per-row scale; writes codes + scale per row
  kRqWeightAbsmax = 1,  // tensor absmax of the unnormalised transform (atomicMax)
  kRqWeightQuant = 2,   // codes + one tensor scale from that absmax
};

constexpr int kMaxRowsPerCta = 256;

struct RotQuantParams {
  const uint16_t* src;      // [rows, K] bf16 bits
  int64_t rows;
  int64_t K;
  int8_t* dst;              // [rows, K] codes (unused in kRqWeightAbsmax)
  float* scale;             // [rows] (activation) or [1] (weight)
  unsigned* tensor_absmax;  // weight modes: float bits of the unnormalised absmax
  int* status_reset;        // activation mode: status word zeroed by CTA 0, or null
  int threads_per_row;      // filled by launch_rotate_quant
  int rows_per_cta;         // filled by launch_rotate_quant
};

// Threads per row (K/32) and rows per CTA for a given K; false if K is not a
// multiple of 128 or above 32768.
bool rotquant_shape(int64_t K, int* threads_per_row, int* rows_per_cta);

cudaError_t launch_rotate_quant(int g, int mode, RotQuantParams p, cudaStream_t stream);

}  // namespace convrot
