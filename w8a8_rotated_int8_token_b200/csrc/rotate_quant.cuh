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
// Input slots per CTA: the block computed and the ones in flight. Rows of
// K >= kRqDeepMinK (one row per CTA) take a third slot: 35.7 against 37.5 us
// on the 4608 x 12288 activation, while shorter rows lose resident CTAs to it.
constexpr int kRqStages = 2;
constexpr int kRqStagesDeep = 3;
constexpr int64_t kRqDeepMinK = 8192;
constexpr int kRqTimeoutStatus = 5;   // CONVROT_ERR_DEVICE_TIMEOUT
constexpr int kRotQuantMaxThreads = 512;  // K/64 threads per row: K <= 32768

struct RotQuantParams {
  const uint16_t* src;      // [rows, K] bf16 bits (IEEE fp16 bits with in_f16)
  int in_f16;               // 0: bf16 input, 1: fp16 input
  int64_t rows;
  int64_t K;
  int64_t ldx;              // row stride of src in elements (>= K, a multiple of 8); 0 = K
  int8_t* dst;              // [rows, K] codes (unused in kRqWeightAbsmax)
  float* scale;             // [rows] (activation) or [1] (weight)
  unsigned* tensor_absmax;  // weight modes: float bits of the unnormalised absmax
  int* status_reset;        // activation mode: status word zeroed by CTA 0, or null
  unsigned* zero_words;     // activation mode: words zeroed by CTA 0 for the next kernel (or null)
  int zero_count;
  int* status;              // a timed-out wait ORs 5 into it (may be null)
  uint64_t timeout_ns;      // bound of every device-side wait
  int late_trigger;         // 1: dependents launch only at exit (dst is a weight a GEMM reads early)
  int threads_per_row;      // filled by launch_rotate_quant
  int rows_per_cta;         // filled by launch_rotate_quant
};

// Threads per row (K/64) and rows per CTA for a given K; false if K is not a
// multiple of 128 or above 32768. The CTA has rows*K/64 threads rounded up to
// whole warps; the padding threads hold zeros.
bool rotquant_shape(int64_t K, int* threads_per_row, int* rows_per_cta);

// Bytes of one input slot: rows_per_cta rows of K bf16, rounded up to whole
// 4 KB regions (one per warp of the CTA; 32 lanes x 64 bf16).
__host__ __device__ inline uint32_t rotquant_slot_bytes(int rows_per_cta, int64_t K) {
  const uint32_t bytes = static_cast<uint32_t>(rows_per_cta) * static_cast<uint32_t>(K) * 2u;
  return (bytes + 4095u) / 4096u * 4096u;
}

cudaError_t launch_rotate_quant(int g, int mode, RotQuantParams p, cudaStream_t stream);

}  // namespace convrot
