// Measured peaks of the units the hot kernels are bound by. The int8 tensor pipe: the same instruction the layer's GEMM
// issues (tcgen05.mma.cta_group::2.kind::i8, M = 256, N = 256, K = 32 per
// instruction, both operands from shared memory) in a loop with no global
// memory traffic, so that a timed launch gives the rate the tensor cores
// sustain on this GPU at its current clock. The operands are zero or copied
// from a caller buffer (the layer's own codes): the rate at a fixed clock does
// not depend on them, but the power drawn does, and with it the clock the
// GPU holds under its power limit. The special-function unit's exp2
// (the unit the attention softmax is bound by): independent chains of
// ex2.approx in every thread of a full grid. Measurement aids for the
// rooflines; they compute nothing of the layer.

#include <cuda_runtime.h>

#include <cstdint>

#include "convrot.h"
#include "ptx_sm100.cuh"

namespace convrot {

namespace {

constexpr int kProbeTile = 128 * 128;  // bytes of this CTA's A (and of its B) operand tile
constexpr int kProbeThreads = 128;
constexpr int kTimeoutStatus = 5;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kProbeThreads, 1)
    i8_peak_pair_kernel(int64_t iters, const uint4* operands, int64_t operand_chunks, int* status,
                        unsigned long long* clock_rec, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t done;
  __shared__ uint32_t tmem_ptr;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool leader = cluster_ctarank() == 0;

  // this CTA's A and B tiles: zeros, or 2 * kProbeTile consecutive bytes of the
  // caller's buffer starting at chunk (blockIdx.x * 2 * kProbeTile / 16) modulo
  // its length (16-byte chunks); the tensor cores read them through the async proxy
  constexpr int kChunks = 2 * kProbeTile / 16;
  for (int i = threadIdx.x; i < kChunks; i += blockDim.x) {
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (operands != nullptr) v = operands[(static_cast<int64_t>(blockIdx.x) * kChunks + i) % operand_chunks];
    reinterpret_cast<uint4*>(smem)[i] = v;
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_ptr, 256);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = tmem_ptr;

  if (warp == 1 && lane == 0 && leader) {
    const uint32_t a_base = smem_addr(smem);
    const uint32_t b_base = smem_addr(smem + kProbeTile);
    constexpr uint32_t idesc = idesc_i8(256, 256);
    if (blockIdx.x == 0) {
      clock_rec[0] = clock64();
      clock_rec[1] = global_timer_ns();
    }
    for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_i8_pair(tmem_base, smem_desc_k_sw128(a_base + k * 32), smem_desc_k_sw128(b_base + k * 32), idesc,
                    (i | k) != 0 ? 1u : 0u);
    }
    mma_commit_pair_mc(&done, 0x3);  // both CTAs learn that every MMA has finished
  }
  if (threadIdx.x == 0) {
    if (!mbar_wait_bounded(&done, 0u, nullptr, timeout_ns)) {
      atomicOr(status, kTimeoutStatus);
    } else if (blockIdx.x == 0) {
      clock_rec[2] = clock64();
      clock_rec[3] = global_timer_ns();
    }
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 256);
}

constexpr int kEx2Threads = 256;
constexpr int kEx2CtasPerSm = 8;
constexpr int kEx2Chains = 8;

__global__ void __launch_bounds__(kEx2Threads) ex2_peak_kernel(int64_t iters, float* sink) {
  float y[kEx2Chains];
#pragma unroll
  for (int i = 0; i < kEx2Chains; ++i) y[i] = 0.5f + 0.01f * static_cast<float>(threadIdx.x & 7) + 0.001f * i;
  for (int64_t it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kEx2Chains; ++i) y[i] = ex2_approx(-y[i]);  // stays in [0.5, 1)
  }
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < kEx2Chains; ++i) s += y[i];
  if (s == 12345.0f) sink[threadIdx.x] = s;  // never true: keeps the chains live
}

}  // namespace

}  // namespace convrot

extern "C" {

convrot_status convrot_probe_ex2_peak(int64_t iters, void* ws, size_t ws_bytes, convrot_stream_t stream) {
  if (iters < 1 || iters > (int64_t(1) << 24)) return CONVROT_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % 256) != 0 || ws_bytes < 256 * sizeof(float))
    return CONVROT_ERR_WORKSPACE;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  convrot::ex2_peak_kernel<<<sms * convrot::kEx2CtasPerSm, convrot::kEx2Threads, 0,
                             reinterpret_cast<cudaStream_t>(stream)>>>(iters, static_cast<float*>(ws));
  return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

int64_t convrot_probe_ex2_per_iter(void) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return static_cast<int64_t>(sms) * convrot::kEx2CtasPerSm * convrot::kEx2Threads * convrot::kEx2Chains;
}

convrot_status convrot_probe_i8_peak(int64_t iters, const void* operands, size_t operand_bytes, void* ws,
                                     size_t ws_bytes, convrot_stream_t stream) {
  // at most 2^20 x 512 tensor cycles (about 0.3 s at 1.9 GHz): well inside the 2 s bound of the final wait
  if (iters < 1 || iters > (int64_t(1) << 20)) return CONVROT_ERR_INVALID_ARG;
  if (operands != nullptr &&
      ((reinterpret_cast<uintptr_t>(operands) % 16) != 0 || operand_bytes < 16 || (operand_bytes % 16) != 0))
    return CONVROT_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % 256) != 0 || ws_bytes < 256) return CONVROT_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  const int smem = 2 * convrot::kProbeTile + 1024;
  if (cudaFuncSetAttribute(convrot::i8_peak_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return CONVROT_ERR_CUDA;
  int* status = static_cast<int*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return CONVROT_ERR_CUDA;
  // one CTA pair per two SMs, every SM busy
  convrot::i8_peak_pair_kernel<<<(sms / 2) * 2, convrot::kProbeThreads, smem, s>>>(
      iters, static_cast<const uint4*>(operands), static_cast<int64_t>(operand_bytes / 16), status,
      reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + CONVROT_WS_CLOCK_RECORD_OFFSET), 2000000000ull);
  return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

int convrot_probe_i8_peak_ctas(void) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return (sms / 2) * 2;
}

}  // extern "C"
