// convrot_linear_noalloc: convrot_linear for callers that cannot allocate
// device memory. Such callers include host applications that own the whole
// device-memory budget and hand a plugin nothing but its input and output
// buffers (an inference server's arena, a fixed-budget deployment), and
// latency-critical loops where a cudaMalloc/cudaFree could synchronise the
// device or fail at a bad time.
//
// The scratch that convrot_linear takes as `ws` (status word, token scales,
// int8 activation codes) lives here in one file-scope device array of fixed
// size, allocated when the library's device code is loaded on a GPU and held
// until the process exits. Host code cannot use the array's name as a device
// address (it is a host-side stand-in), so the first call on each device asks
// the runtime for the array's device address with cudaGetSymbolAddress, with
// that device current, and keeps it for later calls.
//
// Every call shares the one array and leaves its contents behind. The status
// word is cleared by the first kernel of every call, and the codes and scales
// are fully rewritten, so nothing from an earlier call leaks into a result.
// Calls that may overlap on the GPU (different streams without ordering, or
// several host threads) race on the array and must not be issued.

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "convrot.h"

// The scratch of every convrot_linear_noalloc call on this device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CONVROT_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_noalloc_scratch on the current device (set up once per device).
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p != nullptr) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr) return nullptr;
  g_scratch_addr[dev].store(addr, std::memory_order_release);
  return addr;
}

}  // namespace

extern "C" convrot_status convrot_linear_noalloc(const void* X, int64_t M, int64_t K, int g, const int8_t* Wq,
                                                 const float* w_scale, int64_t N, const void* bias, void* Y,
                                                 int* device_status, convrot_stream_t stream) {
  if (device_status != nullptr && (reinterpret_cast<uintptr_t>(device_status) % 4) != 0)
    return CONVROT_ERR_INVALID_ARG;
  const size_t need = convrot_linear_workspace_bytes(M, N, K, g);
  if (need == 0 || M == 0) {
    // an invalid shape (convrot_linear reports which check failed, before any
    // setup) or no tokens (it returns without launching; the scratch is not
    // used, and this call's status, 0, is what device_status receives)
    const convrot_status st = convrot_linear(X, M, K, g, Wq, w_scale, N, bias, Y, nullptr, 0, stream);
    if (st != CONVROT_OK || device_status == nullptr) return st;
    return cudaMemsetAsync(device_status, 0, sizeof(int), reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? CONVROT_OK
               : CONVROT_ERR_CUDA;
  }
  if (need > static_cast<size_t>(CONVROT_NOALLOC_SCRATCH_BYTES)) return CONVROT_ERR_WORKSPACE;
  void* ws = scratch_address();
  if (ws == nullptr) return CONVROT_ERR_CUDA;
  const convrot_status st =
      convrot_linear(X, M, K, g, Wq, w_scale, N, bias, Y, ws, CONVROT_NOALLOC_SCRATCH_BYTES, stream);
  if (st != CONVROT_OK || device_status == nullptr) return st;
  // the status word is the first int of the scratch
  if (cudaMemcpyAsync(device_status, ws, sizeof(int), cudaMemcpyDeviceToDevice,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  return CONVROT_OK;
}
