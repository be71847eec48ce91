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
// address (it is a host-side stand-in), so the first call in each CUDA
// context asks the runtime for the array's device address with
// cudaGetSymbolAddress, with that device current, and keeps it together with
// the context's unique id. A later call in another context of the same device
// (after cudaDeviceReset, or once the primary context was released and made
// anew, which loads the module again and may move the array) looks it up
// again.
//
// Every call shares the one array and leaves its contents behind. The status
// word is cleared by the first kernel of every call, and the codes and scales
// are fully rewritten, so nothing from an earlier call leaks into a result.
// Calls that may overlap on the GPU (different streams without ordering, or
// several host threads) race on the array and must not be issued.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "convrot.h"

// The scratch of every convrot_linear_noalloc call on this device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CONVROT_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The driver's context queries, found once through the runtime (the library
// does not link libcuda directly).
bool context_queries(CtxGetCurrentFn* get_current, CtxGetIdFn* get_id) {
  static CtxGetCurrentFn cur = nullptr;
  static CtxGetIdFn id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      cur = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      id = reinterpret_cast<CtxGetIdFn>(f);
  });
  *get_current = cur;
  *get_id = id;
  return cur != nullptr && id != nullptr;
}

// Unique id of the calling thread's current context (0 if there is none).
unsigned long long current_context_id(CtxGetCurrentFn get_current, CtxGetIdFn get_id) {
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

struct ScratchSlot {
  unsigned long long ctx_id = 0;  // context the address belongs to (0: none yet)
  void* addr = nullptr;
};

std::mutex g_scratch_mutex;
ScratchSlot g_scratch_slot[kMaxDevices];

// Device address of g_noalloc_scratch in the current device's current context.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
  if (!context_queries(&get_current, &get_id)) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchSlot& slot = g_scratch_slot[dev];
  unsigned long long id = current_context_id(get_current, get_id);
  if (id != 0 && id == slot.ctx_id) return slot.addr;
  // first call in this context (the lookup also makes the device's primary
  // context current if no context was yet)
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr) return nullptr;
  id = current_context_id(get_current, get_id);
  if (id == 0) return nullptr;
  slot.ctx_id = id;
  slot.addr = addr;
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
