// C ABI of libconvrot (declared in include/convrot.h): argument checks on the
// host, workspace layout, and the launches of the rotation/quantisation and
// GEMM kernels. Nothing here allocates device memory or synchronises, except
// convrot_read_device_status.

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "convrot.h"
#include "gemm_i8.cuh"
#include "rotate_quant.cuh"

namespace {

constexpr int kAbiVersion = 9;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s bound on every device-side wait
// convrot_linear runs two kernels chained with programmatic dependent launch.
// The one-launch form (rotate+quantise worker warps inside the GEMM kernel,
// convrot_linear_one_launch) is correct but, measured on the DiT QKV layer,
// its workers fall behind the tensor cores (137 us against 94 + 16 us for the
// two kernels at the time), so it is offered only as its own entry point.

// Workspace of convrot_linear:
// [status word | 256 B][M-block ready counters, 8 B each][token scales][int8 codes]
// and, for the weight-streaming GEMM (M <= 64) split over all SMs,
// [arrival counters, one per 128 weight rows][int32 partial accumulators].
constexpr size_t kStatusBytes = 256;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct LinearWs {
  size_t ready_off, scale_off, codes_off, split_count_off, split_part_off, total;
  bool split;
};

#ifndef CONVROT_SMALLM_SPLIT
#define CONVROT_SMALLM_SPLIT 0
#endif

// Whether the workspace of a shape holds the split buffers of the
// weight-streaming GEMM (the layout depends on the shape only) ...
bool linear_has_split_buffers(int64_t M, int64_t N) {
  return M >= 1 && M <= convrot::kSmallM && (N + 127) / 128 <= convrot::kMaxSplitTiles;
}

// ... and whether convrot_linear uses them (the split is compiled out by default:
// it measured slower than whole tiles on every shape tried).
bool linear_uses_split(int64_t M, int64_t N) { return CONVROT_SMALLM_SPLIT != 0 && linear_has_split_buffers(M, N); }

LinearWs linear_ws_layout(int64_t M, int64_t K, int64_t N) {
  LinearWs w;
  w.ready_off = kStatusBytes;
  const size_t mblocks = (static_cast<size_t>(M) + 127) / 128;
  w.scale_off = align_up(w.ready_off + 8 * mblocks, 256);
  w.codes_off = align_up(w.scale_off + 4 * static_cast<size_t>(M), 1024);
  w.total = align_up(w.codes_off + static_cast<size_t>(M) * static_cast<size_t>(K), 256);
  w.split = linear_has_split_buffers(M, N);
  w.split_count_off = w.split_part_off = 0;
  if (w.split) {
    w.split_count_off = w.total;
    w.split_part_off = align_up(w.split_count_off + convrot::split_count_bytes(N), 1024);
    w.total = align_up(w.split_part_off + convrot::split_part_bytes(static_cast<int>(M)), 256);
  }
  return w;
}

// Epoch of a fused call: unique in the process, never 0, so that ready
// counters left in a workspace by earlier calls never look finished.
uint32_t next_epoch() {
  static std::atomic<uint32_t> counter{0x5A17u};
  uint32_t e;
  do {
    e = counter.fetch_add(1u, std::memory_order_relaxed) + 1u;
  } while (e == 0u);
  return e;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

convrot_status from_cuda(cudaError_t e) { return e == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA; }

// Checks shared by every entry point that rotates rows of length K in groups of g.
// rows = 0 passes: the callers return before touching a buffer (an empty batch).
convrot_status check_rotation_shape(int64_t rows, int64_t K, int g) {
  if (rows < 0 || K < 1) return CONVROT_ERR_INVALID_ARG;
  if (g != 128 && g != 256) return CONVROT_ERR_UNSUPPORTED;
  if (K % g != 0) return CONVROT_ERR_INVALID_ARG;
  if (K > CONVROT_MAX_K) return CONVROT_ERR_UNSUPPORTED;
  if (rows > (int64_t(1) << 31) - 1) return CONVROT_ERR_UNSUPPORTED;
  return CONVROT_OK;
}

// Checks of the GEMM shape: TMA needs 16-byte row strides; coordinates are int32.
// M = 0 passes, as above.
convrot_status check_gemm_shape(int64_t M, int64_t N, int64_t K, int n_multiple) {
  if (M < 0 || N < 1 || K < 1) return CONVROT_ERR_INVALID_ARG;
  if (K % 16 != 0 || N % n_multiple != 0) return CONVROT_ERR_INVALID_ARG;
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (M > lim || N > lim || K > lim) return CONVROT_ERR_UNSUPPORTED;
  // the GEMM kernels count output tiles (128 x 128 at the finest) in int
  if (((M + 127) / 128) * ((N + 127) / 128) > lim) return CONVROT_ERR_UNSUPPORTED;
  return CONVROT_OK;
}

// Options of the general dequant epilogue (convrot_linear_ex); the defaults
// are convrot_linear's (bf16, one tensor scale, no activation).
struct EpiOptions {
  int out_f16 = 0;
  int wscale_per_channel = 0;
  int act = 0;
  const void* addend = nullptr;  // [M, ldy] in the output dtype, added before the activation
  int64_t ldx = 0;               // row strides in elements (0 = dense)
  int64_t ldy = 0;
  bool general() const {
    return out_f16 != 0 || wscale_per_channel != 0 || act != 0 || addend != nullptr || ldy != 0;
  }
};

convrot::GemmParams gemm_params(int64_t M, int64_t N, int64_t K, const float* x_scale, const float* w_scale,
                                const void* bias, int* status, const EpiOptions& opt) {
  convrot::GemmParams p{};
  p.out_f16 = opt.out_f16;
  p.wscale_per_channel = opt.wscale_per_channel;
  p.addend = static_cast<const uint16_t*>(opt.addend);
  p.ldy = opt.ldy;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.x_scale = x_scale;
  p.w_scale = w_scale;
  p.bias = static_cast<const uint16_t*>(bias);
  p.status = status;
  p.clock_rec = status == nullptr ? nullptr
                                  : reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(status) +
                                                                          CONVROT_WS_CLOCK_RECORD_OFFSET);
  p.timeout_ns = kWaitTimeoutNs;
  p.group_m = 0;
  return p;
}

convrot_status run_gemm(int epi, const int8_t* Xq, const int8_t* Wq, void* out, int64_t M, int64_t N, int64_t K,
                        const float* x_scale, const float* w_scale, const void* bias, int* status,
                        cudaStream_t stream, EpiOptions opt = EpiOptions(), int32_t* split_part = nullptr,
                        unsigned* split_count = nullptr) {
  convrot::GemmParams p = gemm_params(M, N, K, x_scale, w_scale, bias, status, opt);
  p.split_part = split_part;
  p.split_count = split_count;
  return from_cuda(convrot::launch_gemm_i8(epi, Xq, Wq, out, p, stream));
}


}  // namespace

extern "C" {

int convrot_abi_version(void) { return kAbiVersion; }

const char* convrot_status_string(int status) {
  switch (status) {
    case CONVROT_OK: return "ok";
    case CONVROT_ERR_INVALID_ARG: return "invalid argument (null pointer, size, or alignment)";
    case CONVROT_ERR_UNSUPPORTED: return "unsupported configuration (group size or size limit)";
    case CONVROT_ERR_WORKSPACE: return "workspace null, misaligned or too small";
    case CONVROT_ERR_CUDA: return "CUDA call or kernel launch failed";
    case CONVROT_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
    default: return "unknown status";
  }
}

size_t convrot_prepare_weight_workspace_bytes(void) { return 256; }

convrot_status convrot_prepare_weight_ex(const void* W, int dtype, int64_t N, int64_t K, int g, int wscale_mode,
                                         int8_t* Wq, float* w_scale, void* ws, size_t ws_bytes,
                                         convrot_stream_t stream) {
  if (N < 1) return CONVROT_ERR_INVALID_ARG;  // a weight has at least one output channel
  const convrot_status sh = check_rotation_shape(N, K, g);
  if (sh != CONVROT_OK) return sh;
  if (dtype != CONVROT_DTYPE_BF16 && dtype != CONVROT_DTYPE_F16) return CONVROT_ERR_UNSUPPORTED;
  if (wscale_mode != CONVROT_WSCALE_TENSOR && wscale_mode != CONVROT_WSCALE_CHANNEL) return CONVROT_ERR_UNSUPPORTED;
  if (W == nullptr || Wq == nullptr || w_scale == nullptr) return CONVROT_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(Wq, 16) || !aligned(w_scale, wscale_mode == CONVROT_WSCALE_CHANNEL ? 16 : 4))
    return CONVROT_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  convrot::RotQuantParams p{};
  p.src = static_cast<const uint16_t*>(W);
  p.in_f16 = dtype == CONVROT_DTYPE_F16 ? 1 : 0;
  p.rows = N;
  p.K = K;
  p.dst = Wq;
  p.scale = w_scale;
  p.status_reset = nullptr;
  p.status = nullptr;
  p.timeout_ns = kWaitTimeoutNs;
  if (wscale_mode == CONVROT_WSCALE_CHANNEL) {
    // one scale per weight row: the per-row (activation) form of the kernel,
    // which lets its dependents launch only at exit (they may read the weight early)
    p.tensor_absmax = nullptr;
    p.late_trigger = 1;
    return from_cuda(convrot::launch_rotate_quant(g, convrot::kRqActivation, p, s));
  }
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < convrot_prepare_weight_workspace_bytes())
    return CONVROT_ERR_WORKSPACE;
  unsigned* amax = static_cast<unsigned*>(ws);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return CONVROT_ERR_CUDA;
  p.tensor_absmax = amax;
  e = convrot::launch_rotate_quant(g, convrot::kRqWeightAbsmax, p, s);
  if (e != cudaSuccess) return CONVROT_ERR_CUDA;
  return from_cuda(convrot::launch_rotate_quant(g, convrot::kRqWeightQuant, p, s));
}

convrot_status convrot_prepare_weight(const void* W, int64_t N, int64_t K, int g, int8_t* Wq, float* w_scale,
                                      void* ws, size_t ws_bytes, convrot_stream_t stream) {
  return convrot_prepare_weight_ex(W, CONVROT_DTYPE_BF16, N, K, g, CONVROT_WSCALE_TENSOR, Wq, w_scale, ws, ws_bytes,
                                   stream);
}

convrot_status convrot_quant_act_ex(const void* X, int dtype, int64_t M, int64_t K, int64_t ldx, int g,
                                    int8_t* Xq, float* x_scale, convrot_stream_t stream) {
  const convrot_status sh = check_rotation_shape(M, K, g);
  if (sh != CONVROT_OK) return sh;
  if (dtype != CONVROT_DTYPE_BF16 && dtype != CONVROT_DTYPE_F16) return CONVROT_ERR_UNSUPPORTED;
  if (ldx != 0 && (ldx < K || ldx % 8 != 0)) return CONVROT_ERR_INVALID_ARG;
  if (M == 0) return CONVROT_OK;  // no tokens: nothing to write, nothing launched
  if (X == nullptr || Xq == nullptr || x_scale == nullptr) return CONVROT_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(Xq, 16) || !aligned(x_scale, 4)) return CONVROT_ERR_INVALID_ARG;
  convrot::RotQuantParams p{};
  p.src = static_cast<const uint16_t*>(X);
  p.in_f16 = dtype == CONVROT_DTYPE_F16 ? 1 : 0;
  p.rows = M;
  p.K = K;
  p.ldx = ldx;
  p.dst = Xq;
  p.scale = x_scale;
  p.tensor_absmax = nullptr;
  p.status_reset = nullptr;
  p.status = nullptr;
  p.timeout_ns = kWaitTimeoutNs;
  return from_cuda(
      convrot::launch_rotate_quant(g, convrot::kRqActivation, p, reinterpret_cast<cudaStream_t>(stream)));
}

convrot_status convrot_quant_act(const void* X, int64_t M, int64_t K, int g, int8_t* Xq, float* x_scale,
                                 convrot_stream_t stream) {
  return convrot_quant_act_ex(X, CONVROT_DTYPE_BF16, M, K, 0, g, Xq, x_scale, stream);
}

size_t convrot_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int g) {
  if (check_rotation_shape(M, K, g) != CONVROT_OK || check_gemm_shape(M, N, K, 8) != CONVROT_OK) return 0;
  return linear_ws_layout(M, K, N).total;
}

}  // extern "C"

namespace {

// Whether convrot_linear (and its variants) run the layer as the one fused
// weight-streaming kernel: M * K <= 16384 (at most 16 tokens), bf16 dense rows.
bool linear_is_one_kernel(int64_t M, int64_t K, const EpiOptions& opt) {
  return opt.out_f16 == 0 && opt.ldx == 0 && convrot::smallm_fused_shape(M, K);
}

// The layer: the rotate+quantise kernel followed by the GEMM, or (one_launch)
// the single kernel whose worker warps rotate and quantise while its tensor
// cores multiply the finished M-blocks (K <= 20480, default options only).
// Events (may be null) are recorded before, between and after the launches.
convrot_status linear_impl(const void* X, int64_t M, int64_t K, int g, const int8_t* Wq, const float* w_scale,
                           int64_t N, const void* bias, void* Y, void* ws, size_t ws_bytes, cudaEvent_t ev0,
                           cudaEvent_t ev1, cudaEvent_t ev2, cudaStream_t s, EpiOptions opt = EpiOptions(),
                           bool one_launch = false) {
  convrot_status sh = check_rotation_shape(M, K, g);
  if (sh != CONVROT_OK) return sh;
  sh = check_gemm_shape(M, N, K, 8);
  if (sh != CONVROT_OK) return sh;
  if ((opt.ldx != 0 && (opt.ldx < K || opt.ldx % 8 != 0)) || (opt.ldy != 0 && (opt.ldy < N || opt.ldy % 8 != 0)))
    return CONVROT_ERR_INVALID_ARG;
  int tpr = 0, rpp = 0, cta_threads = 0;
  if (one_launch && (opt.general() || opt.ldx != 0 || !convrot::fused_shape(K, &tpr, &rpp, &cta_threads)))
    return CONVROT_ERR_UNSUPPORTED;
  if (M == 0) {
    // no tokens: Y is empty; nothing is launched and no buffer is touched (the
    // caller's events, if any, are still recorded so that they complete)
    for (cudaEvent_t ev : {ev0, ev1, ev2})
      if (ev != nullptr && cudaEventRecord(ev, s) != cudaSuccess) return CONVROT_ERR_CUDA;
    return CONVROT_OK;
  }
  if (X == nullptr || Wq == nullptr || w_scale == nullptr || Y == nullptr) return CONVROT_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(Wq, 16) || !aligned(w_scale, opt.wscale_per_channel ? 16 : 4) ||
      !aligned(Y, 16) || (bias != nullptr && !aligned(bias, 16)) ||
      (opt.addend != nullptr && !aligned(opt.addend, 16)))
    return CONVROT_ERR_INVALID_ARG;
  const LinearWs lay = linear_ws_layout(M, K, N);
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < lay.total) return CONVROT_ERR_WORKSPACE;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(wsb);
  float* x_scale = reinterpret_cast<float*>(wsb + lay.scale_off);
  int8_t* Xq = reinterpret_cast<int8_t*>(wsb + lay.codes_off);

  if (one_launch) {
    // The call's epoch is drawn here on the host: a CUDA graph would replay
    // the captured value, and from the second replay on the readiness
    // counters would already hold it. So a capturing stream is refused.
    cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &capture) != cudaSuccess) return CONVROT_ERR_CUDA;
    if (capture != cudaStreamCaptureStatusNone) return CONVROT_ERR_UNSUPPORTED;
    // one launch: worker warps rotate + quantise while the GEMM consumes finished M-blocks
    convrot::GemmParams gp{};
    gp.M = static_cast<int>(M);
    gp.N = static_cast<int>(N);
    gp.K = static_cast<int>(K);
    gp.x_scale = x_scale;
    gp.w_scale = w_scale;
    gp.bias = static_cast<const uint16_t*>(bias);
    gp.status = status;
    gp.timeout_ns = kWaitTimeoutNs;
    gp.group_m = 0;
    gp.X = static_cast<const uint16_t*>(X);
    gp.Xq = Xq;
    gp.x_scale_out = x_scale;
    gp.ready = reinterpret_cast<unsigned long long*>(wsb + lay.ready_off);
    gp.epoch = next_epoch();
    // the status word is cleared before the launch, so that no CTA's report of a
    // timed-out wait can come before the clear
    if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return CONVROT_ERR_CUDA;
    if (ev0 != nullptr && cudaEventRecord(ev0, s) != cudaSuccess) return CONVROT_ERR_CUDA;
    const cudaError_t fe = convrot::launch_linear_fused(g, Wq, Y, gp, s);
    if (fe == cudaErrorNotSupported) return CONVROT_ERR_UNSUPPORTED;  // the grid cannot be resident at once
    if (fe != cudaSuccess) return CONVROT_ERR_CUDA;
    if (ev1 != nullptr && cudaEventRecord(ev1, s) != cudaSuccess) return CONVROT_ERR_CUDA;
    if (ev2 != nullptr && cudaEventRecord(ev2, s) != cudaSuccess) return CONVROT_ERR_CUDA;
    return CONVROT_OK;
  }

  const int epi = opt.act ? convrot::kEpiDequantGenGelu
                           : (opt.general() ? convrot::kEpiDequantGen : convrot::kEpiDequantBf16);
  if (linear_is_one_kernel(M, K, opt)) {
    // a few tokens: one kernel rotates and quantises them into shared
    // memory and streams the weight; its CTA 0 also leaves the codes and the
    // token scales in the workspace
    convrot::GemmParams gp = gemm_params(M, N, K, nullptr, w_scale, bias, status, opt);
    gp.X = static_cast<const uint16_t*>(X);
    gp.Xq = Xq;
    gp.x_scale_out = x_scale;
    for (cudaEvent_t ev : {ev0, ev1})
      if (ev != nullptr && cudaEventRecord(ev, s) != cudaSuccess) return CONVROT_ERR_CUDA;
    if (convrot::launch_linear_smallm_fused(epi, g, Wq, Y, gp, s) != cudaSuccess) return CONVROT_ERR_CUDA;
    if (ev2 != nullptr && cudaEventRecord(ev2, s) != cudaSuccess) return CONVROT_ERR_CUDA;
    return CONVROT_OK;
  }

  convrot::RotQuantParams p{};
  p.src = static_cast<const uint16_t*>(X);
  p.in_f16 = opt.out_f16;  // X, bias and Y share the compute dtype
  p.rows = M;
  p.K = K;
  p.ldx = opt.ldx;
  p.dst = Xq;
  p.scale = x_scale;
  p.tensor_absmax = nullptr;
  p.status_reset = status;  // CTA 0 of the first kernel clears the status word of this call
  p.status = status;
  p.timeout_ns = kWaitTimeoutNs;
  int32_t* split_part = nullptr;
  unsigned* split_count = nullptr;
  if (lay.split && linear_uses_split(M, N)) {
    // the weight-streaming GEMM split over all SMs: its arrival counters are
    // zeroed by the first kernel, before the GEMM may start
    split_part = reinterpret_cast<int32_t*>(wsb + lay.split_part_off);
    split_count = reinterpret_cast<unsigned*>(wsb + lay.split_count_off);
    p.zero_words = split_count;
    p.zero_count = static_cast<int>((N + 127) / 128);
  }
  if (ev0 != nullptr && cudaEventRecord(ev0, s) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (convrot::launch_rotate_quant(g, convrot::kRqActivation, p, s) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (ev1 != nullptr && cudaEventRecord(ev1, s) != cudaSuccess) return CONVROT_ERR_CUDA;
  const convrot_status st =
      run_gemm(epi, Xq, Wq, Y, M, N, K, x_scale, w_scale, bias, status, s, opt, split_part, split_count);
  if (st != CONVROT_OK) return st;
  if (ev2 != nullptr && cudaEventRecord(ev2, s) != cudaSuccess) return CONVROT_ERR_CUDA;
  return CONVROT_OK;
}

}  // namespace

extern "C" {

convrot_status convrot_linear(const void* X, int64_t M, int64_t K, int g, const int8_t* Wq, const float* w_scale,
                              int64_t N, const void* bias, void* Y, void* ws, size_t ws_bytes,
                              convrot_stream_t stream) {
  return linear_impl(X, M, K, g, Wq, w_scale, N, bias, Y, ws, ws_bytes, nullptr, nullptr, nullptr,
                     reinterpret_cast<cudaStream_t>(stream));
}

convrot_status convrot_linear_timed(const void* X, int64_t M, int64_t K, int g, const int8_t* Wq,
                                    const float* w_scale, int64_t N, const void* bias, void* Y, void* ws,
                                    size_t ws_bytes, void* ev_start, void* ev_mid, void* ev_end,
                                    convrot_stream_t stream) {
  if (ev_start == nullptr || ev_end == nullptr) return CONVROT_ERR_INVALID_ARG;
  return linear_impl(X, M, K, g, Wq, w_scale, N, bias, Y, ws, ws_bytes, static_cast<cudaEvent_t>(ev_start),
                     static_cast<cudaEvent_t>(ev_mid), static_cast<cudaEvent_t>(ev_end),
                     reinterpret_cast<cudaStream_t>(stream));
}

convrot_status convrot_linear_ex(const void* X, int dtype, int64_t M, int64_t K, int64_t ldx, int g,
                                 const int8_t* Wq, const float* w_scale, int wscale_mode, int64_t N,
                                 const void* bias, const void* addend, int activation, void* Y, int64_t ldy,
                                 void* ws, size_t ws_bytes, convrot_stream_t stream) {
  if (dtype != CONVROT_DTYPE_BF16 && dtype != CONVROT_DTYPE_F16) return CONVROT_ERR_UNSUPPORTED;
  if (wscale_mode != CONVROT_WSCALE_TENSOR && wscale_mode != CONVROT_WSCALE_CHANNEL) return CONVROT_ERR_UNSUPPORTED;
  if (activation != CONVROT_ACT_NONE && activation != CONVROT_ACT_GELU_ERF) return CONVROT_ERR_UNSUPPORTED;
  EpiOptions opt;
  opt.out_f16 = dtype == CONVROT_DTYPE_F16 ? 1 : 0;
  opt.wscale_per_channel = wscale_mode == CONVROT_WSCALE_CHANNEL ? 1 : 0;
  opt.act = activation == CONVROT_ACT_GELU_ERF ? 1 : 0;
  opt.addend = addend;
  opt.ldx = (ldx == K) ? 0 : ldx;
  opt.ldy = (ldy == N) ? 0 : ldy;
  return linear_impl(X, M, K, g, Wq, w_scale, N, bias, Y, ws, ws_bytes, nullptr, nullptr, nullptr,
                     reinterpret_cast<cudaStream_t>(stream), opt);
}

int convrot_linear_launch_count(int64_t M, int64_t N, int64_t K, int g) {
  if (check_rotation_shape(M, K, g) != CONVROT_OK || check_gemm_shape(M, N, K, 8) != CONVROT_OK) return 0;
  return M == 0 ? 0 : linear_is_one_kernel(M, K, EpiOptions()) ? 1 : 2;
}

convrot_status convrot_linear_one_launch(const void* X, int64_t M, int64_t K, int g, const int8_t* Wq,
                                         const float* w_scale, int64_t N, const void* bias, void* Y, void* ws,
                                         size_t ws_bytes, convrot_stream_t stream) {
  return linear_impl(X, M, K, g, Wq, w_scale, N, bias, Y, ws, ws_bytes, nullptr, nullptr, nullptr,
                     reinterpret_cast<cudaStream_t>(stream), EpiOptions(), true);
}

size_t convrot_gemm_workspace_bytes(void) { return kStatusBytes; }

convrot_status convrot_gemm_dequant(const int8_t* Xq, const float* x_scale, const int8_t* Wq, const float* w_scale,
                                    int64_t M, int64_t N, int64_t K, const void* bias, void* Y, void* ws,
                                    size_t ws_bytes, convrot_stream_t stream) {
  const convrot_status sh = check_gemm_shape(M, N, K, 8);
  if (sh != CONVROT_OK) return sh;
  if (M == 0) return CONVROT_OK;  // no tokens: nothing launched
  if (Xq == nullptr || x_scale == nullptr || Wq == nullptr || w_scale == nullptr || Y == nullptr)
    return CONVROT_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || !aligned(x_scale, 4) || !aligned(w_scale, 4) ||
      (bias != nullptr && !aligned(bias, 16)))
    return CONVROT_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < kStatusBytes) return CONVROT_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return CONVROT_ERR_CUDA;
  return run_gemm(convrot::kEpiDequantBf16, Xq, Wq, Y, M, N, K, x_scale, w_scale, bias, status, s);
}

convrot_status convrot_gemm_s32(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K, int32_t* acc,
                                void* ws, size_t ws_bytes, convrot_stream_t stream) {
  const convrot_status sh = check_gemm_shape(M, N, K, 4);
  if (sh != CONVROT_OK) return sh;
  if (M == 0) return CONVROT_OK;  // no tokens: nothing launched
  if (Xq == nullptr || Wq == nullptr || acc == nullptr) return CONVROT_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(acc, 16)) return CONVROT_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < kStatusBytes) return CONVROT_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return CONVROT_ERR_CUDA;
  return run_gemm(convrot::kEpiRawS32, Xq, Wq, acc, M, N, K, nullptr, nullptr, nullptr, status, s);
}

convrot_status convrot_read_device_status(const void* ws, convrot_stream_t stream) {
  if (ws == nullptr || !aligned(ws, 256)) return CONVROT_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int host = 0;
  if (cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (host == 0) return CONVROT_OK;
  return host == CONVROT_ERR_DEVICE_TIMEOUT ? CONVROT_ERR_DEVICE_TIMEOUT : CONVROT_ERR_CUDA;
}

convrot_status convrot_test_wait_timeout(void* ws, size_t ws_bytes, int64_t timeout_ns, convrot_stream_t stream) {
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < kStatusBytes) return CONVROT_ERR_WORKSPACE;
  if (timeout_ns < 1000 || timeout_ns > 1000000000) return CONVROT_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return CONVROT_ERR_CUDA;
  return from_cuda(convrot::launch_wait_timeout(status, static_cast<uint64_t>(timeout_ns), s));
}

}  // extern "C"
