/*
 * convrot.h -- C ABI of libconvrot, the INT8 ConvRot linear layer for NVIDIA B200 (sm_100a).
 *
 * What the layer computes (restated from the pages that describe the method):
 *   - The weight is stored as int8 with one scale for the whole tensor
 *     ("int8_tensorwise"; InvokeAI "int8 Compute" page, opening section).
 *   - Each call rotates its input, quantises it to int8 with one scale per
 *     token, and multiplies int8 by int8 on the tensor cores (same page,
 *     second paragraph).
 *   - The rotation works on groups of input channels, 256 wide in every
 *     published build (same page, "What stays on the default path"); it is a
 *     group-wise rotation slid block by block along the channel axis, so that
 *     an outlier channel is spread over its group ("Explanation of INT8
 *     ConvRot", section "What is INT8 ConvRot?").
 *
 * Readings this library fixes where the pages are silent:
 *   R = blockdiag(H_g/sqrt(g), ...), H_g the Sylvester Walsh-Hadamard matrix
 *   (H[i][j] = (-1)^popcount(i & j)), g in {128, 256}, applied to both X and W
 *   so that X R (W R)^T = X W^T. Symmetric quantisation, codes in [-127, 127],
 *   round to nearest with ties to even. Token scale s_x[m] = absmax_k |(X R)[m,k]| / 127
 *   in float32 (0 for an all-zero token, whose codes are then 0). Output
 *   Y[m,n] = bf16_rne(float(acc[m,n]) * (s_x[m] * s_w) + bias[n]).
 *
 * Conventions for every entry point:
 *   - Matrices are row-major with K contiguous: X [M,K], W/Wq [N,K], Y [M,N].
 *     X, W, bias and Y are bf16 (IEEE bfloat16 bit patterns, 2 bytes each),
 *     except in the *_ex entry points, which also take fp16 and row strides.
 *   - Every data pointer is a DEVICE pointer owned by the caller, 16-byte
 *     aligned (workspaces: 256-byte aligned). The library never allocates,
 *     never frees and never synchronises, except where an entry point says so.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) on the calling thread's current device.
 *   - Arguments are checked on the host before anything is launched; a bad
 *     argument returns an error code and enqueues nothing.
 *   - M = 0 (no tokens: an empty batch, an expert no token was routed to) is
 *     valid wherever M appears. The call checks its other arguments, returns
 *     CONVROT_OK and enqueues nothing; the M-sized pointers may then be NULL
 *     and the workspace is not touched (its status word keeps its value).
 *     convrot_linear_timed still records the caller's events, and
 *     convrot_linear_noalloc writes 0 to its device_status.
 *   - A launch failure returns CONVROT_ERR_CUDA.
 *   - Every wait inside a kernel is bounded (about 2 s). If one runs out, the
 *     kernel records CONVROT_ERR_DEVICE_TIMEOUT in the workspace status word
 *     (where the entry point has one) and returns without faulting;
 *     convrot_read_device_status reports it. convrot_linear's status word is
 *     cleared by the first CTA of its first kernel as it starts, before the
 *     GEMM may launch (in the one-kernel form, by the first CTA once its
 *     predecessor has finished; a memset instead costs 3.7 us per call on the
 *     weight-streaming layers); the clear is not ordered against a timeout
 *     reported by another CTA of that kernel, which could be lost only
 *     if that CTA had waited 2 s before the first CTA started. The other entry
 *     points with a workspace clear it with a 4-byte memset before launching.
 *   - Entry points hold no state between calls (convrot_linear_noalloc's
 *     built-in scratch aside) and are safe to call from several host threads
 *     on different streams with separate workspaces.
 *   - Calls that only enqueue work may be captured into a CUDA graph (stream
 *     capture); each replay recomputes everything from the current contents
 *     of the captured buffers. The exceptions: convrot_linear_one_launch
 *     refuses a capturing stream, convrot_read_device_status synchronises and
 *     so cannot be captured, and convrot_linear_noalloc needs one call on the
 *     device before any capture begins.
 */
#ifndef CONVROT_H
#define CONVROT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CONVROT_API __attribute__((visibility("default")))
#else
#define CONVROT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* convrot_stream_t;

typedef enum {
  CONVROT_OK = 0,
  CONVROT_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer     */
  CONVROT_ERR_UNSUPPORTED = 2,   /* g not in {128,256}, K above the kernel limit    */
  CONVROT_ERR_WORKSPACE = 3,     /* workspace null, misaligned or too small         */
  CONVROT_ERR_CUDA = 4,          /* a CUDA call or kernel launch failed             */
  CONVROT_ERR_DEVICE_TIMEOUT = 5 /* a bounded device-side wait ran out (see above)  */
} convrot_status;

/* Largest K the rotation/quantisation kernels take (one CTA holds a token). */
#define CONVROT_MAX_K 32768

/*
 * Byte offset, inside the workspace of convrot_linear, convrot_linear_timed,
 * convrot_gemm_dequant and convrot_gemm_s32, of a measurement record the
 * tensor-core GEMM for M > 64 writes on every call: four uint64, the SM clock
 * counter (%clock64) and the global timer in ns (%globaltimer) read by one
 * thread of its first CTA when that CTA's first operands have landed, then
 * again after it has issued its last tile's MMAs. (clock difference) / (time
 * difference) is the SM clock the GEMM ran at, in GHz. The weight-streaming
 * GEMM (M <= 64) and the one-launch form leave the record untouched. Not
 * part of any result; no call reads it.
 */
#define CONVROT_WS_CLOCK_RECORD_OFFSET 64

/* Version of this ABI; bumped when a signature or a layout changes. */
CONVROT_API int convrot_abi_version(void);

/* Static English description of a status code. Never NULL. */
CONVROT_API const char* convrot_status_string(int status);

/*
 * convrot_prepare_weight -- rotate and quantise a bf16 weight once per layer.
 *   Wq = clamp(rne((W R) / s_w), -127, 127),  s_w = max |W R| / 127 (float32).
 * The stored weight of a ConvRot layer is int8 with one tensorwise scale,
 * pre-rotated (InvokeAI "int8 Compute", opening section).
 *   W        [N,K] bf16, device.           N >= 1; K % g == 0; K <= CONVROT_MAX_K.
 *   g        group size, 128 or 256.
 *   Wq       [N,K] int8 out, device.
 *   w_scale  1 float out, device.
 *   ws       device workspace of ws_bytes >= convrot_prepare_weight_workspace_bytes();
 *            overwritten; only needed until the enqueued work has run.
 * Enqueues three operations (a 4-byte memset and two kernels) on `stream`.
 */
CONVROT_API size_t convrot_prepare_weight_workspace_bytes(void);
CONVROT_API convrot_status convrot_prepare_weight(const void* W, int64_t N, int64_t K, int g,
                                      int8_t* Wq, float* w_scale,
                                      void* ws, size_t ws_bytes, convrot_stream_t stream);

/*
 * convrot_quant_act -- the fused activation pass: per token, rotate each
 * length-g group (fast Walsh-Hadamard transform in float32, never stored),
 * take the token's absmax, and write int8 codes and the float32 scale
 * (InvokeAI "int8 Compute", second paragraph: rotate, then quantise per token).
 *   X        [M,K] bf16, device.            M >= 0; K % g == 0; K <= CONVROT_MAX_K.
 *   Xq       [M,K] int8 out, device.
 *   x_scale  [M] float out, device.
 * One kernel launch.
 */
CONVROT_API convrot_status convrot_quant_act(const void* X, int64_t M, int64_t K, int g,
                                 int8_t* Xq, float* x_scale, convrot_stream_t stream);

/*
 * convrot_linear -- one ConvRot linear call:
 *   Y = bf16_rne( (Xq Wq^T) * (s_x[m] * s_w) + bias[n] ),  (Xq, s_x) = quant_act(X).
 * The int8 x int8 product accumulates exactly in int32 on the tcgen05 tensor
 * cores (InvokeAI "int8 Compute", second paragraph); dequantisation and the
 * bias are fused into the GEMM epilogue. Two kernels (rotate+quantise, then
 * the GEMM, chained with programmatic dependent launch), or, for a few tokens
 * (M * K <= 16384, M <= 16, K <= 8192; bf16 dense rows), one weight-streaming
 * kernel that rotates and quantises the tokens into shared memory itself
 * (every CTA redundantly; the same arithmetic in the same order, so the same
 * codes, scales and output bits as the two kernels);
 * convrot_linear_launch_count reports the number for a shape. The GEMM
 * kernels read the weight before they wait for the previous kernel on the
 * stream (so that its stream overlaps that kernel's tail): Wq must not be
 * written by a kernel that lets its dependents launch before it finishes
 * (convrot_prepare_weight's kernels do not).
 *   X        [M,K] bf16, device.   M >= 0, N >= 1, K % g == 0, K <= CONVROT_MAX_K,
 *                                   N % 8 == 0.
 *   Wq       [N,K] int8, device (from convrot_prepare_weight with the same g).
 *   w_scale  1 float, device.
 *   bias     [N] bf16, device, or NULL for none.
 *   Y        [M,N] bf16 out, device. Must not overlap any input.
 *   ws       device workspace, 256-byte aligned, ws_bytes >=
 *            convrot_linear_workspace_bytes(M, N, K, g). It holds the status
 *            word, per-128-token readiness counters, the token scales and the
 *            int8 activation codes of this call, and for M <= 64 with
 *            N <= 8192 (the weight-streaming GEMM split over all SMs) one
 *            arrival counter per 128 weight rows and 2 * 160 slots of
 *            128 x (16, 32 or 64) int32 partial sums; calls that may run at the same time need separate
 *            workspaces. Its contents need no initialisation (the readiness
 *            counters carry a per-call tag; the first kernel of a call zeroes
 *            the arrival counters).
 */
CONVROT_API size_t convrot_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int g);
CONVROT_API convrot_status convrot_linear(const void* X, int64_t M, int64_t K, int g,
                              const int8_t* Wq, const float* w_scale, int64_t N,
                              const void* bias, void* Y,
                              void* ws, size_t ws_bytes, convrot_stream_t stream);

/*
 * convrot_linear_one_launch -- the same layer as convrot_linear in ONE kernel
 * launch: worker warps of the GEMM kernel rotate and quantise the tokens
 * block by block and release each 128-token block to the tensor cores through
 * a per-call tagged counter in the workspace, while the tensor cores already
 * multiply the finished blocks (single-SM 128x256 tiles). For callers for whom
 * a launch costs more than the slower schedule: on the DiT QKV layer it
 * measured slower than the two-kernel convrot_linear (137 against 110 us).
 * Same arguments, workspace and errors as convrot_linear, plus
 * CONVROT_ERR_UNSUPPORTED when K > 20480 (the worker warps of one CTA hold a
 * token) or K % 128 != 0, or when the device cannot hold one CTA of the kernel
 * on every SM at once (checked on the host). Not for CUDA graphs: the counters'
 * per-call tag is drawn on the host at each call, so a replayed graph would
 * reuse it. A call on a stream that is capturing returns CONVROT_ERR_UNSUPPORTED
 * and enqueues nothing.
 * The GEMM roles of one CTA wait (bounded) for token blocks that worker warps
 * of OTHER CTAs quantise, so every CTA of the grid (one per SM) must be
 * resident at the same time. On a GPU whose SMs are partly held by other work
 * (another process under MPS, a concurrent kernel), a CTA may not start until
 * others finish, the wait runs out after about 2 s, and the call reports
 * CONVROT_ERR_DEVICE_TIMEOUT through the status word without a fault; the
 * two-kernel convrot_linear has no such dependency.
 */
CONVROT_API convrot_status convrot_linear_one_launch(const void* X, int64_t M, int64_t K, int g,
                                                     const int8_t* Wq, const float* w_scale, int64_t N,
                                                     const void* bias, void* Y, void* ws, size_t ws_bytes,
                                                     convrot_stream_t stream);

/*
 * Variants of the layer: compute dtype, weight-scale granularity, activation.
 *   CONVROT_DTYPE_F16: X, W, bias and Y are IEEE fp16 instead of bf16 (the
 *     pages' kernels run in BF16 and FP16 only: InvokeAI "int8 Compute",
 *     "What stays on the default path").
 *   CONVROT_WSCALE_CHANNEL: one float32 weight scale per output channel (row
 *     of W R), s_w[n] = max_k |(W R)[n,k]| / 127 -- the "Row-wise" scaling of
 *     INT8 ConvRot in the format table of "Explanation of INT8 ConvRot"
 *     (section "Representative Model Formats and INT8 ConvRot").
 *   CONVROT_ACT_GELU_ERF: y -> y * Phi(y) = 0.5 y (1 + erf(y / sqrt(2))) applied
 *     in float32 before the output rounding: the activation between the two
 *     MLP projections of the diffusion transformers the pages measure, fused
 *     into the up projection. The pages themselves describe no activation.
 */
typedef enum { CONVROT_DTYPE_BF16 = 0, CONVROT_DTYPE_F16 = 1 } convrot_dtype;
typedef enum { CONVROT_WSCALE_TENSOR = 0, CONVROT_WSCALE_CHANNEL = 1 } convrot_wscale_mode;
typedef enum { CONVROT_ACT_NONE = 0, CONVROT_ACT_GELU_ERF = 1 } convrot_activation;

/*
 * convrot_prepare_weight_ex -- convrot_prepare_weight with a dtype and a scale mode.
 *   W        [N,K] in `dtype` (bf16 or fp16 bits), device.
 *   wscale_mode  CONVROT_WSCALE_TENSOR: w_scale is 1 float (as convrot_prepare_weight);
 *            CONVROT_WSCALE_CHANNEL: w_scale is [N] floats, 16-byte aligned, and
 *            ws may be NULL (one kernel launch, no workspace).
 * Other arguments and errors as convrot_prepare_weight; an unknown dtype or
 * mode returns CONVROT_ERR_UNSUPPORTED.
 */
CONVROT_API convrot_status convrot_prepare_weight_ex(const void* W, int dtype, int64_t N, int64_t K, int g,
                                                     int wscale_mode, int8_t* Wq, float* w_scale, void* ws,
                                                     size_t ws_bytes, convrot_stream_t stream);

/*
 * convrot_quant_act_ex -- convrot_quant_act with X in `dtype` (bf16 or fp16)
 * and a row stride: row m of X starts ldx elements after row m-1 (ldx >= K,
 * a multiple of 8; 0 means K). Xq and x_scale stay dense.
 */
CONVROT_API convrot_status convrot_quant_act_ex(const void* X, int dtype, int64_t M, int64_t K, int64_t ldx,
                                                int g, int8_t* Xq, float* x_scale, convrot_stream_t stream);

/*
 * convrot_linear_ex -- convrot_linear with the variants above, an addend and row strides:
 *   Y = out_rne( act( (Xq Wq^T) * (s_x[m] * s_w[n or 0]) + bias[n] + addend[m,n] ) ).
 *   dtype        type of X, bias, addend and Y (CONVROT_DTYPE_BF16 or CONVROT_DTYPE_F16).
 *   ldx          row stride of X in elements (>= K, a multiple of 8; 0 = K).
 *   w_scale      1 float (CONVROT_WSCALE_TENSOR) or [N] floats, 16-byte aligned
 *                (CONVROT_WSCALE_CHANNEL), from convrot_prepare_weight_ex.
 *   addend       [M, ldy] in `dtype`, 16-byte aligned, or NULL: a term computed
 *                beside the int8 layer in the compute precision and never
 *                quantised -- how the pages apply a LoRA to an int8 layer
 *                (InvokeAI "int8 Compute", after the list in "What stays on
 *                the default path") -- added in float32 before the activation
 *                and the single output rounding. It may not overlap Y.
 *   activation   CONVROT_ACT_NONE or CONVROT_ACT_GELU_ERF.
 *   ldy          row stride of Y and of addend in elements (>= N, a multiple of 8; 0 = N).
 * Other arguments, the workspace and the errors as convrot_linear. With bf16,
 * dense rows, a tensor scale, no addend and no activation it is exactly
 * convrot_linear.
 */
CONVROT_API convrot_status convrot_linear_ex(const void* X, int dtype, int64_t M, int64_t K, int64_t ldx, int g,
                                             const int8_t* Wq, const float* w_scale, int wscale_mode, int64_t N,
                                             const void* bias, const void* addend, int activation, void* Y,
                                             int64_t ldy, void* ws, size_t ws_bytes, convrot_stream_t stream);

/*
 * convrot_linear_timed -- convrot_linear that also records caller-created CUDA
 * events (cudaEvent_t, passed as void*) on `stream`: ev_start before its first
 * launch, ev_mid after the rotate+quantise kernel (may be NULL), ev_end
 * after the GEMM. The layer's and each kernel's device time can then be read with
 * cudaEventElapsedTime on the launching stream. ev_mid keeps the GEMM from
 * overlapping the first kernel's tail. In the one-kernel form ev_mid is
 * recorded right after ev_start (the rotate+quantise share reads 0).
 */
CONVROT_API convrot_status convrot_linear_timed(const void* X, int64_t M, int64_t K, int g,
                                                const int8_t* Wq, const float* w_scale, int64_t N,
                                                const void* bias, void* Y,
                                                void* ws, size_t ws_bytes,
                                                void* ev_start, void* ev_mid, void* ev_end,
                                                convrot_stream_t stream);

/* Kernel launches one convrot_linear call of this shape enqueues: 2, 1 (the one-kernel form for a few
 * tokens, see convrot_linear), or 0 for M = 0 or an invalid shape. */
CONVROT_API int convrot_linear_launch_count(int64_t M, int64_t N, int64_t K, int g);

/*
 * convrot_gemm_dequant -- the GEMM + epilogue half of convrot_linear, on codes
 * that are already quantised:  Y = bf16_rne(float(Xq Wq^T) * (x_scale[m] * s_w) + bias[n]).
 *   Xq [M,K] int8, x_scale [M] float, Wq [N,K] int8, w_scale 1 float, bias [N]
 *   bf16 or NULL, Y [M,N] bf16 out -- all device. K % 16 == 0, N % 8 == 0.
 *   ws: at least convrot_gemm_workspace_bytes() bytes (the status word).
 */
CONVROT_API size_t convrot_gemm_workspace_bytes(void);
CONVROT_API convrot_status convrot_gemm_dequant(const int8_t* Xq, const float* x_scale,
                                    const int8_t* Wq, const float* w_scale,
                                    int64_t M, int64_t N, int64_t K,
                                    const void* bias, void* Y,
                                    void* ws, size_t ws_bytes, convrot_stream_t stream);

/*
 * convrot_gemm_s32 -- the raw int32 accumulators acc = Xq Wq^T of the same
 * tcgen05 GEMM (for exactness tests): acc [M,N] int32 out, device.
 *   K % 16 == 0, N % 4 == 0. ws as for convrot_gemm_dequant.
 */
CONVROT_API convrot_status convrot_gemm_s32(const int8_t* Xq, const int8_t* Wq,
                                int64_t M, int64_t N, int64_t K, int32_t* acc,
                                void* ws, size_t ws_bytes, convrot_stream_t stream);

/*
 * convrot_linear_noalloc -- convrot_linear without a caller-provided workspace,
 * for callers that cannot allocate device memory: a plugin inside a host
 * application that owns the device-memory budget and passes only input and
 * output buffers, or a latency-critical loop where cudaMalloc/cudaFree could
 * synchronise the device or fail. The pages describe no such entry point;
 * it has no counterpart there.
 *   Arguments as convrot_linear, minus the workspace. The scratch (status
 *   word, token scales, int8 codes) is one built-in device array of
 *   CONVROT_NOALLOC_SCRATCH_BYTES that every GPU loading this library holds
 *   until the process exits. A call needing more
 *   (convrot_linear_workspace_bytes(M, N, K, g) > CONVROT_NOALLOC_SCRATCH_BYTES,
 *   roughly M*K > 64 MiB) returns CONVROT_ERR_WORKSPACE and enqueues nothing.
 *   device_status: NULL, or a device int that receives the call's status word
 *   (0, or CONVROT_ERR_DEVICE_TIMEOUT) once the call has run on `stream`.
 * Allocates nothing. The first call in each CUDA context looks up the array's
 * device address (cudaGetSymbolAddress, with that device current) and keeps it
 * with the context's id; make that first call before any stream capture
 * begins. cudaDeviceReset between calls is supported: the next call is the
 * first one in the new context and looks the address up again (before any
 * capture, as above). All calls share the array:
 * calls that may overlap on the GPU (unordered streams, several host threads)
 * race on it and must not be issued. Each call clears the status word and
 * rewrites the codes and scales, so no result depends on an earlier call.
 */
#define CONVROT_NOALLOC_SCRATCH_BYTES (64u << 20)
CONVROT_API convrot_status convrot_linear_noalloc(const void* X, int64_t M, int64_t K, int g,
                                                  const int8_t* Wq, const float* w_scale, int64_t N,
                                                  const void* bias, void* Y, int* device_status,
                                                  convrot_stream_t stream);

/*
 * convrot_read_device_status -- copy the status word of a workspace used by
 * convrot_linear / convrot_gemm_* back to the host and return it
 * (CONVROT_OK, or CONVROT_ERR_DEVICE_TIMEOUT if a bounded wait ran out).
 * SYNCHRONISES `stream`. The word is reset at the start of every call that
 * uses the workspace (except a call with M = 0, which enqueues nothing).
 */
CONVROT_API convrot_status convrot_read_device_status(const void* ws, convrot_stream_t stream);

/*
 * convrot_attention_int8 -- INT8 attention, O = softmax(S) V per (batch*head):
 *   S[i, j] = (Qq[i] . Kq[j]) * s_q[i] * s_k[j] * softmax_scale, where Qq/Kq are
 *   the per-token int8 codes of the head vectors of Q and K after the
 *   normalised Walsh-Hadamard rotation along the head dimension (the same
 *   rotate + quantise as convrot_quant_act with g = D), the integer dot products
 *   exact; softmax over the keys in float32; P rounded to bf16 and P V
 *   accumulated in float32; O rounded to bf16.
 *   The Hugging Face discussion "INT8 ConvRot on 2xT4" (section "Attention
 *   kernel alone") measures INT8 attention at 4096 + 128 tokens, 32 heads,
 *   head dimension 128 against FP32 attention; the pages do not give the
 *   quantisation scheme, which this entry point fixes as above.
 *   Q [BH, Sq, D], K and V [BH, Skv, D], O [BH, Sq, D]: bf16, row-major (D
 *   contiguous), device pointers, 16-byte aligned; BH = batch * heads
 *   (<= 65535). D must be 128 (else CONVROT_ERR_UNSUPPORTED). Skv >= 1;
 *   Sq = 0 or BH = 0 enqueues nothing. softmax_scale > 0 and finite (usually
 *   1/sqrt(D)). ws: >= convrot_attention_workspace_bytes(BH, Sq, Skv, D),
 *   256-byte aligned; its first word is the status word
 *   (convrot_read_device_status). Launches a 4-byte memset and three kernels
 *   (rotate+quantise of Q and of K, the attention kernel, which reads V as
 *   given).
 */
CONVROT_API size_t convrot_attention_workspace_bytes(int64_t BH, int64_t Sq, int64_t Skv, int64_t D);
CONVROT_API convrot_status convrot_attention_int8(const void* Q, const void* K, const void* V, int64_t BH,
                                                  int64_t Sq, int64_t Skv, int64_t D, float softmax_scale,
                                                  void* O, void* ws, size_t ws_bytes, convrot_stream_t stream);

/*
 * convrot_probe_i8_peak -- measurement aid for the GEMM's roofline (not part
 * of the layer): launches one CTA pair per two SMs, each issuing `iters`
 * times four tcgen05.mma.cta_group::2.kind::i8 instructions (M = 256, N = 256,
 * K = 32: the instruction the layer's GEMM uses) on shared-memory operands,
 * with no global memory traffic in the loop. The caller times the launch with
 * events on `stream`; the work is 2 * 256 * 256 * 128 * iters operations per
 * pair, convrot_probe_i8_peak_ctas() / 2 pairs. iters in [1, 2^20].
 * operands: null (zero operands) or a device buffer of operand_bytes bytes
 * (16-byte aligned, a positive multiple of 16) from which every CTA copies its
 * 32 KB of A and B tiles once, before the loop (wrapping around the buffer).
 * The rate at a fixed clock does not depend on the values, but the power
 * drawn does: the layer's own codes give the clock the GPU holds under its
 * power limit while the GEMM runs. `ws` (>= 256 bytes, 256-byte aligned)
 * receives the status word (CONVROT_ERR_DEVICE_TIMEOUT if the final wait ran
 * out) and, at CONVROT_WS_CLOCK_RECORD_OFFSET, the same clock record as the
 * GEMM's (one CTA: before its first MMA and after its last has completed).
 */
CONVROT_API convrot_status convrot_probe_i8_peak(int64_t iters, const void* operands, size_t operand_bytes,
                                                 void* ws, size_t ws_bytes, convrot_stream_t stream);
/* CTAs that convrot_probe_i8_peak launches on the current device (0 on error). */
CONVROT_API int convrot_probe_i8_peak_ctas(void);

/*
 * convrot_probe_ex2_peak -- measurement aid for the attention softmax's
 * roofline (not part of the layer): a full grid in which every thread runs
 * independent chains of the special-function unit's exp2 (ex2.approx), iters
 * steps each, convrot_probe_ex2_per_iter() exp2 per step over the grid. The
 * caller times it with events on `stream`. iters in [1, 2^24]; ws >= 1 KB,
 * 256-byte aligned (never written in practice).
 */
CONVROT_API convrot_status convrot_probe_ex2_peak(int64_t iters, void* ws, size_t ws_bytes, convrot_stream_t stream);
CONVROT_API int64_t convrot_probe_ex2_per_iter(void);

/*
 * convrot_test_wait_timeout -- exercises the bounded device wait: launches one
 * CTA that waits on a barrier nothing will complete, for at most timeout_ns
 * nanoseconds (1e3 .. 1e9), then records CONVROT_ERR_DEVICE_TIMEOUT in the
 * status word of `ws` (>= convrot_gemm_workspace_bytes()) and returns. For tests.
 */
CONVROT_API convrot_status convrot_test_wait_timeout(void* ws, size_t ws_bytes, int64_t timeout_ns,
                                         convrot_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H */
