// Launch interface of the tcgen05 int8 GEMM (+ epilogue).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace convrot {

enum GemmEpilogue : int {
  kEpiDequantBf16 = 0,  // Y = bf16_rne(float(acc) * (x_scale[m] * w_scale) + bias[n])
  kEpiRawS32 = 1,       // acc as int32
  // Y = out_rne(float(acc) * (x_scale[m] * w_scale[n or 0]) + bias[n]) with the
  // run-time options below (per-channel weight scale, fp16 output and bias)
  kEpiDequantGen = 2,
  kEpiDequantGenGelu = 3,  // the same followed by GELU (exact erf)
};

// true for the epilogues that write a 2-byte dequantised output
__host__ __device__ constexpr bool epi_is_dequant(int epi) { return epi != kEpiRawS32; }
__host__ __device__ constexpr bool epi_is_general(int epi) { return epi == kEpiDequantGen || epi == kEpiDequantGenGelu; }

struct GemmParams {
  int M, N, K;
  const float* x_scale;   // [M]   (dequant epilogue)
  const float* w_scale;   // [1]   (dequant epilogue)
  const uint16_t* bias;   // [N] bf16 (fp16 with out_f16) bits or null
  int wscale_per_channel; // kEpiDequantGen(Gelu): w_scale holds N floats (one per output channel)
  int out_f16;            // kEpiDequantGen(Gelu): Y and bias are IEEE fp16 instead of bf16
  const uint16_t* addend; // kEpiDequantGen(Gelu): [M, ldy] term added before the activation, or null
  int64_t ldy;            // row stride of Y (and addend) in elements (>= N); 0 = N
  int* status;            // status word: a timed-out wait ORs 5 into it
  uint64_t timeout_ns;    // bound of every device-side wait
  int group_m;            // M-blocks per raster group (0 = default)
  int num_m_blocks, num_n_blocks, num_k_blocks;  // filled by the launcher
  // fused form (launch_linear_fused): the kernel also rotates and quantises X
  const uint16_t* X;              // [M,K] bf16 bits
  int8_t* Xq;                     // [M,K] codes (the A operand)
  float* x_scale_out;             // [M] token scales (same buffer as x_scale)
  unsigned long long* ready;      // [num_m_blocks] epoch << 32 | rows quantised
  uint32_t epoch;                 // unique per call, never 0
  int q_threads_per_row, q_rows_per_pass;  // filled by the launcher
  // weight-streaming form split over all SMs (launch_gemm_i8 with M <= kSmallM):
  // null = one CTA per 128 weight rows; else the (weight tile, k-block) units
  // are divided evenly over the CTAs, and partial tiles meet in these buffers
  int32_t* split_part;            // [2 * kMaxSplitCtas][BNT][128] int32 partial accumulators
  unsigned* split_count;          // [weight tiles] arrival counters, zero when the kernel starts
  // pair form: CTA 0's MMA issuer writes {%clock64, %globaltimer} when its first
  // tile's first operands have landed and again after its last tile's MMAs are
  // issued (the SM clock the kernel ran at), or null
  unsigned long long* clock_rec;
  // weight-streaming form: weight rows per CTA tile (a multiple of 8, at most
  // 128; filled by the launcher)
  int tile_rows;
};

constexpr int kMaxFusedRows = 64;  // rows one CTA rotates and quantises per pass (fused form)
constexpr int kSmallM = 64;  // up to this many tokens the GEMM runs in the weight-streaming (swap-AB) form
constexpr int kMaxSplitCtas = 160;    // CTAs of the split weight-streaming form (at most)
// The split pays a partial-tile epilogue (a store, a fence, a counter and the
// last CTA's sum) at the end of most CTAs' ranges: on the 96-tile text-encoder
// layer it measured slower than whole tiles on 96 SMs, so it is used only where
// whole tiles would leave most SMs idle.
constexpr int kMaxSplitTiles = 64;  // weight tiles (128 rows each) up to which the split form is used (N <= 8192)

// Token columns of the weight-streaming form's MMA for M tokens (16, 32 or 64).
__host__ __device__ constexpr int smallm_bnt(int M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

// Bytes of the split form's partial buffers and counters for M tokens and N outputs.
__host__ __device__ constexpr size_t split_part_bytes(int M) {
  return static_cast<size_t>(2 * kMaxSplitCtas) * smallm_bnt(M) * 128 * 4;
}
__host__ __device__ constexpr size_t split_count_bytes(int64_t N) { return static_cast<size_t>((N + 127) / 128) * 4; }

// Worker layout of the fused kernel for a given K; false if K is not a
// multiple of 128 or too large for one CTA's worker warps (then the layer runs
// as two kernels).
bool fused_shape(int64_t K, int* threads_per_row, int* rows_per_pass, int* cta_threads);

// A = Xq [M,K] int8, B = Wq [N,K] int8, out = Y [M,N] bf16 or acc [M,N] int32.
cudaError_t launch_gemm_i8(int epi, const int8_t* A, const int8_t* B, void* out, GemmParams p,
                           cudaStream_t stream);

// The whole ConvRot linear layer in one launch: p.X is rotated and quantised
// into p.Xq / p.x_scale_out by worker warps while the GEMM consumes finished
// M-blocks. p.ready holds num_m_blocks counters; p.epoch must differ from
// every earlier call's epoch on the same workspace.
cudaError_t launch_linear_fused(int g, const int8_t* Wq, void* Y, GemmParams p, cudaStream_t stream);

// The fused weight-streaming form: whether it takes M tokens of K channels
// (M <= 16, K <= 8192, M * K <= 16384: one quantisation pass), and its launch (Y = dequant(quant(X) Wq^T) in one
// kernel; p.X holds the bf16 tokens, p.x_scale is not used; epi is one of the
// dequantising epilogues).
bool smallm_fused_shape(int64_t M, int64_t K);
cudaError_t launch_linear_smallm_fused(int epi, int g, const int8_t* Wq, void* Y, GemmParams p,
                                       cudaStream_t stream);

// One CTA waits on a barrier that nothing completes, for at most timeout_ns,
// then ORs 5 into *status.
cudaError_t launch_wait_timeout(int* status, uint64_t timeout_ns, cudaStream_t stream);

}  // namespace convrot
