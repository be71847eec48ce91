// INT8 attention on the 5th-generation tensor cores: O = softmax(S) V with
// S = (Qq Kq^T) s_q s_k softmax_scale, where Qq and Kq are the per-token int8
// codes of the head vectors of Q and K after the normalised Walsh-Hadamard
// rotation along the head dimension (the linear layer's rotate+quantise,
// g = 128 = D).
//
// The Hugging Face discussion "INT8 ConvRot on 2xT4" (section "Attention
// kernel alone") measures an INT8 attention call of this shape (4096 + 128
// tokens, 32 heads, head dimension 128) against FP32 attention; the pages do
// not give its quantisation scheme, so the per-token int8 rule of the linear
// layer is applied to Q and K, and P V runs in bf16 with float32 accumulation.
//
// One call: Q and K through the rotate+quantise kernel (codes + one scale per
// token), V transposed once into key-contiguous rows (the K-major B operand of
// the P V product), then one CTA per SM at a time, each on one
// (batch*head, 128-query tile):
//   warp 0, one lane : TMA producer: the tile's 128 x 128 query codes once,
//                      then per 128-key block j the key codes into stage j%2
//                      (once S of block j-2 is computed) and the transposed
//                      values, two 64-key halves, into stage j%2 (once P V of
//                      block j-2 is done).
//   warp 1           : allocates 512 TMEM columns; one lane issues
//                      S_j = Qq Kq_j^T (tcgen05.mma kind::i8, M = N = 128,
//                      K = 4 x 32) into S buffer j%2 (TMEM columns 0..127 or
//                      128..255) and O += P_j V_j (kind::f16 with bf16
//                      operands, M = N = 128, K = 8 x 16) into columns
//                      256..383, in the order S_0, S_1, PV_0, S_2, PV_1, ...
//   warps 2..17      : softmax, four warps per query row (TMEM lane), each
//                      taking 32 keys of every block and 32 O columns. One pass per
//                      block straight from TMEM: t = c_i s_k[j] S_ij in base-2
//                      units (c_i = s_q[i] softmax_scale log2(e)),
//                      p = 2^(t - m) against the current reference maximum m
//                      (packed f32x2 arithmetic), P rounded to bf16 into the
//                      128-byte-swizzled P buffer j%2, the row sums in
//                      float32; the block maximum of the row is combined
//                      across the four warps through shared memory. When a block
//                      raises the maximum by more than 8 (p would pass 256)
//                      the reference moves, the block's pass is redone (S is
//                      still in TMEM) and O is rescaled in TMEM once the
//                      previous block's P V is done. The four warps of a row
//                      meet at a named barrier every block, also after a
//                      timed-out wait (they then skip the work), so none can
//                      be left waiting for another. At the end
//                      O / (sum of the four parts) is rounded to bf16 and stored.
// Every buffer is double: the next block's QK^T and loads run while this
// block's softmax runs on the CUDA cores and the previous block's P V on the
// tensor cores. Every mbarrier is waited on phase by phase in order, and every
// wait is bounded (status word + abort flag, as in the GEMM).

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cstdint>

#include "convrot.h"
#include "fwht_dev.cuh"
#include "ptx_sm100.cuh"
#include "rotate_quant.cuh"

namespace convrot {

namespace {

constexpr int AT_BQ = 128;  // queries per CTA tile
constexpr int AT_BK = 128;  // keys per block
constexpr int AT_D = 128;   // head dimension
constexpr int AT_SOFTMAX_WARPS = 16;  // four per TMEM lane quarter: 32 keys (and 32 O columns) each
constexpr int AT_SUB = 32;            // keys of a block (and O columns) per softmax warp
constexpr int AT_THREADS = 64 + 32 * AT_SOFTMAX_WARPS;
constexpr int kQBytes = AT_BQ * AT_D;      // int8 query codes: 16 KB
constexpr int kKBytes = AT_BK * AT_D;      // int8 key codes of one block: 16 KB
constexpr int kHalf = 128 * 128;           // one 64-key half of a bf16 operand: 128 rows x 128 B
constexpr int kVBytes = 2 * kHalf;         // transposed values of one block: 32 KB
constexpr int kPBytes = 2 * kHalf;         // probabilities of one block (bf16): 32 KB
constexpr uint32_t IDESC_S = idesc_i8(AT_BQ, AT_BK);
constexpr uint32_t IDESC_O = idesc_bf16(AT_BQ, AT_D);
constexpr int kTimeoutStatus = 5;
constexpr float kRescaleThreshold = 8.0f;  // base-2 units: probabilities stay below 2^8

struct AttnSmem {
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;       // two stages
  static constexpr int kOffV = kOffK + 2 * kKBytes;   // two stages
  static constexpr int kOffP = kOffV + 2 * kVBytes;   // two buffers
  static constexpr int kOffSk = kOffP + 2 * kPBytes;  // per softmax warp, two buffers of its 32 key scales
  static constexpr int kOffMx = kOffSk + AT_SOFTMAX_WARPS * 2 * AT_SUB * 4;  // [2 blocks][4 parts][128 rows] maxima
  static constexpr int kOffLs = kOffMx + 2 * 4 * AT_BQ * 4;                  // [4 parts][128 rows] row sums
  static constexpr int kOffBar = kOffLs + 4 * AT_BQ * 4;
  // q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], s_empty[2], p_full, o_done, drain
  static constexpr int kNumBars = 16;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 8;
  static constexpr int kBytes = kOffAbort + 8;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
};

struct AttnParams {
  int BH, Sq, Skv, J;  // J = number of 128-key blocks
  const float* sq;     // [BH * Sq] query scales
  const float* sk;     // [BH * Skv] key scales
  uint16_t* O;         // [BH, Sq, 128] bf16
  float c_scale;       // softmax_scale * log2(e)
  int* status;
  uint64_t timeout_ns;
};

__device__ __forceinline__ void attn_abort(volatile int* abort, int* status) {
  *abort = 1;
  atomicOr(status, kTimeoutStatus);
}

// A bounded wait whose outcome the whole warp shares: the softmax warps follow
// each wait with warp-collective instructions (tcgen05.ld, __any_sync), which
// every lane must reach together, also when the wait has run out.
__device__ __forceinline__ bool warp_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                  uint64_t timeout_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, abort, timeout_ns);
  return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// float(acc) for |acc| < 2^22 without a conversion instruction: the integer
// added to the bits of 1.5 * 2^23 is exact, and subtracting 1.5 * 2^23 leaves it.
__device__ __forceinline__ float small_int_to_float(uint32_t acc) {
  return __uint_as_float(acc + 0x4B400000u) - 12582912.0f;
}

// One pass over this thread's 32 logits of a block, straight from TMEM (both
// 16-column loads in flight together): t = c * s_k[key] * S[row, key] (base-2
// units); with WRITE_P the probabilities p = 2^(t - m_ref) are rounded to bf16
// into the four 16-byte pieces `piece0`.. of the row's 128-byte-swizzled
// shared-memory line and their float32 sum returned. The maximum over the
// valid keys of s_k[key] * S[row, key] goes to *mh.
template <bool WRITE_P, bool MASKED>
__device__ __forceinline__ float softmax_pass(uint32_t t_s, const float* skb, float c, float m_ref, int nvalid,
                                              uint8_t* row, int piece0, int sw, float* mh) {
  const float2 mg = make_float2(-12582912.0f, -12582912.0f);
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m_ref, -m_ref);
  float2 sum2 = make_float2(0.0f, 0.0f);
  float ma = -INFINITY, mc = -INFINITY;
  uint32_t a[2][16];
  tmem_ld_32x32b_x16(t_s, a[0]);
  tmem_ld_32x32b_x16(t_s + 16, a[1]);
  tmem_ld_wait_regs16(a[0]);
  tmem_ld_wait_regs16(a[1]);
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = ch * 16 + 2 * i;  // key (within this warp's 32) of the pair's first element
      // float(acc) for |acc| < 2^22: the integer added to the bits of 1.5 * 2^23, minus 1.5 * 2^23
      const float2 x =
          make_float2(__uint_as_float(a[ch][2 * i] + 0x4B400000u), __uint_as_float(a[ch][2 * i + 1] + 0x4B400000u));
      const float2 u = __fmul2_rn(__fadd2_rn(x, mg), *reinterpret_cast<const float2*>(skb + k));
      if (MASKED) {
        ma = (k < nvalid) ? fmaxf(ma, u.x) : ma;
        mc = (k + 1 < nvalid) ? fmaxf(mc, u.y) : mc;
      } else if (i & 1) {
        mc = fwht::fmax3f(mc, u.x, u.y);
      } else {
        ma = fwht::fmax3f(ma, u.x, u.y);
      }
      if (WRITE_P) {
        const float2 t = __ffma2_rn(c2, u, nm2);
        float2 pp = make_float2(ex2_approx(t.x), ex2_approx(t.y));
        if (MASKED) {
          pp.x = (k < nvalid) ? pp.x : 0.0f;
          pp.y = (k + 1 < nvalid) ? pp.y : 0.0f;
        }
        sum2 = __fadd2_rn(sum2, pp);
        w[i] = pack_bf16x2(pp.x, pp.y);
      }
    }
    if (WRITE_P) {  // keys 16 ch .. 16 ch + 15 of this warp: pieces piece0 + 2 ch, piece0 + 2 ch + 1
      *reinterpret_cast<uint4*>(row + (((piece0 + 2 * ch) ^ sw) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(row + (((piece0 + 2 * ch + 1) ^ sw) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
  *mh = fmaxf(ma, mc);
  return sum2.x + sum2.y;
}

template <bool WRITE_P>
__device__ __forceinline__ float softmax_pass_any(uint32_t t_s, const float* skb, float c, float m_ref, int nvalid,
                                                  uint8_t* row, int piece0, int sw, float* mh) {
  return nvalid == AT_SUB ? softmax_pass<WRITE_P, false>(t_s, skb, c, m_ref, nvalid, row, piece0, sw, mh)
                          : softmax_pass<WRITE_P, true>(t_s, skb, c, m_ref, nvalid, row, piece0, sw, mh);
}

// The four softmax warps of one TMEM lane quarter (128 threads) meet here. The
// non-aligned form: a warp need not arrive converged.
__device__ __forceinline__ void quarter_bar(int id) {
  asm volatile("barrier.sync %0, 128;" ::"r"(id) : "memory");
}

__global__ void __launch_bounds__(AT_THREADS, 1)
    attention_i8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = AttnSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* k_empty = bars + 3;   // [2]
  uint64_t* v_full = bars + 5;    // [2]
  uint64_t* v_empty = bars + 7;   // [2]
  uint64_t* s_full = bars + 9;    // [2]
  uint64_t* s_empty = bars + 11;  // [2]
  uint64_t* p_full = bars + 13;
  uint64_t* o_done = bars + 14;
  uint64_t* drain = bars + 15;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + L::kOffTmemPtr);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * AT_BQ;
  const int J = p.J;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    mbar_init(q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&k_full[b], 1);
      mbar_init(&k_empty[b], 1);
      mbar_init(&v_full[b], 1);
      mbar_init(&v_empty[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], AT_SOFTMAX_WARPS);  // every softmax warp
    }
    mbar_init(p_full, AT_SOFTMAX_WARPS);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_ptr, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;
  const uint32_t tO = tmem_base + 256;  // O: columns 256..383; S buffer b: columns 128 b ..

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int issued_k = 0, issued_v = 0;
      auto load_k = [&](int j) {
        const int b = j & 1;
        mbar_arrive_expect_tx(&k_full[b], kKBytes);
        tma_load_3d(smem + L::kOffK + b * kKBytes, &tmK, &k_full[b], 0, j * AT_BK, bh);
        issued_k = j + 1;
      };
      auto load_v = [&](int j) {
        const int b = j & 1;
        uint8_t* dst = smem + L::kOffV + b * kVBytes;
        mbar_arrive_expect_tx(&v_full[b], kVBytes);
        tma_load_3d(dst, &tmV, &v_full[b], j * AT_BK, 0, bh);
        tma_load_3d(dst + kHalf, &tmV, &v_full[b], j * AT_BK + 64, 0, bh);
        issued_v = j + 1;
      };
      mbar_arrive_expect_tx(q_full, kQBytes);
      tma_load_3d(smem + L::kOffQ, &tmQ, q_full, 0, q0, bh);
      load_k(0);
      load_v(0);
      if (J > 1) {
        load_k(1);
        load_v(1);
      }
      for (int j = 0; j + 2 < J; ++j) {
        // stage j%2 again once block j is done with it (the (j/2)-th use of the stage)
        const uint32_t par = static_cast<uint32_t>((j >> 1) & 1);
        if (!mbar_wait_bounded(&k_empty[j & 1], par, abort, p.timeout_ns)) {
          ok = false;
          break;
        }
        load_k(j + 2);
        if (!mbar_wait_bounded(&v_empty[j & 1], par, abort, p.timeout_ns)) {
          ok = false;
          break;
        }
        load_v(j + 2);
      }
      if (!ok) {
        attn_abort(abort, p.status);
        // every copy already issued lands before the shared memory goes away
        mbar_wait_bounded(q_full, 0u, nullptr, p.timeout_ns);
        for (int j = (issued_k > 2 ? issued_k - 2 : 0); j < issued_k; ++j)
          mbar_wait_bounded(&k_full[j & 1], static_cast<uint32_t>((j >> 1) & 1), nullptr, p.timeout_ns);
        for (int j = (issued_v > 2 ? issued_v - 2 : 0); j < issued_v; ++j)
          mbar_wait_bounded(&v_full[j & 1], static_cast<uint32_t>((j >> 1) & 1), nullptr, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t qa = smem_addr(smem + L::kOffQ);
      auto mma_s = [&](int j) -> bool {
        const int b = j & 1;
        const uint32_t par = static_cast<uint32_t>((j >> 1) & 1);
        // S buffer b free (the softmax of block j-2 has read it) and K_j landed
        if (j >= 2 && !mbar_wait_bounded(&s_empty[b], par ^ 1u, abort, p.timeout_ns)) return false;
        if (!mbar_wait_bounded(&k_full[b], par, abort, p.timeout_ns)) return false;
        tc_fence_after();
        const uint32_t kb = smem_addr(smem + L::kOffK + b * kKBytes);
        const uint32_t ts = tmem_base + static_cast<uint32_t>(b * 128);
#pragma unroll
        for (int k = 0; k < AT_D / 32; ++k)
          mma_i8(ts, smem_desc_k_sw128(qa + k * 32), smem_desc_k_sw128(kb + k * 32), IDESC_S, k > 0 ? 1u : 0u);
        mma_commit(&s_full[b]);
        mma_commit(&k_empty[b]);
        return true;
      };
      bool ok = mbar_wait_bounded(q_full, 0u, abort, p.timeout_ns);
      if (ok) ok = mma_s(0);
      if (ok && J > 1) ok = mma_s(1);
      for (int j = 0; j < J && ok; ++j) {
        const int b = j & 1;
        if (!mbar_wait_bounded(p_full, static_cast<uint32_t>(j & 1), abort, p.timeout_ns) ||
            !mbar_wait_bounded(&v_full[b], static_cast<uint32_t>((j >> 1) & 1), abort, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t pa = smem_addr(smem + L::kOffP + b * kPBytes);
        const uint32_t va = smem_addr(smem + L::kOffV + b * kVBytes);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16(tO, smem_desc_k_sw128(pa + h * kHalf + k * 32), smem_desc_k_sw128(va + h * kHalf + k * 32),
                     IDESC_O, (j | h | k) != 0 ? 1u : 0u);
        mma_commit(o_done);
        mma_commit(&v_empty[b]);
        if (j + 2 < J && !mma_s(j + 2)) {
          ok = false;
          break;
        }
      }
      if (!ok) attn_abort(abort, p.status);
      // every MMA this thread issued has finished before TMEM is released
      mma_commit(drain);
      mbar_wait_bounded(drain, 0u, nullptr, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int sub = (warp - 2) >> 2;  // which 32 keys of a block (and O columns) this warp takes
    const int qd = warp & 3;          // TMEM lane quarter this warp may access
    const int r = qd * 32 + lane;
    const int qrow = q0 + r;
    const int bar_id = 1 + qd;  // the four warps of this lane quarter
    const float sqv = (qrow < p.Sq) ? __ldg(p.sq + static_cast<int64_t>(bh) * p.Sq + qrow) : 0.0f;
    const float c = sqv * p.c_scale;  // >= 0
    const uint32_t t_row = (static_cast<uint32_t>(qd * 32) << 16) + static_cast<uint32_t>(sub * AT_SUB);
    const int sw = r & 7;
    const int piece0 = (sub & 1) * 4;  // this warp's 32 keys: four 16-byte pieces of a P half's row
    const float* skh = p.sk + static_cast<int64_t>(bh) * p.Skv + sub * AT_SUB;
    float* skw = reinterpret_cast<float*>(smem + L::kOffSk) + (warp - 2) * 2 * AT_SUB;
    float* mxb = reinterpret_cast<float*>(smem + L::kOffMx);
    float* lsb = reinterpret_cast<float*>(smem + L::kOffLs);
    float m_ref = 0.0f;
    float l = 0.0f;
    bool ok = true;
    // lane loads the scale of key `lane` of this warp's 32, one block ahead
    float skn = (sub * AT_SUB + lane < p.Skv) ? __ldg(skh + lane) : 0.0f;
    for (int j = 0; j < J; ++j) {
      const int b = j & 1;
      float* skb = skw + b * AT_SUB;
      skb[lane] = skn;
      {
        const int kn = (j + 1) * AT_BK + sub * AT_SUB + lane;
        skn = (j + 1 < J && kn < p.Skv) ? __ldg(skh + (j + 1) * AT_BK + lane) : 0.0f;
      }
      __syncwarp();  // the block's key scales are in this warp's buffer
      int nvalid = p.Skv - j * AT_BK - sub * AT_SUB;  // valid keys among this warp's 32
      nvalid = nvalid < 0 ? 0 : (nvalid > AT_SUB ? AT_SUB : nvalid);
      uint8_t* prow = smem + L::kOffP + b * kPBytes + (sub >> 1) * kHalf + r * 128;
      const uint32_t t_s = tmem_base + static_cast<uint32_t>(b * 128) + t_row;

      // S_j is in TMEM. P buffer b was last read by P V of block j-2, which was
      // done before this warp signalled block j-1 (it waited for it there).
      if (ok) ok = warp_wait_bounded(&s_full[b], static_cast<uint32_t>((j >> 1) & 1), abort, p.timeout_ns);
      if (ok) tc_fence_after();
      float mh = -INFINITY;
      float bl = 0.0f;
      if (ok) {
        if (j == 0)  // the first block sets the reference maximum: its maximum first
          softmax_pass_any<false>(t_s, skb, c, 0.0f, nvalid, prow, piece0, sw, &mh);
        else  // later blocks: probabilities against the current reference, maximum alongside
          bl = softmax_pass_any<true>(t_s, skb, c, m_ref, nvalid, prow, piece0, sw, &mh);
      }
      // the row's block maximum over its four parts (every block has a valid key)
      mxb[(b * 4 + sub) * AT_BQ + r] = mh;
      quarter_bar(bar_id);
      const float* mrow = mxb + b * 4 * AT_BQ + r;
      const float t_max = c * fmaxf(fmaxf(mrow[0], mrow[AT_BQ]), fmaxf(mrow[2 * AT_BQ], mrow[3 * AT_BQ]));
      float alpha = 1.0f;
      bool need = false;   // O has to follow a raised reference
      bool redo = j == 0;  // P has to be (re)written against the new reference
      if (j == 0) {
        m_ref = t_max;
      } else if (t_max > m_ref + kRescaleThreshold) {
        alpha = ex2_approx(m_ref - t_max);
        m_ref = t_max;
        need = redo = true;
      }
      if (ok) {
        // The pass reads TMEM with warp-collective loads, so the whole warp runs
        // it when any of its rows needs it; for the others the reference did not
        // move and the pass writes the same probabilities again.
        if (__any_sync(0xFFFFFFFFu, redo)) {
          float unused;
          const float bl2 = softmax_pass_any<true>(t_s, skb, c, m_ref, nvalid, prow, piece0, sw, &unused);
          if (redo) bl = bl2;
        }
        l = l * alpha + bl;
        // S_j has been read: its buffer may take S_{j+2}
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[b]);
      }
      // P V of block j-1 is done: O is stable (and, for block j+1, P buffer b^1 is free)
      if (ok && j >= 1) ok = warp_wait_bounded(o_done, static_cast<uint32_t>((j - 1) & 1), abort, p.timeout_ns);
      if (ok) {
        tc_fence_after();
        // this warp's 32 columns of O to the new reference maximum before this block's P V adds to them
        if (__any_sync(0xFFFFFFFFu, need)) {
          const float2 a2 = make_float2(alpha, alpha);
          uint32_t o[32];
          tmem_ld_32x32b_x32(tO + t_row, o);
          tmem_ld_wait_regs(o);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), a2);
            o[2 * i] = __float_as_uint(v.x);
            o[2 * i + 1] = __float_as_uint(v.y);
          }
          tmem_st_32x32b_x32(tO + t_row, o);
          tmem_st_wait();
        }
        // P is read by the tensor cores (async proxy); O's rescale is complete
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
    }
    if (ok) ok = warp_wait_bounded(o_done, static_cast<uint32_t>((J - 1) & 1), abort, p.timeout_ns);
    // the row sum over the four parts
    lsb[sub * AT_BQ + r] = l;
    quarter_bar(bar_id);
    const float inv = 1.0f / ((lsb[r] + lsb[AT_BQ + r]) + (lsb[2 * AT_BQ + r] + lsb[3 * AT_BQ + r]));
    if (ok) {
      tc_fence_after();
      uint16_t* orow = p.O + (static_cast<int64_t>(bh) * p.Sq + qrow) * AT_D + sub * AT_SUB;
      uint32_t o[32];
      tmem_ld_32x32b_x32(tO + t_row, o);
      tmem_ld_wait_regs(o);
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
      if (qrow < p.Sq) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
    if (!ok && lane == 0) attn_abort(abort, p.status);
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// V [BH, Skv, 128] -> Vt [BH, 128, Skv_pad] (keys contiguous), zero beyond Skv.
// CTA: one head and 64 keys; 256 threads.
__global__ void __launch_bounds__(256) transpose_v_kernel(const uint16_t* __restrict__ V, uint16_t* __restrict__ Vt,
                                                          int Skv, int Skv_pad) {
  __shared__ __align__(16) uint16_t tile[64][AT_D + 8];
  const int bh = blockIdx.y;
  const int k0 = blockIdx.x * 64;
  const uint16_t* src = V + static_cast<int64_t>(bh) * Skv * AT_D;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int c = threadIdx.x + it * 256;  // 16-byte chunk: row c / 16, columns 8 * (c % 16) ..
    const int row = c >> 4;
    const int col = (c & 15) * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k0 + row < Skv) v = __ldg(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(k0 + row) * AT_D + col));
    *reinterpret_cast<uint4*>(&tile[row][col]) = v;
  }
  __syncthreads();
  uint16_t* dst = Vt + static_cast<int64_t>(bh) * AT_D * Skv_pad;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int c = threadIdx.x + it * 256;  // 8 keys of one head dimension: d = c / 8, keys 8 * (c % 8) ..
    const int d = c >> 3;
    const int kc = (c & 7) * 8;
    if (k0 + kc >= Skv_pad) continue;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[e] = static_cast<uint32_t>(tile[kc + 2 * e][d]) | (static_cast<uint32_t>(tile[kc + 2 * e + 1][d]) << 16);
    *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(d) * Skv_pad + k0 + kc) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 attn_tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// A 3-D tiled tensor map with a 128-byte swizzle; dims/strides in elements/bytes.
bool encode_3d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = attn_tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(tm, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct AttnWs {
  size_t qq, sq, kq, sk, vt, total;
  int64_t skv_pad;
};

AttnWs attn_ws_layout(int64_t BH, int64_t Sq, int64_t Skv) {
  AttnWs w;
  w.skv_pad = (Skv + 7) / 8 * 8;
  w.qq = 256;
  w.sq = align_up(w.qq + static_cast<size_t>(BH * Sq) * AT_D, 256);
  w.kq = align_up(w.sq + 4 * static_cast<size_t>(BH * Sq), 1024);
  w.sk = align_up(w.kq + static_cast<size_t>(BH * Skv) * AT_D, 256);
  w.vt = align_up(w.sk + 4 * static_cast<size_t>(BH * Skv), 1024);
  w.total = align_up(w.vt + 2 * static_cast<size_t>(BH) * AT_D * static_cast<size_t>(w.skv_pad), 256);
  return w;
}

bool attn_shape_ok(int64_t BH, int64_t Sq, int64_t Skv, int64_t D) {
  return D == AT_D && BH >= 0 && Sq >= 0 && Skv >= 1 && BH <= 65535 && Sq <= (int64_t(1) << 24) &&
         Skv <= (int64_t(1) << 24) && BH * Sq < (int64_t(1) << 31) && BH * Skv < (int64_t(1) << 31);
}

}  // namespace

}  // namespace convrot

extern "C" {

size_t convrot_attention_workspace_bytes(int64_t BH, int64_t Sq, int64_t Skv, int64_t D) {
  if (!convrot::attn_shape_ok(BH, Sq, Skv, D)) return 0;
  return convrot::attn_ws_layout(BH, Sq, Skv).total;
}

convrot_status convrot_attention_int8(const void* Q, const void* K, const void* V, int64_t BH, int64_t Sq,
                                      int64_t Skv, int64_t D, float softmax_scale, void* O, void* ws, size_t ws_bytes,
                                      convrot_stream_t stream) {
  using namespace convrot;
  if (D != AT_D) return CONVROT_ERR_UNSUPPORTED;
  if (!attn_shape_ok(BH, Sq, Skv, D)) return Skv < 1 || BH < 0 || Sq < 0 ? CONVROT_ERR_INVALID_ARG
                                                                        : CONVROT_ERR_UNSUPPORTED;
  if (!(softmax_scale > 0.0f) || !(softmax_scale < 3.0e38f)) return CONVROT_ERR_INVALID_ARG;
  if (BH == 0 || Sq == 0) return CONVROT_OK;  // no queries: nothing to compute
  auto aligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; };
  if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr) return CONVROT_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16)) return CONVROT_ERR_INVALID_ARG;
  const AttnWs lay = attn_ws_layout(BH, Sq, Skv);
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < lay.total) return CONVROT_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(wsb);
  int8_t* Qq = reinterpret_cast<int8_t*>(wsb + lay.qq);
  float* sq = reinterpret_cast<float*>(wsb + lay.sq);
  int8_t* Kq = reinterpret_cast<int8_t*>(wsb + lay.kq);
  float* sk = reinterpret_cast<float*>(wsb + lay.sk);
  uint16_t* Vt = reinterpret_cast<uint16_t*>(wsb + lay.vt);

  CUtensorMap tq, tk, tv;
  if (!encode_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Qq, AT_D, Sq, BH, AT_D, Sq * AT_D, AT_D, AT_BQ) ||
      !encode_3d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, Kq, AT_D, Skv, BH, AT_D, Skv * AT_D, AT_D, AT_BK) ||
      !encode_3d(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Vt, lay.skv_pad, AT_D, BH, 2 * lay.skv_pad,
                 2 * AT_D * lay.skv_pad, 64, AT_D))
    return CONVROT_ERR_INVALID_ARG;

  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return CONVROT_ERR_CUDA;
  // Q and K: the linear layer's rotate + per-token quantise over head vectors (g = D)
  RotQuantParams rq{};
  rq.in_f16 = 0;
  rq.K = AT_D;
  rq.ldx = 0;
  rq.tensor_absmax = nullptr;
  rq.status_reset = nullptr;
  rq.status = status;
  rq.timeout_ns = 2000000000ull;
  rq.src = static_cast<const uint16_t*>(Q);
  rq.rows = BH * Sq;
  rq.dst = Qq;
  rq.scale = sq;
  if (launch_rotate_quant(AT_D, kRqActivation, rq, s) != cudaSuccess) return CONVROT_ERR_CUDA;
  rq.src = static_cast<const uint16_t*>(K);
  rq.rows = BH * Skv;
  rq.dst = Kq;
  rq.scale = sk;
  if (launch_rotate_quant(AT_D, kRqActivation, rq, s) != cudaSuccess) return CONVROT_ERR_CUDA;
  transpose_v_kernel<<<dim3(static_cast<unsigned>((lay.skv_pad + 63) / 64), static_cast<unsigned>(BH)), 256, 0, s>>>(
      static_cast<const uint16_t*>(V), Vt, static_cast<int>(Skv), static_cast<int>(lay.skv_pad));
  if (cudaGetLastError() != cudaSuccess) return CONVROT_ERR_CUDA;

  AttnParams ap{};
  ap.BH = static_cast<int>(BH);
  ap.Sq = static_cast<int>(Sq);
  ap.Skv = static_cast<int>(Skv);
  ap.J = static_cast<int>((Skv + AT_BK - 1) / AT_BK);
  ap.sq = sq;
  ap.sk = sk;
  ap.O = static_cast<uint16_t*>(O);
  ap.c_scale = softmax_scale * 1.4426950408889634f;
  ap.status = status;
  ap.timeout_ns = 2000000000ull;
  static std::atomic<int> attr_done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (dev < 0 || dev >= 64 || attr_done[dev].load(std::memory_order_acquire) == 0) {
    if (cudaFuncSetAttribute(attention_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnSmem::kAlloc) !=
        cudaSuccess)
      return CONVROT_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_done[dev].store(1, std::memory_order_release);
  }
  const dim3 grid(static_cast<unsigned>((Sq + AT_BQ - 1) / AT_BQ), static_cast<unsigned>(BH));
  attention_i8_kernel<<<grid, AT_THREADS, AttnSmem::kAlloc, s>>>(tq, tk, tv, ap);
  return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

}  // extern "C"
