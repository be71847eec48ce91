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
// token), then one CTA per (batch*head, 128-query tile):
//   warp 0, one lane : TMA producer: the tile's 128 x 128 query codes once,
//                      then per 128-key block the key codes (loaded as soon
//                      as the previous block's S is computed) and the values
//                      as given (two 64-column halves of the head dimension,
//                      the MN-major B operand of P V, loaded as soon as the
//                      previous block's P V is done).
//   warp 1           : allocates 256 TMEM columns; one lane issues
//                      S = Qq Kq^T (tcgen05.mma kind::i8, M = N = 128,
//                      K = 4 x 32) into TMEM columns 0..127 and
//                      O += P V (kind::f16 with bf16 operands, M = N = 128,
//                      K = 8 x 16) into columns 128..255.
//   warps 2..5       : softmax, one query row per thread (TMEM lane): S from
//                      TMEM, t = c_i s_k[j] S_ij in base-2 units with
//                      c_i = s_q[i] softmax_scale log2(e), p = 2^(t - m) in
//                      float32, the row sum in float32, P rounded to bf16 into
//                      128-byte-swizzled shared memory for the MMA. The
//                      reference maximum m moves only when a block raises it
//                      by more than 8 (p <= 256), and then O is rescaled in
//                      TMEM once the previous block's P V has finished. At
//                      the end O / sum is rounded to bf16 and stored.
// S is read out of TMEM before the next block's S is written, so the next
// QK^T runs on the tensor cores while this block's softmax runs on the CUDA
// cores. Every wait is bounded (status word + abort flag, as in the GEMM).

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
constexpr int AT_THREADS = 192;
constexpr int kQBytes = AT_BQ * AT_D;      // int8 query codes: 16 KB
constexpr int kKBytes = AT_BK * AT_D;      // int8 key codes of one block: 16 KB
constexpr int kHalf = 128 * 128;           // 128 rows x 128 B: one half of a block's bf16 operand
constexpr int kVBytes = 2 * kHalf;         // values of one block: 32 KB (two 64-column halves)
constexpr int kPBytes = 2 * kHalf;         // probabilities of one block (bf16): 32 KB
constexpr uint32_t IDESC_S = idesc_i8(AT_BQ, AT_BK);
// P V: A = P (K-major), B = V as stored, keys along K and the head dimension
// along N contiguous (MN-major: bit 16 of the instruction descriptor)
constexpr uint32_t IDESC_O = idesc_bf16(AT_BQ, AT_D) | (1u << 16);
constexpr int kTimeoutStatus = 5;
constexpr float kRescaleThreshold = 8.0f;  // base-2 units: probabilities stay below 2^8

// 2 CTAs per SM: everything below (plus the alignment slack) stays under
// half of the SM's 228 KB of shared memory.
struct AttnSmem {
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKBytes;
  static constexpr int kOffP = kOffV + kVBytes;
  static constexpr int kOffSk = kOffP + kPBytes;  // per softmax warp, two buffers of a block's key scales
  static constexpr int kOffBar = kOffSk + 4 * 2 * AT_BK * 4;
  // q_full, k_full, k_empty, v_full, v_empty, s_full, s_empty, p_full, o_done, drain
  static constexpr int kNumBars = 10;
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

// The probabilities of one row for 64 keys (one half), packed to bf16 into the
// row's 128-byte-swizzled shared-memory line; returns their float32 sum.
template <bool MASKED>
__device__ __forceinline__ float write_p_half(const float (&u)[128], int h, float c, float m_ref, int nvalid,
                                              uint8_t* row, int sw) {
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m_ref, -m_ref);
  // four partial sums: one chain of 64 dependent adds per half would leave its
  // latency exposed with two softmax warps per scheduler (3 % of the call)
  float2 sum2[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                    make_float2(0.0f, 0.0f)};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = h * 64 + i * 8 + 2 * e;
      // t = c u - m for two keys at once, then p = 2^t
      const float2 t = __ffma2_rn(c2, make_float2(u[k], u[k + 1]), nm2);
      float2 pp = make_float2(ex2_approx(t.x), ex2_approx(t.y));
      if (MASKED) {
        pp.x = (k < nvalid) ? pp.x : 0.0f;
        pp.y = (k + 1 < nvalid) ? pp.y : 0.0f;
      }
      sum2[e] = __fadd2_rn(sum2[e], pp);
      w[e] = pack_bf16x2(pp.x, pp.y);
    }
    *reinterpret_cast<uint4*>(row + ((i ^ sw) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  const float2 st = __fadd2_rn(__fadd2_rn(sum2[0], sum2[1]), __fadd2_rn(sum2[2], sum2[3]));
  return st.x + st.y;
}

__global__ void __launch_bounds__(AT_THREADS, 2)
    attention_i8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = AttnSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 2;
  uint64_t* v_full = bars + 3;
  uint64_t* v_empty = bars + 4;
  uint64_t* s_full = bars + 5;
  uint64_t* s_empty = bars + 6;
  uint64_t* p_full = bars + 7;
  uint64_t* o_done = bars + 8;
  uint64_t* drain = bars + 9;
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
    mbar_init(k_full, 1);
    mbar_init(k_empty, 1);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);  // the four softmax warps
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_ptr, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;
  const uint32_t tS = tmem_base;        // S: columns 0..127
  const uint32_t tO = tmem_base + 128;  // O: columns 128..255

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Tensor-pipe order is S_0, S_1, PV_0, S_2, PV_1, ...: K_{j+1} goes out
    // when S_j is done, V_{j+1} when PV_j is done.
    if (lane == 0) {
      bool ok = true;
      int issued_k = 0, issued_v = 0;
      auto load_k = [&](int j) {
        mbar_arrive_expect_tx(k_full, kKBytes);
        tma_load_3d(smem + L::kOffK, &tmK, k_full, 0, j * AT_BK, bh);
        issued_k = j + 1;
      };
      auto load_v = [&](int j) {
        mbar_arrive_expect_tx(v_full, kVBytes);
        tma_load_3d(smem + L::kOffV, &tmV, v_full, 0, j * AT_BK, bh);
        tma_load_3d(smem + L::kOffV + kHalf, &tmV, v_full, 64, j * AT_BK, bh);
        issued_v = j + 1;
      };
      mbar_arrive_expect_tx(q_full, kQBytes);
      tma_load_3d(smem + L::kOffQ, &tmQ, q_full, 0, q0, bh);
      load_k(0);
      load_v(0);
      for (int j = 0; j + 1 < J; ++j) {
        if (!mbar_wait_bounded(k_empty, static_cast<uint32_t>(j & 1), abort, p.timeout_ns)) {
          ok = false;
          break;
        }
        load_k(j + 1);
        if (!mbar_wait_bounded(v_empty, static_cast<uint32_t>(j & 1), abort, p.timeout_ns)) {
          ok = false;
          break;
        }
        load_v(j + 1);
      }
      if (!ok) {
        attn_abort(abort, p.status);
        // every copy already issued lands before the shared memory goes away
        mbar_wait_bounded(q_full, 0u, nullptr, p.timeout_ns);
        if (issued_k > 0) mbar_wait_bounded(k_full, static_cast<uint32_t>((issued_k - 1) & 1), nullptr, p.timeout_ns);
        if (issued_v > 0) mbar_wait_bounded(v_full, static_cast<uint32_t>((issued_v - 1) & 1), nullptr, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t qa = smem_addr(smem + L::kOffQ);
      const uint32_t pa = smem_addr(smem + L::kOffP);
      const uint32_t va = smem_addr(smem + L::kOffV);
      const uint32_t kb = smem_addr(smem + L::kOffK);
      auto mma_s = [&](int j) -> bool {
        if (!mbar_wait_bounded(k_full, static_cast<uint32_t>(j & 1), abort, p.timeout_ns)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < AT_D / 32; ++k)
          mma_i8(tS, smem_desc_k_sw128(qa + k * 32), smem_desc_k_sw128(kb + k * 32), IDESC_S, k > 0 ? 1u : 0u);
        mma_commit(s_full);
        mma_commit(k_empty);
        return true;
      };
      bool ok = mbar_wait_bounded(q_full, 0u, abort, p.timeout_ns);
      if (ok) ok = mma_s(0);
      for (int j = 0; j < J && ok; ++j) {
        if (j + 1 < J) {
          // S_{j+1} once the softmax has read S_j out of TMEM
          if (!mbar_wait_bounded(s_empty, static_cast<uint32_t>(j & 1), abort, p.timeout_ns) || !mma_s(j + 1)) {
            ok = false;
            break;
          }
        }
        if (!mbar_wait_bounded(p_full, static_cast<uint32_t>(j & 1), abort, p.timeout_ns) ||
            !mbar_wait_bounded(v_full, static_cast<uint32_t>(j & 1), abort, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // 16 keys per MMA: P's K-major rows advance 32 B inside a 64-key half; V's
        // MN-major atoms are 8 keys x 64 columns (1 KB apart along the keys, the
        // second 64 columns 16 KB on)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16(tO, smem_desc_k_sw128(pa + h * kHalf + k * 32),
                     smem_desc_mn_sw128(va + (4 * h + k) * 2048, kHalf, 1024), IDESC_O, (j | h | k) != 0 ? 1u : 0u);
        mma_commit(o_done);
        mma_commit(v_empty);
      }
      if (!ok) attn_abort(abort, p.status);
      // every MMA this thread issued has finished before TMEM is released
      mma_commit(drain);
      mbar_wait_bounded(drain, 0u, nullptr, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int qd = warp & 3;  // TMEM lane quarter this warp may access
    const int r = qd * 32 + lane;
    const int qrow = q0 + r;
    const float sqv = (qrow < p.Sq) ? __ldg(p.sq + static_cast<int64_t>(bh) * p.Sq + qrow) : 0.0f;
    const float c = sqv * p.c_scale;  // >= 0
    const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
    uint8_t* prow = smem + L::kOffP + r * 128;
    const int sw = r & 7;
    const float* skh = p.sk + static_cast<int64_t>(bh) * p.Skv;
    // this warp's two buffers of a block's 128 key scales (no barrier across warps)
    float* skw = reinterpret_cast<float*>(smem + L::kOffSk) + (warp - 2) * 2 * AT_BK;
    float m_ref = 0.0f;
    float l = 0.0f;
    bool ok = true;
    // lane loads keys 4 * lane .. 4 * lane + 3 of each block, one block ahead
    float skn[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) skn[e] = (4 * lane + e < p.Skv) ? __ldg(skh + 4 * lane + e) : 0.0f;
    for (int j = 0; j < J; ++j) {
      float* skb = skw + (j & 1) * AT_BK;
      *reinterpret_cast<float4*>(skb + 4 * lane) = make_float4(skn[0], skn[1], skn[2], skn[3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kn = (j + 1) * AT_BK + 4 * lane + e;
        skn[e] = (j + 1 < J && kn < p.Skv) ? __ldg(skh + kn) : 0.0f;
      }
      __syncwarp();  // the block's key scales are in this warp's buffer
      const int nvalid = (p.Skv - j * AT_BK) < AT_BK ? (p.Skv - j * AT_BK) : AT_BK;

      if (!warp_wait_bounded(s_full, static_cast<uint32_t>(j & 1), abort, p.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float u[128];  // s_k[key] * S[row, key]: the logit without the row factor c
      {
        // two 32-column loads in flight at a time, converted as they land
        uint32_t a0[32], a1[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          tmem_ld_32x32b_x32(tS + lane_off + half * 64, a0);
          tmem_ld_32x32b_x32(tS + lane_off + half * 64 + 32, a1);
          tmem_ld_wait_regs(a0);
          tmem_ld_wait_regs(a1);
          if (half == 1) {
            // S has been read: the next block's QK^T may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty);
          }
          // u = float(acc) * s_k, two keys per packed f32x2 operation
          const float2 mg = make_float2(-12582912.0f, -12582912.0f);
#pragma unroll
          for (int k4 = 0; k4 < 16; ++k4) {
            const float4 s4 = *reinterpret_cast<const float4*>(skb + half * 64 + 4 * k4);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int k = 4 * k4 + 2 * e;
              const uint32_t acc0 = (k < 32) ? a0[k] : a1[k - 32];
              const uint32_t acc1 = (k + 1 < 32) ? a0[k + 1] : a1[k - 31];
              // float(acc) for |acc| < 2^22: the integer added to the bits of 1.5 * 2^23, minus 1.5 * 2^23
              const float2 x = make_float2(__uint_as_float(acc0 + 0x4B400000u), __uint_as_float(acc1 + 0x4B400000u));
              const float2 v = __fmul2_rn(__fadd2_rn(x, mg), e == 0 ? make_float2(s4.x, s4.y) : make_float2(s4.z, s4.w));
              u[half * 64 + k] = v.x;
              u[half * 64 + k + 1] = v.y;
            }
          }
        }
      }
      // the block maximum over its valid keys, in base-2 units
      float mb;
      if (nvalid == AT_BK) {
        // 128 -> 43 -> 15 -> 5 -> 1 with three-input maxima
        float a[43], b[15], c5[5];
#pragma unroll
        for (int i = 0; i < 42; ++i) a[i] = fwht::fmax3f(u[3 * i], u[3 * i + 1], u[3 * i + 2]);
        a[42] = fmaxf(u[126], u[127]);
#pragma unroll
        for (int i = 0; i < 14; ++i) b[i] = fwht::fmax3f(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
        b[14] = a[42];
#pragma unroll
        for (int i = 0; i < 5; ++i) c5[i] = fwht::fmax3f(b[3 * i], b[3 * i + 1], b[3 * i + 2]);
        mb = fmaxf(fwht::fmax3f(c5[0], c5[1], c5[2]), fmaxf(c5[3], c5[4]));
      } else {
        mb = -INFINITY;
#pragma unroll
        for (int k = 0; k < AT_BK; ++k) mb = (k < nvalid) ? fmaxf(mb, u[k]) : mb;
      }
      const float t_max = c * mb;
      float alpha = 1.0f;
      bool need = false;
      if (j == 0) {
        m_ref = t_max;
      } else if (t_max > m_ref + kRescaleThreshold) {
        alpha = ex2_approx(m_ref - t_max);
        m_ref = t_max;
        need = true;
      }
      // the previous block's P V has finished: O is stable and the P buffer free
      if (j >= 1 && !warp_wait_bounded(o_done, static_cast<uint32_t>((j - 1) & 1), abort, p.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float bl;
      if (nvalid == AT_BK) {
        bl = write_p_half<false>(u, 0, c, m_ref, nvalid, prow, sw) +
             write_p_half<false>(u, 1, c, m_ref, nvalid, prow + kHalf, sw);
      } else {
        bl = write_p_half<true>(u, 0, c, m_ref, nvalid, prow, sw) +
             write_p_half<true>(u, 1, c, m_ref, nvalid, prow + kHalf, sw);
      }
      l = l * alpha + bl;
      // O to the new reference maximum before this block's P V adds to it
      // (after the P writes, so that the logits are no longer live)
      if (__any_sync(0xFFFFFFFFu, need)) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(tO + lane_off + ch * 32, o);
          tmem_ld_wait_regs(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st_32x32b_x32(tO + lane_off + ch * 32, o);
        }
        tmem_st_wait();
      }
      // P is read by the tensor cores (async proxy); O's rescale is complete
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) {
      if (!warp_wait_bounded(o_done, static_cast<uint32_t>((J - 1) & 1), abort, p.timeout_ns)) {
        ok = false;
      } else {
        tc_fence_after();
        const float inv = 1.0f / l;
        uint16_t* orow = p.O + (static_cast<int64_t>(bh) * p.Sq + qrow) * AT_D;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(tO + lane_off + ch * 32, o);
          tmem_ld_wait_regs(o);
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
          if (qrow < p.Sq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      }
    }
    if (!ok && lane == 0) attn_abort(abort, p.status);
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
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
  size_t qq, sq, kq, sk, total;
};

AttnWs attn_ws_layout(int64_t BH, int64_t Sq, int64_t Skv) {
  AttnWs w;
  w.qq = 256;
  w.sq = align_up(w.qq + static_cast<size_t>(BH * Sq) * AT_D, 256);
  w.kq = align_up(w.sq + 4 * static_cast<size_t>(BH * Sq), 1024);
  w.sk = align_up(w.kq + static_cast<size_t>(BH * Skv) * AT_D, 256);
  w.total = align_up(w.sk + 4 * static_cast<size_t>(BH * Skv), 256);
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

  CUtensorMap tq, tk, tv;
  if (!encode_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Qq, AT_D, Sq, BH, AT_D, Sq * AT_D, AT_D, AT_BQ) ||
      !encode_3d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, Kq, AT_D, Skv, BH, AT_D, Skv * AT_D, AT_D, AT_BK) ||
      !encode_3d(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, AT_D, Skv, BH, 2 * AT_D, 2 * AT_D * Skv, 64, AT_BK))
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
