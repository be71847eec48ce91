// int8 x int8 -> int32 GEMM on the 5th-generation tensor cores (tcgen05,
// kind::i8) with a fused epilogue, for Y = Xq Wq^T: both operands K-major.
// In its fused form the same kernel also produces Xq: the whole ConvRot
// linear layer in one launch.
//
// The int8-by-int8 product with int32 accumulation is the multiply step of
// the ConvRot layer (InvokeAI "int8 Compute", second paragraph); the
// epilogue applies the token and tensor scales and the bias and rounds to
// bf16 (or, for exactness tests, stores the raw int32 accumulators).
//
// Three forms share the roles below: the CTA-pair kernel (256x256 tiles on two
// SMs, the layer's GEMM for M > 64), the weight-streaming kernel (M <= 64) and
// the single-SM kernel described here, which carries the rotate+quantise
// workers of the one-launch form of the layer.
//
// Structure of the single-SM form: a persistent kernel, one CTA per SM.
//   warp 0, one lane : TMA producer. 128x128 (A) and 256x128 (B) int8 tiles,
//                      128-byte swizzle, into a 4-stage shared-memory ring.
//   warp 1           : allocates 512 TMEM columns; one lane issues
//                      tcgen05.mma M=128 N=256 K=32 (4 per stage) into one of
//                      two 128x256 int32 accumulators, commits each stage back
//                      to the producer and each finished tile to the epilogue.
//   warps 2..5       : epilogue. Warp w reads TMEM lanes 32*(w%4).. with
//                      tcgen05.ld (one accumulator row per thread), scales,
//                      adds bias, packs bf16, stages 32x32 chunks in swizzled
//                      shared memory and writes them with TMA stores. Two
//                      accumulators let the epilogue of tile i overlap the
//                      MMAs of tile i+1.
//   warps 6..        : (fused form only) rotate + quantise workers. The CTAs
//                      together walk the token rows in order, a few rows per
//                      CTA per pass, and write the int8 codes and token scales
//                      of A. After each pass one thread publishes the rows it
//                      finished in a per-M-block counter tagged with the call's
//                      epoch (release); the producer acquires the counter of
//                      an M-block before its first TMA load of that block, and
//                      the epilogue before reading the block's token scales.
//                      The workers never wait on the GEMM roles, so the GEMM
//                      runs on the tensor cores while the rotation still runs
//                      on the CUDA cores for later rows.
// Tiles are visited in groups of `group_m` M-blocks so that the CTAs in flight
// share A and B panels in L2. Every wait is bounded; a wait that runs out
// records CONVROT_ERR_DEVICE_TIMEOUT (5) in the status word, every role
// unwinds, in-flight copies and MMAs are drained (bounded), TMEM is freed, and
// the CTA returns.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cstdint>

#include "fwht_dev.cuh"
#include "gemm_i8.cuh"
#include "ptx_sm100.cuh"

namespace convrot {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // bytes (= int8 elements) per stage along K: one swizzle row
constexpr int UMMA_K = 32;
constexpr int STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK;
constexpr int B_STAGE_BYTES = BN * BK;
constexpr int EPI_WARPS = 4;
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr int CHUNK = 32;  // epilogue columns per TMEM load / TMA store
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t IDESC = idesc_i8(BM, BN);
constexpr int kTimeoutStatus = 5;
constexpr int kFusedMaxThreads = 512;  // 6 GEMM warps + up to 10 rotate+quantise warps

template <int EPI>
struct Smem {
  static constexpr int kEpiBuf = epi_is_dequant(EPI) ? CHUNK * CHUNK * 2 : CHUNK * CHUNK * 4;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = STAGES * A_STAGE_BYTES;
  static constexpr int kOffEpi = STAGES * (A_STAGE_BYTES + B_STAGE_BYTES);
  static constexpr int kOffBar = kOffEpi + EPI_WARPS * 2 * kEpiBuf;
  static constexpr int kNumBars = 2 * STAGES + 2 + 2 + 1;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 8;
  static constexpr int kOffRowMax = kOffAbort + 8;  // fused form: 2 x kMaxFusedRows row maxima
  static constexpr int kBytes = kOffRowMax + 2 * kMaxFusedRows * 4;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
};

__device__ __forceinline__ void tile_coords(int tile, const GemmParams& p, int& mb, int& nb) {
  const int per_group = p.group_m * p.num_n_blocks;
  const int grp = tile / per_group;
  const int first_m = grp * p.group_m;
  const int rem_m = p.num_m_blocks - first_m;
  const int gsz = rem_m < p.group_m ? rem_m : p.group_m;
  const int r = tile - grp * per_group;
  mb = first_m + r % gsz;
  nb = r / gsz;
}

__device__ __forceinline__ void raise_abort(volatile int* abort, int* status) {
  *abort = 1;
  atomicOr(status, kTimeoutStatus);
}

__device__ __forceinline__ uint64_t ld_acquire_u64(const unsigned long long* p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ float ld_relaxed_f32(const float* p) {
  float v;
  asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier that also ORs a predicate over the participating threads.
__device__ __forceinline__ bool named_barrier_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %3, 0;\n\t"
      "bar.red.or.pred q, %1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(threads), "r"(static_cast<uint32_t>(pred))
      : "memory");
  return r != 0;
}

// Rows of M-block mb that the fused workers must finish, tagged with the epoch.
__device__ __forceinline__ uint64_t ready_target(const GemmParams& p, int mb) {
  const int rows = (p.M - mb * BM) < BM ? (p.M - mb * BM) : BM;
  return (static_cast<uint64_t>(p.epoch) << 32) | static_cast<uint64_t>(rows);
}

// Bounded wait until every row of M-block mb has been quantised in this call.
__device__ __forceinline__ bool wait_block_ready(const GemmParams& p, int mb, volatile int* abort) {
  const uint64_t target = ready_target(p, mb);
  if (ld_acquire_u64(p.ready + mb) == target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (ld_acquire_u64(p.ready + mb) == target) return true;
    if ((it & 15u) == 0) {
      if (abort != nullptr && *abort) return false;
      if (global_timer_ns() - t0 > p.timeout_ns) return false;
    }
  }
}

// Add n finished rows to M-block mb's counter for this epoch (a stale epoch
// restarts the count). Called after a gpu-scope fence: release.
__device__ __forceinline__ void publish_rows(const GemmParams& p, int mb, int n) {
  unsigned long long* c = p.ready + mb;
  unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(c);
  while (true) {
    const unsigned long long nw = ((old >> 32) == p.epoch)
                                      ? old + static_cast<unsigned long long>(n)
                                      : ((static_cast<unsigned long long>(p.epoch) << 32) | static_cast<unsigned>(n));
    const unsigned long long prev = atomicCAS(c, old, nw);
    if (prev == old) break;
    old = prev;
  }
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// A 16-bit output-dtype value (bf16 or fp16 bits), widened exactly.
__device__ __forceinline__ float out16_to_f32(uint32_t bits16, bool f16) {
  return f16 ? __half2float(__ushort_as_half(static_cast<unsigned short>(bits16)))
             : __uint_as_float(bits16 << 16);
}

// erf(x) by the rational approximation of Abramowitz and Stegun, Handbook of
// Mathematical Functions (1964), formula 7.1.26: for x >= 0,
//   erf(x) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-x^2),  t = 1/(1 + p x),
// with |error| <= 1.5e-7; odd symmetry for x < 0. Branch-free, so a warp's
// lanes never diverge on it (the epilogue applies it to every output).
__device__ __forceinline__ float erf_as7126(float x) {
  const float ax = fabsf(x);
  const float t = __fdividef(1.0f, fmaf(0.3275911f, ax, 1.0f));
  float poly = fmaf(1.061405429f, t, -1.453152027f);
  poly = fmaf(poly, t, 1.421413741f);
  poly = fmaf(poly, t, -0.284496736f);
  poly = fmaf(poly, t, 0.254829592f);
  poly *= t;
  const float e = 1.0f - poly * __expf(-ax * ax);
  return copysignf(e, x);
}

// GELU with the Gaussian CDF: y * Phi(y) = 0.5 y (1 + erf(y / sqrt(2))).
__device__ __forceinline__ float gelu_erf(float y) {
  return 0.5f * y * (1.0f + erf_as7126(y * 0.70710678118654752f));
}

// The general epilogue for 32 consecutive output columns n0..n0+31 of one
// row: y = acc * (sc * wv[e]) + bv[e] (then GELU), packed to the output dtype.
// sc is x_scale[row] times the tensor weight scale, or x_scale[row] alone when
// the weight scale is per channel (then wv holds w_scale[n]).
template <bool GELU>
__device__ __forceinline__ void dequant_gen32(const GemmParams& p, int row, int n0, float sc,
                                              const uint32_t (&r)[32], uint32_t (&packed)[16]) {
  const bool f16 = p.out_f16 != 0;
  float bv[32], wv[32];
#pragma unroll
  for (int pc = 0; pc < 4; ++pc) {
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (p.bias != nullptr && n0 + 8 * pc < p.N) w = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + 8 * pc));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      bv[8 * pc + 2 * e] = out16_to_f32(ws[e] & 0xFFFFu, f16);
      bv[8 * pc + 2 * e + 1] = out16_to_f32(ws[e] >> 16, f16);
    }
  }
  if (p.wscale_per_channel) {
#pragma unroll
    for (int pc = 0; pc < 8; ++pc) {
      float4 w = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (n0 + 4 * pc < p.N) w = __ldg(reinterpret_cast<const float4*>(p.w_scale + n0 + 4 * pc));
      wv[4 * pc] = w.x;
      wv[4 * pc + 1] = w.y;
      wv[4 * pc + 2] = w.z;
      wv[4 * pc + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) wv[e] = 1.0f;
  }
  if (p.addend != nullptr && row < p.M) {  // this row's 32 addend values join the bias
    const int64_t ld = p.ldy ? p.ldy : p.N;
    const uint16_t* a = p.addend + static_cast<int64_t>(row) * ld + n0;
#pragma unroll
    for (int pc = 0; pc < 4; ++pc) {
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (n0 + 8 * pc < p.N) w = __ldg(reinterpret_cast<const uint4*>(a + 8 * pc));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        bv[8 * pc + 2 * e] += out16_to_f32(ws[e] & 0xFFFFu, f16);
        bv[8 * pc + 2 * e + 1] += out16_to_f32(ws[e] >> 16, f16);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    float y0 = fmaf(static_cast<float>(static_cast<int32_t>(r[2 * e])), sc * wv[2 * e], bv[2 * e]);
    float y1 = fmaf(static_cast<float>(static_cast<int32_t>(r[2 * e + 1])), sc * wv[2 * e + 1], bv[2 * e + 1]);
    if (GELU) {
      y0 = gelu_erf(y0);
      y1 = gelu_erf(y1);
    }
    packed[e] = f16 ? f16x2(y0, y1) : bf16x2(y0, y1);
  }
}

// The weight scale a row's multiplier carries: the tensor scale, or 1 when
// the general epilogue applies a per-channel scale column by column.
template <int EPI>
__device__ __forceinline__ float epi_weight_scale(const GemmParams& p) {
  if (EPI == kEpiDequantBf16) return __ldg(p.w_scale);
  if (epi_is_general(EPI)) return p.wscale_per_channel ? 1.0f : __ldg(p.w_scale);
  return 0.0f;
}

// One tile's epilogue for one warp: kChunks chunks of 32 accumulator columns
// of the warp's 32 TMEM lanes (rows row0..row0+31), from t_row / n_base on:
// load, scale + bias, pack, stage in swizzled shared memory, TMA store.
// release() is called by lane 0 once the warp has read its columns.
template <int EPI, int kChunks = BN / CHUNK, class Release>
__device__ __forceinline__ void epilogue_tile(const CUtensorMap* tmOut, const GemmParams& p, uint32_t t_row,
                                              int row0, int n_base, float sc, uint8_t* ebuf0, int& chunk_count,
                                              int lane, Release release) {
  constexpr int kEpiBuf = epi_is_dequant(EPI) ? CHUNK * CHUNK * 2 : CHUNK * CHUNK * 4;
  // two register buffers: the load of chunk c+1 is in flight while chunk c
  // is converted and stored
  uint32_t buf[2][32];
  tmem_ld_32x32b_x32(t_row, buf[0]);
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    uint32_t (&r)[32] = buf[c & 1];
    tmem_ld_wait_regs(r);
    if (c + 1 < kChunks) {
      tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((c + 1) * CHUNK), buf[(c + 1) & 1]);
    } else {  // accumulator fully read: hand it back to the MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) release();
    }
    const int n0 = n_base + c * CHUNK;
    if (n0 >= p.N) continue;
    uint8_t* ebuf = ebuf0 + (chunk_count & 1) * kEpiBuf;
    if (lane == 0) bulk_wait_group_read<1>();  // the store that last read this buffer is done
    __syncwarp();
    if (epi_is_general(EPI)) {
      uint32_t packed[16];
      dequant_gen32<EPI == kEpiDequantGenGelu>(p, row0 + lane, n0, sc, r, packed);
      uint8_t* rowp = ebuf + lane * 64;  // same 64-byte-swizzled staging as below
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int pj = j ^ ((lane >> 1) & 3);
        *reinterpret_cast<uint4*>(rowp + pj * 16) =
            make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
      }
    } else if (EPI == kEpiDequantBf16) {
      float bv[32];
      if (p.bias != nullptr) {
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (n0 + 8 * pc < p.N) w = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + 8 * pc));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            bv[8 * pc + 2 * e] = __uint_as_float(ws[e] << 16);
            bv[8 * pc + 2 * e + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) bv[e] = 0.0f;
      }
      uint32_t packed[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {  // two fused multiply-adds per packed instruction (each rounded once)
        const float2 y = __ffma2_rn(make_float2(static_cast<float>(static_cast<int32_t>(r[2 * e])),
                                                static_cast<float>(static_cast<int32_t>(r[2 * e + 1]))),
                                    make_float2(sc, sc), make_float2(bv[2 * e], bv[2 * e + 1]));
        packed[e] = bf16x2(y.x, y.y);
      }
      // 32 rows x 64 bytes, 64-byte swizzle: 16-byte piece j of row r at piece j ^ ((r >> 1) & 3)
      uint8_t* rowp = ebuf + lane * 64;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int pj = j ^ ((lane >> 1) & 3);
        *reinterpret_cast<uint4*>(rowp + pj * 16) =
            make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
      }
    } else {
      // 32 rows x 128 bytes, 128-byte swizzle: piece j of row r at piece j ^ (r & 7)
      uint8_t* rowp = ebuf + lane * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int pj = j ^ (lane & 7);
        *reinterpret_cast<uint4*>(rowp + pj * 16) = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmOut, ebuf, n0, row0);
      bulk_commit_group();
    }
    ++chunk_count;
  }
}

// Fused rotate + quantise worker (warps 6.. of the fused kernel): rows
// [pass*rpp, pass*rpp + rpp) for pass = blockIdx.x, blockIdx.x + gridDim.x, ...
// Same thread layout and arithmetic as the standalone rotate+quantise kernel
// (64 elements per lane, g/64 lanes per group, f32x2 butterflies, shuffles
// across the group's lanes), reading X straight from global memory.
template <int G>
__device__ __forceinline__ void quant_worker(const GemmParams& p, int qtid, int nq, unsigned* rmax2,
                                             volatile int* abort) {
  using namespace fwht;
  constexpr int LG = G / 64;
  constexpr int PIECE = G / 8;
  const int tpr = p.q_threads_per_row;
  const int rpp = p.q_rows_per_pass;
  const int row_in_pass = qtid / tpr;
  const int t = qtid - row_in_pass * tpr;
  const int grp = t / LG;
  const int l = t - grp * LG;
  const bool lane_active = row_in_pass < rpp;
  int pass = 0;
  for (int64_t gp = blockIdx.x; gp * rpp < p.M; gp += gridDim.x, ++pass) {
    const int64_t r0 = gp * rpp;
    const int64_t row = r0 + row_in_pass;
    const bool valid = lane_active && row < p.M;
    unsigned* rmax = rmax2 + (pass & 1) * kMaxFusedRows;
    if (qtid < rpp) rmax[qtid] = 0u;
    const int64_t base = row * p.K + static_cast<int64_t>(grp) * G + 8 * l;
    float2 v[4][8];
    if (valid) {
      uint4 raw[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint16_t* src = p.X + base + j * PIECE;
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(raw[j].x), "=r"(raw[j].y), "=r"(raw[j].z), "=r"(raw[j].w)
                     : "l"(src));
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const uint32_t aw[4] = {raw[jj].x, raw[jj].y, raw[jj].z, raw[jj].w};
        const uint32_t bw[4] = {raw[jj + 4].x, raw[jj + 4].y, raw[jj + 4].z, raw[jj + 4].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          v[jj][2 * q] = make_float2(__uint_as_float(aw[q] << 16), __uint_as_float(bw[q] << 16));
          v[jj][2 * q + 1] =
              make_float2(__uint_as_float(aw[q] & 0xFFFF0000u), __uint_as_float(bw[q] & 0xFFFF0000u));
        }
      }
    } else {
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int e = 0; e < 8; ++e) v[jj][e] = make_float2(0.0f, 0.0f);
    }
    fwht_group<G>(v, l);
    float m = 0.0f;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fmaxf(fabsf(v[jj][e].x), fabsf(v[jj][e].y)));
#pragma unroll
    for (int s = 1; s < LG; s <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, s));
    named_barrier_sync(1, nq);  // rmax initialised
    if (valid && l == 0) atomicMax(&rmax[row_in_pass], __float_as_uint(m));
    named_barrier_sync(1, nq);
    if (valid) {
      const QuantScale qs = make_scale<G>(__uint_as_float(rmax[row_in_pass]));
      if (t == 0) p.x_scale_out[row] = qs.s;
      if (qs.pre != 1.0f) {
        const float2 pre2 = make_float2(qs.pre, qs.pre);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
#pragma unroll
          for (int e = 0; e < 8; ++e) v[jj][e] = __fmul2_rn(v[jj][e], pre2);
      }
      const float2 ci2 = make_float2(qs.ci, qs.ci);
      const float2 magic2 = make_float2(kRoundMagic, kRoundMagic);
      int8_t* dst = p.Xq + base;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        float2 r[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = __ffma2_rn(v[jj][e], ci2, magic2);
        uint2 lo, hi;
        lo.x = pack4(r[0].x, r[1].x, r[2].x, r[3].x);
        lo.y = pack4(r[4].x, r[5].x, r[6].x, r[7].x);
        hi.x = pack4(r[0].y, r[1].y, r[2].y, r[3].y);
        hi.y = pack4(r[4].y, r[5].y, r[6].y, r[7].y);
        *reinterpret_cast<uint2*>(dst + jj * PIECE) = lo;
        *reinterpret_cast<uint2*>(dst + (jj + 4) * PIECE) = hi;
      }
    }
    // the codes are read by TMA (async proxy) in other CTAs
    fence_proxy_async_global();
    // every worker's stores of this pass are done; all workers agree on stopping
    // early when another role of the CTA has given up
    const bool stop = named_barrier_or(1, nq, *abort != 0);
    if (qtid == 0) {
      __threadfence();
      const int64_t r1 = (r0 + rpp) < p.M ? (r0 + rpp) : p.M;
      for (int64_t r = r0; r < r1;) {
        const int mb = static_cast<int>(r / BM);
        const int64_t end = (static_cast<int64_t>(mb) + 1) * BM < r1 ? (static_cast<int64_t>(mb) + 1) * BM : r1;
        publish_rows(p, mb, static_cast<int>(end - r));
        r = end;
      }
    }
    if (stop) break;
  }
}

}  // namespace

template <int EPI, int FG>
__global__ void __launch_bounds__(FG ? kFusedMaxThreads : NUM_THREADS, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  using L = Smem<EPI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tmem_full = bars + 2 * STAGES;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* drain = tmem_empty + 2;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + L::kOffTmemPtr);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmOut);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_ptr, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;
  // Everything above overlaps the previous kernel (programmatic launch); its
  // outputs (and, fused, the workspace it may still read) are touched only
  // after this point.
  griddep_wait();

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int pending_phase[STAGES];
      for (int i = 0; i < STAGES; ++i) pending_phase[i] = -1;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, p, mb, nb);
        if (FG != 0) {
          if (!wait_block_ready(p, mb, abort)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();  // the codes were written by generic stores
        }
        for (int kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], A_STAGE_BYTES + B_STAGE_BYTES);
          tma_load_2d(smem + L::kOffA + s * A_STAGE_BYTES, &tmA, &full[s], kb * BK, mb * BM);
          tma_load_2d(smem + L::kOffB + s * B_STAGE_BYTES, &tmB, &full[s], kb * BK, nb * BN);
          pending_phase[s] = static_cast<int>(ph);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // all of this CTA's loads are issued: the next kernel may start launching
      griddep_launch_dependents();
      if (!ok) {
        raise_abort(abort, p.status);
        // let every copy already issued land before the CTA's shared memory goes away
        for (int i = 0; i < STAGES; ++i)
          if (pending_phase[i] >= 0)
            mbar_wait_bounded(&full[i], static_cast<uint32_t>(pending_phase[i]), nullptr, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int b = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait_bounded(&tmem_empty[b], (use & 1u) ^ 1u, abort, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(b * BN);
        for (int kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait_bounded(&full[s], ph, abort, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_addr(smem + L::kOffA + s * A_STAGE_BYTES);
          const uint32_t b_base = smem_addr(smem + L::kOffB + s * B_STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            mma_i8(d, smem_desc_k_sw128(a_base + k * UMMA_K), smem_desc_k_sw128(b_base + k * UMMA_K), IDESC,
                   (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tmem_full[b]);
      }
      if (!ok) raise_abort(abort, p.status);
      // every MMA this thread issued has finished before TMEM is released
      mma_commit(drain);
      mbar_wait_bounded(drain, 0u, nullptr, p.timeout_ns);
    }
  } else if (warp < 2 + EPI_WARPS) {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const float sw = epi_weight_scale<EPI>(p);
    uint8_t* ebuf0 = smem + L::kOffEpi + (q * 2) * L::kEpiBuf;
    int chunk_count = 0;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      int mb, nb;
      tile_coords(tile, p, mb, nb);
      const int b = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      if (!mbar_wait_bounded(&tmem_full[b], use & 1u, abort, p.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int row0 = mb * BM + q * 32;
      const int row = row0 + lane;
      float sc = 0.0f;
      if (FG != 0) {
        // the token scales of this block were written in this launch: acquire, then coherent loads
        if (!wait_block_ready(p, mb, abort)) {
          ok = false;
          break;
        }
        sc = (row < p.M ? ld_relaxed_f32(p.x_scale + row) : 0.0f) * sw;
      } else if (epi_is_dequant(EPI)) {
        sc = (row < p.M ? __ldg(p.x_scale + row) : 0.0f) * sw;
      }
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * BN);
      epilogue_tile<EPI>(&tmOut, p, t_row, row0, nb * BN, sc, ebuf0, chunk_count, lane,
                         [&]() { mbar_arrive(&tmem_empty[b]); });
    }
    if (!ok && lane == 0) raise_abort(abort, p.status);
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  } else {
    // ------------------------------------------------ fused rotate + quantise
    if constexpr (FG != 0) {
      unsigned* rmax2 = reinterpret_cast<unsigned*>(smem + L::kOffRowMax);
      quant_worker<FG>(p, static_cast<int>(threadIdx.x) - NUM_THREADS, static_cast<int>(blockDim.x) - NUM_THREADS,
                       rmax2, abort);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ===================================================== CTA-pair (2-SM) form
//
// Two CTAs of a cluster compute a 256x256 tile together with
// tcgen05.mma.cta_group::2 (M=256, N=256, K=32): CTA r of the pair loads rows
// r*128.. of the A tile and rows r*128.. of the B tile (its half of N) into its
// own shared memory, so per SM the operand traffic is 32 KB per 128-byte K
// step instead of 48 KB. The leader (rank 0) issues the MMAs; its full
// barrier collects both CTAs' TMA bytes; tcgen05.commit multicasts stage and
// accumulator completion to both CTAs; the follower's epilogue warps release
// the accumulator by arriving on the leader's barrier. Each CTA holds its 128
// rows x 256 columns of the accumulator (two buffers, 512 columns), and runs
// the same epilogue routine as the single-SM form on them, split over eight
// warps of 128 columns each. No TMA multicast is used.

constexpr int BN_HALF = BN / 2;
// Eight epilogue warps per CTA: two per TMEM lane quarter, each draining 128
// of a tile's 256 accumulator columns, so that the epilogue of a tile (with
// GELU the heaviest part of the kernel) stays shorter than the next tile's MMAs.
constexpr int PAIR_EPI_WARPS = 8;
constexpr int PAIR_THREADS = 64 + 32 * PAIR_EPI_WARPS;
// Two consecutive 128-byte k-blocks per ring stage: one barrier wait, fence
// and commit of the MMA issuer per eight MMAs instead of four (3.6-6.2 %
// faster on the measured layers than one k-block per stage with six stages).
#ifndef CONVROT_PAIR_KPS
#define CONVROT_PAIR_KPS 2
#endif
#ifndef CONVROT_PAIR_STAGES
#define CONVROT_PAIR_STAGES (CONVROT_PAIR_KPS == 1 ? 6 : 3)
#endif
#ifndef CONVROT_PAIR_GROUP_M
#define CONVROT_PAIR_GROUP_M 16
#endif
constexpr int PAIR_STAGES = CONVROT_PAIR_STAGES;
constexpr int PKPS = CONVROT_PAIR_KPS;                // k-blocks per ring stage
constexpr int PA_BOX_BYTES = BM * BK;                  // 16 KB: this CTA's 128 rows of A, one k-block
constexpr int PB_BOX_BYTES = BN_HALF * BK;             // 16 KB: this CTA's 128 rows of B, one k-block
constexpr int PA_STAGE_BYTES = PA_BOX_BYTES * PKPS;
constexpr int PB_STAGE_BYTES = PB_BOX_BYTES * PKPS;

// k-blocks of ring stage ks that lie inside K (the last stage may hold fewer)
__device__ __forceinline__ int stage_kblocks(int ks, int num_k_blocks) {
  const int left = num_k_blocks - ks * PKPS;
  return left < PKPS ? left : PKPS;
}
constexpr uint32_t IDESC_PAIR = idesc_i8(2 * BM, BN);

template <int EPI>
struct PairSmem {
  static constexpr int kStages = epi_is_dequant(EPI) ? PAIR_STAGES : PAIR_STAGES - 1;
  static constexpr int kEpiBuf = epi_is_dequant(EPI) ? CHUNK * CHUNK * 2 : CHUNK * CHUNK * 4;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kStages * PA_STAGE_BYTES;
  static constexpr int kOffEpi = kStages * (PA_STAGE_BYTES + PB_STAGE_BYTES);
  static constexpr int kOffBar = kOffEpi + PAIR_EPI_WARPS * 2 * kEpiBuf;
  // full[S], empty[S], tmem_full[2], tmem_empty[2], drain, teardown
  static constexpr int kNumBars = 2 * kStages + 2 + 2 + 1 + 1;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 8;
  static constexpr int kBytes = kOffAbort + 8;
  static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ void pair_tile_coords(int tile, const GemmParams& p, int& mb2, int& nb) {
  const int per_group = p.group_m * p.num_n_blocks;
  const int grp = tile / per_group;
  const int first_m = grp * p.group_m;
  const int rem_m = p.num_m_blocks - first_m;  // here: 256-row blocks
  const int gsz = rem_m < p.group_m ? rem_m : p.group_m;
  const int r = tile - grp * per_group;
  mb2 = first_m + r % gsz;
  nb = r / gsz;
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
    gemm_i8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  using L = PairSmem<EPI>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tmem_full = bars + 2 * S;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* drain = tmem_empty + 2;
  uint64_t* teardown = drain + 1;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + L::kOffTmemPtr);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int num_pairs = static_cast<int>(gridDim.x >> 1);

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmOut);
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], 2 * PAIR_EPI_WARPS);  // both CTAs' epilogue warps
    }
    mbar_init(drain, 1);
    mbar_init(teardown, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_ptr, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers exist before any remote arrive or TMA completion targets them
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;
  const int num_tiles = p.num_m_blocks * p.num_n_blocks;  // pair tiles
  if (warp == 0 && lane == 0 && pair < num_tiles) {
    // the weight does not come from the previous kernel in a forward pass:
    // start pulling this CTA's first B panel into L2 while that kernel finishes
    int mb2, nb;
    pair_tile_coords(pair, p, mb2, nb);
    const int nk = p.num_k_blocks < 32 ? p.num_k_blocks : 32;
    for (int kb = 0; kb < nk; ++kb) tma_prefetch_2d(&tmB, kb * BK, nb * BN + static_cast<int>(rank) * BN_HALF);
  }
  // Only the activation codes and token scales come from the previous kernel
  // (the rotate+quantise launch, which releases this one only after its own
  // predecessor has finished): the producer waits for it before its first A
  // load, the epilogue before its first token scale; the weight loads of the
  // first S stages go out before that wait.

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      bool ok = true;
      const int nks = (p.num_k_blocks + PKPS - 1) / PKPS;  // ring stages per tile
      auto load_a = [&](int st, int ks, int mb2) {
        const int nv = stage_kblocks(ks, p.num_k_blocks);
        for (int i = 0; i < nv; ++i)
          tma_load_2d_pair(smem + L::kOffA + st * PA_STAGE_BYTES + i * PA_BOX_BYTES, &tmA, map_to_rank(&full[st], 0),
                           (ks * PKPS + i) * BK, mb2 * 2 * BM + static_cast<int>(rank) * BM);
      };
      int early_s[S], early_kb[S], early_mb[S];
      int n_early = 0;
      bool waited = false;
      auto release_early = [&]() {  // wait for the previous kernel, then the A loads held back
        griddep_wait();
        waited = true;
        for (int i = 0; i < n_early; ++i) load_a(early_s[i], early_kb[i], early_mb[i]);
      };
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int mb2, nb;
        pair_tile_coords(tile, p, mb2, nb);
        for (int kb = 0; kb < nks; ++kb) {  // kb: ring stage of the tile (PKPS k-blocks)
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort, p.timeout_ns)) {
            ok = false;
            break;
          }
          const int nv = stage_kblocks(kb, p.num_k_blocks);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * nv * (PA_BOX_BYTES + PB_BOX_BYTES));
          const uint32_t bar_leader = map_to_rank(&full[s], 0);
          for (int i = 0; i < nv; ++i)
            tma_load_2d_pair(smem + L::kOffB + s * PB_STAGE_BYTES + i * PB_BOX_BYTES, &tmB, bar_leader,
                             (kb * PKPS + i) * BK, nb * BN + static_cast<int>(rank) * BN_HALF);
          if (waited) {
            load_a(s, kb, mb2);
          } else {
            early_s[n_early] = s;
            early_kb[n_early] = kb;
            early_mb[n_early] = mb2;
            if (++n_early == S) release_early();
          }
          ++issued;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!waited) release_early();  // fewer than S stages in all, or a timed-out wait
      griddep_launch_dependents();
      if (!ok) raise_abort(abort, p.status);
      // the last stages are released (MMAs done reading this CTA's operands and
      // their commits delivered) before this CTA may go away
      for (int64_t k = (issued > S ? issued - S : 0); k < issued; ++k)
        mbar_wait_bounded(&empty[k % S], static_cast<uint32_t>((k / S) & 1), nullptr, p.timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA (leader)
    if (lane == 0 && leader) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int it = 0;
      const bool rec = p.clock_rec != nullptr && blockIdx.x == 0;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++it) {
        const int b = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait_bounded(&tmem_empty[b], (use & 1u) ^ 1u, abort, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(b * BN);
        const int nks = (p.num_k_blocks + PKPS - 1) / PKPS;
        for (int kb = 0; kb < nks; ++kb) {  // kb: ring stage of the tile
          if (!mbar_wait_bounded(&full[s], ph, abort, p.timeout_ns)) {
            ok = false;
            break;
          }
          if (rec && it == 0 && kb == 0) {
            p.clock_rec[0] = clock64();
            p.clock_rec[1] = global_timer_ns();
          }
          tc_fence_after();
          const uint32_t a_base = smem_addr(smem + L::kOffA + s * PA_STAGE_BYTES);
          const uint32_t b_base = smem_addr(smem + L::kOffB + s * PB_STAGE_BYTES);
          const int nv = stage_kblocks(kb, p.num_k_blocks);
#pragma unroll
          for (int i = 0; i < PKPS; ++i) {
            if (i < nv) {
#pragma unroll
              for (int k = 0; k < BK / UMMA_K; ++k) {
                mma_i8_pair(d, smem_desc_k_sw128(a_base + i * PA_BOX_BYTES + k * UMMA_K),
                            smem_desc_k_sw128(b_base + i * PB_BOX_BYTES + k * UMMA_K), IDESC_PAIR,
                            (kb | i | k) != 0 ? 1u : 0u);
              }
            }
          }
          mma_commit_pair_mc(&empty[s], 0x3);  // the stage is free in both CTAs
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_mc(&tmem_full[b], 0x3);  // both halves of the accumulator are final
      }
      if (!ok) raise_abort(abort, p.status);
      if (rec && ok && it > 0) {
        p.clock_rec[2] = clock64();
        p.clock_rec[3] = global_timer_ns();
      }
      mma_commit_pair_mc(drain, 0x1);
      mbar_wait_bounded(drain, 0u, nullptr, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------ epilogue (both)
    griddep_wait();            // the token scales come from the previous kernel
    const int ew = warp - 2;   // 0..7
    const int q = warp & 3;    // TMEM lane quarter this warp may access
    const int half = ew >> 2;  // which 128 of the tile's 256 columns
    const float sw = epi_weight_scale<EPI>(p);
    uint8_t* ebuf0 = smem + L::kOffEpi + (ew * 2) * L::kEpiBuf;
    int chunk_count = 0;
    int it = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++it) {
      int mb2, nb;
      pair_tile_coords(tile, p, mb2, nb);
      const int b = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      if (!mbar_wait_bounded(&tmem_full[b], use & 1u, abort, p.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int row0 = mb2 * 2 * BM + static_cast<int>(rank) * BM + q * 32;
      const int row = row0 + lane;
      float sc = 0.0f;
      if (epi_is_dequant(EPI)) sc = (row < p.M ? __ldg(p.x_scale + row) : 0.0f) * sw;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(b * BN + half * BN_HALF);
      const uint32_t release_addr = map_to_rank(&tmem_empty[b], 0);
      epilogue_tile<EPI, BN_HALF / CHUNK>(&tmOut, p, t_row, row0, nb * BN + half * BN_HALF, sc, ebuf0, chunk_count,
                                          lane, [&]() { mbar_arrive_cluster(release_addr); });
    }
    if (!ok && lane == 0) raise_abort(abort, p.status);
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    // both CTAs are done with the pair's TMEM and with each other's barriers
    if (lane == 0) {
      mbar_arrive_cluster(map_to_rank(teardown, rank ^ 1u));
      mbar_wait_bounded(teardown, 0u, nullptr, p.timeout_ns);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ===================================================== small-M (swap-AB) form
//
// For at most 64 tokens the layer is bound by streaming the int8 weight. The
// MMA then takes the weight as its M side (128 weight rows per tile) and the
// tokens as its N side (16..64): D[n][m] = sum_k Wq[n][k] Xq[m][k]. The
// weight streams through a deep TMA ring per CTA (the activation codes are
// tiny and stay in L2); the weight loads of the first ring stages go out
// before waiting on the previous kernel, so the weight streams while the
// rotate+quantise kernel runs. TMEM lane n holds weight row n, so the
// epilogue writes Y[m][n] with 32 consecutive n per warp store.
//
// Work split. Without split buffers, CTA c takes weight tiles c, c + grid,
// ... whole (one CTA per 128 weight rows, so N/128 of the SMs stream). With
// them, the (weight tile, 128-wide k-block) units are divided evenly into
// contiguous ranges, one per CTA on every SM, so a tile's K loop may be
// shared by two or three consecutive CTAs. A CTA that holds only part of a
// tile's K stores its int32 partial accumulators in its own slot and counts
// itself in at the tile's arrival counter; the CTA that arrives last adds the
// other slots to its own partial and runs the epilogue. Integer addition is
// exact, so the result does not depend on the order of arrival, and no CTA
// ever waits for another.

constexpr int SM_BW = 128;  // weight rows the MMA covers (M = 128); a tile loads at most this many

// KPS: consecutive 128-byte k-blocks per ring stage (one TMA box each), so
// that each weight row is read in runs of KPS * 128 bytes.
#ifndef CONVROT_SMALLM_KPS
#define CONVROT_SMALLM_KPS 2
#endif
// Whole-tile form, off: size the weight tile so that the tiles cover the SMs
// once (ceil(N / SMs) rows, rounded up to the 8-row swizzle atom) instead of
// 128 rows on ceil(N / 128) SMs. Measured slower on every text-encoder shape
// (M = 1, N = 12288: 15.4 against 14.5 us per layer call on 140 SMs; N = 4096:
// 15.8 against 13.0 us).
#ifndef CONVROT_SMALLM_FIT_ROWS
#define CONVROT_SMALLM_FIT_ROWS 0
#endif

// Fused form (FQ): for a few tokens the kernel rotates and quantises them
// itself, into a shared-memory copy of all K codes, so that a layer call is
// one launch whose weight stream starts while the previous kernel still runs.
// Its CTAs have kSmallQuantWarps more warps, and warps 2.. (the epilogue warps
// and those) do the quantisation, redundantly in every CTA, in passes of
// kSmallQuantThreads * 64 values. Used where one pass holds all tokens
// (M * K <= 16384): each further pass costs about 2.5 us (a pass waits for
// its token loads, issued while the weight stream is in flight), so at M = 16, K = 4096
// the two-kernel form is faster (14.6 against 23.6 us); at M = 1 the fused
// form saves the rotate kernel and two dependent-launch hops (13.3 against
// 14.5 us).
#ifndef CONVROT_SMALLM_FUSED
#define CONVROT_SMALLM_FUSED 1
#endif
// Whole tiles, off: the weight panel of each tile (a contiguous range of rows)
// prefetched into L2 once the first ring stages are requested. Measured
// slower on every text-encoder shape (0.5-1.5 us per layer call).
#ifndef CONVROT_SMALLM_PANEL_PREFETCH
#define CONVROT_SMALLM_PANEL_PREFETCH 0
#endif
constexpr int kSmallQuantM = 16;                          // tokens (one 16-column MMA)
constexpr int kSmallQuantMaxK = 8192;                     // codes: 16 x K bytes of shared memory
constexpr int kSmallQuantWarps = 4;                       // warps added to the CTA
constexpr int kSmallQuantThreads = (EPI_WARPS + kSmallQuantWarps) * 32;  // warps 2..9
constexpr uint32_t kSmallPanelChunk = 32 * 1024;          // bytes per L2 prefetch instruction

// Shared memory of the weight-streaming kernel: a 1 KB header (barriers,
// TMEM address, flags, the fused form's token scales and row maxima), then
// (fused form) the token codes, then the weight ring (S stages of R weight
// rows x KPS k-blocks, packed: k-block i of stage s starts (s * KPS + i) * R *
// 128 bytes in), then (two-kernel form) the token ring. The MMA always reads
// 128 weight rows from a k-block's start; the rows past R belong to the next
// box (or, for the ring's last box, to what follows, inside the allocation)
// and only fill TMEM lanes the epilogue never reads.
template <int BNT, int KPS = 1, bool FQ = false>
struct SmallSmem {
  static constexpr int kX1 = BNT * BK;  // 2..8 KB: one token k-block
  static constexpr int kX = FQ ? 0 : kX1 * KPS;
  static constexpr int kMaxStages = 16;
  static constexpr int kRing = KPS == 1 ? 200 * 1024 : 216 * 1024;
  static constexpr int kNumBars = 2 * kMaxStages + 2 + 2 + 1 + 1;
  static constexpr int kOffBar = 0;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 8;
  static constexpr int kOffLast = kOffAbort + 8;  // split form: "this CTA finishes the tile"
  static constexpr int kOffXs = 512;                       // fused form: the token scales
  static constexpr int kOffRmax = kOffXs + 4 * kSmallQuantM;  // fused form: 2 x 16 row maxima
  static constexpr int kHeader = 1024;
  static_assert(kOffLast + 8 <= kOffXs && kOffRmax + 8 * kSmallQuantM <= kHeader, "header overflow");
  static_assert(!FQ || BNT == kSmallQuantM, "the fused form has one 16-token MMA column block");
  static constexpr int kAlloc = 1024 + kHeader + kRing;  // + the 1 KB alignment slack
  // bytes of the fused form's codes (all K of BNT tokens)
  __host__ __device__ static constexpr int codes_bytes(int K) { return FQ ? BNT * K : 0; }
  // weight bytes of one stage for R rows
  __host__ __device__ static constexpr int w_stage(int rows) { return rows * BK * KPS; }
  // ring stages for R rows: the MMA's overrun past the last box ((128 - R)
  // rows) stays inside the allocation
  __host__ __device__ static constexpr int stages(int rows, int K) {
    const int fit = (kRing - codes_bytes(K) - (SM_BW - rows) * BK) / (w_stage(rows) + kX);
#ifdef CONVROT_SMALLM_STAGES
    const int cap = CONVROT_SMALLM_STAGES < kMaxStages ? CONVROT_SMALLM_STAGES : kMaxStages;
#else
    const int cap = kMaxStages;
#endif
    return fit < cap ? fit : cap;
  }
};

// The sequence of (weight tile, k-block range) segments a CTA works on; every
// role of the CTA walks the same sequence.
struct SmallSegments {
  bool split;
  int KB, tiles, G;
  int64_t u, u1;  // split: the CTA's unit range [u, u1)
  int next;       // no split: the next whole tile
  __device__ __forceinline__ SmallSegments(const GemmParams& p, int num_tiles) {
    split = p.split_part != nullptr;
    KB = p.num_k_blocks;
    tiles = num_tiles;
    G = static_cast<int>(gridDim.x);
    const int64_t U = static_cast<int64_t>(tiles) * KB;
    u = static_cast<int64_t>(blockIdx.x) * U / G;
    u1 = static_cast<int64_t>(blockIdx.x + 1) * U / G;
    next = static_cast<int>(blockIdx.x);
  }
  __device__ __forceinline__ bool get(int& tile, int& k0, int& k1) {
    if (split) {
      if (u >= u1) return false;
      tile = static_cast<int>(u / KB);
      k0 = static_cast<int>(u - static_cast<int64_t>(tile) * KB);
      const int64_t left = u1 - u;
      k1 = (KB - k0) < left ? KB : k0 + static_cast<int>(left);
      u += k1 - k0;
      return true;
    }
    if (next >= tiles) return false;
    tile = next;
    k0 = 0;
    k1 = KB;
    next += G;
    return true;
  }
  // split form: the CTA holding unit x, and the first unit of CTA c
  __device__ __forceinline__ int cta_of(int64_t x) const {
    const int64_t U = static_cast<int64_t>(tiles) * KB;
    return static_cast<int>(((x + 1) * G - 1) / U);
  }
  __device__ __forceinline__ int64_t first_unit(int c) const {
    return static_cast<int64_t>(c) * (static_cast<int64_t>(tiles) * KB) / G;
  }
};

__device__ __forceinline__ void epi_named_barrier() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// One output value of the weight-streaming epilogue: token m, output channel n.
template <int EPI>
__device__ __forceinline__ void smallm_store(const GemmParams& p, void* out, int m, int n, int32_t acc, float xs,
                                             float sw, float swn, float bn) {
  if (EPI == kEpiDequantBf16) {
    const float y = fmaf(static_cast<float>(acc), xs * sw, bn);
    static_cast<__nv_bfloat16*>(out)[static_cast<int64_t>(m) * p.N + n] = __float2bfloat16_rn(y);
  } else if (epi_is_general(EPI)) {
    const int64_t at = static_cast<int64_t>(m) * (p.ldy ? p.ldy : p.N) + n;
    float bias_add = bn;
    if (p.addend != nullptr) bias_add += out16_to_f32(__ldg(p.addend + at), p.out_f16 != 0);
    float y = fmaf(static_cast<float>(acc), xs * swn, bias_add);
    if (EPI == kEpiDequantGenGelu) y = gelu_erf(y);
    if (p.out_f16)
      static_cast<__half*>(out)[at] = __float2half_rn(y);
    else
      static_cast<__nv_bfloat16*>(out)[at] = __float2bfloat16_rn(y);
  } else {
    static_cast<int32_t*>(out)[static_cast<int64_t>(m) * p.N + n] = acc;
  }
}

// Fused form: the rotation and quantisation of the M <= 16 tokens by the
// kSmallQuantThreads threads of warps 2.. (qt = their index), straight from
// X in global memory into the shared-memory B operand: code k of token m at
// codes + (k / 128) * BNT * 128 + m * 128 + (k % 128), its 16-byte chunk
// swizzled by m % 8 (the layout a 128-byte-swizzled TMA box of BNT rows
// gives), the token scales into xs. The arithmetic and its order are those
// of the rotate+quantise kernel (pair stage on the top piece bit from the
// input words, the lane's own stages, the shuffle stages on the lane bits;
// absmax; the correctly rounded scale; code = rne(u * 127 / absmax_u)), so
// every code and scale equals that kernel's. Rows past M are not written:
// their MMA columns are never stored. With gcodes (CTA 0) the codes and
// scales also go to global memory ([M, K] row-major and [M]).
template <int G, int BNT>
__device__ __forceinline__ void smallm_quant(const GemmParams& p, uint8_t* codes, float* xs, unsigned* rmax2,
                                             int qt, int8_t* gcodes, float* gscale) {
  using namespace fwht;
  constexpr int LG = G / 64;
  constexpr int PIECE = G / 8;
  const int K = p.K;
  const int tpr = K / 64;                     // threads per token (64 values each)
  const int rpp = kSmallQuantThreads / tpr;   // tokens per pass (>= 2 for K <= 8192)
  const int row_in_pass = qt / tpr;
  const int t = qt - row_in_pass * tpr;
  const int grp = t / LG;
  const int l = t - grp * LG;
  const bool lane_active = row_in_pass < rpp;
  for (int pass = 0; pass * rpp < p.M; ++pass) {
    const int row = pass * rpp + row_in_pass;
    const bool valid = lane_active && row < p.M;
    unsigned* rmax = rmax2 + (pass & 1) * BNT;
    if (qt < BNT) rmax[qt] = 0u;
    float2 v[4][8];
    if (valid) {
      const uint16_t* src = p.X + static_cast<int64_t>(row) * K + grp * G + 8 * l;
      uint4 raw[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(raw[j].x), "=r"(raw[j].y), "=r"(raw[j].z), "=r"(raw[j].w)
                     : "l"(src + j * PIECE));
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const uint32_t aw[4] = {raw[jj].x, raw[jj].y, raw[jj].z, raw[jj].w};
        const uint32_t bw[4] = {raw[jj + 4].x, raw[jj + 4].y, raw[jj + 4].z, raw[jj + 4].w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          fwht_first_pair<false>(aw[q],
                                 make_float2(__uint_as_float(bw[q] << 16), __uint_as_float(bw[q] & 0xFFFF0000u)),
                                 v[jj][2 * q], v[jj][2 * q + 1]);
      }
    } else {
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int e = 0; e < 8; ++e) v[jj][e] = make_float2(0.0f, 0.0f);
    }
    fwht_lane_local(v);
    fwht_lane_shuffle<LG>(v, l);
    float m = absmax64_v3(v);
#pragma unroll
    for (int s = 1; s < LG; s <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, s));
    named_barrier_sync(2, kSmallQuantThreads);  // this pass's row maxima are zero
    if (valid && l == 0) atomicMax(&rmax[row_in_pass], __float_as_uint(m));
    named_barrier_sync(2, kSmallQuantThreads);
    if (valid) {
      const float amax_u = __uint_as_float(rmax[row_in_pass]);
      if (t == 0) {
        const float sc = scale_of<G>(amax_u);
        xs[row] = sc;
        if (gscale != nullptr) gscale[row] = sc;
      }
      const CodeFactor cf = code_factor(amax_u);
      if (cf.pre != 1.0f) {  // tiny row: multiply by 2^64 first (exact), then by ci
        const float2 pre2 = make_float2(cf.pre, cf.pre);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
#pragma unroll
          for (int e = 0; e < 8; ++e) v[jj][e] = __fmul2_rn(v[jj][e], pre2);
      }
      const float2 ci2 = make_float2(cf.ci, cf.ci);
      const float2 magic2 = make_float2(kRoundMagic, kRoundMagic);
      uint8_t* const row_base = codes + row * BK;
      const int sw = row & 7;
      auto put8 = [&](int k, uint2 val) {  // 8 codes at columns k..k+7 (k % 8 == 0)
        const int j = k & (BK - 1);
        *reinterpret_cast<uint2*>(row_base + (k / BK) * (BNT * BK) + ((((j >> 4) ^ sw) << 4) | (j & 15))) = val;
      };
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        float2 r[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = __ffma2_rn(v[jj][e], ci2, magic2);
        // piece jj from the .x halves, piece jj+4 from the .y halves
        uint2 lo, hi;
        lo.x = pack4(r[0].x, r[1].x, r[2].x, r[3].x);
        lo.y = pack4(r[4].x, r[5].x, r[6].x, r[7].x);
        hi.x = pack4(r[0].y, r[1].y, r[2].y, r[3].y);
        hi.y = pack4(r[4].y, r[5].y, r[6].y, r[7].y);
        const int k = grp * G + jj * PIECE + 8 * l;
        put8(k, lo);
        put8(k + 4 * PIECE, hi);
        if (gcodes != nullptr) {
          int8_t* g8 = gcodes + static_cast<int64_t>(row) * K + k;
          *reinterpret_cast<uint2*>(g8) = lo;
          *reinterpret_cast<uint2*>(g8 + 4 * PIECE) = hi;
        }
      }
    }
  }
  // the codes are read by the tensor cores (async proxy)
  fence_proxy_async_smem();
  named_barrier_sync(2, kSmallQuantThreads);
}

template <int EPI, int BNT, int KPS, int QG = 0>
__global__ void __launch_bounds__(QG != 0 ? NUM_THREADS + 32 * kSmallQuantWarps : NUM_THREADS, 1)
    gemm_i8_smallm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                          void* __restrict__ out, const int8_t* __restrict__ Wq, const GemmParams p) {
  constexpr bool FQ = QG != 0;  // fused form: the kernel quantises the tokens itself
  using L = SmallSmem<BNT, KPS, FQ>;
  const int R = p.tile_rows;  // weight rows per tile
  const int S = L::stages(R, p.K);
  const int kW1 = R * BK;  // one weight box
  const int kW = kW1 * KPS;
  const int off_w = L::kHeader + L::codes_bytes(p.K);
  const int off_x = off_w + S * kW;
  constexpr int kMaxS = L::kMaxStages;
  constexpr uint32_t kIdesc = idesc_i8(SM_BW, BNT);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tmem_full = bars + 2 * S;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* drain = tmem_empty + 2;
  uint64_t* x_ready = drain + 1;  // fused form: the token codes are in shared memory
  uint8_t* const codes = smem + L::kHeader;
  float* const xs_s = reinterpret_cast<float*>(smem + L::kOffXs);
  unsigned* const rmax_s = reinterpret_cast<unsigned*>(smem + L::kOffRmax);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + L::kOffTmemPtr);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::kOffLast);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = (p.N + R - 1) / R;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], EPI_WARPS);
    }
    mbar_init(drain, 1);
    mbar_init(x_ready, 1);
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
  // The weight stream does not depend on the previous kernel (see the pair
  // kernel): the weight loads of the first S stages go out before the wait,
  // the activation-code loads and the token scales after it. The fused form
  // loads no tokens: its producer never waits. Either form lets the next
  // kernel launch once every load of this CTA is out (letting it launch after
  // the first stages instead measured 0.7 us slower per call at M = 1).

  if (warp == 0) {
    if (lane == 0) {
      SmallSegments seg(p, num_tiles);
      int s = 0;
      uint32_t ph = 0;
      int pending_phase[kMaxS];
      for (int i = 0; i < S; ++i) pending_phase[i] = -1;
      bool ok = true;
      int early_s[kMaxS], early_kb[kMaxS];
      int n_early = 0;
      bool waited = FQ;
      int issued = 0;
      bool prefetched = !(CONVROT_SMALLM_PANEL_PREFETCH && !seg.split &&
                          static_cast<int64_t>(p.N) * p.K <= (int64_t(64) << 20));
      auto prefetch_panels = [&]() {
        // this CTA's tiles (each R contiguous weight rows) into L2
        for (int t = static_cast<int>(blockIdx.x); t < num_tiles; t += static_cast<int>(gridDim.x)) {
          const int64_t r0 = static_cast<int64_t>(t) * R;
          const int64_t r1 = r0 + R < p.N ? r0 + R : p.N;
          const uint8_t* base = reinterpret_cast<const uint8_t*>(Wq) + r0 * p.K;
          const int64_t bytes = (r1 - r0) * p.K;
          for (int64_t off = 0; off < bytes; off += kSmallPanelChunk)
            bulk_prefetch_l2(base + off, static_cast<uint32_t>(bytes - off < kSmallPanelChunk ? bytes - off
                                                                                             : kSmallPanelChunk));
        }
        prefetched = true;
      };
      auto load_x = [&](int st, int kb) {
#pragma unroll
        for (int i = 0; i < KPS; ++i)
          tma_load_2d(smem + off_x + st * L::kX + i * L::kX1, &tmX, &full[st], (kb + i) * BK, 0);
      };
      auto release_early = [&]() {
        griddep_wait();
        waited = true;
        for (int i = 0; i < n_early; ++i) load_x(early_s[i], early_kb[i]);
      };
      int tile, k0, k1;
      while (ok && seg.get(tile, k0, k1)) {
        // KPS k-blocks per stage (blocks past K arrive as zeros: whole tiles only when KPS > 1)
        for (int kb = k0; kb < k1; kb += KPS) {
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kW + L::kX));
#pragma unroll
          for (int i = 0; i < KPS; ++i)
            tma_load_2d(smem + off_w + s * kW + i * kW1, &tmW, &full[s], (kb + i) * BK, tile * R);
          if (FQ) {
          } else if (waited) {
            load_x(s, kb);
          } else {
            early_s[n_early] = s;
            early_kb[n_early] = kb;
            if (++n_early == S) release_early();
          }
          pending_phase[s] = static_cast<int>(ph);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
          if (!prefetched && ++issued == S) prefetch_panels();
        }
      }
      if (!waited) release_early();
      if (!prefetched && ok) prefetch_panels();
      griddep_launch_dependents();
      if (!ok) {
        raise_abort(abort, p.status);
        for (int i = 0; i < S; ++i)
          if (pending_phase[i] >= 0)
            mbar_wait_bounded(&full[i], static_cast<uint32_t>(pending_phase[i]), nullptr, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      SmallSegments seg(p, num_tiles);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      bool x_in = !FQ;  // fused form: the token codes are in shared memory
      int it = 0;
      int tile, k0, k1;
      while (ok && seg.get(tile, k0, k1)) {
        const int b = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait_bounded(&tmem_empty[b], (use & 1u) ^ 1u, abort, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(b * 128);
        for (int kb = k0; kb < k1; kb += KPS) {
          if (!mbar_wait_bounded(&full[s], ph, abort, p.timeout_ns)) {
            ok = false;
            break;
          }
          if (!x_in) {
            if (!mbar_wait_bounded(x_ready, 0u, abort, p.timeout_ns)) {
              ok = false;
              break;
            }
            x_in = true;
          }
          tc_fence_after();
#pragma unroll
          for (int i = 0; i < KPS; ++i) {
            if (FQ && kb + i >= p.num_k_blocks) break;  // no codes past K (the weight box there is zeros)
            const uint32_t w_base = smem_addr(smem + off_w + s * kW + i * kW1);
            const uint32_t x_base = FQ ? smem_addr(codes + (kb + i) * L::kX1)
                                       : smem_addr(smem + off_x + s * L::kX + i * L::kX1);
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              mma_i8(d, smem_desc_k_sw128(w_base + k * UMMA_K), smem_desc_k_sw128(x_base + k * UMMA_K), kIdesc,
                     (kb > k0 || i > 0 || k > 0) ? 1u : 0u);
            }
          }
          mma_commit(&empty[s]);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tmem_full[b]);
        ++it;
      }
      if (!ok) raise_abort(abort, p.status);
      mma_commit(drain);
      mbar_wait_bounded(drain, 0u, nullptr, p.timeout_ns);
    }
  } else {
    if constexpr (FQ) {
      // warps 2..: wait for the previous kernel (X may be its output; this
      // call's status word and output may still be read by it), clear the
      // status word (CTA 0), rotate and quantise the tokens
      griddep_wait();
      if (blockIdx.x == 0 && threadIdx.x == 64 && p.status != nullptr) *p.status = 0;
      const bool keep = blockIdx.x == 0 && p.Xq != nullptr && p.x_scale_out != nullptr;
      smallm_quant<QG, BNT>(p, codes, xs_s, rmax_s, static_cast<int>(threadIdx.x) - 64, keep ? p.Xq : nullptr,
                            keep ? p.x_scale_out : nullptr);
      if (threadIdx.x == 64) mbar_arrive(x_ready);
    } else {
      griddep_wait();  // the token scales (and the split counters' zeroing) come from the previous kernel
    }
  }
  if (warp >= 2 && warp < 2 + EPI_WARPS) {
    SmallSegments seg(p, num_tiles);
    const int q = warp & 3;
    const int nl = q * 32 + lane;  // weight row within the tile (TMEM lane)
    const bool row_ok = nl < R;    // lanes past the tile's rows hold no output
    const float sw = epi_weight_scale<EPI>(p);
    int it = 0;
    int si = 0;  // segment index within this CTA
    bool ok = true;
    int tile, k0, k1;
    while (seg.get(tile, k0, k1)) {
      const int b = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      const int n = row_ok ? tile * R + nl : p.N;
      const bool whole = (k0 == 0 && k1 == seg.KB);
      float bn = 0.0f;
      float swn = sw;  // this thread's output channel's weight scale
      if (epi_is_dequant(EPI) && n < p.N) {
        if (p.bias != nullptr) bn = out16_to_f32(__ldg(p.bias + n), epi_is_general(EPI) && p.out_f16 != 0);
        if (epi_is_general(EPI) && p.wscale_per_channel) swn = __ldg(p.w_scale + n);
      }
      if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&tmem_full[b], use & 1u, abort, p.timeout_ns));
      // the accumulators of this segment: token m of weight row n in acc[m]
      int32_t acc[BNT];
#pragma unroll
      for (int m = 0; m < BNT; ++m) acc[m] = 0;
      if (ok) {
        tc_fence_after();
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * 128);
#pragma unroll
        for (int c = 0; c < BNT / 16; ++c) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(t_row + static_cast<uint32_t>(c * 16), r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[c * 16 + j] = static_cast<int32_t>(r[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tmem_empty[b]);
      }
      bool write_out = whole;
      if (!whole) {
        // split form, part of a tile: this CTA's partial to its slot (slot 0:
        // its first segment, 1: its last), counted in at the tile's counter
        int32_t* part = p.split_part + static_cast<int64_t>(2 * blockIdx.x + (si == 0 ? 0 : 1)) * BNT * 128;
        if (ok) {
#pragma unroll
          for (int m = 0; m < BNT; ++m) part[m * 128 + nl] = acc[m];
        }
        __threadfence();
        epi_named_barrier();  // every epilogue thread's partial is stored (all four warps, also after a timeout)
        if (threadIdx.x == 64) {
          const int c_first = seg.cta_of(static_cast<int64_t>(tile) * seg.KB);
          const int c_last = seg.cta_of(static_cast<int64_t>(tile) * seg.KB + seg.KB - 1);
          const unsigned prev = atomicAdd(p.split_count + tile, 1u);
          *last_flag = (prev == static_cast<unsigned>(c_last - c_first)) ? 1 : 0;
        }
        epi_named_barrier();
        write_out = *last_flag != 0;
        if (write_out && ok) {
          __threadfence();
          // add the other contributors' partials (read through L2)
          const int c_first = seg.cta_of(static_cast<int64_t>(tile) * seg.KB);
          const int c_last = seg.cta_of(static_cast<int64_t>(tile) * seg.KB + seg.KB - 1);
          for (int c = c_first; c <= c_last; ++c) {
            if (c == static_cast<int>(blockIdx.x)) continue;
            const int slot = 2 * c + ((seg.first_unit(c) / seg.KB) == tile ? 0 : 1);
            const int32_t* op = p.split_part + static_cast<int64_t>(slot) * BNT * 128;
#pragma unroll
            for (int m = 0; m < BNT; ++m) acc[m] += __ldcg(op + m * 128 + nl);
          }
        }
      }
      if (write_out && ok && n < p.N) {
#pragma unroll
        for (int m = 0; m < BNT; ++m)
          if (m < p.M) smallm_store<EPI>(p, out, m, n, acc[m], FQ ? xs_s[m] : __ldg(p.x_scale + m), sw, swn, bn);
      }
      ++it;
      ++si;
    }
    if (!ok && lane == 0) raise_abort(abort, p.status);
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

// -------------------------------------------------------------------- host

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// A 2-D tiled tensor map; row_elems = distance between rows in elements (0 = inner).
bool encode_2d(CUtensorMap* tm, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
               uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz,
               uint64_t row_elems = 0) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {(row_elems ? row_elems : inner) * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;

// SM count of the current device, looked up once per device.
int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < kMaxDevices) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// cudaFuncSetAttribute(max dynamic shared memory) once per device and kernel.
template <class Kernel>
cudaError_t ensure_smem_attr(Kernel kern, int bytes, std::atomic<int>* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(bytes, std::memory_order_release);
  return e;
}

template <int EPI, int FG>
cudaError_t launch_impl(const int8_t* A, const int8_t* B, void* out, GemmParams p, cudaStream_t stream) {
  CUtensorMap ta, tb, to;
  if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, p.K, p.M, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, p.K, p.N, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  bool ok_out;
  if (epi_is_dequant(EPI))
    ok_out = encode_2d(&to, (epi_is_general(EPI) && p.out_f16) ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                       2, out, p.N, p.M, CHUNK, 32, CU_TENSOR_MAP_SWIZZLE_64B, static_cast<uint64_t>(p.ldy));
  else
    ok_out = encode_2d(&to, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, out, p.N, p.M, CHUNK, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok_out) return cudaErrorInvalidValue;

  p.num_m_blocks = (p.M + BM - 1) / BM;
  p.num_n_blocks = (p.N + BN - 1) / BN;
  p.num_k_blocks = (p.K + BK - 1) / BK;
  if (p.group_m <= 0) p.group_m = FG ? 4 : 16;
  int threads = NUM_THREADS;
  if (FG != 0) {
    if (!fused_shape(p.K, &p.q_threads_per_row, &p.q_rows_per_pass, &threads)) return cudaErrorInvalidValue;
  }
  const int tiles = p.num_m_blocks * p.num_n_blocks;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = tiles < sms ? tiles : sms;
  constexpr int smem = Smem<EPI>::kAlloc;
  static std::atomic<int> attr_done[kMaxDevices];
  cudaError_t e = ensure_smem_attr(gemm_i8_kernel<EPI, FG>, smem, attr_done);
  if (e != cudaSuccess) return e;
  if (FG != 0) {
    // the fused form's CTAs wait for one another's quantised blocks: the whole
    // grid (one CTA per SM) must fit on the device at once
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemm_i8_kernel<EPI, FG>, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1 || static_cast<int64_t>(per_sm) * sms < grid) return cudaErrorNotSupported;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_i8_kernel<EPI, FG>, ta, tb, to, p);
}

}  // namespace

bool fused_shape(int64_t K, int* threads_per_row, int* rows_per_pass, int* cta_threads) {
  if (K <= 0 || K % 128 != 0) return false;
  const int64_t tpr = K / 64;
  if (tpr > 32 * (kFusedMaxThreads - NUM_THREADS) / 32) return false;
  int64_t rpp = 256 / tpr;
  if (rpp < 1) rpp = 1;
  if (rpp > kMaxFusedRows) rpp = kMaxFusedRows;
  const int64_t workers = (rpp * tpr + 31) / 32 * 32;
  if (NUM_THREADS + workers > kFusedMaxThreads) return false;
  *threads_per_row = static_cast<int>(tpr);
  *rows_per_pass = static_cast<int>(rpp);
  *cta_threads = static_cast<int>(NUM_THREADS + workers);
  return true;
}

namespace {

template <int EPI>
cudaError_t launch_pair(const int8_t* A, const int8_t* B, void* out, GemmParams p, cudaStream_t stream) {
  CUtensorMap ta, tb, to;
  if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, p.K, p.M, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, p.K, p.N, BK, BN_HALF, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  bool ok_out;
  if (epi_is_dequant(EPI))
    ok_out = encode_2d(&to, (epi_is_general(EPI) && p.out_f16) ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                       2, out, p.N, p.M, CHUNK, 32, CU_TENSOR_MAP_SWIZZLE_64B, static_cast<uint64_t>(p.ldy));
  else
    ok_out = encode_2d(&to, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, out, p.N, p.M, CHUNK, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok_out) return cudaErrorInvalidValue;
  p.num_m_blocks = (p.M + 2 * BM - 1) / (2 * BM);  // 256-row pair blocks
  p.num_n_blocks = (p.N + BN - 1) / BN;
  p.num_k_blocks = (p.K + BK - 1) / BK;
  // Tile order by what stays in L2 for the whole launch. Activation codes of at
  // most 32 MiB: one group over every pair-row (N outside), so the codes stay and
  // each weight panel is read from DRAM once (1.8-2.9 % faster on the 4608-token
  // K = 3072 layers than groups of 16). Else a weight of at most 40 MiB: groups
  // of one pair-row (N inside), so the weight stays and each pair-row of codes is
  // read once (1.5-4.5 % faster on the 2048² MLP and the down projection). Else
  // groups of 16 pair-rows.
  if (p.group_m <= 0) {
    const int64_t a_bytes = static_cast<int64_t>(p.M) * p.K, b_bytes = static_cast<int64_t>(p.N) * p.K;
    p.group_m = a_bytes <= (int64_t(32) << 20)   ? p.num_m_blocks
                : b_bytes <= (int64_t(40) << 20) ? 1
                                                  : CONVROT_PAIR_GROUP_M;
  }
  const int tiles = p.num_m_blocks * p.num_n_blocks;
  const int sms = sm_count();
  if (sms < 2) return cudaErrorInvalidDevice;
  const int pairs = tiles < sms / 2 ? tiles : sms / 2;
  constexpr int smem = PairSmem<EPI>::kAlloc;
  static std::atomic<int> attr_done[kMaxDevices];
  cudaError_t e = ensure_smem_attr(gemm_i8_pair_kernel<EPI>, smem, attr_done);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(PAIR_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_i8_pair_kernel<EPI>, ta, tb, to, p);
}

}  // namespace

namespace {

// Weight rows per tile of the weight-streaming form: whole tiles take the
// fewest rows (a multiple of 8) that cover the N rows with one tile per SM;
// the split form keeps 128-row tiles.
int smallm_tile_rows(int N, int sms, bool split) {
  if (!CONVROT_SMALLM_FIT_ROWS || split) return SM_BW;
  const int per_sm = (N + sms - 1) / sms;
  const int rows = (per_sm + 7) / 8 * 8;
  return rows < SM_BW ? rows : SM_BW;
}

template <int EPI, int BNT, int KPS>
cudaError_t launch_smallm_t(const int8_t* A, const int8_t* B, void* out, GemmParams p, cudaStream_t stream) {
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  p.tile_rows = smallm_tile_rows(p.N, sms, p.split_part != nullptr);
  CUtensorMap tw, tx;
  if (!encode_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, p.K, p.N, BK, p.tile_rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, p.K, p.M, BK, BNT, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  p.num_k_blocks = (p.K + BK - 1) / BK;
  const int tiles = (p.N + p.tile_rows - 1) / p.tile_rows;
  int grid = tiles < sms ? tiles : sms;
  if (p.split_part != nullptr) {
    // every SM streams an equal share of the (tile, k-block) units
    if (tiles > kMaxSplitTiles || BNT != smallm_bnt(p.M)) return cudaErrorInvalidValue;
    const int64_t units = static_cast<int64_t>(tiles) * p.num_k_blocks;
    const int cap = sms < kMaxSplitCtas ? sms : kMaxSplitCtas;
    grid = static_cast<int>(units < cap ? units : cap);
  }
  constexpr int smem = SmallSmem<BNT, KPS>::kAlloc;
  static std::atomic<int> attr_done[kMaxDevices];
  cudaError_t e = ensure_smem_attr(gemm_i8_smallm_kernel<EPI, BNT, KPS>, smem, attr_done);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_i8_smallm_kernel<EPI, BNT, KPS>, tw, tx, out, B, p);
}

// The fused weight-streaming form (M <= kSmallQuantM): one kernel that
// rotates and quantises the tokens (group size G) and multiplies them with
// the weight; whole tiles only.
template <int EPI, int G>
cudaError_t launch_smallm_fq(const int8_t* B, void* out, GemmParams p, cudaStream_t stream) {
  constexpr int BNT = 16, KPS = CONVROT_SMALLM_KPS;
  using L = SmallSmem<BNT, KPS, true>;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  p.split_part = nullptr;
  p.tile_rows = smallm_tile_rows(p.N, sms, false);
  if (p.X == nullptr || p.M < 1 || p.M > kSmallQuantM || p.K > kSmallQuantMaxK || L::stages(p.tile_rows, p.K) < 2)
    return cudaErrorInvalidValue;
  CUtensorMap tw;
  if (!encode_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, p.K, p.N, BK, p.tile_rows, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  p.num_k_blocks = (p.K + BK - 1) / BK;
  const int tiles = (p.N + p.tile_rows - 1) / p.tile_rows;
  const int grid = tiles < sms ? tiles : sms;
  constexpr int smem = L::kAlloc;
  static std::atomic<int> attr_done[kMaxDevices];
  cudaError_t e = ensure_smem_attr(gemm_i8_smallm_kernel<EPI, BNT, KPS, G>, smem, attr_done);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(NUM_THREADS + 32 * kSmallQuantWarps);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_i8_smallm_kernel<EPI, BNT, KPS, G>, tw, tw, out, B, p);
}

template <int EPI, int KPS>
cudaError_t launch_smallm_k(const int8_t* A, const int8_t* B, void* out, GemmParams p, cudaStream_t stream) {
  if (p.M <= 16) return launch_smallm_t<EPI, 16, KPS>(A, B, out, p, stream);
  if (p.M <= 32) return launch_smallm_t<EPI, 32, KPS>(A, B, out, p, stream);
  return launch_smallm_t<EPI, 64, KPS>(A, B, out, p, stream);
}

template <int EPI>
cudaError_t launch_smallm(const int8_t* A, const int8_t* B, void* out, GemmParams p, cudaStream_t stream) {
  // several k-blocks per stage only for whole tiles (the split form walks single k-blocks)
  if (p.split_part == nullptr && CONVROT_SMALLM_KPS > 1)
    return launch_smallm_k<EPI, CONVROT_SMALLM_KPS>(A, B, out, p, stream);
  return launch_smallm_k<EPI, 1>(A, B, out, p, stream);
}

}  // namespace

cudaError_t launch_gemm_i8(int epi, const int8_t* A, const int8_t* B, void* out, GemmParams p,
                           cudaStream_t stream) {
  if (p.M <= kSmallM) {
    if (epi == kEpiDequantBf16) return launch_smallm<kEpiDequantBf16>(A, B, out, p, stream);
    if (epi == kEpiDequantGen) return launch_smallm<kEpiDequantGen>(A, B, out, p, stream);
    if (epi == kEpiDequantGenGelu) return launch_smallm<kEpiDequantGenGelu>(A, B, out, p, stream);
    if (epi == kEpiRawS32) return launch_smallm<kEpiRawS32>(A, B, out, p, stream);
    return cudaErrorInvalidValue;
  }
  if (epi == kEpiDequantBf16) return launch_pair<kEpiDequantBf16>(A, B, out, p, stream);
  if (epi == kEpiDequantGen) return launch_pair<kEpiDequantGen>(A, B, out, p, stream);
  if (epi == kEpiDequantGenGelu) return launch_pair<kEpiDequantGenGelu>(A, B, out, p, stream);
  if (epi == kEpiRawS32) return launch_pair<kEpiRawS32>(A, B, out, p, stream);
  return cudaErrorInvalidValue;
}

bool smallm_fused_shape(int64_t M, int64_t K) {
  using L = SmallSmem<16, CONVROT_SMALLM_KPS, true>;
  return CONVROT_SMALLM_FUSED && M >= 1 && M <= kSmallQuantM && K >= BK && K <= kSmallQuantMaxK &&
         M * K <= int64_t(kSmallQuantThreads) * 64 && L::stages(SM_BW, static_cast<int>(K)) >= 2;
}

cudaError_t launch_linear_smallm_fused(int epi, int g, const int8_t* Wq, void* Y, GemmParams p,
                                       cudaStream_t stream) {
  if (g == 128) {
    if (epi == kEpiDequantBf16) return launch_smallm_fq<kEpiDequantBf16, 128>(Wq, Y, p, stream);
    if (epi == kEpiDequantGen) return launch_smallm_fq<kEpiDequantGen, 128>(Wq, Y, p, stream);
    if (epi == kEpiDequantGenGelu) return launch_smallm_fq<kEpiDequantGenGelu, 128>(Wq, Y, p, stream);
  } else if (g == 256) {
    if (epi == kEpiDequantBf16) return launch_smallm_fq<kEpiDequantBf16, 256>(Wq, Y, p, stream);
    if (epi == kEpiDequantGen) return launch_smallm_fq<kEpiDequantGen, 256>(Wq, Y, p, stream);
    if (epi == kEpiDequantGenGelu) return launch_smallm_fq<kEpiDequantGenGelu, 256>(Wq, Y, p, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_linear_fused(int g, const int8_t* Wq, void* Y, GemmParams p, cudaStream_t stream) {
  if (g == 256) return launch_impl<kEpiDequantBf16, 256>(p.Xq, Wq, Y, p, stream);
  if (g == 128) return launch_impl<kEpiDequantBf16, 128>(p.Xq, Wq, Y, p, stream);
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------- bounded-wait probe

__global__ void wait_timeout_kernel(int* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing arrives on this barrier: the wait must give up by itself
    if (!mbar_wait_bounded(&bar, 0u, &abort, timeout_ns)) atomicOr(status, kTimeoutStatus);
  }
}

cudaError_t launch_wait_timeout(int* status, uint64_t timeout_ns, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace convrot
