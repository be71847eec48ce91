// Rotation + int8 quantisation kernels: one pass over a bf16 matrix whose rows
// are rotated group by group with the normalised Walsh-Hadamard transform
// (X R with R = blockdiag(H_g/sqrt(g))) and quantised symmetrically to int8.
//
// Activations get one scale per token (row); the weight gets one scale for the
// whole tensor, found by a first pass over all rows (InvokeAI "int8 Compute"
// page: input rotated and quantised per token, weights int8_tensorwise).
//
// Thread layout. A token row of K elements is K/g groups. A group is owned by
// LG = g/64 consecutive lanes, 64 elements per lane: lane l of the group loads
// eight 16-byte pieces at group offsets j*(g/8) + 8*l (j = 0..7), so one warp
// load instruction reads LG*16 contiguous bytes per group, fully coalesced.
// The group index bits split as e (bits 0-2, inside a piece), l (log2 LG lane
// bits) and j (top three bits): six butterfly stages run in registers. For
// g = 128 the one stage on the lane bit uses shuffles. For g = 256 the lanes
// of a group transpose their values through shared memory so that the two
// lane bits come into registers (two more register stages); that costs one
// 16-byte store and one 16-byte load per four values instead of two shuffles
// per value.
//
// Arithmetic is packed: the 64 values live as 32 float2 pairs (piece j, piece
// j+4), so every butterfly stage except the one on j's top bit is one f32x2
// add or fma per two butterflies; that stage is done on scalars. The transform
// is computed unnormalised in float32 and 1/sqrt(g) is folded into the scale.
// A CTA handles `rpc` whole rows at a time (K/64 threads per row, about three
// warps) and loops over row blocks (persistent grid, several CTAs per SM);
// thread 0 streams the blocks into shared memory with bulk asynchronous
// copies, the next block in flight while the current one is computed. The row
// absmax is reduced in shared memory, with one CTA barrier per block.

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "fwht_dev.cuh"
#include "ptx_sm100.cuh"
#include "rotate_quant.cuh"

namespace convrot {

using namespace fwht;


// bf16 (F16IN false) or IEEE fp16 (true) input words: two elements each,
// widened exactly to float32 (low half first).
template <bool F16IN>
__device__ __forceinline__ float2 widen2(uint32_t w) {
  if (F16IN) {
    __half2 h;
    *reinterpret_cast<uint32_t*>(&h) = w;
    return __half22float2(h);
  }
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

#ifndef CONVROT_RQ_MAXNREG
#define CONVROT_RQ_MAXNREG 112
#endif

// register cap: g = 128 keeps its lane-pair shuffles' operands live longer
template <int G>
constexpr int rq_maxnreg() { return G == 256 ? CONVROT_RQ_MAXNREG : 128; }

template <int G, int MODE, bool F16IN, int S>
__global__ void __maxnreg__(rq_maxnreg<G>()) rotate_quant_kernel(RotQuantParams p) {
  constexpr int LG = G / 64;
  constexpr int PIECE = G / 8;  // elements between consecutive pieces of a lane
  // S input slots of rows_per_cta x K bf16, each rounded up to whole 4 KB
  // warp regions (g = 256 reuses a warp's region for its exchange)
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ uint64_t full[S];
  __shared__ unsigned row_max[3][kMaxRowsPerCta];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int rpc = p.rows_per_cta;
  const int K = static_cast<int>(p.K);
  const int rows = static_cast<int>(p.rows);
  const int row_in_cta = tid / p.threads_per_row;  // >= rpc for the padding threads of the last warp
  const int t = tid - row_in_cta * p.threads_per_row;
  const int grp = t / LG;
  const int l = t - grp * LG;
  const bool lane_active = row_in_cta < rpc;
  // Group k reads its pieces in the order j ^ (k mod F), F = 2 (g=256) or 4
  // (g=128), so that the F groups sharing a 128-byte bank window hit
  // different banks. The transform then comes out with piece r multiplied by
  // (-1)^popcount(r & flip), which the quantisation multiplier undoes. The
  // flip never changes the top piece bit, so pieces jj and jj+4 still pair.
  constexpr int F = (G == 256) ? 2 : 4;
  const int flip = grp & (F - 1);
  const int nblocks = (rows + rpc - 1) / rpc;
  const uint32_t stage_bytes = rotquant_slot_bytes(rpc, p.K);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < rpc) row_max[0][tid] = 0u;
  __syncthreads();
  // The input may be the previous kernel's output: wait for it (launches are
  // programmatic), then let the next kernel start its prologue early.
  griddep_wait();
  if (MODE == kRqActivation && blockIdx.x == 0) {
    // words the next kernel of the call counts in (its split arrival counters),
    // and the call's status word: cleared before the next kernel may start
    if (p.zero_words != nullptr)
      for (int i = tid; i < p.zero_count; i += blockDim.x) p.zero_words[i] = 0u;
    if (p.status_reset != nullptr && tid == 0) *p.status_reset = 0;
    __threadfence();
    __syncthreads();
  }
  // A kernel that follows may read a weight before it waits for this one (the
  // GEMMs stream the weight from their start): the weight-quantising passes
  // therefore let it launch only when the codes are written (at exit).
  const bool late = MODE == kRqWeightQuant || p.late_trigger != 0;
  if (!late) griddep_launch_dependents();

  // The producer (thread 0) keeps S-1 row blocks of this CTA in flight: block
  // it+S-1 goes out as soon as block it has landed, into the slot that block
  // it-1 released at its barrier.
  int issued = 0;
  auto issue = [&](int it) {
    const int blk = static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
    if (blk >= nblocks) return;
    const int r0 = blk * rpc;
    const int nrows = (rows - r0) < rpc ? (rows - r0) : rpc;
    const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
    const uint32_t bytes = static_cast<uint32_t>(nrows) * row_bytes;
    const int slot = it % S;
    uint8_t* const dst = stage_mem + static_cast<size_t>(slot) * stage_bytes;
    mbar_arrive_expect_tx(&full[slot], bytes);
    if (p.ldx == 0 || p.ldx == p.K) {  // dense rows: one copy for the block
      bulk_load(dst, p.src + static_cast<int64_t>(r0) * K, bytes, &full[slot]);
    } else {  // strided rows: one copy per row, packed densely in the slot
      for (int r = 0; r < nrows; ++r)
        bulk_load(dst + r * row_bytes, p.src + static_cast<int64_t>(r0 + r) * p.ldx, row_bytes, &full[slot]);
    }
    issued = it + 1;
  };
  static_assert(S >= 2, "the block after the current one needs its own slot");
  if (tid == 0)
    for (int i = 0; i < S - 1; ++i) issue(i);

  // byte offset of the lane's first piece inside a slot (loop-invariant)
  const uint32_t lane_off = (static_cast<uint32_t>(row_in_cta) * static_cast<uint32_t>(K) +
                             static_cast<uint32_t>(grp * G + 8 * l)) * 2u;
  // the g = 256 exchange region of this warp inside a slot
  const uint32_t xoff = static_cast<uint32_t>(tid >> 5) * kX256RegionBytes;

  int it = 0;
  int slot = 0;
  uint32_t ph = 0;
  int rsel = 0;  // which of the three row-maximum buffers this block uses
  bool timed_out = false;
  for (int blk = blockIdx.x; blk < nblocks; blk += gridDim.x, ++it) {
    const int row = blk * rpc + row_in_cta;
    const bool valid = lane_active && row < rows;
    // Row maxima rotate over three buffers: this block's, the next block's
    // (cleared now, before this block's barrier), and the previous block's,
    // which slower threads may still be reading.
    const int rnext = (rsel == 2) ? 0 : rsel + 1;
    unsigned* rmax = row_max[rsel];
    if (tid < rpc) row_max[rnext][tid] = 0u;

    const bool ok = mbar_wait_bounded(&full[slot], ph, &abort_flag, p.timeout_ns);
    // the slot of block it+S-1 was released by the barrier of block it-1
    if (tid == 0 && ok) issue(it + S - 1);
    uint8_t* slot_mem = stage_mem + static_cast<size_t>(slot) * stage_bytes;
    // Every lane loads, also those of rows past the end or of padding
    // threads: their bytes lie inside the slot (stale but harmless) and only
    // their stores are skipped. The stage on the top piece bit is taken
    // straight from the input words.
    float2 v[4][8];
    {
      const uint8_t* src = slot_mem + lane_off;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const uint4 a = *reinterpret_cast<const uint4*>(src + ((jj ^ flip) * PIECE) * 2);
        const uint4 b = *reinterpret_cast<const uint4*>(src + (((jj + 4) ^ flip) * PIECE) * 2);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) fwht_first_pair<F16IN>(aw[q], widen2<F16IN>(bw[q]), v[jj][2 * q], v[jj][2 * q + 1]);
      }
    }
    if (++slot == S) {
      slot = 0;
      ph ^= 1u;
    }
    rsel = rnext;

    // the other stages; afterwards w holds the lane's values (layout per g below)
    float2 w[4][8];
    fwht_lane_local(v);
    if constexpr (G == 256) {
      fwht256_exchange(v, w, slot_mem + xoff, (tid & 31) >> 2, l);
      // the slot is refilled by an asynchronous copy after the barrier below
      fence_proxy_async_smem();
      fwht256_after_exchange(w);
    } else {
      fwht_lane_shuffle<LG>(v, l);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int e = 0; e < 8; ++e) w[jj][e] = v[jj][e];
    }
    float m = absmax64_v3(w);
#pragma unroll
    for (int s = 1; s < LG; s <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, s));
    // non-negative floats order like their bit patterns
    if (valid && l == 0) atomicMax(&rmax[row_in_cta], __float_as_uint(m));

    // every thread has its input in registers (the slot may be refilled) and
    // its row maximum posted; the CTA also agrees on a timed-out wait here
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      break;
    }

    if (MODE == kRqWeightAbsmax) {
      if (valid && t == 0) atomicMax(p.tensor_absmax, rmax[row_in_cta]);
      continue;
    }
    const float amax_u =
        (MODE == kRqActivation) ? __uint_as_float(rmax[row_in_cta]) : __uint_as_float(*p.tensor_absmax);
    // the stored scale, one correctly rounded division, by the one thread that stores it
    if (MODE == kRqActivation) {
      if (valid && t == 0) p.scale[row] = scale_of<G>(amax_u);
    } else {
      if (blk == 0 && tid == 0) *p.scale = scale_of<G>(amax_u);
    }
    if (!valid) continue;
    const CodeFactor cf = code_factor(amax_u);
    if (cf.pre != 1.0f) {  // tiny row: multiply by 2^64 first (exact), then by ci
      const float2 pre2 = make_float2(cf.pre, cf.pre);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int e = 0; e < 8; ++e) w[jj][e] = __fmul2_rn(w[jj][e], pre2);
    }
    const float2 magic2 = make_float2(kRoundMagic, kRoundMagic);
    int8_t* dst = p.dst + static_cast<int64_t>(row) * K + grp * G;
    if constexpr (G == 256) {
      // the lane holds elements 32*l + (0..31) (.x) and 128 + 32*l + (0..31)
      // (.y), in the order w[src][e] = element 8*src + e of the run; the
      // piece-order flip left them multiplied by (-1)^(flip & l)
      const float ci = (flip & l & 1) ? -cf.ci : cf.ci;
      const float2 ci2 = make_float2(ci, ci);
      uint32_t lo[8], hi[8];
#pragma unroll
      for (int src = 0; src < 4; ++src) {
        float2 r[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = __ffma2_rn(w[src][e], ci2, magic2);
        lo[2 * src] = pack4(r[0].x, r[1].x, r[2].x, r[3].x);
        lo[2 * src + 1] = pack4(r[4].x, r[5].x, r[6].x, r[7].x);
        hi[2 * src] = pack4(r[0].y, r[1].y, r[2].y, r[3].y);
        hi[2 * src + 1] = pack4(r[4].y, r[5].y, r[6].y, r[7].y);
      }
      int8_t* o = dst + 32 * l;
      *reinterpret_cast<uint4*>(o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(o + 16) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
      *reinterpret_cast<uint4*>(o + 128) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(o + 144) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
    } else {
      int8_t* d8 = dst + 8 * l;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float cij = (__popc(jj & flip) & 1) ? -cf.ci : cf.ci;
        const float2 ci2 = make_float2(cij, cij);
        float2 r[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = __ffma2_rn(w[jj][e], ci2, magic2);
        // piece jj from the .x halves, piece jj+4 from the .y halves
        uint2 lo, hi;
        lo.x = pack4(r[0].x, r[1].x, r[2].x, r[3].x);
        lo.y = pack4(r[4].x, r[5].x, r[6].x, r[7].x);
        hi.x = pack4(r[0].y, r[1].y, r[2].y, r[3].y);
        hi.y = pack4(r[4].y, r[5].y, r[6].y, r[7].y);
        *reinterpret_cast<uint2*>(d8 + jj * PIECE) = lo;
        *reinterpret_cast<uint2*>(d8 + (jj + 4) * PIECE) = hi;
      }
    }
  }
  if (late) __threadfence();  // the codes are visible before the implicit trigger at exit
  if (timed_out && tid == 0) {
    if (p.status != nullptr) atomicOr(p.status, kRqTimeoutStatus);
    // let the copies already issued land before the shared memory goes away
    for (int k = it; k < issued; ++k)
      mbar_wait_bounded(&full[k % S], static_cast<uint32_t>((k / S) & 1), nullptr, p.timeout_ns);
  }
}

// ------------------------------------------------------------------ launch

bool rotquant_shape(int64_t K, int* threads_per_row, int* rows_per_cta) {
  if (K <= 0 || K % 128 != 0 || K > 32768) return false;
  const int tpr = static_cast<int>(K / 64);
  int rpc = (96 + tpr / 2) / tpr;
  if (rpc < 1) rpc = 1;
  if (rpc > kMaxRowsPerCta) rpc = kMaxRowsPerCta;
  if ((rpc * tpr + 31) / 32 * 32 > kRotQuantMaxThreads) return false;
  *threads_per_row = tpr;
  *rows_per_cta = rpc;
  return true;
}

namespace {

template <int G, int MODE, bool F16IN, int S>
cudaError_t launch_typed(RotQuantParams p, cudaStream_t stream) {
  void (*kern)(RotQuantParams) = rotate_quant_kernel<G, MODE, F16IN, S>;
  const int threads = (p.rows_per_cta * p.threads_per_row + 31) / 32 * 32;
  const size_t smem = static_cast<size_t>(S) * rotquant_slot_bytes(p.rows_per_cta, p.K);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // per device and kernel: the largest dynamic shared memory set so far, and
  // the occupancy found for the last (threads, smem) shape
  constexpr int kDevs = 64;
  static std::atomic<int> smem_set[kDevs];
  static std::atomic<long long> occ_key[kDevs];
  static std::atomic<int> occ_val[kDevs];
  static std::atomic<int> sm_cache[kDevs];
  const bool cacheable = dev >= 0 && dev < kDevs;
  if (!cacheable || smem_set[dev].load(std::memory_order_acquire) < static_cast<int>(smem)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (cacheable) smem_set[dev].store(static_cast<int>(smem), std::memory_order_release);
  }
  const long long key = (static_cast<long long>(threads) << 32) | static_cast<long long>(smem);
  int per_sm = 0;
  if (cacheable && occ_key[dev].load(std::memory_order_acquire) == key) {
    per_sm = occ_val[dev].load(std::memory_order_relaxed);
  } else {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (e != cudaSuccess) return e;
    if (cacheable) {
      occ_val[dev].store(per_sm, std::memory_order_relaxed);
      occ_key[dev].store(key, std::memory_order_release);
    }
  }
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  int sms = cacheable ? sm_cache[dev].load(std::memory_order_relaxed) : 0;
  if (sms <= 0) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if (cacheable) sm_cache[dev].store(sms, std::memory_order_relaxed);
  }
  const int64_t nblocks = (p.rows + p.rows_per_cta - 1) / p.rows_per_cta;
  const int64_t grid = nblocks < static_cast<int64_t>(sms) * per_sm ? nblocks : static_cast<int64_t>(sms) * per_sm;
  // programmatic stream serialisation: the kernel waits for its predecessor
  // itself (griddepcontrol.wait), so its launch can overlap the predecessor's tail
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
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

template <int G, bool F16IN, int S>
cudaError_t launch_mode_s(int mode, RotQuantParams p, cudaStream_t stream) {
  if (mode == kRqActivation) return launch_typed<G, kRqActivation, F16IN, S>(p, stream);
  if (mode == kRqWeightAbsmax) return launch_typed<G, kRqWeightAbsmax, F16IN, S>(p, stream);
  return launch_typed<G, kRqWeightQuant, F16IN, S>(p, stream);
}

template <int G, bool F16IN>
cudaError_t launch_mode(int mode, RotQuantParams p, cudaStream_t stream) {
  if (p.K >= kRqDeepMinK) return launch_mode_s<G, F16IN, kRqStagesDeep>(mode, p, stream);
  return launch_mode_s<G, F16IN, kRqStages>(mode, p, stream);
}

cudaError_t launch_rotate_quant(int g, int mode, RotQuantParams p, cudaStream_t stream) {
  int tpr = 0, rpc = 0;
  if (!rotquant_shape(p.K, &tpr, &rpc)) return cudaErrorInvalidValue;
  p.threads_per_row = tpr;
  p.rows_per_cta = rpc;
  if (g == 256) return p.in_f16 ? launch_mode<256, true>(mode, p, stream) : launch_mode<256, false>(mode, p, stream);
  if (g == 128) return p.in_f16 ? launch_mode<128, true>(mode, p, stream) : launch_mode<128, false>(mode, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace convrot
