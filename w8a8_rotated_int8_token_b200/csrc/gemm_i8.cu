// int8 x int8 -> int32 GEMM on the 5th-generation tensor cores (tcgen05,
// kind::i8) with a fused epilogue, for Y = Xq Wq^T: both operands K-major.
//
// The int8-by-int8 product with int32 accumulation is the multiply step of
// the ConvRot layer (InvokeAI "int8 Compute", second paragraph); the
// epilogue applies the token and tensor scales and the bias and rounds to
// bf16 (or, for exactness tests, stores the raw int32 accumulators).
//
// Structure: a persistent kernel, one CTA per SM, 6 warps.
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
// Tiles are visited in groups of `group_m` M-blocks so that the CTAs in flight
// share A and B panels in L2. Every wait is bounded; a wait that runs out
// records CONVROT_ERR_DEVICE_TIMEOUT (5) in the status word, every role
// unwinds, in-flight copies and MMAs are drained (bounded), TMEM is freed, and
// the CTA returns.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cstdint>

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

template <int EPI>
struct Smem {
  static constexpr int kEpiBuf = (EPI == kEpiDequantBf16) ? CHUNK * CHUNK * 2 : CHUNK * CHUNK * 4;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = STAGES * A_STAGE_BYTES;
  static constexpr int kOffEpi = STAGES * (A_STAGE_BYTES + B_STAGE_BYTES);
  static constexpr int kOffBar = kOffEpi + EPI_WARPS * 2 * kEpiBuf;
  static constexpr int kNumBars = 2 * STAGES + 2 + 2 + 1;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 8;
  static constexpr int kBytes = kOffAbort + 8;
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

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
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
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const float sw = (EPI == kEpiDequantBf16) ? __ldg(p.w_scale) : 0.0f;
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
      if (EPI == kEpiDequantBf16) sc = (row < p.M ? __ldg(p.x_scale + row) : 0.0f) * sw;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * BN);
#pragma unroll 1
      for (int c = 0; c < BN / CHUNK; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * CHUNK), r);
        tmem_ld_wait();
        if (c == BN / CHUNK - 1) {  // accumulator fully read: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tmem_empty[b]);
        }
        const int n0 = nb * BN + c * CHUNK;
        if (n0 >= p.N) continue;
        uint8_t* ebuf = ebuf0 + (chunk_count & 1) * L::kEpiBuf;
        if (lane == 0) bulk_wait_group_read<1>();  // the store that last read this buffer is done
        __syncwarp();
        if (EPI == kEpiDequantBf16) {
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
          for (int e = 0; e < 16; ++e) {
            const float y0 = fmaf(static_cast<float>(static_cast<int32_t>(r[2 * e])), sc, bv[2 * e]);
            const float y1 = fmaf(static_cast<float>(static_cast<int32_t>(r[2 * e + 1])), sc, bv[2 * e + 1]);
            packed[e] = bf16x2(y0, y1);
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
          tma_store_2d(&tmOut, ebuf, n0, row0);
          bulk_commit_group();
        }
        ++chunk_count;
      }
    }
    if (!ok && lane == 0) raise_abort(abort, p.status);
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
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

bool encode_2d(CUtensorMap* tm, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
               uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <int EPI>
cudaError_t launch_impl(const int8_t* A, const int8_t* B, void* out, GemmParams p, cudaStream_t stream) {
  CUtensorMap ta, tb, to;
  if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, p.K, p.M, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, p.K, p.N, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  bool ok_out;
  if (EPI == kEpiDequantBf16)
    ok_out = encode_2d(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, p.N, p.M, CHUNK, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  else
    ok_out = encode_2d(&to, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, out, p.N, p.M, CHUNK, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok_out) return cudaErrorInvalidValue;

  p.num_m_blocks = (p.M + BM - 1) / BM;
  p.num_n_blocks = (p.N + BN - 1) / BN;
  p.num_k_blocks = (p.K + BK - 1) / BK;
  if (p.group_m <= 0) p.group_m = 16;
  const int tiles = p.num_m_blocks * p.num_n_blocks;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = tiles < sms ? tiles : sms;
  constexpr int smem = Smem<EPI>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(gemm_i8_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gemm_i8_kernel<EPI><<<grid, NUM_THREADS, smem, stream>>>(ta, tb, to, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_i8(int epi, const int8_t* A, const int8_t* B, void* out, GemmParams p,
                           cudaStream_t stream) {
  if (epi == kEpiDequantBf16) return launch_impl<kEpiDequantBf16>(A, B, out, p, stream);
  if (epi == kEpiRawS32) return launch_impl<kEpiRawS32>(A, B, out, p, stream);
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
