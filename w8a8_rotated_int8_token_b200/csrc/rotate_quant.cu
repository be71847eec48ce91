// Rotation + int8 quantisation kernels: one pass over a bf16 matrix whose rows
// are rotated group by group with the normalised Walsh-Hadamard transform
// (X R with R = blockdiag(H_g/sqrt(g))) and quantised symmetrically to int8.
//
// Activations get one scale per token (row); the weight gets one scale for the
// whole tensor, found by a first pass over all rows (InvokeAI "int8 Compute"
// page: input rotated and quantised per token, weights int8_tensorwise).
//
// Thread layout. A token row of K elements is K/g groups. A group of g
// elements is owned by LG = g/32 consecutive lanes, 32 elements per lane:
// lane l of the group loads four 16-byte pieces at group offsets
// j*(g/4) + 8*l (j = 0..3). With i = 64*j + 8*l + e (g = 256) the element
// index bits split as e (bits 0-2, inside one 16-byte piece), l (lane bits)
// and j (top two bits), so five butterfly stages run in registers and
// log2(LG) stages (3 for g=256, 2 for g=128) run across lanes with shuffles. Each warp
// load instruction covers LG*16-byte contiguous runs, fully coalesced.
// A CTA holds `rpc` whole rows (K/32 threads per row); the row absmax is
// reduced in shared memory. The transform is computed unnormalised in float32
// and the 1/sqrt(g) factor is folded into the scale.

#include <cuda_runtime.h>

#include <cstdint>

#include "rotate_quant.cuh"

namespace convrot {

namespace {

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + magic rounds x to an integer (ties to even)

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint4 load_streaming(const uint16_t* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Unnormalised Walsh-Hadamard transform of one group held as v[j][e] by the
// LG lanes of the group (see the file comment for the index split).
template <int G>
__device__ __forceinline__ void fwht_group(float (&v)[4][8], int l) {
  // bits 0..2: inside each 16-byte piece
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if ((e & h) == 0) {
          const float a = v[j][e], b = v[j][e + h];
          v[j][e] = a + b;
          v[j][e + h] = a - b;
        }
      }
    }
  }
  // top two bits: across the four pieces of this lane
#pragma unroll
  for (int h = 1; h < 4; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if ((j & h) == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float a = v[j][e], b = v[j + h][e];
          v[j][e] = a + b;
          v[j + h][e] = a - b;
        }
      }
    }
  }
  // middle bits: across the LG lanes of the group. The lower partner keeps
  // a + b, the upper one b_partner - own = a - b.
  constexpr int LG = G / 32;
#pragma unroll
  for (int m = 1; m < LG; m <<= 1) {
    const float sgn = (l & m) ? -1.0f : 1.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float p = __shfl_xor_sync(0xFFFFFFFFu, v[j][e], m);
        v[j][e] = fmaf(sgn, v[j][e], p);
      }
    }
  }
}

// The scale of a row (or tensor) from the absmax of its unnormalised
// transform, and the factor that maps an unnormalised value to code units.
struct QuantScale {
  float s;        // stored scale: float32(absmax(X R) / 127)
  float ci;       // code = rne(u * ci) for an unnormalised value u (after `pre`)
  float pre;      // 1, or 2^64 for rows whose scale is below 2^-100
};

template <int G>
__device__ __forceinline__ QuantScale make_scale(float amax_u) {
  // 1/sqrt(g) and 127*sqrt(g): exact for g = 256 (1/16 and 2032); nearest
  // floats for g = 128. The scale takes one rounding for g = 256:
  // s = absmax(X R)/127 = absmax_u / (127 sqrt(g)).
  const float cg = (G == 256) ? 0.0625f : 0.0883883461356163f;
  const float div = (G == 256) ? 2032.0f : 1436.8409423828125f;
  QuantScale q;
  q.s = amax_u / div;
  q.pre = 1.0f;
  if (q.s == 0.0f) {
    q.ci = 0.0f;
  } else if (q.s >= 0x1p-100f) {
    q.ci = cg * (1.0f / q.s);
  } else {  // tiny row: lift by 2^64 (exact) so that 1/s cannot overflow
    q.pre = 0x1p64f;
    q.ci = cg * (1.0f / (q.s * 0x1p64f));
  }
  return q;
}

__device__ __forceinline__ uint32_t pack4(float a, float b, float c, float d, float ci) {
  // low byte of (u*ci + magic) is the two's-complement int8 code of rne(u*ci)
  const uint32_t qa = __float_as_uint(fmaf(a, ci, kRoundMagic));
  const uint32_t qb = __float_as_uint(fmaf(b, ci, kRoundMagic));
  const uint32_t qc = __float_as_uint(fmaf(c, ci, kRoundMagic));
  const uint32_t qd = __float_as_uint(fmaf(d, ci, kRoundMagic));
  const uint32_t ab = __byte_perm(qa, qb, 0x0040);
  const uint32_t cd = __byte_perm(qc, qd, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

}  // namespace

template <int G, int MODE>
__global__ void __launch_bounds__(1024) rotate_quant_kernel(RotQuantParams p) {
  constexpr int LG = G / 32;
  __shared__ unsigned row_max[kMaxRowsPerCta];

  const int tid = threadIdx.x;
  const int row_in_cta = tid / p.threads_per_row;
  const int t = tid - row_in_cta * p.threads_per_row;
  const int grp = t / LG;
  const int l = t - grp * LG;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * p.rows_per_cta + row_in_cta;
  const bool valid = row < p.rows;

  if (tid < p.rows_per_cta) row_max[tid] = 0u;
  if (MODE == kRqActivation && p.status_reset != nullptr && blockIdx.x == 0 && tid == 0) *p.status_reset = 0;

  float v[4][8];
  const int64_t base = row * p.K + static_cast<int64_t>(grp) * G + 8 * l;
  if (valid) {
    uint4 raw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) raw[j] = load_streaming(p.src + base + j * (G / 4));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[j][2 * q] = bf16lo(w[q]);
        v[j][2 * q + 1] = bf16hi(w[q]);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) v[j][e] = 0.0f;
  }

  fwht_group<G>(v, l);  // all lanes take part in the shuffles

  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[j][e]));
#pragma unroll
  for (int s = 1; s < LG; s <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, s));

  __syncthreads();  // row_max initialised
  // non-negative floats order like their bit patterns
  if (valid && l == 0) atomicMax(&row_max[row_in_cta], __float_as_uint(m));
  __syncthreads();

  if (MODE == kRqWeightAbsmax) {
    if (valid && t == 0) atomicMax(p.tensor_absmax, row_max[row_in_cta]);
    return;
  }

  const float amax_u =
      (MODE == kRqActivation) ? __uint_as_float(row_max[row_in_cta]) : __uint_as_float(*p.tensor_absmax);
  const QuantScale qs = make_scale<G>(amax_u);
  if (MODE == kRqActivation) {
    if (valid && t == 0) p.scale[row] = qs.s;
  } else {
    if (blockIdx.x == 0 && tid == 0) *p.scale = qs.s;
  }
  if (!valid) return;
  if (qs.pre != 1.0f) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) v[j][e] *= qs.pre;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint2 out;
    out.x = pack4(v[j][0], v[j][1], v[j][2], v[j][3], qs.ci);
    out.y = pack4(v[j][4], v[j][5], v[j][6], v[j][7], qs.ci);
    *reinterpret_cast<uint2*>(p.dst + base + j * (G / 4)) = out;
  }
}

// ------------------------------------------------------------------ launch

bool rotquant_shape(int64_t K, int* threads_per_row, int* rows_per_cta) {
  if (K <= 0 || K % 128 != 0 || K > 32768) return false;
  const int tpr = static_cast<int>(K / 32);
  int rpc = (256 + tpr - 1) / tpr;
  if (rpc < 1) rpc = 1;
  while ((rpc * tpr) % 32 != 0) ++rpc;
  if (rpc * tpr > 1024 || rpc > kMaxRowsPerCta) return false;
  *threads_per_row = tpr;
  *rows_per_cta = rpc;
  return true;
}

cudaError_t launch_rotate_quant(int g, int mode, RotQuantParams p, cudaStream_t stream) {
  int tpr = 0, rpc = 0;
  if (!rotquant_shape(p.K, &tpr, &rpc)) return cudaErrorInvalidValue;
  p.threads_per_row = tpr;
  p.rows_per_cta = rpc;
  const int64_t ctas = (p.rows + rpc - 1) / rpc;
  if (ctas > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(ctas));
  const dim3 block(static_cast<unsigned>(rpc * tpr));
  if (g == 256) {
    if (mode == kRqActivation) rotate_quant_kernel<256, kRqActivation><<<grid, block, 0, stream>>>(p);
    else if (mode == kRqWeightAbsmax) rotate_quant_kernel<256, kRqWeightAbsmax><<<grid, block, 0, stream>>>(p);
    else rotate_quant_kernel<256, kRqWeightQuant><<<grid, block, 0, stream>>>(p);
  } else if (g == 128) {
    if (mode == kRqActivation) rotate_quant_kernel<128, kRqActivation><<<grid, block, 0, stream>>>(p);
    else if (mode == kRqWeightAbsmax) rotate_quant_kernel<128, kRqWeightAbsmax><<<grid, block, 0, stream>>>(p);
    else rotate_quant_kernel<128, kRqWeightQuant><<<grid, block, 0, stream>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace convrot
