// Device building blocks of the per-token rotation and quantisation, shared by
// the standalone rotate+quantise kernel and the fused ConvRot linear kernel:
// the unnormalised fast Walsh-Hadamard transform of a 64-element lane slice
// (packed f32x2 butterflies), the scale rule and the int8 code packing.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace convrot {

namespace fwht {

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + magic rounds x to an integer (ties to even)

__device__ __forceinline__ float2 bfly_sum(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 bfly_diff(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

// Unnormalised Walsh-Hadamard transform of one group. p[jj][e] holds the
// elements of pieces jj (.x) and jj+4 (.y) at in-piece position e.
template <int G>
__device__ __forceinline__ void fwht_group(float2 (&p)[4][8], int l) {
  // in-piece bits (e: 1, 2, 4), packed
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if ((e & h) == 0) {
          const float2 a = p[jj][e], b = p[jj][e + h];
          p[jj][e] = bfly_sum(a, b);
          p[jj][e + h] = bfly_diff(a, b);
        }
      }
    }
  }
  // piece bits 0 and 1, packed
#pragma unroll
  for (int h = 1; h < 4; h <<= 1) {
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if ((jj & h) == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 a = p[jj][e], b = p[jj + h][e];
          p[jj][e] = bfly_sum(a, b);
          p[jj + h][e] = bfly_diff(a, b);
        }
      }
    }
  }
  // piece bit 2: the two halves of each pair
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float a = p[jj][e].x, b = p[jj][e].y;
      p[jj][e] = make_float2(a + b, a - b);
    }
  }
  // lane bits: the lower partner keeps a + b, the upper one b_partner - own = a - b
  constexpr int LG = G / 64;
#pragma unroll
  for (int m = 1; m < LG; m <<= 1) {
    const float sgn = (l & m) ? -1.0f : 1.0f;
    const float2 s2 = make_float2(sgn, sgn);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float2 q;
        q.x = __shfl_xor_sync(0xFFFFFFFFu, p[jj][e].x, m);
        q.y = __shfl_xor_sync(0xFFFFFFFFu, p[jj][e].y, m);
        p[jj][e] = __ffma2_rn(s2, p[jj][e], q);
      }
    }
  }
}

// g = 256, first half: the five stages on the bits a lane holds in registers
// (in-piece bits 0-2 and piece bits 5-6; bit 7 is the .x/.y half of a pair).
__device__ __forceinline__ void fwht256_in_lane(float2 (&p)[4][8]) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if ((e & h) == 0) {
          const float2 a = p[jj][e], b = p[jj][e + h];
          p[jj][e] = bfly_sum(a, b);
          p[jj][e + h] = bfly_diff(a, b);
        }
      }
    }
  }
#pragma unroll
  for (int h = 1; h < 4; h <<= 1) {
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if ((jj & h) == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 a = p[jj][e], b = p[jj + h][e];
          p[jj][e] = bfly_sum(a, b);
          p[jj + h][e] = bfly_diff(a, b);
        }
      }
    }
  }
}

// g = 256, the exchange: lane l of a group holds the elements whose bits 3-4
// equal l; afterwards it holds those whose bits 5-6 equal l, as
// w[b7][q] = (element 128*b7 + 32*l + 2*q, ... + 1), q = bits 1-4. The 4 KB of
// shared memory the warp's own input came from are reused in two rounds, one
// per value of bit 2, so that whole float2 pairs retire on both sides of each
// round. In a round a group's 128 values form 32 16-byte chunks
// c = bits 3-7 of the element index; chunk c is stored at
// (c & ~7) | ((c ^ ((c >> 3) & 1) << 1 ^ 5 * (group & 1)) & 7), which keeps the
// writes and the reads of a warp on all 32 banks (4 wavefronts each).
__device__ __forceinline__ int xchg_chunk(int c, int gw5) {
  return (c & ~7) | ((c ^ (((c >> 3) & 1) << 1) ^ gw5) & 7);
}

__device__ __forceinline__ void fwht256_exchange(const float2 (&p)[4][8], float2 (&w)[2][16], uint8_t* region,
                                                 int gw, int l, bool active) {
  float* blk = reinterpret_cast<float*>(region + gw * 512);
  const int gw5 = (gw & 1) ? 5 : 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {  // bit 2 of the element index
    __syncwarp();  // the previous use of the region (input pieces or round 0) is finished
    if (active) {
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {    // bits 5-6
#pragma unroll
        for (int b7 = 0; b7 < 2; ++b7) {
          const int c = l + 4 * jj + 16 * b7;
          float4 f;
          f.x = b7 ? p[jj][4 * h + 0].y : p[jj][4 * h + 0].x;
          f.y = b7 ? p[jj][4 * h + 1].y : p[jj][4 * h + 1].x;
          f.z = b7 ? p[jj][4 * h + 2].y : p[jj][4 * h + 2].x;
          f.w = b7 ? p[jj][4 * h + 3].y : p[jj][4 * h + 3].x;
          *reinterpret_cast<float4*>(blk + 4 * xchg_chunk(c, gw5)) = f;
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k) {         // bits 3-4
#pragma unroll
      for (int b7 = 0; b7 < 2; ++b7) {
        const int q = 8 * (k >> 1) + 4 * (k & 1) + 2 * h;
        if (active) {
          const int c = k + 4 * l + 16 * b7;
          const float4 f = *reinterpret_cast<const float4*>(blk + 4 * xchg_chunk(c, gw5));
          w[b7][q] = make_float2(f.x, f.y);
          w[b7][q + 1] = make_float2(f.z, f.w);
        } else {
          w[b7][q] = make_float2(0.0f, 0.0f);
          w[b7][q + 1] = make_float2(0.0f, 0.0f);
        }
      }
    }
  }
}

// g = 256, second half: stages on bits 3 (q bit 2), 4 (q bit 3) and 7.
__device__ __forceinline__ void fwht256_after_exchange(float2 (&w)[2][16]) {
#pragma unroll
  for (int h = 4; h < 16; h <<= 1) {
#pragma unroll
    for (int b7 = 0; b7 < 2; ++b7) {
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if ((q & h) == 0) {
          const float2 a = w[b7][q], b = w[b7][q + h];
          w[b7][q] = bfly_sum(a, b);
          w[b7][q + h] = bfly_diff(a, b);
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const float2 a = w[0][q], b = w[1][q];
    w[0][q] = bfly_sum(a, b);
    w[1][q] = bfly_diff(a, b);
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

// Four codes from four magic-rounded floats: the low byte of (u*ci + 1.5*2^23)
// is the two's-complement int8 code of rne(u*ci).
__device__ __forceinline__ uint32_t pack4(float a, float b, float c, float d) {
  const uint32_t lo = __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040);
  const uint32_t hi = __byte_perm(__float_as_uint(c), __float_as_uint(d), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

}  // namespace fwht

}  // namespace convrot
