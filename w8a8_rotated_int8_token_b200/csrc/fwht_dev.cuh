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

// A float2 as one 64-bit register pair, and back (no instruction when the
// pair already sits in one).
__device__ __forceinline__ unsigned long long f2_as_b64(float2 v) {
  unsigned long long u;
  asm("mov.b64 %0, {%1, %2};" : "=l"(u) : "f"(v.x), "f"(v.y));
  return u;
}
__device__ __forceinline__ float2 b64_as_f2(unsigned long long u) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(u));
  return v;
}

// Packed butterflies (a + b, a - b) on f32x2, each lane rounded once. Written
// on 64-bit operands, the packed add and subtract keep every pair in one
// register pair through the stages: 8% fewer instructions in the
// rotate+quantise kernel than the same arithmetic through float2 intrinsics.
__device__ __forceinline__ float2 bfly_sum(float2 a, float2 b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_as_b64(a)), "l"(f2_as_b64(b)));
  return b64_as_f2(d);
}
__device__ __forceinline__ float2 bfly_diff(float2 a, float2 b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_as_b64(a)), "l"(f2_as_b64(b)));
  return b64_as_f2(d);
}

// The stage on the top piece bit (the .x and .y halves of a pair), on scalars.
__device__ __forceinline__ void fwht_pair_stage(float2 (&p)[4][8]) {
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float a = p[jj][e].x, b = p[jj][e].y;
      p[jj][e] = make_float2(a + b, a - b);
    }
  }
}

// The stage on the top piece bit taken first, straight from the input words:
// with a from piece jj and b from piece jj+4 (two elements per 32-bit word),
// lo = (a0 + b0, a0 - b0) and hi = (a1 + b1, a1 - b1). Only b is widened to
// float32; a enters the sm_100 mixed-precision add/sub as a 16-bit operand
// (exact), so each sum or difference is one float32 rounding, as after an
// explicit widening, at one instruction less per butterfly.
template <bool F16IN>
__device__ __forceinline__ void fwht_first_pair(uint32_t wa, float2 b, float2& lo, float2& hi) {
  if (F16IN) {
    asm("{\n\t.reg .b16 a0, a1;\n\tmov.b32 {a0, a1}, %4;\n\t"
        "add.rn.f32.f16 %0, a0, %5;\n\tsub.rn.f32.f16 %1, a0, %5;\n\t"
        "add.rn.f32.f16 %2, a1, %6;\n\tsub.rn.f32.f16 %3, a1, %6;\n\t}"
        : "=f"(lo.x), "=f"(lo.y), "=f"(hi.x), "=f"(hi.y)
        : "r"(wa), "f"(b.x), "f"(b.y));
  } else {
    asm("{\n\t.reg .b16 a0, a1;\n\tmov.b32 {a0, a1}, %4;\n\t"
        "add.rn.f32.bf16 %0, a0, %5;\n\tsub.rn.f32.bf16 %1, a0, %5;\n\t"
        "add.rn.f32.bf16 %2, a1, %6;\n\tsub.rn.f32.bf16 %3, a1, %6;\n\t}"
        : "=f"(lo.x), "=f"(lo.y), "=f"(hi.x), "=f"(hi.y)
        : "r"(wa), "f"(b.x), "f"(b.y));
  }
}

// max(a, b, c) in one sm_100 three-input instruction.
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// max |value| of a lane's 64 values in 32 sm_100 three-input maxima, |.|
// taken on the inputs of the first level: 64 -> 22 -> 8 -> 3 -> 1 (four
// dependent steps).
__device__ __forceinline__ float absmax64_v3(const float2 (&w)[4][8]) {
  auto val = [&](int v) {  // value v of the lane: pair v / 2, its .x or .y half
    const float2 p = w[v >> 4][(v >> 1) & 7];
    return (v & 1) ? p.y : p.x;
  };
  float a[22];
#pragma unroll
  for (int i = 0; i < 21; ++i) a[i] = fmax3f(fabsf(val(3 * i)), fabsf(val(3 * i + 1)), fabsf(val(3 * i + 2)));
  a[21] = fabsf(val(63));
  float b[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) b[i] = fmax3f(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
  b[7] = a[21];
  return fmax3f(fmax3f(b[0], b[1], b[2]), fmax3f(b[3], b[4], b[5]), fmaxf(b[6], b[7]));
}

// The five packed stages on the index bits a lane holds apart from the top
// piece bit: p[jj][e] holds the elements of pieces jj (.x) and jj+4 (.y) at
// in-piece position e; the stages run on e (1, 2, 4) and jj (1, 2) as f32x2.
__device__ __forceinline__ void fwht_lane_local(float2 (&p)[4][8]) {
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

// The stages on the lane bits of a group (LG = g/64 lanes), with shuffles:
// the lower partner keeps a + b, the upper one b_partner - own = a - b.
template <int LG>
__device__ __forceinline__ void fwht_lane_shuffle(float2 (&p)[4][8], int l) {
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

// Unnormalised Walsh-Hadamard transform of one group, all in registers and
// shuffles; lane l of the group holds pieces jj, jj+4 at group offset 8l.
template <int G>
__device__ __forceinline__ void fwht_group(float2 (&p)[4][8], int l) {
  fwht_lane_local(p);
  fwht_pair_stage(p);
  fwht_lane_shuffle<G / 64>(p, l);
}

// g = 256 through shared memory instead of shuffles. Before the exchange
// lane l (0..3) of a group holds the elements whose index bits 3-4 equal l;
// the 8-byte pair p[jj][e] = (element 32jj + 8l + e, element 128 + the same).
// Lane jj receives that pair: afterwards q[src][e] holds the pair of
// elements 32*l + 8*src + e (and +128), so the lane owns two runs of 32
// consecutive elements and index bits 3-4 are in registers.
//
// The transposition runs in four rounds (e in {2r, 2r+1}) through the 4 KB
// of shared memory the warp's own input came from. In a round, the 16-byte
// chunk that lane src sends to lane d of warp group gw sits at chunk index
// 38*(gw/2) + (gw%2) + 10*d + 2*src: the two groups of a pair interleave on
// even and odd chunks, so every 8-lane phase of a 16-byte store (fixed d) or
// load (fixed src) touches 8 different bank quads, and every address is a
// per-thread base plus a constant. A round spans 2432 bytes.
constexpr int kX256RegionBytes = 4096;  // the input bytes of one warp: 32 lanes x 64 bf16 (see rotquant_slot_bytes)

__device__ __forceinline__ void fwht256_exchange(const float2 (&p)[4][8], float2 (&q)[4][8], uint8_t* warp_region,
                                                 int gw, int l) {
  uint8_t* const pair_base = warp_region + 16 * (38 * (gw >> 1) + (gw & 1));
  uint8_t* const wr = pair_base + 32 * l;        // + 160 d
  const uint8_t* const rd = pair_base + 160 * l;  // + 32 src
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    __syncwarp();  // the warp's input loads, or the previous round's loads, are done
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      const float2 a = p[d][2 * r], b = p[d][2 * r + 1];
      *reinterpret_cast<float4*>(wr + 160 * d) = make_float4(a.x, a.y, b.x, b.y);
    }
    __syncwarp();
#pragma unroll
    for (int src = 0; src < 4; ++src) {
      const float4 f = *reinterpret_cast<const float4*>(rd + 32 * src);
      q[src][2 * r] = make_float2(f.x, f.y);
      q[src][2 * r + 1] = make_float2(f.z, f.w);
    }
  }
}

// g = 256, the two stages left after the exchange (index bits 3-4, the first
// index of q), packed.
__device__ __forceinline__ void fwht256_after_exchange(float2 (&q)[4][8]) {
#pragma unroll
  for (int h = 1; h < 4; h <<= 1) {
#pragma unroll
    for (int src = 0; src < 4; ++src) {
      if ((src & h) == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 a = q[src][e], b = q[src + h][e];
          q[src][e] = bfly_sum(a, b);
          q[src + h][e] = bfly_diff(a, b);
        }
      }
    }
  }
}

// max |value| of a lane's 64 values, as a balanced tree (six dependent steps
// instead of a 64-long chain).
__device__ __forceinline__ float absmax64(const float2 (&w)[4][8]) {
  float a[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 x = w[i >> 2][2 * (i & 3)], y = w[i >> 2][2 * (i & 3) + 1];
    a[i] = fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(y.x), fabsf(y.y)));
  }
#pragma unroll
  for (int n = 8; n >= 1; n >>= 1)
#pragma unroll
    for (int i = 0; i < n; ++i) a[i] = fmaxf(a[i], a[i + n]);
  return a[0];
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

// The stored scale of a row (or tensor): float32(absmax(X R) / 127) =
// absmax_u / (127 sqrt(g)), correctly rounded (for g = 256 the divisor 2032 is
// exact; for g = 128 it is the nearest float to 127 sqrt(128)). From 2^-100 up
// the quotient is the product with the rounded reciprocal r of the divisor,
// corrected once by the exact remainder (two fused multiply-adds); that this
// equals the correctly rounded quotient for every float in that range is
// checked exhaustively on the CPU by the test suite. Below 2^-100 (where the
// remainder could leave the normal range) it is the plain division.
template <int G>
__device__ __forceinline__ float scale_of(float amax_u) {
  constexpr float div = (G == 256) ? 2032.0f : 1436.8409423828125f;
  constexpr float r = (G == 256) ? 0x1.020408p-11f : 0x1.6ce3aep-11f;  // nearest floats to 1/div
  if (amax_u >= 0x1p-100f) {
    const float q0 = __fmul_rn(amax_u, r);
    const float e = fmaf(-q0, div, amax_u);  // exact remainder amax_u - q0 * div
    return fmaf(e, r, q0);
  }
  return amax_u / div;
}

// The factor that maps an unnormalised value u to code units:
// code = rne(u * ci) with ci = 127 / absmax_u, the same quotient as u / (sqrt(g) s)
// up to float32 rounding (which can move a code only at a near-tie). The row
// maximum maps to 127 * (1 +- 2^-22), so no code leaves [-127, 127].
struct CodeFactor {
  float ci;   // 0 for an all-zero row
  float pre;  // 1, or 2^64 for rows whose absmax is below 2^-90
};

__device__ __forceinline__ CodeFactor code_factor(float amax_u) {
  CodeFactor c;
  c.pre = 1.0f;
  if (amax_u == 0.0f) {
    c.ci = 0.0f;
  } else if (amax_u >= 0x1p-90f) {
    c.ci = 127.0f * __frcp_rn(amax_u);
  } else {  // tiny row: lift by 2^64 (exact) so that the reciprocal cannot overflow
    c.pre = 0x1p64f;
    c.ci = 127.0f * __frcp_rn(amax_u * 0x1p64f);
  }
  return c;
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
