// The HeadQ codec on the GPU, bit-exact: base 2-bit code, residual, projection
// and 4-bit side code ("HeadQ: Model-Visible Distortion and Score-Space
// Correction for KV-Cache Quantization", gist.science summary, section 3, step 2).
// Shared by the cache-write kernel and the fused append of the decode kernel.
//
// Every arithmetic step is one IEEE fp32 operation through an explicit *_rn
// intrinsic, so no compiler contraction can change a result.
#pragma once

#include "headq_internal.cuh"

namespace headq {
namespace codec {

// rint(RN(a / b)) for finite a and b != 0, without a division in the common case.
// With rb = RN(1/b), q = RN(a * rb) lies within |a/b| * 2^-22.9 of a/b, and RN(a/b)
// within |a/b| * 2^-24.  For |q| < 16 both errors are below 2^-18.9, so when q is
// more than 2^-16 away from every rounding boundary k + 1/2, a/b and RN(a/b) lie
// strictly on the same side of it and round to the same integer as q.  Otherwise
// (or when rb or q is not a small finite number) the quotient is formed exactly.
__device__ __forceinline__ float rint_quot(float a, float b, float rb) {
  const float q = __fmul_rn(a, rb);
  const float f = __fsub_rn(q, floorf(q));
  if (fabsf(q) < 16.0f && fabsf(__fsub_rn(f, 0.5f)) > 0x1p-16f) return rintf(q);
  return rintf(__fdiv_rn(a, b));
}

// Packed fp32 pairs (sm_100).  A packed multiply followed by a packed add is
// contracted into a fused multiply-add by the compiler even with explicit .rn
// (measured: the results are those of fma.rn.f32x2), so a sum that must be
// rounded on its own after a product is formed as fma.rn.f32x2(a, one, b) with
// `one` a runtime 1.0 (from the kernel parameters, unknown to the compiler):
// a * 1.0 is exact, so the lane is RN(a + b), and the product feeding it cannot
// be fused into it.
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// y = RN(y + RN(u * e)) in each lane: the projection's multiply, then add
__device__ __forceinline__ void muladd2_pk(uint64_t& y, uint64_t u, uint64_t e2, uint64_t one2) {
  uint64_t t;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(u), "l"(e2));
  y = fma2(t, one2, y);
}
// Packed fp32 pair helpers (sm_100), each lane one IEEE round-to-nearest op
// (mind the contraction of mul2 followed by add2 / sub2: see fma2 above).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) |
         (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float pk_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float pk_hi(uint64_t v) {
  return __uint_as_float(static_cast<uint32_t>(v >> 32));
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t dup2(float e) {
  const uint64_t b = __float_as_uint(e);
  return b | (b << 32);
}

// Base code B_b of one group of GS channels held by one thread: per-token,
// per-group asymmetric 2-bit min/max code.  Returns the packed code bytes
// (channel k of the group at bits 2(k%4) of byte k/4), the scale and minimum;
// with RESIDUAL, x is replaced by the residual x - (mn + code*scale) (product
// rounded first).
template <int GS, bool RESIDUAL>
__device__ __forceinline__ void quantize_group(float (&x)[GS], uint32_t (&packed)[GS / 16 > 0 ? GS / 16 : 1],
                                               float& scale_out, float& min_out) {
  float lo = x[0], hi = x[0];
#pragma unroll
  for (int k = 1; k < GS; ++k) {
    lo = fminf(lo, x[k]);
    hi = fmaxf(hi, x[k]);
  }
  lo = __fadd_rn(lo, 0.0f);  // a -0 extreme is stored as +0
  hi = __fadd_rn(hi, 0.0f);
  const float scale = __fdiv_rn(__fsub_rn(hi, lo), 3.0f);
  const float rs = __frcp_rn(scale);
#pragma unroll
  for (int w = 0; w < (GS / 16 > 0 ? GS / 16 : 1); ++w) packed[w] = 0u;
#pragma unroll
  for (int k = 0; k < GS; ++k) {
    int code = 0;
    if (scale != 0.0f) {
      const float t = rint_quot(__fsub_rn(x[k], lo), scale, rs);
      code = t < 0.0f ? 0 : (t > 3.0f ? 3 : static_cast<int>(t));
    }
    if constexpr (RESIDUAL)
      x[k] = __fsub_rn(x[k], __fadd_rn(lo, __fmul_rn(static_cast<float>(code), scale)));
    packed[k / 16] |= static_cast<uint32_t>(code) << (2 * (k % 16));
  }
  scale_out = scale;
  min_out = lo;
}

// Q_q: 4-bit symmetric absmax side code of r values; s = max|y| / 7,
// w = clamp(rint(y / s), -7, 7), all 0 when s == 0.
__device__ __forceinline__ float side_scale(float absmax) { return __fdiv_rn(absmax, 7.0f); }

__device__ __forceinline__ int side_level(float y, float s, float rs) {
  if (s == 0.0f) return 0;
  const float t = rint_quot(y, s, rs);
  return t < -7.0f ? -7 : (t > 7.0f ? 7 : static_cast<int>(t));
}

// Load n (multiple of 8 for bf16 / 4 for fp32) consecutive fp32 values.
template <int N>
__device__ __forceinline__ void load_row(const void* base, size_t off, bool bf16, float (&x)[N]) {
  if (bf16) {
    const uint16_t* p = static_cast<const uint16_t*>(base) + off;
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int k = 0; k < N / 8; ++k) {
        const uint4 u = reinterpret_cast<const uint4*>(p)[k];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          x[8 * k + 2 * j] = __uint_as_float(w[j] << 16);
          x[8 * k + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < N; ++k) x[k] = bf16_bits_to_f32(p[k]);
    }
  } else {
    const float* p = static_cast<const float*>(base) + off;
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int k = 0; k < N / 4; ++k) {
        const float4 u = reinterpret_cast<const float4*>(p)[k];
        x[4 * k] = u.x; x[4 * k + 1] = u.y; x[4 * k + 2] = u.z; x[4 * k + 3] = u.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < N; ++k) x[k] = p[k];
    }
  }
}

// Store the packed 2-bit code of one group (GS/4 bytes).
template <int GS>
__device__ __forceinline__ void store_codes(uint8_t* dst, const uint32_t (&packed)[GS / 16 > 0 ? GS / 16 : 1]) {
  if constexpr (GS == 32) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
  } else if constexpr (GS == 16) {
    *reinterpret_cast<uint32_t*>(dst) = packed[0];
  } else {
#pragma unroll
    for (int k = 0; k < GS / 4; ++k) dst[k] = static_cast<uint8_t>(packed[0] >> (8 * k));
  }
}

// Store GS values of a dense value row in the cache's value dtype.
template <int GS>
__device__ __forceinline__ void store_values(void* v, size_t off, bool cache_bf16, const float (&x)[GS]) {
  if (cache_bf16) {
    uint16_t* dst = static_cast<uint16_t*>(v) + off;
    if constexpr (GS % 8 == 0) {
#pragma unroll
      for (int k = 0; k < GS / 8; ++k) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          w[j] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(x[8 * k + 2 * j]))) |
                 (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(x[8 * k + 2 * j + 1])))
                  << 16);
        reinterpret_cast<uint4*>(dst)[k] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
#pragma unroll
      for (int k = 0; k < GS; ++k) dst[k] = __bfloat16_as_ushort(__float2bfloat16_rn(x[k]));
    }
  } else {
    float* dst = static_cast<float*>(v) + off;
    if constexpr (GS % 4 == 0) {
#pragma unroll
      for (int k = 0; k < GS / 4; ++k)
        reinterpret_cast<float4*>(dst)[k] = make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]);
    } else {
#pragma unroll
      for (int k = 0; k < GS; ++k) dst[k] = x[k];
    }
  }
}

}  // namespace codec
}  // namespace headq
