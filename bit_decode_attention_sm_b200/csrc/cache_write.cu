// HeadQ cache write: the base 2-bit key code, the residual, its projection onto
// the query-PCA basis U_h and the 4-bit side code ("HeadQ: Model-Visible
// Distortion and Score-Space Correction for KV-Cache Quantization", gist.science
// summary, section 3, step 2), plus the value store (dense copy, or the same
// 2-bit code for the full-KV composition of section 5).
//
// Every codec operation is a single IEEE fp32 operation through the *_rn
// intrinsics (this file is also compiled with -fmad=false), so the stored
// planes are bit-identical to the exact-arithmetic definition in headq.h.
//
// Work split: one CTA per (64-token tile, kv, b).
//   phase A  one warp per token, lanes over channels: group min/max by shuffles,
//            codes, packing, dequantisation, residual -> shared memory
//   phase B  one thread per (token, block of RB side-code rows): the projection
//            y = U_h^T e, channel by channel in order, one FMA per term
//   phase C  one thread per token: side scale, side codes, nibble packing
#include "headq_internal.cuh"

namespace headq {
namespace {

constexpr int kTT = 64;        // tokens per CTA
constexpr int kThreads = 256;  // 8 warps
constexpr unsigned kFull = 0xffffffffu;

template <int D>
struct Lanes {
  static constexpr int kActive = D < 32 ? D : 32;  // lanes that hold channels
  static constexpr int kCPL = D / kActive;         // channels per lane
  static constexpr int kGS = group_size(D);        // channels per group
  static constexpr int kLPG = kGS / kCPL;          // lanes per group
};

// Load CPL consecutive elements (fp32 or bf16) starting at element `off`.
template <int CPL>
__device__ __forceinline__ void load_vec(const void* base, size_t off, bool bf16,
                                         float (&x)[CPL]) {
  if (bf16) {
    const uint16_t* p = static_cast<const uint16_t*>(base) + off;
    if constexpr (CPL == 4) {
      uint2 u = *reinterpret_cast<const uint2*>(p);
      x[0] = __uint_as_float(u.x << 16);
      x[1] = __uint_as_float(u.x & 0xffff0000u);
      x[2] = __uint_as_float(u.y << 16);
      x[3] = __uint_as_float(u.y & 0xffff0000u);
    } else {
#pragma unroll
      for (int k = 0; k < CPL; ++k) x[k] = bf16_bits_to_f32(p[k]);
    }
  } else {
    const float* p = static_cast<const float*>(base) + off;
    if constexpr (CPL == 4) {
      float4 u = *reinterpret_cast<const float4*>(p);
      x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
    } else {
#pragma unroll
      for (int k = 0; k < CPL; ++k) x[k] = p[k];
    }
  }
}

// The base code B_b of one token: this lane holds channels lane*CPL .. +CPL-1.
// Writes the packed code bytes, scale and minimum of its group(s); returns the
// dequantised values mn + code*scale in xh.  All 32 lanes must call it.
template <int D>
__device__ __forceinline__ void base_code(const float (&x)[Lanes<D>::kCPL], int lane,
                                          bool store, uint8_t* code_row,
                                          float* scale_row, float* min_row,
                                          float (&xh)[Lanes<D>::kCPL]) {
  using L = Lanes<D>;
  constexpr int CPL = L::kCPL;
  float lo = x[0], hi = x[0];
#pragma unroll
  for (int k = 1; k < CPL; ++k) {
    lo = fminf(lo, x[k]);
    hi = fmaxf(hi, x[k]);
  }
#pragma unroll
  for (int off = 1; off < L::kLPG; off <<= 1) {
    lo = fminf(lo, __shfl_xor_sync(kFull, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(kFull, hi, off));
  }
  lo = __fadd_rn(lo, 0.0f);  // a -0 extreme is stored as +0
  hi = __fadd_rn(hi, 0.0f);
  const float scale = __fdiv_rn(__fsub_rn(hi, lo), 3.0f);
  uint32_t bits = 0;
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    int code = 0;
    if (scale != 0.0f) {
      const float t = rintf(__fdiv_rn(__fsub_rn(x[k], lo), scale));
      code = t < 0.0f ? 0 : (t > 3.0f ? 3 : static_cast<int>(t));
    }
    xh[k] = __fadd_rn(lo, __fmul_rn(static_cast<float>(code), scale));
    const int c = lane * CPL + k;
    bits |= static_cast<uint32_t>(code) << (CPL >= 4 ? 2 * k : 2 * (c & 3));
  }
  if constexpr (CPL < 4) {
#pragma unroll
    for (int off = 1; off * CPL < 4; off <<= 1) bits |= __shfl_xor_sync(kFull, bits, off);
  }
  if (!store) return;
  if constexpr (CPL >= 4) {
    if constexpr (CPL == 4) {
      code_row[lane] = static_cast<uint8_t>(bits);
    } else {
      reinterpret_cast<uint16_t*>(code_row)[lane] = static_cast<uint16_t>(bits);
    }
  } else {
    if (((lane * CPL) & 3) == 0) code_row[(lane * CPL) >> 2] = static_cast<uint8_t>(bits);
  }
  if (((lane * CPL) % L::kGS) == 0) {
    const int g = lane * CPL / L::kGS;
    scale_row[g] = scale;
    min_row[g] = lo;
  }
}

template <int D, int RB>
__global__ void __launch_bounds__(kThreads)
cache_write_kernel(const CacheWriteParams p) {
  using L = Lanes<D>;
  constexpr int CPL = L::kCPL;
  constexpr int NG = num_groups(D);
  constexpr int ES = D + 1;  // padded row of the residual tile

  extern __shared__ float smem[];
  float* e_s = smem;                 // [kTT][ES]
  float* u_s = e_s + kTT * ES;       // [D][r]
  const int r = p.c.r;
  float* y_s = u_s + D * r;          // [kTT][r + 1]

  const int b = blockIdx.z, kv = blockIdx.y;
  const int tile0 = blockIdx.x * kTT;
  const int Hkv = p.c.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t bk = static_cast<size_t>(b) * Hkv + kv;

  if (r > 0) {
    const float* U = p.U + static_cast<size_t>(kv) * D * r;
    for (int i = threadIdx.x; i < D * r; i += kThreads) u_s[i] = U[i];
  }

  // ---- phase A: base code, residual, values --------------------------------
  for (int tt = warp; tt < kTT; tt += kThreads / 32) {
    const int t = tile0 + tt;
    if (t >= p.n) break;  // warp-uniform
    const bool act = lane < L::kActive;
    const size_t in_off = (bk * p.n + t) * D + lane * CPL;
    const size_t row = bk * p.c.T_cap + p.t0 + t;
    float x[CPL], xh[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) x[k] = 0.0f;
    if (act) load_vec<CPL>(p.k, in_off, p.in_bf16, x);
    base_code<D>(x, lane, act, p.c.k_codes + row * (D / 4), p.c.k_scale + row * NG,
                 p.c.k_min + row * NG, xh);
    if (act) {
#pragma unroll
      for (int k = 0; k < CPL; ++k) e_s[tt * ES + lane * CPL + k] = __fsub_rn(x[k], xh[k]);
    }
    if (p.v != nullptr) {
      float vv[CPL];
#pragma unroll
      for (int k = 0; k < CPL; ++k) vv[k] = 0.0f;
      if (act) load_vec<CPL>(p.v, in_off, p.in_bf16, vv);
      if (p.c.vmode == HEADQ_V_2BIT) {
        float vh[CPL];
        base_code<D>(vv, lane, act, p.c.v_codes + row * (D / 4), p.c.v_scale + row * NG,
                     p.c.v_min + row * NG, vh);
      } else if (act) {
        const size_t vo = row * D + lane * CPL;
        if (p.c.v_dtype == HEADQ_BF16) {
          uint16_t* dst = static_cast<uint16_t*>(p.c.v) + vo;
          if (p.in_bf16) {
            const uint16_t* src = static_cast<const uint16_t*>(p.v) + in_off;
#pragma unroll
            for (int k = 0; k < CPL; ++k) dst[k] = src[k];
          } else {
#pragma unroll
            for (int k = 0; k < CPL; ++k)
              dst[k] = __bfloat16_as_ushort(__float2bfloat16_rn(vv[k]));
          }
        } else {
          float* dst = static_cast<float*>(p.c.v) + vo;
#pragma unroll
          for (int k = 0; k < CPL; ++k) dst[k] = vv[k];
        }
      }
    }
  }
  if (r == 0) return;  // no side code
  __syncthreads();

  // ---- phase B: y = U_h^T e, channel order, one FMA per term ---------------
  const int blocks_per_tok = r / RB;
  for (int pr = threadIdx.x; pr < kTT * blocks_per_tok; pr += kThreads) {
    const int tt = pr / blocks_per_tok;
    const int i0 = (pr - tt * blocks_per_tok) * RB;
    if (tile0 + tt >= p.n) continue;
    float y[RB];
#pragma unroll
    for (int k = 0; k < RB; ++k) y[k] = 0.0f;
    const float* er = e_s + tt * ES;
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
      const float ec = er[c];
      float u[RB];
      if constexpr (RB == 4) {
        const float4 q4 = *reinterpret_cast<const float4*>(u_s + c * r + i0);
        u[0] = q4.x; u[1] = q4.y; u[2] = q4.z; u[3] = q4.w;
      } else {
        const float2 q2 = *reinterpret_cast<const float2*>(u_s + c * r + i0);
        u[0] = q2.x; u[1] = q2.y;
      }
#pragma unroll
      for (int k = 0; k < RB; ++k) y[k] = __fmaf_rn(u[k], ec, y[k]);
    }
#pragma unroll
    for (int k = 0; k < RB; ++k) y_s[tt * (r + 1) + i0 + k] = y[k];
  }
  __syncthreads();

  // ---- phase C: side code -------------------------------------------------
  for (int tt = threadIdx.x; tt < kTT; tt += kThreads) {
    if (tile0 + tt >= p.n) continue;
    const float* y = y_s + tt * (r + 1);
    float a = 0.0f;
    for (int i = 0; i < r; ++i) a = fmaxf(a, fabsf(y[i]));
    const float s = __fdiv_rn(a, 7.0f);
    const size_t row = bk * p.c.T_cap + p.t0 + tile0 + tt;
    uint8_t* zr = p.c.z_codes + row * (r / 2);
    for (int i = 0; i < r; i += 2) {
      int w[2] = {0, 0};
      if (s != 0.0f) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const float t = rintf(__fdiv_rn(y[i + k], s));
          w[k] = t < -7.0f ? -7 : (t > 7.0f ? 7 : static_cast<int>(t));
        }
      }
      zr[i >> 1] = static_cast<uint8_t>((w[0] & 0xF) | ((w[1] & 0xF) << 4));
    }
    p.c.z_scale[row] = s;
  }
}

template <int D>
cudaError_t launch_d(const CacheWriteParams& p, cudaStream_t s) {
  const int r = p.c.r;
  const size_t smem = sizeof(float) * (static_cast<size_t>(kTT) * (D + 1) +
                                       static_cast<size_t>(D) * r +
                                       static_cast<size_t>(kTT) * (r + 1));
  dim3 grid((p.n + kTT - 1) / kTT, p.c.Hkv, p.c.B);
  auto k = r % 4 == 0 ? cache_write_kernel<D, 4> : cache_write_kernel<D, 2>;
  if (smem > 48 * 1024) {  // only the largest head dims need the opt-in
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  k<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cache_write(const CacheWriteParams& p, cudaStream_t s) {
  switch (p.c.d) {
    case 8: return launch_d<8>(p, s);
    case 16: return launch_d<16>(p, s);
    case 32: return launch_d<32>(p, s);
    case 64: return launch_d<64>(p, s);
    case 128: return launch_d<128>(p, s);
    case 256: return launch_d<256>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace headq
