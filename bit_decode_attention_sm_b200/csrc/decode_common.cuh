// Device helpers shared by the tensor-core decode and diagnostic kernels
// (decode_mma.cu, attn_kl_hm.cu): PTX
// wrappers for mbarriers, bulk and tensor copies and the MMAs, the exact
// unpacking of 2-bit codes and 4-bit side codes into fp16 operands, the fp16 /
// bf16 high-low splits, the per-head power-of-two prescale of the query, and
// the bit-exact encoding of an appended token ("HeadQ: Model-Visible Distortion
// and Score-Space Correction for KV-Cache Quantization", gist.science summary,
// section 3, steps 2 and 3).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "codec.cuh"
#include "headq_internal.cuh"

namespace headq {
namespace dc {

constexpr long long kWaitCycles = 4000000000LL;  // about 2 s at B200 clocks
constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Up to kSuspendNs the waiting warp is suspended by the hardware (it resumes as
// soon as the phase completes) instead of spinning through issue slots.
constexpr uint32_t kSuspendNs = 1000000;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}
// Wait for the phase of the given parity to complete; false after ~2 s (the
// clock is read every 32 tries, each of which suspends for at most kSuspendNs).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long start = clock64();
  for (;;) {
    for (int k = 0; k < 32; ++k)
      if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - start > kWaitCycles) return false;
  }
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                       uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4],
                                        const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// ---------------------------------------------------------------- unpacking
// y holds one 16-bit word of eight 2-bit codes c0..c7 (code k at bits 2k) in both
// halves.  Returns fp16 pairs (c0,c1) (c2,c3) (c4,c5) (c6,c7), exactly.
__device__ __forceinline__ void unpack_codes(uint32_t y, uint32_t (&v)[4]) {
  const uint32_t z = y >> 8;
  // (1024 + c, 1024 + 4c') * (1, 1/4) - (1024, 256)
  v[0] = hfma2((y & 0x000C0003u) | 0x64006400u, 0x34003C00u, 0xDC00E400u);
  // (1024 + 16c, 1024 + 64c') * (1/16, 1/64) - (64, 16)
  v[1] = hfma2((y & 0x00C00030u) | 0x64006400u, 0x24002C00u, 0xCC00D400u);
  v[2] = hfma2((z & 0x000C0003u) | 0x64006400u, 0x34003C00u, 0xDC00E400u);
  v[3] = hfma2((z & 0x00C00030u) | 0x64006400u, 0x24002C00u, 0xCC00D400u);
}
// y holds one 16-bit word of four offset nibbles (w + 8, nibble k at bits 4k) in
// both halves.  Returns fp16 pairs (w0,w1) (w2,w3), exactly.
__device__ __forceinline__ void unpack_side(uint32_t y, uint32_t& n01, uint32_t& n23) {
  const uint32_t z = y >> 8;
  // (1024 + n, 1024 + 16n') * (1, 1/16) - (1032, 72)
  n01 = hfma2((y & 0x00F0000Fu) | 0x64006400u, 0x2C003C00u, 0xD480E408u);
  n23 = hfma2((z & 0x00F0000Fu) | 0x64006400u, 0x2C003C00u, 0xD480E408u);
}
__device__ __forceinline__ uint32_t half_part_pair(float a, float b, bool lo) {
  __half ha = __float2half_rn(a), hb = __float2half_rn(b);
  if (lo) {
    ha = __float2half_rn(a - __half2float(ha));
    hb = __float2half_rn(b - __half2float(hb));
  }
  return static_cast<uint32_t>(__half_as_ushort(ha)) |
         (static_cast<uint32_t>(__half_as_ushort(hb)) << 16);
}
// 2^-e (f) and 2^e (finv), e the binary exponent of the largest |q| of query
// head h (from its per-group maxima), clamped to [-126, 126].  The head's query
// times 2^-e has its largest element in [1, 2), so its fp16 high and low parts,
// its group sums and sigma U_h^T q stay inside fp16 range whatever the query's
// magnitude; the logit is scaled back by 2^e in fp32 (a power of two: exact).
template <int NG>
__device__ __forceinline__ void head_prescale(const float* qmax_s, int h, float& f, float& finv) {
  float m = 0.f;
#pragma unroll
  for (int gg = 0; gg < NG; ++gg) m = fmaxf(m, qmax_s[h * NG + gg]);
  int e = m > 0.f ? static_cast<int>((__float_as_uint(m) >> 23) & 0xffu) - 127 : 0;
  e = max(-126, min(126, e));
  f = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
  finv = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}
// 2^-e (f) and 2^e (finv), e the binary exponent of m >= 0 clamped to
// [-126, 126] (0 for m == 0): m * f lies in [1, 2)
__device__ __forceinline__ void pow2_prescale(float m, float& f, float& finv) {
  int e = m > 0.f ? static_cast<int>((__float_as_uint(m) >> 23) & 0xffu) - 127 : 0;
  e = max(-126, min(126, e));
  f = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
  finv = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}
// 2^-E for a power-of-two exponent E in [-126, 126]
__device__ __forceinline__ float pow2_neg(int E) {
  return __uint_as_float(static_cast<uint32_t>(127 - E) << 23);
}
__device__ __forceinline__ uint32_t bf16_part_pair(float a, float b, bool lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 f = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - f.x, b - f.y);
  const __nv_bfloat162 r = lo ? l : h;
  return *reinterpret_cast<const uint32_t*>(&r);
}
// The new token of sequence b, KV head kv, encoded into cache position pos
// exactly as the cache write does (bit-exact codec): lanes 0..NG-1 take the key
// groups, NG..2NG-1 the value groups, lanes < R the side rows.  Warp-wide; U_h
// is in shared memory, enew_s is [D] scratch.
template <int D, int R, bool V2>
__device__ __forceinline__ void encode_new_token(const DecodeParams& p, int b, int kv, int pos,
                                                 const float* u_s, float* enew_s, int lane) {
  constexpr int NG = D / 32;
  const size_t bk = static_cast<size_t>(b) * p.c.Hkv + kv;
  const long long orow = cache_row(p.c, b, kv, pos);
  if (orow < 0 && lane == 0 && p.err) atomicOr(p.err, kDevErrBadPage);
  const size_t row = orow < 0 ? 0 : static_cast<size_t>(orow);
  const size_t in = bk * D;
  if (orow < 0) {
    // a block-table entry outside the pool: the token is not written
  } else if (lane < NG) {
    float x[32];
    uint32_t packed[2];
    float sc, mn;
    codec::load_row<32>(p.k_new, in + lane * 32, p.new_bf16, x);
    codec::quantize_group<32, true>(x, packed, sc, mn);
    codec::store_codes<32>(p.c.k_codes + row * (D / 4) + lane * 8, packed);
    p.c.k_scale[row * NG + lane] = sc;
    p.c.k_min[row * NG + lane] = mn;
#pragma unroll
    for (int k = 0; k < 32; ++k) enew_s[lane * 32 + k] = x[k];
  } else if (lane < 2 * NG && p.v_new != nullptr) {
    const int gv = lane - NG;
    float vv[32];
    codec::load_row<32>(p.v_new, in + gv * 32, p.new_bf16, vv);
    if constexpr (V2) {
      uint32_t packed[2];
      float sc, mn;
      codec::quantize_group<32, false>(vv, packed, sc, mn);
      codec::store_codes<32>(p.c.v_codes + row * (D / 4) + gv * 8, packed);
      p.c.v_scale[row * NG + gv] = sc;
      p.c.v_min[row * NG + gv] = mn;
    } else {
      codec::store_values<32>(p.c.v, row * D + gv * 32, true, vv);
    }
  }
  __syncwarp();
  if (R > 0 && orow >= 0) {
    float y = 0.0f;
    // channels in order (the codec's rounding sequence); unrolled so that the
    // loads of U_h (shared or global memory) are issued ahead of the adds
    if (lane < R) {
#pragma unroll 16
      for (int c = 0; c < D; ++c) y = __fadd_rn(y, __fmul_rn(u_s[c * R + lane], enew_s[c]));
    }
    float a = lane < R ? fabsf(y) : 0.0f;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o2));
    const float zs = codec::side_scale(a);
    const int w = lane < R ? codec::side_level(y, zs, __frcp_rn(zs)) : 0;
    const int w_next = __shfl_down_sync(kFull, w, 1);
    if (lane < R && (lane & 1) == 0)
      p.c.z_codes[row * (R / 2) + (lane >> 1)] =
          static_cast<uint8_t>((w & 0xF) | ((w_next & 0xF) << 4));
    if (lane == 0) p.c.z_scale[row] = zs;
  }
}

}  // namespace dc
}  // namespace headq
