// HeadQ cache write: the base 2-bit key code, the residual, its projection onto
// the query-PCA basis U_h and the 4-bit side code ("HeadQ: Model-Visible
// Distortion and Score-Space Correction for KV-Cache Quantization", gist.science
// summary, section 3, step 2), plus the value store (dense copy, or the same
// 2-bit code for the full-KV composition of section 5).
//
// Bit-exact: every codec operation is one IEEE fp32 operation (codec.cuh; this
// file is also compiled with -fmad=false).
//
// One CTA per (64-token tile, kv, b), two phases:
//   A  one thread per (token, 32-channel group): the group's keys and values
//      loaded straight from HBM together, base code (a short path per channel,
//      the exact codec near a rounding tie), codes/scale/min stored, the
//      residual written to shared memory, values copied or coded
//   B  one thread per (token, RB side rows), two threads per token for r = 16:
//      y = U_h^T e in channel order, each term a rounded product then a rounded
//      sum (packed fp32x2 multiply and add, two rows per instruction), U_h read
//      as (nearly) warp-wide broadcasts; then max|y|
//      shared by a warp shuffle and the 4-bit side code of each thread's rows
#include "codec.cuh"

namespace headq {
namespace {

constexpr int kTT = 64;        // tokens per CTA
constexpr int kThreads = 256;
constexpr unsigned kFull = 0xffffffffu;

// The residual tile in shared memory, one fp32 per channel.  Group g of a
// token starts at 16-byte chunk g*GC (two chunks of padding per group: GC = 10,
// 2 mod 8, for 32-channel groups) and a token row spans RC chunks (RC odd): the
// (token, group) writes of phase A and the per-token reads of phase B then fall
// in distinct banks.
template <int D>
struct ResTile {
  static constexpr int GS = group_size(D);
  static constexpr int NG = num_groups(D);
  static constexpr int GC = GS / 4 + 2;
  static constexpr int RC = NG * GC + 1;
  static constexpr int kFloats = kTT * RC * 4;
  // float offset of channel c within a token row
  __device__ static int off(int c) { return 4 * ((c / GS) * GC + (c % GS) / 4) + (c & 3); }
};

// U_h in shared memory as [r / RB][D][RB]: the RB rows a phase-B thread owns are
// contiguous for every channel; blocks are padded apart by 16 bytes (8 for RB 2)
// so the threads of a token (when it has several) read distinct banks.
template <int D, int RB>
struct BasisTile {
  static constexpr int kPad = RB >= 4 ? 4 : 2;
  static constexpr int kBlock = D * RB + kPad;
  __host__ __device__ static int floats(int r) { return (r / RB) * kBlock; }
};

__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// GS values of one group as loaded: GS/8 16-byte words of bf16, or GS/4 of fp32.
template <int GS, bool BF16>
struct RawGroup {
  static constexpr int kWords = BF16 ? GS / 8 : GS / 4;
  uint4 w[kWords];
};

template <int GS, bool BF16>
__device__ __forceinline__ void load_raw(const void* base, size_t off, RawGroup<GS, BF16>& g) {
  if constexpr (BF16) {
    const uint4* s = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off);
#pragma unroll
    for (int k = 0; k < GS / 8; ++k) g.w[k] = s[k];
  } else {
    const uint4* s = reinterpret_cast<const uint4*>(static_cast<const float*>(base) + off);
#pragma unroll
    for (int k = 0; k < GS / 4; ++k) g.w[k] = s[k];
  }
}

template <int GS, bool BF16>
__device__ __forceinline__ void unpack_raw(const RawGroup<GS, BF16>& g, float (&x)[GS]) {
  if constexpr (BF16) {
#pragma unroll
    for (int k = 0; k < GS / 8; ++k) {
      const uint32_t w[4] = {g.w[k].x, g.w[k].y, g.w[k].z, g.w[k].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[8 * k + 2 * j] = __uint_as_float(w[j] << 16);
        x[8 * k + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < GS / 4; ++k) {
      x[4 * k] = __uint_as_float(g.w[k].x);
      x[4 * k + 1] = __uint_as_float(g.w[k].y);
      x[4 * k + 2] = __uint_as_float(g.w[k].z);
      x[4 * k + 3] = __uint_as_float(g.w[k].w);
    }
  }
}

// The per-token base code of one group: the codes, scale, minimum and residuals
// of codec::quantize_group, with fewer operations per channel.  With the scale
// a normal number of at most 2^126, every product q = RN((x - min) * RN(1/scale))
// lies in [0, 3(1 + 2^-21)]: RN(x - min) <= RN(max - min) = R, scale = RN(R/3),
// and the three roundings (scale, 1/scale, the product) are each within a
// relative 2^-24.  Then q rounds to the same integer
// as RN((x - min)/scale) whenever q is more than 2^-16 away from a half-integer
// (the error argument of codec::rint_quot), so no clamp is needed there; a
// channel whose q lies that close to a half-integer (exact ties are common with
// bf16 inputs) takes the exact quotient, as codec::rint_quot does.  Returns false,
// with x partly overwritten, when the scale is outside that range: the caller
// then runs the exact codec on the group.
template <int GS, bool RESIDUAL>
__device__ __forceinline__ bool quantize_group_fast(float (&x)[GS],
                                                    uint32_t (&packed)[GS / 16 > 0 ? GS / 16 : 1],
                                                    float& scale_out, float& min_out, float one) {
  float lo = x[0], hi = x[0];
#pragma unroll
  for (int k = 1; k + 1 < GS; k += 2) {
    lo = fmin3(lo, x[k], x[k + 1]);
    hi = fmax3(hi, x[k], x[k + 1]);
  }
  lo = fminf(lo, x[GS - 1]);
  hi = fmaxf(hi, x[GS - 1]);
  lo = __fadd_rn(lo, 0.0f);  // a -0 extreme is stored as +0
  hi = __fadd_rn(hi, 0.0f);
  const float scale = __fdiv_rn(__fsub_rn(hi, lo), 3.0f);
  scale_out = scale;
  min_out = lo;
#pragma unroll
  for (int w = 0; w < (GS / 16 > 0 ? GS / 16 : 1); ++w) packed[w] = 0u;
  if (scale == 0.0f) {  // all codes 0; the residual is x - (min + 0) = x - min
    if constexpr (RESIDUAL) {
#pragma unroll
      for (int k = 0; k < GS; ++k) x[k] = __fsub_rn(x[k], lo);
    }
    return true;
  }
  if (!(scale >= 0x1p-126f && scale <= 0x1p126f)) return false;
  const float rs = __frcp_rn(scale);
  // Channel pairs (k, k+1) in packed fp32x2 registers: every lane of sub2 / mul2 /
  // add2 is the same round-to-nearest operation as the scalar form, so codes and
  // residuals are unchanged bit for bit.  The codes are summed as c * 4^(k % 8)
  // (exact small integers), even and odd channels in separate lanes.
  const uint64_t lo2 = codec::pk2(lo, lo), rs2 = codec::pk2(rs, rs), sc2 = codec::pk2(scale, scale);
  const uint64_t one2 = codec::pk2(one, one), mone2 = codec::pk2(-one, -one);
  uint64_t acc2[GS / 8 > 0 ? GS / 8 : 1];
#pragma unroll
  for (int i = 0; i < (GS / 8 > 0 ? GS / 8 : 1); ++i) acc2[i] = 0ull;
#pragma unroll
  for (int k = 0; k < GS; k += 2) {
    const uint64_t a2 = codec::sub2(codec::pk2(x[k], x[k + 1]), lo2);
    const uint64_t q2 = codec::mul2(a2, rs2);
    float c0 = rintf(codec::pk_lo(q2)), c1 = rintf(codec::pk_hi(q2));
    const uint64_t d2 = codec::fma2(codec::pk2(c0, c1), mone2, q2);  // RN(q - c)
    // near a half-integer (or NaN): that channel takes the exact quotient
    const bool ok0 = fabsf(codec::pk_lo(d2)) < 0.5f - 0x1p-16f;
    const bool ok1 = fabsf(codec::pk_hi(d2)) < 0.5f - 0x1p-16f;
    if (!(ok0 && ok1)) {
      if (!ok0) {
        const float t = rintf(__fdiv_rn(codec::pk_lo(a2), scale));
        c0 = static_cast<float>(t < 0.0f ? 0 : (t > 3.0f ? 3 : static_cast<int>(t)));
      }
      if (!ok1) {
        const float t = rintf(__fdiv_rn(codec::pk_hi(a2), scale));
        c1 = static_cast<float>(t < 0.0f ? 0 : (t > 3.0f ? 3 : static_cast<int>(t)));
      }
    }
    const uint64_t c2 = codec::pk2(c0, c1);
    const int j = k % 8;  // weights 4^j, 4^(j+1)
    acc2[k / 8] = codec::add2(acc2[k / 8], codec::mul2(c2, codec::pk2(static_cast<float>(1u << (2 * j)),
                                                                     static_cast<float>(1u << (2 * j + 2)))));
    if constexpr (RESIDUAL) {
      // RN(x - RN(min + RN(c * scale))): the product rounded before the sum
      const uint64_t r2 = codec::sub2(codec::pk2(x[k], x[k + 1]),
                                      codec::fma2(codec::mul2(c2, sc2), one2, lo2));
      x[k] = codec::pk_lo(r2);
      x[k + 1] = codec::pk_hi(r2);
    }
  }
  if constexpr (GS >= 16) {
#pragma unroll
    for (int w = 0; w < GS / 16; ++w) {
      const uint32_t a = static_cast<uint32_t>(codec::pk_lo(acc2[2 * w]) + codec::pk_hi(acc2[2 * w]));
      const uint32_t b = static_cast<uint32_t>(codec::pk_lo(acc2[2 * w + 1]) + codec::pk_hi(acc2[2 * w + 1]));
      packed[w] = a | (b << 16);
    }
  } else {
    packed[0] = static_cast<uint32_t>(codec::pk_lo(acc2[0]) + codec::pk_hi(acc2[0]));
  }
  return true;
}

// Base code of a group loaded as raw words from base + off: the short path, or,
// for a scale outside its range, the group loaded again through the exact codec.
template <int GS, bool RESIDUAL, bool BF16>
__device__ __forceinline__ void quantize_raw(const void* base, size_t off, RawGroup<GS, BF16>& raw,
                                             float (&x)[GS],
                                             uint32_t (&packed)[GS / 16 > 0 ? GS / 16 : 1],
                                             float& sc, float& mn, float one) {
  unpack_raw<GS, BF16>(raw, x);
  if (!quantize_group_fast<GS, RESIDUAL>(x, packed, sc, mn, one)) {
    load_raw<GS, BF16>(base, off, raw);
    unpack_raw<GS, BF16>(raw, x);
    codec::quantize_group<GS, RESIDUAL>(x, packed, sc, mn);
  }
}

// Plane rows of a tile's tokens: when its first and last token share a slab, the
// tile occupies consecutive rows from row0 (the common case: contiguous planes,
// or a tile inside one page); otherwise each token is looked up.
struct TileRows {
  long long row0;
  bool consecutive;
};

__device__ __forceinline__ TileRows tile_rows(const headq_cache& c, int b, int kv, int t_first,
                                              int nt) {
  const CacheSlab a = cache_slab(c, b, kv, t_first);
  const CacheSlab z = cache_slab(c, b, kv, t_first + nt - 1);
  if (a.slab >= 0 && a.slab == z.slab) return {a.slab * slab_rows(c) + a.off, true};
  return {-1, false};
}

__device__ __forceinline__ long long tile_row(const headq_cache& c, const TileRows& tr, int b,
                                              int kv, int t_first, int tt) {
  return tr.consecutive ? tr.row0 + tt : cache_row(c, b, kv, t_first + tt);
}

// Dense values whose cache dtype is the input dtype are copied as 16-byte chunks
// with consecutive lanes on consecutive chunks (whole rows of the tile), in
// batches of kBatch chunks per thread.
template <int D, bool BF16>
struct ValueCopy {
  static constexpr int kCPR = D * (BF16 ? 2 : 4) / 16;  // chunks per row
  static constexpr int kBatch = 4;
};

// The value of one (token, group): a plain copy when the cache holds the input
// dtype, else converted; or the 2-bit code of the full-KV composition.
template <int D, bool BF16>
__device__ __forceinline__ void store_value_group(const CacheWriteParams& p, size_t in_off,
                                                  RawGroup<group_size(D), BF16>& raw,
                                                  size_t row, int g) {
  constexpr int GS = group_size(D);
  constexpr int NG = num_groups(D);
  constexpr int NW = GS / 16 > 0 ? GS / 16 : 1;
  float vv[GS];
  if (p.c.vmode == HEADQ_V_2BIT) {
    uint32_t packed[NW];
    float sc, mn;
    quantize_raw<GS, false, BF16>(p.v, in_off, raw, vv, packed, sc, mn, p.one);
    codec::store_codes<GS>(p.c.v_codes + row * (D / 4) + g * (GS / 4), packed);
    p.c.v_scale[row * NG + g] = sc;
    p.c.v_min[row * NG + g] = mn;
    return;
  }
  const bool cache_bf16 = p.c.v_dtype == HEADQ_BF16;
  if (cache_bf16 == BF16) {  // same dtype: the input bits are the cached bits
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.c.v) +
                                          (row * D + g * GS) * (BF16 ? 2 : 4));
#pragma unroll
    for (int k = 0; k < RawGroup<GS, BF16>::kWords; ++k) dst[k] = raw.w[k];
    return;
  }
  unpack_raw<GS, BF16>(raw, vv);
  codec::store_values<GS>(p.c.v, row * D + g * GS, cache_bf16, vv);
}

// U_h of this KV head into the [r / RB][D][RB] tile, by 16-byte vectors (8-byte
// for RB 2): a vector's rows fall in one block.
template <int D, int RB>
__device__ __forceinline__ void load_basis(const CacheWriteParams& p, int kv, float* u_s) {
  using BT = BasisTile<D, RB>;
  constexpr int V = RB >= 4 ? 4 : 2;  // floats per vector
  const int r = p.c.r, rv = r / V;
  const float* U = p.U + static_cast<size_t>(kv) * D * r;
  for (int i = threadIdx.x; i < D * rv; i += kThreads) {
    const int c = i / rv, row = (i - c * rv) * V;
    float* dst = u_s + (row / RB) * BT::kBlock + c * RB + (row % RB);
    if constexpr (V == 4)
      *reinterpret_cast<float4*>(dst) = reinterpret_cast<const float4*>(U)[i];
    else
      *reinterpret_cast<float2*>(dst) = reinterpret_cast<const float2*>(U)[i];
  }
}

// y (RB rows, as packed pairs) += U[c][rows] * e, for one channel c (each
// product rounded, then each sum).
template <int RB>
__device__ __forceinline__ void muladd_rows(uint64_t (&y)[RB / 2], const float* u, uint64_t e2,
                                            uint64_t one2) {
  if constexpr (RB == 2) {
    codec::muladd2_pk(y[0], *reinterpret_cast<const uint64_t*>(u), e2, one2);
  } else {
#pragma unroll
    for (int k = 0; k < RB / 4; ++k) {
      const ulonglong2 uu = reinterpret_cast<const ulonglong2*>(u)[k];
      codec::muladd2_pk(y[2 * k], uu.x, e2, one2);
      codec::muladd2_pk(y[2 * k + 1], uu.y, e2, one2);
    }
  }
}

__device__ __forceinline__ float lo32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

// Phase B: from the tile's residuals, y = U_h^T e and the 4-bit side code of
// every token.  When the threads of a token are a power of two (aligned lanes
// of one warp) max|y| goes round by shuffles and each thread codes its own
// rows; otherwise y passes through shared memory first.
template <int D, int RB>
__device__ __forceinline__ void side_code_tile(const CacheWriteParams& p, const float* e_s,
                                               const float* u_s, float* y_s, int b, int kv,
                                               int tile0, int t0, const TileRows& tr) {
  using L = ResTile<D>;
  using BT = BasisTile<D, RB>;
  const int r = p.c.r, tid = threadIdx.x;
  const int bpt = r / RB;                      // threads per token
  const uint64_t one2 = codec::pk2(p.one, p.one);  // runtime 1.0: see codec::fma2
  const bool fused = (bpt & (bpt - 1)) == 0;   // kTT * bpt is a multiple of 32 either way
  for (int pr = tid; pr < kTT * bpt; pr += kThreads) {
    const int tt = pr / bpt, blk = pr - tt * bpt, i0 = blk * RB;
    uint64_t y[RB / 2];
#pragma unroll
    for (int k = 0; k < RB / 2; ++k) y[k] = 0ull;
    const float4* er = reinterpret_cast<const float4*>(e_s) + tt * L::RC;
    const float* ub = u_s + blk * BT::kBlock;
#pragma unroll 1
    for (int g = 0; g < L::NG; ++g) {  // rolled: keeps the loop in the instruction cache
#pragma unroll
      for (int j = 0; j < L::GS / 4; ++j) {
        const int c = g * L::GS + 4 * j;
        const float4 ev = er[g * L::GC + j];  // e_c .. e_c+3
        muladd_rows<RB>(y, ub + c * RB, codec::dup2(ev.x), one2);
        muladd_rows<RB>(y, ub + (c + 1) * RB, codec::dup2(ev.y), one2);
        muladd_rows<RB>(y, ub + (c + 2) * RB, codec::dup2(ev.z), one2);
        muladd_rows<RB>(y, ub + (c + 3) * RB, codec::dup2(ev.w), one2);
      }
    }
    const bool live = tile0 + tt < p.n;
    if (fused) {
      float a = 0.0f;
#pragma unroll
      for (int k = 0; k < RB / 2; ++k) a = fmax3(a, fabsf(lo32(y[k])), fabsf(hi32(y[k])));
      for (int m = 1; m < bpt; m <<= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, m));
      if (!live) continue;
      const long long row_s = tile_row(p.c, tr, b, kv, t0 + tile0, tt);
      if (row_s < 0) continue;
      const size_t row = static_cast<size_t>(row_s);
      const float s = codec::side_scale(a);
      const float rs = __frcp_rn(s);
      uint64_t bits = 0u;
#pragma unroll
      for (int k = 0; k < RB / 2; ++k) {
        const int w0 = codec::side_level(lo32(y[k]), s, rs);
        const int w1 = codec::side_level(hi32(y[k]), s, rs);
        bits |= static_cast<uint64_t>((w0 & 0xF) | ((w1 & 0xF) << 4)) << (8 * k);
      }
      uint8_t* dst = p.c.z_codes + row * (r / 2) + i0 / 2;
      if constexpr (RB == 2) *dst = static_cast<uint8_t>(bits);
      else if constexpr (RB == 4) *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(bits);
      else if constexpr (RB == 8) *reinterpret_cast<uint32_t*>(dst) = static_cast<uint32_t>(bits);
      else *reinterpret_cast<uint64_t*>(dst) = bits;
      if (blk == 0) p.c.z_scale[row] = s;
    } else if (live) {
#pragma unroll
      for (int k = 0; k < RB / 2; ++k) {
        y_s[tt * (r + 1) + i0 + 2 * k] = lo32(y[k]);
        y_s[tt * (r + 1) + i0 + 2 * k + 1] = hi32(y[k]);
      }
    }
  }
  if (fused) return;
  __syncthreads();
  // one byte (two rows) per thread
  const int pairs = r / 2;
  for (int pr = tid; pr < kTT * pairs; pr += kThreads) {
    const int tt = pr / pairs, i = 2 * (pr - tt * pairs);
    if (tile0 + tt >= p.n) continue;
    const float* y = y_s + tt * (r + 1);
    float a = 0.0f;
    for (int k = 0; k < r; ++k) a = fmaxf(a, fabsf(y[k]));
    const float s = codec::side_scale(a);
    const float rs = __frcp_rn(s);
    const int w0 = codec::side_level(y[i], s, rs);
    const int w1 = codec::side_level(y[i + 1], s, rs);
    const long long row_s = tile_row(p.c, tr, b, kv, t0 + tile0, tt);
    if (row_s < 0) continue;
    const size_t row = static_cast<size_t>(row_s);
    p.c.z_codes[row * (r / 2) + (i >> 1)] = static_cast<uint8_t>((w0 & 0xF) | ((w1 & 0xF) << 4));
    if (i == 0) p.c.z_scale[row] = s;
  }
}

// Shared-memory carve-up of both kernels: residual tile, basis tile, y rows
// (side code through shared memory) and, for the per-channel code, the block's
// per-channel minimum and scale.
template <int D, int RB>
__host__ __device__ inline size_t cache_write_smem_floats(int r, bool channel) {
  return static_cast<size_t>(ResTile<D>::kFloats) + BasisTile<D, RB>::floats(r) +
         static_cast<size_t>(kTT) * (r + 1) + (channel ? 2 * D : 0);
}

template <int D, int RB, bool BF16>
__global__ void __launch_bounds__(kThreads, BF16 ? 3 : 2)
cache_write_kernel(const CacheWriteParams p) {
  constexpr int GS = group_size(D);
  constexpr int NG = num_groups(D);
  constexpr int NW = GS / 16 > 0 ? GS / 16 : 1;
  using L = ResTile<D>;

  extern __shared__ float4 smem4[];
  const int r = p.c.r;
  float* e_s = reinterpret_cast<float*>(smem4);      // [kTT][RC chunks]
  float* u_s = e_s + L::kFloats;                     // [r/RB][D][RB] (+ pad)
  float* y_s = u_s + BasisTile<D, RB>::floats(r);    // [kTT][r + 1]

  const int b = blockIdx.z, kv = blockIdx.y;
  const int tile0 = blockIdx.x * kTT;
  const int tid = threadIdx.x;
  const size_t bk = static_cast<size_t>(b) * p.c.Hkv + kv;
  int t0 = p.t0;
  if (p.append) {  // one new token per sequence, at position T_b - 1
    const int Tb = p.seq_lens ? max(0, min(p.seq_lens[b], p.T)) : p.T;
    if (Tb == 0) return;
    t0 = Tb - 1;
  }
  if (r > 0) load_basis<D, RB>(p, kv, u_s);
  const int nt = min(kTT, p.n - tile0);
  const TileRows tr = tile_rows(p.c, b, kv, t0 + tile0, nt);

  // dense values in the input dtype: one contiguous copy of the tile's rows
  using VC = ValueCopy<D, BF16>;
  const bool v_copy = p.v != nullptr && p.c.vmode != HEADQ_V_2BIT &&
                      ((p.c.v_dtype == HEADQ_BF16) == BF16);
  const int v_chunks = nt * VC::kCPR;
  const uint4* v_src = v_copy ? reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.v) +
                                                               (bk * p.n + tile0) * D * (BF16 ? 2 : 4))
                              : nullptr;
  uint4* v_dst = reinterpret_cast<uint4*>(p.c.v);
  uint4 vb[VC::kBatch];
  auto v_load = [&](int base) {
#pragma unroll
    for (int j = 0; j < VC::kBatch; ++j) {
      const int i = base + j * kThreads + tid;
      if (i < v_chunks) vb[j] = v_src[i];
    }
  };
  auto v_store = [&](int base) {
    if (tr.consecutive) {  // the tile's rows are one contiguous run of the plane
      uint4* dst = v_dst + static_cast<size_t>(tr.row0) * VC::kCPR;
#pragma unroll
      for (int j = 0; j < VC::kBatch; ++j) {
        const int i = base + j * kThreads + tid;
        if (i < v_chunks) dst[i] = vb[j];
      }
      return;
    }
#pragma unroll
    for (int j = 0; j < VC::kBatch; ++j) {
      const int i = base + j * kThreads + tid;
      if (i >= v_chunks) continue;
      const int tt = i / VC::kCPR;
      const long long row_s = cache_row(p.c, b, kv, t0 + tile0 + tt);
      if (row_s >= 0) v_dst[static_cast<size_t>(row_s) * VC::kCPR + (i - tt * VC::kCPR)] = vb[j];
    }
  };
  // ---- phase A: base code, residual, values ---------------------------------
  // one (token, group) task: the keys' code and residual from kraw
  auto key_group = [&](int tt, int g, size_t in_off, size_t row, RawGroup<GS, BF16>& kraw) {
    float x[GS];
    uint32_t packed[NW];
    float sc, mn;
    quantize_raw<GS, true, BF16>(p.k, in_off, kraw, x, packed, sc, mn, p.one);  // x: the residual e
    codec::store_codes<GS>(p.c.k_codes + row * (D / 4) + g * (GS / 4), packed);
    p.c.k_scale[row * NG + g] = sc;
    p.c.k_min[row * NG + g] = mn;
    float4* er = reinterpret_cast<float4*>(e_s) + tt * L::RC + g * L::GC;
#pragma unroll
    for (int j = 0; j < GS / 4; ++j) er[j] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
  };
  if (v_copy) {
    v_load(0);
    bool stored = false;
    for (int task = tid; task < kTT * NG; task += kThreads) {
      const int tt = task / NG, g = task - tt * NG;
      if (tt >= nt) continue;
      const size_t in_off = (bk * p.n + tile0 + tt) * D + g * GS;
      RawGroup<GS, BF16> kraw;
      load_raw<GS, BF16>(p.k, in_off, kraw);
      if (!stored) {  // the copy's first batch, while the keys load
        v_store(0);
        stored = true;
      }
      const long long row_s = tile_row(p.c, tr, b, kv, t0 + tile0, tt);
      if (row_s < 0) continue;  // block-table entry outside the pool: not written
      key_group(tt, g, in_off, static_cast<size_t>(row_s), kraw);
    }
    if (!stored) v_store(0);
    for (int base = VC::kBatch * kThreads; base < v_chunks; base += VC::kBatch * kThreads) {
      v_load(base);
      v_store(base);
    }
  } else {
    for (int task = tid; task < kTT * NG; task += kThreads) {
      const int tt = task / NG, g = task - tt * NG;
      if (tt >= nt) continue;
      const size_t in_off = (bk * p.n + tile0 + tt) * D + g * GS;
      RawGroup<GS, BF16> kraw, vraw;
      load_raw<GS, BF16>(p.k, in_off, kraw);
      if (p.v != nullptr) load_raw<GS, BF16>(p.v, in_off, vraw);
      const long long row_s = tile_row(p.c, tr, b, kv, t0 + tile0, tt);
      if (row_s < 0) continue;
      const size_t row = static_cast<size_t>(row_s);
      key_group(tt, g, in_off, row, kraw);
      if (p.v != nullptr) store_value_group<D, BF16>(p, in_off, vraw, row, g);
    }
  }
  if (r == 0) return;  // no side code
  __syncthreads();
  side_code_tile<D, RB>(p, e_s, u_s, y_s, b, kv, tile0, t0, tr);
}

// The alternative base code, per channel over a block of 64 tokens: the CTA's
// tile is one block (writes start on a block boundary).  Phase A1 stages the
// keys (in the residual tile's layout) and stores the values; A2, one thread per
// channel: minimum, maximum and scale over the block's tokens; A3, one thread
// per (token, 4 channels): codes, packed byte, residual in place.  Every step is
// the same IEEE fp32 operation as in the per-token code.
template <int D, int RB, bool BF16>
__global__ void __launch_bounds__(kThreads, BF16 ? 3 : 2)
cache_write_channel_kernel(const CacheWriteParams p) {
  constexpr int GS = group_size(D);
  constexpr int NG = num_groups(D);
  using L = ResTile<D>;
  static_assert(D <= kThreads, "one thread per channel");

  extern __shared__ float4 smem4[];
  const int r = p.c.r;
  float* e_s = reinterpret_cast<float*>(smem4);      // [kTT][RC chunks]: keys, then residuals
  float* u_s = e_s + L::kFloats;
  float* y_s = u_s + BasisTile<D, RB>::floats(r);
  float* mn_s = y_s + kTT * (r + 1);                 // [D]
  float* sc_s = mn_s + D;                            // [D]

  const int b = blockIdx.z, kv = blockIdx.y;
  const int tile0 = blockIdx.x * kTT;
  const int tid = threadIdx.x;
  const size_t bk = static_cast<size_t>(b) * p.c.Hkv + kv;
  const int t0 = p.t0;
  const int nt = min(kTT, p.n - tile0);
  const TileRows tr = tile_rows(p.c, b, kv, t0 + tile0, nt);
  if (r > 0) load_basis<D, RB>(p, kv, u_s);

  // A1: the block's keys, and the values (as for the per-token code)
  for (int task = tid; task < kTT * NG; task += kThreads) {
    const int tt = task / NG, g = task - tt * NG;
    if (tt >= nt) continue;
    const size_t in_off = (bk * p.n + tile0 + tt) * D + g * GS;
    RawGroup<GS, BF16> kraw, vraw;
    load_raw<GS, BF16>(p.k, in_off, kraw);
    if (p.v != nullptr) load_raw<GS, BF16>(p.v, in_off, vraw);
    float x[GS];
    unpack_raw<GS, BF16>(kraw, x);
    float4* er = reinterpret_cast<float4*>(e_s) + tt * L::RC + g * L::GC;
#pragma unroll
    for (int j = 0; j < GS / 4; ++j) er[j] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
    if (p.v != nullptr) {
      const long long row_s = tile_row(p.c, tr, b, kv, t0 + tile0, tt);
      if (row_s >= 0) store_value_group<D, BF16>(p, in_off, vraw, static_cast<size_t>(row_s), g);
    }
  }
  __syncthreads();
  const long long brow_s = cache_row(p.c, b, kv, t0 + tile0);  // the block's first row
  // A2: per channel, over the block's tokens
  if (tid < D) {
    const int o = L::off(tid);
    float lo = e_s[o], hi = e_s[o];
    for (int tt = 1; tt < nt; ++tt) {
      lo = fminf(lo, e_s[tt * 4 * L::RC + o]);
      hi = fmaxf(hi, e_s[tt * 4 * L::RC + o]);
    }
    lo = __fadd_rn(lo, 0.0f);  // a -0 extreme is stored as +0
    hi = __fadd_rn(hi, 0.0f);
    const float scale = __fdiv_rn(__fsub_rn(hi, lo), 3.0f);
    mn_s[tid] = lo;
    sc_s[tid] = scale;
    if (brow_s >= 0) {
      const size_t brow = static_cast<size_t>(brow_s) >> 6;
      p.c.k_min[brow * D + tid] = lo;
      p.c.k_scale[brow * D + tid] = scale;
    }
  }
  __syncthreads();
  // A3: codes of 4 channels of one token -> one byte; residuals in place
  for (int task = tid; task < kTT * (D / 4); task += kThreads) {
    const int tt = task / (D / 4), c4 = (task - tt * (D / 4)) * 4;
    if (tt >= nt) continue;
    float4* ch = reinterpret_cast<float4*>(e_s + tt * 4 * L::RC + L::off(c4));
    const float4 h = *ch;
    const float xs[4] = {h.x, h.y, h.z, h.w};
    float res[4];
    uint32_t byte = 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = c4 + k;
      const float x = xs[k], lo = mn_s[c], scale = sc_s[c];
      int code = 0;
      if (scale != 0.0f) {
        const float tq = codec::rint_quot(__fsub_rn(x, lo), scale, __frcp_rn(scale));
        code = tq < 0.0f ? 0 : (tq > 3.0f ? 3 : static_cast<int>(tq));
      }
      byte |= static_cast<uint32_t>(code) << (2 * k);
      res[k] = __fsub_rn(x, __fadd_rn(lo, __fmul_rn(static_cast<float>(code), scale)));
    }
    *ch = make_float4(res[0], res[1], res[2], res[3]);
    const long long row_s = tile_row(p.c, tr, b, kv, t0 + tile0, tt);
    if (row_s >= 0) p.c.k_codes[static_cast<size_t>(row_s) * (D / 4) + c4 / 4] = static_cast<uint8_t>(byte);
  }
  if (r == 0) return;
  __syncthreads();  // residuals complete
  side_code_tile<D, RB>(p, e_s, u_s, y_s, b, kv, tile0, t0, tr);
}

template <int D, int RB>
cudaError_t launch_rb(const CacheWriteParams& p, cudaStream_t s) {
  const bool channel = p.c.kmode == HEADQ_K_CHANNEL;
  if (channel && D > kThreads) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * cache_write_smem_floats<D, RB>(p.c.r, channel);
  dim3 grid((p.n + kTT - 1) / kTT, p.c.Hkv, p.c.B);
  auto k = channel ? (p.in_bf16 ? cache_write_channel_kernel<D, RB, true>
                               : cache_write_channel_kernel<D, RB, false>)
                   : (p.in_bf16 ? cache_write_kernel<D, RB, true> : cache_write_kernel<D, RB, false>);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  k<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// RB side rows per phase-B thread: half the rank when that is 16, 8, 4 or 2 (two
// threads per token: four warps of the CTA share the projection, and U_h reads
// stay two addresses per warp instruction); else the largest of 8, 4, 2 dividing r.
template <int D>
cudaError_t launch_d(const CacheWriteParams& p, cudaStream_t s) {
  const int r = p.c.r;
  if constexpr (D >= 32)
    if (r == 32) return launch_rb<D, 16>(p, s);
  if (r == 16) return launch_rb<D, 8>(p, s);
  if (r == 8) return launch_rb<D, 4>(p, s);
  if (r == 4) return launch_rb<D, 2>(p, s);
  if (r % 8 == 0) return launch_rb<D, 8>(p, s);
  if (r % 4 == 0) return launch_rb<D, 4>(p, s);
  return launch_rb<D, 2>(p, s);
}

}  // namespace

cudaError_t launch_cache_write(const CacheWriteParams& p0, cudaStream_t s) {
  CacheWriteParams p = p0;
  p.one = 1.0f;  // see codec::fma2
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
