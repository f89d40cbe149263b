// HeadQ cache write: the base 2-bit key code, the residual, its projection onto
// the query-PCA basis U_h and the 4-bit side code ("HeadQ: Model-Visible
// Distortion and Score-Space Correction for KV-Cache Quantization", gist.science
// summary, section 3, step 2), plus the value store (dense copy, or the same
// 2-bit code for the full-KV composition of section 5).
//
// Bit-exact: every codec operation is one IEEE fp32 operation (codec.cuh; this
// file is also compiled with -fmad=false).
//
// One CTA per (64-token tile, kv, b), three phases:
//   A  one thread per (token, 32-channel group): vector loads of the group's keys
//      and values straight from HBM (all issued before any arithmetic), base code,
//      codes/scale/min stored, residual e -> shared memory, values stored/coded
//   B  one thread per (token, 8 side rows): y = U_h^T e in channel order, one
//      fused multiply-add per term, two rows per packed fp32x2 FMA
//   C  one thread per (token, pair of side rows): absmax scale and the two nibbles
#include "codec.cuh"

namespace headq {
namespace {

constexpr int kTT = 64;        // tokens per CTA
constexpr int kThreads = 256;

// The value of token tt, group g of the tile: dense copy or 2-bit code.
template <int D>
__device__ __forceinline__ void store_value_group(const CacheWriteParams& p, size_t in_off,
                                                  size_t row, int g) {
  constexpr int GS = group_size(D);
  constexpr int NG = num_groups(D);
  constexpr int NW = GS / 16 > 0 ? GS / 16 : 1;
  float vv[GS];
  codec::load_row<GS>(p.v, in_off, p.in_bf16, vv);
  if (p.c.vmode == HEADQ_V_2BIT) {
    uint32_t packed[NW];
    float sc, mn;
    codec::quantize_group<GS, false>(vv, packed, sc, mn);
    codec::store_codes<GS>(p.c.v_codes + row * (D / 4) + g * (GS / 4), packed);
    p.c.v_scale[row * NG + g] = sc;
    p.c.v_min[row * NG + g] = mn;
  } else {
    codec::store_values<GS>(p.c.v, row * D + g * GS, p.c.v_dtype == HEADQ_BF16, vv);
  }
}

// Phases B and C, shared by both base codes: from the residuals e_s of the
// tile's tokens, y = U_h^T e and the 4-bit side code of every token.
template <int D, int RB>
__device__ __forceinline__ void side_code_tile(const CacheWriteParams& p, float* e_s, float* u_s,
                                               float* y_s, int b, int kv, int tile0, int t0) {
  constexpr int ES = D + 4;
  const int r = p.c.r, tid = threadIdx.x;
  {
    const float4* U4 = reinterpret_cast<const float4*>(p.U + static_cast<size_t>(kv) * D * r);
    for (int i = tid; i < D * r / 4; i += kThreads) reinterpret_cast<float4*>(u_s)[i] = U4[i];
  }
  __syncthreads();

  // ---- phase B: y = U_h^T e, channel order, one FMA per term ---------------
  // RB side rows per thread as RB/2 packed pairs, one fp32x2 FMA per pair and
  // channel (the pairs and U stay in 64-bit registers)
  const int blocks_per_tok = r / RB;
  for (int pr = tid; pr < kTT * blocks_per_tok; pr += kThreads) {
    const int tt = pr / blocks_per_tok;
    const int i0 = (pr - tt * blocks_per_tok) * RB;
    if (tile0 + tt >= p.n) continue;
    uint64_t y[RB / 2];
#pragma unroll
    for (int k = 0; k < RB / 2; ++k) y[k] = 0ull;
    const float* er = e_s + tt * ES;
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      const uint64_t e2 = codec::dup2(er[c]);
      const uint64_t* ur = reinterpret_cast<const uint64_t*>(u_s + c * r + i0);
      if constexpr (RB >= 4) {
#pragma unroll
        for (int k = 0; k < RB / 4; ++k) {
          const ulonglong2 u = reinterpret_cast<const ulonglong2*>(ur)[k];
          codec::fma2_pk(y[2 * k], u.x, e2);
          codec::fma2_pk(y[2 * k + 1], u.y, e2);
        }
      } else {
        codec::fma2_pk(y[0], ur[0], e2);
      }
    }
#pragma unroll
    for (int k = 0; k < RB / 2; ++k) {
      y_s[tt * (r + 1) + i0 + 2 * k] = __uint_as_float(static_cast<uint32_t>(y[k]));
      y_s[tt * (r + 1) + i0 + 2 * k + 1] = __uint_as_float(static_cast<uint32_t>(y[k] >> 32));
    }
  }
  __syncthreads();

  // ---- phase C: side code, one byte (two rows) per thread --------------------
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
    const long long row_s = cache_row(p.c, b, kv, t0 + tile0 + tt);
    if (row_s < 0) continue;
    const size_t row = static_cast<size_t>(row_s);
    p.c.z_codes[row * (r / 2) + (i >> 1)] = static_cast<uint8_t>((w0 & 0xF) | ((w1 & 0xF) << 4));
    if (i == 0) p.c.z_scale[row] = s;
  }
}

template <int D, int RB>
__global__ void __launch_bounds__(kThreads, 3)
cache_write_kernel(const CacheWriteParams p) {
  constexpr int GS = group_size(D);
  constexpr int NG = num_groups(D);
  constexpr int NW = GS / 16 > 0 ? GS / 16 : 1;
  constexpr int ES = D + 4;  // residual row stride (floats): 16-byte rows, spread banks

  extern __shared__ float smem[];
  const int r = p.c.r;
  float* e_s = smem;                 // [kTT][ES]
  float* u_s = e_s + kTT * ES;       // [D][r]
  float* y_s = u_s + D * r;          // [kTT][r + 1]

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

  // ---- phase A: base code, residual, values ---------------------------------
  for (int task = tid; task < kTT * NG; task += kThreads) {
    const int tt = task / NG, g = task - tt * NG;
    const int t = tile0 + tt;
    if (t >= p.n) continue;
    const size_t in_off = (bk * p.n + t) * D + g * GS;
    const long long row_s = cache_row(p.c, b, kv, t0 + t);
    if (row_s < 0) continue;  // block-table entry outside the pool: not written
    const size_t row = static_cast<size_t>(row_s);
    float x[GS];
    codec::load_row<GS>(p.k, in_off, p.in_bf16, x);
    uint32_t packed[NW];
    float sc, mn;
    codec::quantize_group<GS, true>(x, packed, sc, mn);  // x becomes the residual e
    codec::store_codes<GS>(p.c.k_codes + row * (D / 4) + g * (GS / 4), packed);
    p.c.k_scale[row * NG + g] = sc;
    p.c.k_min[row * NG + g] = mn;
#pragma unroll
    for (int k = 0; k < GS; k += 4)
      *reinterpret_cast<float4*>(e_s + tt * ES + g * GS + k) =
          make_float4(x[k], x[k + 1], x[k + 2], x[k + 3]);
    if (p.v != nullptr) store_value_group<D>(p, in_off, row, g);
  }
  if (r == 0) return;  // no side code
  side_code_tile<D, RB>(p, e_s, u_s, y_s, b, kv, tile0, t0);
}

// The alternative base code, per channel over a block of 64 tokens: the CTA's
// tile is one block (writes start on a block boundary).  Phase A1 stages the
// keys; A2, one thread per channel: minimum, maximum and scale over the block's
// tokens; A3, one thread per (token, 4 channels): codes, packed byte, residual.
// Every step is the same IEEE fp32 operation as in the per-token code.
template <int D, int RB>
__global__ void __launch_bounds__(kThreads, 3)
cache_write_channel_kernel(const CacheWriteParams p) {
  constexpr int GS = group_size(D);
  constexpr int NG = num_groups(D);
  constexpr int ES = D + 4;
  static_assert(D <= kThreads, "one thread per channel");

  extern __shared__ float smem[];
  const int r = p.c.r;
  float* e_s = smem;                 // [kTT][ES]   keys, then residuals
  float* u_s = e_s + kTT * ES;       // [D][r]      (phase A2 borrows it: [2][D])
  float* y_s = u_s + D * (r > 2 ? r : 2);

  const int b = blockIdx.z, kv = blockIdx.y;
  const int tile0 = blockIdx.x * kTT;
  const int tid = threadIdx.x;
  const size_t bk = static_cast<size_t>(b) * p.c.Hkv + kv;
  const int t0 = p.t0;
  const int nt = min(kTT, p.n - tile0);

  // A1: the block's keys, and the values (as for the per-token code)
  for (int task = tid; task < kTT * NG; task += kThreads) {
    const int tt = task / NG, g = task - tt * NG;
    if (tt >= nt) continue;
    const size_t in_off = (bk * p.n + tile0 + tt) * D + g * GS;
    float x[GS];
    codec::load_row<GS>(p.k, in_off, p.in_bf16, x);
#pragma unroll
    for (int k = 0; k < GS; k += 4)
      *reinterpret_cast<float4*>(e_s + tt * ES + g * GS + k) =
          make_float4(x[k], x[k + 1], x[k + 2], x[k + 3]);
    if (p.v != nullptr) {
      const long long row_s = cache_row(p.c, b, kv, t0 + tile0 + tt);
      if (row_s >= 0) store_value_group<D>(p, in_off, static_cast<size_t>(row_s), g);
    }
  }
  __syncthreads();
  const long long brow_s = cache_row(p.c, b, kv, t0 + tile0);  // the block's first row
  float* mn_s = u_s;
  float* sc_s = u_s + D;
  // A2: per channel, over the block's tokens
  if (tid < D) {
    float lo = e_s[tid], hi = e_s[tid];
    for (int tt = 1; tt < nt; ++tt) {
      lo = fminf(lo, e_s[tt * ES + tid]);
      hi = fmaxf(hi, e_s[tt * ES + tid]);
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
    uint32_t byte = 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = c4 + k;
      const float x = e_s[tt * ES + c], lo = mn_s[c], scale = sc_s[c];
      int code = 0;
      if (scale != 0.0f) {
        const float tq = codec::rint_quot(__fsub_rn(x, lo), scale, __frcp_rn(scale));
        code = tq < 0.0f ? 0 : (tq > 3.0f ? 3 : static_cast<int>(tq));
      }
      byte |= static_cast<uint32_t>(code) << (2 * k);
      e_s[tt * ES + c] = __fsub_rn(x, __fadd_rn(lo, __fmul_rn(static_cast<float>(code), scale)));
    }
    const long long row_s = cache_row(p.c, b, kv, t0 + tile0 + tt);
    if (row_s >= 0) p.c.k_codes[static_cast<size_t>(row_s) * (D / 4) + c4 / 4] = static_cast<uint8_t>(byte);
  }
  if (r == 0) return;
  __syncthreads();  // residuals complete; u_s is reloaded with U below
  side_code_tile<D, RB>(p, e_s, u_s, y_s, b, kv, tile0, t0);
}

template <int D>
cudaError_t launch_d(const CacheWriteParams& p, cudaStream_t s) {
  const int r = p.c.r;
  const bool channel = p.c.kmode == HEADQ_K_CHANNEL;
  if (channel && D > kThreads) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * (static_cast<size_t>(kTT) * (D + 4) +
                                       static_cast<size_t>(D) * (r > 2 ? r : 2) +
                                       static_cast<size_t>(kTT) * (r + 1));
  dim3 grid((p.n + kTT - 1) / kTT, p.c.Hkv, p.c.B);
  auto k = channel ? (r % 8 == 0 ? cache_write_channel_kernel<D, 8>
                                 : (r % 4 == 0 ? cache_write_channel_kernel<D, 4>
                                               : cache_write_channel_kernel<D, 2>))
                   : (r % 8 == 0 ? cache_write_kernel<D, 8>
                                 : (r % 4 == 0 ? cache_write_kernel<D, 4> : cache_write_kernel<D, 2>));
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
