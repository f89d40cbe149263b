// HeadQ decode attention (cache read): "HeadQ: Model-Visible Distortion and
// Score-Space Correction for KV-Cache Quantization", gist.science summary,
// section 3, step 3 -- the runtime query turns the stored side code into an
// additive logit correction,
//   s^_j = sm_scale * ( q . k^base_j + sigma * (U_h^T q) . z^_j ),
// followed by softmax and the attention-weighted readout o = sum_j p_j v_j
// (section 2.2).
//
// The base-code logit is evaluated in factored form: with group sums
// Q_g = sum_{c in g} q_c,
//   q . k^base_j = sum_g ( min_{j,g} Q_g + scale_{j,g} sum_{c in g} q_c code_{j,c} ),
// which is exact algebra of the dequantisation min + code*scale, so each code is
// used once per query head without rebuilding the key.
//
// Split-T flash decoding: CTA (split, kv, b) covers a contiguous chunk of tokens
// for the G query heads of one KV head and keeps a running max m, sum l and
// unnormalised output o (online softmax); a combine kernel merges the splits by
// their log-sum-exp.  When there is a single split the CTA writes the result.
#include <math.h>

#include <algorithm>

#include "headq_internal.cuh"

namespace headq {
namespace {

constexpr int kTile = 32;      // tokens per inner step (one per lane in phase 2)
constexpr int kThreads = 128;
constexpr int kMaxOut = 16;    // (G * d) / kThreads outputs per thread at most
static_assert(kThreads == 4 * kTile, "phase 1 maps the four warps to four channel quarters");
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// A staged tile row of 2-bit key codes: d/16 32-bit words (for d = 8, the row's
// two bytes in one word); rows padded by one word so that the 32 tokens a warp
// reads at once fall in distinct banks.
template <int D>
struct CodeRow {
  static constexpr int kWords = D >= 16 ? D / 16 : 1;
  static constexpr int kCodes = D >= 16 ? 16 : D;  // codes per word
  static constexpr int kStride = kWords + 1;
};

// Code k of w as an exact float: the bits of 2^23 + code, less 2^23 (an FMA-pipe
// add instead of an integer conversion).
__device__ __forceinline__ float code_f(uint32_t w, int k) {
  return __int_as_float(0x4B000000u | ((w >> (2 * k)) & 3u)) - 8388608.0f;
}

// Generic split kernel, every shape the tensor-core kernel does not take.  Per
// 32-token tile: the tile's codes, scales, side codes and values are staged in
// shared memory with vector loads; one thread per (head, token) forms the logit
// from the staged code words; one warp per head updates the online softmax; one
// thread per (channel, head set) accumulates p_j v_j.
template <int D, int GM>
__global__ void __launch_bounds__(kThreads, D >= 256 ? 2 : 4)
decode_split_kernel(const DecodeParams p) {
  // (G * d) / kThreads outputs per thread: at most GM * d / kThreads for G <= GM;
  // the 16-head batch also serves G > 16 (several passes), up to kMaxOut (G * d <= 2048)
  constexpr int KO = GM == 16 ? kMaxOut
                              : (GM * D / kThreads < 1 ? 1
                                                       : (GM * D / kThreads > kMaxOut ? kMaxOut
                                                                                      : GM * D / kThreads));
  constexpr int NG = num_groups(D);
  constexpr int GS = group_size(D);
  using CR = CodeRow<D>;
  constexpr int KS = NG + 1;  // padded row of per-token group scales / minima
  const int G = p.G, r = p.c.r;
  const bool channel = p.c.kmode == HEADQ_K_CHANNEL;
  const int ZB = r > 0 ? ((r / 2 + 3) / 4 + 1) * 4 : 0;  // padded side-code row, bytes
  extern __shared__ float4 sm4[];
  float* v_s = reinterpret_cast<float*>(sm4);  // [kTile][D] the tile's values (float4 stores)
  float* q_s = v_s + kTile * D;      // [G][D]
  float* qs_s = q_s + G * D;         // [G][D]    per-channel code: q * scale of the block
  float* qg_s = qs_s + (channel ? G * D : 0);  // [G][NG] group sums of q
  float* qt_s = qg_s + G * NG;       // [G][r]    sigma * U_h^T q
  float* s_s = qt_s + G * r;         // [G][kTile] weights
  float* ps_s = s_s + G * kTile;     // [4][G][kTile] partial logits of the channel quarters
  float* m_s = ps_s + 4 * G * kTile; // [G]
  float* l_s = m_s + G;              // [G]
  float* a_s = l_s + G;              // [G]
  float* qm_s = a_s + G;             // [G]       per-channel code: q . minimum of the block
  float* ks_s = qm_s + G;            // [kTile][KS] per-token code: group scales
  float* km_s = ks_s + kTile * KS;   // [kTile][KS] and minima
  float* zs_s = km_s + kTile * KS;   // [kTile] side scales
  uint32_t* kc_s = reinterpret_cast<uint32_t*>(zs_s + kTile);  // [kTile][CR::kStride]
  uint8_t* zb_s = reinterpret_cast<uint8_t*>(kc_s + kTile * CR::kStride);  // [kTile][ZB]

  const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int Tb = p.T;
  if (p.seq_lens) Tb = max(0, min(p.seq_lens[b], p.T));
  const int t_begin = split * p.chunk;
  const int t_end = min(Tb, t_begin + p.chunk);
  const int h0 = kv * G;

  for (int i = tid; i < G * D; i += kThreads)
    q_s[i] = load_elem(p.q, (static_cast<size_t>(b) * p.Hq + h0) * D + i, p.q_bf16);
  for (int h = tid; h < G; h += kThreads) {
    m_s[h] = -INFINITY;
    l_s[h] = 0.0f;
  }
  __syncthreads();
  for (int i = tid; i < G * NG; i += kThreads) {
    const int h = i / NG, g = i - h * NG;
    float acc = 0.0f;
    for (int c = 0; c < GS; ++c) acc += q_s[h * D + g * GS + c];
    qg_s[i] = acc;
  }
  for (int i = tid; i < G * r; i += kThreads) {
    const int h = i / r, ii = i - h * r;
    const float* U = p.U + static_cast<size_t>(kv) * D * r;
    float acc = 0.0f;
    for (int c = 0; c < D; ++c) acc = fmaf(U[c * r + ii], q_s[h * D + c], acc);
    qt_s[i] = p.corr_sign * acc;
  }

  float o[KO];
#pragma unroll
  for (int k = 0; k < KO; ++k) o[k] = 0.0f;

  for (int t0 = t_begin; t0 < t_end; t0 += kTile) {
    const int nt = min(kTile, t_end - t0);
    // the tile's rows are consecutive: chunks start at multiples of 64 tokens
    const size_t row0 = cache_row_read(p.c, b, kv, t0, tid == 0 ? p.err : nullptr);
    // ---- staging ------------------------------------------------------------
    if constexpr (D >= 16) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(p.c.k_codes + row0 * (D / 4));
      for (int e = tid; e < nt * CR::kWords; e += kThreads) {
        const int j = e / CR::kWords, w = e - j * CR::kWords;
        kc_s[j * CR::kStride + w] = src[e];
      }
    } else {
      const uint16_t* src = reinterpret_cast<const uint16_t*>(p.c.k_codes + row0 * (D / 4));
      for (int j = tid; j < nt; j += kThreads) kc_s[j * CR::kStride] = src[j];
    }
    if (!channel) {
      for (int e = tid; e < nt * NG; e += kThreads) {
        const int j = e / NG, g = e - j * NG;
        ks_s[j * KS + g] = p.c.k_scale[row0 * NG + e];
        km_s[j * KS + g] = p.c.k_min[row0 * NG + e];
      }
    } else if (((t0 - t_begin) & 63) == 0) {  // a new 64-token block: fold its scale into q
      const size_t bi = (row0 >> 6) * D;
      for (int i = tid; i < G * D; i += kThreads) qs_s[i] = q_s[i] * p.c.k_scale[bi + (i % D)];
      for (int h = warp; h < G; h += kThreads / 32) {
        float acc = 0.0f;
        for (int c = lane; c < D; c += 32) acc = fmaf(q_s[h * D + c], p.c.k_min[bi + c], acc);
        acc = warp_sum(acc);
        if (lane == 0) qm_s[h] = acc;
      }
    }
    if (r > 0) {
      for (int e = tid; e < nt * (r / 2); e += kThreads) {
        const int j = e / (r / 2), i = e - j * (r / 2);
        zb_s[j * ZB + i] = p.c.z_codes[row0 * (r / 2) + e];
      }
      for (int j = tid; j < nt; j += kThreads) zs_s[j] = p.c.z_scale[row0 + j];
    }
    if (p.c.vmode == HEADQ_V_2BIT) {  // one thread per (token, 4 channels)
      for (int e = tid; e < nt * (D / 4); e += kThreads) {
        const int j = e / (D / 4), c4 = e - j * (D / 4), g = (4 * c4) / GS;
        const size_t row = row0 + j;
        const uint32_t cb = p.c.v_codes[row * (D / 4) + c4];
        const float vsc = p.c.v_scale[row * NG + g], vmn = p.c.v_min[row * NG + g];
        float4 v;
        v.x = __fadd_rn(vmn, __fmul_rn(static_cast<float>(cb & 3u), vsc));
        v.y = __fadd_rn(vmn, __fmul_rn(static_cast<float>((cb >> 2) & 3u), vsc));
        v.z = __fadd_rn(vmn, __fmul_rn(static_cast<float>((cb >> 4) & 3u), vsc));
        v.w = __fadd_rn(vmn, __fmul_rn(static_cast<float>(cb >> 6), vsc));
        *reinterpret_cast<float4*>(v_s + j * D + 4 * c4) = v;
      }
    } else if (p.c.v_dtype == HEADQ_BF16) {  // one thread per (token, 8 channels)
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.c.v) + row0 * D);
      for (int e = tid; e < nt * (D / 8); e += kThreads) {
        const uint4 u = src[e];
        float* dst = v_s + 8 * e;
        *reinterpret_cast<float4*>(dst) =
            make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                        __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
        *reinterpret_cast<float4*>(dst + 4) =
            make_float4(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xffff0000u),
                        __uint_as_float(u.w << 16), __uint_as_float(u.w & 0xffff0000u));
      }
    } else {  // fp32
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.c.v) + row0 * D);
      for (int e = tid; e < nt * (D / 4); e += kThreads)
        reinterpret_cast<float4*>(v_s)[e] = src[e];
    }
    __syncthreads();
    // ---- phase 1: partial logits; warp = quarter of the channels, lane = token --
    // Each code is decoded once for a batch of GM heads; a warp's lanes read the
    // same query words (broadcasts) and code rows 9 words apart (distinct banks).
    // The softmax warps add the four quarters in a fixed order.
    {
      constexpr int NP = kThreads / kTile;  // quarters (one per warp)
      constexpr int PS = D / NP;            // channels per thread
      constexpr int CS = PS >= 4 ? 4 : PS;  // channels per step
      const int j = lane, part = warp;
      const bool live = j < nt;
      const int c0 = part * PS;
      const uint32_t* kw = kc_s + j * CR::kStride;
      for (int hb = 0; hb < G; hb += GM) {  // one pass unless G > 16
        const int gn = min(GM, G - hb);
        float acc[GM];
#pragma unroll
        for (int h = 0; h < GM; ++h) acc[h] = 0.0f;
        // sum_{c in [cb, cb + n)} q'_{h,c} code_c into sum[h], q' rows at qb
        auto dot = [&](const float* qb, int cb, int n, float (&sum)[GM]) {
#pragma unroll
          for (int i = 0; i < n; i += CS) {
            const int c = cb + i;
            const uint32_t word = kw[c / CR::kCodes] >> (2 * (c % CR::kCodes));
            float e[CS];
#pragma unroll
            for (int k = 0; k < CS; ++k) e[k] = code_f(word, k);
#pragma unroll
            for (int h = 0; h < GM; ++h) {
              if (h < gn) {
                const float* qh = qb + h * D + c;
                if constexpr (CS == 4) {
                  const float4 q4 = *reinterpret_cast<const float4*>(qh);
                  sum[h] = fmaf(q4.x, e[0], sum[h]);
                  sum[h] = fmaf(q4.y, e[1], sum[h]);
                  sum[h] = fmaf(q4.z, e[2], sum[h]);
                  sum[h] = fmaf(q4.w, e[3], sum[h]);
                } else {
#pragma unroll
                  for (int k = 0; k < CS; ++k) sum[h] = fmaf(qh[k], e[k], sum[h]);
                }
              }
            }
          }
        };
        if (live) {
          if (channel) {  // q.k^ = q.min + sum_c (q_c scale_c) code_c, per block
            if (part == 0) {
#pragma unroll
              for (int h = 0; h < GM; ++h)
                if (h < gn) acc[h] = qm_s[hb + h];
            }
            dot(qs_s + hb * D, c0, PS, acc);
          } else {  // sum_g ( min_g Q_g + scale_g sum_{c in g} q_c code_c )
            constexpr int SEG = PS < GS ? PS : GS;  // channels of one group in this thread
#pragma unroll
            for (int sg = 0; sg < PS / SEG; ++sg) {
              const int cb = c0 + sg * SEG, g = cb / GS;
              float pg[GM];
#pragma unroll
              for (int h = 0; h < GM; ++h) pg[h] = 0.0f;
              dot(q_s + hb * D, cb, SEG, pg);
              const float km = km_s[j * KS + g], ks = ks_s[j * KS + g];
              const bool first = cb % GS == 0;  // this thread holds the group's start
#pragma unroll
              for (int h = 0; h < GM; ++h) {
                if (h < gn) {
                  if (first) acc[h] = fmaf(km, qg_s[(hb + h) * NG + g], acc[h]);
                  acc[h] = fmaf(ks, pg[h], acc[h]);
                }
              }
            }
          }
          if (r > 0) {  // side rows part, part + NP, ...
            const uint8_t* zr = zb_s + j * ZB;
            float cz[GM];
#pragma unroll
            for (int h = 0; h < GM; ++h) cz[h] = 0.0f;
            for (int i = part; i < r; i += NP) {
              const float w = static_cast<float>(nibble(zr, i));
#pragma unroll
              for (int h = 0; h < GM; ++h)
                if (h < gn) cz[h] = fmaf(qt_s[(hb + h) * r + i], w, cz[h]);
            }
            const float zs = zs_s[j];
#pragma unroll
            for (int h = 0; h < GM; ++h) acc[h] = fmaf(zs, cz[h], acc[h]);
          }
        }
#pragma unroll
        for (int h = 0; h < GM; ++h)
          if (h < gn) ps_s[(part * G + hb + h) * kTile + j] = acc[h];
      }
    }
    __syncthreads();
    // ---- phase 2: online softmax update, one warp per head --------------------
    for (int h = warp; h < G; h += kThreads / 32) {
      const float* ph = ps_s + h * kTile + lane;
      const float s = lane < nt ? ((ph[0] + ph[G * kTile]) + (ph[2 * G * kTile] + ph[3 * G * kTile])) *
                                      p.sm_scale
                                : -INFINITY;
      const float m_old = m_s[h];
      const float m_new = fmaxf(m_old, warp_max(s));
      const float pj = lane < nt ? expf(s - m_new) : 0.0f;
      const float alpha = expf(m_old - m_new);
      const float sum = warp_sum(pj);
      s_s[h * kTile + lane] = pj;
      __syncwarp();
      if (lane == 0) {
        l_s[h] = l_s[h] * alpha + sum;
        m_s[h] = m_new;
        a_s[h] = alpha;
      }
    }
    __syncthreads();
    // ---- phase 3: rescale and accumulate p_j v_j ------------------------------
#pragma unroll
    for (int k = 0; k < KO; ++k) {
      const int idx = tid + k * kThreads;
      if (idx < G * D) {
        const int h = idx / D, c = idx - h * D;
        float acc = o[k] * a_s[h];
        const float* pw = s_s + h * kTile;
        for (int j = 0; j < nt; ++j) acc = fmaf(pw[j], v_s[j * D + c], acc);
        o[k] = acc;
      }
    }
    __syncthreads();
  }

  // epilogue: partial (o, m, l) or the final result
  const PartView pv = part_view(p.part, static_cast<size_t>(p.c.B) * p.Hq, p.splits, D);
#pragma unroll
  for (int k = 0; k < KO; ++k) {
    const int idx = tid + k * kThreads;
    if (idx < G * D) {
      const int h = idx / D, c = idx - h * D;
      const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
      if (p.splits == 1) {
        const float l = l_s[h];
        p.out[bh * D + c] = l > 0.0f ? o[k] / l : 0.0f;
      } else {
        pv.o[(bh * p.splits + split) * D + c] = o[k];
      }
    }
  }
  for (int h = tid; h < G; h += kThreads) {
    const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
    if (p.splits == 1) {
      if (p.lse) p.lse[bh] = l_s[h] > 0.0f ? m_s[h] + logf(l_s[h]) : -INFINITY;
    } else {
      pv.m[bh * p.splits + split] = m_s[h];
      pv.l[bh * p.splits + split] = l_s[h];
    }
  }
}

// Merge the T-splits of one (b, h): exact log-sum-exp combination.  Warp 0
// forms the split weights e^{m_s - M} in shared memory; every thread then
// streams one output column over the splits with independent loads in flight.
constexpr int kCombineThreads = 128;
constexpr int kCombineMaxSplits = 2048;

template <int D>
__global__ void __launch_bounds__(kCombineThreads)
decode_combine_kernel(const DecodeParams p) {
  __shared__ float w_s[kCombineMaxSplits];
  __shared__ float ML[2];
  const size_t bh = blockIdx.x;
  const int S = p.splits;
  const PartView pv = part_view(p.part, static_cast<size_t>(p.c.B) * p.Hq, S, D);
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    float M = -INFINITY;
    for (int s = lane; s < S; s += 32) M = fmaxf(M, pv.m[bh * S + s]);
    M = warp_max(M);
    float L = 0.0f;
    for (int s = lane; s < S; s += 32) {
      const float m = pv.m[bh * S + s];
      const float w = m > -INFINITY ? expf(m - M) : 0.0f;
      w_s[s] = w;
      L = fmaf(w, pv.l[bh * S + s], L);
    }
    L = warp_sum(L);
    if (lane == 0) {
      ML[0] = M;
      ML[1] = L;
    }
  }
  __syncthreads();
  const float L = ML[1];
  for (int c = threadIdx.x; c < D; c += kCombineThreads) {
    const float* po = pv.o + bh * S * D + c;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int s = 0;
    for (; s + 4 <= S; s += 4) {
      a0 = fmaf(w_s[s], po[(s + 0) * D], a0);
      a1 = fmaf(w_s[s + 1], po[(s + 1) * D], a1);
      a2 = fmaf(w_s[s + 2], po[(s + 2) * D], a2);
      a3 = fmaf(w_s[s + 3], po[(s + 3) * D], a3);
    }
    for (; s < S; ++s) a0 = fmaf(w_s[s], po[s * D], a0);
    const float acc = (a0 + a1) + (a2 + a3);
    p.out[bh * D + c] = L > 0.0f ? acc / L : 0.0f;
  }
  if (threadIdx.x == 0 && p.lse) p.lse[bh] = L > 0.0f ? ML[0] + logf(L) : -INFINITY;
}

// shared memory of decode_split_kernel, in the order it is carved up
template <int D>
size_t decode_split_smem(int G, int r, bool channel) {
  const int NG = num_groups(D), KS = NG + 1;
  const int ZB = r > 0 ? ((r / 2 + 3) / 4 + 1) * 4 : 0;
  size_t f = static_cast<size_t>(kTile) * D + G * D + (channel ? G * D : 0) + G * NG + G * r +
             5 * G * kTile + 4 * G + 2 * kTile * KS + kTile;
  return f * sizeof(float) + sizeof(uint32_t) * kTile * CodeRow<D>::kStride + kTile * ZB;
}

// The split kernel for a batch of GM >= G heads (G > 16: several 16-head passes)
template <int D, int GM>
cudaError_t launch_split_gm(const DecodeParams& p, cudaStream_t s) {
  const size_t smem = decode_split_smem<D>(p.G, p.c.r, p.c.kmode == HEADQ_K_CHANNEL);
  auto k = decode_split_kernel<D, GM>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(p.splits, p.c.Hkv, p.c.B);
  k<<<grid, kThreads, smem, s>>>(p);
  return cudaSuccess;
}

template <int D>
cudaError_t launch_split(const DecodeParams& p, cudaStream_t s) {
  if (p.G <= 1) return launch_split_gm<D, 1>(p, s);
  if (p.G <= 2) return launch_split_gm<D, 2>(p, s);
  if (p.G <= 4) return launch_split_gm<D, 4>(p, s);
  if (p.G <= 8) return launch_split_gm<D, 8>(p, s);
  if constexpr (16 * D <= 2048) return launch_split_gm<D, 16>(p, s);  // G * d <= 2048
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_d(const DecodeParams& p, bool mma, cudaStream_t s) {
  if (mma) {
    const cudaError_t e = launch_decode_mma(p, s);
    if (e != cudaSuccess) return e;
  } else {
    const cudaError_t e = launch_split<D>(p, s);
    if (e != cudaSuccess) return e;
  }
  if (p.splits > 1 && !(mma && p.fused)) {  // unless the split kernel merged its splits
    if (p.splits > kCombineMaxSplits) return cudaErrorInvalidConfiguration;
    decode_combine_kernel<D><<<p.c.B * p.Hq, kCombineThreads, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace

DecodePlan decode_plan(const headq_cache& c, int Hq, int T) {
  DecodePlan dp{1, 64, 1, false, false};
  const int G = c.Hkv > 0 ? Hq / c.Hkv : 0;
  const int units = c.B * c.Hkv;
  if (T <= 0 || units <= 0) return dp;
  // the tensor-core kernel reads either base code: per-channel keys fold each
  // 64-token block's scale into the query fragments tile by tile
  const bool mma = mma_decode_supported(c, G);
  const int occ = mma ? mma_decode_ctas_per_sm(c, G) : 0;
  if (occ > 0) {
    // Each CTA streams one contiguous chunk; the last CTA of each (b, kv)
    // merges the splits, so one kernel per call.  The split count minimises
    // waves x (tiles per CTA + kTileOverhead): with `slots` resident CTAs a
    // call takes ceil(units * splits / slots) waves of CTAs whose time is their
    // tile count plus a fixed cost (query preparation, merge) worth about
    // kTileOverhead tiles.  Ties go to fewer splits.
    constexpr long long kTileOverhead = 2;
    const long long slots = static_cast<long long>(occ) * sm_count();
    const int max_s = (T + 63) / 64;
    // a multiple of 16 tokens (so every bulk copy stays 16-byte aligned); of
    // 64 for a paged cache, so that no 64-token tile straddles two pages, and
    // for per-channel keys, so that every tile is one block
    const int align = (c.page_size > 0 || c.kmode == HEADQ_K_CHANNEL) ? 64 : 16;
    const long long per_unit = (slots + units - 1) / units;
    const int s_hi = static_cast<int>(
        std::min<long long>({static_cast<long long>(max_s), kMaxMmaSplits, 4 * per_unit + 4}));
    long long best = -1;
    int chunk = T;
    for (int s = 1; s <= s_hi; ++s) {
      int ch = (T + s - 1) / s;
      ch = (ch + align - 1) / align * align;
      const int sp = (T + ch - 1) / ch;
      if (sp != s) continue;  // the same chunk as a smaller count
      const long long waves = (static_cast<long long>(units) * sp + slots - 1) / slots;
      const long long cost = waves * ((ch + 63) / 64 + kTileOverhead);
      if (best < 0 || cost < best) {
        best = cost;
        chunk = ch;
      }
    }
    dp.chunk = chunk;
    dp.splits = (T + chunk - 1) / chunk;
    dp.mma = true;
    dp.fused = units <= kMaxFusedUnits;
    dp.kernels = (dp.splits > 1 && !dp.fused) ? 2 : 1;
  } else {
    // the generic kernel is latency-bound per warp (4 warps per CTA): fill
    // the SMs with about 4 CTAs each, chunks down to 64 tokens
    const SplitPlan sp = plan_splits(units, T, 64, 4);
    dp.splits = sp.splits;
    dp.chunk = sp.chunk;
    dp.kernels = dp.splits > 1 ? 2 : 1;
  }
  return dp;
}

cudaError_t launch_decode(const DecodeParams& p, bool mma, cudaStream_t s) {
  switch (p.c.d) {
    case 8: return launch_d<8>(p, false, s);
    case 16: return launch_d<16>(p, false, s);
    case 32: return launch_d<32>(p, false, s);
    case 64: return launch_d<64>(p, mma, s);
    case 128: return launch_d<128>(p, mma, s);
    case 256: return launch_d<256>(p, false, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace headq
