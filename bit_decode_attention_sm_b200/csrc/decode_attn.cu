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

#include "headq_internal.cuh"

namespace headq {
namespace {

constexpr int kTile = 32;      // tokens per inner step (one per lane in phase 2)
constexpr int kThreads = 128;
constexpr int kMaxOut = 16;    // (G * d) / kThreads outputs per thread at most
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

template <int D>
__device__ __forceinline__ float value_at(const DecodeParams& p, size_t row, int c) {
  if (p.c.vmode == HEADQ_V_2BIT) {
    constexpr int NG = num_groups(D);
    const int g = c / group_size(D);
    const float code = static_cast<float>(code2(p.c.v_codes + row * (D / 4), c));
    return __fadd_rn(p.c.v_min[row * NG + g], __fmul_rn(code, p.c.v_scale[row * NG + g]));
  }
  return load_elem(p.c.v, row * D + c, p.c.v_dtype == HEADQ_BF16);
}

template <int D>
__global__ void __launch_bounds__(kThreads)
decode_split_kernel(const DecodeParams p) {
  constexpr int NG = num_groups(D);
  constexpr int GS = group_size(D);
  const int G = p.G, r = p.c.r;
  extern __shared__ float sm[];
  float* q_s = sm;                // [G][D]
  float* qg_s = q_s + G * D;      // [G][NG]   group sums of q
  float* qt_s = qg_s + G * NG;    // [G][r]    sigma * U_h^T q
  float* s_s = qt_s + G * r;      // [G][kTile] logits, then weights
  float* m_s = s_s + G * kTile;   // [G]
  float* l_s = m_s + G;           // [G]
  float* a_s = l_s + G;           // [G]
  float* v_s = a_s + G;           // [kTile][D] the tile's values, dequantised
  float* kmn_s = v_s + kTile * D; // [D] per-channel key minima of the tile's block
  float* ksc_s = kmn_s + D;       // [D] and scales (per-channel base code)

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
  __syncthreads();

  float o[kMaxOut];
#pragma unroll
  for (int k = 0; k < kMaxOut; ++k) o[k] = 0.0f;

  for (int t0 = t_begin; t0 < t_end; t0 += kTile) {
    const int nt = min(kTile, t_end - t0);
    // the tile's rows are consecutive: chunks start at multiples of 64 tokens
    const size_t row0 = cache_row_read(p.c, b, kv, t0, tid == 0 ? p.err : nullptr);
    // the tile's values (and, per-channel code, its block's minima and scales)
    // staged once with coalesced loads, so the readout below reads shared memory
    for (int e = tid; e < nt * D; e += kThreads) {
      const int j = e / D, c = e - j * D;
      v_s[e] = value_at<D>(p, row0 + j, c);
    }
    if (p.c.kmode == HEADQ_K_CHANNEL)
      for (int c = tid; c < D; c += kThreads) {
        kmn_s[c] = p.c.k_min[(row0 >> 6) * D + c];
        ksc_s[c] = p.c.k_scale[(row0 >> 6) * D + c];
      }
    __syncthreads();
    // phase 1: logits of (head, token) pairs
    for (int idx = tid; idx < G * kTile; idx += kThreads) {
      const int h = idx / kTile, j = idx - h * kTile;
      float s = -INFINITY;
      if (j < nt) {
        const size_t row = row0 + j;
        const uint8_t* cr = p.c.k_codes + row * (D / 4);
        const float* qh = q_s + h * D;
        float acc = 0.0f;
        if (p.c.kmode == HEADQ_K_CHANNEL) {  // per-channel minimum and scale of the block
          for (int c = 0; c < D; ++c) {
            const float kh =
                __fadd_rn(kmn_s[c], __fmul_rn(static_cast<float>(code2(cr, c)), ksc_s[c]));
            acc = fmaf(qh[c], kh, acc);
          }
        } else {
          for (int g = 0; g < NG; ++g) {
            float pg = 0.0f;
            for (int c = 0; c < GS; ++c)
              pg = fmaf(qh[g * GS + c], static_cast<float>(code2(cr, g * GS + c)), pg);
            acc = fmaf(p.c.k_min[row * NG + g], qg_s[h * NG + g], acc);
            acc = fmaf(p.c.k_scale[row * NG + g], pg, acc);
          }
        }
        if (r > 0) {
          const uint8_t* zr = p.c.z_codes + row * (r / 2);
          float cz = 0.0f;
          for (int i = 0; i < r; ++i)
            cz = fmaf(qt_s[h * r + i], static_cast<float>(nibble(zr, i)), cz);
          acc = fmaf(p.c.z_scale[row], cz, acc);
        }
        s = acc * p.sm_scale;
      }
      s_s[idx] = s;
    }
    __syncthreads();
    // phase 2: online softmax update, one warp per head
    for (int h = warp; h < G; h += kThreads / 32) {
      const float s = s_s[h * kTile + lane];
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
    // phase 3: rescale and accumulate p_j v_j
#pragma unroll
    for (int k = 0; k < kMaxOut; ++k) {
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
  for (int k = 0; k < kMaxOut; ++k) {
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

template <int D>
cudaError_t launch_d(const DecodeParams& p, bool mma, cudaStream_t s) {
  if (mma) {
    const cudaError_t e = launch_decode_mma(p, s);
    if (e != cudaSuccess) return e;
  } else {
    const int G = p.G, r = p.c.r;
    const size_t smem = sizeof(float) * (static_cast<size_t>(G) * D + G * num_groups(D) +
                                         G * r + G * kTile + 3 * G + kTile * D + 2 * D);
    auto k = decode_split_kernel<D>;
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
      if (e != cudaSuccess) return e;
    }
    dim3 grid(p.splits, p.c.Hkv, p.c.B);
    k<<<grid, kThreads, smem, s>>>(p);
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
  // the tensor-core kernel reads the per-token base code; the per-channel code
  // goes to the generic kernel
  const bool mma = c.kmode == HEADQ_K_TOKEN && mma_decode_supported(c, G);
  const int occ = mma ? mma_decode_ctas_per_sm(c, G) : 0;
  if (occ > 0) {
    // one wave: every CTA resident, each streaming one contiguous chunk; the
    // last CTA of each (b, kv) merges the splits, so one kernel per call
    int s = (occ * sm_count()) / units;
    const int max_s = (T + 63) / 64;
    s = s < 1 ? 1 : (s > max_s ? max_s : s);
    if (s > kMaxMmaSplits) s = kMaxMmaSplits;
    // a multiple of 16 tokens (so every bulk copy stays 16-byte aligned); of
    // 64 for a paged cache, so that no 64-token tile straddles two pages
    const int align = c.page_size > 0 ? 64 : 16;
    int chunk = (T + s - 1) / s;
    chunk = (chunk + align - 1) / align * align;
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
