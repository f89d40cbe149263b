// HeadQ model-visible distortion diagnostics ("HeadQ: Model-Visible Distortion
// and Score-Space Correction for KV-Cache Quantization", gist.science summary,
// section 2.1 -- score perturbation delta_j = s^_j - s_j, attention KL and its
// local Fisher-weighted variance form -- and section 2.2 -- readout error
// sum_j p_j dv_j at fixed p and the A^2 = p_j^2 weighted token distortion).
//
// One streaming pass over the cache and the full-precision K/V per split:
// logits s_j = sm*q.k_j and delta_j = sm*(q.(k^base_j - k_j) + sigma*(U^T q).z^_j)
// in fp32 (delta from the per-channel key error, so it keeps its own relative
// precision), then fp64 running sums rescaled by the running maxima m of s and
// md of delta:
//   W = sum w, w = e^{s-m};  X = sum w e^{delta-md};  M1 = sum w delta;
//   M2 = sum w delta^2;  A2 = sum w^2 |dv|^2;  dov = sum w dv.
// With p = w/W, KL(p || softmax(s + delta)) = log sum_j p_j e^{delta_j}
// - sum_j p_j delta_j, so a combine kernel merges the splits and forms
//   KL = log(X/W) + md - M1/W,  Var = M2/W - (M1/W)^2,  A2V = A2/W^2,
//   dout2 = |dov/W|^2.
// This form never subtracts two log-sum-exps of the (large) logits, so the KL
// keeps its relative precision even when it is tiny.
#include <math.h>

#include "headq_internal.cuh"

namespace headq {
namespace {

constexpr int kTile = 32;
constexpr int kThreads = 128;
constexpr int kMaxOut = 16;
constexpr int kPartHead = 7;  // m, W, md, X, M1, M2, A2 then dov[D]
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_maxf(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ double warp_sumd(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

template <int D>
__device__ __forceinline__ float cached_value(const AttnKlParams& p, size_t row, int c) {
  if (p.c.vmode == HEADQ_V_2BIT) {
    constexpr int NG = num_groups(D);
    const int g = c / group_size(D);
    const float code = static_cast<float>(code2(p.c.v_codes + row * (D / 4), c));
    return __fadd_rn(p.c.v_min[row * NG + g], __fmul_rn(code, p.c.v_scale[row * NG + g]));
  }
  return load_elem(p.c.v, row * D + c, p.c.v_dtype == HEADQ_BF16);
}

template <int D>
__device__ __forceinline__ float base_key(const AttnKlParams& p, size_t row, int c) {
  constexpr int NG = num_groups(D);
  const int g = c / group_size(D);
  const float code = static_cast<float>(code2(p.c.k_codes + row * (D / 4), c));
  return __fadd_rn(p.c.k_min[row * NG + g], __fmul_rn(code, p.c.k_scale[row * NG + g]));
}

template <int D>
__global__ void __launch_bounds__(kThreads)
attn_kl_split_kernel(const AttnKlParams p) {
  const int G = p.G, r = p.c.r, Hkv = p.c.Hkv;
  extern __shared__ double smd[];
  double* acc_s = smd;                                  // [G][6]: W, X, M1, M2, A2, -
  float* q_s = reinterpret_cast<float*>(acc_s + G * 6); // [G][D]
  float* qt_s = q_s + G * D;                            // [G][r]
  float* s_s = qt_s + G * r;                            // [G][kTile] s, then w
  float* d_s = s_s + G * kTile;                         // [G][kTile] delta
  float* n2_s = d_s + G * kTile;                        // [kTile] |dv_j|^2
  float* m_s = n2_s + kTile;                            // [G]
  float* md_s = m_s + G;                                // [G] running max of delta
  float* a_s = md_s + G;                                // [G]

  const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int Tb = p.T;
  if (p.seq_lens) Tb = max(0, min(p.seq_lens[b], p.T));
  const int t_begin = split * p.chunk;
  const int t_end = min(Tb, t_begin + p.chunk);
  const size_t bk = static_cast<size_t>(b) * Hkv + kv;
  const int h0 = kv * G;

  for (int i = tid; i < G * D; i += kThreads)
    q_s[i] = load_elem(p.q, (static_cast<size_t>(b) * p.Hq + h0) * D + i, p.q_bf16);
  for (int h = tid; h < G; h += kThreads) {
    m_s[h] = -INFINITY;
    md_s[h] = -INFINITY;
    for (int k = 0; k < 6; ++k) acc_s[h * 6 + k] = 0.0;
  }
  __syncthreads();
  for (int i = tid; i < G * r; i += kThreads) {
    const int h = i / r, ii = i - h * r;
    const float* U = p.U + static_cast<size_t>(kv) * D * r;
    float acc = 0.0f;
    for (int c = 0; c < D; ++c) acc = fmaf(U[c * r + ii], q_s[h * D + c], acc);
    qt_s[i] = p.corr_sign * acc;
  }
  __syncthreads();

  double dov[kMaxOut];
#pragma unroll
  for (int k = 0; k < kMaxOut; ++k) dov[k] = 0.0;

  for (int t0 = t_begin; t0 < t_end; t0 += kTile) {
    const int nt = min(kTile, t_end - t0);
    // per-token value distortion |v^_j - v_j|^2
    for (int j = tid; j < kTile; j += kThreads) {
      float n2 = 0.0f;
      if (j < nt) {
        const size_t row = bk * p.c.T_cap + t0 + j;
        const size_t frow = bk * p.T + t0 + j;
        for (int c = 0; c < D; ++c) {
          const float dv = cached_value<D>(p, row, c) - load_elem(p.v_full, frow * D + c, p.kv_bf16);
          n2 = fmaf(dv, dv, n2);
        }
      }
      n2_s[j] = n2;
    }
    // logits and score perturbations per (head, token)
    for (int idx = tid; idx < G * kTile; idx += kThreads) {
      const int h = idx / kTile, j = idx - h * kTile;
      float s = -INFINITY, dl = 0.0f;
      if (j < nt) {
        const size_t row = bk * p.c.T_cap + t0 + j;
        const size_t frow = bk * p.T + t0 + j;
        const float* qh = q_s + h * D;
        float sf = 0.0f, de = 0.0f;
        for (int c = 0; c < D; ++c) {
          const float kf = load_elem(p.k_full, frow * D + c, p.kv_bf16);
          sf = fmaf(qh[c], kf, sf);
          de = fmaf(qh[c], base_key<D>(p, row, c) - kf, de);
        }
        if (r > 0) {
          const uint8_t* zr = p.c.z_codes + row * (r / 2);
          float cz = 0.0f;
          for (int i = 0; i < r; ++i)
            cz = fmaf(qt_s[h * r + i], static_cast<float>(nibble(zr, i)), cz);
          de = fmaf(p.c.z_scale[row], cz, de);
        }
        s = sf * p.sm_scale;
        dl = de * p.sm_scale;
      }
      s_s[idx] = s;
      d_s[idx] = dl;
    }
    __syncthreads();
    for (int h = warp; h < G; h += kThreads / 32) {
      const bool valid = lane < nt;
      const float s = s_s[h * kTile + lane];
      const float dl = d_s[h * kTile + lane];
      const float m_old = m_s[h], md_old = md_s[h];
      const float m_new = fmaxf(m_old, warp_maxf(s));
      const float md_new = fmaxf(md_old, warp_maxf(valid ? dl : -INFINITY));
      const double w = valid ? exp(static_cast<double>(s) - m_new) : 0.0;
      const double x = valid ? w * exp(static_cast<double>(dl) - md_new) : 0.0;
      const double alpha = exp(static_cast<double>(m_old) - m_new);
      const double beta = exp(static_cast<double>(md_old) - md_new);
      const double d = dl;
      const double sW = warp_sumd(w), sX = warp_sumd(x);
      const double sM1 = warp_sumd(w * d), sM2 = warp_sumd(w * d * d);
      const double sA2 = warp_sumd(w * w * static_cast<double>(n2_s[lane]));
      s_s[h * kTile + lane] = static_cast<float>(w);
      __syncwarp();
      if (lane == 0) {
        double* a = acc_s + h * 6;
        a[0] = a[0] * alpha + sW;
        a[1] = a[1] * alpha * beta + sX;
        a[2] = a[2] * alpha + sM1;
        a[3] = a[3] * alpha + sM2;
        a[4] = a[4] * alpha * alpha + sA2;
        m_s[h] = m_new;
        md_s[h] = md_new;
        a_s[h] = static_cast<float>(alpha);
      }
    }
    __syncthreads();
    // readout error accumulator sum_j w_j (v^_j - v_j)
#pragma unroll
    for (int k = 0; k < kMaxOut; ++k) {
      const int idx = tid + k * kThreads;
      if (idx < G * D) {
        const int h = idx / D, c = idx - h * D;
        double acc = dov[k] * static_cast<double>(a_s[h]);
        const float* pw = s_s + h * kTile;
        for (int j = 0; j < nt; ++j) {
          const size_t row = bk * p.c.T_cap + t0 + j;
          const size_t frow = bk * p.T + t0 + j;
          const float dv = cached_value<D>(p, row, c) - load_elem(p.v_full, frow * D + c, p.kv_bf16);
          acc += static_cast<double>(pw[j]) * dv;
        }
        dov[k] = acc;
      }
    }
    __syncthreads();
  }

  const int PS = kPartHead + D;
#pragma unroll
  for (int k = 0; k < kMaxOut; ++k) {
    const int idx = tid + k * kThreads;
    if (idx < G * D) {
      const int h = idx / D, c = idx - h * D;
      const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
      p.part[(bh * p.splits + split) * PS + kPartHead + c] = dov[k];
    }
  }
  for (int h = tid; h < G; h += kThreads) {
    const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
    double* pt = p.part + (bh * p.splits + split) * PS;
    const double* a = acc_s + h * 6;
    pt[0] = m_s[h];
    pt[1] = a[0];
    pt[2] = md_s[h];
    pt[3] = a[1];
    pt[4] = a[2];
    pt[5] = a[3];
    pt[6] = a[4];
  }
}

template <int D>
__global__ void attn_kl_combine_kernel(const AttnKlParams p) {
  const size_t bh = blockIdx.x;
  const int S = p.splits, PS = kPartHead + D;
  const double* pb = p.part + bh * S * PS;
  double M = -INFINITY, MD = -INFINITY;
  for (int s = 0; s < S; ++s) {
    M = fmax(M, pb[s * PS + 0]);
    MD = fmax(MD, pb[s * PS + 2]);
  }
  double W = 0, X = 0, M1 = 0, M2 = 0, A2 = 0;
  for (int s = 0; s < S; ++s) {
    const double* q = pb + s * PS;
    if (q[0] > -INFINITY) {
      const double f = exp(q[0] - M);
      W += f * q[1];
      X += f * exp(q[2] - MD) * q[3];
      M1 += f * q[4];
      M2 += f * q[5];
      A2 += f * f * q[6];
    }
  }
  __shared__ double red[32];
  double o2 = 0.0;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    double acc = 0.0;
    for (int s = 0; s < S; ++s) {
      const double* q = pb + s * PS;
      if (q[0] > -INFINITY) acc += exp(q[0] - M) * q[kPartHead + c];
    }
    const double dv = W > 0 ? acc / W : 0.0;
    o2 += dv * dv;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) o2 += __shfl_xor_sync(kFull, o2, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = o2;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) tot += red[w];
    if (W > 0) {
      const double m1 = M1 / W;
      p.kl[bh] = static_cast<float>(log(X / W) + MD - m1);
      p.fvar[bh] = static_cast<float>(M2 / W - m1 * m1);
      p.a2v[bh] = static_cast<float>(A2 / (W * W));
      if (p.dout2) p.dout2[bh] = static_cast<float>(tot);
    } else {
      p.kl[bh] = 0.0f;
      p.fvar[bh] = 0.0f;
      p.a2v[bh] = 0.0f;
      if (p.dout2) p.dout2[bh] = 0.0f;
    }
  }
}

template <int D>
cudaError_t launch_d(const AttnKlParams& p, cudaStream_t s) {
  const int G = p.G, r = p.c.r;
  const size_t smem = sizeof(double) * G * 6 +
                      sizeof(float) * (static_cast<size_t>(G) * D + G * r + 2 * G * kTile +
                                       kTile + 3 * G);
  auto k = attn_kl_split_kernel<D>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(p.splits, p.c.Hkv, p.c.B);
  k<<<grid, kThreads, smem, s>>>(p);
  attn_kl_combine_kernel<D><<<p.c.B * p.Hq, D < 32 ? 32 : (D > 128 ? 128 : D), 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_kl(const AttnKlParams& p, cudaStream_t s) {
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
