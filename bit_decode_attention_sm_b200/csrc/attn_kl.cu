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
  const float code = static_cast<float>(code2(p.c.k_codes + row * (D / 4), c));
  if (p.c.kmode == HEADQ_K_CHANNEL) {  // per channel, per 64-token block (row / 64)
    const size_t bi = (row >> 6) * D + c;
    return __fadd_rn(p.c.k_min[bi], __fmul_rn(code, p.c.k_scale[bi]));
  }
  constexpr int NG = num_groups(D);
  const int g = c / group_size(D);
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
    // the tile's cache rows are consecutive: chunks start at multiples of 64
    const size_t crow0 = cache_row_read(p.c, b, kv, t0, tid == 0 ? p.err : nullptr);
    // per-token value distortion |v^_j - v_j|^2
    for (int j = tid; j < kTile; j += kThreads) {
      float n2 = 0.0f;
      if (j < nt) {
        const size_t row = crow0 + j;
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
        const size_t row = crow0 + j;
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
          const size_t row = crow0 + j;
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

// ---------------------------------------------------------------------------
// Staged kernel (d = 64 or 128): 32-token tiles of every plane and of the full
// K and V are copied to shared memory with double-buffered cp.async (rows past
// the end zero-filled); the key error dk = k^ - k and the value error
// dv = v^ - v are formed once per token and shared by the G query heads.
constexpr int kSTT = 32;         // tokens per tile
constexpr int kSThreads = 256;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <int D>
struct KlStage {
  static constexpr int NG = D / 32;
  int frow;   // bytes per staged full-precision row (padded)
  int cvrow;  // bytes per staged cache-value row (dense, padded)
  int kf, vf, cv, kc, ks, km, zc, zs, vc, vs, vm, bytes;
  __host__ __device__ KlStage(int esz, int cv_esz, int r, bool v2) {
    frow = D * esz + 16;
    cvrow = D * cv_esz + 16;
    kf = 0;
    vf = kf + kSTT * frow;
    cv = vf + kSTT * frow;
    kc = cv + (v2 ? 0 : kSTT * cvrow);
    ks = kc + kSTT * (D / 4);
    km = ks + kSTT * NG * 4;
    zc = km + kSTT * NG * 4;
    zs = zc + kSTT * (r / 2 > 0 ? r / 2 : 0);
    vc = zs + (r > 0 ? kSTT * 4 : 0);
    vs = vc + (v2 ? kSTT * (D / 4) : 0);
    vm = vs + (v2 ? kSTT * NG * 4 : 0);
    bytes = (vm + (v2 ? kSTT * NG * 4 : 0) + 127) / 128 * 128;
  }
};

// copy kSTT rows of CH 16-byte chunks (contiguous in global) into shared rows of
// stride `dst_stride`, zero-filling rows >= valid
template <int CH>
__device__ __forceinline__ void stage_rows_ch(uint8_t* dst, int dst_stride, const uint8_t* src,
                                              int valid, int tid) {
  for (int e = tid; e < kSTT * CH; e += kSThreads) {
    const int row = e / CH, c = e - row * CH;
    const bool ok = row < valid;
    cp_async16(dst + row * dst_stride + c * 16, ok ? src + static_cast<size_t>(row) * CH * 16 + c * 16 : src,
               ok);
  }
}
// rows of rb = D * 2 or D * 4 bytes (the chunk count a compile-time constant)
template <int D>
__device__ __forceinline__ void stage_rows(uint8_t* dst, int dst_stride, const uint8_t* src, int rb,
                                           int valid, int tid) {
  if (rb == D * 2)
    stage_rows_ch<D * 2 / 16>(dst, dst_stride, src, valid, tid);
  else
    stage_rows_ch<D * 4 / 16>(dst, dst_stride, src, valid, tid);
}
// a contiguous block (rows of rb bytes packed), valid rows only
__device__ __forceinline__ void stage_block(uint8_t* dst, const uint8_t* src, int rb, int valid,
                                            int tid) {
  const int total = (kSTT * rb) / 16;
  const int vbytes = valid * rb;
  for (int e = tid; e < total; e += kSThreads) {
    const bool ok = e * 16 < vbytes;
    cp_async16(dst + e * 16, ok ? src + e * 16 : src, ok);
  }
}

// channels c .. c+7 of a staged row (bf16 or fp32), c a multiple of 8
__device__ __forceinline__ void ld8(const uint8_t* row, int c, bool bf16, float (&x)[8]) {
  if (bf16) {
    const uint4 u = *reinterpret_cast<const uint4*>(row + 2 * c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  } else {
    const float4 a = *reinterpret_cast<const float4*>(row + 4 * c);
    const float4 b = *reinterpret_cast<const float4*>(row + 4 * c + 16);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

template <int D>
__global__ void __launch_bounds__(kSThreads)
attn_kl_staged_kernel(const AttnKlParams p) {
  constexpr int NG = D / 32;
  constexpr int DS = D + 4;  // padded fp32 rows of dk / dv
  const int G = p.G, r = p.c.r, Hkv = p.c.Hkv;
  const bool v2 = p.c.vmode == HEADQ_V_2BIT;
  const bool cv_bf16 = p.c.v_dtype == HEADQ_BF16;
  const int esz = p.kv_bf16 ? 2 : 4;
  const KlStage<D> L(esz, cv_bf16 ? 2 : 4, r, v2);

  extern __shared__ __align__(128) uint8_t sm8[];
  uint8_t* stg[2] = {sm8, sm8 + L.bytes};
  float* dk_s = reinterpret_cast<float*>(sm8 + 2 * L.bytes);  // [kSTT][DS]
  float* dv_s = dk_s + kSTT * DS;                              // [kSTT][DS]
  float* q_s = dv_s + kSTT * DS;                               // [G][D]
  float* qt_s = q_s + G * D;                                   // [G][r]
  float* s_s = qt_s + G * (r > 0 ? r : 1);                     // [2][G][kSTT] s halves, then w
  float* d_s = s_s + 2 * G * kSTT;                             // [2][G][kSTT] delta halves
  float* n2_s = d_s + 2 * G * kSTT;                            // [kSTT]
  float* m_s = n2_s + kSTT;                                    // [G]
  float* md_s = m_s + G;                                       // [G]
  float* a_s = md_s + G;                                       // [G]
  double* acc_s = reinterpret_cast<double*>(smem_align(a_s + G, 8));  // [G][5]

  const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int Tb = p.T;
  if (p.seq_lens) Tb = max(0, min(p.seq_lens[b], p.T));
  const int t_begin = split * p.chunk;
  const int t_end = min(Tb, t_begin + p.chunk);
  const int ntiles = t_end > t_begin ? (t_end - t_begin + kSTT - 1) / kSTT : 0;
  const size_t bk = static_cast<size_t>(b) * Hkv + kv;
  const int h0 = kv * G;

  auto issue = [&](int i) {
    const int t0 = t_begin + i * kSTT;
    const int nv = min(kSTT, t_end - t0);
    uint8_t* st = stg[i & 1];
    const size_t frow0 = bk * p.T + t0;
    const size_t crow0 = cache_row_read(p.c, b, kv, t0, tid == 0 ? p.err : nullptr);
    stage_rows<D>(st + L.kf, L.frow, static_cast<const uint8_t*>(p.k_full) + frow0 * D * esz,
               D * esz, nv, tid);
    stage_rows<D>(st + L.vf, L.frow, static_cast<const uint8_t*>(p.v_full) + frow0 * D * esz,
               D * esz, nv, tid);
    if (!v2) {
      const int cesz = cv_bf16 ? 2 : 4;
      stage_rows<D>(st + L.cv, L.cvrow, static_cast<const uint8_t*>(p.c.v) + crow0 * D * cesz,
                 D * cesz, nv, tid);
    } else {
      stage_block(st + L.vc, p.c.v_codes + crow0 * (D / 4), D / 4, nv, tid);
      stage_block(st + L.vs, reinterpret_cast<const uint8_t*>(p.c.v_scale + crow0 * NG), NG * 4, nv, tid);
      stage_block(st + L.vm, reinterpret_cast<const uint8_t*>(p.c.v_min + crow0 * NG), NG * 4, nv, tid);
    }
    stage_block(st + L.kc, p.c.k_codes + crow0 * (D / 4), D / 4, nv, tid);
    stage_block(st + L.ks, reinterpret_cast<const uint8_t*>(p.c.k_scale + crow0 * NG), NG * 4, nv, tid);
    stage_block(st + L.km, reinterpret_cast<const uint8_t*>(p.c.k_min + crow0 * NG), NG * 4, nv, tid);
    if (r > 0) {
      if ((kSTT * (r / 2)) % 16 == 0)
        stage_block(st + L.zc, p.c.z_codes + crow0 * (r / 2), r / 2, nv, tid);
      stage_block(st + L.zs, reinterpret_cast<const uint8_t*>(p.c.z_scale + crow0), 4, nv, tid);
    }
    cp_async_commit();
  };
  if (ntiles > 0) issue(0);

  for (int i = tid; i < G * D; i += kSThreads)
    q_s[i] = load_elem(p.q, (static_cast<size_t>(b) * p.Hq + h0) * D + i, p.q_bf16);
  for (int h = tid; h < G; h += kSThreads) {
    m_s[h] = -INFINITY;
    md_s[h] = -INFINITY;
    for (int k = 0; k < 5; ++k) acc_s[h * 5 + k] = 0.0;
  }
  __syncthreads();
  for (int i = tid; i < G * r; i += kSThreads) {
    const int h = i / r, ii = i - h * r;
    const float* U = p.U + static_cast<size_t>(kv) * D * r;
    float acc = 0.0f;
    for (int c = 0; c < D; ++c) acc = fmaf(U[c * r + ii], q_s[h * D + c], acc);
    qt_s[i] = p.corr_sign * acc;
  }

  constexpr int kMaxDov = 8;  // (G * D) / kSThreads outputs per thread at most
  double dov[kMaxDov];
#pragma unroll
  for (int k = 0; k < kMaxDov; ++k) dov[k] = 0.0;

  for (int i = 0; i < ntiles; ++i) {
    if (i + 1 < ntiles) {
      issue(i + 1);
      cp_async_wait1();
    } else {
      cp_async_wait0();
    }
    __syncthreads();
    const uint8_t* st = stg[i & 1];
    const int t0 = t_begin + i * kSTT;
    const int nt = min(kSTT, t_end - t0);
    // phase 0: key and value errors per (token, 8 channels); |dv|^2 per token
    {
      constexpr int CPT = D / 8;  // tasks per token
      for (int task = tid; task < kSTT * CPT; task += kSThreads) {
        const int tt = task / CPT, c8 = task - tt * CPT, c = 8 * c8, g = c / 32;
        float n2 = 0.0f;
        if (tt < nt) {
          const uint32_t kb = *reinterpret_cast<const uint16_t*>(st + L.kc + tt * (D / 4) + 2 * c8);
          const float ksc = reinterpret_cast<const float*>(st + L.ks)[tt * NG + g];
          const float kmn = reinterpret_cast<const float*>(st + L.km)[tt * NG + g];
          float kf[8], vf[8], vh[8];
          ld8(st + L.kf + tt * L.frow, c, p.kv_bf16, kf);
          ld8(st + L.vf + tt * L.frow, c, p.kv_bf16, vf);
          if (v2) {
            const uint32_t vb = *reinterpret_cast<const uint16_t*>(st + L.vc + tt * (D / 4) + 2 * c8);
            const float vsc = reinterpret_cast<const float*>(st + L.vs)[tt * NG + g];
            const float vmn = reinterpret_cast<const float*>(st + L.vm)[tt * NG + g];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              vh[k] = __fadd_rn(vmn, __fmul_rn(static_cast<float>((vb >> (2 * k)) & 3), vsc));
          } else {
            ld8(st + L.cv + tt * L.cvrow, c, cv_bf16, vh);
          }
          float dk[8], dv[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float kh = __fadd_rn(kmn, __fmul_rn(static_cast<float>((kb >> (2 * k)) & 3), ksc));
            dk[k] = kh - kf[k];
            dv[k] = vh[k] - vf[k];
            n2 = fmaf(dv[k], dv[k], n2);
          }
          float4* dkw = reinterpret_cast<float4*>(dk_s + tt * DS + c);
          float4* dvw = reinterpret_cast<float4*>(dv_s + tt * DS + c);
          dkw[0] = make_float4(dk[0], dk[1], dk[2], dk[3]);
          dkw[1] = make_float4(dk[4], dk[5], dk[6], dk[7]);
          dvw[0] = make_float4(dv[0], dv[1], dv[2], dv[3]);
          dvw[1] = make_float4(dv[4], dv[5], dv[6], dv[7]);
        }
        // the CPT tasks of a token are CPT consecutive lanes of one warp
#pragma unroll
        for (int o = CPT / 2; o > 0; o >>= 1) n2 += __shfl_xor_sync(kFull, n2, o);
        if (c8 == 0) n2_s[tt] = tt < nt ? n2 : 0.0f;
      }
    }
    __syncthreads();
    // phase 1: partial logits s and score perturbations delta per (half of the
    // channels, head, token): the halves of a (head, token) are in different
    // warps (one token per lane, distinct banks) and phase 2 adds them
    for (int task = tid; task < 2 * G * kSTT; task += kSThreads) {
      const int half = task / (G * kSTT), pair = task - half * (G * kSTT);
      const int h = pair / kSTT, tt = pair - h * kSTT;
      float sf = 0.0f, de = 0.0f;
      if (tt < nt) {
        const float* qh = q_s + h * D;
        const uint8_t* kfr = st + L.kf + tt * L.frow;
        const float* dkr = dk_s + tt * DS;
        const int c_lo = half * (D / 2);
        if (p.kv_bf16) {
#pragma unroll 4
          for (int c = c_lo; c < c_lo + D / 2; c += 8) {
            const uint4 kw = *reinterpret_cast<const uint4*>(kfr + 2 * c);
            const uint32_t w4[4] = {kw.x, kw.y, kw.z, kw.w};
            const float4 d0 = *reinterpret_cast<const float4*>(dkr + c);
            const float4 d1 = *reinterpret_cast<const float4*>(dkr + c + 4);
            const float4 q0 = *reinterpret_cast<const float4*>(qh + c);
            const float4 q1 = *reinterpret_cast<const float4*>(qh + c + 4);
            const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
            const float dvv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              sf = fmaf(qv[2 * k], __uint_as_float(w4[k] << 16), sf);
              sf = fmaf(qv[2 * k + 1], __uint_as_float(w4[k] & 0xffff0000u), sf);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) de = fmaf(qv[k], dvv[k], de);
          }
        } else {
          for (int c = c_lo; c < c_lo + D / 2; ++c) {
            sf = fmaf(qh[c], reinterpret_cast<const float*>(kfr)[c], sf);
            de = fmaf(qh[c], dkr[c], de);
          }
        }
        if (r > 0 && half == 1) {
          const uint8_t* zr = (kSTT * (r / 2)) % 16 == 0
                                  ? st + L.zc + tt * (r / 2)
                                  : p.c.z_codes + (cache_row_read(p.c, b, kv, t0, nullptr) + tt) * (r / 2);
          float cz = 0.0f;
          for (int ii = 0; ii < r; ++ii)
            cz = fmaf(qt_s[h * r + ii], static_cast<float>(nibble(zr, ii)), cz);
          de = fmaf(reinterpret_cast<const float*>(st + L.zs)[tt], cz, de);
        }
      }
      s_s[task] = sf;
      d_s[task] = de;
    }
    __syncthreads();
    // phase 2: running fp64 accumulators, one warp per head
    for (int h = warp; h < G; h += kSThreads / 32) {
      const bool valid = lane < nt;
      const int e0 = h * kSTT + lane, e1 = e0 + G * kSTT;
      const float sv = valid ? (s_s[e0] + s_s[e1]) * p.sm_scale : -INFINITY;
      const float dl = valid ? (d_s[e0] + d_s[e1]) * p.sm_scale : 0.0f;
      const float m_old = m_s[h], md_old = md_s[h];
      const float m_new = fmaxf(m_old, warp_maxf(sv));
      const float md_new = fmaxf(md_old, warp_maxf(valid ? dl : -INFINITY));
      const double w = valid ? exp(static_cast<double>(sv) - m_new) : 0.0;
      const double x = valid ? w * exp(static_cast<double>(dl) - md_new) : 0.0;
      const double alpha = exp(static_cast<double>(m_old) - m_new);
      const double beta = exp(static_cast<double>(md_old) - md_new);
      const double dd = dl;
      const double sW = warp_sumd(w), sX = warp_sumd(x);
      const double sM1 = warp_sumd(w * dd), sM2 = warp_sumd(w * dd * dd);
      const double sA2 = warp_sumd(w * w * static_cast<double>(n2_s[lane]));
      s_s[h * kSTT + lane] = static_cast<float>(w);
      __syncwarp();
      if (lane == 0) {
        double* a = acc_s + h * 5;
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
    // phase 3: readout error sum_j w_j dv_j per (head, dim)
#pragma unroll
    for (int k = 0; k < kMaxDov; ++k) {
      const int idx = tid + k * kSThreads;
      if (idx < G * D) {
        const int h = idx / D, c = idx - h * D;
        const float* pw = s_s + h * kSTT;
        float part = 0.0f;
        for (int j = 0; j < nt; ++j) part = fmaf(pw[j], dv_s[j * DS + c], part);
        dov[k] = dov[k] * static_cast<double>(a_s[h]) + part;
      }
    }
    __syncthreads();
  }

  const int PS = kPartHead + D;
#pragma unroll
  for (int k = 0; k < kMaxDov; ++k) {
    const int idx = tid + k * kSThreads;
    if (idx < G * D) {
      const int h = idx / D, c = idx - h * D;
      const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
      p.part[(bh * p.splits + split) * PS + kPartHead + c] = dov[k];
    }
  }
  for (int h = tid; h < G; h += kSThreads) {
    const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
    double* pt = p.part + (bh * p.splits + split) * PS;
    const double* a = acc_s + h * 5;
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
size_t staged_smem(const AttnKlParams& p) {
  const KlStage<D> L(p.kv_bf16 ? 2 : 4, p.c.v_dtype == HEADQ_BF16 ? 2 : 4, p.c.r,
                     p.c.vmode == HEADQ_V_2BIT);
  const int G = p.G, r = p.c.r;
  return 2 * size_t(L.bytes) + sizeof(float) * (2 * kSTT * (D + 4) + G * D + G * (r > 0 ? r : 1) +
                                                4 * G * kSTT + kSTT + 3 * G) +
         8 + sizeof(double) * G * 5;
}

template <int D>
cudaError_t launch_d(const AttnKlParams& p, cudaStream_t s) {
  const int G = p.G, r = p.c.r;
  if (p.hm) {
    const cudaError_t e = launch_attn_kl_hm(p, s);
    if (e != cudaSuccess) return e;
    attn_kl_combine_kernel<D><<<p.c.B * p.Hq, D < 32 ? 32 : (D > 128 ? 128 : D), 0, s>>>(p);
    return cudaGetLastError();
  }
  const size_t smem = sizeof(double) * G * 6 +
                      sizeof(float) * (static_cast<size_t>(G) * D + G * r + 2 * G * kTile +
                                       kTile + 3 * G);
  dim3 grid(p.splits, p.c.Hkv, p.c.B);
  if constexpr (D == 64 || D == 128) {
    if (p.G * D <= 8 * kSThreads && p.c.kmode == HEADQ_K_TOKEN) {
      const size_t ssm = staged_smem<D>(p);
      auto k = attn_kl_staged_kernel<D>;
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(ssm));
      if (e != cudaSuccess) return e;
      k<<<grid, kSThreads, ssm, s>>>(p);
      attn_kl_combine_kernel<D><<<p.c.B * p.Hq, D < 32 ? 32 : (D > 128 ? 128 : D), 0, s>>>(p);
      return cudaGetLastError();
    }
  }
  auto k = attn_kl_split_kernel<D>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
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
