// A^2 value policy for the full-KV composition ("HeadQ: Model-Visible
// Distortion and Score-Space Correction for KV-Cache Quantization"; abstract,
// and the gist.science summary, section 2: under fixed attention the readout
// error of value distortions dv_j has the A^2-weighted diagonal surrogate
// D_V = sum_j p_j^2 |dv_j|^2, and value compression should put its precision
// where that weight is large; section 5 composes HeadQ keys with 2-bit values
// under an A^2 value policy, which the pages do not spell out).
//
// Policy as built here: with a budget of K tokens per (b, kv) whose values stay
// exact (the input precision) and 2-bit codes for the rest, D_V (summed over a
// set of observation queries and the G query heads of the KV head) loses the
// term of every kept token, so the K tokens with the largest
//   a_j = |v^_j - v_j|^2 * sum_{obs o, head h} p_{o,h,j}^2
// minimise it exactly (top-K, ties to the lower position).  p is the attention
// of the observation queries over the exact keys.
//
//   a2 pass kernel (x2)  pass 0: per 64-token tile, each observation query's
//                        logit max and exp-sum (two halves per tile); lse
//                        kernel merges them.  Pass 1: a_j per token.
//   a2 select kernel     per (b, kv): radix select of the K-th largest a_j over
//                        the 32-bit patterns (a_j >= 0, so the bit order is the
//                        value order), ordered compaction of the kept positions
//                        (ascending), and a copy of their exact values.
//   a2 fixup kernel      after a decode: out += sum_{kept j < T_b}
//                        exp(s^_j - lse) (v_j - v^_j), which turns the decode's
//                        readout over v^_j into the readout over the mixed values
//                        (same softmax weights; exact algebra).
#include <math.h>

#include <algorithm>
#include <mutex>

#include "codec.cuh"
#include "headq_internal.cuh"

#define HEADQ_API extern "C" __attribute__((visibility("default")))

namespace headq {
namespace {

constexpr int kAT = 64;          // tokens per score tile
constexpr int kAThreads = 256;   // 64 tokens x 4 query lanes
constexpr int kAQC = 16;         // observation queries staged per chunk
constexpr int kSelThreads = 1024;
constexpr int kSelReg = 4;       // scores per select thread kept in registers
constexpr int kFixThreads = 512;
constexpr int kFixTok = 64;      // kept tokens per fixup step
constexpr int kFixIdx = 512;     // kept-token indices loaded at once (a multiple of kFixTok)
constexpr int kFixMaxOut = 2048 / kFixThreads;
constexpr int kFixHeads = 8;     // heads per KV head accumulated per thread (G <= 8)

struct A2Params {
  headq_cache c;
  const void* q_obs;
  bool q_bf16;
  int n_obs, Hq, G, T;
  const int32_t* seq_lens;
  const void* k_full;
  const void* v_full;
  bool kv_bf16;
  float sm_scale;
  int ntiles;
  int ppt;        // partials per tile: 2 (CUDA-core pass) or 4 (tensor-core pass)
  float2* part;   // [B*Hkv, ntiles, ppt, NQ] (max, exp-sum) per tile part
  float* lse;     // [B*Hkv, NQ], query index o*G + g
  float* scores;  // [B*Hkv, T]
  unsigned* err;
};

__device__ __forceinline__ int seq_len(const int32_t* seq_lens, int b, int T) {
  return seq_lens ? max(0, min(seq_lens[b], T)) : T;
}

// the cached (dequantised) value of channel c at plane row `row`
__device__ __forceinline__ float value_hat(const headq_cache& c, size_t row, int ch, int d) {
  if (c.vmode == HEADQ_V_2BIT) {
    const int GS = d < 32 ? d : 32, NG = d / GS;
    const int g = ch / GS;
    const float mn = c.v_min[row * NG + g], sc = c.v_scale[row * NG + g];
    return __fadd_rn(mn, __fmul_rn(static_cast<float>(code2(c.v_codes + row * (d / 4), ch)), sc));
  }
  return load_elem(c.v, row * d + ch, c.v_dtype == HEADQ_BF16);
}

// 8 consecutive elements (offset a multiple of 8) of an fp32 or bf16 tensor
__device__ __forceinline__ void load8(const void* base, size_t off, bool bf16, float (&x)[8]) {
  if (bf16) {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  } else {
    const float4* f = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
    const float4 a = f[0], b = f[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

// value_hat of channels c0 .. c0+7 (c0 a multiple of 8, inside one group)
__device__ __forceinline__ void value_hat8(const headq_cache& c, size_t row, int c0, int d,
                                           float (&x)[8]) {
  if (c.vmode == HEADQ_V_2BIT) {
    const int GS = d < 32 ? d : 32, NG = d / GS;
    const int g = c0 / GS;
    const float mn = c.v_min[row * NG + g], sc = c.v_scale[row * NG + g];
    const uint32_t w = *reinterpret_cast<const uint16_t*>(c.v_codes + row * (d / 4) + c0 / 4);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      x[k] = __fadd_rn(mn, __fmul_rn(static_cast<float>((w >> (2 * k)) & 3u), sc));
  } else {
    load8(c.v, row * d + c0, c.v_dtype == HEADQ_BF16, x);
  }
}

// Pass 0 (SCORE false): tile partials of the softmax normaliser of each
// observation query.  Pass 1 (SCORE true): a_j of each token of the tile.
template <int D, bool SCORE>
__global__ void __launch_bounds__(kAThreads) a2_pass_kernel(const A2Params p) {
  extern __shared__ float sm[];
  constexpr int KS = D + 4;             // key row stride: 16-byte rows, 8 rows per bank sweep
  float* k_s = sm;                      // [kAT][KS]
  float* q_s = k_s + kAT * KS;          // [kAQC][D]
  float* red_s = q_s + kAQC * D;        // [kAThreads]
  float* dv2_s = red_s + kAThreads;     // [kAT]

  const int tile = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, j = tid % kAT, lane4 = tid / kAT;  // 4 query lanes
  const int Tb = seq_len(p.seq_lens, b, p.T);
  const int t0 = tile * kAT;
  const int G = p.G, NQ = p.n_obs * G;
  const size_t bk = static_cast<size_t>(b) * p.c.Hkv + kv;
  const bool valid = t0 + j < Tb;

  for (int e = tid; e < kAT * D; e += kAThreads) {
    const int jj = e / D, ch = e - jj * D;
    float x = 0.0f;
    if (t0 + jj < Tb) x = load_elem(p.k_full, (bk * p.T + t0 + jj) * D + ch, p.kv_bf16);
    k_s[jj * KS + ch] = x;
  }
  if constexpr (SCORE) {  // |v^_j - v_j|^2, channels split over the 4 lanes
    float a = 0.0f;
    if (valid) {
      const size_t row = cache_row_read(p.c, b, kv, t0 + j, lane4 == 0 ? p.err : nullptr);
      for (int ch = lane4 * (D / 4); ch < (lane4 + 1) * (D / 4); ++ch) {
        const float dv = value_hat(p.c, row, ch, D) -
                         load_elem(p.v_full, (bk * p.T + t0 + j) * D + ch, p.kv_bf16);
        a = fmaf(dv, dv, a);
      }
    }
    red_s[tid] = a;
    __syncthreads();
    if (tid < kAT) dv2_s[tid] = (red_s[tid] + red_s[tid + kAT]) + (red_s[tid + 2 * kAT] + red_s[tid + 3 * kAT]);
  }

  float acc2 = 0.0f;  // SCORE: sum of p^2 of token j over this lane's queries
  for (int q0 = 0; q0 < NQ; q0 += kAQC) {
    const int nq = min(kAQC, NQ - q0);
    __syncthreads();
    for (int e = tid; e < kAQC * D; e += kAThreads) {
      const int qq = e / D, ch = e - qq * D;
      float x = 0.0f;
      if (qq < nq) {
        const int qi = q0 + qq, o = qi / G, g = qi - o * G;
        x = load_elem(p.q_obs, ((static_cast<size_t>(b) * p.n_obs + o) * p.Hq + kv * G + g) * D + ch,
                      p.q_bf16);
      }
      q_s[e] = x;
    }
    __syncthreads();
    // lane4 takes queries lane4, lane4 + 4, lane4 + 8, lane4 + 12 of the chunk
    float s[kAQC / 4];
#pragma unroll
    for (int u = 0; u < kAQC / 4; ++u) s[u] = 0.0f;
    // 128-bit loads: the 4 queries of a lane are the same for the whole warp
    // (broadcast), the key rows differ by token (no bank conflict at stride KS)
    const float4* kr = reinterpret_cast<const float4*>(k_s + j * KS);
#pragma unroll 4
    for (int c4 = 0; c4 < D / 4; ++c4) {
      const float4 kc = kr[c4];
#pragma unroll
      for (int u = 0; u < kAQC / 4; ++u) {
        const float4 qv = reinterpret_cast<const float4*>(q_s + (lane4 + 4 * u) * D)[c4];
        s[u] = fmaf(qv.x, kc.x, s[u]);
        s[u] = fmaf(qv.y, kc.y, s[u]);
        s[u] = fmaf(qv.z, kc.z, s[u]);
        s[u] = fmaf(qv.w, kc.w, s[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kAQC / 4; ++u) {
      const int qq = lane4 + 4 * u;
      if (qq >= nq) break;  // uniform across the warp (lane4 is per warp)
      const float sv = valid ? s[u] * p.sm_scale : -INFINITY;
      if constexpr (!SCORE) {
        float m = sv;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o2));
        float l = valid ? expf(sv - m) : 0.0f;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o2);
        if ((tid & 31) == 0) {
          const int half = (j >> 5);
          p.part[((bk * p.ntiles + tile) * p.ppt + half) * NQ + q0 + qq] = make_float2(m, l);
        }
      } else {
        const float pj = valid ? expf(sv - p.lse[bk * NQ + q0 + qq]) : 0.0f;
        acc2 = fmaf(pj, pj, acc2);
      }
    }
  }
  if constexpr (SCORE) {
    __syncthreads();
    red_s[tid] = acc2;
    __syncthreads();
    if (tid < kAT && t0 + tid < p.T) {
      const float w = (red_s[tid] + red_s[tid + kAT]) + (red_s[tid + 2 * kAT] + red_s[tid + 3 * kAT]);
      p.scores[bk * p.T + t0 + tid] = t0 + tid < Tb ? w * dv2_s[tid] : 0.0f;
    }
  }
}

// ---- the same two passes on tensor cores, for bf16 keys and queries ---------
// Observation queries on the MMA M side: warp w holds queries [16 w, 16 w + 16)
// of a chunk of kQW * 16 as A fragments (all k-steps, in registers for the
// CTA's whole walk), and a CTA walks kTPC 64-token tiles of one (b, kv), each
// tile's keys (the B operand: tokens on N, from padded rows with 32-bit loads,
// lanes on distinct banks) streamed through two cp.async buffers so the next
// tile loads during the current tile's MMAs.  Logits = Q K^T on mma.sync
// m16n8k16 bf16 -> fp32: products of bf16 values are exact, so this differs from
// the CUDA-core pass only in the order of the fp32 sums.
//   pass 0: a running max and sum per query row in each lane (its sixteen
//           columns of a tile: the tile's maximum first, then one exponential
//           per logit and one rescale of the sum), merged over the row's four
//           lanes at the end: one (max, sum) partial per (CTA, query)
//   pass 1: p^2 per (query, token) summed over the chunk's queries per token:
//           the row pair in each lane, the warp's rows by a butterfly over the
//           lanes of a column (each step keeps half of the columns), the warps
//           in shared memory
// |v^_j - v_j|^2 comes from a2_dv2_kernel, already in `scores`.
constexpr int kQW = 8;           // query warps: 16 queries each
constexpr int kMT = 32 * kQW;    // threads
constexpr int kTPC = 16;         // tiles per CTA

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
constexpr float kLog2eF = 1.4426950408889634f;
// 2^x, results below 2^-126 flushed to zero (2^-inf = 0)
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 16 bytes global -> shared, asynchronously; zero-filled when `valid` is false
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// four 8x8 b16 matrices; lane l gives the row address of matrix l / 8, row l % 8
__device__ __forceinline__ void ldsm_x4(const void* row, uint32_t (&r)[4]) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(row));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}

template <int D>
constexpr size_t a2_mma_smem() {
  return sizeof(uint16_t) * (2 * kAT + 16 * kQW) * (D + 8) +
         sizeof(float) * (kQW * kAT + kTPC * kAT);
}

template <int D, bool SCORE>
__global__ void __launch_bounds__(kMT, 3) a2_pass_mma_kernel(const A2Params p) {
  constexpr int RS = D + 8;  // bf16 elements per shared row
  constexpr int KSTEPS = D / 16;
  constexpr int CPR = D / 8; // 16-byte chunks per row
  constexpr int QC = 16 * kQW;
  constexpr float kL2e = 1.4426950408889634f;
  constexpr float kLn2f = 0.6931471805599453f;
  extern __shared__ __align__(16) unsigned char a2m_smem[];
  uint16_t* k_s = reinterpret_cast<uint16_t*>(a2m_smem);          // [2][kAT][RS]
  uint16_t* q_s = k_s + 2 * kAT * RS;                               // [QC][RS]
  float* red_s = reinterpret_cast<float*>(q_s + QC * RS);          // [kQW][kAT] per-warp sums
  float* acc_s = red_s + kQW * kAT;                                 // [kTPC][kAT] sum p^2

  const int kv = blockIdx.y, b = blockIdx.z;
  const int tile_first = blockIdx.x * kTPC;
  const int ntl = min(kTPC, p.ntiles - tile_first);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int Tb = seq_len(p.seq_lens, b, p.T);
  const int G = p.G, NQ = p.n_obs * G;
  const size_t bk = static_cast<size_t>(b) * p.c.Hkv + kv;
  const uint16_t* kf = static_cast<const uint16_t*>(p.k_full);
  const uint16_t* qo = static_cast<const uint16_t*>(p.q_obs);
  const float s2 = p.sm_scale * kL2e;  // logits in log2 units

  // the key rows of local tile k into buffer buf (rows past T_b read as zero)
  auto load_tile = [&](int k, int buf) {
    const int t0 = (tile_first + k) * kAT;
    uint16_t* dst = k_s + buf * kAT * RS;
    for (int e = tid; e < kAT * CPR; e += kMT) {
      const int row = e / CPR, c8 = e - row * CPR;
      const bool valid = t0 + row < Tb;
      const uint16_t* src = kf + (bk * p.T + (valid ? t0 + row : 0)) * D + c8 * 8;
      cp_async16(dst + row * RS + c8 * 8, src, valid);
    }
    cp_async_commit();
  };
  if constexpr (SCORE)
    for (int e = tid; e < kTPC * kAT; e += kMT) acc_s[e] = 0.0f;

  for (int q0 = 0; q0 < NQ; q0 += QC) {
    const int nq = min(QC, NQ - q0);
    __syncthreads();  // every warp is done with the previous query chunk
    for (int e = tid; e < QC * CPR; e += kMT) {
      const int qq = e / CPR, c8 = e - qq * CPR;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (qq < nq) {
        const int qi = q0 + qq, o = qi / G, gq = qi - o * G;
        v = *reinterpret_cast<const uint4*>(
            qo + ((static_cast<size_t>(b) * p.n_obs + o) * p.Hq + kv * G + gq) * D + c8 * 8);
      }
      *reinterpret_cast<uint4*>(q_s + qq * RS + c8 * 8) = v;
    }
    load_tile(0, 0);
    __syncthreads();  // the query chunk in shared memory
    // this warp's 16 queries as A fragments (rows g and g + 8)
    const bool wlive = 16 * warp < nq;
    const int qr0 = q0 + 16 * warp + g, qr1 = qr0 + 8;  // query indices of the two rows
    const bool r0 = qr0 < q0 + nq, r1 = qr1 < q0 + nq;
    uint32_t qa[KSTEPS][4];
    {
      const uint16_t* a0 = q_s + (16 * warp + g) * RS + 2 * t;
      const uint16_t* a1 = a0 + 8 * RS;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        qa[ks][0] = *reinterpret_cast<const uint32_t*>(a0 + 16 * ks);
        qa[ks][1] = *reinterpret_cast<const uint32_t*>(a1 + 16 * ks);
        qa[ks][2] = *reinterpret_cast<const uint32_t*>(a0 + 16 * ks + 8);
        qa[ks][3] = *reinterpret_cast<const uint32_t*>(a1 + 16 * ks + 8);
      }
    }
    // pass 0: running max (log2 units) and sum of the two rows over this lane's
    // columns; pass 1: the rows' lse in log2 units
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};
    float lse2[2] = {0.0f, 0.0f};
    if constexpr (SCORE) {
      if (r0) lse2[0] = p.lse[bk * NQ + qr0] * kL2e;
      if (r1) lse2[1] = p.lse[bk * NQ + qr1] * kL2e;
    }

    for (int k = 0; k < ntl; ++k) {
      const int tile = tile_first + k;
      if (k + 1 < ntl) {
        load_tile(k + 1, (k + 1) & 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();  // tile k in shared memory
      const uint16_t* kb = k_s + (k & 1) * kAT * RS;
      if (wlive) {
        // the tile's logits of this lane: rows g | g + 8 x tokens 8 nt + 2t, + 1
        float cv[kAT / 8][4];
#pragma unroll
        for (int nt = 0; nt < kAT / 8; ++nt) {
          cv[nt][0] = cv[nt][1] = cv[nt][2] = cv[nt][3] = 0.0f;
          // B fragments of two k-steps per ldmatrix: matrices = channels
          // [32 kk, +8), [+8, +16), [+16, +24), [+24, +32) of tokens 8 nt .. 8 nt + 7
          const uint16_t* br = kb + (8 * nt + (lane & 7)) * RS + 8 * (lane >> 3);
#pragma unroll
          for (int kk = 0; kk < KSTEPS / 2; ++kk) {
            uint32_t bf[4];
            ldsm_x4(br + 32 * kk, bf);
            mma_bf16_16816(cv[nt], qa[2 * kk], bf[0], bf[1]);
            mma_bf16_16816(cv[nt], qa[2 * kk + 1], bf[2], bf[3]);
          }
        }
        // tokens past T_b (the last tile of a sequence) take logit -inf
        if ((tile + 1) * kAT > Tb) {
#pragma unroll
          for (int nt = 0; nt < kAT / 8; ++nt) {
            const int j = tile * kAT + 8 * nt + 2 * t;
            if (j >= Tb) cv[nt][0] = cv[nt][2] = -INFINITY;
            if (j + 1 >= Tb) cv[nt][1] = cv[nt][3] = -INFINITY;
          }
        }
        if constexpr (!SCORE) {
          // per row: the tile's maximum, then one rescale of the running sum
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < kAT / 8; ++nt)
              mx = fmaxf(mx, fmaxf(cv[nt][2 * rr], cv[nt][2 * rr + 1]));
            const float mnew = fmaxf(m[rr], mx * s2);  // log2 units (s2 > 0)
            if (mnew != -INFINITY) {
              float acc = 0.0f;
#pragma unroll
              for (int nt = 0; nt < kAT / 8; ++nt)
                acc += ex2_ftz(fmaf(cv[nt][2 * rr], s2, -mnew)) +
                       ex2_ftz(fmaf(cv[nt][2 * rr + 1], s2, -mnew));
              l[rr] = fmaf(l[rr], ex2_ftz(m[rr] - mnew), acc);  // 2^-inf = 0
              m[rr] = mnew;
            }
          }
        } else {
          // p^2 summed over the warp's 16 rows for each of the lane's 16 columns
          // (v[2 nt + e] = token 8 nt + 2t + e), then a butterfly over the lanes
          // of the same t (xor 16, 8, 4): each step keeps half of the columns,
          // so that lane (g, t) ends with the sums of tokens 8g + 2t + {0, 1}
          float v[kAT / 4];
#pragma unroll
          for (int nt = 0; nt < kAT / 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float pa = r0 ? ex2_ftz(fmaf(cv[nt][e], s2, -lse2[0])) : 0.0f;
              const float pb = r1 ? ex2_ftz(fmaf(cv[nt][2 + e], s2, -lse2[1])) : 0.0f;
              v[2 * nt + e] = fmaf(pa, pa, pb * pb);
            }
          }
#pragma unroll
          for (int step = 0; step < 3; ++step) {
            const int bit = 16 >> step, n = 8 >> step;  // lanes apart, values kept
            const bool up = (lane & bit) != 0;
#pragma unroll
            for (int i = 0; i < n; ++i) {
              const float keep = up ? v[n + i] : v[i];
              const float give = up ? v[i] : v[n + i];
              v[i] = keep + __shfl_xor_sync(0xffffffffu, give, bit);
            }
          }
          red_s[warp * kAT + 8 * g + 2 * t] = v[0];
          red_s[warp * kAT + 8 * g + 2 * t + 1] = v[1];
        }
      }
      if constexpr (SCORE) {
        __syncthreads();  // every warp's token sums in red_s
        if (tid < kAT) {
          float a = 0.0f;
          for (int w = 0; w < kQW; ++w)
            if (16 * w < nq) a += red_s[w * kAT + tid];
          acc_s[k * kAT + tid] += a;
        }
      }
      __syncthreads();  // every warp is done with buffer k & 1 (and red_s) before reuse
    }
    if constexpr (!SCORE) {
      // merge the rows' (max, sum) over their four lanes; one partial per query
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
#pragma unroll
        for (int o2 = 1; o2 < 4; o2 <<= 1) {
          const float mo = __shfl_xor_sync(0xffffffffu, m[rr], o2);
          const float lo = __shfl_xor_sync(0xffffffffu, l[rr], o2);
          const float mx = fmaxf(m[rr], mo);
          if (mx != -INFINITY) {
            l[rr] = (m[rr] == -INFINITY ? 0.0f : l[rr] * exp2f(m[rr] - mx)) +
                    (mo == -INFINITY ? 0.0f : lo * exp2f(mo - mx));
            m[rr] = mx;
          }
        }
      }
      if (wlive && t == 0) {
        float2* dst = p.part + (bk * gridDim.x + blockIdx.x) * NQ;  // gridDim.x partials per (b, kv)
        // natural-log max; the sum is the same in either base
        if (r0) dst[qr0] = make_float2(m[0] == -INFINITY ? -INFINITY : m[0] * kLn2f, l[0]);
        if (r1) dst[qr1] = make_float2(m[1] == -INFINITY ? -INFINITY : m[1] * kLn2f, l[1]);
      }
    }
  }
  if constexpr (SCORE) {
    // scores holds |v^_j - v_j|^2 (a2_dv2_kernel); times sum_{o,h} p^2
    for (int e = tid; e < ntl * kAT; e += kMT) {
      const int tok = tile_first * kAT + e;
      if (tok >= p.T) continue;
      float* sc = p.scores + bk * p.T + tok;
      *sc = tok < Tb ? acc_s[e] * *sc : 0.0f;
    }
  }
}

// |v^_j - v_j|^2 of every token j < T into scores (0 for j >= T_b): one lane per
// (token, 32-channel group), summed over the token's D/32 lanes by shuffles;
// CTA (token block, kv, b).  2-bit values: the group's 32 exact bf16 values (four
// 16-byte loads), its 8 code bytes, scale and minimum; v^ = min + code * scale
// rounded as the codec rounds it (a rounded product, then a rounded sum), in
// packed fp32 pairs (each lane one IEEE round-to-nearest operation; separate
// PTX statements, so nothing is contracted); each code becomes an exact float
// as (2^23 | code) - 2^23.  Dense values: the cached values.
template <int D>
__global__ void __launch_bounds__(256) a2_dv2_kernel(const A2Params p) {
  constexpr int LPT = D / 32;          // lanes per token (one per group)
  constexpr int TPB = 256 / LPT;       // tokens per CTA
  const int kv = blockIdx.y, b = blockIdx.z;
  const int tt = blockIdx.x * TPB + threadIdx.x / LPT;
  const int g = threadIdx.x % LPT;
  const size_t bk = static_cast<size_t>(b) * p.c.Hkv + kv;
  const bool live = tt < seq_len(p.seq_lens, b, p.T);
  float a = 0.0f;
  if (live) {
    const size_t row = cache_row_read(p.c, b, kv, tt, g == 0 ? p.err : nullptr);
    const uint4* vp = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.v_full) +
                                                     (bk * p.T + tt) * D + 32 * g);
    uint32_t vw[16];  // the 32 exact values, bf16 pairs
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 u = vp[k];
      vw[4 * k] = u.x; vw[4 * k + 1] = u.y; vw[4 * k + 2] = u.z; vw[4 * k + 3] = u.w;
    }
    uint64_t acc = 0;  // (+0, +0)
    if (p.c.vmode == HEADQ_V_2BIT) {
      const uint2 cw = *reinterpret_cast<const uint2*>(p.c.v_codes + row * (D / 4) + 8 * g);
      const uint64_t sc = codec::dup2(p.c.v_scale[row * (D / 32) + g]);
      const uint64_t mn = codec::dup2(p.c.v_min[row * (D / 32) + g]);
      const uint64_t magic = codec::dup2(8388608.0f);  // 2^23
#pragma unroll
      for (int w = 0; w < 16; ++w) {  // channels 2w, 2w + 1 of the group
        const uint32_t word = w < 8 ? cw.x : cw.y;
        const uint32_t sh = 4 * (w & 7);
        const uint64_t code =
            codec::sub2(codec::pk2(__uint_as_float(((word >> sh) & 3u) | 0x4B000000u),
                                   __uint_as_float(((word >> (sh + 2)) & 3u) | 0x4B000000u)),
                        magic);
        const uint64_t vh = codec::add2(mn, codec::mul2(code, sc));
        const uint64_t v = codec::pk2(__uint_as_float(vw[w] << 16), __uint_as_float(vw[w] & 0xffff0000u));
        const uint64_t dv = codec::sub2(vh, v);
        acc = codec::fma2(dv, dv, acc);
      }
    } else {
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float vh[8];
        value_hat8(p.c, row, 32 * g + 8 * c8, D, vh);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t u = vw[4 * c8 + k];
          const uint64_t dv = codec::sub2(codec::pk2(vh[2 * k], vh[2 * k + 1]),
                                          codec::pk2(__uint_as_float(u << 16),
                                                     __uint_as_float(u & 0xffff0000u)));
          acc = codec::fma2(dv, dv, acc);
        }
      }
    }
    a = codec::pk_lo(acc) + codec::pk_hi(acc);
  }
#pragma unroll
  for (int o2 = 1; o2 < LPT; o2 <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o2);
  if (tt < p.T && g == 0) p.scores[bk * p.T + tt] = live ? a : 0.0f;
}

// lse of every observation query from the tile partials; one CTA per (b, kv)
__global__ void a2_lse_kernel(const A2Params p) {
  const size_t bk = blockIdx.x;
  const int NQ = p.n_obs * p.G;
  for (int qi = threadIdx.x; qi < NQ; qi += blockDim.x) {
    const int ne = p.ppt * p.ntiles;
    float M = -INFINITY;
    for (int e = 0; e < ne; ++e) M = fmaxf(M, p.part[(bk * ne + e) * NQ + qi].x);
    float L = 0.0f;
    if (M != -INFINITY)
      for (int e = 0; e < ne; ++e) {
        const float2 ml = p.part[(bk * ne + e) * NQ + qi];
        if (ml.x != -INFINITY) L += ml.y * expf(ml.x - M);
      }
    p.lse[bk * NQ + qi] = M == -INFINITY ? -INFINITY : M + logf(L);
  }
}

// exclusive prefix count of `flag` over the CTA (threads in order); returns it
// and the CTA total through *total.  Uses wsum (kSelThreads / 32 entries).
__device__ __forceinline__ int block_excl_count(bool flag, int* wsum, int* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  __syncthreads();
  if (lane == 0) wsum[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    const int v = lane < kSelThreads / 32 ? wsum[lane] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane < kSelThreads / 32) wsum[lane] = x - v;  // exclusive
    if (lane == 31) wsum[kSelThreads / 32] = x;       // total
  }
  __syncthreads();
  *total = wsum[kSelThreads / 32];
  return wsum[warp] + in_warp;
}

__global__ void __launch_bounds__(kSelThreads)
a2_select_kernel(const float* scores, int Hkv, const int32_t* seq_lens, int T, int K,
                 const void* v_full, int esz, int d, int32_t* keep_idx, void* keep_v) {
  __shared__ unsigned hist[256];
  __shared__ unsigned s_pre;
  __shared__ int s_rem;
  __shared__ int wsum[kSelThreads / 32 + 1];
  const size_t bk = blockIdx.x;
  const int b = static_cast<int>(bk / Hkv);
  const int tid = threadIdx.x;
  const int Tb = seq_len(seq_lens, b, T);
  const int Keff = min(K, Tb);
  const unsigned* key = reinterpret_cast<const unsigned*>(scores + bk * T);
  int32_t* out_idx = keep_idx + bk * K;

  // radix select, 8 bits at a time from the top: s_pre ends as the bit pattern
  // of the Keff-th largest score, s_rem as how many of the kept tokens equal it
  if (tid == 0) {
    s_pre = 0u;
    s_rem = Keff;
  }
  // the first kSelReg * kSelThreads scores stay in registers for all passes
  unsigned kr[kSelReg];
#pragma unroll
  for (int c = 0; c < kSelReg; ++c) {
    const int t = c * kSelThreads + tid;
    kr[c] = t < Tb ? key[t] : 0u;
  }
  unsigned mask = 0u;
  const int lane = tid & 31;
  for (int shift = 24; shift >= 0 && Keff > 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0u;
    __syncthreads();
    const unsigned pre = s_pre;
    // the lanes of a warp with the same bin (lanes outside share 256): one atomic
    // per distinct bin, by its lowest lane
    auto count = [&](unsigned u, bool valid) {
      const bool in = valid && (u & mask) == pre;
      const unsigned bin = in ? (u >> shift) & 255u : 256u;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<unsigned>(__popc(peers)));
    };
#pragma unroll
    for (int c = 0; c < kSelReg; ++c)
      if (c * kSelThreads < Tb) count(kr[c], c * kSelThreads + tid < Tb);
    for (int t0 = kSelReg * kSelThreads; t0 < Tb; t0 += kSelThreads) {
      const int t = t0 + tid;
      count(t < Tb ? key[t] : 0u, t < Tb);
    }
    __syncthreads();
    // the bin holding the s_rem-th largest: counts summed from the top bin down
    // (thread i <-> bin 255 - i), an inclusive scan over the 256 threads
    if (tid < 256) {
      const int rem = s_rem;
      const unsigned h = hist[255 - tid];
      unsigned c = h;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, c, o);
        if (lane >= o) c += y;
      }
      if (lane == 31) wsum[tid >> 5] = static_cast<int>(c);
      asm volatile("bar.sync 2, 256;" ::: "memory");
      unsigned before = 0u;
      for (int w = 0; w < (tid >> 5); ++w) before += static_cast<unsigned>(wsum[w]);
      c += before;
      if (c >= static_cast<unsigned>(rem) && c - h < static_cast<unsigned>(rem)) {
        s_rem = rem - static_cast<int>(c - h);
        s_pre = pre | (static_cast<unsigned>(255 - tid) << shift);
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  const unsigned tau = s_pre;
  const int need_eq = s_rem;

  // ordered compaction: every token above tau, and the first need_eq equal to it
  int base = 0, eq_base = 0;
  auto compact = [&](unsigned u, int t) {
    const bool eq = t < Tb && u == tau;
    int eq_total = 0;
    const int eq_rank = block_excl_count(eq, wsum, &eq_total);
    const bool take = t < Tb && (u > tau || (eq && eq_base + eq_rank < need_eq));
    int take_total = 0;
    const int pos = block_excl_count(take, wsum, &take_total);
    if (take && base + pos < Keff) out_idx[base + pos] = t;
    base += take_total;
    eq_base += eq_total;
  };
  if (Keff > 0) {
#pragma unroll
    for (int c = 0; c < kSelReg; ++c)
      if (c * kSelThreads < Tb) compact(kr[c], c * kSelThreads + tid);
    for (int t0 = kSelReg * kSelThreads; t0 < Tb; t0 += kSelThreads) {
      const int t = t0 + tid;
      compact(t < Tb ? key[t] : 0u, t);
    }
  }
  for (int k = Keff + tid; k < K; k += kSelThreads) out_idx[k] = -1;
  __syncthreads();

  // exact values of the kept tokens (raw elements of v_full), zero for the pad
  const int row_bytes = d * esz;
  const uint8_t* vsrc = static_cast<const uint8_t*>(v_full);
  uint8_t* vdst = static_cast<uint8_t*>(keep_v) + bk * K * row_bytes;
  for (int e = tid; e < K * (row_bytes / 4); e += kSelThreads) {
    const int k = e / (row_bytes / 4), w = e - k * (row_bytes / 4);
    uint32_t x = 0u;
    if (k < Keff) {
      const int t = out_idx[k];
      x = reinterpret_cast<const uint32_t*>(vsrc + (bk * T + t) * row_bytes)[w];
    }
    reinterpret_cast<uint32_t*>(vdst + static_cast<size_t>(k) * row_bytes)[w] = x;
  }
}

struct FixParams {
  headq_cache c;
  const void* q;
  bool q_bf16;
  int Hq, G, T;
  const int32_t* seq_lens;
  const float* U;
  float sm_scale, corr_sign;
  const int32_t* keep_idx;
  const void* keep_v;
  bool keep_bf16;
  int K;
  float* out;
  const float* lse;
};

// shared-memory layout of one fixup chunk: the kept tokens' key planes
template <int D>
struct FixStage {
  static constexpr int NG = num_groups(D);
  static constexpr int kKcWords = (D + 15) / 16;  // 2-bit codes, 16 per word (d = 8: half)
  static constexpr int kZcBytes = 16;      // side codes, r <= 32
  static constexpr size_t bytes() {
    return sizeof(uint32_t) * kFixTok * kKcWords + sizeof(float) * kFixTok * (2 * NG + 1) +
           kFixTok * kZcBytes;
  }
};

template <int D>
__global__ void __launch_bounds__(kFixThreads) a2_fixup_kernel(const FixParams p) {
  constexpr int GS = group_size(D), NG = num_groups(D);
  using FS = FixStage<D>;
  extern __shared__ float sm[];
  const int G = p.G, r = p.c.r;
  float* dv_s = sm;                   // [kFixTok][D]  (first: 16-byte aligned rows)
  float* q_s = dv_s + kFixTok * D;    // [G][D]
  float* qg_s = q_s + G * D;          // [G][NG]
  float* qt_s = qg_s + G * NG;        // [G][r]
  float* lse_s = qt_s + G * r;        // [G]
  // weights exp(s^_j - lse) [kFixTok][PS]: PS = kFixHeads (16-byte rows, heads
  // G.. zero) when the accumulation is blocked by channel, else G
  const bool blocked = D >= 64 && G <= kFixHeads;
  const int PS = blocked ? kFixHeads : G;
  float* p_s = smem_align(lse_s + G, 16);
  // kept-token indices and cache rows of a chunk of kFixIdx (every step of it)
  int* idx_all = reinterpret_cast<int*>(p_s + kFixTok * PS);         // [kFixIdx]
  size_t* row_all = reinterpret_cast<size_t*>(smem_align(idx_all + kFixIdx, 8));  // [kFixIdx]
  uint32_t* kc_s = reinterpret_cast<uint32_t*>(row_all + kFixIdx);   // [kFixTok][D/16]
  float* ks_s = reinterpret_cast<float*>(kc_s + kFixTok * FS::kKcWords);  // [kFixTok][NG]
  float* km_s = ks_s + kFixTok * NG;                                  // [kFixTok][NG]
  float* zs_s = km_s + kFixTok * NG;                                  // [kFixTok]
  uint8_t* zc_s = reinterpret_cast<uint8_t*>(zs_s + kFixTok);         // [kFixTok][16]

  const int kv = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int h0 = kv * G;
  const int Tb = seq_len(p.seq_lens, b, p.T);
  if (Tb == 0) return;  // out = 0, lse = -inf: nothing to correct
  const size_t bk = static_cast<size_t>(b) * p.c.Hkv + kv;

  for (int i = tid; i < G * D; i += kFixThreads)
    q_s[i] = load_elem(p.q, (static_cast<size_t>(b) * p.Hq + h0) * D + i, p.q_bf16);
  for (int h = tid; h < G; h += kFixThreads) lse_s[h] = p.lse[static_cast<size_t>(b) * p.Hq + h0 + h];
  for (int e = tid; e < kFixTok * PS; e += kFixThreads) p_s[e] = 0.0f;  // padded heads stay 0
  __syncthreads();
  for (int i = tid; i < G * NG; i += kFixThreads) {
    const int h = i / NG, g = i - h * NG;
    float acc = 0.0f;
    for (int c = 0; c < GS; ++c) acc += q_s[h * D + g * GS + c];
    qg_s[i] = acc;
  }
  // sigma U_h^T q, with U_h staged in the (not yet used) value-difference buffer
  float* u_s = dv_s;
  for (int i = tid; i < D * r; i += kFixThreads) u_s[i] = p.U[static_cast<size_t>(kv) * D * r + i];
  __syncthreads();
  for (int i = tid; i < G * r; i += kFixThreads) {
    const int h = i / r, ii = i - h * r;
    float acc = 0.0f;
    for (int c = 0; c < D; ++c) acc = fmaf(u_s[c * r + ii], q_s[h * D + c], acc);
    qt_s[i] = p.corr_sign * acc;
  }

  // blocked (G <= kFixHeads, D >= 64, so that the [TQ][kFixHeads][D] class sums
  // fit in the value-difference tile): acc[h] = head h, channel cf, the tokens of
  // class tq; else acc[k] = output tid + k * kFixThreads over all tokens
  static_assert(D < 64 || kFixThreads * kFixHeads <= kFixTok * D, "class sums fit");
  constexpr int kAcc = kFixMaxOut > kFixHeads ? kFixMaxOut : kFixHeads;
  const int cf = tid % D, tq = tid / D;
  float acc[kAcc];
#pragma unroll
  for (int k = 0; k < kAcc; ++k) acc[k] = 0.0f;

  for (int k0 = 0; k0 < p.K; k0 += kFixTok) {
    __syncthreads();
    if (k0 % kFixIdx == 0) {  // a new chunk: every step's indices and rows at once
      for (int k = tid; k < kFixIdx; k += kFixThreads) {
        const int t = k0 + k < p.K ? p.keep_idx[bk * p.K + k0 + k] : -1;
        const bool ok = t >= 0 && t < Tb;
        idx_all[k] = ok ? t : -1;
        row_all[k] = ok ? cache_row_read(p.c, b, kv, t, nullptr) : 0;
      }
      __syncthreads();
    }
    const int* idx_s = idx_all + k0 % kFixIdx;     // this step's kFixTok entries
    const size_t* row_s = row_all + k0 % kFixIdx;
    // stage the kept tokens' key planes (word-wide, all threads)
    if constexpr (D >= 16) {
      for (int e = tid; e < kFixTok * FS::kKcWords; e += kFixThreads) {
        const int tt = e / FS::kKcWords, w = e - tt * FS::kKcWords;
        kc_s[e] = idx_s[tt] >= 0
                      ? reinterpret_cast<const uint32_t*>(p.c.k_codes + row_s[tt] * (D / 4))[w]
                      : 0u;
      }
    } else {  // d = 8: a 2-byte code row, staged byte by byte into the low half
      for (int tt = tid; tt < kFixTok; tt += kFixThreads) {
        uint32_t x = 0u;
        if (idx_s[tt] >= 0)
          for (int by = 0; by < D / 4; ++by)
            x |= static_cast<uint32_t>(p.c.k_codes[row_s[tt] * (D / 4) + by]) << (8 * by);
        kc_s[tt] = x;
      }
    }
    for (int e = tid; e < kFixTok * NG; e += kFixThreads) {
      const int tt = e / NG, g = e - tt * NG;
      const bool ok = idx_s[tt] >= 0;
      ks_s[e] = ok ? p.c.k_scale[row_s[tt] * NG + g] : 0.0f;
      km_s[e] = ok ? p.c.k_min[row_s[tt] * NG + g] : 0.0f;
    }
    if (r > 0) {
      for (int e = tid; e < kFixTok * (r / 2); e += kFixThreads) {
        const int tt = e / (r / 2), w = e - tt * (r / 2);
        zc_s[tt * FS::kZcBytes + w] = idx_s[tt] >= 0 ? p.c.z_codes[row_s[tt] * (r / 2) + w] : 0;
      }
      for (int tt = tid; tt < kFixTok; tt += kFixThreads)
        zs_s[tt] = idx_s[tt] >= 0 ? p.c.z_scale[row_s[tt]] : 0.0f;
    }
    // exact value minus cached value, 8 channels per task (wide loads)
    for (int e = tid; e < kFixTok * (D / 8); e += kFixThreads) {
      const int tt = e / (D / 8), c0 = (e - tt * (D / 8)) * 8;
      float dv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (idx_s[tt] >= 0) {
        float v[8], vh[8];
        load8(p.keep_v, (bk * p.K + k0 + tt) * D + c0, p.keep_bf16, v);
        value_hat8(p.c, row_s[tt], c0, D, vh);
#pragma unroll
        for (int k = 0; k < 8; ++k) dv[k] = v[k] - vh[k];
      }
      float4* dst = reinterpret_cast<float4*>(dv_s + tt * D + c0);
      dst[0] = make_float4(dv[0], dv[1], dv[2], dv[3]);
      dst[1] = make_float4(dv[4], dv[5], dv[6], dv[7]);
    }
    __syncthreads();
    // weights exp(s^_j - lse) of the kept tokens, per head.  D >= 16: kFP lanes
    // per token (aligned in a warp), each with one 16-channel slice (inside one
    // group) for every head and every kFP-th side row; the slices are summed by
    // shuffles.  d = 8: one lane per (token, head).
    if constexpr (D >= 16) {
      constexpr int kFP = D / 16;                  // lanes per token, a power of two <= 16
      constexpr int kTPP = kFixThreads / kFP;      // tokens per pass
      const int part = tid % kFP, c0 = 16 * part, g = c0 / GS;
      const bool first_of_group = (c0 % GS) == 0;
      for (int tt = tid / kFP; tt < kFixTok; tt += kTPP) {
        const bool live = idx_s[tt] >= 0;
        const uint32_t cw = kc_s[tt * FS::kKcWords + part];
        float code[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) code[k] = static_cast<float>((cw >> (2 * k)) & 3u);
        const float ksc = ks_s[tt * NG + g], kmn = km_s[tt * NG + g];
        const float zs = r > 0 ? zs_s[tt] : 0.0f;  // (not staged without a side code)
        const uint8_t* zr = zc_s + tt * FS::kZcBytes;
        for (int h = 0; h < G; ++h) {
          const float4* qh = reinterpret_cast<const float4*>(q_s + h * D + c0);
          float pg = 0.0f;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const float4 qv = qh[k4];
            pg = fmaf(qv.x, code[4 * k4], pg);
            pg = fmaf(qv.y, code[4 * k4 + 1], pg);
            pg = fmaf(qv.z, code[4 * k4 + 2], pg);
            pg = fmaf(qv.w, code[4 * k4 + 3], pg);
          }
          float sp = ksc * pg;
          if (first_of_group) sp = fmaf(kmn, qg_s[h * NG + g], sp);
          if (r > 0) {
            float cz = 0.0f;
            for (int i = part; i < r; i += kFP)
              cz = fmaf(qt_s[h * r + i], static_cast<float>(nibble(zr, i)), cz);
            sp = fmaf(zs, cz, sp);
          }
#pragma unroll
          for (int o2 = 1; o2 < kFP; o2 <<= 1) sp += __shfl_xor_sync(0xffffffffu, sp, o2);
          if (part == 0) p_s[tt * PS + h] = live ? ex2_ftz((sp * p.sm_scale - lse_s[h]) * kLog2eF) : 0.0f;
        }
      }
    } else {
      for (int pr = tid; pr < kFixTok * G; pr += kFixThreads) {
        const int tt = pr / G, h = pr - tt * G;
        float w = 0.0f;
        if (idx_s[tt] >= 0) {
          const uint32_t* cw = kc_s + tt * FS::kKcWords;
          const float* qh = q_s + h * D;
          float s = 0.0f;
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            float pg = 0.0f;
#pragma unroll
            for (int c = 0; c < GS; ++c) {
              const int ch = g * GS + c;
              const uint32_t code = (cw[ch >> 4] >> (2 * (ch & 15))) & 3u;
              pg = fmaf(qh[ch], static_cast<float>(code), pg);
            }
            s = fmaf(km_s[tt * NG + g], qg_s[h * NG + g], s);
            s = fmaf(ks_s[tt * NG + g], pg, s);
          }
          if (r > 0) {
            const uint8_t* zr = zc_s + tt * FS::kZcBytes;
            float cz = 0.0f;
            for (int i = 0; i < r; ++i) cz = fmaf(qt_s[h * r + i], static_cast<float>(nibble(zr, i)), cz);
            s = fmaf(zs_s[tt], cz, s);
          }
          w = expf(s * p.sm_scale - lse_s[h]);
        }
        p_s[tt * PS + h] = w;
      }
    }
    __syncthreads();
    if (blocked) {
      // thread (c, tq): channel c for every head over the tokens tt = tq mod TQ
      // of the step (one value load, the heads' weights as broadcasts)
#pragma unroll 4
      for (int tt = tq; tt < kFixTok; tt += kFixThreads / D) {
        const float dv = dv_s[tt * D + cf];
        const float4 pa = reinterpret_cast<const float4*>(p_s + tt * kFixHeads)[0];
        const float4 pb = reinterpret_cast<const float4*>(p_s + tt * kFixHeads)[1];
        acc[0] = fmaf(pa.x, dv, acc[0]); acc[1] = fmaf(pa.y, dv, acc[1]);
        acc[2] = fmaf(pa.z, dv, acc[2]); acc[3] = fmaf(pa.w, dv, acc[3]);
        acc[4] = fmaf(pb.x, dv, acc[4]); acc[5] = fmaf(pb.y, dv, acc[5]);
        acc[6] = fmaf(pb.z, dv, acc[6]); acc[7] = fmaf(pb.w, dv, acc[7]);
      }
    } else {
#pragma unroll
      for (int k = 0; k < kFixMaxOut; ++k) {
        const int idx = tid + k * kFixThreads;
        if (idx < G * D) {
          const int h = idx / D, c = idx - h * D;
          float a = acc[k];
#pragma unroll
          for (int tt = 0; tt < kFixTok; ++tt) a = fmaf(p_s[tt * PS + h], dv_s[tt * D + c], a);
          acc[k] = a;
        }
      }
    }
  }
  if (blocked) {
    // the token classes' sums, in a fixed order, through shared memory
    constexpr int TQ = kFixThreads / D;
    __syncthreads();
    float* red = dv_s;  // [TQ][kFixHeads][D], inside the (consumed) value-difference tile
#pragma unroll
    for (int h = 0; h < kFixHeads; ++h)
      if (h < G) red[(tq * kFixHeads + h) * D + cf] = acc[h];
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kFixThreads) {
      const int h = idx / D, c = idx - h * D;
      float a = 0.0f;
      for (int q = 0; q < TQ; ++q) a += red[(q * kFixHeads + h) * D + c];
      p.out[(static_cast<size_t>(b) * p.Hq + h0 + h) * D + c] += a;
    }
  } else {
#pragma unroll
    for (int k = 0; k < kFixMaxOut; ++k) {
      const int idx = tid + k * kFixThreads;
      if (idx < G * D) {
        const int h = idx / D, c = idx - h * D;
        p.out[(static_cast<size_t>(b) * p.Hq + h0 + h) * D + c] += acc[k];
      }
    }
  }
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

int score_tiles(int T) { return (T + kAT - 1) / kAT; }

size_t a2_ws_bytes(const headq_cache* c, int n_obs, int Hq, int T) {
  const size_t NQ = static_cast<size_t>(n_obs) * (Hq / c->Hkv);
  const size_t units = static_cast<size_t>(c->B) * c->Hkv;
  return kWsHeaderBytes + round256(sizeof(float2) * units * score_tiles(T) * 4 * NQ) +
         round256(sizeof(float) * units * NQ);
}

template <int D>
cudaError_t launch_scores(A2Params p, cudaStream_t s) {
  dim3 grid(p.ntiles, p.c.Hkv, p.c.B);
  const int NQ = p.n_obs * p.G;
  if constexpr (D == 64 || D == 128) {
    if (p.kv_bf16 && p.q_bf16) {  // tensor cores
      p.ppt = 4;
      constexpr size_t smem = a2_mma_smem<D>();
      static std::once_flag once;
      static cudaError_t attr = cudaSuccess;
      std::call_once(once, [] {
        attr = cudaFuncSetAttribute(a2_pass_mma_kernel<D, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (attr == cudaSuccess)
          attr = cudaFuncSetAttribute(a2_pass_mma_kernel<D, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      });
      if (attr != cudaSuccess) return attr;
      const int parts = (p.ntiles + kTPC - 1) / kTPC;  // CTAs per (b, kv)
      const dim3 mgrid(parts, p.c.Hkv, p.c.B);
      a2_pass_mma_kernel<D, false><<<mgrid, kMT, smem, s>>>(p);
      A2Params pl = p;  // the normaliser merges one partial per CTA
      pl.ntiles = parts;
      pl.ppt = 1;
      a2_lse_kernel<<<p.c.B * p.c.Hkv, NQ < 1024 ? (NQ + 31) / 32 * 32 : 1024, 0, s>>>(pl);
      constexpr int kDv2Tok = 256 / (D / 32);
      a2_dv2_kernel<D><<<dim3((p.T + kDv2Tok - 1) / kDv2Tok, p.c.Hkv, p.c.B), 256, 0, s>>>(p);
      a2_pass_mma_kernel<D, true><<<mgrid, kMT, smem, s>>>(p);
      return cudaGetLastError();
    }
  }
  p.ppt = 2;
  const size_t smem = sizeof(float) * (kAT * (D + 4) + kAQC * D + kAThreads + kAT);
  auto k0 = a2_pass_kernel<D, false>;
  auto k1 = a2_pass_kernel<D, true>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k0, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  k0<<<grid, kAThreads, smem, s>>>(p);
  a2_lse_kernel<<<p.c.B * p.c.Hkv, NQ < 1024 ? (NQ + 31) / 32 * 32 : 1024, 0, s>>>(p);
  k1<<<grid, kAThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_fixup(const FixParams& p, cudaStream_t s) {
  const int G = p.G;
  const size_t smem = sizeof(float) * (static_cast<size_t>(G) * D + G * num_groups(D) +
                                       G * p.c.r + G + kFixTok * std::max(G, kFixHeads) +
                                       kFixTok * D) + 16 +
                      sizeof(int) * (kFixIdx + 2) + sizeof(size_t) * kFixIdx + FixStage<D>::bytes();
  auto k = a2_fixup_kernel<D>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  k<<<dim3(p.c.Hkv, p.c.B), kFixThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace headq

using namespace headq;

HEADQ_API size_t headq_a2_workspace_bytes(const headq_cache* cache, int n_obs, int Hq, int T) {
  if (!cache || cache->Hkv <= 0 || n_obs <= 0 || Hq <= 0 || T < 0) return 0;
  return a2_ws_bytes(cache, n_obs, Hq, T);
}

HEADQ_API headq_status headq_a2_scores(const headq_cache* cache, const void* q_obs,
                                       headq_dtype q_dtype, int n_obs, int Hq,
                                       const int32_t* seq_lens, int T, const void* k_full,
                                       const void* v_full, headq_dtype kv_dtype, float sm_scale,
                                       float* scores, void* ws, size_t ws_bytes,
                                       headq_stream_t stream) {
  headq_status st = check_cache(cache);
  if (st != HEADQ_OK) return st;
  if (!q_obs || !aligned16(q_obs)) return HEADQ_ERR_INVALID_ARG;
  if (q_dtype != HEADQ_F32 && q_dtype != HEADQ_BF16) return HEADQ_ERR_INVALID_ARG;
  if (Hq <= 0 || Hq % cache->Hkv != 0 || T < 0 || T > cache->T_cap || n_obs <= 0)
    return HEADQ_ERR_INVALID_ARG;
  if (kv_dtype != HEADQ_F32 && kv_dtype != HEADQ_BF16) return HEADQ_ERR_INVALID_ARG;
  if (!k_full || !v_full || !scores || !aligned16(k_full) || !aligned16(v_full) ||
      !aligned16(scores) || (seq_lens && !aligned16(seq_lens)))
    return HEADQ_ERR_INVALID_ARG;
  if (cache->d < 8 || cache->d > 256) return HEADQ_ERR_UNSUPPORTED;
  if (!ws || !aligned16(ws) || ws_bytes < a2_ws_bytes(cache, n_obs, Hq, T))
    return HEADQ_ERR_WORKSPACE;
  if (cache->B == 0 || T == 0) return HEADQ_OK;
  A2Params p{};
  p.c = *cache;
  p.q_obs = q_obs;
  p.q_bf16 = q_dtype == HEADQ_BF16;
  p.n_obs = n_obs;
  p.Hq = Hq;
  p.G = Hq / cache->Hkv;
  p.T = T;
  p.seq_lens = seq_lens;
  p.k_full = k_full;
  p.v_full = v_full;
  p.kv_bf16 = kv_dtype == HEADQ_BF16;
  p.sm_scale = sm_scale;
  p.ntiles = score_tiles(T);
  p.err = static_cast<unsigned*>(ws);
  const size_t units = static_cast<size_t>(cache->B) * cache->Hkv;
  const size_t NQ = static_cast<size_t>(n_obs) * p.G;
  p.part = reinterpret_cast<float2*>(static_cast<char*>(ws) + kWsHeaderBytes);
  p.lse = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsHeaderBytes +
                                   round256(sizeof(float2) * units * p.ntiles * 4 * NQ));
  p.scores = scores;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (cache->d) {
    case 8: e = launch_scores<8>(p, s); break;
    case 16: e = launch_scores<16>(p, s); break;
    case 32: e = launch_scores<32>(p, s); break;
    case 64: e = launch_scores<64>(p, s); break;
    case 128: e = launch_scores<128>(p, s); break;
    case 256: e = launch_scores<256>(p, s); break;
    default: return HEADQ_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? HEADQ_OK : HEADQ_ERR_CUDA;
}

HEADQ_API headq_status headq_a2_select(const float* scores, int B, int Hkv,
                                       const int32_t* seq_lens, int T, int K, const void* v_full,
                                       headq_dtype kv_dtype, int d, int32_t* keep_idx,
                                       void* keep_v, headq_stream_t stream) {
  if (B < 0 || Hkv <= 0 || T < 0 || K < 0 || d <= 0 || d % 8 != 0) return HEADQ_ERR_INVALID_ARG;
  if (kv_dtype != HEADQ_F32 && kv_dtype != HEADQ_BF16) return HEADQ_ERR_INVALID_ARG;
  if (B == 0 || K == 0) return HEADQ_OK;
  if (!scores || !v_full || !keep_idx || !keep_v || !aligned16(scores) || !aligned16(v_full) ||
      !aligned16(keep_idx) || !aligned16(keep_v) || (seq_lens && !aligned16(seq_lens)))
    return HEADQ_ERR_INVALID_ARG;
  a2_select_kernel<<<B * Hkv, kSelThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      scores, Hkv, seq_lens, T, K, v_full, kv_dtype == HEADQ_BF16 ? 2 : 4, d, keep_idx, keep_v);
  return cudaGetLastError() == cudaSuccess ? HEADQ_OK : HEADQ_ERR_CUDA;
}

HEADQ_API headq_status headq_a2_value_fixup(const headq_cache* cache, const void* q,
                                            headq_dtype q_dtype, int Hq, const int32_t* seq_lens,
                                            int T, const float* U, float sm_scale, int corr_sign,
                                            const int32_t* keep_idx, const void* keep_v,
                                            headq_dtype keep_dtype, int K, float* out,
                                            const float* lse, headq_stream_t stream) {
  headq_status st = check_read_args(cache, q, q_dtype, Hq, T, U, corr_sign);
  if (st != HEADQ_OK) return st;
  if (cache->kmode != HEADQ_K_TOKEN) return HEADQ_ERR_UNSUPPORTED;
  if (K < 0 || (keep_dtype != HEADQ_F32 && keep_dtype != HEADQ_BF16)) return HEADQ_ERR_INVALID_ARG;
  if (!out || !lse || !aligned16(out) || !aligned16(lse) || (seq_lens && !aligned16(seq_lens)))
    return HEADQ_ERR_INVALID_ARG;
  if (cache->B == 0 || K == 0) return HEADQ_OK;
  if (!keep_idx || !keep_v || !aligned16(keep_idx) || !aligned16(keep_v))
    return HEADQ_ERR_INVALID_ARG;
  FixParams p{};
  p.c = *cache;
  p.q = q;
  p.q_bf16 = q_dtype == HEADQ_BF16;
  p.Hq = Hq;
  p.G = Hq / cache->Hkv;
  p.T = T;
  p.seq_lens = seq_lens;
  p.U = U;
  p.sm_scale = sm_scale;
  p.corr_sign = static_cast<float>(corr_sign);
  p.keep_idx = keep_idx;
  p.keep_v = keep_v;
  p.keep_bf16 = keep_dtype == HEADQ_BF16;
  p.K = K;
  p.out = out;
  p.lse = lse;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (cache->d) {
    case 8: e = launch_fixup<8>(p, s); break;
    case 16: e = launch_fixup<16>(p, s); break;
    case 32: e = launch_fixup<32>(p, s); break;
    case 64: e = launch_fixup<64>(p, s); break;
    case 128: e = launch_fixup<128>(p, s); break;
    case 256: e = launch_fixup<256>(p, s); break;
    default: return HEADQ_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? HEADQ_OK : HEADQ_ERR_CUDA;
}
