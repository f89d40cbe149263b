// HeadQ model-visible distortion diagnostics on tensor cores ("HeadQ: Model-Visible
// Distortion and Score-Space Correction for KV-Cache Quantization", gist.science
// summary, section 2.1 -- the score perturbation delta_j = s^_j - s_j, the
// attention KL and its local Fisher-weighted variance -- and section 2.2 -- the
// readout error sum_j p_j dv_j at fixed p and the A^2 = p_j^2 weighted value
// distortion).  Same quantities, same split partials and the same combine kernel
// as attn_kl.cu; this kernel computes the per-token terms with MMAs:
//
//  * Logits with the query heads on M (rows h: bf16 high part of head h's query,
//    rows h + 8: its low part) and 8 tokens on N.  The exact keys come straight
//    from a 128-byte-swizzled TMA tile through ldmatrix; the 2-bit codes are
//    unpacked exactly to bf16 with the same channel order.  Both products use the
//    same query fragments and keep one accumulator per 32-channel group g, so
//        delta_j = sm * sum_g (min_jg Q_g + scale_jg q.code_jg - q.k_jg)
//                  + sm * sigma * z_scale_j (U^T q).w_j
//    is formed group by group from fp32 partial sums of the same rounded query:
//    the query's rounding enters delta only through the key error itself.  The
//    side-code term is one fp16 MMA (as in the decode kernels).
//  * Per (token, head): w = e^{s - m}, fp64 running sums W, X = sum w e^{delta -
//    md}, M1 = sum w delta, M2 = sum w delta^2, A2 = sum w^2 |dv|^2, with m and
//    md the running maxima of s and delta.
//  * The value error dv = v^ - v (cached value against the exact one) is formed
//    per (token, dim) from two swizzled tiles and enters
//    dov = sum_j w_j dv_j as bf16 high/low MMA operands (dims on M, tokens on K,
//    heads on N: w is already in the B layout of the logit accumulators).
//  * One TMA producer warp, two stages of 112 tokens, seven consumer warps of 16
//    tokens each; bounded mbarrier waits that flag the workspace error word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "decode_common.cuh"

namespace headq {
namespace {
using namespace dc;

// seven consumer warps and the producer: 256 threads, the most a CTA can have at
// the 224 registers a thread this kernel uses
constexpr int kCW = 7;                    // consumer warps
constexpr int kTile = 16 * kCW;           // tokens per stage (112)
constexpr int kThreads = (kCW + 1) * 32;  // + one producer warp
constexpr int kCT = kCW * 32;
constexpr int kGM = 8;                    // head rows
constexpr int kStages = 2;
constexpr int kPartHead = 7;              // partial: m, W, md, X, M1, M2, A2, then dov[D]

template <int D, int R, bool V2>
struct KLayout {
  static constexpr int NG = D / 32;
  static constexpr int RR = R > 0 ? R : 1;
  static constexpr int kBoxes = D / 64;          // 64-channel swizzled boxes per row
  static constexpr int kBox = kTile * 128;       // one box: kTile rows of 128 bytes
  static constexpr int kKf = 0;                  // exact keys (swizzled boxes)
  static constexpr int kVf = kKf + kBoxes * kBox;   // exact values (swizzled boxes)
  static constexpr int kVc = kVf + kBoxes * kBox;   // cached values: dense boxes or codes
  static constexpr int kVcBytes = V2 ? kTile * (D / 4) : kBoxes * kBox;
  static constexpr int kVs = kVc + kVcBytes;     // 2-bit value scale / minimum
  static constexpr int kVm = kVs + (V2 ? kTile * NG * 4 : 0);
  static constexpr int kKc = kVm + (V2 ? kTile * NG * 4 : 0);
  static constexpr int kKs = kKc + kTile * (D / 4);
  static constexpr int kKm = kKs + kTile * NG * 4;
  static constexpr int kZc = kKm + kTile * NG * 4;
  static constexpr int kZs = kZc + kTile * (R / 2);
  static constexpr int kEnd = kZs + (R > 0 ? kTile * 4 : 0);
  static constexpr int kStage = (kEnd + 1023) / 1024 * 1024;
  // bytes of the 1-D copies per token row (the boxes are counted whole)
  static constexpr int kRowBytes =
      (V2 ? D / 4 + 8 * NG : 0) + D / 4 + 8 * NG + (R > 0 ? R / 2 + 4 : 0);
  static constexpr int kBoxBytes = (V2 ? 2 : 3) * kBoxes * kBox;
  // query state: q [kGM][D] fp32, group sums [kGM][NG], maxima [kGM][NG],
  // sigma U^T q [kGM][RR].  The raw query [kGM][D] and U_h [D][RR] arrive in the
  // memory of stage 1, which takes its first tile once the consumers are done
  // with them.
  static constexpr int kQFloats = kGM * D + 2 * kGM * NG + kGM * RR;
  static constexpr int kQBytes = (kQFloats * 4 + 15) / 16 * 16;
  static constexpr int kRawBytes = kGM * D * 4;
  // the final merge of the warps: [kCW][kGM] x 7 doubles, dov [kCW][kGM][D]
  // floats -- in the stage memory once the stream is done
  static constexpr int kSmem = 1024 + kStages * kStage + kQBytes + 16 * (2 * kStages + 2) + 64;
  static_assert(kCW * kGM * 7 * 8 + kCW * kGM * D * 4 <= kStages * kStage, "merge space");
  static_assert(kRawBytes + D * RR * 4 <= kStage, "query staging space");
  static_assert(kSmem <= 232448, "shared memory");
};

__device__ __forceinline__ uint32_t bfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// bf16 value (as float) of the low / high half of a packed pair
__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
// bf16 high and low parts of a pair of floats (a in the low half)
__device__ __forceinline__ void bf_split(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - bf_lo(hi), b - bf_hi(hi));
  lo = *reinterpret_cast<const uint32_t*>(&l);
}
// Two k-slot pairs of 2-bit codes as exact bf16 B-operand registers.  x holds the
// codes of channels (2t, 2t+1) of a 16-channel k-step at bits 0-3 and those of
// (2t+8, 2t+9) at bits 16-19; 0x4300 | c is the bf16 value 128 + c, and
// (128 + c0, 128 + 4 c1) * (1, 1/4) - (128, 32) = (c0, c1) exactly.
__device__ __forceinline__ void unpack_codes_bf16(uint32_t x, uint32_t& b0, uint32_t& b1) {
  const uint32_t up = x << 16;
  const uint32_t r0 = (x & 0x3u) | (up & 0xC0000u) | 0x43004300u;
  const uint32_t dn = x >> 16;
  const uint32_t r1 = (dn & 0x3u) | (x & 0xC0000u) | 0x43004300u;
  // multiplier (1, 1/4) = (0x3F80, 0x3E80), offset (-128, -32) = (0xC300, 0xC200)
  b0 = bfma2(r0, 0x3E803F80u, 0xC200C300u);
  b1 = bfma2(r1, 0x3E803F80u, 0xC200C300u);
}
__device__ __forceinline__ int seq_len(const AttnKlParams& p, int b) {
  return p.seq_lens ? max(0, min(p.seq_lens[b], p.T)) : p.T;
}

// one CTA of 256 threads per SM: up to 224 registers a thread
template <int D, int R, bool V2>
__global__ void __maxnreg__(224)
attn_kl_hm_kernel(const AttnKlParams p, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap cmap) {
  using L = KLayout<D, R, V2>;
  constexpr int NG = L::NG;
  constexpr int KS = D / 16;
  constexpr int MT = D / 16;  // 16-dim row blocks of the readout-error product

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align(smem_raw, 1024);
  uint8_t* stages = smem;
  float* q_s = reinterpret_cast<float*>(stages + size_t(kStages) * L::kStage);  // [kGM][D]
  float* qsum_s = q_s + kGM * D;     // [kGM][NG]
  float* qmax_s = qsum_s + kGM * NG; // [kGM][NG]
  float* qt_s = qmax_s + kGM * NG;   // [kGM][RR]
  float* qraw_s = reinterpret_cast<float*>(stages + L::kStage);            // in stage 1
  float* u_s = reinterpret_cast<float*>(stages + L::kStage + L::kRawBytes);  // in stage 1
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(q_s) + L::kQBytes);
  // bars[s] full, bars[kStages + s] empty, bars[2 kStages] query and U_h in,
  // bars[2 kStages + 1] the consumers are done with them (stage 1 is free)
  int* stile_s = reinterpret_cast<int*>(bars + 2 * kStages + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int G = p.G, Hkv = p.c.Hkv;
  const int Tb = seq_len(p, b);
  const int t_begin = split * p.chunk;
  const int t_end = min(Tb, t_begin + p.chunk);
  const int ntiles = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
  const size_t bk = static_cast<size_t>(b) * Hkv + kv;
  const int h0 = kv * G;
  const uint32_t qbar = smem_addr(&bars[2 * kStages]);
  const uint32_t qdone = smem_addr(&bars[2 * kStages + 1]);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&bars[s]), 1);
      mbar_init(smem_addr(&bars[kStages + s]), kCW);
    }
    mbar_init(qbar, 1);
    mbar_init(qdone, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // ------------------------------------------------------------ producer warp
  if (warp == kCW) {
    if (lane == 0) {
      const uint32_t qbytes = static_cast<uint32_t>(G * D * (p.q_bf16 ? 2 : 4));
      mbar_expect_tx(qbar, qbytes + (R > 0 ? D * R * 4 : 0));
      bulk_g2s(smem_addr(qraw_s),
               static_cast<const uint8_t*>(p.q) +
                   (static_cast<size_t>(b) * p.Hq + h0) * D * (p.q_bf16 ? 2 : 4),
               qbytes, qbar);
      if constexpr (R > 0)
        bulk_g2s(smem_addr(u_s), p.U + static_cast<size_t>(kv) * D * R, D * R * 4, qbar);
      bool ok = true;
      int issued = 0;
      for (int i = 0; ok; ++i) {
        const int s = i % kStages, use = i / kStages;
        if (use > 0 && !mbar_wait(smem_addr(&bars[kStages + s]), (use - 1) & 1)) {
          ok = false;
          break;
        }
        // stage 1 holds the raw query and U_h until the consumers are done
        if (i == 1 && !mbar_wait(qdone, 0)) {
          ok = false;
          break;
        }
        const uint32_t full = smem_addr(&bars[s]);
        if (i >= ntiles) {
          stile_s[s] = -1;
          mbar_arrive(full);
          ++issued;
          break;
        }
        const int t0 = t_begin + i * kTile;
        stile_s[s] = t0;
        const int n16 = (min(kTile, t_end - t0) + 15) & ~15;
        mbar_expect_tx(full, L::kBoxBytes + n16 * L::kRowBytes);
        uint8_t* st = stages + size_t(s) * L::kStage;
        const CacheSlab sl = cache_slab_read(p.c, b, kv, t0, p.err);
        const size_t row0 = static_cast<size_t>(sl.slab) * slab_rows(p.c) + sl.off;
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx) {
          tma_3d(smem_addr(st + L::kKf + bx * L::kBox), &kmap, bx * 64, t0, static_cast<int>(bk), full);
          tma_3d(smem_addr(st + L::kVf + bx * L::kBox), &vmap, bx * 64, t0, static_cast<int>(bk), full);
          if constexpr (!V2)
            tma_3d(smem_addr(st + L::kVc + bx * L::kBox), &cmap, bx * 64, sl.off,
                   static_cast<int>(sl.slab), full);
        }
        if constexpr (V2) {
          bulk_g2s(smem_addr(st + L::kVc), p.c.v_codes + row0 * (D / 4), n16 * (D / 4), full);
          bulk_g2s(smem_addr(st + L::kVs), p.c.v_scale + row0 * NG, n16 * NG * 4, full);
          bulk_g2s(smem_addr(st + L::kVm), p.c.v_min + row0 * NG, n16 * NG * 4, full);
        }
        bulk_g2s(smem_addr(st + L::kKc), p.c.k_codes + row0 * (D / 4), n16 * (D / 4), full);
        bulk_g2s(smem_addr(st + L::kKs), p.c.k_scale + row0 * NG, n16 * NG * 4, full);
        bulk_g2s(smem_addr(st + L::kKm), p.c.k_min + row0 * NG, n16 * NG * 4, full);
        if constexpr (R > 0) {
          bulk_g2s(smem_addr(st + L::kZc), p.c.z_codes + row0 * (R / 2), n16 * (R / 2), full);
          bulk_g2s(smem_addr(st + L::kZs), p.c.z_scale + row0, n16 * 4, full);
        }
        ++issued;
      }
      if (!ok && p.err) atomicOr(p.err, kDevErrWaitTimeout);
      for (int s = 0; s < kStages && s < issued; ++s)
        mbar_wait(smem_addr(&bars[s]), ((issued - 1 - s) / kStages) & 1);
    }
    return;
  }

  // ------------------------------------------------------------ consumer warps
  if (!mbar_wait(qbar, 0) && tid == 0 && p.err) atomicOr(p.err, kDevErrWaitTimeout);
  // the query as the MMAs see it: its bf16 high part plus bf16 low part, so that
  // the group sums Q_g use the same rounded values as the code and key products
  for (int k = tid; k < kGM * D; k += kCT) {
    const float v = k < G * D ? load_elem(qraw_s, k, p.q_bf16) : 0.0f;
    const float hi = __bfloat162float(__float2bfloat16_rn(v));
    q_s[k] = hi + __bfloat162float(__float2bfloat16_rn(v - hi));
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  for (int k = tid; k < kGM * NG; k += kCT) {
    const int h = k / NG, g = k - h * NG;
    float acc = 0.0f, amax = 0.0f;
    for (int c = 0; c < 32; ++c) {
      const float v = q_s[h * D + g * 32 + c];
      acc += v;
      amax = fmaxf(amax, fabsf(v));
    }
    qsum_s[k] = acc;
    qmax_s[k] = amax;
  }
  if constexpr (R > 0) {
    for (int k = tid; k < kGM * R; k += kCT) {
      const int h = k / R, ii = k - h * R;
      float acc = 0.0f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = fmaf(u_s[c * R + ii], q_s[h * D + c], acc);
      qt_s[k] = p.corr_sign * acc;
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  if (tid == 0) mbar_arrive(qdone);  // the raw query and U_h are no longer read

  const int gq = lane >> 2, t = lane & 3;
  const int jw = 16 * warp;
  // A fragments: the query of head gq as bf16 high (row gq) and low (row gq + 8)
  // parts, natural channel order: k-slots (2t, 2t+1) <-> channels 16 ks + 2t + {0, 1},
  // (2t+8, 2t+9) <-> 16 ks + 2t + 8 + {0, 1}
  uint32_t aq[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const float* qh = q_s + gq * D + 16 * ks + 2 * t;
    bf_split(qh[0], qh[1], aq[ks][0], aq[ks][1]);
    bf_split(qh[8], qh[9], aq[ks][2], aq[ks][3]);
  }
  // side-code A fragment (fp16 high/low, prescaled by the head's power of two)
  float fq, finv;
  head_prescale<NG>(qmax_s, gq, fq, finv);
  uint32_t az[4] = {0u, 0u, 0u, 0u};
  if constexpr (R == 16) {
    const float* z = qt_s + gq * R + 4 * t;
    az[0] = half_part_pair(z[0] * fq, z[1] * fq, false);
    az[1] = half_part_pair(z[0] * fq, z[1] * fq, true);
    az[2] = half_part_pair(z[2] * fq, z[3] * fq, false);
    az[3] = half_part_pair(z[2] * fq, z[3] * fq, true);
  } else if constexpr (R == 8) {
    const float* z = qt_s + gq * R + 2 * t;
    az[0] = half_part_pair(z[0] * fq, z[1] * fq, false);
    az[1] = half_part_pair(z[0] * fq, z[1] * fq, true);
  }
  float qsum[NG];
#pragma unroll
  for (int gg = 0; gg < NG; ++gg) qsum[gg] = qsum_s[gq * NG + gg];
  const uint32_t sel = (2 * t) | ((2 * t + 1) << 4) | ((2 * t) << 8) | ((2 * t + 1) << 12);
  const uint32_t sel8 = t | (4 << 4) | (t << 8) | (4 << 12);
  const float sm = p.sm_scale;
  constexpr float L2E = kLog2e;

  // running state of head gq (per lane: its tokens; merged at the end)
  float m = -INFINITY, md = -INFINITY;   // running maxima of s and delta
  double W = 0.0, X = 0.0, M1 = 0.0, M2 = 0.0, A2 = 0.0;
  float dov[MT][4];  // rows: this lane's dims, columns: heads 2t, 2t+1
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) dov[mt][0] = dov[mt][1] = dov[mt][2] = dov[mt][3] = 0.f;

  bool ok = true;
  for (int i = 0;; ++i) {
    const int s = i % kStages;
    if (!mbar_wait(smem_addr(&bars[s]), (i / kStages) & 1)) {
      ok = false;
      break;
    }
    const int t0 = stile_s[s];
    if (t0 < 0) break;
    const uint8_t* st = stages + size_t(s) * L::kStage;
    const int nvalid = min(kTile, t_end - t0);

    // ---- value errors: this lane's dims (16-byte chunks gq and gq + 8) of the
    // tokens jw + {2t, 2t+1, 2t+8, 2t+9}; |dv|^2 per token summed over the lanes
    // of the same t
    uint32_t ahi[MT][4], alo[MT][4];
    float n2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int tok = jw + 2 * t + (k & 1) + 8 * (k >> 1);
      const bool valid = tok < nvalid;
      float part = 0.f;
#pragma unroll
      for (int cb = 0; cb < L::kBoxes; ++cb) {
        // chunk gq of box cb of row tok, 128-byte swizzle: physical chunk gq ^ (tok & 7)
        const int off = cb * L::kBox + tok * 128 + ((gq ^ (tok & 7)) << 4);
        const uint4 vf = *reinterpret_cast<const uint4*>(st + L::kVf + off);
        float dv[8];
        if constexpr (V2) {
          const int dim0 = 64 * cb + 8 * gq;  // 8 dims, one group
          const int g = dim0 / 32;
          const uint16_t cw = *reinterpret_cast<const uint16_t*>(st + L::kVc + tok * (D / 4) + dim0 / 4);
          const float vsc = reinterpret_cast<const float*>(st + L::kVs)[tok * NG + g];
          const float vmn = reinterpret_cast<const float*>(st + L::kVm)[tok * NG + g];
          const uint32_t fw[4] = {vf.x, vf.y, vf.z, vf.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float code = static_cast<float>((cw >> (2 * e)) & 3);
            const float vh = __fadd_rn(vmn, __fmul_rn(code, vsc));
            const float vx = (e & 1) ? bf_hi(fw[e >> 1]) : bf_lo(fw[e >> 1]);
            dv[e] = valid ? vh - vx : 0.f;
          }
        } else {
          const uint4 vc = *reinterpret_cast<const uint4*>(st + L::kVc + off);
          const uint32_t fw[4] = {vf.x, vf.y, vf.z, vf.w}, cw4[4] = {vc.x, vc.y, vc.z, vc.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            dv[2 * e] = valid ? bf_lo(cw4[e]) - bf_lo(fw[e]) : 0.f;
            dv[2 * e + 1] = valid ? bf_hi(cw4[e]) - bf_hi(fw[e]) : 0.f;
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) part = fmaf(dv[e], dv[e], part);
        // A operand of m-tile mt = 4 cb + e/2: row gq <-> dim 64 cb + 8 gq + e (e
        // even), row gq + 8 <-> the next dim (e odd); k-slots (2t, 2t+1) <->
        // tokens k = 0, 1, (2t+8, 2t+9) <-> k = 2, 3; register j = (e & 1) +
        // 2 (k >> 1).  A pair holds tokens (k even, k odd): the even token's
        // errors wait in ahi until the odd token's arrive.
        if ((k & 1) == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) ahi[4 * cb + e / 2][(e & 1) + 2 * (k >> 1)] = __float_as_uint(dv[e]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int mt = 4 * cb + e / 2;
            const int j = (e & 1) + 2 * (k >> 1);  // a0 (row gq, tok 2t..), a1 (row gq + 8), a2, a3
            uint32_t hi, lo;
            bf_split(__uint_as_float(ahi[mt][j]), dv[e], hi, lo);
            ahi[mt][j] = hi;
            alo[mt][j] = lo;
          }
        }
      }
      n2[k] = part;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {  // sum over the 8 lanes of this t (their dims)
      n2[k] += __shfl_xor_sync(kFull, n2[k], 4);
      n2[k] += __shfl_xor_sync(kFull, n2[k], 8);
      n2[k] += __shfl_xor_sync(kFull, n2[k], 16);
    }

    // ---- logits s and perturbations delta of head gq, tokens jw + 8 nb + {2t, 2t+1}
    float sv[4], dl[4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
      float accS[NG][4], accK[NG][4], accZ[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        accS[gg][0] = accS[gg][1] = accS[gg][2] = accS[gg][3] = 0.f;
        accK[gg][0] = accK[gg][1] = accK[gg][2] = accK[gg][3] = 0.f;
      }
      // exact keys: ldmatrix of token rows jw + 8 nb + (lane & 7), chunk 4 kp + (lane >> 3)
      const int lrow = jw + 8 * nb + (lane & 7);
#pragma unroll
      for (int kp = 0; kp < KS / 2; ++kp) {
        const int chunk = 4 * kp + (lane >> 3);
        const uint32_t addr = smem_addr(st + L::kKf + (chunk >> 3) * L::kBox + lrow * 128 +
                                        (((chunk & 7) ^ (lrow & 7)) << 4));
        uint32_t kb[4];
        ldsm_x4(addr, kb);
        const uint32_t b0[2] = {kb[0], kb[1]}, b1[2] = {kb[2], kb[3]};
        mma_bf16(accS[kp], aq[2 * kp], b0);
        mma_bf16(accS[kp], aq[2 * kp + 1], b1);
      }
      // the base code of token jw + 8 nb + gq, same channel order
      const int tb = jw + 8 * nb + gq;
      uint32_t cw[D / 16];
#pragma unroll
      for (int v4 = 0; v4 < D / 64; ++v4) {
        const uint4 a = *reinterpret_cast<const uint4*>(st + L::kKc + tb * (D / 4) + 16 * v4);
        cw[4 * v4 + 0] = a.x; cw[4 * v4 + 1] = a.y; cw[4 * v4 + 2] = a.z; cw[4 * v4 + 3] = a.w;
      }
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t bb[2];
        unpack_codes_bf16(cw[ks] >> (4 * t), bb[0], bb[1]);
        mma_bf16(accK[ks >> 1], aq[ks], bb);
      }
      if constexpr (R > 0) {
        uint32_t bzv[2];
        if constexpr (R == 16) {
          const uint2 z = *reinterpret_cast<const uint2*>(st + L::kZc + tb * 8);
          unpack_side(__byte_perm(z.x, z.y, sel) ^ 0x88888888u, bzv[0], bzv[1]);
        } else {
          const uint32_t z = *reinterpret_cast<const uint32_t*>(st + L::kZc + tb * 4);
          uint32_t dummy;
          unpack_side(__byte_perm(z, 0u, sel8) ^ 0x00880088u, bzv[0], dummy);
          bzv[1] = 0u;
        }
        mma_f16(accZ, az, bzv);
      }
      const int ta = jw + 8 * nb + 2 * t;  // this lane's output tokens ta, ta + 1
      const float* ksp = reinterpret_cast<const float*>(st + L::kKs);
      const float* kmp = reinterpret_cast<const float*>(st + L::kKm);
      float sa = 0.f, sb = 0.f, da = 0.f, db = 0.f;
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const float s_a = accS[gg][0] + accS[gg][2], s_b = accS[gg][1] + accS[gg][3];
        const float k_a = accK[gg][0] + accK[gg][2], k_b = accK[gg][1] + accK[gg][3];
        da += fmaf(kmp[ta * NG + gg], qsum[gg], fmaf(ksp[ta * NG + gg], k_a, -s_a));
        db += fmaf(kmp[(ta + 1) * NG + gg], qsum[gg], fmaf(ksp[(ta + 1) * NG + gg], k_b, -s_b));
        sa += s_a;
        sb += s_b;
      }
      if constexpr (R > 0) {
        const float2 zs = reinterpret_cast<const float2*>(st + L::kZs)[ta / 2];
        da = fmaf(zs.x * finv, accZ[0] + accZ[2], da);
        db = fmaf(zs.y * finv, accZ[1] + accZ[3], db);
      }
      const bool va = ta < nvalid, vb = ta + 1 < nvalid;
      sv[2 * nb] = va ? sa * sm : -INFINITY;
      sv[2 * nb + 1] = vb ? sb * sm : -INFINITY;
      dl[2 * nb] = va ? da * sm : -INFINITY;
      dl[2 * nb + 1] = vb ? db * sm : -INFINITY;
    }

    // ---- running maxima of s and delta for head gq (its four lanes)
    float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
    float mxd = fmaxf(fmaxf(dl[0], dl[1]), fmaxf(dl[2], dl[3]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    mxd = fmaxf(mxd, __shfl_xor_sync(kFull, mxd, 1));
    mxd = fmaxf(mxd, __shfl_xor_sync(kFull, mxd, 2));
    const float mnew = fmaxf(m, mx), mdnew = fmaxf(md, mxd);
    const bool grow = mnew > m;
    if (__any_sync(kFull, grow)) {
      const float alpha = grow ? exp2f((m - mnew) * L2E) : 1.0f;
      if (grow) {
        const double a = alpha;
        W *= a;
        X *= a;
        M1 *= a;
        M2 *= a;
        A2 *= a * a;
        m = mnew;
      }
      const float a0 = __shfl_sync(kFull, alpha, 8 * t);      // head 2t
      const float a1 = __shfl_sync(kFull, alpha, 8 * t + 4);  // head 2t + 1
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        dov[mt][0] *= a0; dov[mt][1] *= a1; dov[mt][2] *= a0; dov[mt][3] *= a1;
      }
    }
    if (mdnew > md) {
      X *= static_cast<double>(exp2f((md - mdnew) * L2E));
      md = mdnew;
    }
    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      w[k] = sv[k] == -INFINITY ? 0.f : exp2f((sv[k] - m) * L2E);
      if (w[k] > 0.f) {
        const float x = w[k] * exp2f((dl[k] - md) * L2E);
        const float wd = w[k] * dl[k];
        W += static_cast<double>(w[k]);
        X += static_cast<double>(x);
        M1 += static_cast<double>(wd);
        M2 += static_cast<double>(wd) * static_cast<double>(dl[k]);
        // n2 index: sv[k] is token jw + 8 (k >> 1) + 2t + (k & 1); n2[j] is token
        // jw + 2t + (j & 1) + 8 (j >> 1): the same order
        A2 += static_cast<double>(w[k]) * static_cast<double>(w[k]) * static_cast<double>(n2[k]);
      }
    }

    // ---- readout error: dov += dv^T w (B = w of head gq, tokens 2t, 2t+1 | 2t+8, 2t+9)
    uint32_t bwh[2], bwl[2];
    bf_split(w[0], w[1], bwh[0], bwl[0]);
    bf_split(w[2], w[3], bwh[1], bwl[1]);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      mma_bf16(dov[mt], ahi[mt], bwh);
      mma_bf16(dov[mt], ahi[mt], bwl);
      mma_bf16(dov[mt], alo[mt], bwh);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&bars[kStages + s]));
  }
  if (!ok && lane == 0 && p.err) atomicOr(p.err, kDevErrWaitTimeout);

  // ---- merge: lanes of a head, then the warps, into this split's partial
  W += __shfl_xor_sync(kFull, W, 1);  W += __shfl_xor_sync(kFull, W, 2);
  X += __shfl_xor_sync(kFull, X, 1);  X += __shfl_xor_sync(kFull, X, 2);
  M1 += __shfl_xor_sync(kFull, M1, 1); M1 += __shfl_xor_sync(kFull, M1, 2);
  M2 += __shfl_xor_sync(kFull, M2, 1); M2 += __shfl_xor_sync(kFull, M2, 2);
  A2 += __shfl_xor_sync(kFull, A2, 1); A2 += __shfl_xor_sync(kFull, A2, 2);
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");  // every warp is done with the stages
  double* ms = reinterpret_cast<double*>(stages);        // [kCW][kGM][7]
  float* mo = reinterpret_cast<float*>(ms + kCW * kGM * 7);  // [kCW][kGM][D]
  if (t == 0) {
    double* e = ms + (warp * kGM + gq) * 7;
    e[0] = m; e[1] = W; e[2] = md; e[3] = X; e[4] = M1; e[5] = M2; e[6] = A2;
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {  // rows: dims 64 cb + 8 gq + 2 e2 (+1), cb = mt / 4
    const int d0 = 64 * (mt >> 2) + 8 * gq + 2 * (mt & 3);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * t + e;
      mo[(warp * kGM + h) * D + d0] = dov[mt][e];
      mo[(warp * kGM + h) * D + d0 + 1] = dov[mt][2 + e];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  const int PS = kPartHead + D;
  for (int idx = tid; idx < G * D; idx += kCT) {
    const int h = idx / D, c = idx - h * D;
    double M = -INFINITY;
#pragma unroll
    for (int wv = 0; wv < kCW; ++wv) M = fmax(M, ms[(wv * kGM + h) * 7]);
    double acc = 0.0;
    if (M > -INFINITY) {
#pragma unroll
      for (int wv = 0; wv < kCW; ++wv) {
        const double mw = ms[(wv * kGM + h) * 7];
        if (mw > -INFINITY) acc += exp2((mw - M) * static_cast<double>(L2E)) * mo[(wv * kGM + h) * D + c];
      }
    }
    const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
    p.part[(bh * p.splits + split) * PS + kPartHead + c] = acc;
  }
  for (int h = tid; h < G; h += kCT) {
    double M = -INFINITY, MD = -INFINITY;
    for (int wv = 0; wv < kCW; ++wv) {
      M = fmax(M, ms[(wv * kGM + h) * 7]);
      MD = fmax(MD, ms[(wv * kGM + h) * 7 + 2]);
    }
    double sW = 0, sX = 0, s1 = 0, s2 = 0, sA = 0;
    if (M > -INFINITY) {
      for (int wv = 0; wv < kCW; ++wv) {
        const double* e = ms + (wv * kGM + h) * 7;
        if (e[0] == -INFINITY) continue;
        const double f = exp2((e[0] - M) * static_cast<double>(L2E));
        sW += f * e[1];
        sX += f * exp2((e[2] - MD) * static_cast<double>(L2E)) * e[3];
        s1 += f * e[4];
        s2 += f * e[5];
        sA += f * f * e[6];
      }
    }
    const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
    double* pt = p.part + (bh * p.splits + split) * PS;
    pt[0] = M;
    pt[1] = sW;
    pt[2] = MD;
    pt[3] = sX;
    pt[4] = s1;
    pt[5] = s2;
    pt[6] = sA;
  }
}

// ---------------------------------------------------------------- host side
// bf16 rows of D channels in slabs: [slab][row][channel], 64-channel x kTile-row
// boxes with the 128-byte swizzle
template <int D>
bool encode_rows(CUtensorMap* map, const void* base, uint64_t rows, uint64_t slabs) {
  return encode_bf16_rows(map, base, D, rows, slabs, kTile);
}

template <int D, int R, bool V2>
cudaError_t launch_variant(const AttnKlParams& p, cudaStream_t s) {
  using L = KLayout<D, R, V2>;
  auto k = attn_kl_hm_kernel<D, R, V2>;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [&] {
    attr = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  });
  if (attr != cudaSuccess) return attr;
  CUtensorMap kmap, vmap, cmap;
  memset(&cmap, 0, sizeof(cmap));
  const uint64_t seqs = static_cast<uint64_t>(p.c.B) * p.c.Hkv;
  if (!encode_rows<D>(&kmap, p.k_full, static_cast<uint64_t>(p.T), seqs) ||
      !encode_rows<D>(&vmap, p.v_full, static_cast<uint64_t>(p.T), seqs))
    return cudaErrorInvalidValue;
  if (!V2) {
    const bool paged = p.c.page_size > 0;
    const uint64_t rows = static_cast<uint64_t>(paged ? p.c.page_size : p.c.T_cap);
    const uint64_t slabs = static_cast<uint64_t>(paged ? p.c.num_pages : p.c.B) * p.c.Hkv;
    if (!encode_rows<D>(&cmap, p.c.v, rows, slabs)) return cudaErrorInvalidValue;
  }
  dim3 grid(p.splits, p.c.Hkv, p.c.B);
  k<<<grid, kThreads, L::kSmem, s>>>(p, kmap, vmap, cmap);
  return cudaGetLastError();
}

}  // namespace

bool kl_hm_supported(const headq_cache& c, int G, bool kv_bf16) {
  if (!kv_bf16 || c.kmode != HEADQ_K_TOKEN) return false;
  if (c.d != 64 && c.d != 128) return false;
  if (G < 1 || G > kGM) return false;
  if (c.r != 0 && c.r != 8 && c.r != 16) return false;
  if (c.page_size > 0 && c.page_size % kTile != 0) return false;  // whole tiles per page
  if (c.vmode == HEADQ_V_2BIT) return true;
  return c.v_dtype == HEADQ_BF16 && tensor_maps_available();
}

// Splits for one CTA per SM: chunks a multiple of the tile (112 tokens), the
// count chosen so the grid fills whole waves best (ties: fewer splits).
SplitPlan kl_hm_plan(int units, int T) {
  // One CTA per SM.  The split count minimises waves x (tiles per CTA +
  // kTileOverhead), the 2 standing for a CTA's fixed cost (query and U_h
  // preparation, the fp64 merge and partial store); ties go to fewer splits.
  constexpr long long kTileOverhead = 2;
  SplitPlan best{1, (T + kTile - 1) / kTile * kTile};
  if (units <= 0 || T <= 0) return best;
  const long long slots = sm_count();
  long long best_cost = -1;
  const int max_s = (T + kTile - 1) / kTile;
  for (int s = 1; s <= max_s && s <= 256; ++s) {
    int chunk = (T + s - 1) / s;
    chunk = (chunk + kTile - 1) / kTile * kTile;
    const int sp = (T + chunk - 1) / chunk;
    if (sp != s) continue;
    const long long waves = (static_cast<long long>(units) * sp + slots - 1) / slots;
    const long long cost = waves * (chunk / kTile + kTileOverhead);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = SplitPlan{sp, chunk};
    }
  }
  return best;
}

cudaError_t launch_attn_kl_hm(const AttnKlParams& p, cudaStream_t s) {
  const bool v2 = p.c.vmode == HEADQ_V_2BIT;
#define HEADQ_KL_CASE(DD, RR, VV) \
  if (p.c.d == DD && p.c.r == RR && v2 == VV) return launch_variant<DD, RR, VV>(p, s);
  HEADQ_KL_CASE(128, 16, false) HEADQ_KL_CASE(128, 8, false) HEADQ_KL_CASE(128, 0, false)
  HEADQ_KL_CASE(128, 16, true) HEADQ_KL_CASE(128, 8, true) HEADQ_KL_CASE(128, 0, true)
  HEADQ_KL_CASE(64, 16, false) HEADQ_KL_CASE(64, 8, false) HEADQ_KL_CASE(64, 0, false)
  HEADQ_KL_CASE(64, 16, true) HEADQ_KL_CASE(64, 8, true) HEADQ_KL_CASE(64, 0, true)
#undef HEADQ_KL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace headq
