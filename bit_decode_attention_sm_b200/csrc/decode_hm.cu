// HeadQ decode attention for 5 to 8 query heads per KV head (GQA), tensor-core
// kernel for sm_100a ("HeadQ: Model-Visible Distortion and Score-Space Correction
// for KV-Cache Quantization", gist.science summary, section 3, step 3: the
// runtime query turns the side code into an additive logit correction; the
// readout is the attention-weighted sum of values, the values dequantised as
// min + code * scale per 32-channel group when they are 2-bit coded).
//
// Same mathematics and cache layout as decode_mma.cu; the MMA operand roles
// are chosen for G = 5..8 heads so that one m16n8k16 serves all of them:
//
//  * q . code: A = the query, head g's fp16 high part in row g and its low part
//    in row g + 8 (8 head slots fill M = 16); B = the 2-bit codes with the 8
//    tokens of an n-tile on N.  Each thread's codes come straight out of the
//    packed 32-bit word: one AND keeps two 2-bit fields 16 bits apart, and the
//    16-bit halves, read as fp16 with a zero exponent, are the exact values
//    code * 2^(p - 24) (p = the field's bit position 0..6 within its half, after
//    a shift of 0 or 8).  The query operand carries the compensating 2^(6 - p),
//    so every product is q * code * 2^-18 and one fp32 factor restores the
//    logit.  Each 32-channel group keeps its own accumulator; the group's scale
//    and minimum apply as the dequantisation defines them.  The side code is one
//    more MMA on offset nibbles (w + 8, exact subnormals the same way) against
//    sigma U_h^T q; the offset's contribution is subtracted per head.
//  * p . V: A = the values transposed (channels on M, tokens on K), B = the
//    probabilities with the 8 head slots on N.  The logit accumulator of an
//    n-tile pair already holds, per thread, the B fragment of its k-step, so p
//    never leaves the registers.  Dense bf16 values come from the swizzled tile
//    by ldmatrix.trans, p as bf16 high + low parts (two MMAs).  2-bit values:
//    one byte-permute pairs the same code byte of two tokens, four ANDs give
//    the A registers of two 16-channel row blocks (exact subnormals again,
//    with a power of two per row undone at the end); B is p * scale_{j,g} per
//    group g, in fp16 relative to a power of two 2^E per (warp, head, group)
//    that is raised once an entry reaches 2^12 of it; the minimum enters as
//    sum_j p_j min_{j,g} in fp32.
//  * five consumer warps take the four 16-token slices of the 64-token stages in
//    turn, each with its own online softmax (log2 domain, lazily rescaled max);
//    a stage is released after its four slices.  Five, because two CTAs of six
//    warps at this register count still fit an SM.  The warps merge through
//    shared memory at the end and the splits by the last CTA.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "decode_pipe.cuh"
#include "headq_internal.cuh"

namespace headq {
namespace {
using namespace dc;

constexpr int kCW = 5;                    // consumer warps
constexpr int kSlices = 4;                // 16-token slices per 64-token stage
constexpr int kTile = kPipeTile;          // tokens per stage
constexpr int kThreads = (kCW + 1) * 32;  // + one producer warp
constexpr int kGM = 8;                    // head slots
constexpr int kCT = kCW * 32;             // consumer threads
constexpr float kRescale = 8.0f;          // log2 units the stale max may lag (p <= 2^8)
constexpr int kRaiseLog2 = 12;            // 2-bit values: entries stay below 2^(E + 12)
constexpr float kMaxInit = -1e30f;        // running max before the first logit (finite)

// pipeline depth (the stages also hold the merging CTA's [G][splits] weights)
// and CTAs per SM: two, with registers for the operand fragments, the output
// and the per-(head, group) exponents without spilling
template <bool V2>
constexpr int kStagesHM = V2 ? 8 : 4;
constexpr int kMinCtasHM = 2;

// stages | q [8][D] | group sums and maxima [8][NG] each | sigma U^T q [8][R] |
// U_h [D][R] | the query as bulk-copied [8][D] | appended token's residual [D]
// | barriers (2 kStages + 1) | stage tile starts
template <int D, int R, bool V2>
constexpr size_t hm_smem_bytes() {
  using L = StageLayout<D, R, V2>;
  constexpr int RR = R > 0 ? R : 1;
  return 1024 + size_t(kStagesHM<V2>) * L::kStage +
         sizeof(float) * (kGM * D + 2 * kGM * L::NG + kGM * RR + D * RR + kGM * D + D) + 16 +
         8 * (2 * kStagesHM<V2> + 1) + 4 * kStagesHM<V2> + 16;
}

// 2^x, flushing results below 2^-126 to zero (2^-inf = 0)
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^e as a float, e in [-126, 127]
__device__ __forceinline__ float pow2f(int e) {
  return __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}
__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t f16x2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// the N (= 2 or 4) per-group floats of one token's row of a plane, as one
// vector load (rows are 8- or 16-byte aligned in the stage)
template <int N>
__device__ __forceinline__ void load_groups(const uint8_t* row, float (&v)[N]) {
  if constexpr (N == 4) {
    const float4 a = *reinterpret_cast<const float4*>(row);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else {
    static_assert(N == 2, "2 or 4 groups");
    const float2 a = *reinterpret_cast<const float2*>(row);
    v[0] = a.x; v[1] = a.y;
  }
}

template <int D, int R, bool V2>
__global__ void __launch_bounds__(kThreads, kMinCtasHM)
decode_hm_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap vmap) {
  using L = StageLayout<D, R, V2>;
  constexpr int NG = L::NG;
  constexpr int KS = D / 16;   // k-steps of 16 channels
  constexpr int MT = D / 16;   // 16-channel row blocks of the output
  constexpr int RR = R > 0 ? R : 1;
  constexpr int kStages = kStagesHM<V2>;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = smem_align(smem_raw, 1024);
  float* q_s = reinterpret_cast<float*>(stages + size_t(kStages) * L::kStage);  // [8][D]
  float* qsum_s = q_s + kGM * D;    // [8][NG]
  float* qmax_s = qsum_s + kGM * NG;  // [8][NG]
  float* qt_s = qmax_s + kGM * NG;    // [8][RR]
  float* u_s = smem_align(qt_s + kGM * RR, 16);  // [D][RR] (bulk-copy destination)
  float* qraw_s = u_s + D * RR;                  // [8][D] (bulk-copy destination)
  float* enew_s = qraw_s + kGM * D;              // [D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_align(enew_s + D, 16));
  // bars[s] = stage full, bars[kStages + s] = stage empty, bars[2 kStages] = the
  // query and U_h are in shared memory
  int* stile_s = reinterpret_cast<int*>(bars + 2 * kStages + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int G = p.G, Hkv = p.c.Hkv;
  int Tb = p.T;
  if (p.seq_lens) Tb = max(0, min(p.seq_lens[b], p.T));
  const int t_begin = split * p.chunk;
  const int tile_end = min(Tb, t_begin + p.chunk);
  const int ntiles = tile_end > t_begin ? (tile_end - t_begin + kTile - 1) / kTile : 0;
  const size_t bk = static_cast<size_t>(b) * Hkv + kv;
  const int h0 = kv * G;
  const int pos = (p.k_new != nullptr && Tb > 0) ? Tb - 1 : -1;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&bars[s]), 1);
      mbar_init(smem_addr(&bars[kStages + s]), kSlices);
    }
    mbar_init(smem_addr(&bars[2 * kStages]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kCW) {
    produce_tiles<D, R, V2, false, kStages, true>(p, &vmap, stages, bars, bars + kStages,
                                                  bars + 2 * kStages, stile_s, qraw_s, u_s,
                                                  enew_s, b, kv, h0, t_begin, tile_end,
                                                  ntiles, pos, lane);
    return;
  }

  // ------------------------------------------------------------ consumer warps
  // query prep: q and U_h (bulk-copied by the producer), group sums and maxima,
  // sigma U_h^T q
  if (!mbar_wait(smem_addr(&bars[2 * kStages]), 0) && tid == 0 && p.err)
    atomicOr(p.err, kDevErrWaitTimeout);
  for (int i = tid; i < kGM * D; i += kCT)
    q_s[i] = i < G * D ? load_elem(qraw_s, i, p.q_bf16) : 0.0f;
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  for (int i = tid; i < kGM * NG; i += kCT) {
    const int h = i / NG, gg = i - h * NG;
    float acc = 0.0f, amax = 0.0f;
    for (int c = 0; c < 32; ++c) {
      const float v = q_s[h * D + gg * 32 + c];
      acc += v;
      amax = fmaxf(amax, fabsf(v));
    }
    qsum_s[i] = acc;
    qmax_s[i] = amax;
  }
  if constexpr (R > 0) {
    for (int i = tid; i < kGM * R; i += kCT) {
      const int h = i / R, ii = i - h * R;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains
#pragma unroll 8
      for (int c = 0; c < D; c += 4)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = fmaf(u_s[(c + k) * R + ii], q_s[h * D + c + k], acc[k]);
      qt_s[i] = p.corr_sign * ((acc[0] + acc[1]) + (acc[2] + acc[3]));
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");

  const int g = lane >> 2, t = lane & 3;

  // Operand fields of this thread: its code bits sit at 4t (and 4t + 16) of each
  // 32-bit key-code word; after the shift sh they sit at p0 = 4 (t & 1), so the
  // masks m0 / m1 keep the fields at p0 and p0 + 2 of both halves, worth
  // code * 2^(p0 - 24) and code * 2^(p0 - 22).  The query carries 2^(6 - p0) and
  // 2^(4 - p0): every product is q * code * 2^-18.
  const int sh = 8 * (t >> 1);
  const uint32_t m0 = 0x00030003u << (4 * (t & 1)), m1 = m0 << 2;
  const uint32_t mz = 0x000F000Fu << (4 * (t & 1));
  float f, finv;  // head g's power-of-two prescale (largest |q| * f in [1, 2))
  head_prescale<NG>(qmax_s, g, f, finv);
  const float fa0 = f * pow2f(6 - 4 * (t & 1)), fa1 = f * pow2f(4 - 4 * (t & 1));
  // A operands of q . code, k-step ks = 2 gg + e (channels 32 gg + 16 e + 0..15):
  // k-slots (2t, 2t+1) <-> channels (2t, 2t+8), (2t+8, 2t+9) <-> (2t+1, 2t+9)
  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const float* qh = q_s + g * D + 16 * ks;
    const float c0 = qh[2 * t] * fa0, c1 = qh[2 * t + 8] * fa0;
    const float c2 = qh[2 * t + 1] * fa1, c3 = qh[2 * t + 9] * fa1;
    qa[ks][0] = half_part_pair(c0, c1, false);
    qa[ks][1] = half_part_pair(c0, c1, true);
    qa[ks][2] = half_part_pair(c2, c3, false);
    qa[ks][3] = half_part_pair(c2, c3, true);
  }
  // side code: k-slots (2t, 2t+1) <-> components (t, t+4), (2t+8, 2t+9) <-> (8+t,
  // 12+t); nibble fields at p0 = 4 (t & 1) worth (w + 8) * 2^(p0 - 24)
  uint32_t qz[4] = {0u, 0u, 0u, 0u};
  float zoff = 0.f;  // sum_i 8 * (high + low part)_i * 2^(p0_i - 24) over head g's slots
  if constexpr (R > 0) {
    const float* z = qt_s + g * R;
    const float fz = f * pow2f(6 - 4 * (t & 1));
    const float c0 = z[t] * fz, c1 = z[t + 4] * fz;
    qz[0] = half_part_pair(c0, c1, false);
    qz[1] = half_part_pair(c0, c1, true);
    float part = 0.f;
    {
      const __half2 hi = *reinterpret_cast<const __half2*>(&qz[0]);
      const __half2 lo = *reinterpret_cast<const __half2*>(&qz[1]);
      part = (__low2float(hi) + __low2float(lo)) + (__high2float(hi) + __high2float(lo));
    }
    if constexpr (R == 16) {
      const float c2 = z[8 + t] * fz, c3 = z[12 + t] * fz;
      qz[2] = half_part_pair(c2, c3, false);
      qz[3] = half_part_pair(c2, c3, true);
      const __half2 hi = *reinterpret_cast<const __half2*>(&qz[2]);
      const __half2 lo = *reinterpret_cast<const __half2*>(&qz[3]);
      part += (__low2float(hi) + __low2float(lo)) + (__high2float(hi) + __high2float(lo));
    }
    part *= pow2f(4 * (t & 1));  // field weight 2^p0 (times 2^-24, with the 8 below)
    part += __shfl_xor_sync(kFull, part, 1);
    part += __shfl_xor_sync(kFull, part, 2);
    zoff = part * 0x1p-21f;  // 8 * 2^-24
  }
  // group sums of head g in the accumulator's units (2^-18 f)
  float qs[NG];
#pragma unroll
  for (int gg = 0; gg < NG; ++gg) qs[gg] = qsum_s[g * NG + gg] * f * 0x1p-18f;
  const float scale2 = p.sm_scale * kLog2e * 0x1p18f * finv;

  // readout state: the softmax of head g (this thread's logit rows), the output
  // with rows = channels and columns = head slots 2t, 2t+1
  float m2 = kMaxInit, l = 0.f;
  float o[V2 ? 1 : MT][4];       // dense values: row block mt (channels 16 mt + g, + 8)
  float oa[V2 ? NG : 1][4], ob[V2 ? NG : 1][4];  // 2-bit values, group gg: channels
                                                 // 32 gg + 4 g + {0, 1 | 2, 3}
  float vmin[V2 ? NG : 1];       // sum_j p_j min_{j,g} of head g (this thread's tokens)
  int ve[V2 ? NG : 1];           // 2-bit values: the exponent E of (head g, group gg)
#pragma unroll
  for (int mt = 0; mt < (V2 ? 1 : MT); ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
#pragma unroll
  for (int gg = 0; gg < (V2 ? NG : 1); ++gg) {
    oa[gg][0] = oa[gg][1] = oa[gg][2] = oa[gg][3] = 0.f;
    ob[gg][0] = ob[gg][1] = ob[gg][2] = ob[gg][3] = 0.f;
    vmin[gg] = 0.f;
    ve[gg] = -126;
  }
  // the byte of a value-code row holding channels 32 gg + 4 g .. + 3 is byte g & 3
  // of word 2 gg + (g >> 2); the permute puts it into byte 0 (token 2t or 2t+8)
  // and byte 2 (token 2t+1 or 2t+9)
  const uint32_t vsel = static_cast<uint32_t>((g & 3) | ((4 + (g & 3)) << 8));
  // ldmatrix row owned by this lane (dense values): matrix (lane >> 3), row (lane & 7)
  const int lm_row = 8 * (lane >> 4) + (lane & 7);  // + the slice's first token
  const int lm_chunk_hi = (lane >> 3) & 1;

  bool ok = true;
  // The kCW warps take the kSlices 16-token slices of the stages in turn (slice
  // j = tile j / kSlices, tokens 16 (j % kSlices) ..), each with its own online
  // softmax; a stage is released after its kSlices slices.
  for (int j = warp; j < ntiles * kSlices; j += kCW) {
    const int i = j / kSlices, jw = 16 * (j - i * kSlices);
    const int s = i % kStages;
    if (!mbar_wait(smem_addr(&bars[s]), (i / kStages) & 1)) {
      ok = false;
      break;
    }
    const int t0 = t_begin + i * kTile;
    uint8_t* st = stages + size_t(s) * L::kStage;
    const int nvalid = min(kTile, tile_end - t0);

    if (nvalid < jw + 16) {
      // tail of the split: rows past the end may hold anything (earlier tiles,
      // never-written shared memory): the planes whose values meet p = 0 in a
      // product are cleared (codes and key planes only meet masked logits)
      if constexpr (V2) {
        for (int idx = lane; idx < 16 * NG * 2; idx += 32) {
          const int pl = idx / (16 * NG), rem = idx - pl * 16 * NG;
          const int row = jw + rem / NG, gg = rem % NG;
          if (row >= nvalid)
            reinterpret_cast<float*>(st + (pl ? L::kVm : L::kVs))[row * NG + gg] = 0.f;
        }
      } else {
        for (int idx = lane; idx < 16 * 8 * L::kVBoxes; idx += 32) {
          const int bx = idx % L::kVBoxes, rem = idx / L::kVBoxes;
          const int row = jw + rem / 8, c16 = rem % 8;
          if (row >= nvalid)
            *reinterpret_cast<uint4*>(st + bx * L::kVBox + row * 128 + c16 * 16) =
                make_uint4(0, 0, 0, 0);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
    }

    // ---- logits of head g for the tokens jw + 8 nt + 2t, + 1 (C columns)
    float x[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int jb = jw + 8 * nt + g;      // this thread's B column (token)
      const int ja = jw + 8 * nt + 2 * t;  // its C columns
      uint32_t kw[D / 16];
#pragma unroll
      for (int v4 = 0; v4 < D / 64; ++v4) {
        const uint4 a = *reinterpret_cast<const uint4*>(st + L::kKc + jb * (D / 4) + 16 * v4);
        kw[4 * v4 + 0] = a.x; kw[4 * v4 + 1] = a.y; kw[4 * v4 + 2] = a.z; kw[4 * v4 + 3] = a.w;
      }
      float ksa[NG], ksb[NG], kma[NG], kmb[NG];
      load_groups<NG>(st + L::kKs + ja * NG * 4, ksa);
      load_groups<NG>(st + L::kKs + (ja + 1) * NG * 4, ksb);
      load_groups<NG>(st + L::kKm + ja * NG * 4, kma);
      load_groups<NG>(st + L::kKm + (ja + 1) * NG * 4, kmb);
      float sa = 0.f, sb = 0.f;
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t y = kw[2 * gg + e] >> sh;
          const uint32_t bb[2] = {y & m0, y & m1};
          mma_f16(acc, qa[2 * gg + e], bb);
        }
        const float2 hl = __fadd2_rn(make_float2(acc[0], acc[1]), make_float2(acc[2], acc[3]));
        sa = fmaf(ksa[gg], hl.x, sa);
        sb = fmaf(ksb[gg], hl.y, sb);
        sa = fmaf(kma[gg], qs[gg], sa);
        sb = fmaf(kmb[gg], qs[gg], sb);
      }
      if constexpr (R > 0) {
        uint32_t bz[2];
        if constexpr (R == 16) {
          const uint2 zw = *reinterpret_cast<const uint2*>(st + L::kZc + jb * 8);
          bz[0] = ((zw.x ^ 0x88888888u) >> sh) & mz;
          bz[1] = ((zw.y ^ 0x88888888u) >> sh) & mz;
        } else {
          const uint32_t zw = *reinterpret_cast<const uint32_t*>(st + L::kZc + jb * 4);
          bz[0] = ((zw ^ 0x88888888u) >> sh) & mz;
          bz[1] = 0u;
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        mma_f16(acc, qz, bz);
        const float2 zs = *reinterpret_cast<const float2*>(st + L::kZs + ja * 4);
        const float2 hl = __fadd2_rn(
            __fadd2_rn(make_float2(acc[0], acc[1]), make_float2(acc[2], acc[3])),
            make_float2(-zoff, -zoff));
        sa = fmaf(zs.x, hl.x, sa);
        sb = fmaf(zs.y, hl.y, sb);
      }
      x[nt][0] = ja < nvalid ? sa * scale2 : -INFINITY;
      x[nt][1] = ja + 1 < nvalid ? sb * scale2 : -INFINITY;
    }

    // ---- online softmax of head g over the warp's 16 tokens (m2 stays finite:
    // masked logits give p = 2^-inf = 0)
    float mx = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    const bool resc = mx > m2 + kRescale;
    float alpha = 1.0f;
    if (resc) {
      alpha = ex2_ftz(m2 - mx);
      m2 = mx;
    }
    float pr[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) pr[k] = ex2_ftz(x[k >> 1][k & 1] - m2);
    l = fmaf(l, alpha, (pr[0] + pr[1]) + (pr[2] + pr[3]));

    if constexpr (V2) {
      // tokens of this thread's B rows: jw + 2t, + 1 (pr[0], pr[1]) and
      // jw + 8 + 2t, + 1 (pr[2], pr[3])
      const int jr[4] = {jw + 2 * t, jw + 2 * t + 1, jw + 8 + 2 * t, jw + 9 + 2 * t};
      float vs[4][NG];
#pragma unroll
      for (int k = 0; k < 4; ++k) load_groups<NG>(st + L::kVs + jr[k] * NG * 4, vs[k]);
      // A operands of p . V: this thread's code byte (channels 32 gg + 4 g .. + 3)
      // of its four tokens, paired by token and split into two row blocks
      uint32_t aa[NG][4], ab[NG][4];
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const uint8_t* vc = st + L::kVc + 8 * gg + 4 * (g >> 2);
        const uint32_t c0 = *reinterpret_cast<const uint32_t*>(vc + jr[0] * (D / 4));
        const uint32_t c1 = *reinterpret_cast<const uint32_t*>(vc + jr[1] * (D / 4));
        const uint32_t c2 = *reinterpret_cast<const uint32_t*>(vc + jr[2] * (D / 4));
        const uint32_t c3 = *reinterpret_cast<const uint32_t*>(vc + jr[3] * (D / 4));
        const uint32_t z01 = __byte_perm(c0, c1, vsel), z23 = __byte_perm(c2, c3, vsel);
        aa[gg][0] = z01 & 0x00030003u; aa[gg][1] = z01 & 0x000C000Cu;
        aa[gg][2] = z23 & 0x00030003u; aa[gg][3] = z23 & 0x000C000Cu;
        ab[gg][0] = z01 & 0x00300030u; ab[gg][1] = z01 & 0x00C000C0u;
        ab[gg][2] = z23 & 0x00300030u; ab[gg][3] = z23 & 0x00C000C0u;
      }
      // B entries p_j scale_{j,g} of head g; their largest in the 16 tokens
      // (the quad's lanes) decides whether 2^E of (head g, group g) is raised
      // (branch-free: a raise is rare, but keeps the block one basic block)
      float w[NG][4];
      float rf[NG];
      bool raise = false;
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
#pragma unroll
        for (int k = 0; k < 4; ++k) w[gg][k] = pr[k] * vs[k][gg];
        float hx = fmaxf(fmaxf(w[gg][0], w[gg][1]), fmaxf(w[gg][2], w[gg][3]));
        hx = fmaxf(hx, __shfl_xor_sync(kFull, hx, 1));
        hx = fmaxf(hx, __shfl_xor_sync(kFull, hx, 2));
        const uint32_t hb = __float_as_uint(hx);
        const bool up = hb >= static_cast<uint32_t>(127 + ve[gg] + kRaiseLog2) << 23;
        const int en = max(-126, min(126, static_cast<int>(hb >> 23) - 127));
        // 2^(E_old - E_new) on a raise
        rf[gg] = up ? alpha * (pow2_neg(-ve[gg]) * pow2_neg(en)) : alpha;
        ve[gg] = up ? en : ve[gg];
        raise |= up;
      }
      {
        float vm[4][NG];
#pragma unroll
        for (int k = 0; k < 4; ++k) load_groups<NG>(st + L::kVm + jr[k] * NG * 4, vm[k]);
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) {
          float a = vmin[gg] * alpha;
#pragma unroll
          for (int k = 0; k < 4; ++k) a = fmaf(pr[k], vm[k][gg], a);
          vmin[gg] = a;
        }
      }
      if (__any_sync(kFull, resc || raise)) {
        // output columns = head slots 2t, 2t+1: their factors live in lanes 8t, 8t+4
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) {
          const float r0 = __shfl_sync(kFull, rf[gg], 8 * t);
          const float r1 = __shfl_sync(kFull, rf[gg], 8 * t + 4);
          oa[gg][0] *= r0; oa[gg][1] *= r1; oa[gg][2] *= r0; oa[gg][3] *= r1;
          ob[gg][0] *= r0; ob[gg][1] *= r1; ob[gg][2] *= r0; ob[gg][3] *= r1;
        }
      }
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const float fe = pow2_neg(ve[gg]);
        const uint32_t bv[2] = {f16x2(w[gg][0] * fe, w[gg][1] * fe),
                                f16x2(w[gg][2] * fe, w[gg][3] * fe)};
        mma_f16(oa[gg], aa[gg], bv);
        mma_f16(ob[gg], ab[gg], bv);
      }
    } else {
      if (__any_sync(kFull, resc)) {
        const float r0 = __shfl_sync(kFull, alpha, 8 * t), r1 = __shfl_sync(kFull, alpha, 8 * t + 4);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          o[mt][0] *= r0; o[mt][1] *= r1; o[mt][2] *= r0; o[mt][3] *= r1;
        }
      }
      // B = p of head g, tokens (2t, 2t+1 | 8+2t, 9+2t), as bf16 high + low parts
      const uint32_t bh[2] = {bf16x2(pr[0], pr[1]), bf16x2(pr[2], pr[3])};
      float2 hf[2];
      hf[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bh[0]));
      hf[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bh[1]));
      const uint32_t bl[2] = {bf16x2(pr[0] - hf[0].x, pr[1] - hf[0].y),
                              bf16x2(pr[2] - hf[1].x, pr[3] - hf[1].y)};
      const uint32_t vbase = smem_addr(st);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int chunk = 2 * mt + lm_chunk_hi;
        const uint32_t addr = vbase + (chunk >> 3) * L::kVBox + (jw + lm_row) * 128 +
                              (((chunk & 7) ^ ((jw + lm_row) & 7)) << 4);
        uint32_t a[4];
        ldsm_x4_trans(addr, a);
        mma_bf16(o[mt], a, bh);
        mma_bf16(o[mt], a, bl);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&bars[kStages + s]));
  }
  if (!ok && lane == 0 && p.err) atomicOr(p.err, kDevErrWaitTimeout);

  // ---- merge the consumer warps' partial softmax states
  l += __shfl_xor_sync(kFull, l, 1);
  l += __shfl_xor_sync(kFull, l, 2);
#pragma unroll
  for (int gg = 0; gg < (V2 ? NG : 0); ++gg) {
    vmin[gg] += __shfl_xor_sync(kFull, vmin[gg], 1);
    vmin[gg] += __shfl_xor_sync(kFull, vmin[gg], 2);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  float* mo = reinterpret_cast<float*>(stages);  // [kCW][8][D]
  float* mm = mo + kCW * kGM * D;                // [kCW][8]
  float* ml = mm + kCW * kGM;                    // [kCW][8]
  float* vms = ml + kCW * kGM;                   // [kCW][8][NG] (2-bit values)
  __shared__ int flags[2];                       // [0] a warp failed, [1] last CTA
  if (tid == 0) flags[0] = 0;
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  if (!ok) flags[0] = 1;
  float* mw = mo + warp * kGM * D;
  if constexpr (V2) {
    // back from the field weights (2^-24, 2^-22, 2^-20, 2^-18 for the channels
    // 4g + 0..3 of a group) and from units of 2^E of each column's head slot
    // (held by lanes 8t, 8t + 4)
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) {
      const float u = pow2_neg(-ve[gg]);
      const float ue[2] = {__shfl_sync(kFull, u, 8 * t), __shfl_sync(kFull, u, 8 * t + 4)};
      const int c = 32 * gg + 4 * g;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float* row = mw + (2 * t + e) * D + c;
        row[0] = (oa[gg][e] * 0x1p24f) * ue[e];
        row[1] = (oa[gg][2 + e] * 0x1p22f) * ue[e];
        row[2] = (ob[gg][e] * 0x1p20f) * ue[e];
        row[3] = (ob[gg][2 + e] * 0x1p18f) * ue[e];
      }
    }
  } else {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        mw[(2 * t + e) * D + 16 * mt + g] = o[mt][e];
        mw[(2 * t + e) * D + 16 * mt + g + 8] = o[mt][2 + e];
      }
    }
  }
  if (t == 0) {
    mm[warp * kGM + g] = m2;
    ml[warp * kGM + g] = l;
#pragma unroll
    for (int gg = 0; gg < (V2 ? NG : 0); ++gg) vms[(warp * kGM + g) * NG + gg] = vmin[gg];
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  const bool failed = flags[0] != 0;
  const bool single = p.splits == 1;
  if (failed && single) return;
  const PartView pv = part_view(p.part, static_cast<size_t>(p.c.B) * p.Hq, p.splits, D);
  for (int idx = tid; idx < G * D; idx += kCT) {
    const int h = idx / D, c = idx - h * D;
    float M = kMaxInit;
#pragma unroll
    for (int w = 0; w < kCW; ++w) M = fmaxf(M, mm[w * kGM + h]);
    float O = 0.f, Ls = 0.f;
    {
#pragma unroll
      for (int w = 0; w < kCW; ++w) {
        const float fw = exp2f(mm[w * kGM + h] - M);
        float ow = mo[(w * kGM + h) * D + c];
        if constexpr (V2) ow += vms[(w * kGM + h) * NG + c / 32];
        O = fmaf(fw, ow, O);
        Ls = fmaf(fw, ml[w * kGM + h], Ls);
      }
    }
    const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
    if (single) {
      p.out[bh * D + c] = Ls > 0.f ? O / Ls : 0.f;
      if (c == 0 && p.lse) p.lse[bh] = Ls > 0.f ? (M + log2f(Ls)) * kLn2 : -INFINITY;
    } else if (!failed) {
      pv.o[(bh * p.splits + split) * D + c] = O;
      if (c == 0) {
        pv.m[bh * p.splits + split] = Ls > 0.f ? M * kLn2 : -INFINITY;
        pv.l[bh * p.splits + split] = Ls;
      }
    }
  }
  if (single || !p.fused) return;  // unfused: the combine kernel merges the splits

  // ---- split arrival; the last CTA of this (b, kv) merges all splits.  Every
  // CTA arrives (also one that failed), so the counter always returns to zero.
  __threadfence();
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  if (tid == 0) {
    const unsigned old = atomicAdd(p.counters + bk, 1u);
    flags[1] = old == static_cast<unsigned>(p.splits - 1);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  if (!flags[1]) return;
  __threadfence();
  // the split weights overwrite the (consumed) warp partials
  merge_splits_last<D>(p, b, h0, reinterpret_cast<float*>(stages), warp, kCW, lane);
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  if (tid == 0) p.counters[bk] = 0;  // ready for the next call
}

// ---------------------------------------------------------------- host side
constexpr int kMaxDev = 64;

template <int D, int R, bool V2>
struct HmVariant {
  static int occupancy[kMaxDev];  // CTAs per SM, 0 = not yet known
  static std::mutex mu;

  static constexpr size_t smem() { return hm_smem_bytes<D, R, V2>(); }
  // the warps' partials (outputs, maxima, sums, group minima), and later the
  // merging CTA's [G][splits] split weights, lie inside the stages
  static_assert(sizeof(float) * kCW * kGM * (D + 2 + D / 32) <=
                    size_t(kStagesHM<V2>) * StageLayout<D, R, V2>::kStage,
                "warp partials fit in the stages");
  static_assert(sizeof(float) * kGM * kMaxMmaSplits <=
                    size_t(kStagesHM<V2>) * StageLayout<D, R, V2>::kStage,
                "split weights fit in the stages");

  static int ctas_per_sm() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
      cudaGetLastError();
      return 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (occupancy[dev] == 0) {
      auto k = decode_hm_kernel<D, R, V2>;
      const int sm = static_cast<int>(smem());
      int n = 0;
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) !=
              cudaSuccess ||
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kThreads, sm) != cudaSuccess) {
        cudaGetLastError();
        n = -1;
      }
      occupancy[dev] = n > 0 ? n : -1;
    }
    return occupancy[dev] > 0 ? occupancy[dev] : 0;
  }

  static cudaError_t launch(const DecodeParams& p, cudaStream_t s) {
    if (ctas_per_sm() == 0) return cudaErrorInvalidConfiguration;
    CUtensorMap vmap;
    memset(&vmap, 0, sizeof(vmap));
    const dim3 grid(p.splits, p.c.Hkv, p.c.B);
    if (!V2) {
      if (!tensor_maps_available()) return cudaErrorNotSupported;
      // [slab][row in slab][channel]: one slab per (b, kv), or per (page, kv)
      const bool paged = p.c.page_size > 0;
      const uint64_t rows = static_cast<uint64_t>(paged ? p.c.page_size : p.c.T_cap);
      const uint64_t slabs = static_cast<uint64_t>(paged ? p.c.num_pages : p.c.B) * p.c.Hkv;
      if (!encode_bf16_rows(&vmap, p.c.v, D, rows, slabs, kTile)) return cudaErrorInvalidValue;
    }
    decode_hm_kernel<D, R, V2><<<grid, kThreads, smem(), s>>>(p, vmap);
    return cudaGetLastError();
  }
};
template <int D, int R, bool V2>
int HmVariant<D, R, V2>::occupancy[kMaxDev];
template <int D, int R, bool V2>
std::mutex HmVariant<D, R, V2>::mu;

template <typename F>
auto hm_dispatch(int d, int r, bool v2, F&& f) -> decltype(f(HmVariant<128, 16, false>{})) {
#define HEADQ_HM_CASE(DD, RR, VV) \
  if (d == DD && r == RR && v2 == VV) return f(HmVariant<DD, RR, VV>{});
  HEADQ_HM_CASE(128, 16, false) HEADQ_HM_CASE(128, 8, false) HEADQ_HM_CASE(128, 0, false)
  HEADQ_HM_CASE(64, 16, false) HEADQ_HM_CASE(64, 8, false) HEADQ_HM_CASE(64, 0, false)
  HEADQ_HM_CASE(128, 16, true) HEADQ_HM_CASE(128, 8, true)
  HEADQ_HM_CASE(64, 16, true) HEADQ_HM_CASE(64, 8, true)
#undef HEADQ_HM_CASE
  return decltype(f(HmVariant<128, 16, false>{}))();
}

}  // namespace

bool hm_decode_supported(const headq_cache& c, int G) {
  if (c.d != 64 && c.d != 128) return false;
  if (c.kmode != HEADQ_K_TOKEN || G < 5 || G > kGM) return false;
  if (c.vmode == HEADQ_V_2BIT) return c.r == 8 || c.r == 16;
  return c.vmode == HEADQ_V_DENSE && c.v_dtype == HEADQ_BF16 &&
         (c.r == 0 || c.r == 8 || c.r == 16) && tensor_maps_available();
}

int hm_decode_ctas_per_sm(const headq_cache& c) {
  return hm_dispatch(c.d, c.r, c.vmode == HEADQ_V_2BIT,
                     [](auto v) { return decltype(v)::ctas_per_sm(); });
}

cudaError_t launch_decode_hm(const DecodeParams& p, cudaStream_t s) {
  // 0 means no variant matched; otherwise the launch status + 1
  const int e = hm_dispatch(p.c.d, p.c.r, p.c.vmode == HEADQ_V_2BIT, [&](auto v) {
    return static_cast<int>(decltype(v)::launch(p, s)) + 1;
  });
  return e == 0 ? cudaErrorInvalidValue : static_cast<cudaError_t>(e - 1);
}

}  // namespace headq
