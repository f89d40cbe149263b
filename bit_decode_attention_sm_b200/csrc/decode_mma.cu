// HeadQ decode attention, bandwidth kernel for sm_100a ("HeadQ: Model-Visible
// Distortion and Score-Space Correction for KV-Cache Quantization", gist.science
// summary, section 3, step 3: the runtime query turns the side code into an
// additive logit correction; the readout is the attention-weighted sum of values).
//
// Same mathematics as decode_attn.cu's generic kernel; this one is built to stream
// the packed cache at HBM speed:
//
//  * TMA pipeline.  One producer warp fills 3-4 shared-memory stages of 64
//    tokens with 1-D bulk copies of the contiguous code / scale / side planes and
//    a 3-D tensor copy (128-byte swizzle) of the bf16 value tile; four consumer
//    warps each take 16 tokens of every stage.  mbarriers carry completion; every
//    wait is bounded and flags the workspace error word on expiry.
//  * q . code on tensor cores.  mma.m16n8k16 (fp16 in, fp32 accumulate) with the
//    16 tokens of a warp on M and the query heads on N, each head's query split
//    into an fp16 high and low part in adjacent columns (so 4 heads fill N = 8 and
//    high + low add up inside one thread).  2-bit codes are exact small integers:
//    0x6400 | (code << 2k) is the fp16 value 1024 + code*4^k, and one exact fp16
//    FMA turns it back into the code.  Channels map to MMA k-slots so that each
//    thread's codes are one 16-bit word per 32-channel group, and each group keeps
//    its own accumulator, so the per-group scale and minimum are applied exactly as
//    the dequantisation min + code*scale defines them:
//        q.k^base_j = sum_g ( min_{j,g} Q_g + scale_{j,g} sum_{c in g} q_c code_{j,c} ).
//    The side-code correction is one more MMA on the unpacked signed nibbles
//    against sigma * U_h^T q (also split high / low), scaled by the side scale.
//  * softmax in the log2 domain with a lazily refreshed running max (the output is
//    rescaled only when the max grows by more than 2^8), per warp.
//  * p . V on tensor cores.  mma.m16n8k16 (bf16) with the value dims on M (A = V^T
//    fed by ldmatrix.trans from the swizzled tile) and the heads on N, p split into
//    bf16 high and low parts in adjacent columns; the probabilities move from the
//    logit layout to the B-operand layout with four warp shuffles.
//  * the four warps' (max, sum, output) are merged through shared memory at the
//    end; splits are merged by the common log-sum-exp combine kernel.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "codec.cuh"
#include "decode_pipe.cuh"
#include "headq_internal.cuh"

namespace headq {
namespace {
using namespace dc;

constexpr int kCW = 4;                   // consumer warps
constexpr int kTile = kPipeTile;         // tokens per stage (16 per consumer warp)
constexpr int kThreads = (kCW + 1) * 32; // + one producer warp
// pipeline depth: 4 stages of 64 tokens, 3 for the two-N-tile variants (their
// q fragments take the shared memory of the fourth) so that two CTAs fit per SM
template <int NT>
constexpr int kStagesFor = NT == 1 ? 4 : 3;
constexpr float kRescale = 8.0f;         // log2 units the stale max may lag (p <= 2^8)
// 2-bit values: p * scale enters the fp16 operand relative to a power of two
// 2^E per (warp, head slot, group) that is raised once a product reaches
// 2^kRaiseLog2 of it (fp16 holds up to 2^16).
constexpr int kRaiseLog2 = 12;

// Shared-memory stage of kTile tokens (StageLayout), plus this kernel's
// per-warp scratch for 2-bit values.
template <int D, int R, bool V2 = false, bool KCH = false>
struct Layout : StageLayout<D, R, V2, KCH> {
  // 2-bit values: per consumer warp, the fp16 codes of its D/4 channels for the
  // kTile tokens of a stage (the warp's readout slice)
  static constexpr int kCodeTile = V2 ? kTile * (D / kCW) * 2 : 0;
  // 2-bit values: the probabilities p [2 buffers][kCW warps][8 head slots][24]
  // (16 tokens, rows padded for conflict-free stores and loads) and each warp's
  // running max [2][8 head slots][kCW], passed from the logit warps to the
  // readout warps
  static constexpr int kPexFloats = 2 * kCW * 8 * 24;
  static constexpr int kExBytes = V2 ? (kPexFloats + 2 * 8 * kCW) * 4 : 0;
};

// the two-N-tile variants keep each thread's q B-operand fragments in shared
// memory instead of 32 registers, so that two CTAs fit on an SM
template <int NT>
constexpr bool kBqInSmem = NT == 2;

template <int D, int R, int NT, bool V2, bool KCH>
constexpr size_t smem_bytes() {
  using L = Layout<D, R, V2, KCH>;
  constexpr size_t bq_bytes = kBqInSmem<NT> ? size_t(kCW) * 32 * (D / 16) * NT * 8 : 0;
  // stages | per-warp value code tiles | p exchange | q fragments | q [GM][D] |
  // group sums [GM][NG] | sigma U^T q [GM][R] | U [D][R] | appended token's
  // residual [D] and projection [R] | max |q| per (head, group) [GM][NG] | the
  // query as bulk-copied (raw bf16 or fp32) [GM][D] | barriers.  2-bit values
  // (three CTAs per SM) land the raw query and U_h in the code tiles, which are
  // free until the main loop (the fused append then reads U_h from global
  // memory).
  return 1024 + size_t(kStagesFor<NT>) * L::kStage + size_t(kCW) * L::kCodeTile + L::kExBytes +
         bq_bytes +
         sizeof(float) * ((4 * NT) * (D + L::NG + (R > 0 ? R : 1)) +
                          (V2 ? 0 : D * (R > 0 ? R : 1)) + D + (R > 0 ? R : 1) +
                          (4 * NT) * L::NG + (V2 ? 0 : (4 * NT) * D)) +
         32 * kStagesFor<NT> + 80;  // barriers (2 kStages + 4), stage tile starts,
                                    // two 16-byte alignments
}

// ---------------------------------------------------------------- the kernel
// CTAs per SM the registers are budgeted for: 2-bit values keep a small
// readout accumulator (their channel slice), so three fit
template <bool V2>
constexpr int kMinCtas = V2 ? 3 : 2;

template <int D, int R, int NT, bool V2, bool KCH>
__global__ void __launch_bounds__(kThreads, kMinCtas<V2>)
decode_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap vmap) {
  using L = Layout<D, R, V2, KCH>;
  constexpr int NG = L::NG;
  constexpr int KS = D / 16;   // k-steps of 16 channels
  constexpr int MT = D / 16;   // 16-dim row blocks of the output
  constexpr int GM = 4 * NT;   // head slots
  constexpr int RR = R > 0 ? R : 1;
  constexpr int kCT = kCW * 32;  // consumer threads
  constexpr int kStages = kStagesFor<NT>;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align(smem_raw, 1024);
  uint8_t* stages = smem;
  uint8_t* ctiles = smem + size_t(kStagesFor<NT>) * L::kStage;  // [kCW][16][D] fp16 value codes
  float* pex_s = reinterpret_cast<float*>(ctiles + size_t(kCW) * L::kCodeTile);  // 2-bit values
  float* mex_s = pex_s + L::kPexFloats;
  uint2* bq_s = reinterpret_cast<uint2*>(ctiles + size_t(kCW) * L::kCodeTile +
                                         L::kExBytes);  // [KS][NT][128]
  float* q_s = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bq_s) +
                                        (kBqInSmem<NT> ? size_t(kCW) * 32 * KS * NT * 8 : 0));
  float* qsum_s = q_s + GM * D;                                               // [GM][NG]
  float* qt_s = qsum_s + GM * NG;                                             // [GM][RR]
  // U_h [D][RR] in shared memory (2-bit values: in the code tiles, after the query)
  float* u_s = V2 ? reinterpret_cast<float*>(ctiles + GM * D * 4) : qt_s + GM * RR;
  static_assert(!V2 || (4 * NT) * D * 4 + D * (R > 0 ? R : 1) * 4 <= kCW * L::kCodeTile,
                "the query and U_h fit in the code tiles");
  float* enew_s = qt_s + GM * RR + (V2 ? 0 : D * RR);                         // [D]
  float* ynew_s = enew_s + D;                                                 // [RR]
  float* qmax_s = ynew_s + RR;                                                // [GM][NG]
  // [GM][D] floats of room, 16-byte aligned (a bulk-copy destination): the query
  // as copied (bf16 or fp32)
  float* qraw_s = V2 ? reinterpret_cast<float*>(ctiles) : smem_align(qmax_s + GM * NG, 16);
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(smem_align(V2 ? qmax_s + GM * NG : qraw_s + GM * D, 16));
  // bars[s] = stage full, bars[kStages + s] = stage empty, bars[2 kStages + 1] =
  // the query and U_h are in shared memory (bars[2 kStages] unused),
  // bars[2 kStages + 2 + b] = exchange buffer b holds every warp's p (2-bit values)
  int* stile_s = reinterpret_cast<int*>(bars + 2 * kStages + 4);  // [kStages] tile start, -1: end

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int G = p.G, Hkv = p.c.Hkv;
  int Tb = p.T;
  if (p.seq_lens) Tb = max(0, min(p.seq_lens[b], p.T));
  const int t_begin = split * p.chunk;
  const int t_end = min(Tb, t_begin + p.chunk);
  const int ntiles = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
  const size_t bk = static_cast<size_t>(b) * Hkv + kv;
  const int h0 = kv * G;
  // position of this step's new token (fused append), -1 when none
  const int pos = (p.k_new != nullptr && Tb > 0) ? Tb - 1 : -1;
  const int tile_end = t_end;  // a tile's tokens stop at the chunk end

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&bars[s]), 1);
      mbar_init(smem_addr(&bars[kStages + s]), kCW);
    }
    mbar_init(smem_addr(&bars[2 * kStages]), 1);
    mbar_init(smem_addr(&bars[2 * kStages + 1]), 1);
    mbar_init(smem_addr(&bars[2 * kStages + 2]), kCW);
    mbar_init(smem_addr(&bars[2 * kStages + 3]), kCW);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // ------------------------------------------------------------ producer warp
  // starts streaming at once; the consumers prepare the query meanwhile
  if (warp == kCW) {
    // 2-bit values reuse u_s (in the code tiles) once the main loop starts: the
    // fused append's encoder reads U_h from global memory
    produce_tiles<D, R, V2, KCH, kStages, !V2>(p, &vmap, stages, bars, bars + kStages,
                                               bars + 2 * kStages + 1, stile_s, qraw_s, u_s,
                                               enew_s, b, kv, h0, t_begin, tile_end, ntiles,
                                               pos, lane);
    return;
  }

  // ------------------------------------------------------------ consumer warps
  // query prep: q and U_h (bulk-copied by the producer), group sums, sigma U_h^T q
  if (!mbar_wait(smem_addr(&bars[2 * kStages + 1]), 0) && tid == 0 && p.err)
    atomicOr(p.err, kDevErrWaitTimeout);
  for (int i = tid; i < GM * D; i += kCT)
    q_s[i] = i < G * D ? load_elem(qraw_s, i, p.q_bf16) : 0.0f;
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  for (int i = tid; i < GM * NG; i += kCT) {
    const int h = i / NG, g = i - h * NG;
    float acc = 0.0f, amax = 0.0f;
    for (int c = 0; c < 32; ++c) {
      const float v = q_s[h * D + g * 32 + c];
      acc += v;
      amax = fmaxf(amax, fabsf(v));
    }
    qsum_s[i] = acc;
    qmax_s[i] = amax;
  }
  if constexpr (R > 0) {
    for (int i = tid; i < GM * R; i += kCT) {
      const int h = i / R, ii = i - h * R;
      float acc = 0.0f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = fmaf(u_s[c * R + ii], q_s[h * D + c], acc);
      qt_s[i] = p.corr_sign * acc;
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");

  const int g = lane >> 2, t = lane & 3;
  const int jw = 16 * warp;

  // B operands of q . code: column n = g is head (g >> 1), fp16 high (g even) or
  // low (g odd) part; k-step ks = 2*grp + e, k-slots (2t, 2t+1) <-> channels
  // 32*grp + 8t + 4e + {0, 1}, (2t+8, 2t+9) <-> 32*grp + 8t + 4e + {2, 3}.
  // Every head's query enters the fp16 operands scaled by its own power of two
  // (head_prescale): fb for the head of this thread's B column, fo / scale2 for
  // the head of its output column.
  float fb[NT], fo[NT], scale2[NT], foinv[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float finv;
    head_prescale<NG>(qmax_s, 4 * nt + (g >> 1), fb[nt], finv);
    head_prescale<NG>(qmax_s, 4 * nt + t, fo[nt], finv);
    scale2[nt] = p.sm_scale * kLog2e * finv;
    foinv[nt] = finv;
  }
  uint32_t bq[kBqInSmem<NT> ? 1 : KS][NT][2];
#pragma unroll
  for (int ks = 0; ks < (KCH ? 0 : KS); ++ks) {  // per-channel keys: rebuilt per tile
    const int ch0 = 32 * (ks >> 1) + 8 * t + 4 * (ks & 1);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float* qh = q_s + (4 * nt + (g >> 1)) * D + ch0;
      const float f = fb[nt];
      const uint32_t b0 = half_part_pair(qh[0] * f, qh[1] * f, g & 1);
      const uint32_t b1 = half_part_pair(qh[2] * f, qh[3] * f, g & 1);
      if constexpr (kBqInSmem<NT>) {
        bq_s[(ks * NT + nt) * kCT + tid] = make_uint2(b0, b1);
      } else {
        bq[ks][nt][0] = b0;
        bq[ks][nt][1] = b1;
      }
    }
  }
  uint32_t bz[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    bz[nt][0] = bz[nt][1] = 0;
    if constexpr (R == 16) {
      const float* z = qt_s + (4 * nt + (g >> 1)) * R + 4 * t;
      const float f = fb[nt];
      bz[nt][0] = half_part_pair(z[0] * f, z[1] * f, g & 1);
      bz[nt][1] = half_part_pair(z[2] * f, z[3] * f, g & 1);
    } else if constexpr (R == 8) {
      const float* z = qt_s + (4 * nt + (g >> 1)) * R + 2 * t;
      const float f = fb[nt];
      bz[nt][0] = half_part_pair(z[0] * f, z[1] * f, g & 1);
    }
  }
  // group sums of this thread's output head (4*nt + t)
  float qsum[NT][NG];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) qsum[nt][gg] = qsum_s[(4 * nt + t) * NG + gg] * fo[nt];

  const uint32_t sel = (2 * t) | ((2 * t + 1) << 4) | ((2 * t) << 8) | ((2 * t + 1) << 12);
  const uint32_t sel8 = t | (4 << 4) | (t << 8) | (4 << 12);
  // ldmatrix row owned by this lane: matrix (lane >> 3), row (lane & 7)
  const int lm_tok = jw + 8 * (lane >> 4) + (lane & 7);
  const int lm_chunk_hi = (lane >> 3) & 1;

  float m2[NT], l[NT];
  float o[V2 ? 1 : MT][NT][4];      // dense values: columns (head, high/low part)
  // 2-bit values.  Logits and softmax are per warp (its 16 tokens of each tile,
  // as for dense values); the readout is split by channel: this warp reads out
  // channels [cw0, cw0 + CW) of all kTile tokens of each tile (p of the other
  // warps' tokens through shared memory), into ov with columns = the 8 head
  // slots (C columns 2t, 2t+1).  ov is relative to Mref, the running maximum of
  // the warps' maxima for head slot g (this thread's B column), and in units of
  // 2^ve, the exponent of head slot g in this channel slice.
  constexpr int CW = D / kCW, MTW = CW / 16, CPR = CW / 8;
  const int cw0 = warp * CW, gw = cw0 / 32;
  float ov[V2 ? MTW : 1][4];
  int ve = -126;
  float Mref = -INFINITY;
  float vmin_acc[NT][V2 ? NG : 1];  // 2-bit values: sum_j p_j min_{j,g} per group (this warp's tokens)
  uint8_t* ctile = ctiles + size_t(warp) * L::kCodeTile;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int gg = 0; gg < (V2 ? NG : 1); ++gg) vmin_acc[nt][gg] = 0.f;
    m2[nt] = -INFINITY;
    l[nt] = 0.0f;
#pragma unroll
    for (int mt = 0; mt < (V2 ? 1 : MT); ++mt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
  }
#pragma unroll
  for (int mt = 0; mt < (V2 ? MTW : 1); ++mt) ov[mt][0] = ov[mt][1] = ov[mt][2] = ov[mt][3] = 0.f;

  bool ok = true;
  for (int i = 0;; ++i) {
    const int s = i % kStages;
    if (!mbar_wait(smem_addr(&bars[s]), (i / kStages) & 1)) {
      ok = false;
      break;
    }
    const int t0 = stile_s[s];  // the producer's tile for this stage, -1: no more
    if (t0 < 0) break;
    uint8_t* st = stages + size_t(s) * L::kStage;
    const int nvalid = min(kTile, tile_end - t0);
    const int j0 = jw + g, j1 = j0 + 8;
    const bool val0 = j0 < nvalid, val1 = j1 < nvalid;

    if constexpr (V2) {
      // the fp16 codes of this warp's channel slice for all kTile tokens: row r =
      // token r (CW * 2 bytes), its 16-byte chunk c stored at c ^ sz(r),
      // sz(r) = (r / (8 / CPR)) % CPR, so that the 16-byte stores of 8 lanes and
      // the 8 rows read by an ldmatrix each cover all 8 bank groups
      constexpr int WPT = CW / 16;  // 32-bit code words of the slice per token
      for (int task = lane; task < kTile * WPT; task += 32) {
        const int r = task / WPT, wd = task - r * WPT;
        const uint32_t wv = *reinterpret_cast<const uint32_t*>(st + L::kVc + r * (D / 4) +
                                                               cw0 / 4 + 4 * wd);
        uint32_t v1[4], v2[4];
        unpack_codes(__byte_perm(wv, 0u, 0x1010u), v1);  // channels 16 wd + 0..7 of the slice
        unpack_codes(__byte_perm(wv, 0u, 0x3232u), v2);  // 16 wd + 8..15
        const int sz = (r / (8 / CPR)) % CPR;
        uint8_t* row = ctile + r * (CW * 2);
        *reinterpret_cast<uint4*>(row + (((2 * wd) ^ sz) << 4)) = make_uint4(v1[0], v1[1], v1[2], v1[3]);
        *reinterpret_cast<uint4*>(row + (((2 * wd + 1) ^ sz) << 4)) =
            make_uint4(v2[0], v2[1], v2[2], v2[3]);
      }
      __syncwarp();
    } else if (nvalid < jw + 16) {  // tail of the split: clear value rows past the end
      for (int idx = lane; idx < 16 * 8 * L::kVBoxes; idx += 32) {
        const int bx = idx % L::kVBoxes, rem = idx / L::kVBoxes;
        const int row = jw + rem / 8, c16 = rem % 8;
        if (row >= nvalid)
          *reinterpret_cast<uint4*>(st + bx * L::kVBox + row * 128 + c16 * 16) =
              make_uint4(0, 0, 0, 0);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
    }

    // ---- per-channel keys: the B operands of q . code are the query times the
    // block's scale, (q * scale)_c, rebuilt for each tile (one 64-token block),
    // prescaled by a power of two per (head, block) from their largest
    // magnitude; the minimum enters as one term q . min per (head, block)
    float kfinv[KCH ? NT : 1], kqmin[KCH ? NT : 1];
    if constexpr (KCH) {
      const float* ksc = reinterpret_cast<const float*>(st + L::kKs);  // [D] block scale
      const float* kmn = reinterpret_cast<const float*>(st + L::kKm);  // [D] block minimum
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float* qh = q_s + (4 * nt + (g >> 1)) * D;
        float qv[KS][4];
        float mx = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const int ch0 = 32 * (ks >> 1) + 8 * t + 4 * (ks & 1);
          const float4 a = *reinterpret_cast<const float4*>(qh + ch0);
          const float4 c = *reinterpret_cast<const float4*>(ksc + ch0);
          qv[ks][0] = a.x * c.x; qv[ks][1] = a.y * c.y; qv[ks][2] = a.z * c.z; qv[ks][3] = a.w * c.w;
          mx = fmaxf(mx, fmaxf(fmaxf(fabsf(qv[ks][0]), fabsf(qv[ks][1])),
                               fmaxf(fabsf(qv[ks][2]), fabsf(qv[ks][3]))));
        }
        // the head of this B column: its eight lanes (lane >> 3)
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
        float fk, fkinv;
        pow2_prescale(mx, fk, fkinv);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const uint32_t b0 = half_part_pair(qv[ks][0] * fk, qv[ks][1] * fk, g & 1);
          const uint32_t b1 = half_part_pair(qv[ks][2] * fk, qv[ks][3] * fk, g & 1);
          if constexpr (kBqInSmem<NT>) {
            bq_s[(ks * NT + nt) * kCT + tid] = make_uint2(b0, b1);
          } else {
            bq[ks][nt][0] = b0;
            bq[ks][nt][1] = b1;
          }
        }
        // the output head 4 nt + t: its factor from lane 8t; q . min over the
        // eight lanes of the same t, 16 channels each
        kfinv[nt] = __shfl_sync(kFull, fkinv, 8 * t);
        const int cb = (D / 8) * g;  // this lane's d/8 channels
        const float* qo = q_s + (4 * nt + t) * D + cb;
        float qm = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          const float4 a = *reinterpret_cast<const float4*>(qo + 4 * c4);
          const float4 m = *reinterpret_cast<const float4*>(kmn + cb + 4 * c4);
          qm = fmaf(a.x, m.x, fmaf(a.y, m.y, fmaf(a.z, m.z, fmaf(a.w, m.w, qm))));
        }
        qm += __shfl_xor_sync(kFull, qm, 4);
        qm += __shfl_xor_sync(kFull, qm, 8);
        qm += __shfl_xor_sync(kFull, qm, 16);
        kqmin[nt] = qm;
      }
    }

    // ---- q . code and the side-code correction on tensor cores
    float acc[NG + (R > 0 ? 1 : 0)][NT][4];
#pragma unroll
    for (int a = 0; a < NG + (R > 0 ? 1 : 0); ++a)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[a][nt][0] = acc[a][nt][1] = acc[a][nt][2] = acc[a][nt][3] = 0.f;

    uint32_t cw0[D / 16], cw1[D / 16];
#pragma unroll
    for (int v4 = 0; v4 < D / 64; ++v4) {
      const uint4 a = *reinterpret_cast<const uint4*>(st + L::kKc + j0 * (D / 4) + 16 * v4);
      const uint4 c = *reinterpret_cast<const uint4*>(st + L::kKc + j1 * (D / 4) + 16 * v4);
      cw0[4 * v4 + 0] = a.x; cw0[4 * v4 + 1] = a.y; cw0[4 * v4 + 2] = a.z; cw0[4 * v4 + 3] = a.w;
      cw1[4 * v4 + 0] = c.x; cw1[4 * v4 + 1] = c.y; cw1[4 * v4 + 2] = c.z; cw1[4 * v4 + 3] = c.w;
    }
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) {
      uint32_t u0[4], u1[4];
      unpack_codes(__byte_perm(cw0[2 * gg], cw0[2 * gg + 1], sel), u0);
      unpack_codes(__byte_perm(cw1[2 * gg], cw1[2 * gg + 1], sel), u1);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t a[4] = {u0[2 * e], u1[2 * e], u0[2 * e + 1], u1[2 * e + 1]};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if constexpr (kBqInSmem<NT>) {
            const uint2 bv = bq_s[((2 * gg + e) * NT + nt) * kCT + tid];
            const uint32_t b[2] = {bv.x, bv.y};
            mma_f16(acc[gg][nt], a, b);
          } else {
            mma_f16(acc[gg][nt], a, bq[2 * gg + e][nt]);
          }
        }
      }
    }
    float zs0 = 0.f, zs1 = 0.f;
    if constexpr (R > 0) {
      uint32_t a[4];
      if constexpr (R == 16) {
        const uint2 z0 = *reinterpret_cast<const uint2*>(st + L::kZc + j0 * 8);
        const uint2 z1 = *reinterpret_cast<const uint2*>(st + L::kZc + j1 * 8);
        unpack_side(__byte_perm(z0.x, z0.y, sel) ^ 0x88888888u, a[0], a[2]);
        unpack_side(__byte_perm(z1.x, z1.y, sel) ^ 0x88888888u, a[1], a[3]);
      } else {
        const uint32_t z0 = *reinterpret_cast<const uint32_t*>(st + L::kZc + j0 * 4);
        const uint32_t z1 = *reinterpret_cast<const uint32_t*>(st + L::kZc + j1 * 4);
        uint32_t dummy;
        unpack_side(__byte_perm(z0, 0u, sel8) ^ 0x00880088u, a[0], dummy);
        unpack_side(__byte_perm(z1, 0u, sel8) ^ 0x00880088u, a[1], dummy);
        a[2] = a[3] = 0u;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_f16(acc[NG][nt], a, bz[nt]);
      zs0 = reinterpret_cast<const float*>(st + L::kZs)[j0];
      zs1 = reinterpret_cast<const float*>(st + L::kZs)[j1];
    }
    float ks0[NG], km0[NG], ks1[NG], km1[NG];
#pragma unroll
    for (int gg = 0; gg < (KCH ? 0 : NG); ++gg) {
      ks0[gg] = reinterpret_cast<const float*>(st + L::kKs)[j0 * NG + gg];
      km0[gg] = reinterpret_cast<const float*>(st + L::kKm)[j0 * NG + gg];
      ks1[gg] = reinterpret_cast<const float*>(st + L::kKs)[j1 * NG + gg];
      km1[gg] = reinterpret_cast<const float*>(st + L::kKm)[j1 * NG + gg];
    }

    // ---- logits, online softmax, p in the B-operand layout
    uint32_t bp[NT][2];
    const int pb = i & 1;  // 2-bit values: the exchange buffer of this tile
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float s0 = 0.f, s1 = 0.f;
      float x0, x1;
      if constexpr (KCH) {  // q . k^ = q . min + sum_c (q scale)_c code_c, in true units
        float c0 = 0.f, c1 = 0.f;
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) {
          c0 += acc[gg][nt][0] + acc[gg][nt][1];
          c1 += acc[gg][nt][2] + acc[gg][nt][3];
        }
        s0 = fmaf(c0, kfinv[nt], kqmin[nt]);
        s1 = fmaf(c1, kfinv[nt], kqmin[nt]);
        if constexpr (R > 0) {  // the side term is in units of the head's prescale
          s0 = fmaf(zs0 * foinv[nt], acc[NG][nt][0] + acc[NG][nt][1], s0);
          s1 = fmaf(zs1 * foinv[nt], acc[NG][nt][2] + acc[NG][nt][3], s1);
        }
        x0 = val0 ? s0 * (p.sm_scale * kLog2e) : -INFINITY;
        x1 = val1 ? s1 * (p.sm_scale * kLog2e) : -INFINITY;
      } else {
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) {
          s0 = fmaf(ks0[gg], acc[gg][nt][0] + acc[gg][nt][1], s0);
          s0 = fmaf(km0[gg], qsum[nt][gg], s0);
          s1 = fmaf(ks1[gg], acc[gg][nt][2] + acc[gg][nt][3], s1);
          s1 = fmaf(km1[gg], qsum[nt][gg], s1);
        }
        if constexpr (R > 0) {
          s0 = fmaf(zs0, acc[NG][nt][0] + acc[NG][nt][1], s0);
          s1 = fmaf(zs1, acc[NG][nt][2] + acc[NG][nt][3], s1);
        }
        x0 = val0 ? s0 * scale2[nt] : -INFINITY;
        x1 = val1 ? s1 * scale2[nt] : -INFINITY;
      }
      float mx = fmaxf(x0, x1);
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      const float mnew = fmaxf(m2[nt], mx);
      const bool resc = mnew > m2[nt] + kRescale;
      if (__any_sync(kFull, resc)) {
        const float alpha = resc ? exp2f(m2[nt] - mnew) : 1.0f;
        if (resc) m2[nt] = mnew;
        l[nt] *= alpha;
        if constexpr (V2) {  // the readout rescales to the warps' common maximum itself
#pragma unroll
          for (int gg = 0; gg < NG; ++gg) vmin_acc[nt][gg] *= alpha;
        } else {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            o[mt][nt][0] *= alpha; o[mt][nt][1] *= alpha;
            o[mt][nt][2] *= alpha; o[mt][nt][3] *= alpha;
          }
        }
      }
      const float p0 = x0 == -INFINITY ? 0.f : exp2f(x0 - m2[nt]);
      const float p1 = x1 == -INFINITY ? 0.f : exp2f(x1 - m2[nt]);
      l[nt] += p0 + p1;
      if constexpr (V2) {
        // p and this warp's maximum to the readout warps
        float* pw = pex_s + ((pb * kCW + warp) * 8 + 4 * nt + t) * 24;
        pw[g] = p0;
        pw[g + 8] = p1;
        if (g == 0) mex_s[(pb * 8 + 4 * nt + t) * kCW + warp] = m2[nt];
        // the running sum of p_j * min_{j,g} (masked tokens add nothing)
        const float* vm = reinterpret_cast<const float*>(st + L::kVm);
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) {
          if (p0 > 0.f) vmin_acc[nt][gg] = fmaf(p0, vm[j0 * NG + gg], vmin_acc[nt][gg]);
          if (p1 > 0.f) vmin_acc[nt][gg] = fmaf(p1, vm[j1 * NG + gg], vmin_acc[nt][gg]);
        }
      } else {
        // B operand of p . V: (tokens 2t, 2t+1 | 2t+8, 2t+9) x column g
        const int sa = 8 * t + (g >> 1), sb = sa + 4;
        const float va = __shfl_sync(kFull, p0, sa), vb = __shfl_sync(kFull, p0, sb);
        const float vc = __shfl_sync(kFull, p1, sa), vd = __shfl_sync(kFull, p1, sb);
        bp[nt][0] = bf16_part_pair(va, vb, g & 1);
        bp[nt][1] = bf16_part_pair(vc, vd, g & 1);
      }
    }

    // ---- 2-bit values: the readout of this warp's channel slice over the
    // kTile tokens.  Column g of the B operand is head slot g; its entries for
    // the tokens 16 kb + {2t, 2t+1 | 2t+8, 2t+9} are p_j * scale_{j,gw} of logit
    // warp kb, brought to the common reference Mref (factor 2^(m_kb - Mref), m_kb
    // that warp's running maximum) and to 2^-E, E the running exponent of
    // (head slot, slice): raised, with that column of ov rescaled by the exact
    // power of two, as soon as an entry reaches 2^kRaiseLog2 * 2^E, so the fp16
    // operand never overflows and entries within 2^-14 of 2^E keep the full
    // 11-bit mantissa.  p <= 2^8 (the lazy rescale); the codes are exact in fp16.
    if constexpr (V2) {
      __syncwarp();
      const uint32_t xbar = smem_addr(&bars[2 * kStages + 2 + pb]);
      if (lane == 0) mbar_arrive(xbar);
      if (!mbar_wait(xbar, (i >> 1) & 1)) {
        ok = false;
        break;
      }
      const bool hv = g < GM;  // head slot g exists
      float mw[kCW];
      {
        const float4 m4 = *reinterpret_cast<const float4*>(mex_s + (pb * 8 + g) * kCW);
        mw[0] = hv ? m4.x : -INFINITY;
        mw[1] = hv ? m4.y : -INFINITY;
        mw[2] = hv ? m4.z : -INFINITY;
        mw[3] = hv ? m4.w : -INFINITY;
      }
      float Mn = Mref;
#pragma unroll
      for (int kb = 0; kb < kCW; ++kb) Mn = fmaxf(Mn, mw[kb]);
      float rfac = 1.0f;  // factor of the ov column of head slot g
      if (Mn > Mref) {
        rfac = exp2f(Mref - Mn);
        Mref = Mn;
      }
      float fk[kCW];
#pragma unroll
      for (int kb = 0; kb < kCW; ++kb) fk[kb] = mw[kb] == -INFINITY ? 0.f : exp2f(mw[kb] - Mref);
      const float* vs = reinterpret_cast<const float*>(st + L::kVs);
      float wq[kCW][4];
      float hx = 0.f;
#pragma unroll
      for (int kb = 0; kb < kCW; ++kb) {
        const float* pr = pex_s + ((pb * kCW + kb) * 8 + g) * 24 + 2 * t;
        const float2 pa = hv ? *reinterpret_cast<const float2*>(pr) : make_float2(0.f, 0.f);
        const float2 pc = hv ? *reinterpret_cast<const float2*>(pr + 8) : make_float2(0.f, 0.f);
        const int ja = 16 * kb + 2 * t;
        // masked tokens have p = 0 and may have no scale in the stage
        wq[kb][0] = pa.x > 0.f ? pa.x * vs[ja * NG + gw] : 0.f;
        wq[kb][1] = pa.y > 0.f ? pa.y * vs[(ja + 1) * NG + gw] : 0.f;
        wq[kb][2] = pc.x > 0.f ? pc.x * vs[(ja + 8) * NG + gw] : 0.f;
        wq[kb][3] = pc.y > 0.f ? pc.y * vs[(ja + 9) * NG + gw] : 0.f;
        hx = fmaxf(hx, fk[kb] * fmaxf(fmaxf(wq[kb][0], wq[kb][1]), fmaxf(wq[kb][2], wq[kb][3])));
      }
      // the largest entry of head slot g (its four lanes; non-negative floats
      // order like their bit patterns)
      hx = fmaxf(hx, __shfl_xor_sync(kFull, hx, 1));
      hx = fmaxf(hx, __shfl_xor_sync(kFull, hx, 2));
      const uint32_t mxb = __float_as_uint(hx);
      if (mxb >= static_cast<uint32_t>(127 + ve + kRaiseLog2) << 23) {
        const int en = max(-126, min(126, static_cast<int>(mxb >> 23) - 127));
        rfac *= pow2_neg(-ve) * pow2_neg(en);  // 2^(E_old - E_new)
        ve = en;
      }
      if (__any_sync(kFull, rfac != 1.0f)) {
        // the output columns are head slots 2t, 2t+1: their factors live in
        // lanes 8t and 8t + 4
        const float r0 = __shfl_sync(kFull, rfac, 8 * t), r1 = __shfl_sync(kFull, rfac, 8 * t + 4);
#pragma unroll
        for (int mt = 0; mt < MTW; ++mt) {
          ov[mt][0] *= r0; ov[mt][1] *= r1; ov[mt][2] *= r0; ov[mt][3] *= r1;
        }
      }
      const float fE = pow2_neg(ve);
      uint32_t bpf[kCW][2];
#pragma unroll
      for (int kb = 0; kb < kCW; ++kb) {
        const float c = fk[kb] * fE;
        const __half2 h0 = __floats2half2_rn(wq[kb][0] * c, wq[kb][1] * c);
        const __half2 h1 = __floats2half2_rn(wq[kb][2] * c, wq[kb][3] * c);
        bpf[kb][0] = *reinterpret_cast<const uint32_t*>(&h0);
        bpf[kb][1] = *reinterpret_cast<const uint32_t*>(&h1);
      }
      // p . V on tensor cores: A = V^T of the slice from the code tile
      const uint32_t cbase = smem_addr(ctile);
      const int lr = 8 * (lane >> 4) + (lane & 7);  // ldmatrix row of this lane in a k-step
#pragma unroll
      for (int kb = 0; kb < kCW; ++kb) {
        const int r = 16 * kb + lr;
        const int sz = (r / (8 / CPR)) % CPR;
#pragma unroll
        for (int mt = 0; mt < MTW; ++mt) {
          const int chunk = 2 * mt + lm_chunk_hi;
          uint32_t a[4];
          ldsm_x4_trans(cbase + r * (CW * 2) + ((chunk ^ sz) << 4), a);
          mma_f16(ov[mt], a, bpf[kb]);
        }
      }
    } else {
      // ---- p . V on tensor cores (A = V^T from the swizzled tile)
      const uint32_t vbase = smem_addr(st);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int chunk = 2 * mt + lm_chunk_hi;
        const uint32_t addr = vbase + (chunk >> 3) * L::kVBox + lm_tok * 128 +
                              (((chunk & 7) ^ (lm_tok & 7)) << 4);
        uint32_t a[4];
        ldsm_x4_trans(addr, a);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16(o[mt][nt], a, bp[nt]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&bars[kStages + s]));
  }
  if (!ok && lane == 0 && p.err) atomicOr(p.err, kDevErrWaitTimeout);

  // ---- merge the consumer warps' partial softmax states
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    l[nt] += __shfl_xor_sync(kFull, l[nt], 4);
    l[nt] += __shfl_xor_sync(kFull, l[nt], 8);
    l[nt] += __shfl_xor_sync(kFull, l[nt], 16);
    if constexpr (V2) {
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        vmin_acc[nt][gg] += __shfl_xor_sync(kFull, vmin_acc[nt][gg], 4);
        vmin_acc[nt][gg] += __shfl_xor_sync(kFull, vmin_acc[nt][gg], 8);
        vmin_acc[nt][gg] += __shfl_xor_sync(kFull, vmin_acc[nt][gg], 16);
      }
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  float* mo = reinterpret_cast<float*>(stages);  // [kCW][GM][D] ([GM][D] for 2-bit values)
  float* mm = mo + kCW * GM * D;                 // [kCW][GM]
  float* ml = mm + kCW * GM;                     // [kCW][GM]
  float* vms = ml + kCW * GM;                    // [kCW][GM][NG] (2-bit values) sum p min
  int* flags = reinterpret_cast<int*>(vms + (V2 ? kCW * GM * NG : 0));  // [0] a warp failed, [1] last CTA
  if (tid == 0) flags[0] = 0;
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  if (!ok) flags[0] = 1;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = 4 * nt + t;
    if constexpr (!V2) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        mo[(warp * GM + h) * D + 16 * mt + g] = o[mt][nt][0] + o[mt][nt][1];
        mo[(warp * GM + h) * D + 16 * mt + g + 8] = o[mt][nt][2] + o[mt][nt][3];
      }
    }
    if (g == 0) {
      mm[warp * GM + h] = m2[nt];
      ml[warp * GM + h] = l[nt];
      if constexpr (V2) {
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) vms[(warp * GM + h) * NG + gg] = vmin_acc[nt][gg];
      }
    }
  }
  if constexpr (V2) {
    // this warp's channel slice, columns = head slots 2t, 2t+1: back from units
    // of 2^ve of each column's head slot (held by lanes 8t, 8t + 4); relative to
    // Mref, the largest of the warps' final maxima
    const float u = pow2_neg(-ve);
    const float ue[2] = {__shfl_sync(kFull, u, 8 * t), __shfl_sync(kFull, u, 8 * t + 4)};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * t + e;
      if (h < GM) {
#pragma unroll
        for (int mt = 0; mt < MTW; ++mt) {
          mo[h * D + cw0 + 16 * mt + g] = ov[mt][e] * ue[e];
          mo[h * D + cw0 + 16 * mt + g + 8] = ov[mt][2 + e] * ue[e];
        }
      }
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  const bool failed = flags[0] != 0;
  const bool single = p.splits == 1;
  if (failed && single) return;
  const PartView pv = part_view(p.part, static_cast<size_t>(p.c.B) * p.Hq, p.splits, D);
  for (int idx = tid; idx < G * D; idx += kCT) {
    const int h = idx / D, c = idx - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCW; ++w) M = fmaxf(M, mm[w * GM + h]);
    float O = 0.f, Ls = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < kCW; ++w) {
        const float f = exp2f(mm[w * GM + h] - M);
        if constexpr (V2)  // sum_j p_j min_{j,g}
          O = fmaf(f, vms[(w * GM + h) * NG + c / 32], O);
        else
          O = fmaf(f, mo[(w * GM + h) * D + c], O);
        Ls = fmaf(f, ml[w * GM + h], Ls);
      }
      if constexpr (V2) O += mo[h * D + c];  // sum_j p_j scale_{j,g} code_{j,c}, relative to M
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
  merge_splits_last<D>(p, b, h0, reinterpret_cast<float*>(flags + 4), warp, kCW, lane);
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
  if (tid == 0) p.counters[bk] = 0;  // ready for the next call
}

// ---------------------------------------------------------------- host side
constexpr int kMaxDev = 64;

template <int D, int R, int NT, bool V2, bool KCH>
struct Variant {
  static int occupancy[kMaxDev];  // CTAs per SM, 0 = not yet known
  static std::mutex mu;

  // Once per device: raise the dynamic shared memory limit and ask the
  // occupancy calculator how many CTAs fit on one SM.
  static int ctas_per_sm() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
      cudaGetLastError();
      return 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (occupancy[dev] == 0) {
      auto k = decode_mma_kernel<D, R, NT, V2, KCH>;
      const int smem = static_cast<int>(smem_bytes<D, R, NT, V2, KCH>());
      int n = 0;
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
              cudaSuccess ||
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kThreads, smem) != cudaSuccess) {
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
    dim3 grid(p.splits, p.c.Hkv, p.c.B);
    if (V2) {  // no value tensor map: the 2-bit value planes are bulk-copied
      memset(&vmap, 0, sizeof(vmap));
      decode_mma_kernel<D, R, NT, V2, KCH><<<grid, kThreads, smem_bytes<D, R, NT, V2, KCH>(), s>>>(p, vmap);
      return cudaGetLastError();
    }
    if (!tensor_maps_available()) return cudaErrorNotSupported;
    // [slab][row in slab][channel]: one slab per (b, kv), or per (page, kv)
    const bool paged = p.c.page_size > 0;
    const uint64_t rows = static_cast<uint64_t>(paged ? p.c.page_size : p.c.T_cap);
    const uint64_t slabs = static_cast<uint64_t>(paged ? p.c.num_pages : p.c.B) * p.c.Hkv;
    if (!encode_bf16_rows(&vmap, p.c.v, D, rows, slabs, kTile)) return cudaErrorInvalidValue;
    decode_mma_kernel<D, R, NT, V2, KCH><<<grid, kThreads, smem_bytes<D, R, NT, V2, KCH>(), s>>>(p, vmap);
    return cudaGetLastError();
  }
};
template <int D, int R, int NT, bool V2, bool KCH>
int Variant<D, R, NT, V2, KCH>::occupancy[kMaxDev];
template <int D, int R, int NT, bool V2, bool KCH>
std::mutex Variant<D, R, NT, V2, KCH>::mu;

template <typename F>
auto dispatch(int d, int r, int G, bool v2, bool kch, F&& f)
    -> decltype(f(Variant<128, 16, 1, false, false>{})) {
  const int nt = G <= 4 ? 1 : 2;
#define HEADQ_MMA_CASE(DD, RR, NN, VV, KK) \
  if (d == DD && r == RR && nt == NN && v2 == VV && kch == KK) \
    return f(Variant<DD, RR, NN, VV, KK>{});
// per-token keys with G > 4 run in decode_hm.cu: only one N-tile here
#define HEADQ_MMA_CASES_NT(NN, KK)                                               \
  HEADQ_MMA_CASE(128, 16, NN, false, KK) HEADQ_MMA_CASE(128, 8, NN, false, KK)   \
  HEADQ_MMA_CASE(128, 0, NN, false, KK) HEADQ_MMA_CASE(64, 16, NN, false, KK)    \
  HEADQ_MMA_CASE(64, 8, NN, false, KK) HEADQ_MMA_CASE(64, 0, NN, false, KK)      \
  HEADQ_MMA_CASE(128, 16, NN, true, KK) HEADQ_MMA_CASE(128, 8, NN, true, KK)     \
  HEADQ_MMA_CASE(64, 16, NN, true, KK) HEADQ_MMA_CASE(64, 8, NN, true, KK)
  HEADQ_MMA_CASES_NT(1, false)
  HEADQ_MMA_CASES_NT(1, true)
  HEADQ_MMA_CASES_NT(2, true)
#undef HEADQ_MMA_CASES_NT
#undef HEADQ_MMA_CASE
  return decltype(f(Variant<128, 16, 1, false, false>{}))();
}

bool is_v2(const headq_cache& c) { return c.vmode == HEADQ_V_2BIT; }

}  // namespace

bool mma_decode_supported(const headq_cache& c, int G) {
  if (c.d != 64 && c.d != 128) return false;
  if (c.kmode != HEADQ_K_TOKEN && c.kmode != HEADQ_K_CHANNEL) return false;
  if (G < 1 || G > 8) return false;
  if (c.vmode == HEADQ_V_2BIT) return c.r == 8 || c.r == 16;
  return c.vmode == HEADQ_V_DENSE && c.v_dtype == HEADQ_BF16 &&
         (c.r == 0 || c.r == 8 || c.r == 16) && tensor_maps_available();
}

int mma_decode_ctas_per_sm(const headq_cache& c, int G) {
  if (hm_decode_supported(c, G)) return hm_decode_ctas_per_sm(c);
  return dispatch(c.d, c.r, G, is_v2(c), c.kmode == HEADQ_K_CHANNEL,
                  [](auto v) { return decltype(v)::ctas_per_sm(); });
}

cudaError_t launch_decode_mma(const DecodeParams& p, cudaStream_t s) {
  if (hm_decode_supported(p.c, p.G)) return launch_decode_hm(p, s);
  // 0 means no variant matched; otherwise the launch status + 1
  const int e = dispatch(p.c.d, p.c.r, p.G, is_v2(p.c), p.c.kmode == HEADQ_K_CHANNEL, [&](auto v) {
    return static_cast<int>(decltype(v)::launch(p, s)) + 1;
  });
  return e == 0 ? cudaErrorInvalidValue : static_cast<cudaError_t>(e - 1);
}

}  // namespace headq
