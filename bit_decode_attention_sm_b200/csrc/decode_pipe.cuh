// The streaming skeleton shared by the tensor-core decode kernels (decode_mma.cu,
// decode_hm.cu): the shared-memory stage of 64 tokens, the producer warp that
// fills the stages with bulk / tensor copies of the packed cache planes (and
// encodes the appended token first, when the call appends one), and the merge
// of a (b, kv)'s T-splits by the last CTA to finish ("HeadQ: Model-Visible
// Distortion and Score-Space Correction for KV-Cache Quantization", gist.science
// summary, section 3, step 3: the decode reads the stored base code, side code
// and values of every cached token).
#pragma once

#include "decode_common.cuh"

namespace headq {
namespace dc {

constexpr int kPipeTile = 64;  // tokens per stage

// Shared-memory stage of kPipeTile tokens.  Dense bf16 values (V2 = false): the
// swizzled value boxes come first (64 tokens x 64 dims x bf16 each).  2-bit
// values (V2 = true): their code, scale and minimum planes are bulk-copied like
// the keys'.  Per-channel keys (KCH): the tile is one 64-token block, whose scale
// and minimum rows (d floats each) take the place of the per-token key scale and
// minimum planes.
template <int D, int R, bool V2 = false, bool KCH = false>
struct StageLayout {
  static constexpr int kTile = kPipeTile;
  static constexpr int NG = D / 32;
  static constexpr int kVBoxes = V2 ? 0 : D / 64;    // 64-dim boxes per token row
  static constexpr int kVBox = kTile * 128;          // 64 tokens x 128 bytes
  static constexpr int kKc = kVBoxes * kVBox;
  static constexpr int kKs = kKc + kTile * (D / 4);
  static constexpr int kKm = kKs + kTile * NG * 4;
  static constexpr int kZc = kKm + kTile * NG * 4;
  static constexpr int kZs = kZc + kTile * (R / 2);
  static constexpr int kVc = kZs + (R > 0 ? kTile * 4 : 0);
  static constexpr int kVs = kVc + (V2 ? kTile * (D / 4) : 0);
  static constexpr int kVm = kVs + (V2 ? kTile * NG * 4 : 0);
  static constexpr int kEnd = kVm + (V2 ? kTile * NG * 4 : 0);
  static constexpr int kStage = (kEnd + 1023) / 1024 * 1024;
  static constexpr int kRowBytes =
      D / 4 + (KCH ? 0 : 8 * NG) + (R > 0 ? R / 2 + 4 : 0) + (V2 ? D / 4 + 8 * NG : 0);
  static constexpr int kTileBytes = KCH ? 2 * D * 4 : 0;  // bytes per tile, besides the rows
  static_assert(!KCH || D * 4 <= kTile * NG * 4, "a block row fits the per-token plane space");
};

// The producer warp of a decode CTA.  Bulk-copies the query of the CTA's G
// heads (into qraw_s) and U_h (into u_s, when R > 0) behind barrier qbar,
// then the tiles of [t_begin, tile_end) in order, one per stage, each behind
// its stage's full barrier; then an end marker (stile_s[s] = -1).  A stage is
// reused once its empty barrier completes (the consumers' arrivals).  When the
// call appends (pos inside the chunk), the warp encodes the new token once the
// first stages are in flight, or before the tile holding it if that comes
// sooner, and publishes it to the copies (async proxy) before that tile is
// issued; the encoder reads U_h from u_s (after qbar) when kEncSmemU, else from
// global memory (a kernel that reuses u_s once its main loop starts).  Every
// wait is bounded; on expiry the error word is flagged and the warp stops
// issuing, and it never leaves with copies in flight.
template <int D, int R, bool V2, bool KCH, int kStages, bool kEncSmemU>
__device__ __forceinline__ void produce_tiles(const DecodeParams& p, const CUtensorMap* vmap,
                                              uint8_t* stages, uint64_t* full_bars,
                                              uint64_t* empty_bars, uint64_t* qbar_p,
                                              int* stile_s, float* qraw_s, float* u_s,
                                              float* enew_s, int b, int kv, int h0,
                                              int t_begin, int tile_end, int ntiles, int pos,
                                              int lane) {
  using L = StageLayout<D, R, V2, KCH>;
  constexpr int NG = L::NG;
  constexpr int kTile = L::kTile;
  const int G = p.G;
  const uint32_t qbar = smem_addr(qbar_p);
  if (lane == 0) {
    // the query and U_h first: they head the copy queue, so the consumers'
    // preparation does not wait behind the cache stream
    const uint32_t qbytes = static_cast<uint32_t>(G * D * (p.q_bf16 ? 2 : 4));
    mbar_expect_tx(qbar, qbytes + (R > 0 ? D * R * 4 : 0));
    bulk_g2s(smem_addr(qraw_s),
             static_cast<const uint8_t*>(p.q) +
                 (static_cast<size_t>(b) * p.Hq + h0) * D * (p.q_bf16 ? 2 : 4),
             qbytes, qbar);
    if (R > 0)
      bulk_g2s(smem_addr(u_s), p.U + static_cast<size_t>(kv) * D * R, D * R * 4, qbar);
  }
  bool ok = true;
  int issued = 0;
  const int enc_i =
      (pos >= t_begin && pos < tile_end) ? min((pos - t_begin) / kTile, kStages) : -1;
  for (int i = 0;; ++i) {
    const int s = i % kStages, use = i / kStages;
    if (i == enc_i) {
      if (kEncSmemU && !mbar_wait(qbar, 0) && lane == 0 && p.err)
        atomicOr(p.err, kDevErrWaitTimeout);
      encode_new_token<D, R, V2>(p, b, kv, pos,
                                 kEncSmemU ? u_s : p.U + static_cast<size_t>(kv) * D * R,
                                 enew_s, lane);
      // publish the token's planes to the bulk copies (async proxy): every
      // lane's writes, then the issuing lane
      __threadfence();
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __syncwarp();
      if (lane == 0) asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    int t0 = -1;
    if (lane == 0) {
      if (use > 0 && !mbar_wait(smem_addr(&empty_bars[s]), (use - 1) & 1)) ok = false;
      if (ok && i < ntiles) t0 = t_begin + i * kTile;
    }
    ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    t0 = __shfl_sync(kFull, t0, 0);
    if (!ok) break;
    if (lane == 0) {
      stile_s[s] = t0;
      const uint32_t full = smem_addr(&full_bars[s]);
      if (t0 < 0) {
        mbar_arrive(full);  // no more tiles: the consumers stop at this stage
      } else {
        const int n16 = (min(kTile, tile_end - t0) + 15) & ~15;
        mbar_expect_tx(full, L::kVBoxes * L::kVBox + n16 * L::kRowBytes + L::kTileBytes);
        uint8_t* st = stages + size_t(s) * L::kStage;
        const CacheSlab sl = cache_slab_read(p.c, b, kv, t0, p.err);
        const size_t row0 = static_cast<size_t>(sl.slab) * slab_rows(p.c) + sl.off;
        bulk_g2s(smem_addr(st + L::kKc), p.c.k_codes + row0 * (D / 4), n16 * (D / 4), full);
        if constexpr (KCH) {  // the tile is one block: its scale and minimum rows
          const size_t brow = row0 / kTile;
          bulk_g2s(smem_addr(st + L::kKs), p.c.k_scale + brow * D, D * 4, full);
          bulk_g2s(smem_addr(st + L::kKm), p.c.k_min + brow * D, D * 4, full);
        } else {
          bulk_g2s(smem_addr(st + L::kKs), p.c.k_scale + row0 * NG, n16 * NG * 4, full);
          bulk_g2s(smem_addr(st + L::kKm), p.c.k_min + row0 * NG, n16 * NG * 4, full);
        }
        if constexpr (R > 0) {
          bulk_g2s(smem_addr(st + L::kZc), p.c.z_codes + row0 * (R / 2), n16 * (R / 2), full);
          bulk_g2s(smem_addr(st + L::kZs), p.c.z_scale + row0, n16 * 4, full);
        }
        if constexpr (V2) {
          bulk_g2s(smem_addr(st + L::kVc), p.c.v_codes + row0 * (D / 4), n16 * (D / 4), full);
          bulk_g2s(smem_addr(st + L::kVs), p.c.v_scale + row0 * NG, n16 * NG * 4, full);
          bulk_g2s(smem_addr(st + L::kVm), p.c.v_min + row0 * NG, n16 * NG * 4, full);
        } else {
#pragma unroll
          for (int bx = 0; bx < L::kVBoxes; ++bx)
            tma_3d(smem_addr(st + bx * L::kVBox), vmap, bx * 64, sl.off,
                   static_cast<int>(sl.slab), full);
        }
      }
      ++issued;
    }
    if (t0 < 0) break;
  }
  if (lane == 0) {
    if (!ok && p.err) atomicOr(p.err, kDevErrWaitTimeout);
    // never leave with copies in flight: wait (bounded) for the last use of each stage
    for (int s = 0; s < kStages && s < issued; ++s) {
      const int last_use = (issued - 1 - s) / kStages;
      mbar_wait(smem_addr(&full_bars[s]), last_use & 1);
    }
  }
}

// The last CTA of a (b, kv) merges all p.splits partials of its G heads into
// the output (log-sum-exp combine), one warp per head (warps 0..nwarps-1), no
// CTA barrier, few round trips to L2: the first round issues the (m, l) of the
// splits (lane-strided) together with the partial outputs of the first kMR
// splits (lane = 4 output dims); while those are in flight the warp reduces
// the maximum and writes the split weights to w_s ([G][splits] floats of
// shared memory); further rounds load the remaining splits' outputs.
template <int D>
__device__ __forceinline__ void merge_splits_last(const DecodeParams& p, int b, int h0,
                                                  float* w_s, int warp, int nwarps, int lane) {
  const int S = p.splits, G = p.G;
  const PartView pv = part_view(p.part, static_cast<size_t>(p.c.B) * p.Hq, S, D);
  constexpr int kSPL = 4;   // splits per lane held in registers (S <= 128)
  constexpr int kMR = 16;   // splits per round of output loads
  for (int h = warp; h < G; h += nwarps) {
    const size_t bh = static_cast<size_t>(b) * p.Hq + h0 + h;
    const bool has_c4 = lane < D / 4;
    const float4* po = reinterpret_cast<const float4*>(pv.o + bh * S * D) + lane;
    float4 v[kMR];
#pragma unroll
    for (int u = 0; u < kMR; ++u)
      v[u] = (has_c4 && u < S) ? __ldcg(po + u * (D / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
    float mv[kSPL], lv[kSPL];
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < kSPL; ++k) {
      const int sI = lane + 32 * k;
      mv[k] = -INFINITY;
      lv[k] = 0.f;
      if (sI < S) {
        mv[k] = __ldcg(pv.m + bh * S + sI);
        lv[k] = __ldcg(pv.l + bh * S + sI);
      }
      mx = fmaxf(mx, mv[k]);
    }
    for (int sI = lane + 32 * kSPL; sI < S; sI += 32) mx = fmaxf(mx, __ldcg(pv.m + bh * S + sI));
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o2));
    float ls = 0.f;
    float* w = w_s + h * S;
#pragma unroll
    for (int k = 0; k < kSPL; ++k) {
      const int sI = lane + 32 * k;
      if (sI < S) {
        const float wk = mv[k] > -INFINITY ? expf(mv[k] - mx) : 0.f;
        w[sI] = wk;
        ls = fmaf(wk, lv[k], ls);
      }
    }
    for (int sI = lane + 32 * kSPL; sI < S; sI += 32) {
      const float m = __ldcg(pv.m + bh * S + sI);
      const float wk = m > -INFINITY ? expf(m - mx) : 0.f;
      w[sI] = wk;
      ls = fmaf(wk, __ldcg(pv.l + bh * S + sI), ls);
    }
    for (int o2 = 16; o2 > 0; o2 >>= 1) ls += __shfl_xor_sync(kFull, ls, o2);
    __syncwarp();
    float4 acc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0;;) {
#pragma unroll
      for (int u = 0; u < kMR; ++u) {
        const float wu = s0 + u < S ? w[s0 + u] : 0.f;
        float4& a4 = acc[u & 3];
        a4.x = fmaf(wu, v[u].x, a4.x); a4.y = fmaf(wu, v[u].y, a4.y);
        a4.z = fmaf(wu, v[u].z, a4.z); a4.w = fmaf(wu, v[u].w, a4.w);
      }
      s0 += kMR;
      if (s0 >= S) break;
#pragma unroll
      for (int u = 0; u < kMR; ++u)
        v[u] = (has_c4 && s0 + u < S) ? __ldcg(po + (s0 + u) * (D / 4))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float inv = ls > 0.f ? 1.0f / ls : 0.f;
    if (has_c4) {
      float4 r;
      r.x = ((acc[0].x + acc[1].x) + (acc[2].x + acc[3].x)) * inv;
      r.y = ((acc[0].y + acc[1].y) + (acc[2].y + acc[3].y)) * inv;
      r.z = ((acc[0].z + acc[1].z) + (acc[2].z + acc[3].z)) * inv;
      r.w = ((acc[0].w + acc[1].w) + (acc[2].w + acc[3].w)) * inv;
      reinterpret_cast<float4*>(p.out + bh * D)[lane] = r;
    }
    if (lane == 0 && p.lse) p.lse[bh] = ls > 0.f ? mx + logf(ls) : -INFINITY;
  }
}

}  // namespace dc
}  // namespace headq
