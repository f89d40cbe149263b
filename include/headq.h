/*
 * headq.h -- C ABI of libheadq, HeadQ decode attention for NVIDIA B200 (sm_100a).
 *
 * HeadQ ("HeadQ: Model-Visible Distortion and Score-Space Correction for
 * KV-Cache Quantization"; arXiv abstract and the gist.science technical summary,
 * section 3 "Methodology: HeadQ") stores every cached key as
 *   - a 2-bit base code  k^base_j = B_b(k_j)                    (section 3, step 2)
 *   - a low-rank side code z_j = Q_q(U_h^T (k_j - k^base_j))     (section 3, step 2)
 * in a rank-r basis U_h learned from post-RoPE calibration queries (step 1), and
 * reads it with an additive logit correction                     (section 3, step 3)
 *   s^_j = q^T k^base_j / sqrt(d) + q^T U_h z^_j / sqrt(d),
 * followed by softmax and the attention-weighted value readout.  Section 2 of the
 * summary defines the diagnostics (attention KL, the Fisher-weighted score-error
 * variance, the A^2-weighted value distortion) that headq_attn_kl computes.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers, allocated and owned by the caller;
 *     the library allocates no memory and keeps no state between calls.
 *   - Work is enqueued asynchronously on `stream`; results are valid once the
 *     stream has reached that point.  Argument errors are detected on the host,
 *     before anything is launched, and returned synchronously.
 *   - Every pointer must be 16-byte aligned.  Layouts are dense, row-major, with
 *     the last index fastest.
 *   - Shapes: d is 8, 16, 32, 64, 128 or 256; the base code works on groups of
 *     32 channels (group = d when d < 32); r is even with 0 <= r <= min(d, 32);
 *     Hq is a multiple of Hkv and query head h reads KV head h / (Hq / Hkv);
 *     T_cap (the cache capacity in tokens) is a multiple of 16.
 *   - Codec bit layout: channel c of a 2-bit code is bits 2*(c%4)..2*(c%4)+1 of
 *     byte c/4; side-code entry i is a 4-bit two's-complement nibble in byte i/2
 *     (even i in the low nibble).  Scales and minima are IEEE fp32.
 *   - Exact codec arithmetic (bit-reproducible): for each token and group of 32
 *     channels, mn = min x, mx = max x (a -0 extreme stored as +0),
 *     scale = (mx - mn) / 3, code = clamp(rint((x - mn) / scale), 0, 3) with
 *     round-half-even (all codes 0 when scale == 0); the residual is
 *     e = x - (mn + code*scale) (product rounded first); the projection
 *     y = U_h^T e accumulates channel by channel in order with one fused
 *     multiply-add per term; the side scale is s = max|y| / 7 and the side code
 *     w = clamp(rint(y / s), -7, 7) (all 0 when s == 0).  Every operation is one
 *     IEEE fp32 operation (division correctly rounded, no flush-to-zero).
 */
#ifndef HEADQ_H
#define HEADQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *headq_stream_t;

typedef enum {
    HEADQ_OK = 0,
    HEADQ_ERR_INVALID_ARG = 1, /* null/misaligned pointer, inconsistent sizes    */
    HEADQ_ERR_UNSUPPORTED = 2, /* valid request outside the supported shapes     */
    HEADQ_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required     */
    HEADQ_ERR_CUDA = 4,        /* a CUDA call or kernel launch failed            */
    HEADQ_ERR_DEVICE = 5       /* a kernel flagged a device-side error (timeout) */
} headq_status;

typedef enum { HEADQ_F32 = 0, HEADQ_BF16 = 1 } headq_dtype;

/* The base code of the keys (B_b of summary section 3, step 2). */
typedef enum {
    HEADQ_K_TOKEN = 0,   /* per token, per group of 32 channels (the pages' reading) */
    HEADQ_K_CHANNEL = 1  /* per channel, per block of 64 tokens (KIVI-style keys)   */
} headq_kmode;

typedef enum {
    HEADQ_V_DENSE = 0, /* V stored as v_dtype, [B, Hkv, T_cap, d]               */
    HEADQ_V_2BIT = 1   /* V stored with the 2-bit base code of the keys, no side */
} headq_vmode;

/*
 * The packed HeadQ cache: structure-of-arrays planes in HBM, each indexed
 * [b][kv][t] with t < T_cap (contiguous layout, page_size == 0; the paged
 * layout is described below).  Planes (NG = d / min(32, d) groups per token):
 *   k_codes  uint8 [B, Hkv, T_cap, d/4]   2-bit base key code
 *   k_scale  fp32  [B, Hkv, T_cap, NG]    base-code scale per group
 *   k_min    fp32  [B, Hkv, T_cap, NG]    base-code minimum per group
 *   z_codes  uint8 [B, Hkv, T_cap, r/2]   4-bit side code (unused when r == 0)
 *   z_scale  fp32  [B, Hkv, T_cap]        side-code scale
 *   v        v_dtype [B, Hkv, T_cap, d]   dense values   (vmode DENSE)
 *   v_codes/v_scale/v_min as k_codes/k_scale/k_min        (vmode 2BIT)
 * Pointers of planes the mode does not use may be NULL.
 *
 * Paged layout (page_size > 0), for serving loops that hand out cache memory in
 * fixed pages.  Every plane is a pool of num_pages pages, indexed
 * [page][kv][t % page_size] in place of [b][kv][t]:
 *   k_codes  uint8 [num_pages, Hkv, page_size, d/4]   (and so on for each plane)
 * block_table int32 [B, max_pages] (device) gives the pool page that holds
 * tokens [i*page_size, (i+1)*page_size) of sequence b at block_table[b*max_pages+i];
 * pages may be shared by no two (b, i) that are written.  page_size is a
 * multiple of 64 and T_cap == max_pages * page_size is the capacity of one
 * sequence.  Entries a call reaches must lie in [0, num_pages): a read of an
 * entry outside that range is redirected to page 0 and sets the device error
 * word (decode and diagnostic calls), a write to one is dropped.  With
 * page_size == 0 the page fields are ignored.
 *
 * Key base code (kmode).  HEADQ_K_TOKEN is the layout above.  HEADQ_K_CHANNEL
 * (an alternative base quantizer under the same side-code correction): each
 * channel of each block of 64 consecutive tokens has its own minimum and scale
 * (same arithmetic as the per-token code, taken along the block's tokens), so
 * k_scale and k_min hold one row of d floats per block: plane row p of a token
 * (b*Hkv + kv)*T_cap + t, or its paged row) has its block row at p / 64, i.e.
 *   k_scale, k_min  fp32 [B, Hkv, T_cap/64, d]  (paged: [num_pages, Hkv, page_size/64, d])
 * T_cap is a multiple of 64, writes start on a block boundary (t0 % 64 == 0)
 * and a block's codes are fixed once written (headq_decode_append and the A^2
 * fixup are unsupported in this mode).
 */
typedef struct {
    int B, Hkv, T_cap, d, r;
    headq_vmode vmode;
    headq_dtype v_dtype;
    uint8_t *k_codes;
    float *k_scale, *k_min;
    uint8_t *z_codes;
    float *z_scale;
    void *v;
    uint8_t *v_codes;
    float *v_scale, *v_min;
    int page_size;               /* 0: contiguous planes; else tokens per page   */
    int num_pages;               /* pages in each plane's pool (paged)           */
    int max_pages;               /* block_table entries per sequence (paged)     */
    const int32_t *block_table;  /* [B, max_pages] pool page of each logical page */
    headq_kmode kmode;           /* key base code, HEADQ_K_TOKEN by default       */
} headq_cache;

/* Library version as 10000*major + 100*minor + patch. */
int headq_version(void);

/* Static, human-readable text for a status code. */
const char *headq_status_string(headq_status s);

/*
 * headq_calibrate -- query-PCA basis U_h per KV head (summary section 3, step 1:
 * each layer and head gets a rank-r basis from a PCA of its post-RoPE
 * calibration queries).
 *   q_cal   [N, Hq, d] (dtype), calibration queries after RoPE.
 *   U_out   fp32 [Hkv, d, r]: U_out[(kv*d + c)*r + i] is entry c of basis vector i.
 *   eig_out fp32 [Hkv, r] (nullable): the matching eigenvalues, descending.
 * The basis is the top-r eigenvectors of the second moment (1/M) X^T X of the
 * M = N*G calibration queries of the G query heads that share KV head kv
 * (center != 0 subtracts their mean first), computed in fp64 by cyclic Jacobi
 * rotations; each column is signed so that its largest-magnitude entry is
 * positive (lowest index on a tie).
 *   ws: device workspace of at least headq_calibrate_workspace_bytes(...) bytes.
 * Requires 1 <= r <= d <= 128.
 */
headq_status headq_calibrate(const void *q_cal, headq_dtype dtype, int N, int Hq,
                             int Hkv, int d, int r, int center, float *U_out,
                             float *eig_out, void *ws, size_t ws_bytes,
                             headq_stream_t stream);
size_t headq_calibrate_workspace_bytes(int N, int Hq, int Hkv, int d);

/*
 * headq_cache_write -- encode n new tokens per (b, kv) into cache positions
 * [t0, t0 + n) (summary section 3, step 2: base code, residual, projection onto
 * U_h, side quantizer, store base code and side code).
 *   k, v  [B, Hkv, n, d] of kv_dtype.  k is encoded; v is copied (DENSE, rounded
 *         to nearest-even when the cache is bf16 and v is fp32) or encoded with
 *         the 2-bit base code (2BIT).  v may be NULL to leave V untouched.
 *   U     fp32 [Hkv, d, r] from headq_calibrate (ignored when r == 0).
 * Bit-exact with the arithmetic stated at the top of this header.
 * Requires 0 <= t0, 0 <= n, t0 + n <= T_cap.  n == 0 is a no-op (k, v and U
 * are then not read and may be NULL).
 */
headq_status headq_cache_write(const headq_cache *cache, const void *k, const void *v,
                               headq_dtype kv_dtype, int t0, int n, const float *U,
                               headq_stream_t stream);

/*
 * headq_decode_attn -- one decode step of attention over the HeadQ cache
 * (summary section 3, step 3: the runtime query decodes the side code into the
 * additive logit correction; softmax and the readout o = sum_j p_j v_j of
 * section 2.2).  For every (b, h), kv = h / (Hq/Hkv), tokens j < T_b:
 *   s^_j = sm_scale * ( q.k^base_j + corr_sign * (U_h^T q) . z^_j )
 *   out[b,h] = sum_j softmax(s^)_j v^_j ,  lse[b,h] = log sum_j exp(s^_j)
 * with k^base_j = mn + code*scale per group, z^_j = w_j * s_j, and v^_j the dense
 * value or its 2-bit dequantisation.
 *   q         [B, Hq, d] (q_dtype)
 *   seq_lens  int32 [B] (nullable): T_b; NULL means T_b = T for every b.
 *             0 <= T_b <= T <= T_cap.  T_b == 0 gives out = 0, lse = -inf.
 *   sm_scale  logit scale; pass 1/sqrt(d) for the pages' formula.
 *   corr_sign +1 HeadQ, 0 base code only, -1 the wrong-sign control (section 4).
 *   out       fp32 [B, Hq, d];  lse fp32 [B, Hq] (nullable).
 *   ws        device workspace of at least headq_decode_workspace_bytes(...)
 *             bytes, zero-filled before its first use: it holds the device error
 *             word (see headq_workspace_status) and per-(b, kv) arrival counters
 *             that every call leaves at zero again.  Calls sharing a workspace
 *             must not overlap on the GPU.
 * Accumulation is fp32; the result matches the fp64 definition to a relative
 * error of about 1e-5 of the row maximum.
 */
headq_status headq_decode_attn(const headq_cache *cache, const void *q,
                               headq_dtype q_dtype, int Hq, const int32_t *seq_lens,
                               int T, const float *U, float sm_scale, int corr_sign,
                               float *out, float *lse, void *ws, size_t ws_bytes,
                               headq_stream_t stream);
size_t headq_decode_workspace_bytes(const headq_cache *cache, int Hq, int T);

/*
 * headq_decode_plan -- the launch plan headq_decode_attn uses for these sizes on
 * the current device: *splits T-splits of *chunk tokens per (b, kv), the number
 * of kernels one headq_decode_append call launches (*append_kernels, nullable),
 * and the number of kernels one headq_decode_attn call launches (returned).
 * 0 on invalid sizes.
 */
int headq_decode_plan(const headq_cache *cache, int Hq, int T, int *splits, int *chunk,
                      int *append_kernels);

/*
 * headq_decode_append -- one serving decode step: write each sequence's new token
 * into the cache, then attend over the cache including it (summary section 3,
 * steps 2 and 3 in one call).  For every b with T_b >= 1 (T_b = seq_lens[b], or
 * T when seq_lens is NULL) the new key k_new[b, kv] and value v_new[b, kv]
 * ([B, Hkv, d] of kv_dtype; v_new may be NULL) are encoded into position T_b - 1
 * bit-exactly as headq_cache_write would, and out/lse are those of
 * headq_decode_attn over tokens j < T_b.  Sequences with T_b = 0 write nothing.
 * Same arguments, workspace and conventions as headq_decode_attn.  On the
 * tensor-core path this is a single kernel: the CTA that owns position T_b - 1
 * encodes the token while the others stream the cache.
 */
headq_status headq_decode_append(const headq_cache *cache, const void *k_new,
                                 const void *v_new, headq_dtype kv_dtype, const void *q,
                                 headq_dtype q_dtype, int Hq, const int32_t *seq_lens, int T,
                                 const float *U, float sm_scale, int corr_sign, float *out,
                                 float *lse, void *ws, size_t ws_bytes, headq_stream_t stream);

/*
 * headq_decode_attn_noalloc -- headq_decode_attn without a caller workspace.
 * The HeadQ pages have no counterpart to this: it exists for callers that hold
 * only their input and output buffers and cannot allocate device memory (a
 * plugin inside a host framework that hands it tensors but no allocator,
 * code running where cudaMalloc is forbidden after start-up, or a caller that
 * must not grow its memory footprint per request).
 *   Arguments and results are those of headq_decode_attn minus ws/ws_bytes.
 *   Scratch: a fixed 4 MiB array inside the library (per GPU, resident from
 *   load until process exit).  A request whose workspace
 *   (headq_decode_workspace_bytes) exceeds 4 MiB returns HEADQ_ERR_WORKSPACE
 *   and launches nothing.
 *   The first call on a device does a one-time, synchronous set-up on that
 *   device (looks up the array's device address, zero-fills it); make that
 *   first call before any stream capture.
 *   Every call on a device shares the one array and leaves its contents behind:
 *   calls whose work overlaps on the GPU (different streams, or different host
 *   threads, without ordering between them) race on it and must be serialised
 *   by the caller.  Allocates nothing (no cudaMalloc, no cudaFree).
 */
headq_status headq_decode_attn_noalloc(const headq_cache *cache, const void *q,
                                       headq_dtype q_dtype, int Hq,
                                       const int32_t *seq_lens, int T, const float *U,
                                       float sm_scale, int corr_sign, float *out,
                                       float *lse, headq_stream_t stream);

/*
 * headq_decode_noalloc_status -- headq_workspace_status for the built-in scratch
 * of headq_decode_attn_noalloc on the current device (the pages have no
 * counterpart to this either).  A no-alloc call reports a device-side error the
 * way headq_decode_attn does, through the error word at the start of its
 * scratch: a bounded wait that gave up (no result written) or a block-table
 * entry outside the page pool (result undefined).  Its caller does not hold the
 * scratch's address, so this call waits for `stream`, reads the word, clears
 * it and returns HEADQ_ERR_DEVICE if it was set, else HEADQ_OK (also when no
 * no-alloc call has run on the device yet).  Because every no-alloc call on a
 * device shares the one word, the status covers all of them since the last
 * check.  Synchronous; allocates nothing; call it off the hot path.
 */
headq_status headq_decode_noalloc_status(headq_stream_t stream);

/*
 * headq_attn_kl -- model-visible distortion of the cache against the
 * full-precision keys and values (summary section 2.1: score perturbation
 * delta_j = s^_j - s_j, attention KL and its local Fisher form; section 2.2:
 * readout error and the A^2 weighting).  With s_j = sm_scale * q.k_j (full
 * keys), p = softmax(s), p~ = softmax(s^) and v^ as read from the cache:
 *   kl         = KL(p || p~)                    fp32 [B, Hq]
 *   fisher_var = Var_p(s^ - s)                  fp32 [B, Hq]
 *   a2_vdist   = sum_j p_j^2 |v^_j - v_j|^2     fp32 [B, Hq]
 *   dout2      = |sum_j p_j (v^_j - v_j)|^2     fp32 [B, Hq] (nullable)
 *   k_full, v_full [B, Hkv, T, d] of kv_dtype (the unquantised cache).
 * Other arguments as headq_decode_attn; workspace from
 * headq_attn_kl_workspace_bytes (first 256 bytes zero before first use).
 * Accumulators are fp64.
 */
headq_status headq_attn_kl(const headq_cache *cache, const void *q, headq_dtype q_dtype,
                           int Hq, const int32_t *seq_lens, int T, const void *k_full,
                           const void *v_full, headq_dtype kv_dtype, const float *U,
                           float sm_scale, int corr_sign, float *kl, float *fisher_var,
                           float *a2_vdist, float *dout2, void *ws, size_t ws_bytes,
                           headq_stream_t stream);
size_t headq_attn_kl_workspace_bytes(const headq_cache *cache, int Hq, int T);

/*
 * A^2 value policy for the full-KV composition (2-bit values).  The pages give
 * the value-side distortion as an A^2-weighted surrogate (abstract; summary
 * section 2: under fixed attention p the readout error of value distortions
 * dv_j is summarised by D_V = sum_j p_j^2 |dv_j|^2) and compose HeadQ keys with
 * 2-bit values under an "A^2 value policy" they do not define (section 5).
 * This library's reading: a budget of K tokens per (b, kv) keeps its values
 * exact (the input precision) and the rest use the 2-bit code; D_V, summed over
 * a set of n_obs observation queries per sequence and the G query heads of the
 * KV head, loses exactly the terms of the kept tokens, so keeping the K tokens
 * with the largest
 *   a_j = |v^_j - v_j|^2 * sum_{o < n_obs} sum_{h in kv's group} p_{o,h,j}^2
 * minimises it (top-K; ties to the lower position).  p_{o,h,.} is the softmax
 * of sm_scale * q_{o,h} . k_j over the exact keys j < T_b.
 *
 * headq_a2_scores -- a_j for every cached token.
 *   q_obs   [B, n_obs, Hq, d] (q_dtype): observation queries of each sequence.
 *   k_full, v_full  [B, Hkv, T, d] (kv_dtype): the exact keys and values.
 *   scores  fp32 [B, Hkv, T]; 0 for j >= T_b.  v^_j is read from the cache.
 *   ws      headq_a2_workspace_bytes(...) bytes (its first word is the device
 *           error word, as for decode).
 * Two passes of the logits (normaliser, then p^2), fp32 accumulation.
 */
size_t headq_a2_workspace_bytes(const headq_cache *cache, int n_obs, int Hq, int T);
headq_status headq_a2_scores(const headq_cache *cache, const void *q_obs, headq_dtype q_dtype,
                             int n_obs, int Hq, const int32_t *seq_lens, int T,
                             const void *k_full, const void *v_full, headq_dtype kv_dtype,
                             float sm_scale, float *scores, void *ws, size_t ws_bytes,
                             headq_stream_t stream);

/*
 * headq_a2_select -- the kept set of each (b, kv): the min(K, T_b) positions
 * j < T_b with the largest scores (scores >= 0, as headq_a2_scores returns;
 * equal scores: lower position first), written to keep_idx int32 [B, Hkv, K]
 * in ascending order and padded with -1, and their exact values copied from
 * v_full [B, Hkv, T, d] (kv_dtype) into keep_v [B, Hkv, K, d] (same dtype,
 * zero rows for the padding).  d is a multiple of 8.
 */
headq_status headq_a2_select(const float *scores, int B, int Hkv, const int32_t *seq_lens,
                             int T, int K, const void *v_full, headq_dtype kv_dtype, int d,
                             int32_t *keep_idx, void *keep_v, headq_stream_t stream);

/*
 * headq_a2_value_fixup -- after headq_decode_attn (or headq_decode_append) with
 * the same cache, q, seq_lens, T, U, sm_scale and corr_sign has written out and
 * lse, turn its readout over the cached values v^_j into the readout over the
 * policy's mixed values (the exact value for every kept j < T_b, v^_j for the
 * rest):  out[b,h] += sum_{kept j} exp(s^_j - lse[b,h]) (v_j - v^_j), where s^_j
 * is the HeadQ logit.  The softmax weights are unchanged, so the result is the
 * mixed-value attention itself.  keep_idx/keep_v as headq_a2_select writes them
 * (entries < 0 or >= T_b are skipped); lse is read, not written.
 */
headq_status headq_a2_value_fixup(const headq_cache *cache, const void *q, headq_dtype q_dtype,
                                  int Hq, const int32_t *seq_lens, int T, const float *U,
                                  float sm_scale, int corr_sign, const int32_t *keep_idx,
                                  const void *keep_v, headq_dtype keep_dtype, int K, float *out,
                                  const float *lse, headq_stream_t stream);

/*
 * Split-T across devices (context-parallel decode).  Each device holds a
 * contiguous range [t_lo, t_lo + n) of every sequence's cached tokens, at local
 * positions [0, n) of its own cache, and runs headq_decode_attn over it with
 * the local lengths from headq_shard_seq_lens.  Its (out, lse) is a normalised
 * partial; after an all-gather of the partials every device combines them with
 * headq_merge_partials into the attention over all tokens.  This is the
 * flash-decoding split merge across devices: HeadQ changes only the logits
 * (summary section 3, step 3), so softmax over a union of token sets is
 * recovered exactly from the parts' log-sum-exps.
 *
 * headq_shard_seq_lens -- out[b] = clamp(T_b - t_lo, 0, n), T_b = seq_lens[b]
 * clamped to [0, T] (or T when seq_lens is NULL).  seq_lens, out: int32 [B].
 */
headq_status headq_shard_seq_lens(const int32_t *seq_lens, int B, int T, int t_lo, int n,
                                  int32_t *out, headq_stream_t stream);

/*
 * headq_merge_partials -- combine S partial decode results of the same BH rows
 * (BH = B * Hq).  Part s has its output at o_parts + s*part_stride, fp32
 * [BH, d], and its log-sum-exp at lse_parts + s*part_stride, fp32 [BH] (one
 * all-gathered buffer of [out | lse] blocks fits this directly); part_stride is
 * in floats and a multiple of 4.  Per row:
 *   M = max_s lse_s,  out = sum_s e^{lse_s - M} o_s / sum_s e^{lse_s - M},
 *   lse = M + log sum_s e^{lse_s - M}
 * A part with lse = -inf (no tokens) contributes nothing; a row no part covers
 * gets out = 0, lse = -inf, as headq_decode_attn gives for T_b = 0.
 *   out fp32 [BH, d]; lse fp32 [BH] (nullable).  Neither may alias a part.
 */
headq_status headq_merge_partials(const float *o_parts, const float *lse_parts, int S, int BH,
                                  int d, size_t part_stride, float *out, float *lse,
                                  headq_stream_t stream);

/*
 * headq_workspace_status -- waits for `stream`, reads the device error word of a
 * decode / attn_kl workspace, clears it, and returns HEADQ_ERR_DEVICE if a
 * kernel that used the workspace gave up a bounded wait (it then wrote no
 * result) or met a block-table entry outside the page pool (its result is
 * then undefined), else HEADQ_OK.  Synchronous; call it off the hot path.
 */
headq_status headq_workspace_status(void *ws, headq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HEADQ_H */
