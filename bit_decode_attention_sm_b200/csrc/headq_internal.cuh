// Internal declarations shared by the CUDA translation units of libheadq.
// Host-side argument checking lives in headq_api.cu; each kernel file exports
// one launcher taking a plain parameter struct.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "headq.h"

namespace headq {

// First bytes of every decode / attn_kl workspace: the device error word.
constexpr size_t kWsHeaderBytes = 256;
// Decode workspaces then hold a fixed region of split arrival counters (one per
// (b, kv), left at zero by every call; never overlapped by partials, whatever
// the shape of the call), then the partials.
constexpr int kMaxFusedUnits = 8192;
constexpr size_t kWsCounterBytes = sizeof(unsigned) * kMaxFusedUnits;
constexpr unsigned kDevErrWaitTimeout = 1u;
constexpr unsigned kDevErrBadPage = 2u;  // a block-table entry outside the pool

__host__ __device__ constexpr int group_size(int d) { return d < 32 ? d : 32; }
__host__ __device__ constexpr int num_groups(int d) { return d / group_size(d); }

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// p (a pointer into shared memory) advanced to the next multiple of `align` (a
// power of two) bytes of the shared window, by pointer arithmetic on p itself so
// that the compiler keeps its address space (shared loads and stores, not
// generic ones)
template <typename T>
__device__ __forceinline__ T* smem_align(T* p, uint32_t align) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(p) +
                              (((a + align - 1) & ~(align - 1)) - a));
}

// element i of a tensor that is either fp32 or bf16
__device__ __forceinline__ float load_elem(const void* p, size_t i, bool bf16) {
  return bf16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(p)[i])
              : static_cast<const float*>(p)[i];
}

// 2-bit code of channel c in a packed row
__device__ __forceinline__ int code2(const uint8_t* row, int c) {
  return (row[c >> 2] >> (2 * (c & 3))) & 3;
}

// signed 4-bit side code i in a packed row
__device__ __forceinline__ int nibble(const uint8_t* row, int i) {
  int v = (row[i >> 1] >> (4 * (i & 1))) & 0xF;
  return v >= 8 ? v - 16 : v;
}

// Where token t of sequence b, KV head kv lives.  The planes are slabs of
// slab_rows() consecutive rows: contiguous planes have one slab per (b, kv)
// ([b][kv][t], slab b*Hkv + kv, offset t); a paged cache one per (page, kv)
// ([page][kv][t % page_size], page from the block table).  slab < 0 when that
// entry lies outside the pool.  The 64 tokens of a 64-aligned tile share one
// page (page_size is a multiple of 64), so they occupy consecutive rows.
struct CacheSlab {
  long long slab;
  int off;
};

__device__ __forceinline__ int slab_rows(const headq_cache& c) {
  return c.page_size ? c.page_size : c.T_cap;
}

__device__ __forceinline__ CacheSlab cache_slab(const headq_cache& c, int b, int kv, int t) {
  if (c.page_size == 0) return {static_cast<long long>(b) * c.Hkv + kv, t};
  const int i = t / c.page_size;
  const int pg = c.block_table[static_cast<size_t>(b) * c.max_pages + i];
  if (pg < 0 || pg >= c.num_pages) return {-1, 0};
  return {static_cast<long long>(pg) * c.Hkv + kv, t - i * c.page_size};
}

// plane row of the token, -1 when its block-table entry is outside the pool
__device__ __forceinline__ long long cache_row(const headq_cache& c, int b, int kv, int t) {
  const CacheSlab s = cache_slab(c, b, kv, t);
  return s.slab < 0 ? -1 : s.slab * slab_rows(c) + s.off;
}

// cache_slab for a read: a bad entry reads slab 0 (always valid memory) and
// raises kDevErrBadPage in the error word, when there is one
__device__ __forceinline__ CacheSlab cache_slab_read(const headq_cache& c, int b, int kv, int t,
                                                     unsigned* err) {
  CacheSlab s = cache_slab(c, b, kv, t);
  if (s.slab < 0) {
    if (err) atomicOr(err, kDevErrBadPage);
    s = {0, t % c.page_size};
  }
  return s;
}

__device__ __forceinline__ size_t cache_row_read(const headq_cache& c, int b, int kv, int t,
                                                 unsigned* err) {
  const CacheSlab s = cache_slab_read(c, b, kv, t, err);
  return static_cast<size_t>(s.slab) * slab_rows(c) + s.off;
}

struct CacheWriteParams {
  headq_cache c;
  const void* k;
  const void* v;
  bool in_bf16;
  int t0, n;
  const float* U;
  // append mode (n == 1): sequence b's token goes to position T_b - 1, with
  // T_b = seq_lens[b] (or T when seq_lens is null); nothing when T_b == 0
  bool append;
  const int32_t* seq_lens;
  int T;
  // 1.0f, set by the host: a value the compiler cannot see, so that the packed
  // "multiply, then add" of the codec is not contracted (codec::fma2)
  float one;
};

// Decode split partials: unnormalised outputs o [B*Hq][splits][d] (rows of d
// floats, 16-byte aligned), then the running max m and sum l [B*Hq][splits].
struct PartView {
  float* o;
  float* m;
  float* l;
};
__host__ __device__ inline PartView part_view(float* base, size_t bhq, int splits, int d) {
  const size_t n = bhq * static_cast<size_t>(splits);
  return {base, base + n * d, base + n * d + n};
}

struct DecodeParams {
  headq_cache c;
  const void* q;
  bool q_bf16;
  int Hq, G, T;
  const int32_t* seq_lens;
  const float* U;
  float sm_scale;
  float corr_sign;
  int splits;      // T-splits per (b, kv)
  int chunk;       // tokens per split (multiple of 64)
  float* part;     // [B, Hq, splits, d + 2] partial (o, m, l)
  unsigned* err;   // device error word
  unsigned* counters;  // [B * Hkv] split arrival counters, zero between calls
  bool fused;          // the split kernel merges its own splits (last CTA)
  // fused append (tensor-core kernel): the new token [B, Hkv, d] of each sequence
  // is encoded into position T_b - 1 before the tile holding it is read
  const void* k_new;
  const void* v_new;
  bool new_bf16;
  float* out;
  float* lse;
};

struct AttnKlParams {
  headq_cache c;
  const void* q;
  bool q_bf16;
  int Hq, G, T;
  const int32_t* seq_lens;
  const void* k_full;
  const void* v_full;
  bool kv_bf16;
  const float* U;
  float sm_scale;
  float corr_sign;
  int splits, chunk;
  bool hm;         // the tensor-core kernel (attn_kl_hm.cu) with its own split plan
  double* part;    // [B, Hq, splits, 7 + d]
  unsigned* err;
  float *kl, *fvar, *a2v, *dout2;
};

struct CalibrateParams {
  const void* q;
  bool bf16;
  int N, Hq, Hkv, G, d, r;
  bool center;
  double* gram;    // [Hkv, d, d]
  double* vt;      // [Hkv, d, d] rotation accumulator (rows = eigenvectors)
  float* U;
  float* eig;
};

// Tensor map of bf16 rows of `inner` channels in slabs ([slab][row][channel],
// row stride inner * 2 bytes), boxes of 64 channels x box_rows rows with the
// 128-byte swizzle (headq_api.cu).  False when the driver offers no encoder or
// the encoding fails (a base or stride not 16-byte aligned).
bool tensor_maps_available();
bool encode_bf16_rows(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                      uint64_t slabs, uint32_t box_rows);

// host-side argument checks shared by the entry points (headq_api.cu)
bool aligned16(const void* p);
headq_status check_cache(const headq_cache* c);
headq_status check_read_args(const headq_cache* c, const void* q, headq_dtype qd, int Hq, int T,
                             const float* U, int corr_sign);

cudaError_t launch_cache_write(const CacheWriteParams& p, cudaStream_t s);
cudaError_t launch_attn_kl(const AttnKlParams& p, cudaStream_t s);
// the tensor-core diagnostic kernel (attn_kl_hm.cu): its shapes, its split plan
// and its launch (the split kernel only; the combine kernel follows it)
struct SplitPlan;
bool kl_hm_supported(const headq_cache& c, int G, bool kv_bf16);
cudaError_t launch_attn_kl_hm(const AttnKlParams& p, cudaStream_t s);
cudaError_t launch_calibrate(const CalibrateParams& p, cudaStream_t s);

// split planning shared by the workspace-size query and the launch
struct SplitPlan {
  int splits, chunk;
};
SplitPlan plan_splits(int units, int T, int min_chunk, int ctas_per_sm = 2);
SplitPlan kl_hm_plan(int units, int T);
int sm_count();

// The decode kernel and T-split plan chosen for these sizes on the current
// device; the workspace query, headq_decode_plan and the launch all use it.
struct DecodePlan {
  int splits, chunk, kernels;
  bool mma;    // tensor-core TMA kernel (decode_mma.cu) instead of the generic one
  bool fused;  // that kernel also merges the splits (no combine launch)
};
DecodePlan decode_plan(const headq_cache& c, int Hq, int T);
cudaError_t launch_decode(const DecodeParams& p, bool mma, cudaStream_t s);  // p.fused set

constexpr int kMaxMmaSplits = 1024;  // the merging CTA keeps per-split weights in smem
bool mma_decode_supported(const headq_cache& c, int G);
int mma_decode_ctas_per_sm(const headq_cache& c, int G);
cudaError_t launch_decode_mma(const DecodeParams& p, cudaStream_t s);
// the tensor-core kernel for 5..8 query heads per KV head with per-token keys
// (decode_hm.cu); launch_decode_mma and mma_decode_ctas_per_sm route to it
bool hm_decode_supported(const headq_cache& c, int G);
int hm_decode_ctas_per_sm(const headq_cache& c);
cudaError_t launch_decode_hm(const DecodeParams& p, cudaStream_t s);


}  // namespace headq
