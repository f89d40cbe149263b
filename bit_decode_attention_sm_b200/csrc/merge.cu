// Split-T across devices (context parallel decode): each device attends over
// its own contiguous range of cached tokens and returns a normalised partial
// (o_s, lse_s); after one all-gather of the partials every device combines
// them.  The combine is the flash-decoding split merge (softmax over the union
// of the token sets, written in terms of each part's log-sum-exp):
//   M = max_s lse_s,  w_s = exp(lse_s - M),
//   out = sum_s w_s o_s / sum_s w_s,   lse = M + log sum_s w_s,
// the same identity the single-device decode uses for its T-splits (HeadQ
// changes only the logits, section 3, step 3 of the gist.science summary; the
// softmax and readout of section 2.2 are unchanged).
#include <math.h>

#include "headq_internal.cuh"

#define HEADQ_API extern "C" __attribute__((visibility("default")))

namespace headq {
namespace {

constexpr int kMergeThreads = 128;

// one CTA per output row (b, h); threads over channels
__global__ void __launch_bounds__(kMergeThreads)
merge_partials_kernel(const float* o_parts, const float* lse_parts, int S, int d,
                      size_t stride, float* out, float* lse) {
  const int bh = blockIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, lse_parts[s * stride + bh]);
  if (M == -INFINITY) {  // no part holds a token: out = 0, lse = -inf
    for (int c = threadIdx.x; c < d; c += kMergeThreads) out[static_cast<size_t>(bh) * d + c] = 0.0f;
    if (lse && threadIdx.x == 0) lse[bh] = -INFINITY;
    return;
  }
  float L = 0.0f;
  for (int s = 0; s < S; ++s) L += expf(lse_parts[s * stride + bh] - M);
  for (int c = threadIdx.x; c < d; c += kMergeThreads) {
    float acc = 0.0f;
    for (int s = 0; s < S; ++s) {
      const float w = expf(lse_parts[s * stride + bh] - M);
      if (w > 0.0f) acc = fmaf(w, o_parts[s * stride + static_cast<size_t>(bh) * d + c], acc);
    }
    out[static_cast<size_t>(bh) * d + c] = acc / L;
  }
  if (lse && threadIdx.x == 0) lse[bh] = M + logf(L);
}

// local length of sequence b on the device holding global tokens [t_lo, t_lo+n)
__global__ void shard_seq_lens_kernel(const int32_t* seq_lens, int B, int T, int t_lo, int n,
                                      int32_t* out) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int Tb = seq_lens ? seq_lens[b] : T;
  Tb = Tb < 0 ? 0 : (Tb > T ? T : Tb);
  const int loc = Tb - t_lo;
  out[b] = loc < 0 ? 0 : (loc > n ? n : loc);
}

}  // namespace
}  // namespace headq

using namespace headq;

HEADQ_API headq_status headq_merge_partials(const float* o_parts, const float* lse_parts,
                                            int S, int BH, int d, size_t part_stride,
                                            float* out, float* lse, headq_stream_t stream) {
  if (S <= 0 || BH < 0 || d <= 0) return HEADQ_ERR_INVALID_ARG;
  if (BH == 0) return HEADQ_OK;
  if (!o_parts || !lse_parts || !out) return HEADQ_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(lse_parts) || !aligned16(out) || (lse && !aligned16(lse)))
    return HEADQ_ERR_INVALID_ARG;
  if (part_stride % 4 != 0) return HEADQ_ERR_INVALID_ARG;
  if (S > 1 && part_stride < static_cast<size_t>(BH) * d) return HEADQ_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  merge_partials_kernel<<<BH, kMergeThreads, 0, s>>>(o_parts, lse_parts, S, d, part_stride,
                                                     out, lse);
  return cudaGetLastError() == cudaSuccess ? HEADQ_OK : HEADQ_ERR_CUDA;
}

HEADQ_API headq_status headq_shard_seq_lens(const int32_t* seq_lens, int B, int T, int t_lo,
                                            int n, int32_t* out, headq_stream_t stream) {
  if (B < 0 || T < 0 || t_lo < 0 || n < 0) return HEADQ_ERR_INVALID_ARG;
  if (B == 0) return HEADQ_OK;
  if (!out || !aligned16(out) || (seq_lens && !aligned16(seq_lens))) return HEADQ_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  shard_seq_lens_kernel<<<(B + 127) / 128, 128, 0, s>>>(seq_lens, B, T, t_lo, n, out);
  return cudaGetLastError() == cudaSuccess ? HEADQ_OK : HEADQ_ERR_CUDA;
}
