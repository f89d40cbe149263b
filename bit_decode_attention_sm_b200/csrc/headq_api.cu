// C ABI of libheadq: argument checking on the host, workspace sizing, and the
// launch of the kernels in the other translation units.  Nothing here
// allocates device memory; a failed check returns before any launch.
#include <string.h>

#include <mutex>

#include "headq_internal.cuh"

#define HEADQ_API extern "C" __attribute__((visibility("default")))

namespace headq {

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

static bool supported_d(int d) {
  return d == 8 || d == 16 || d == 32 || d == 64 || d == 128 || d == 256;
}

namespace {
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library); null when the driver does not offer it
EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(f);
    cudaGetLastError();
  });
  return fn;
}
}  // namespace

bool tensor_maps_available() { return encode_fn() != nullptr; }

bool encode_bf16_rows(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                      uint64_t slabs, uint32_t box_rows) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {inner, rows, slabs};
  const cuuint64_t strides[2] = {inner * 2, rows * inner * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

// Split each (b, kv) sequence into chunks so that the grid covers about
// `ctas_per_sm` CTAs per SM of this GPU, with chunks of at least `min_chunk`
// tokens and a multiple of 64 tokens.
SplitPlan plan_splits(int units, int T, int min_chunk, int ctas_per_sm) {
  SplitPlan sp{1, 64};
  if (T <= 0 || units <= 0) return sp;
  const int target = ctas_per_sm * sm_count();
  int s = (target + units - 1) / units;
  const int max_s = (T + min_chunk - 1) / min_chunk;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  int chunk = (T + s - 1) / s;
  chunk = (chunk + 63) / 64 * 64;
  sp.chunk = chunk;
  sp.splits = (T + chunk - 1) / chunk;
  return sp;
}

headq_status check_cache(const headq_cache* c) {
  if (!c) return HEADQ_ERR_INVALID_ARG;
  if (c->B < 0 || c->Hkv <= 0 || c->T_cap < 0 || c->r < 0) return HEADQ_ERR_INVALID_ARG;
  if (!supported_d(c->d)) return HEADQ_ERR_UNSUPPORTED;
  if (c->r % 2 != 0 || c->r > c->d || c->r > 32) return HEADQ_ERR_UNSUPPORTED;
  if (c->T_cap % 16 != 0) return HEADQ_ERR_UNSUPPORTED;
  if (c->kmode != HEADQ_K_TOKEN && c->kmode != HEADQ_K_CHANNEL) return HEADQ_ERR_INVALID_ARG;
  if (c->kmode == HEADQ_K_CHANNEL && c->T_cap % 64 != 0) return HEADQ_ERR_UNSUPPORTED;
  if (c->page_size < 0) return HEADQ_ERR_INVALID_ARG;
  if (c->page_size > 0) {  // paged pools: whole 64-token tiles per page
    if (c->page_size % 64 != 0) return HEADQ_ERR_UNSUPPORTED;
    if (!c->block_table || !aligned16(c->block_table)) return HEADQ_ERR_INVALID_ARG;
    if (c->num_pages <= 0 || c->max_pages <= 0) return HEADQ_ERR_INVALID_ARG;
    if (static_cast<long long>(c->max_pages) * c->page_size != c->T_cap)
      return HEADQ_ERR_INVALID_ARG;
  }
  if (c->vmode != HEADQ_V_DENSE && c->vmode != HEADQ_V_2BIT) return HEADQ_ERR_INVALID_ARG;
  if (c->v_dtype != HEADQ_F32 && c->v_dtype != HEADQ_BF16) return HEADQ_ERR_INVALID_ARG;
  if (!c->k_codes || !c->k_scale || !c->k_min) return HEADQ_ERR_INVALID_ARG;
  if (!aligned16(c->k_codes) || !aligned16(c->k_scale) || !aligned16(c->k_min))
    return HEADQ_ERR_INVALID_ARG;
  if (c->r > 0) {
    if (!c->z_codes || !c->z_scale) return HEADQ_ERR_INVALID_ARG;
    if (!aligned16(c->z_codes) || !aligned16(c->z_scale)) return HEADQ_ERR_INVALID_ARG;
  }
  if (c->vmode == HEADQ_V_DENSE) {
    if (!c->v || !aligned16(c->v)) return HEADQ_ERR_INVALID_ARG;
  } else {
    if (!c->v_codes || !c->v_scale || !c->v_min) return HEADQ_ERR_INVALID_ARG;
    if (!aligned16(c->v_codes) || !aligned16(c->v_scale) || !aligned16(c->v_min))
      return HEADQ_ERR_INVALID_ARG;
  }
  return HEADQ_OK;
}

headq_status check_read_args(const headq_cache* c, const void* q, headq_dtype qd, int Hq, int T,
                             const float* U, int corr_sign) {
  headq_status st = check_cache(c);
  if (st != HEADQ_OK) return st;
  if (!q || !aligned16(q)) return HEADQ_ERR_INVALID_ARG;
  if (qd != HEADQ_F32 && qd != HEADQ_BF16) return HEADQ_ERR_INVALID_ARG;
  if (Hq <= 0 || Hq % c->Hkv != 0) return HEADQ_ERR_INVALID_ARG;
  if (T < 0 || T > c->T_cap) return HEADQ_ERR_INVALID_ARG;
  if (corr_sign < -1 || corr_sign > 1) return HEADQ_ERR_INVALID_ARG;
  if (c->r > 0 && (!U || !aligned16(U))) return HEADQ_ERR_INVALID_ARG;
  if ((Hq / c->Hkv) * c->d > 2048) return HEADQ_ERR_UNSUPPORTED;
  return HEADQ_OK;
}

static size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// decode workspace: [error word header][fixed arrival-counter region][partials]
static size_t decode_ws(const headq_cache* c, int Hq, int T) {
  const DecodePlan dp = decode_plan(*c, Hq, T);
  return kWsHeaderBytes + kWsCounterBytes +
         round256(sizeof(float) * static_cast<size_t>(c->B) * Hq * dp.splits * (c->d + 2));
}

// the diagnostic's split plan: the tensor-core kernel's when it serves the shape
static SplitPlan kl_plan(const headq_cache& c, int Hq, int T, bool kv_bf16, bool* hm) {
  *hm = kl_hm_supported(c, Hq / c.Hkv, kv_bf16);
  return *hm ? kl_hm_plan(c.B * c.Hkv, T) : plan_splits(c.B * c.Hkv, T, 256);
}

// sized for either kernel (the value dtype of the call is not known here)
static size_t kl_ws(const headq_cache* c, int Hq, int T) {
  bool hm = false;
  SplitPlan sp = plan_splits(c->B * c->Hkv, T, 256);
  const SplitPlan sh = kl_plan(*c, Hq, T, true, &hm);
  if (hm && sh.splits > sp.splits) sp = sh;
  return kWsHeaderBytes +
         round256(sizeof(double) * static_cast<size_t>(c->B) * Hq * sp.splits * (7 + c->d));
}

}  // namespace headq

using namespace headq;

HEADQ_API int headq_version(void) { return 101; }

HEADQ_API const char* headq_status_string(headq_status s) {
  switch (s) {
    case HEADQ_OK: return "ok";
    case HEADQ_ERR_INVALID_ARG: return "invalid argument";
    case HEADQ_ERR_UNSUPPORTED: return "unsupported shape";
    case HEADQ_ERR_WORKSPACE: return "workspace missing or too small";
    case HEADQ_ERR_CUDA: return "CUDA error";
    case HEADQ_ERR_DEVICE: return "device-side error (bounded wait gave up)";
  }
  return "unknown status";
}

HEADQ_API size_t headq_calibrate_workspace_bytes(int N, int Hq, int Hkv, int d) {
  if (N <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return 0;
  (void)Hq;
  return round256(sizeof(double) * (2 * static_cast<size_t>(Hkv) * d * d + Hkv * d));
}

HEADQ_API headq_status headq_calibrate(const void* q_cal, headq_dtype dtype, int N, int Hq,
                                       int Hkv, int d, int r, int center, float* U_out,
                                       float* eig_out, void* ws, size_t ws_bytes,
                                       headq_stream_t stream) {
  if (!q_cal || !U_out || !aligned16(q_cal) || !aligned16(U_out)) return HEADQ_ERR_INVALID_ARG;
  if (eig_out && !aligned16(eig_out)) return HEADQ_ERR_INVALID_ARG;
  if (dtype != HEADQ_F32 && dtype != HEADQ_BF16) return HEADQ_ERR_INVALID_ARG;
  if (N <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0) return HEADQ_ERR_INVALID_ARG;
  if (d < 2 || d % 2 != 0 || d > 128 || r < 1 || r > d) return HEADQ_ERR_UNSUPPORTED;
  if (!ws || !aligned16(ws) || ws_bytes < headq_calibrate_workspace_bytes(N, Hq, Hkv, d))
    return HEADQ_ERR_WORKSPACE;
  CalibrateParams p{};
  p.q = q_cal;
  p.bf16 = dtype == HEADQ_BF16;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.d = d;
  p.r = r;
  p.center = center != 0;
  p.gram = static_cast<double*>(ws);
  p.vt = p.gram + static_cast<size_t>(Hkv) * d * d;
  p.U = U_out;
  p.eig = eig_out;
  return launch_calibrate(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? HEADQ_OK
             : HEADQ_ERR_CUDA;
}

HEADQ_API headq_status headq_cache_write(const headq_cache* cache, const void* k,
                                         const void* v, headq_dtype kv_dtype, int t0, int n,
                                         const float* U, headq_stream_t stream) {
  headq_status st = check_cache(cache);
  if (st != HEADQ_OK) return st;
  if (kv_dtype != HEADQ_F32 && kv_dtype != HEADQ_BF16) return HEADQ_ERR_INVALID_ARG;
  if (t0 < 0 || n < 0 || static_cast<long>(t0) + n > cache->T_cap) return HEADQ_ERR_INVALID_ARG;
  if (cache->kmode == HEADQ_K_CHANNEL && t0 % 64 != 0) return HEADQ_ERR_UNSUPPORTED;
  if (n == 0 || cache->B == 0) return HEADQ_OK;  // nothing to read: k, v, U unused
  if (!k || !aligned16(k) || (v && !aligned16(v))) return HEADQ_ERR_INVALID_ARG;
  if (cache->r > 0 && (!U || !aligned16(U))) return HEADQ_ERR_INVALID_ARG;
  CacheWriteParams p{};
  p.c = *cache;
  p.k = k;
  p.v = v;
  p.in_bf16 = kv_dtype == HEADQ_BF16;
  p.t0 = t0;
  p.n = n;
  p.U = U;
  return launch_cache_write(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? HEADQ_OK
             : HEADQ_ERR_CUDA;
}

HEADQ_API size_t headq_decode_workspace_bytes(const headq_cache* cache, int Hq, int T) {
  if (!cache || cache->B < 0 || cache->Hkv <= 0 || Hq <= 0 || T < 0 || !supported_d(cache->d))
    return 0;
  return decode_ws(cache, Hq, T);
}

HEADQ_API int headq_decode_plan(const headq_cache* cache, int Hq, int T, int* splits,
                                int* chunk, int* append_kernels) {
  if (!cache || cache->B < 0 || cache->Hkv <= 0 || Hq <= 0 || T < 0 || !supported_d(cache->d))
    return 0;
  const DecodePlan dp = decode_plan(*cache, Hq, T);
  if (splits) *splits = dp.splits;
  if (chunk) *chunk = dp.chunk;
  if (append_kernels) *append_kernels = dp.mma ? dp.kernels : dp.kernels + 1;
  return dp.kernels;
}

HEADQ_API headq_status headq_decode_attn(const headq_cache* cache, const void* q,
                                         headq_dtype q_dtype, int Hq,
                                         const int32_t* seq_lens, int T, const float* U,
                                         float sm_scale, int corr_sign, float* out,
                                         float* lse, void* ws, size_t ws_bytes,
                                         headq_stream_t stream) {
  headq_status st = check_read_args(cache, q, q_dtype, Hq, T, U, corr_sign);
  if (st != HEADQ_OK) return st;
  if (!out || !aligned16(out) || (lse && !aligned16(lse))) return HEADQ_ERR_INVALID_ARG;
  if (seq_lens && !aligned16(seq_lens)) return HEADQ_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < decode_ws(cache, Hq, T)) return HEADQ_ERR_WORKSPACE;
  if (cache->B == 0) return HEADQ_OK;
  const DecodePlan sp = decode_plan(*cache, Hq, T);
  DecodeParams p{};
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
  p.splits = sp.splits;
  p.chunk = sp.chunk;
  p.err = static_cast<unsigned*>(ws);
  p.counters = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + kWsHeaderBytes);
  p.fused = sp.fused;
  p.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsHeaderBytes + kWsCounterBytes);
  p.out = out;
  p.lse = lse;
  return launch_decode(p, sp.mma, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? HEADQ_OK
             : HEADQ_ERR_CUDA;
}

HEADQ_API headq_status headq_decode_append(const headq_cache* cache, const void* k_new,
                                           const void* v_new, headq_dtype kv_dtype,
                                           const void* q, headq_dtype q_dtype, int Hq,
                                           const int32_t* seq_lens, int T, const float* U,
                                           float sm_scale, int corr_sign, float* out,
                                           float* lse, void* ws, size_t ws_bytes,
                                           headq_stream_t stream) {
  headq_status st = check_read_args(cache, q, q_dtype, Hq, T, U, corr_sign);
  if (st != HEADQ_OK) return st;
  if (cache->kmode != HEADQ_K_TOKEN) return HEADQ_ERR_UNSUPPORTED;  // sealed key blocks
  if (!k_new || !aligned16(k_new) || (v_new && !aligned16(v_new))) return HEADQ_ERR_INVALID_ARG;
  if (kv_dtype != HEADQ_F32 && kv_dtype != HEADQ_BF16) return HEADQ_ERR_INVALID_ARG;
  if (!out || !aligned16(out) || (lse && !aligned16(lse))) return HEADQ_ERR_INVALID_ARG;
  if (seq_lens && !aligned16(seq_lens)) return HEADQ_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < decode_ws(cache, Hq, T)) return HEADQ_ERR_WORKSPACE;
  if (cache->B == 0) return HEADQ_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const DecodePlan sp = decode_plan(*cache, Hq, T);
  if (!sp.mma) {
    // generic path: the append write, then the decode
    CacheWriteParams w{};
    w.c = *cache;
    w.k = k_new;
    w.v = v_new;
    w.in_bf16 = kv_dtype == HEADQ_BF16;
    w.n = 1;
    w.U = U;
    w.append = true;
    w.seq_lens = seq_lens;
    w.T = T;
    if (launch_cache_write(w, s) != cudaSuccess) return HEADQ_ERR_CUDA;
    return headq_decode_attn(cache, q, q_dtype, Hq, seq_lens, T, U, sm_scale, corr_sign, out,
                             lse, ws, ws_bytes, stream);
  }
  DecodeParams p{};
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
  p.splits = sp.splits;
  p.chunk = sp.chunk;
  p.err = static_cast<unsigned*>(ws);
  p.counters = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + kWsHeaderBytes);
  p.fused = sp.fused;
  p.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsHeaderBytes + kWsCounterBytes);
  p.out = out;
  p.lse = lse;
  p.k_new = k_new;
  p.v_new = v_new;
  p.new_bf16 = kv_dtype == HEADQ_BF16;
  return launch_decode(p, true, s) == cudaSuccess ? HEADQ_OK : HEADQ_ERR_CUDA;
}

HEADQ_API size_t headq_attn_kl_workspace_bytes(const headq_cache* cache, int Hq, int T) {
  if (!cache || cache->B < 0 || cache->Hkv <= 0 || Hq <= 0 || T < 0 || !supported_d(cache->d))
    return 0;
  return kl_ws(cache, Hq, T);
}

HEADQ_API headq_status headq_attn_kl(const headq_cache* cache, const void* q,
                                     headq_dtype q_dtype, int Hq, const int32_t* seq_lens,
                                     int T, const void* k_full, const void* v_full,
                                     headq_dtype kv_dtype, const float* U, float sm_scale,
                                     int corr_sign, float* kl, float* fisher_var,
                                     float* a2_vdist, float* dout2, void* ws, size_t ws_bytes,
                                     headq_stream_t stream) {
  headq_status st = check_read_args(cache, q, q_dtype, Hq, T, U, corr_sign);
  if (st != HEADQ_OK) return st;
  if (!k_full || !v_full || !aligned16(k_full) || !aligned16(v_full))
    return HEADQ_ERR_INVALID_ARG;
  if (kv_dtype != HEADQ_F32 && kv_dtype != HEADQ_BF16) return HEADQ_ERR_INVALID_ARG;
  if (!kl || !fisher_var || !a2_vdist || !aligned16(kl) || !aligned16(fisher_var) ||
      !aligned16(a2_vdist) || (dout2 && !aligned16(dout2)))
    return HEADQ_ERR_INVALID_ARG;
  if (seq_lens && !aligned16(seq_lens)) return HEADQ_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < kl_ws(cache, Hq, T)) return HEADQ_ERR_WORKSPACE;
  if (cache->B == 0) return HEADQ_OK;
  bool hm = false;
  const SplitPlan sp = kl_plan(*cache, Hq, T, kv_dtype == HEADQ_BF16, &hm);
  AttnKlParams p{};
  p.hm = hm;
  p.c = *cache;
  p.q = q;
  p.q_bf16 = q_dtype == HEADQ_BF16;
  p.Hq = Hq;
  p.G = Hq / cache->Hkv;
  p.T = T;
  p.seq_lens = seq_lens;
  p.k_full = k_full;
  p.v_full = v_full;
  p.kv_bf16 = kv_dtype == HEADQ_BF16;
  p.U = U;
  p.sm_scale = sm_scale;
  p.corr_sign = static_cast<float>(corr_sign);
  p.splits = sp.splits;
  p.chunk = sp.chunk;
  p.err = static_cast<unsigned*>(ws);
  p.part = reinterpret_cast<double*>(static_cast<char*>(ws) + kWsHeaderBytes);
  p.kl = kl;
  p.fvar = fisher_var;
  p.a2v = a2_vdist;
  p.dout2 = dout2;
  return launch_attn_kl(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? HEADQ_OK
             : HEADQ_ERR_CUDA;
}

HEADQ_API headq_status headq_workspace_status(void* ws, headq_stream_t stream) {
  if (!ws) return HEADQ_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HEADQ_ERR_CUDA;
  if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return HEADQ_ERR_CUDA;
  if (word != 0) {
    if (cudaMemset(ws, 0, sizeof(word)) != cudaSuccess) return HEADQ_ERR_CUDA;
    return HEADQ_ERR_DEVICE;
  }
  return HEADQ_OK;
}
