// HeadQ calibration: the query-PCA basis U_h ("HeadQ: Model-Visible Distortion
// and Score-Space Correction for KV-Cache Quantization", gist.science summary,
// section 3, step 1 -- a rank-r basis per layer and head, by PCA of post-RoPE
// calibration queries; section 4 -- query-PCA bases recover the active residual).
//
// Per KV head the basis is the top-r eigenvectors of the second moment
// C = (1/M) sum_m x_m x_m^T of the M = N*G calibration queries of its G query
// heads (x centred first when requested).  The score error of a key residual e
// is q.e, with E[(q.e)^2] = e^T E[q q^T] e, so this eigenspace is the rank-r
// subspace that captures the most score error.
//
//   gram kernel    C in fp64, one CTA per (row i, kv)
//   jacobi kernel  one CTA per kv: cyclic two-sided Jacobi rotations in fp64
//                  (Jacobi's method; rotation angle as in Golub & Van Loan,
//                  "Matrix Computations", symmetric Schur decomposition), the
//                  d/2 disjoint pairs of each step from the round-robin
//                  ("circle") schedule applied in parallel; then the r largest
//                  eigenvalues, descending, and a sign rule per vector.
#include <math.h>

#include "headq_internal.cuh"

namespace headq {
namespace {

constexpr int kGramThreads = 128;
constexpr int kJacThreads = 256;
constexpr int kMaxSweeps = 40;

__global__ void mean_kernel(const CalibrateParams p, double* mean) {
  const int kv = blockIdx.x;
  const int d = p.d;
  const long M = static_cast<long>(p.N) * p.G;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double acc = 0.0;
    for (long m = 0; m < M; ++m) {
      const long n = m / p.G, g = m - n * p.G;
      acc += load_elem(p.q, (static_cast<size_t>(n) * p.Hq + kv * p.G + g) * d + c, p.bf16);
    }
    mean[kv * d + c] = acc / static_cast<double>(M);
  }
}

__global__ void __launch_bounds__(kGramThreads)
gram_kernel(const CalibrateParams p, const double* mean) {
  const int i = blockIdx.x, kv = blockIdx.y;
  const int d = p.d;
  const long M = static_cast<long>(p.N) * p.G;
  __shared__ double xi_s[kGramThreads];
  double acc = 0.0;
  const int j = threadIdx.x;
  const double mi = p.center ? mean[kv * d + i] : 0.0;
  const double mj = (p.center && j < d) ? mean[kv * d + j] : 0.0;
  for (long m0 = 0; m0 < M; m0 += kGramThreads) {
    const long mm = m0 + threadIdx.x;
    double xi = 0.0;
    if (mm < M) {
      const long n = mm / p.G, g = mm - n * p.G;
      xi = load_elem(p.q, (static_cast<size_t>(n) * p.Hq + kv * p.G + g) * d + i, p.bf16) - mi;
    }
    xi_s[threadIdx.x] = xi;
    __syncthreads();
    if (j < d) {
      const long cnt = min(static_cast<long>(kGramThreads), M - m0);
      for (long t = 0; t < cnt; ++t) {
        const long m = m0 + t;
        const long n = m / p.G, g = m - n * p.G;
        const double xj =
            load_elem(p.q, (static_cast<size_t>(n) * p.Hq + kv * p.G + g) * d + j, p.bf16) - mj;
        acc += xi_s[t] * xj;
      }
    }
    __syncthreads();
  }
  if (j < d) p.gram[(static_cast<size_t>(kv) * d + i) * d + j] = acc / static_cast<double>(M);
}

// member at position pos of the round-robin schedule at step k (d players)
__device__ __forceinline__ int rr_member(int pos, int k, int d) {
  return pos == 0 ? 0 : ((pos - 1 + k) % (d - 1)) + 1;
}

__global__ void __launch_bounds__(kJacThreads)
jacobi_kernel(const CalibrateParams p) {
  const int kv = blockIdx.x;
  const int d = p.d, r = p.r, half = d / 2;
  extern __shared__ double A[];                 // [d][d]
  double* cs = A + d * d;                       // [half] cosines
  double* sn = cs + half;                       // [half] sines
  int* pp = reinterpret_cast<int*>(sn + half);  // [half]
  int* qq = pp + half;                          // [half]
  __shared__ double red[kJacThreads / 32];
  __shared__ int stop;
  double* Vt = p.vt + static_cast<size_t>(kv) * d * d;  // row k = eigenvector k
  const int tid = threadIdx.x;

  for (int i = tid; i < d * d; i += kJacThreads) {
    A[i] = p.gram[static_cast<size_t>(kv) * d * d + i];
    Vt[i] = (i / d == i % d) ? 1.0 : 0.0;
  }
  __syncthreads();

  for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
    // convergence: off-diagonal mass against the total
    double off = 0.0, tot = 0.0;
    for (int i = tid; i < d * d; i += kJacThreads) {
      const double a2 = A[i] * A[i];
      tot += a2;
      if (i / d != i % d) off += a2;
    }
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
    }
    if ((tid & 31) == 0) red[tid >> 5] = off;
    __syncthreads();
    if (tid == 0) {
      double so = 0.0;
      for (int w = 0; w < kJacThreads / 32; ++w) so += red[w];
      red[0] = so;
    }
    __syncthreads();
    const double off_all = red[0];
    __syncthreads();
    if ((tid & 31) == 0) red[tid >> 5] = tot;
    __syncthreads();
    if (tid == 0) {
      double st = 0.0;
      for (int w = 0; w < kJacThreads / 32; ++w) st += red[w];
      stop = (off_all <= 1e-28 * st) ? 1 : 0;
    }
    __syncthreads();
    if (stop) break;

    for (int step = 0; step < d - 1; ++step) {
      for (int i = tid; i < half; i += kJacThreads) {
        int a = rr_member(i, step, d), b = rr_member(d - 1 - i, step, d);
        if (a > b) { const int t = a; a = b; b = t; }
        pp[i] = a;
        qq[i] = b;
        const double apq = A[a * d + b];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double tau = (A[b * d + b] - A[a * d + a]) / (2.0 * apq);
          const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        cs[i] = c;
        sn[i] = s;
      }
      __syncthreads();
      // rows p, q  (A <- J^T A)
      for (int w = tid; w < half * d; w += kJacThreads) {
        const int i = w / d, j = w - i * d;
        const int a = pp[i], b = qq[i];
        const double c = cs[i], s = sn[i];
        const double ap = A[a * d + j], aq = A[b * d + j];
        A[a * d + j] = c * ap - s * aq;
        A[b * d + j] = s * ap + c * aq;
      }
      __syncthreads();
      // columns p, q  (A <- A J) and the eigenvector rows (V <- V J)
      for (int w = tid; w < half * d; w += kJacThreads) {
        const int i = w / d, j = w - i * d;
        const int a = pp[i], b = qq[i];
        const double c = cs[i], s = sn[i];
        const double ap = A[j * d + a], aq = A[j * d + b];
        A[j * d + a] = c * ap - s * aq;
        A[j * d + b] = s * ap + c * aq;
        const double vp = Vt[a * d + j], vq = Vt[b * d + j];
        Vt[a * d + j] = c * vp - s * vq;
        Vt[b * d + j] = s * vp + c * vq;
      }
      __syncthreads();
      for (int i = tid; i < half; i += kJacThreads) {
        A[pp[i] * d + qq[i]] = 0.0;
        A[qq[i] * d + pp[i]] = 0.0;
      }
      __syncthreads();
    }
  }

  // rank of each eigenvalue (descending, lower index first on ties)
  for (int k = tid; k < d; k += kJacThreads) {
    const double lk = A[k * d + k];
    int rank = 0;
    for (int j = 0; j < d; ++j) {
      const double lj = A[j * d + j];
      rank += (lj > lk) || (lj == lk && j < k);
    }
    if (rank < r) {
      const double* v = Vt + static_cast<size_t>(k) * d;
      int arg = 0;
      double best = fabs(v[0]);
      for (int c = 1; c < d; ++c)
        if (fabs(v[c]) > best) { best = fabs(v[c]); arg = c; }
      const double sgn = v[arg] < 0.0 ? -1.0 : 1.0;
      float* U = p.U + static_cast<size_t>(kv) * d * r;
      for (int c = 0; c < d; ++c) U[c * r + rank] = static_cast<float>(sgn * v[c]);
      if (p.eig) p.eig[kv * r + rank] = static_cast<float>(lk);
    }
  }
}

}  // namespace

cudaError_t launch_calibrate(const CalibrateParams& p, cudaStream_t s) {
  double* mean = p.vt + static_cast<size_t>(p.Hkv) * p.d * p.d;
  if (p.center) mean_kernel<<<p.Hkv, 128, 0, s>>>(p, mean);
  gram_kernel<<<dim3(p.d, p.Hkv), kGramThreads, 0, s>>>(p, mean);
  const size_t smem = sizeof(double) * (static_cast<size_t>(p.d) * p.d + p.d) +
                      sizeof(int) * p.d;
  cudaError_t e = cudaFuncSetAttribute(jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  jacobi_kernel<<<p.Hkv, kJacThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace headq
