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
//   gram kernel    C in fp64, one CTA per (32x32 tile pair, kv), the query rows
//                  staged through shared memory 32 at a time, the next 32 rows
//                  loaded into registers during the current slab's products
//   jacobi kernel  one CTA per kv: cyclic two-sided Jacobi rotations on the
//                  fp64 matrix in shared memory (Jacobi's method; rotation angle
//                  as in Golub & Van Loan, "Matrix Computations", symmetric Schur
//                  decomposition), the d/2 disjoint pairs of each step from the
//                  round-robin ("circle") schedule applied in parallel (one warp
//                  per pair for the row pass, one lane per pair for the column
//                  pass, two barriers per step), the rotations accumulated in
//                  fp32 rows of eigenvectors, also in shared memory; then the r
//                  largest eigenvalues, descending, and a sign rule per vector.
#include <math.h>

#include "headq_internal.cuh"

namespace headq {
namespace {

constexpr int kGramThreads = 128;
constexpr int kJacThreads = 512;
constexpr int kJacWarps = kJacThreads / 32;
constexpr int kJacPairsPerWarp = (128 / 2 + kJacWarps - 1) / kJacWarps;  // d <= 128
constexpr int kMaxSweeps = 40;

__global__ void mean_kernel(const CalibrateParams p, double* mean) {
  const int kv = blockIdx.x;
  const int d = p.d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double acc = 0.0;
    for (int n = 0; n < p.N; ++n)
      for (int g = 0; g < p.G; ++g)
        acc += load_elem(p.q, (static_cast<size_t>(n) * p.Hq + kv * p.G + g) * d + c, p.bf16);
    mean[kv * d + c] = acc / (static_cast<double>(p.N) * p.G);
  }
}

constexpr int kGT = 32;                        // Gram tile edge
constexpr int kGPer = kGT * kGT / kGramThreads;  // tile elements each thread stages

// C tile (i0.., j0..) of kv head: sum over the M = N*G query rows, j0 >= i0;
// the mirrored tile is written too.  Each thread stages the same column c of
// rows mm0 + 4k of every 32-row slab; the next slab is loaded into registers
// while the current one is multiplied.
__global__ void __launch_bounds__(kGramThreads)
gram_kernel(const CalibrateParams p, const double* mean) {
  const int kv = blockIdx.y;
  const int d = p.d, tiles = (d + kGT - 1) / kGT;
  int ti = 0, tj = blockIdx.x;  // linear index over the upper-triangle tile pairs
  while (tj >= tiles - ti) { tj -= tiles - ti; ++ti; }
  tj += ti;
  const int i0 = ti * kGT, j0 = tj * kGT;
  const int M = p.N * p.G;
  __shared__ double xi_s[kGT][kGT + 1];  // [row m][col i]
  __shared__ double xj_s[kGT][kGT + 1];
  const int tid = threadIdx.x;           // 128 threads: 8 x 16, each 4 x 2 outputs
  const int ry = tid / 16, rx = tid % 16;
  const int c = tid % kGT, mm0 = tid / kGT;
  const bool ci = i0 + c < d, cj = j0 + c < d;
  const double mi = (p.center && ci) ? mean[kv * d + i0 + c] : 0.0;
  const double mj = (p.center && cj) ? mean[kv * d + j0 + c] : 0.0;
  double va[kGPer], vb[kGPer];
  auto load = [&](int m0) {
#pragma unroll
    for (int k = 0; k < kGPer; ++k) {
      const int m = m0 + mm0 + 4 * k;
      va[k] = 0.0;
      vb[k] = 0.0;
      if (m < M) {
        const int n = m / p.G, g = m - n * p.G;
        const size_t row = (static_cast<size_t>(n) * p.Hq + kv * p.G + g) * d;
        if (ci) va[k] = load_elem(p.q, row + i0 + c, p.bf16) - mi;
        if (cj) vb[k] = load_elem(p.q, row + j0 + c, p.bf16) - mj;
      }
    }
  };
  double acc[4][2] = {};
  load(0);
  for (int m0 = 0; m0 < M; m0 += kGT) {
#pragma unroll
    for (int k = 0; k < kGPer; ++k) {
      xi_s[mm0 + 4 * k][c] = va[k];
      xj_s[mm0 + 4 * k][c] = vb[k];
    }
    __syncthreads();
    if (m0 + kGT < M) load(m0 + kGT);
#pragma unroll 4
    for (int mm = 0; mm < kGT; ++mm) {
      double xi[4], xj[2];
#pragma unroll
      for (int k = 0; k < 4; ++k) xi[k] = xi_s[mm][ry * 4 + k];
#pragma unroll
      for (int k = 0; k < 2; ++k) xj[k] = xj_s[mm][rx * 2 + k];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b2 = 0; b2 < 2; ++b2) acc[a][b2] = fma(xi[a], xj[b2], acc[a][b2]);
    }
    __syncthreads();
  }
  double* C = p.gram + static_cast<size_t>(kv) * d * d;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b2 = 0; b2 < 2; ++b2) {
      const int i = i0 + ry * 4 + a, j = j0 + rx * 2 + b2;
      if (i < d && j < d) {
        const double v = acc[a][b2] / static_cast<double>(M);
        C[static_cast<size_t>(i) * d + j] = v;
        C[static_cast<size_t>(j) * d + i] = v;
      }
    }
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
  float* Vt = reinterpret_cast<float*>(sn + half);  // [d][d] row k = eigenvector k
  int* pp = reinterpret_cast<int*>(Vt + d * d);     // [half]
  int* qq = pp + half;                              // [half]
  __shared__ double red[kJacThreads / 32];
  __shared__ int stop;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  for (int i = tid; i < d * d; i += kJacThreads) {
    A[i] = p.gram[static_cast<size_t>(kv) * d * d + i];
    Vt[i] = (i / d == i % d) ? 1.0f : 0.0f;
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
      // off-diagonal norm below 1e-8 of the total: converged.  Jacobi converges
      // quadratically near the end, so the eigenvalues then carry errors of order
      // 1e-16 of the total and the eigenvectors of order 1e-8 over the relative gap
      stop = (off_all <= 1e-16 * st) ? 1 : 0;
    }
    __syncthreads();
    if (stop) break;

    for (int step = 0; step < d - 1; ++step) {
      // rows p, q (A <- J^T A) and the eigenvector rows (V <- V J).  The warp
      // that owns a pair also forms its rotation: only that warp writes rows p
      // and q in this pass, so the three entries the angle needs are still the
      // ones the previous step left.  Pair i belongs to warp i % kJacWarps.
      // Lane k of a warp forms the rotation of the warp's k-th pair; then the
      // warp rotates its pairs' rows one pair at a time, the lanes along j.
      int a_l = 0, b_l = 0;
      double c_l = 1.0, s_l = 0.0;
      if (lane < kJacPairsPerWarp && warp + kJacWarps * lane < half) {
        const int i = warp + kJacWarps * lane;
        a_l = rr_member(i, step, d);
        b_l = rr_member(d - 1 - i, step, d);
        if (a_l > b_l) { const int t = a_l; a_l = b_l; b_l = t; }
        const double apq = A[a_l * d + b_l];
        if (apq != 0.0) {
          const double tau = (A[b_l * d + b_l] - A[a_l * d + a_l]) / (2.0 * apq);
          const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c_l = 1.0 / sqrt(1.0 + t * t);
          s_l = t * c_l;
        }
        pp[i] = a_l;
        qq[i] = b_l;
        cs[i] = c_l;
        sn[i] = s_l;
      }
      __syncwarp();  // the pivot entries are read before any row is written
#pragma unroll
      for (int k = 0; k < kJacPairsPerWarp; ++k) {
        if (warp + kJacWarps * k >= half) break;
        const int a = __shfl_sync(0xffffffffu, a_l, k), b = __shfl_sync(0xffffffffu, b_l, k);
        const double c = __shfl_sync(0xffffffffu, c_l, k), s = __shfl_sync(0xffffffffu, s_l, k);
        const float cf = static_cast<float>(c), sf = static_cast<float>(s);
        for (int j = lane; j < d; j += 32) {
          const double ap = A[a * d + j], aq = A[b * d + j];
          A[a * d + j] = c * ap - s * aq;
          A[b * d + j] = s * ap + c * aq;
          const float vp = Vt[a * d + j], vq = Vt[b * d + j];
          Vt[a * d + j] = cf * vp - sf * vq;
          Vt[b * d + j] = sf * vp + cf * vq;
        }
      }
      __syncthreads();
      // columns p, q (A <- A J).  The pair index runs across lanes, so a warp
      // touches distinct columns of one row (a column walk strides d doubles and
      // puts every lane on one bank).  The pivot entries A[p][q] = A[q][p] are
      // set to exactly 0, the value the rotation annihilates them to.
      for (int i0 = 0; i0 < half; i0 += 32) {
        const int i = i0 + lane;
        if (i >= half) break;
        const int a = pp[i], b = qq[i];
        const double c = cs[i], s = sn[i];
        for (int j = warp; j < d; j += kJacWarps) {
          const double ap = A[j * d + a], aq = A[j * d + b];
          A[j * d + a] = j == b ? 0.0 : c * ap - s * aq;
          A[j * d + b] = j == a ? 0.0 : s * ap + c * aq;
        }
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
      const float* v = Vt + static_cast<size_t>(k) * d;
      int arg = 0;
      float best = fabsf(v[0]);
      for (int c = 1; c < d; ++c)
        if (fabsf(v[c]) > best) { best = fabsf(v[c]); arg = c; }
      const float sgn = v[arg] < 0.0f ? -1.0f : 1.0f;
      float* U = p.U + static_cast<size_t>(kv) * d * r;
      for (int c = 0; c < d; ++c) U[c * r + rank] = sgn * v[c];
      if (p.eig) p.eig[kv * r + rank] = static_cast<float>(lk);
    }
  }
}

}  // namespace

cudaError_t launch_calibrate(const CalibrateParams& p, cudaStream_t s) {
  double* mean = p.vt + static_cast<size_t>(p.Hkv) * p.d * p.d;
  if (p.center) mean_kernel<<<p.Hkv, 128, 0, s>>>(p, mean);
  const int tiles = (p.d + kGT - 1) / kGT;
  gram_kernel<<<dim3(tiles * (tiles + 1) / 2, p.Hkv), kGramThreads, 0, s>>>(p, mean);
  const size_t smem = sizeof(double) * (static_cast<size_t>(p.d) * p.d + p.d) +
                      sizeof(float) * static_cast<size_t>(p.d) * p.d + sizeof(int) * p.d;
  cudaError_t e = cudaFuncSetAttribute(jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  jacobi_kernel<<<p.Hkv, kJacThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace headq
