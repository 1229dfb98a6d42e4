// Block-incremental SVD update of a latent basis on the GPU (fp64 throughout).
//
// Method: iS-KV (title "Online Low-Rank KV Cache Compression via Block-Incremental SVD";
// method section, technical framework and key innovation: a dynamically updated low-rank
// basis kept current by an incremental SVD, with the historical coordinates synchronised to
// it).  The pages give no formula; the update is the textbook block update of a truncated
// SVD in the cache's terms (the same steps as the oracle's incsvd module):
//   state   B [r][D] basis rows, S [r][r] the Gram matrix of the history coordinates
//   block   K [n][D] exact rows
//   1  Y = K B^T                                   [n][r]
//   2  P = K - Y B                                 residual outside the basis
//   3  Q^T [k][D]: orthonormal rows spanning P's rows (k = its numerical rank), taken
//      orthogonal to B, and Rp^T = P Q            [n][k]
//   4  G = [[S + Y^T Y, Y^T Rp^T], [Rp Y, Rp Rp^T]]  ((r + k) square)
//   5  the r leading eigenpairs (lam, V) of G
//   out B' = V^T [B; Q^T],  R = V[:r, :] (history sync Z <- Z R),  S' = diag(lam)
//
// GPU structure.  The products of steps 1-5 and the output run as tiled fp64 GEMMs.  Step 3
// is Cholesky QR done twice: a Cholesky factorisation of P P^T with diagonal pivoting (the
// pivots below a threshold end the factorisation: that is the rank), forward substitution
// for the orthonormal rows, a projection off B, and the same again.  Step 5 reduces G to
// tridiagonal form with Householder reflections (one CTA), finds the r largest eigenvalues
// by bisection on Sturm counts (a thread per eigenvalue), their eigenvectors by inverse
// iteration on the tridiagonal matrix (a thread per eigenvector, orthogonalised against the
// earlier members of a cluster of nearly equal eigenvalues), and transforms them back with
// the reflections.  All sizes are fixed by (r, n): directions beyond the rank are zero rows,
// so the host never waits for a device result.
#include "lr_internal.cuh"
#include "k_common.cuh"

#include <algorithm>
#include <cmath>

namespace {

constexpr int kIsvdMaxRows = 128;   // block rows per update

// ---- tiled fp64 GEMM: C[M][N] = alpha op(A) op(B) + beta C ----------------------------------
// op(A)[i][k] = ta ? A[k * lda + i] : A[i * lda + k];  op(B)[k][j] = tb ? B[j * ldb + k] : B[k * ldb + j]
constexpr int kGT = 32;     // output tile
constexpr int kGK = 16;     // K step
__global__ void __launch_bounds__(256) k_gemm64(int M, int N, int K, double alpha, const double* A, int lda, int ta,
                                                const double* B, int ldb, int tb, double beta, double* C, int ldc) {
  __shared__ double As[kGK][kGT + 1];
  __shared__ double Bs[kGK][kGT + 1];
  const int i0 = blockIdx.y * kGT, j0 = blockIdx.x * kGT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16 threads, 2 x 2 outputs each
  double acc[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
  for (int k0 = 0; k0 < K; k0 += kGK) {
    for (int e = threadIdx.x; e < kGK * kGT; e += 256) {
      const int kk = e / kGT, ii = e % kGT;
      const int i = i0 + ii, k = k0 + kk;
      As[kk][ii] = (i < M && k < K) ? (ta ? A[(size_t)k * lda + i] : A[(size_t)i * lda + k]) : 0.0;
      const int j = j0 + ii;
      Bs[kk][ii] = (j < N && k < K) ? (tb ? B[(size_t)j * ldb + k] : B[(size_t)k * ldb + j]) : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      const double a0 = As[kk][ty], a1 = As[kk][ty + 16];
      const double b0 = Bs[kk][tx], b1 = Bs[kk][tx + 16];
      acc[0][0] = fma(a0, b0, acc[0][0]);
      acc[0][1] = fma(a0, b1, acc[0][1]);
      acc[1][0] = fma(a1, b0, acc[1][0]);
      acc[1][1] = fma(a1, b1, acc[1][1]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int i = i0 + ty + 16 * a, j = j0 + tx + 16 * b;
      if (i < M && j < N) {
        const size_t o = (size_t)i * ldc + j;
        C[o] = alpha * acc[a][b] + (beta == 0.0 ? 0.0 : beta * C[o]);
      }
    }
}

cudaError_t gemm64(int M, int N, int K, double alpha, const double* A, int lda, bool ta, const double* B, int ldb,
                   bool tb, double beta, double* C, int ldc, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  const dim3 grid((N + kGT - 1) / kGT, (M + kGT - 1) / kGT);
  return launch_serial(k_gemm64, grid, dim3(256), 0, s, M, N, K, alpha, A, lda, ta ? 1 : 0, B, ldb, tb ? 1 : 0, beta,
                       C, ldc);
}

// ---- conversions ----------------------------------------------------------------------------
__global__ void k_to_f64(const void* src, int dtype, double* dst, long long n) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = (double)elem_f(src, i, dtype);
}
__global__ void k_f32_to_f64(const float* src, double* dst, int rows, int cols, int ld_dst) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < rows * cols) dst[(size_t)(i / cols) * ld_dst + i % cols] = (double)src[i];
}

// the largest squared row norm of K [n][D] (one CTA: a warp per row, then the maximum)
__global__ void __launch_bounds__(256) k_rownorm_max(const double* K, int n, int D, double* out) {
  __shared__ double red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double best = 0.0;
  for (int i = warp; i < n; i += 8) {
    double acc = 0.0;
    for (int c = lane; c < D; c += 32) acc += K[(size_t)i * D + c] * K[(size_t)i * D + c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    best = fmax(best, acc);
  }
  if (lane == 0) red[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = red[0];
    for (int w = 1; w < 8; ++w) t = fmax(t, red[w]);
    *out = t;
  }
}

// ---- Cholesky QR step: pivoted Cholesky of the n x n Gram matrix C (one CTA, in place) -----
// C = Pi L L^T Pi^T; a pivot at or below rel * (*scale) ends the factorisation.  The factor
// grows in the finished columns of the shared-memory copy; written out as L (lower, row-major
// n x n, row i belongs to the i-th pivot, zero past the rank), perm[i] = the row of P that
// pivot i took, and *rank.
constexpr int kCholThreads = 256;
__global__ void __launch_bounds__(kCholThreads) k_pchol(const double* C, int n, const double* scale, double rel,
                                                        double* L, int* perm, int* rank) {
  extern __shared__ double cs[];          // [n][n + 1]
  __shared__ int piv_s[kIsvdMaxRows];
  __shared__ double best_v[kCholThreads / 32];
  __shared__ int best_i[kCholThreads / 32];
  __shared__ int pivot_s, stop_s;
  const int ld = n + 1, tid = threadIdx.x, nt = kCholThreads;
  for (int e = tid; e < n * n; e += nt) cs[(e / n) * ld + e % n] = C[e];
  for (int i = tid; i < n; i += nt) piv_s[i] = i;
  __syncthreads();
  const double tol = rel * *scale;
  int k = 0;
  for (; k < n; ++k) {
    double bv = -1.0;
    int bi = k;
    for (int i = k + tid; i < n; i += nt)
      if (cs[i * ld + i] > bv) { bv = cs[i * ld + i]; bi = i; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if ((tid & 31) == 0) { best_v[tid >> 5] = bv; best_i[tid >> 5] = bi; }
    __syncthreads();
    if (tid == 0) {
      double v = best_v[0];
      int p = best_i[0];
      for (int w = 1; w < nt / 32; ++w)
        if (best_v[w] > v || (best_v[w] == v && best_i[w] < p)) { v = best_v[w]; p = best_i[w]; }
      pivot_s = p;
      stop_s = !(v > tol);
    }
    __syncthreads();
    if (stop_s) break;
    const int p = pivot_s;
    if (p != k) {
      // swap rows k, p (every column: the finished L part and the trailing block), then
      // columns k, p of the trailing rows
      for (int j = tid; j < n; j += nt) {
        const double t = cs[k * ld + j]; cs[k * ld + j] = cs[p * ld + j]; cs[p * ld + j] = t;
      }
      __syncthreads();
      for (int i = k + tid; i < n; i += nt) {
        const double t = cs[i * ld + k]; cs[i * ld + k] = cs[i * ld + p]; cs[i * ld + p] = t;
      }
      if (tid == 0) { const int t = piv_s[k]; piv_s[k] = piv_s[p]; piv_s[p] = t; }
      __syncthreads();
    }
    const double lkk = sqrt(cs[k * ld + k]);
    __syncthreads();
    for (int i = k + 1 + tid; i < n; i += nt) cs[i * ld + k] /= lkk;
    if (tid == 0) cs[k * ld + k] = lkk;
    __syncthreads();
    for (int i = k + 1 + (tid >> 5); i < n; i += nt / 32) {
      const double lik = cs[i * ld + k];
      for (int j = k + 1 + (tid & 31); j < n; j += 32) cs[i * ld + j] -= lik * cs[j * ld + k];
    }
    __syncthreads();
  }
  for (int e = tid; e < n * n; e += nt) {
    const int i = e / n, j = e % n;
    L[e] = (j <= i && j < k) ? cs[i * ld + j] : 0.0;
  }
  for (int i = tid; i < n; i += nt) perm[i] = piv_s[i];
  if (tid == 0) *rank = k;
}

// Q[i] = (P[perm[i]] - sum_{j<i} L[i][j] Q[j]) / L[i][i] for i < rank; rows >= rank are zero.
// Thread = one column; a CTA's 32 columns of Q stay in shared memory during the substitution.
constexpr int kFwdCols = 32;
__global__ void __launch_bounds__(kFwdCols) k_fwd_subst(const double* L, const int* perm, const int* rank,
                                                        const double* P, double* Q, int n, int D) {
  extern __shared__ double fsm[];
  double* ls = fsm;                       // [n][n]
  double* qs = ls + (size_t)n * n;        // [n][kFwdCols]: P's rows in pivot order, then Q
  const int k = *rank;
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) ls[e] = L[e];
  const int c = blockIdx.x * kFwdCols + threadIdx.x;
  const bool live = c < D;
  for (int i = 0; i < k; ++i) qs[i * kFwdCols + threadIdx.x] = live ? P[(size_t)perm[i] * D + c] : 0.0;
  __syncthreads();
  for (int i = 0; i < n; ++i) {
    double v = 0.0;
    if (i < k && live) {
      double s0 = qs[i * kFwdCols + threadIdx.x], s1 = 0.0, s2 = 0.0, s3 = 0.0;
      const double* li = ls + (size_t)i * n;
      int j = 0;
      for (; j + 4 <= i; j += 4) {
        s0 -= li[j] * qs[j * kFwdCols + threadIdx.x];
        s1 -= li[j + 1] * qs[(j + 1) * kFwdCols + threadIdx.x];
        s2 -= li[j + 2] * qs[(j + 2) * kFwdCols + threadIdx.x];
        s3 -= li[j + 3] * qs[(j + 3) * kFwdCols + threadIdx.x];
      }
      for (; j < i; ++j) s0 -= li[j] * qs[j * kFwdCols + threadIdx.x];
      v = ((s0 + s1) + (s2 + s3)) / li[i];
    }
    qs[i * kFwdCols + threadIdx.x] = v;
    if (live) Q[(size_t)i * D + c] = v;
  }
}

// ---- Householder tridiagonalisation of the symmetric m x m matrix G (one cluster) -------------
// The rows of G are spread over the cluster's CTAs (CTA c holds rows [c rpc, +rpc) in shared
// memory).  Step k: every CTA reads row k (by symmetry, column k) from its owner through
// distributed shared memory and forms the reflection u (stored by the owner in U[k][k+1 ..])
// and tau; each CTA computes p_i = tau (A u)_i for its rows and its share of p^T u; after a
// cluster barrier every CTA gathers the whole p, forms w = p - (tau / 2)(p^T u) u and applies
// A -= u w^T + w u^T to its rows; a second barrier ends the step.  d / e: the tridiagonal.
__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cl_map(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ double cl_ld(uint32_t addr) {
  double v;
  asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(addr) : "memory");
  return v;
}

constexpr int kTriThreads = 512;
__global__ void __launch_bounds__(kTriThreads, 1) k_tridiag(const double* Gin, int m, int rpc, double* U, double* tau,
                                                          double* d, double* e) {
  extern __shared__ __align__(16) double tsm[];
  double* A = tsm;                        // [rpc][m] this CTA's rows
  double* u = A + (size_t)rpc * m;        // [m]
  double* pw = u + m;                     // [m] p of the gathered rows, then w
  double* pl = pw + m;                    // [rpc] p of this CTA's rows
  double* red = pl + rpc;                 // [32] reductions; red[16]: this CTA's share of p^T u
  const int cr = blockIdx.x, ncl = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = kTriThreads / 32;
  const int row0 = cr * rpc, nrow = max(0, min(rpc, m - row0));
  for (int li = warp; li < nrow; li += nw)
    for (int j = lane; j < m; j += 32) A[(size_t)li * m + j] = Gin[(size_t)(row0 + li) * m + j];
  cl_sync();
  auto bsum = [&](double v) -> double {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < nw; ++w) t += red[w];
    return t;
  };
  for (int k = 0; k < m - 2; ++k) {
    const int len = m - k - 1;
    const int owner = k / rpc;
    // row k (= column k) from its owner
    const uint32_t rk = cl_map(A + (size_t)(k - owner * rpc) * m, (uint32_t)owner);
    double ss = 0.0;
    for (int j = tid; j < len; j += kTriThreads) {
      const double x = cl_ld(rk + (uint32_t)((k + 1 + j) * 8));
      u[j] = x;
      ss += x * x;
    }
    const double nrm2 = bsum(ss);
    const double x0 = u[0];
    const double nrm = sqrt(nrm2);
    const double alpha = x0 >= 0.0 ? -nrm : nrm;
    const double u0 = x0 - alpha;
    const double unrm2 = nrm2 - x0 * x0 + u0 * u0;
    const double t = unrm2 > 0.0 ? 2.0 / unrm2 : 0.0;
    __syncthreads();
    if (tid == 0) u[0] = u0;
    if (cr == owner && tid == 0) {
      d[k] = A[(size_t)(k - owner * rpc) * m + k];
      e[k] = unrm2 > 0.0 ? alpha : x0;
      tau[k] = t;
    }
    __syncthreads();
    if (cr == owner)
      for (int j = tid; j < m; j += kTriThreads) U[(size_t)k * m + j] = j > k ? u[j - k - 1] : 0.0;
    if (t == 0.0) {   // column already reduced: nothing to apply (uniform over the cluster)
      cl_sync();
      continue;
    }
    // p_i = t (A u)_i for this CTA's rows i > k (a warp per row); share of p^T u
    double pu = 0.0;
    for (int li = warp; li < nrow; li += nw) {
      const int i = row0 + li;
      if (i <= k) continue;
      const double* row = A + (size_t)li * m + (k + 1);
      double acc = 0.0;
      for (int j = lane; j < len; j += 32) acc += row[j] * u[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const double pv = t * acc;
      if (lane == 0) {
        pl[li] = pv;
        pu += pv * u[i - k - 1];
      }
    }
    const double pu_cta = bsum(pu);
    if (tid == 0) red[16] = pu_cta;
    cl_sync();
    // gather p for every row > k and the shares of p^T u
    double put = 0.0;
    for (int c = 0; c < ncl; ++c) put += cl_ld(cl_map(red + 16, (uint32_t)c));
    const double K = 0.5 * t * put;
    for (int j = tid; j < len; j += kTriThreads) {
      const int i = k + 1 + j, c = i / rpc;
      const double pj = cl_ld(cl_map(pl + (i - c * rpc), (uint32_t)c));
      pw[j] = pj - K * u[j];
    }
    __syncthreads();
    // A -= u w^T + w u^T on this CTA's rows i > k, columns j > k
    for (int li = warp; li < nrow; li += nw) {
      const int i = row0 + li;
      if (i <= k) continue;
      const int ii = i - k - 1;
      const double ui = u[ii], wi = pw[ii];
      double* row = A + (size_t)li * m + k + 1;
      for (int j = lane; j < len; j += 32) row[j] -= ui * pw[j] + wi * u[j];
    }
    cl_sync();
  }
  // the last 2 x 2 block
  for (int i = m - 2; i < m; ++i) {
    if (i < 0) continue;
    if (cr == i / rpc && tid == 0) {
      const double* row = A + (size_t)(i - cr * rpc) * m;
      d[i] = row[i];
      if (i == m - 1 && m >= 2) e[m - 2] = row[m - 2];
    }
  }
  if (cr == 0)
    for (int k = max(0, m - 2); k < m; ++k) {
      for (int j = tid; j < m; j += kTriThreads) U[(size_t)k * m + j] = 0.0;
      if (tid == 0) tau[k] = 0.0;
    }
  cl_sync();   // no CTA leaves while another may still read its rows
}

// ---- eigenvalues: the r largest of the tridiagonal (d, e) by bisection (thread per value) ----
__device__ int sturm_below(const double* d, const double* e, int m, double x) {
  // number of eigenvalues below x: negative pivots of the LDL^T factorisation of T - x I
  int cnt = 0;
  double q = d[0] - x;
  if (q < 0.0) ++cnt;
  for (int i = 1; i < m; ++i) {
    const double qq = q != 0.0 ? q : 1e-300;
    q = d[i] - x - e[i - 1] * e[i - 1] / qq;
    if (q < 0.0) ++cnt;
  }
  return cnt;
}

// A warp per eigenvalue: each round evaluates the Sturm count at 31 interior points of the
// current interval (one per lane) and keeps the sub-interval that holds the eigenvalue, so
// 11 rounds shrink it by 2^-55.  d / e are staged in shared memory.
__global__ void __launch_bounds__(256) k_bisect(const double* d, const double* e, int m, int r, double* lam) {
  extern __shared__ double de[];          // d [m], e [m]
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    de[i] = d[i];
    de[m + i] = i < m - 1 ? e[i] : 0.0;
  }
  __syncthreads();
  const double* ds = de;
  const double* es = de + m;
  const int lane = threadIdx.x & 31;
  const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);   // j-th largest
  if (j >= r) return;
  double lo = 1e300, hi = -1e300;
  for (int i = lane; i < m; i += 32) {
    const double rad = (i > 0 ? fabs(es[i - 1]) : 0.0) + (i < m - 1 ? fabs(es[i]) : 0.0);
    lo = fmin(lo, ds[i] - rad);
    hi = fmax(hi, ds[i] + rad);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const double span = fmax(hi - lo, 1e-300);
  lo -= 1e-12 * span;
  hi += 1e-12 * span;
  const int target = m - 1 - j;           // 0-based index from the bottom
  for (int it = 0; it < 16; ++it) {
    const double step = (hi - lo) / 32.0;
    const double x = lo + step * (lane + 1);       // lanes 0..30: interior points
    const int below = lane < 31 ? sturm_below(ds, es, m, x) : m + 1;
    // the first point with more than `target` eigenvalues below it bounds the eigenvalue above
    const unsigned mask = __ballot_sync(0xffffffffu, below > target);
    const int first = __ffs(mask) - 1;             // 0..31 (31: the upper end)
    const double nlo = first == 0 ? lo : lo + step * first;
    const double nhi = first == 31 ? hi : lo + step * (first + 1);
    lo = nlo;
    hi = nhi;
    if (hi - lo <= 4e-16 * fmax(fabs(lo), fabs(hi)) + 1e-300) break;
  }
  if (lane == 0) lam[j] = 0.5 * (lo + hi);
}

// ---- eigenvectors of the tridiagonal by inverse iteration (thread per cluster) --------------
// Thread j handles eigenvalue j when it starts a cluster (j == 0 or lam[j-1] - lam[j] above the
// cluster gap) and then every member of the cluster, orthogonalising each iterate against the
// cluster's earlier vectors.  kInvThreads threads per CTA, each with its LU factors and iterate
// in shared memory ([5][m] doubles).
constexpr int kInvThreads = 4;
__global__ void __launch_bounds__(32) k_inviter(const double* d, const double* e, int m, int r, const double* lam,
                                                double gap_rel, double* X) {
  extern __shared__ double isc[];
  const int j0 = blockIdx.x * kInvThreads + threadIdx.x;
  if (threadIdx.x >= kInvThreads || j0 >= r) return;
  double* a = isc + (size_t)threadIdx.x * 5 * m;   // U diagonal
  double* b = a + m;                               // first superdiagonal
  double* c = b + m;                               // second superdiagonal (from interchanges)
  double* l = c + m;                               // multipliers (interchange: mult + 4)
  double* x = l + m;                               // iterate
  double tn = 0.0;
  for (int i = 0; i < m; ++i) tn = fmax(tn, fabs(d[i]) + (i < m - 1 ? fabs(e[i]) : 0.0) + (i > 0 ? fabs(e[i - 1]) : 0.0));
  const double gap = gap_rel * tn;
  if (j0 > 0 && lam[j0 - 1] - lam[j0] <= gap) return;   // not the first of its cluster
  int j1 = j0 + 1;
  while (j1 < r && lam[j1 - 1] - lam[j1] <= gap) ++j1;
  const double tiny = 1e-300 + 1e-15 * tn;
  for (int jj = j0; jj < j1; ++jj) {
    const double lmb = lam[jj];
    // T - lmb I = P L U by Gaussian elimination with partial pivoting on the tridiagonal
    double dcur = d[0] - lmb, ecur = m > 1 ? e[0] : 0.0;
    for (int i = 0; i < m; ++i) {
      const double sub = i < m - 1 ? e[i] : 0.0;                  // T[i+1][i]
      const double dn = i < m - 1 ? d[i + 1] - lmb : 0.0;         // T[i+1][i+1]
      const double en = i < m - 2 ? e[i + 1] : 0.0;               // T[i+1][i+2]
      if (i < m - 1 && fabs(sub) > fabs(dcur)) {
        a[i] = sub;
        b[i] = dn;
        c[i] = en;
        const double mult = dcur / sub;                           // |mult| < 1
        dcur = ecur - mult * dn;
        ecur = -mult * en;
        l[i] = mult + 4.0;                                        // interchange marked: 3 < mult + 4 < 5
      } else {
        a[i] = fabs(dcur) > tiny ? dcur : (dcur < 0.0 ? -tiny : tiny);
        b[i] = ecur;
        c[i] = 0.0;
        const double mult = i < m - 1 ? sub / a[i] : 0.0;
        l[i] = mult;                                              // |mult| <= 1
        dcur = dn - mult * ecur;
        ecur = en;
      }
    }
    for (int i = 0; i < m; ++i) x[i] = 1.0 + 0.01 * (double)((i * 7 + jj * 13) % 17);
    for (int iter = 0; iter < 4; ++iter) {
      for (int i = 0; i < m - 1; ++i) {
        const double mv = l[i];
        if (mv >= 3.0) {
          const double mult = mv - 4.0;
          const double xi = x[i], xn = x[i + 1];
          x[i] = xn;
          x[i + 1] = xi - mult * xn;
        } else {
          x[i + 1] -= mv * x[i];
        }
      }
      for (int i = m - 1; i >= 0; --i) {
        double v = x[i];
        if (i + 1 < m) v -= b[i] * x[i + 1];
        if (i + 2 < m) v -= c[i] * x[i + 2];
        x[i] = v / a[i];
      }
      for (int q = j0; q < jj; ++q) {
        const double* xq = X + (size_t)q * m;
        double dot = 0.0;
        for (int i = 0; i < m; ++i) dot += xq[i] * x[i];
        for (int i = 0; i < m; ++i) x[i] -= dot * xq[i];
      }
      double nrm = 0.0;
      for (int i = 0; i < m; ++i) nrm += x[i] * x[i];
      const double inv = nrm > 0.0 ? 1.0 / sqrt(nrm) : 0.0;
      for (int i = 0; i < m; ++i) x[i] *= inv;
    }
    for (int i = 0; i < m; ++i) X[(size_t)jj * m + i] = x[i];
    __threadfence_block();
  }
}

// ---- back-transformation: X[j] <- H_0 H_1 ... H_{m-3} X[j], then a sign convention -----------
// (the component of largest magnitude positive).  CTA = kBtVecs eigenvectors (a warp each),
// each reflection vector staged in shared memory once for them.
constexpr int kBtVecs = 4;
constexpr int kBtStage = 8;               // reflection vectors staged together
__global__ void __launch_bounds__(32 * kBtVecs) k_backtrans(const double* U, const double* tau, int m, int r, double* X) {
  extern __shared__ double xs[];          // [kBtVecs][m] vectors, then [kBtStage][m] reflections
  double* us = xs + (size_t)kBtVecs * m;
  const int j0 = blockIdx.x * kBtVecs, nj = min(kBtVecs, r - j0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int idx = tid; idx < nj * m; idx += blockDim.x) xs[idx] = X[(size_t)(j0 + idx / m) * m + idx % m];
  // reflections k = m - 3 .. 0 in groups of kBtStage (highest first)
  for (int kh = m - 3; kh >= 0; kh -= kBtStage) {
    const int kl = max(0, kh - kBtStage + 1);
    __syncthreads();                      // the previous group's reads are done
    for (int q = 0; q <= kh - kl; ++q)
      for (int i = tid; i < m; i += blockDim.x) us[(size_t)q * m + i] = U[(size_t)(kh - q) * m + i];
    __syncthreads();
    if (warp < nj) {
      double* xv = xs + (size_t)warp * m;
      for (int q = 0; q <= kh - kl; ++q) {
        const int k = kh - q;
        const double t = tau[k];
        if (t == 0.0) continue;
        const double* uq = us + (size_t)q * m;
        double acc = 0.0;
        for (int i = k + 1 + lane; i < m; i += 32) acc += uq[i] * xv[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        const double w = t * acc;
        for (int i = k + 1 + lane; i < m; i += 32) xv[i] -= w * uq[i];
        __syncwarp();
      }
    }
  }
  __syncthreads();
  if (warp < nj) {
    const double* xv = xs + (size_t)warp * m;
    double best = 0.0;
    for (int i = lane; i < m; i += 32)
      if (fabs(xv[i]) > fabs(best)) best = xv[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, o);
      if (fabs(ob) > fabs(best) || (fabs(ob) == fabs(best) && ob > best)) best = ob;
    }
    const double sg = best < 0.0 ? -1.0 : 1.0;
    for (int i = lane; i < m; i += 32) X[(size_t)(j0 + warp) * m + i] = sg * xv[i];
  }
}

// ---- outputs --------------------------------------------------------------------------------
// R [r][r] fp32: R[i][j] = v_j[i]; S' = diag(lam) fp32.
__global__ void k_isvd_small_out(const double* X, const double* lam, int m, int r, float* R, float* S) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= r * r) return;
  const int i = e / r, j = e % r;
  R[e] = (float)X[(size_t)j * m + i];
  S[e] = i == j ? (float)lam[i] : 0.f;
}
// B' [r][D] and A' = B'^T [D][r] in the cache dtype
__global__ void k_isvd_basis_out(const double* Bn, int r, int D, int dtype, void* Bout, void* Aout) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)r * D) return;
  const int i = (int)(e / D), c = (int)(e % D);
  const float v = (float)Bn[e];
  if (Bout) store_elem(Bout, e, v, dtype);
  if (Aout) store_elem(Aout, (long long)c * r + i, v, dtype);
}

struct IsvdWork {
  int r = 0, D = 0;                       // sizes the buffers were made for
  double* base = nullptr;
  double *Bd, *Kd, *Y, *P, *C, *L, *Q1, *Q2, *T, *Rpt, *G, *U, *tau, *dd, *ee, *lam, *X, *inv, *Bn;
  int* ibuf = nullptr;                    // perm [n], rank
};

}  // namespace

// Per-cache working memory of the update, made on first use for the larger rank.
void isvd_release(lr_cache* c) {
  IsvdWork* w = reinterpret_cast<IsvdWork*>(c->isvd_state);
  if (w) {
    if (w->base) cudaFree(w->base);
    if (w->ibuf) cudaFree(w->ibuf);
    delete w;
  }
  c->isvd_state = nullptr;
}

static cudaError_t isvd_work(lr_cache* c, IsvdWork** out) {
  const int r = std::max(c->desc.rank_k, c->desc.rank_v), D = c->D, n = kIsvdMaxRows, m = r + n;
  IsvdWork* w = reinterpret_cast<IsvdWork*>(c->isvd_state);
  if (w && w->r == r && w->D == D) {
    *out = w;
    return cudaSuccess;
  }
  isvd_release(c);
  w = new (std::nothrow) IsvdWork();
  if (!w) return cudaErrorMemoryAllocation;
  const size_t sz[] = {(size_t)r * D, (size_t)n * D, (size_t)n * r, (size_t)n * D, (size_t)n * n, (size_t)n * n,
                       (size_t)n * D, (size_t)n * D, (size_t)n * r, (size_t)n * n, (size_t)m * m, (size_t)m * m,
                       (size_t)m, (size_t)m, (size_t)m, (size_t)r, (size_t)r * m, (size_t)5 * m * r, (size_t)r * D};
  size_t total = 0;
  for (size_t s : sz) total += (s + 1) / 2 * 2;   // 16-byte aligned pieces
  cudaError_t e = lr_dev_malloc(&w->base, total * sizeof(double));
  if (e == cudaSuccess) e = lr_dev_malloc(&w->ibuf, (size_t)(n + 1) * sizeof(int));
  if (e != cudaSuccess) {
    if (w->base) cudaFree(w->base);
    delete w;
    return e;
  }
  double** ptrs[] = {&w->Bd, &w->Kd, &w->Y, &w->P, &w->C, &w->L, &w->Q1, &w->Q2, &w->T, &w->Rpt,
                     &w->G, &w->U, &w->tau, &w->dd, &w->ee, &w->lam, &w->X, &w->inv, &w->Bn};
  size_t off = 0;
  for (int i = 0; i < 19; ++i) {
    *ptrs[i] = w->base + off;
    off += (sz[i] + 1) / 2 * 2;
  }
  w->r = r;
  w->D = D;
  c->isvd_state = w;
  *out = w;
  return cudaSuccess;
}

cudaError_t launch_basis_update(lr_cache* c, int side, const void* blk, int n, float* gram, float* R_out,
                                void* B_out, void* A_out, cudaStream_t s) {
  const int r = side ? c->desc.rank_v : c->desc.rank_k, D = c->D, m = r + n;
  const int dtype = c->desc.dtype;
  IsvdWork* w = nullptr;
  cudaError_t e = isvd_work(c, &w);
  if (e != cudaSuccess) return e;
  int* perm = w->ibuf;
  int* rank = w->ibuf + n;
  const void* Bsrc = side ? c->B_v : c->B_k;
  auto blocks = [](long long count, int t) { return (unsigned)((count + t - 1) / t); };
  static std::atomic<uint32_t> o1{0}, o2{0}, o3{0}, o4{0}, o5{0};
  e = smem_optin(k_pchol, o1);
  if (e == cudaSuccess) e = smem_optin(k_fwd_subst, o2);
  if (e == cudaSuccess) e = smem_optin(k_tridiag, o3);
  if (e == cudaSuccess) e = smem_optin(k_backtrans, o4);
  if (e == cudaSuccess) e = smem_optin(k_inviter, o5);
  // fp64 copies of the basis and the block
  if (e == cudaSuccess)
    e = launch_serial(k_to_f64, dim3(blocks((long long)r * D, 256)), dim3(256), 0, s, Bsrc, dtype, w->Bd, (long long)r * D);
  if (e == cudaSuccess)
    e = launch_serial(k_to_f64, dim3(blocks((long long)n * D, 256)), dim3(256), 0, s, blk, dtype, w->Kd, (long long)n * D);
  double* scale = w->lam;   // the block's largest squared row norm (lam is written later)
  if (e == cudaSuccess) e = launch_serial(k_rownorm_max, dim3(1), dim3(256), 0, s, (const double*)w->Kd, n, D, scale);
  // 1. Y = K B^T;  2. P = K - Y B
  if (e == cudaSuccess) e = gemm64(n, r, D, 1.0, w->Kd, D, false, w->Bd, D, true, 0.0, w->Y, r, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(w->P, w->Kd, (size_t)n * D * sizeof(double), cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = gemm64(n, D, r, -1.0, w->Y, r, false, w->Bd, D, false, 1.0, w->P, D, s);
  // 3. Q2 [n][D]: orthonormal rows spanning P's rows (rows past the rank zero), two passes of
  //    Cholesky QR with a projection off B between them; a residual direction whose squared
  //    norm is at most 1e-12 of the block's largest squared row norm is dropped
  const size_t chol_smem = (size_t)n * (n + 1) * sizeof(double);
  const size_t fwd_smem = ((size_t)n * n + (size_t)n * kFwdCols) * sizeof(double);
  const dim3 fgrid(blocks(D, kFwdCols));
  for (int pass = 0; pass < 2 && e == cudaSuccess; ++pass) {
    const double* src = pass == 0 ? w->P : w->Q1;
    double* dst = pass == 0 ? w->Q1 : w->Q2;
    e = gemm64(n, n, D, 1.0, src, D, false, src, D, true, 0.0, w->C, n, s);
    if (e == cudaSuccess)
      e = launch_serial(k_pchol, dim3(1), dim3(kCholThreads), chol_smem, s, (const double*)w->C, n, (const double*)scale,
                        pass == 0 ? 1e-12 : 1e-24, w->L, perm, rank);
    if (e == cudaSuccess)
      e = launch_serial(k_fwd_subst, fgrid, dim3(kFwdCols), fwd_smem, s, (const double*)w->L, (const int*)perm,
                        (const int*)rank, src, dst, n, D);
    if (e == cudaSuccess && pass == 0) {
      // Q1 <- Q1 - (Q1 B^T) B
      e = gemm64(n, r, D, 1.0, w->Q1, D, false, w->Bd, D, true, 0.0, w->T, r, s);
      if (e == cudaSuccess) e = gemm64(n, D, r, -1.0, w->T, r, false, w->Bd, D, false, 1.0, w->Q1, D, s);
    }
  }
  // Rp^T = P Q2^T [n][n]
  if (e == cudaSuccess) e = gemm64(n, n, D, 1.0, w->P, D, false, w->Q2, D, true, 0.0, w->Rpt, n, s);
  // 4. G [m][m] = [[S + Y^T Y, Y^T Rp^T], [Rp Y, Rp Rp^T]]
  if (e == cudaSuccess)
    e = launch_serial(k_f32_to_f64, dim3(blocks((long long)r * r, 256)), dim3(256), 0, s, (const float*)gram, w->G, r,
                      r, m);
  if (e == cudaSuccess) e = gemm64(r, r, n, 1.0, w->Y, r, true, w->Y, r, false, 1.0, w->G, m, s);
  if (e == cudaSuccess) e = gemm64(r, n, n, 1.0, w->Y, r, true, w->Rpt, n, false, 0.0, w->G + r, m, s);
  if (e == cudaSuccess) e = gemm64(n, r, n, 1.0, w->Rpt, n, true, w->Y, r, false, 0.0, w->G + (size_t)r * m, m, s);
  if (e == cudaSuccess) e = gemm64(n, n, n, 1.0, w->Rpt, n, true, w->Rpt, n, false, 0.0, w->G + (size_t)r * m + r, m, s);
  // 5. eigenpairs: tridiagonalisation (one cluster), bisection, inverse iteration,
  //    back-transformation
  if (e == cudaSuccess) {
    const int ncl = m <= 448 ? 8 : 16;
    const int rpc = (m + ncl - 1) / ncl;
    const size_t tsm = ((size_t)rpc * m + 2 * (size_t)m + rpc + 32) * sizeof(double);
    static std::atomic<int> nonportable{0};
    if (ncl > 8 && !nonportable.load()) {
      e = cudaFuncSetAttribute(k_tridiag, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e == cudaSuccess) nonportable.store(1);
    }
    if (e == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(ncl);
      cfg.blockDim = dim3(kTriThreads);
      cfg.dynamicSmemBytes = tsm;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)ncl;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (lr_fault_launch()) e = cudaErrorLaunchFailure;
      else {
        lr_count_launch();
        e = cudaLaunchKernelEx(&cfg, k_tridiag, (const double*)w->G, m, rpc, w->U, w->tau, w->dd, w->ee);
      }
    }
  }
  if (e == cudaSuccess)
    e = launch_serial(k_bisect, dim3(blocks(r, 8)), dim3(256), (size_t)2 * m * sizeof(double), s, (const double*)w->dd,
                      (const double*)w->ee, m, r, w->lam);
  if (e == cudaSuccess)
    e = launch_serial(k_inviter, dim3(blocks(r, kInvThreads)), dim3(32), (size_t)kInvThreads * 5 * m * sizeof(double), s,
                      (const double*)w->dd, (const double*)w->ee, m, r, (const double*)w->lam, 1e-10, w->X);
  if (e == cudaSuccess)
    e = launch_serial(k_backtrans, dim3(blocks(r, kBtVecs)), dim3(32 * kBtVecs),
                      (size_t)(kBtVecs + kBtStage) * m * sizeof(double), s, (const double*)w->U, (const double*)w->tau, m, r,
                      w->X);
  // outputs: R, S', B' = V^T [B; Q2] (X holds V^T: row j = v_j), A' = B'^T
  if (e == cudaSuccess)
    e = launch_serial(k_isvd_small_out, dim3(blocks((long long)r * r, 256)), dim3(256), 0, s, (const double*)w->X,
                      (const double*)w->lam, m, r, R_out, gram);
  if (e == cudaSuccess) e = gemm64(r, D, r, 1.0, w->X, m, false, w->Bd, D, false, 0.0, w->Bn, D, s);
  if (e == cudaSuccess) e = gemm64(r, D, n, 1.0, w->X + r, m, false, w->Q2, D, false, 1.0, w->Bn, D, s);
  if (e == cudaSuccess)
    e = launch_serial(k_isvd_basis_out, dim3(blocks((long long)r * D, 256)), dim3(256), 0, s, (const double*)w->Bn, r,
                      D, dtype, B_out, A_out);
  return e;
}
