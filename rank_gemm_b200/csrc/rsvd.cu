// rsvd.cu -- the low-rank split of W^ = diag(lambda) W on the device (offline
// weight preparation without caller-supplied factors).
//
// The pages split W^ by an SVD into the rank-r 16-bit branch and the residual
// (SVDQuant overview figure, Stage 3, "svdq-int4-flux.1-dev" model card).
// Here the split is the randomized range finder with subspace iteration of
// Halko, Martinsson and Tropp, "Finding structure with randomness" (SIAM
// Review 2011, Algorithms 4.4 and 5.1), in float64:
//   Omega = Rademacher N x l (l = min(r + 8, K, N)) from a Philox4x32-10
//     stream (Salmon et al., SC 2011): entry (n, j) is the top bit of word
//     e = n l + j, block e / 4 at counter (block lo, block hi, 0, 0), key
//     (seed lo, seed hi);
//   Q = orth(W^ Omega); 3 times: Z = orth(W^T Q), Q = orth(W^ Z);
//   Z = W^T Q;  T = Z^T Z = P diag(e) P^T (descending);  sigma = sqrt(e);
//   U = Q P, V = Z P / sigma;  each column of V signed so its largest-|.|
//   entry is positive (first index wins);
//   L1f = bf16(diag(lambda)^-1 U_r Sigma_r), L2 = bf16(V_r^T).
// orth() is CholeskyQR2: twice G = Y^T Y, G = R^T R, Y <- Y R^-1 (a Gram
// matrix that is not positive definite is factored with 2^-40 trace(G) added
// to its diagonal).  The products with W^ (K x N) and the tall-skinny
// products run as float64 tiled GEMMs on the GPU; the l x l Cholesky
// factorizations, triangular inverses and the symmetric eigenproblem (cyclic
// Jacobi) run on the host, in float64, on matrices of at most 264 x 264.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int GT = 64, GK = 16;   // GEMM tile: 64 x 64 outputs, 16-deep k slices; 256 threads, 4 x 4 each

// ---------------------------------------------------------------- device kernels
__device__ __forceinline__ void philox_round(uint32_t (&c)[4], uint32_t k0, uint32_t k1) {
  const uint64_t p0 = (uint64_t)0xD2511F53u * c[0], p1 = (uint64_t)0xCD9E8D57u * c[2];
  const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0, hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
  c[0] = hi1 ^ c[1] ^ k0;
  c[1] = lo1;
  c[2] = hi0 ^ c[3] ^ k1;
  c[3] = lo0;
}

__global__ void rademacher_kernel(double* omega, long long n_words, uint64_t seed) {
  const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // Philox block: 4 words
  if (b * 4 >= n_words) return;
  uint32_t c[4] = {(uint32_t)b, (uint32_t)((uint64_t)b >> 32), 0u, 0u};
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    philox_round(c, k0, k1);
  }
  for (int w = 0; w < 4; ++w)
    if (b * 4 + w < n_words) omega[b * 4 + w] = (c[w] >> 31) ? -1.0 : 1.0;
}

// What[k][n] = lambda_k * W[k][n], W given as W_t[n][k]; 32 x 32 tiles through shared memory
__global__ void what_kernel(const __nv_bfloat16* __restrict__ Wt, const float* __restrict__ lam, double* What, int K,
                            int N) {
  __shared__ double tile[32][33];
  const int k0 = blockIdx.x * 32, n0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int n = n0 + i, k = k0 + threadIdx.x;
    tile[i][threadIdx.x] = (n < N && k < K) ? (double)__bfloat162float(Wt[(size_t)n * K + k]) : 0.0;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int k = k0 + i, n = n0 + threadIdx.x;
    if (k < K && n < N) What[(size_t)k * N + n] = (double)lam[k] * tile[threadIdx.x][i];
  }
}

// C[i][j] = sum_k A(i, k) B(k, j) in float64, A(i, k) = A[i sai + k sak],
// B(k, j) = B[k sbk + j sbj], C row-major with leading dimension ldc.
__global__ void __launch_bounds__(256) dgemm_kernel(int M, int Nc, int Kd, const double* __restrict__ A, long long sai,
                                                    long long sak, const double* __restrict__ B, long long sbk,
                                                    long long sbj, double* __restrict__ C, long long ldc) {
  __shared__ double As[GK][GT + 1];
  __shared__ double Bs[GK][GT + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int i0 = blockIdx.y * GT, j0 = blockIdx.x * GT;
  double acc[4][4] = {};
  for (int k0 = 0; k0 < Kd; k0 += GK) {
    for (int e = threadIdx.x; e < GK * GT; e += 256) {
      // A: consecutive threads walk i when A is stored k-major (sak == 1 walks k)
      const int kk = sak == 1 ? e % GK : e / GT, ii = sak == 1 ? e / GK : e % GT;
      const int gi = i0 + ii, gk = k0 + kk;
      As[kk][ii] = (gi < M && gk < Kd) ? A[gi * sai + gk * sak] : 0.0;
      const int kb = sbj == 1 ? e / GT : e % GK, jj = sbj == 1 ? e % GT : e / GK;
      const int gj = j0 + jj, gk2 = k0 + kb;
      Bs[kb][jj] = (gj < Nc && gk2 < Kd) ? B[gk2 * sbk + gj * sbj] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GK; ++kk) {
      double a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = As[kk][ty + 16 * u];
        b[u] = Bs[kk][tx + 16 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int i = i0 + ty + 16 * u, j = j0 + tx + 16 * v;
      if (i < M && j < Nc) C[i * ldc + j] = acc[u][v];
    }
}

// L1f[k][i] = bf16(U[k][i] sigma_i sgn_i / lambda_k), L2[i][n] = bf16(V[n][i] sgn_i), i < r
__global__ void fold_kernel(const double* __restrict__ U, const double* __restrict__ V, const double* __restrict__ ss,
                            const float* __restrict__ lam, int K, int N, int l, int r, __nv_bfloat16* L1f,
                            __nv_bfloat16* L2) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < (long long)K * r; e += stride) {
    const int k = (int)(e / r), i = (int)(e % r);
    L1f[e] = __double2bfloat16(U[(size_t)k * l + i] * ss[i] / (double)lam[k]);
  }
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < (long long)r * N; e += stride) {
    const int i = (int)(e / N), n = (int)(e % N);
    L2[e] = __double2bfloat16(V[(size_t)n * l + i] * (signbit(ss[i]) ? -1.0 : 1.0));
  }
}

// ---------------------------------------------------------------- host helpers
cudaError_t dgemm(int M, int Nc, int Kd, const double* A, long long sai, long long sak, const double* B, long long sbk,
                  long long sbj, double* C, long long ldc, cudaStream_t s) {
  dim3 grid((Nc + GT - 1) / GT, (M + GT - 1) / GT);
  dgemm_kernel<<<grid, 256, 0, s>>>(M, Nc, Kd, A, sai, sak, B, sbk, sbj, C, ldc);
  return cudaGetLastError();
}

// G = R^T R, R upper triangular (row-major n x n); false if not positive definite
bool cholesky_upper(const std::vector<double>& G, std::vector<double>& R, int n) {
  R.assign((size_t)n * n, 0.0);
  for (int j = 0; j < n; ++j) {
    double d = G[(size_t)j * n + j];
    for (int k = 0; k < j; ++k) d -= R[(size_t)k * n + j] * R[(size_t)k * n + j];
    if (!(d > 0.0)) return false;
    const double rjj = std::sqrt(d);
    R[(size_t)j * n + j] = rjj;
    for (int i = j + 1; i < n; ++i) {
      double v = G[(size_t)j * n + i];
      for (int k = 0; k < j; ++k) v -= R[(size_t)k * n + j] * R[(size_t)k * n + i];
      R[(size_t)j * n + i] = v / rjj;
    }
  }
  return true;
}

// inverse of an upper-triangular R (row-major), by back substitution
void upper_inverse(const std::vector<double>& R, std::vector<double>& Ri, int n) {
  Ri.assign((size_t)n * n, 0.0);
  for (int c = 0; c < n; ++c) {
    for (int i = c; i >= 0; --i) {
      double v = (i == c) ? 1.0 : 0.0;
      for (int k = i + 1; k <= c; ++k) v -= R[(size_t)i * n + k] * Ri[(size_t)k * n + c];
      Ri[(size_t)i * n + c] = v / R[(size_t)i * n + i];
    }
  }
}

// symmetric eigenproblem by cyclic Jacobi rotations: A = P diag(e) P^T
void jacobi_eig(std::vector<double> A, int n, std::vector<double>& e, std::vector<double>& P) {
  P.assign((size_t)n * n, 0.0);
  for (int i = 0; i < n; ++i) P[(size_t)i * n + i] = 1.0;
  for (int sweep = 0; sweep < 60; ++sweep) {
    double off = 0.0, diag = 0.0;
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) (i == j ? diag : off) += A[(size_t)i * n + j] * A[(size_t)i * n + j];
    // off-diagonal norm below 1e-13 of the diagonal's: eigenvalues to ~1e-26, vectors to ~1e-13
    if (off <= 1e-26 * diag) break;
    for (int p = 0; p < n - 1; ++p)
      for (int q = p + 1; q < n; ++q) {
        const double apq = A[(size_t)p * n + q];
        if (apq == 0.0) continue;
        const double app = A[(size_t)p * n + p], aqq = A[(size_t)q * n + q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < n; ++k) {   // A <- J^T A J on rows/columns p, q
          const double akp = A[(size_t)k * n + p], akq = A[(size_t)k * n + q];
          A[(size_t)k * n + p] = c * akp - s * akq;
          A[(size_t)k * n + q] = s * akp + c * akq;
        }
        for (int k = 0; k < n; ++k) {
          const double apk = A[(size_t)p * n + k], aqk = A[(size_t)q * n + k];
          A[(size_t)p * n + k] = c * apk - s * aqk;
          A[(size_t)q * n + k] = s * apk + c * aqk;
        }
        for (int k = 0; k < n; ++k) {
          const double pkp = P[(size_t)k * n + p], pkq = P[(size_t)k * n + q];
          P[(size_t)k * n + p] = c * pkp - s * pkq;
          P[(size_t)k * n + q] = s * pkp + c * pkq;
        }
      }
  }
  e.resize(n);
  for (int i = 0; i < n; ++i) e[i] = A[(size_t)i * n + i];
}

struct Scratch {
  double *what = nullptr, *omega = nullptr, *y = nullptr, *y2 = nullptr, *z = nullptr, *z2 = nullptr, *g = nullptr,
         *ri = nullptr, *u = nullptr, *v = nullptr, *ss = nullptr;
  ~Scratch() {
    for (double* p : {what, omega, y, y2, z, z2, g, ri, u, v, ss}) cudaFree(p);
  }
};

// Y (rows x l, row-major, on the device) <- Y R^-1 twice (CholeskyQR2); tmp is a rows x l buffer
cudaError_t cholqr2(double*& Y, double*& tmp, int rows, int l, Scratch& sc, cudaStream_t s) {
  std::vector<double> G((size_t)l * l), R, Ri;
  for (int pass = 0; pass < 2; ++pass) {
    cudaError_t e = dgemm(l, l, rows, Y, 1, l, Y, l, 1, sc.g, l, s);   // Y^T Y
    if (e == cudaSuccess) e = cudaMemcpyAsync(G.data(), sc.g, G.size() * 8, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    if (!cholesky_upper(G, R, l)) {
      double tr = 0.0;
      for (int i = 0; i < l; ++i) tr += G[(size_t)i * l + i];
      const double shift = tr > 0.0 ? std::ldexp(tr, -40) : 1.0;
      for (int i = 0; i < l; ++i) G[(size_t)i * l + i] += shift;
      if (!cholesky_upper(G, R, l)) return cudaErrorInvalidValue;
    }
    upper_inverse(R, Ri, l);
    e = cudaMemcpyAsync(sc.ri, Ri.data(), Ri.size() * 8, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = dgemm(rows, l, l, Y, l, 1, sc.ri, l, 1, tmp, l, s);   // Y R^-1
    if (e != cudaSuccess) return e;
    std::swap(Y, tmp);
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t lowrank_factors(int K, int N, int r, const __nv_bfloat16* Wt, const float* lam, uint64_t seed,
                            __nv_bfloat16* L1f, __nv_bfloat16* L2, double* sigma_out, cudaStream_t s) {
  const int l = std::min(r + 8, std::min(K, N));
  if (r < 1 || r > l) return cudaErrorInvalidValue;
  Scratch sc;
  const size_t big = (size_t)std::max(K, N) * l * 8;
  if (cudaMalloc(&sc.what, (size_t)K * N * 8) != cudaSuccess || cudaMalloc(&sc.omega, (size_t)N * l * 8) != cudaSuccess ||
      cudaMalloc(&sc.y, big) != cudaSuccess || cudaMalloc(&sc.y2, big) != cudaSuccess ||
      cudaMalloc(&sc.z, big) != cudaSuccess || cudaMalloc(&sc.z2, big) != cudaSuccess ||
      cudaMalloc(&sc.g, (size_t)l * l * 8) != cudaSuccess || cudaMalloc(&sc.ri, (size_t)l * l * 8) != cudaSuccess ||
      cudaMalloc(&sc.u, (size_t)K * l * 8) != cudaSuccess || cudaMalloc(&sc.v, (size_t)N * l * 8) != cudaSuccess ||
      cudaMalloc(&sc.ss, (size_t)l * 8) != cudaSuccess)
    return cudaErrorMemoryAllocation;
  cudaError_t e;
  {
    dim3 grid((K + 31) / 32, (N + 31) / 32), block(32, 8);
    what_kernel<<<grid, block, 0, s>>>(Wt, lam, sc.what, K, N);
    const long long words = (long long)N * l;
    rademacher_kernel<<<(unsigned)((words / 4 + 256) / 256), 256, 0, s>>>(sc.omega, words, seed);
    e = cudaGetLastError();
  }
  double *Y = sc.y, *Yt = sc.y2, *Z = sc.z, *Zt = sc.z2;
  // Q = orth(W^ Omega)
  if (e == cudaSuccess) e = dgemm(K, l, N, sc.what, N, 1, sc.omega, l, 1, Y, l, s);
  if (e == cudaSuccess) e = cholqr2(Y, Yt, K, l, sc, s);
  for (int it = 0; e == cudaSuccess && it < 3; ++it) {
    e = dgemm(N, l, K, sc.what, 1, N, Y, l, 1, Z, l, s);   // W^T Q
    if (e == cudaSuccess) e = cholqr2(Z, Zt, N, l, sc, s);
    if (e == cudaSuccess) e = dgemm(K, l, N, sc.what, N, 1, Z, l, 1, Y, l, s);   // W^ Z
    if (e == cudaSuccess) e = cholqr2(Y, Yt, K, l, sc, s);
  }
  // Z = W^T Q, T = Z^T Z
  std::vector<double> T((size_t)l * l), ev, P;
  if (e == cudaSuccess) e = dgemm(N, l, K, sc.what, 1, N, Y, l, 1, Z, l, s);
  if (e == cudaSuccess) e = dgemm(l, l, N, Z, 1, l, Z, l, 1, sc.g, l, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(T.data(), sc.g, T.size() * 8, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  jacobi_eig(T, l, ev, P);
  // descending order (stable), sigma = sqrt(max(e, 0))
  std::vector<int> ord(l);
  for (int i = 0; i < l; ++i) ord[i] = i;
  std::stable_sort(ord.begin(), ord.end(), [&](int a, int b) { return ev[a] > ev[b]; });
  std::vector<double> Ps((size_t)l * l), sig(l);
  for (int j = 0; j < l; ++j) {
    sig[j] = std::sqrt(std::max(ev[ord[j]], 0.0));
    for (int i = 0; i < l; ++i) Ps[(size_t)i * l + j] = P[(size_t)i * l + ord[j]];
  }
  // U = Q P; V = Z P / sigma (the division folded into P's columns)
  std::vector<double> Pv(Ps);
  for (int j = 0; j < l; ++j)
    for (int i = 0; i < l; ++i) Pv[(size_t)i * l + j] /= (sig[j] > 0.0 ? sig[j] : 1.0);
  e = cudaMemcpyAsync(sc.ri, Ps.data(), Ps.size() * 8, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = dgemm(K, l, l, Y, l, 1, sc.ri, l, 1, sc.u, l, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(sc.ri, Pv.data(), Pv.size() * 8, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = dgemm(N, l, l, Z, l, 1, sc.ri, l, 1, sc.v, l, s);
  // signs: each right singular vector's largest-|.| entry positive (first index wins)
  std::vector<double> V((size_t)N * l);
  if (e == cudaSuccess) e = cudaMemcpyAsync(V.data(), sc.v, V.size() * 8, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  std::vector<double> ss(r);
  for (int i = 0; i < r; ++i) {
    int piv = 0;
    double best = -1.0;
    for (int n = 0; n < N; ++n) {
      const double a = std::fabs(V[(size_t)n * l + i]);
      if (a > best) {
        best = a;
        piv = n;
      }
    }
    const double sgn = V[(size_t)piv * l + i] < 0 ? -1.0 : 1.0;
    ss[i] = std::copysign(sig[i], sgn);   // sigma_i with the column's sign (sigma_i >= 0)
  }
  // ss_i = sign_i sigma_i; for sigma_i = 0 the sign rides on the zero's sign bit
  std::vector<double> sgn_sig(ss);
  e = cudaMemcpyAsync(sc.ss, sgn_sig.data(), r * 8, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) {
    fold_kernel<<<256, 256, 0, s>>>(sc.u, sc.v, sc.ss, lam, K, N, l, r, L1f, L2);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && sigma_out) std::memcpy(sigma_out, sig.data(), (size_t)l * 8);
  return e;
}

}  // namespace svdq
