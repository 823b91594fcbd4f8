// fit.cu -- learned projections: an orthonormal basis of the dominant
// right-singular subspace of a calibration matrix.
//
// SALS page, key designs (the projection choice: a low-rank projection from
// the SVD / PCA of the keys; calibration data).  P is hidden x r with
// orthonormal columns spanning the top-r right singular subspace of a
// calibration matrix X [n x hidden] (keys for Pk, values for Pv).  The decode
// path uses P only through P P^T (Kc = K P, reconstruction Kc P^T), so any
// orthonormal basis of that subspace serves.  This one comes from subspace
// iteration on the Gram matrix:
//   C = X^T X,   V_0 = orth(Omega),   V_{i+1} = orth(C V_i)   (i < iters)
// where Omega [hidden x r] is the caller's random start and orth(W) is
// Cholesky-QR applied twice: G = W^T W = L L^T, W <- W L^{-T}.  Every step is
// fp64 (Cholesky-QR squares the condition number of W); the error of the
// subspace falls as (sigma_{r+1} / sigma_r)^(2 iters).  An offline
// calibration step: plain tiled CUDA-core GEMMs, one-CTA factorisations.
#include "common.cuh"

namespace salsc {
namespace {

constexpr int kGemmTile = 64;   // output tile (kGemmTile x kGemmTile) per CTA
constexpr int kGemmK = 16;      // k-chunk staged in shared memory
constexpr int kGemmThreads = 256;  // 16 x 16 threads, 4 x 4 outputs each
constexpr int kFactorThreads = 1024;
constexpr uint32_t FLAG_FIT_NOT_SPD = 1u << 2;  // a Cholesky pivot was not positive

__device__ __forceinline__ double ld64(const double* p) { return *p; }
__device__ __forceinline__ double ld64(const float* p) { return (double)*p; }
__device__ __forceinline__ double ld64(const __nv_bfloat16* p) { return (double)__bfloat162float(*p); }

// C[M x N] = op(A) . op(B), fp64 accumulation.  A is [M x K] with row stride
// lda (TA false) or stored as [K x M] (TA true); B is [K x N] with row stride
// ldb (TB false) or stored as [N x K] (TB true).
template <typename TA_t, bool TA, typename TB_t, bool TB>
__global__ void __launch_bounds__(kGemmThreads)
gemm_f64_kernel(int M, int N, int K, const TA_t* __restrict__ A, int64_t lda,
                const TB_t* __restrict__ B, int64_t ldb, double* __restrict__ C, int64_t ldc) {
  __shared__ double As[kGemmK][kGemmTile + 1];
  __shared__ double Bs[kGemmK][kGemmTile + 1];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * kGemmTile, n0 = blockIdx.x * kGemmTile;
  double acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kGemmK) {
    for (int e = tid; e < kGemmK * kGemmTile; e += kGemmThreads) {
      const int kk = e / kGemmTile, mm = e % kGemmTile;
      const int gm = m0 + mm, gk = k0 + kk;
      double a = 0.0;
      if (gm < M && gk < K) a = TA ? ld64(A + (int64_t)gk * lda + gm) : ld64(A + (int64_t)gm * lda + gk);
      As[kk][mm] = a;
      const int gn = n0 + mm;
      double b = 0.0;
      if (gn < N && gk < K) b = TB ? ld64(B + (int64_t)gn * ldb + gk) : ld64(B + (int64_t)gk * ldb + gn);
      Bs[kk][mm] = b;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGemmK; ++kk) {
      double a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty + 16 * i];
        b[i] = Bs[kk][tx + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gm = m0 + ty + 16 * i, gn = n0 + tx + 16 * j;
      if (gm < M && gn < N) C[(int64_t)gm * ldc + gn] = acc[i][j];
    }
}

template <typename TA_t, bool TA, typename TB_t, bool TB>
cudaError_t gemm(int M, int N, int K, const TA_t* A, int64_t lda, const TB_t* B, int64_t ldb,
                 double* C, int64_t ldc, cudaStream_t s) {
  const dim3 grid((unsigned)((N + kGemmTile - 1) / kGemmTile),
                  (unsigned)((M + kGemmTile - 1) / kGemmTile));
  gemm_f64_kernel<TA_t, TA, TB_t, TB><<<grid, kGemmThreads, 0, s>>>(M, N, K, A, lda, B, ldb, C, ldc);
  return cudaGetLastError();
}

// In place: the lower triangle of G [m x m] (symmetric positive definite)
// becomes L with G = L L^T (right-looking, one CTA).  A pivot that is not
// positive sets FLAG_FIT_NOT_SPD and is replaced by 1.
__global__ void __launch_bounds__(kFactorThreads)
cholesky_kernel(double* __restrict__ G, int m, uint32_t* __restrict__ flags) {
  __shared__ double s_d;
  const int tid = threadIdx.x;
  for (int j = 0; j < m; ++j) {
    if (tid == 0) {
      double a = G[(int64_t)j * m + j];
      if (!(a > 0.0)) {
        atomicOr(flags, FLAG_FIT_NOT_SPD);
        a = 1.0;
      }
      s_d = sqrt(a);
      G[(int64_t)j * m + j] = s_d;
    }
    __syncthreads();
    const double d = s_d;
    for (int i = j + 1 + tid; i < m; i += kFactorThreads) G[(int64_t)i * m + j] /= d;
    __syncthreads();
    // trailing update of the lower triangle: G[i][k] -= L[i][j] L[k][j], j < k <= i
    const int len = m - j - 1;
    for (int e = tid; e < len * len; e += kFactorThreads) {
      const int i = j + 1 + e / len, k = j + 1 + e % len;
      if (k <= i) G[(int64_t)i * m + k] -= G[(int64_t)i * m + j] * G[(int64_t)k * m + j];
    }
    __syncthreads();
  }
}

// X = L^{-1} for L the lower triangle of Lm [m x m]: column c by forward
// substitution (one thread per column); the upper triangle of X is zero.
__global__ void __launch_bounds__(kFactorThreads)
lower_inverse_kernel(const double* __restrict__ Lm, double* __restrict__ X, int m) {
  for (int c = threadIdx.x; c < m; c += kFactorThreads) {
    for (int i = 0; i < c; ++i) X[(int64_t)i * m + c] = 0.0;
    for (int i = c; i < m; ++i) {
      double s = i == c ? 1.0 : 0.0;
      for (int k = c; k < i; ++k) s -= Lm[(int64_t)i * m + k] * X[(int64_t)k * m + c];
      X[(int64_t)i * m + c] = s / Lm[(int64_t)i * m + i];
    }
  }
}

__global__ void widen_kernel(const float* __restrict__ src, double* __restrict__ dst, int64_t count) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < count;
       e += (int64_t)gridDim.x * blockDim.x)
    dst[e] = (double)src[e];
}

template <typename T>
__global__ void cast_out_kernel(const double* __restrict__ V, T* __restrict__ P, int64_t count) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < count;
       e += (int64_t)gridDim.x * blockDim.x)
    P[e] = from_f32<T>((float)V[e]);
}

// V [h x m] <- orth(W): Cholesky-QR, G = W^T W = L L^T, V = W L^{-T}.
cudaError_t cholqr(const double* W, double* V, double* G, double* X, int h, int m,
                   uint32_t* flags, cudaStream_t s) {
  cudaError_t e = gemm<double, true, double, false>(m, m, h, W, m, W, m, G, m, s);
  if (e != cudaSuccess) return e;
  cholesky_kernel<<<1, kFactorThreads, 0, s>>>(G, m, flags);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lower_inverse_kernel<<<1, kFactorThreads, 0, s>>>(G, X, m);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return gemm<double, false, double, true>(h, m, m, W, m, X, m, V, m, s);
}

}  // namespace

size_t fit_workspace_size(int64_t hidden, int64_t rank) {
  const size_t h = (size_t)hidden, m = (size_t)rank;
  return kWsAlign + sizeof(double) * (h * h + 2 * h * m + 2 * m * m);
}

cudaError_t fit_projection(const void* Xc, int64_t n, int hidden, int rank, const float* omega,
                           int iters, void* P_out, salsc_dtype dt, void* ws, cudaStream_t s) {
  const int h = hidden, m = rank;
  uint32_t* flags = (uint32_t*)ws;
  double* C = (double*)((char*)ws + kWsAlign);  // [h x h]
  double* V = C + (size_t)h * h;                // [h x m]
  double* W = V + (size_t)h * m;                // [h x m]
  double* G = W + (size_t)h * m;                // [m x m]
  double* X = G + (size_t)m * m;                // [m x m]
  cudaError_t e = cudaMemsetAsync(flags, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  // C = X^T X over the n calibration rows (stored [n x h])
  if (n > INT32_MAX) return cudaErrorInvalidValue;
  e = dt == SALSC_BF16
          ? gemm<__nv_bfloat16, true, __nv_bfloat16, false>(h, h, (int)n, (const __nv_bfloat16*)Xc,
                                                            h, (const __nv_bfloat16*)Xc, h, C, h, s)
          : gemm<float, true, float, false>(h, h, (int)n, (const float*)Xc, h, (const float*)Xc, h,
                                            C, h, s);
  if (e != cudaSuccess) return e;
  // V_0 = orth(Omega), then V <- orth(C V) iters times; orth is Cholesky-QR
  // twice (the second pass brings V^T V to the identity to fp64 rounding)
  widen_kernel<<<256, 256, 0, s>>>(omega, W, (int64_t)h * m);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  auto orth2 = [&]() -> cudaError_t {  // W -> V
    cudaError_t r = cholqr(W, V, G, X, h, m, flags, s);
    if (r == cudaSuccess) r = cholqr(V, W, G, X, h, m, flags, s);
    if (r == cudaSuccess)
      r = cudaMemcpyAsync(V, W, sizeof(double) * (size_t)h * m, cudaMemcpyDeviceToDevice, s);
    return r;
  };
  if ((e = orth2()) != cudaSuccess) return e;
  for (int it = 0; it < iters; ++it) {
    if ((e = gemm<double, false, double, false>(h, m, h, C, h, V, m, W, m, s)) != cudaSuccess)
      return e;
    if ((e = orth2()) != cudaSuccess) return e;
  }
  if (dt == SALSC_BF16)
    cast_out_kernel<__nv_bfloat16><<<256, 256, 0, s>>>(V, (__nv_bfloat16*)P_out, (int64_t)h * m);
  else
    cast_out_kernel<float><<<256, 256, 0, s>>>(V, (float*)P_out, (int64_t)h * m);
  return cudaGetLastError();
}

}  // namespace salsc
