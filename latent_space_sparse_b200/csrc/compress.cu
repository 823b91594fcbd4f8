// compress.cu -- prefill low-rank projection Y = X . P.
//
// SALS technical framework, stage 1: keys (before RoPE) and values are
// projected into the latent space, Kc = K . Pk and Vc = V . Pv, with fp32
// accumulation and one rounding to the storage type.
#include "common.cuh"

namespace salsc {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kThreads = 256;

// CUDA-core tiled GEMM: each thread computes a 4x4 block of the 64x64 tile.
template <typename T>
__global__ void __launch_bounds__(kThreads)
compress_simt_kernel(const T* __restrict__ X, const T* __restrict__ P, T* __restrict__ Y, int64_t n,
                     int hid, int r) {
  __shared__ float xs[kBK][kBM + 4];
  __shared__ float ps[kBK][kBN];
  const int64_t m0 = (int64_t)blockIdx.x * kBM;
  const int n0 = blockIdx.y * kBN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < hid; k0 += kBK) {
    for (int e = threadIdx.x; e < kBM * kBK; e += kThreads) {
      const int mm = e / kBK, kk = e % kBK;
      const int64_t row = m0 + mm;
      xs[kk][mm] = (row < n && k0 + kk < hid) ? to_f32(X[row * hid + k0 + kk]) : 0.f;
    }
    for (int e = threadIdx.x; e < kBK * kBN; e += kThreads) {
      const int kk = e / kBN, nn = e % kBN;
      ps[kk][nn] = (k0 + kk < hid && n0 + nn < r) ? to_f32(P[(int64_t)(k0 + kk) * r + n0 + nn]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ps[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = m0 + ty * 4 + i;
    if (row >= n) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx * 4 + j;
      if (col < r) Y[row * r + col] = from_f32<T>(acc[i][j]);
    }
  }
}

}  // namespace

cudaError_t launch_compress(const void* X, const void* P, void* Y, int64_t n, int hid, int r,
                            salsc_dtype dt, cudaStream_t s) {
  dim3 grid((unsigned)((n + kBM - 1) / kBM), (unsigned)((r + kBN - 1) / kBN));
  if (dt == SALSC_BF16)
    compress_simt_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
        (const __nv_bfloat16*)X, (const __nv_bfloat16*)P, (__nv_bfloat16*)Y, n, hid, r);
  else
    compress_simt_kernel<float><<<grid, kThreads, 0, s>>>((const float*)X, (const float*)P,
                                                          (float*)Y, n, hid, r);
  return cudaGetLastError();
}

}  // namespace salsc
