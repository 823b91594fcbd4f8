// append.cu -- decode-time append: the new token's latent key and value rows.
//
// SALS technical framework, stage 1, applied to the token being decoded: its
// key (before RoPE) and value are projected into the latent space and written
// into the latent cache,
//   Kc[rows[b]] = K_new[b] . Pk,   Vc[rows[b]] = V_new[b] . Pv,
// with fp32 accumulation and one rounding to the storage type, for every
// sequence b of the batch.
//
// Each output element is a dot product of length `hidden`; the work is tiny
// (B x hidden x r) and the cost is reading Pk and Pv once.  A cluster of 8
// CTAs takes one block of 32 latent columns of one matrix: CTA q of the
// cluster reduces rows q*hidden/8 .. (q+1)*hidden/8 of P for every sequence
// (warp w takes an eighth of those rows, lane l takes column l, so every P
// load of a warp is 64 contiguous bytes), the eight warps' sums are added in
// shared memory, and the cluster's eight partial blocks are added through
// distributed shared memory by its first CTA, which rounds and writes the
// rows.  No global scratch memory.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace salsc {
namespace {

constexpr int kCols = 32;     // latent columns per cluster
constexpr int kWarps = 8;     // hidden-row slices per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kCluster = 8;   // hidden-row parts per cluster
constexpr int kBChunk = 16;   // sequences per pass
constexpr int kMaxRowsPerCta = 1024;  // hidden / 8 rows staged per sequence

template <typename T>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads)
append_kernel(const T* __restrict__ X0, const T* __restrict__ X1, const T* __restrict__ P0,
              const T* __restrict__ P1, T* __restrict__ Y0, T* __restrict__ Y1,
              const int64_t* __restrict__ rows, int B, int hid, int r) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float xs[kBChunk][kMaxRowsPerCta / 4];  // x rows of this CTA's hidden part, chunked
  __shared__ float red[kWarps][kBChunk][kCols];
  __shared__ float part[kBChunk][kCols];             // this CTA's partial block, read by rank 0
  const int q = (int)cluster.block_rank();
  const int cb = blockIdx.y;
  const bool second = blockIdx.z == 1;
  const T* X = second ? X1 : X0;
  const T* P = second ? P1 : P0;
  T* Y = second ? Y1 : Y0;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int c = cb * kCols + lane;
  const int hc = (hid + kCluster - 1) / kCluster;  // hidden rows of this CTA
  const int h0 = q * hc, h1 = min(hid, h0 + hc);
  constexpr int kSub = kMaxRowsPerCta / 4;          // rows staged at a time
  allow_dependent_launch();
  for (int b0 = 0; b0 < B; b0 += kBChunk) {
    const int nb = min(kBChunk, B - b0);
    float acc[kBChunk];
#pragma unroll
    for (int j = 0; j < kBChunk; ++j) acc[j] = 0.f;
    for (int s0 = h0; s0 < h1; s0 += kSub) {
      const int s1 = min(h1, s0 + kSub);
      __syncthreads();  // the previous sub-block is consumed
      for (int e = tid; e < nb * (s1 - s0); e += kThreads) {
        const int bb = e / (s1 - s0), i = e % (s1 - s0);
        xs[bb][i] = to_f32(X[(int64_t)(b0 + bb) * hid + s0 + i]);
      }
      __syncthreads();
      // warp w: rows s0 + w, s0 + w + 8, ...
      for (int i = s0 + warp; i < s1; i += kWarps) {
        const float p = c < r ? to_f32(P[(int64_t)i * r + c]) : 0.f;
#pragma unroll
        for (int j = 0; j < kBChunk; ++j)
          if (j < nb) acc[j] = fmaf(xs[j][i - s0], p, acc[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < kBChunk; ++j) red[warp][j][lane] = acc[j];
    __syncthreads();
    for (int e = tid; e < nb * kCols; e += kThreads) {
      const int j = e / kCols, l = e % kCols;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) sum += red[w][j][l];
      part[j][l] = sum;
    }
    cluster.sync();  // every CTA's partial block is complete
    if (q == 0) {
      for (int e = tid; e < nb * kCols; e += kThreads) {
        const int j = e / kCols, l = e % kCols;
        const int cc = cb * kCols + l;
        float sum = 0.f;
#pragma unroll
        for (int qq = 0; qq < kCluster; ++qq) sum += cluster.map_shared_rank(&part[0][0], qq)[j * kCols + l];
        if (cc < r) Y[rows[b0 + j] * r + cc] = from_f32<T>(sum);
      }
    }
    cluster.sync();  // rank 0 is done reading the partial blocks
  }
}

}  // namespace

cudaError_t launch_append(const void* const X[2], const void* const Pm[2], void* const Y[2],
                          int n_mats, const int64_t* rows, int B, int hid, int r, salsc_dtype dt,
                          cudaStream_t s) {
  if ((hid + kCluster - 1) / kCluster > kMaxRowsPerCta) return cudaErrorInvalidConfiguration;
  const dim3 grid(kCluster, (unsigned)((r + kCols - 1) / kCols), (unsigned)n_mats);
  if (dt == SALSC_BF16) {
    append_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
        (const __nv_bfloat16*)X[0], (const __nv_bfloat16*)X[1], (const __nv_bfloat16*)Pm[0],
        (const __nv_bfloat16*)Pm[1], (__nv_bfloat16*)Y[0], (__nv_bfloat16*)Y[1], rows, B, hid, r);
  } else {
    append_kernel<float><<<grid, kThreads, 0, s>>>((const float*)X[0], (const float*)X[1],
                                                   (const float*)Pm[0], (const float*)Pm[1],
                                                   (float*)Y[0], (float*)Y[1], rows, B, hid, r);
  }
  return cudaGetLastError();
}

}  // namespace salsc
