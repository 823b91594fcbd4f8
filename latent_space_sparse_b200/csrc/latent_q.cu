// latent_q.cu -- latent query of every selection unit.
//
// SALS technical framework, stage 2: tokens are selected in latent space
// with a RoPE-free query-key interaction.  Unit u's score of token t is
//   s_u[t] = sum_{h in u} (q_h . Pk_u) . Kc[t] = ((sum_{h in u} q_h) . Pk_u) . Kc[t],
// so the group sum is taken on the queries first (exact in real arithmetic,
// by linearity) and each unit needs one latent query q_lat = qsum . Pk_u.
//
// Output: q_lat fp32 [B][U][r], and the same values split into bf16 hi/lo
// parts [B][npad][r] (row 2u = hi, row 2u+1 = lo, hi + lo = q_lat to about
// 2^-16 relative; rows 2U..npad-1 zero) for the tensor-core scoring kernel.
#include "common.cuh"

namespace salsc {
namespace {

constexpr int kCols = 16;                  // latent columns per CTA
constexpr int kSlices = 32;                // row slices of Pk_u per CTA
constexpr int kThreads = kCols * kSlices;  // thread (slice, column): 512
constexpr int kWarps = kThreads / 32;
constexpr int kBatchChunk = 8;             // sequences per pass
constexpr int kRowsMax = kMaxHeadDim / kSlices;

// CTA (u, column block): q_lat[b, u, c] = sum_i qsum[b, i] * Pk[u*d + i, c] for
// 16 columns c.  Thread (slice, column) owns d/32 rows of one column of Pk_u;
// Pk is a weight, not an output of the previous kernel, so those loads are
// issued before the dependency wait (the kernel is launched with programmatic
// dependent launch).  After the wait the group sums of the queries are formed
// in shared memory (one query element per thread), each thread adds up its
// rows for every sequence, and the 32 slices are summed: lanes l and l+16 of a
// warp by a shuffle, then the 16 warps through shared memory.  Many short
// threads rather than a few long ones: with one CTA per SM the latency of
// each instruction is hidden only by other warps.
template <typename T>
__global__ void __launch_bounds__(kThreads)
latent_q_kernel(const T* __restrict__ q, const T* __restrict__ Pk, float* __restrict__ qlat,
                __nv_bfloat16* __restrict__ qsplit, uint32_t* __restrict__ krange, int B, int Hq,
                int U, int G, int d, int r, int npad) {
  __shared__ float qsum[kBatchChunk][kMaxHeadDim];
  __shared__ float red[kWarps][kBatchChunk][kCols];
  const int u = blockIdx.x;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int col = tid % kCols, slice = tid / kCols;
  const int c = blockIdx.y * kCols + col;
  const int rows = d / kSlices, i0 = slice * rows;
  float pk[kRowsMax];
#pragma unroll
  for (int j = 0; j < kRowsMax; ++j)
    pk[j] = (j < rows && c < r) ? to_f32(Pk[((size_t)u * d + i0 + j) * r + c]) : 0.f;
  allow_dependent_launch();
  grid_dependency_wait();  // q and the workspace belong to the previous kernel until now
  // empty key range of every unit, narrowed by the scoring kernel's atomics
  if (blockIdx.y == 0)
    for (int b = tid; b < B; b += kThreads) {
      krange[2 * ((size_t)b * U + u)] = 0xffffffffu;
      krange[2 * ((size_t)b * U + u) + 1] = 0u;
    }
  constexpr int kElems = kBatchChunk * kMaxHeadDim / kThreads;  // query sums per thread: 2
  for (int b0 = 0; b0 < B; b0 += kBatchChunk) {
    const int nb = min(kBatchChunk, B - b0);
    float v[kElems][8];
#pragma unroll
    for (int j = 0; j < kElems; ++j) {
      const int e = tid + j * kThreads;
      const int bb = e / d, i = e % d;
      const T* qp = q + ((size_t)(b0 + bb) * Hq + u * G) * d + i;
#pragma unroll
      for (int g = 0; g < 8; ++g) v[j][g] = (e < nb * d && g < G) ? to_f32(qp[(size_t)g * d]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kElems; ++j) {
      const int e = tid + j * kThreads;
      if (e < nb * d)
        qsum[e / d][e % d] = ((v[j][0] + v[j][1]) + (v[j][2] + v[j][3])) +
                             ((v[j][4] + v[j][5]) + (v[j][6] + v[j][7]));
    }
    __syncthreads();
    float acc[kBatchChunk];
#pragma unroll
    for (int bb = 0; bb < kBatchChunk; ++bb) {
      acc[bb] = 0.f;
#pragma unroll
      for (int j = 0; j < kRowsMax; ++j)
        if (j < rows && bb < nb) acc[bb] = fmaf(qsum[bb][i0 + j], pk[j], acc[bb]);
      acc[bb] += __shfl_xor_sync(0xffffffffu, acc[bb], 16);  // the warp's two slices
    }
    if (lane < kCols) {
#pragma unroll
      for (int bb = 0; bb < kBatchChunk; ++bb) red[warp][bb][lane] = acc[bb];
    }
    __syncthreads();
    if (tid < nb * kCols) {
      const int bb = tid / kCols, cl = tid % kCols;
      const int cc = blockIdx.y * kCols + cl;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) sum += red[w][bb][cl];
      if (cc < r) {
        const int b = b0 + bb;
        qlat[((size_t)b * U + u) * r + cc] = sum;
        const __nv_bfloat16 hi = __float2bfloat16_rn(sum);
        const __nv_bfloat16 lo = __float2bfloat16_rn(sum - __bfloat162float(hi));
        qsplit[((size_t)b * npad + 2 * u) * r + cc] = hi;
        qsplit[((size_t)b * npad + 2 * u + 1) * r + cc] = lo;
        // the padding rows are cleared by the last unit's CTAs
        if (u == U - 1)
          for (int row = 2 * U; row < npad; ++row)
            qsplit[((size_t)b * npad + row) * r + cc] = __float2bfloat16_rn(0.f);
      }
    }
    __syncthreads();  // qsum and red are reused by the next chunk
  }
}

}  // namespace

cudaError_t launch_latent_q(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(p.U, (p.r + kCols - 1) / kCols);
  if (p.dtype == SALSC_BF16)
    return launch_k(latent_q_kernel<__nv_bfloat16>, grid, dim3(kThreads), 0, s, true,
                    (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.Pk, a.qlat, a.qsplit,
                    a.krange, p.B, p.Hq, p.U, p.G, p.d, p.r, p.npad);
  return launch_k(latent_q_kernel<float>, grid, dim3(kThreads), 0, s, true, (const float*)a.q,
                  (const float*)a.Pk, a.qlat, a.qsplit, a.krange, p.B, p.Hq, p.U, p.G, p.d, p.r,
                  p.npad);
}

}  // namespace salsc
