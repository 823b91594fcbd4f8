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

constexpr int kThreads = 128;  // one latent column per thread
constexpr int kBatchChunk = 16;

template <typename T>
__global__ void __launch_bounds__(kThreads)
latent_q_kernel(const T* __restrict__ q, const T* __restrict__ Pk, float* __restrict__ qlat,
                __nv_bfloat16* __restrict__ qsplit, int B, int Hq, int U, int G, int d, int r,
                int npad) {
  __shared__ float qsum[kBatchChunk * kMaxHeadDim];
  const int u = blockIdx.x;
  const int c = blockIdx.y * kThreads + threadIdx.x;
  for (int b0 = 0; b0 < B; b0 += kBatchChunk) {
    const int nb = min(kBatchChunk, B - b0);
    __syncthreads();
    for (int e = threadIdx.x; e < kBatchChunk * d; e += kThreads) {
      const int bb = e / d, i = e % d;
      float s = 0.f;
      if (bb < nb)
        for (int g = 0; g < G; ++g) s += to_f32(q[((size_t)(b0 + bb) * Hq + u * G + g) * d + i]);
      qsum[bb * d + i] = s;
    }
    __syncthreads();
    if (c < r) {
      float acc[kBatchChunk];
#pragma unroll
      for (int bb = 0; bb < kBatchChunk; ++bb) acc[bb] = 0.f;
      const T* pcol = Pk + (size_t)u * d * r + c;
      for (int i = 0; i < d; ++i) {
        const float pk = to_f32(pcol[(size_t)i * r]);
#pragma unroll
        for (int bb = 0; bb < kBatchChunk; ++bb) acc[bb] = fmaf(qsum[bb * d + i], pk, acc[bb]);
      }
      for (int bb = 0; bb < nb; ++bb) {
        const int b = b0 + bb;
        const float v = acc[bb];
        qlat[((size_t)b * U + u) * r + c] = v;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
        qsplit[((size_t)b * npad + 2 * u) * r + c] = hi;
        qsplit[((size_t)b * npad + 2 * u + 1) * r + c] = lo;
        // the padding rows are cleared by the last unit's CTAs
        if (u == U - 1)
          for (int row = 2 * U; row < npad; ++row)
            qsplit[((size_t)b * npad + row) * r + c] = __float2bfloat16_rn(0.f);
      }
    }
  }
}

}  // namespace

cudaError_t launch_latent_q(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(p.U, (p.r + kThreads - 1) / kThreads);
  if (p.dtype == SALSC_BF16)
    latent_q_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
        (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.Pk, a.qlat, a.qsplit, p.B, p.Hq, p.U,
        p.G, p.d, p.r, p.npad);
  else
    latent_q_kernel<float><<<grid, kThreads, 0, s>>>((const float*)a.q, (const float*)a.Pk, a.qlat,
                                                     a.qsplit, p.B, p.Hq, p.U, p.G, p.d, p.r,
                                                     p.npad);
  return cudaGetLastError();
}

}  // namespace salsc
