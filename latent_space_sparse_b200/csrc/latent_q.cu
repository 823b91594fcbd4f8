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

constexpr int kThreads = 128;  // 4 warps; each warp takes a quarter of the head dim
constexpr int kCols = 64;      // latent columns per CTA: 2 per lane
constexpr int kBatchChunk = 8;

template <typename T>
__device__ __forceinline__ float2 load2(const T* p);
template <>
__device__ __forceinline__ float2 load2<float>(const float* p) {
  return *(const float2*)p;
}
template <>
__device__ __forceinline__ float2 load2<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat1622float2(*(const __nv_bfloat162*)p);
}

// CTA (u, column block): q_lat[b, u, c] = sum_i qsum[b, i] * Pk[u*d + i, c] for
// its 64 columns.  Each warp reads a quarter of the d rows of Pk_u (coalesced
// 128-byte rows, all loads independent), and the four partial sums are
// added in shared memory.
template <typename T>
__global__ void __launch_bounds__(kThreads)
latent_q_kernel(const T* __restrict__ q, const T* __restrict__ Pk, float* __restrict__ qlat,
                __nv_bfloat16* __restrict__ qsplit, int B, int Hq, int U, int G, int d, int r,
                int npad) {
  __shared__ float qsum[kBatchChunk][kMaxHeadDim];
  __shared__ float2 red[4][kBatchChunk][32];
  const int u = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int c = blockIdx.y * kCols + 2 * lane;
  const int rows = d / 4, i0 = warp * rows;
  for (int b0 = 0; b0 < B; b0 += kBatchChunk) {
    const int nb = min(kBatchChunk, B - b0);
    __syncthreads();
    for (int e = threadIdx.x; e < kBatchChunk * d; e += kThreads) {
      const int bb = e / d, i = e % d;
      float s = 0.f;
      if (bb < nb)
        for (int g = 0; g < G; ++g) s += to_f32(q[((size_t)(b0 + bb) * Hq + u * G + g) * d + i]);
      qsum[bb][i] = s;
    }
    __syncthreads();
    float2 acc[kBatchChunk];
#pragma unroll
    for (int bb = 0; bb < kBatchChunk; ++bb) acc[bb] = make_float2(0.f, 0.f);
    if (c < r) {
      const T* pcol = Pk + ((size_t)u * d + i0) * r + c;
#pragma unroll 8
      for (int i = 0; i < rows; ++i) {
        const float2 pk = load2<T>(pcol + (size_t)i * r);
#pragma unroll
        for (int bb = 0; bb < kBatchChunk; ++bb) {
          const float qv = qsum[bb][i0 + i];
          acc[bb].x = fmaf(qv, pk.x, acc[bb].x);
          acc[bb].y = fmaf(qv, pk.y, acc[bb].y);
        }
      }
    }
#pragma unroll
    for (int bb = 0; bb < kBatchChunk; ++bb) red[warp][bb][lane] = acc[bb];
    __syncthreads();
    // warp w finishes batch rows w, w+4
    for (int bb = warp; bb < nb; bb += 4) {
      if (c >= r) continue;
      float2 v = red[0][bb][lane];
#pragma unroll
      for (int w = 1; w < 4; ++w) {
        v.x += red[w][bb][lane].x;
        v.y += red[w][bb][lane].y;
      }
      const int b = b0 + bb;
      *(float2*)(qlat + ((size_t)b * U + u) * r + c) = v;
      const __nv_bfloat16 hx = __float2bfloat16_rn(v.x), hy = __float2bfloat16_rn(v.y);
      const __nv_bfloat16 lx = __float2bfloat16_rn(v.x - __bfloat162float(hx));
      const __nv_bfloat16 ly = __float2bfloat16_rn(v.y - __bfloat162float(hy));
      *(__nv_bfloat162*)(qsplit + ((size_t)b * npad + 2 * u) * r + c) = __halves2bfloat162(hx, hy);
      *(__nv_bfloat162*)(qsplit + ((size_t)b * npad + 2 * u + 1) * r + c) =
          __halves2bfloat162(lx, ly);
      // the padding rows are cleared by the last unit's CTAs
      if (u == U - 1)
        for (int row = 2 * U; row < npad; ++row)
          *(__nv_bfloat162*)(qsplit + ((size_t)b * npad + row) * r + c) =
              __halves2bfloat162(__float2bfloat16_rn(0.f), __float2bfloat16_rn(0.f));
    }
  }
}

}  // namespace

cudaError_t launch_latent_q(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(p.U, (p.r + kCols - 1) / kCols);
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
