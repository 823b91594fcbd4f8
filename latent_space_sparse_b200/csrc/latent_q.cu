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

constexpr int kThreads = 256;  // 8 warps; each warp takes d/8 rows of Pk_u
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
// its 64 columns.  Each warp owns d/8 rows of Pk_u; its Pk loads are issued
// first, the query sums are formed by the whole CTA meanwhile, and the eight
// warps' partial sums are added in shared memory.  Small loops keep the code
// short (the kernel is too brief to amortise a cold instruction cache).
template <typename T>
__global__ void __launch_bounds__(kThreads)
latent_q_kernel(const T* __restrict__ q, const T* __restrict__ Pk, float* __restrict__ qlat,
                __nv_bfloat16* __restrict__ qsplit, int* __restrict__ unit_count, int B, int Hq,
                int U, int G, int d, int r, int npad) {
  constexpr int kRowsMax = kMaxHeadDim / 8;  // Pk rows per warp
  __shared__ float qsum[kBatchChunk][kMaxHeadDim];
  // per warp: its Pk rows during the row loop, then its partial sums
  static_assert(kBatchChunk <= kRowsMax, "partial sums reuse the Pk staging rows");
  __shared__ float2 wbuf[8][kRowsMax][32];
  allow_dependent_launch();
  if (blockIdx.y == 0 && unit_count)
    for (int b = threadIdx.x; b < B; b += kThreads) unit_count[b * U + blockIdx.x] = 0;
  const int u = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int c = blockIdx.y * kCols + 2 * lane;
  const int rows = d / 8, i0 = warp * rows;
  for (int b0 = 0; b0 < B; b0 += kBatchChunk) {
    const int nb = min(kBatchChunk, B - b0);
    float2 pk[kRowsMax];
#pragma unroll
    for (int i = 0; i < kRowsMax; ++i)
      pk[i] = (i < rows && c < r) ? load2<T>(Pk + ((size_t)u * d + i0 + i) * r + c)
                                  : make_float2(0.f, 0.f);
    // query group sums: thread e covers (bb, i) = e, e+256, ...
    for (int e = threadIdx.x; e < nb * d; e += kThreads) {
      const int bb = e / d, i = e % d;
      const T* qp = q + ((size_t)(b0 + bb) * Hq + u * G) * d + i;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      float sacc = 0.f;
      for (int g0 = 0; g0 < G; g0 += 4) {
#pragma unroll
        for (int g = 0; g < 4; ++g) v[g] = g0 + g < G ? to_f32(qp[(size_t)(g0 + g) * d]) : 0.f;
        sacc += (v[0] + v[1]) + (v[2] + v[3]);
      }
      qsum[bb][i] = sacc;
    }
    __syncthreads();
    // the Pk values go through shared memory so that the row loop stays rolled:
    // code executed once per SM costs a cold instruction fetch per instruction
#pragma unroll
    for (int i = 0; i < kRowsMax; ++i) wbuf[warp][i][lane] = pk[i];
    __syncwarp();
    float2 acc[kBatchChunk];
#pragma unroll
    for (int bb = 0; bb < kBatchChunk; ++bb) acc[bb] = make_float2(0.f, 0.f);
#pragma unroll 1
    for (int i = 0; i < rows; ++i) {
      const float2 pv = wbuf[warp][i][lane];
#pragma unroll
      for (int bb = 0; bb < kBatchChunk; ++bb) {
        const float qv = qsum[bb][i0 + i];
        acc[bb].x = fmaf(qv, pv.x, acc[bb].x);
        acc[bb].y = fmaf(qv, pv.y, acc[bb].y);
      }
    }
    __syncwarp();
#pragma unroll
    for (int bb = 0; bb < kBatchChunk; ++bb) wbuf[warp][bb][lane] = acc[bb];
    __syncthreads();
    // warp w finishes batch row w
    if (warp < nb && c < r) {
      const int bb = warp;
      float2 v = wbuf[0][bb][lane];
      for (int w = 1; w < 8; ++w) {
        v.x += wbuf[w][bb][lane].x;
        v.y += wbuf[w][bb][lane].y;
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
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_latent_q(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(p.U, (p.r + kCols - 1) / kCols);
  if (p.dtype == SALSC_BF16)
    latent_q_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
        (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.Pk, a.qlat, a.qsplit, a.unit_count, p.B,
        p.Hq, p.U, p.G, p.d, p.r, p.npad);
  else
    latent_q_kernel<float><<<grid, kThreads, 0, s>>>((const float*)a.q, (const float*)a.Pk, a.qlat,
                                                     a.qsplit, a.unit_count, p.B, p.Hq, p.U, p.G,
                                                     p.d, p.r, p.npad);
  return cudaGetLastError();
}

}  // namespace salsc
