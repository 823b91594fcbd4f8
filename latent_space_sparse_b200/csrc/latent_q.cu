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

constexpr int kBatchChunk = 8;  // sequences per pass

// Threads and register cap per column width.  COLS = 16 (at most a few hundred
// CTAs, e.g. 128 for 8 units of r = 256): 768 threads of at most 48 registers,
// 36K registers a CTA, so that two CTAs never share an SM (73K > 64K) and the
// scoring kernel's CTAs, launched early two per SM (21K), fit beside each one
// instead of waiting for the SM to drain.  COLS = 64 (many units and a wide
// latent space): 512 threads.
template <int COLS> constexpr int lq_threads() { return COLS == 16 ? 768 : 512; }

// CTA (u, column block): q_lat[b, u, c] = sum_i qsum[b, i] * Pk[u*d + i, c] for
// COLS columns c.  Thread (slice, column) owns d/SLICES rows of one column of
// Pk_u; Pk is a weight, not an output of the previous kernel, so those loads
// are issued before the dependency wait (the kernel is launched with
// programmatic dependent launch).  After the wait the group sums of the
// queries are formed in shared memory (one query element per thread), each
// thread adds up its rows for every sequence, and the slices are summed
// through shared memory.  Many short threads rather than a few long ones:
// with one CTA per SM the latency of each instruction is hidden only by
// other warps.  COLS = 16 spreads a small Pk (GQA) over enough CTAs; COLS = 64
// keeps a large one (MHA, r = 512) to a few hundred CTAs.
template <typename T, int COLS>
__device__ __forceinline__ void latent_q_body(const T* __restrict__ q, const T* __restrict__ Pk,
                                              float* __restrict__ qlat,
                                              __nv_bfloat16* __restrict__ qsplit,
                                              uint32_t* __restrict__ krange,
                                              uint64_t* trace, int B, int Hq, int U, int G,
                                              int d, int r, int npad) {
  constexpr int kThreads = lq_threads<COLS>();
  constexpr int SLICES = kThreads / COLS;
  constexpr int kRowsMax = (kMaxHeadDim + SLICES - 1) / SLICES;
  __shared__ float qsum[kBatchChunk][kMaxHeadDim];
  __shared__ float red[SLICES][kBatchChunk][COLS];
  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid == 0) trace_stamp(trace, TRACE_START);
  const int col = tid % COLS, slice = tid / COLS;
  const int c = blockIdx.y * COLS + col;
  const int rows = (d + SLICES - 1) / SLICES, i0 = slice * rows;
  float pk[kRowsMax];
#pragma unroll
  for (int j = 0; j < kRowsMax; ++j)
    pk[j] = (j < rows && i0 + j < d && c < r) ? to_f32(Pk[((size_t)u * d + i0 + j) * r + c]) : 0.f;
  grid_dependency_wait();  // q and the workspace belong to the previous kernel until now
  if (tid == 0) trace_stamp(trace, TRACE_WAITED);
  // Only now may the step's later kernels start: they read step inputs (Kc,
  // the sequence offsets) before their own dependency waits, and everything
  // the stream did before this step is complete once the wait above returns.
  allow_dependent_launch();
  // empty key range of every unit, narrowed by the scoring kernel's atomics
  if (blockIdx.y == 0)
    for (int b = tid; b < B; b += kThreads) {
      krange[2 * ((size_t)b * U + u)] = 0xffffffffu;
      krange[2 * ((size_t)b * U + u) + 1] = 0u;
    }
  constexpr int kElems = (kBatchChunk * kMaxHeadDim + kThreads - 1) / kThreads;  // query sums per thread
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
    // the chunk's live sequences only (a chain of shared-memory loads and
    // FMAs per sequence: at B = 1 one pass, not kBatchChunk)
#pragma unroll 1
    for (int bb = 0; bb < nb; ++bb) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < kRowsMax; ++j)
        if (j < rows && i0 + j < d) acc = fmaf(qsum[bb][i0 + j], pk[j], acc);
      red[slice][bb][col] = acc;
    }
    __syncthreads();
    for (int e = tid; e < nb * COLS; e += kThreads) {
      const int bb = e / COLS, cl = e % COLS;
      const int cc = blockIdx.y * COLS + cl;
      float sum = 0.f;
#pragma unroll
      for (int sl = 0; sl < SLICES; ++sl) sum += red[sl][bb][cl];
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
  if (tid == 0) trace_stamp(trace, TRACE_END);
}

template <typename T>
__global__ void __maxnreg__(48)
latent_q16_kernel(const T* __restrict__ q, const T* __restrict__ Pk, float* __restrict__ qlat,
                  __nv_bfloat16* __restrict__ qsplit, uint32_t* __restrict__ krange,
                  uint64_t* trace, int B, int Hq, int U, int G, int d, int r, int npad) {
  latent_q_body<T, 16>(q, Pk, qlat, qsplit, krange, trace, B, Hq, U, G, d, r, npad);
}

template <typename T>
__global__ void __launch_bounds__(lq_threads<64>())
latent_q64_kernel(const T* __restrict__ q, const T* __restrict__ Pk, float* __restrict__ qlat,
                  __nv_bfloat16* __restrict__ qsplit, uint32_t* __restrict__ krange,
                  uint64_t* trace, int B, int Hq, int U, int G, int d, int r, int npad) {
  latent_q_body<T, 64>(q, Pk, qlat, qsplit, krange, trace, B, Hq, U, G, d, r, npad);
}

template <typename T, int COLS>
cudaError_t launch_cols(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(p.U, (p.r + COLS - 1) / COLS);
  auto kernel = COLS == 16 ? latent_q16_kernel<T> : latent_q64_kernel<T>;
  return launch_k(kernel, grid, dim3(lq_threads<COLS>()), 0, s, true, (const T*)a.q,
                  (const T*)a.Pk, a.qlat, a.qsplit, a.krange, trace_of(a, 0), p.B, p.Hq,
                  p.U, p.G, p.d, p.r, p.npad);
}

template <typename T>
cudaError_t launch_t(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  // 16 columns per CTA unless that makes more than 512 CTAs
  return (int64_t)p.U * ((p.r + 15) / 16) > 512 ? launch_cols<T, 64>(p, a, s)
                                                  : launch_cols<T, 16>(p, a, s);
}

}  // namespace

cudaError_t launch_latent_q(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  return p.dtype == SALSC_BF16 ? launch_t<__nv_bfloat16>(p, a, s) : launch_t<float>(p, a, s);
}

}  // namespace salsc
