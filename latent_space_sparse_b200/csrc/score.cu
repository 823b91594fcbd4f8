// score.cu -- RoPE-free latent scoring of every cached token.
//
// SALS technical framework, stage 2: s_u[t] = q_lat[b,u] . Kc_b[t] for every
// unit u and every cached token t < n_b.  Kc is read exactly once per step
// for all units of a sequence.
//
// Scores are written fp32, packed per (b,u): unit (b,u)'s n_b scores start at
// seq_off[b]*U + u*n_b.
#include "common.cuh"

namespace salsc {
namespace {

constexpr int kThreads = 256;

// CUDA-core path: one warp per token row; each lane holds its slice of the
// row in registers and reduces U dot products across the warp.
template <typename T>
__global__ void __launch_bounds__(kThreads)
score_simt_kernel(const T* __restrict__ Kc, const float* __restrict__ qlat,
                  const int64_t* __restrict__ seq_off, float* __restrict__ scores, int B, int U,
                  int r, int tile_len) {
  extern __shared__ float sq[];  // [U][r]
  int b;
  int64_t t0;
  find_tile(seq_off, B, tile_len, blockIdx.x, b, t0);
  if (b < 0) return;
  const int64_t off = seq_off[b];
  const int64_t nb = seq_off[b + 1] - off;
  for (int e = threadIdx.x; e < U * r; e += kThreads) sq[e] = qlat[(size_t)b * U * r + e];
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int kPer = kMaxRank / 32;  // row elements held per lane
  const int64_t t_end = min(t0 + (int64_t)tile_len, nb);
  for (int64_t t = t0 + warp; t < t_end; t += kThreads / 32) {
    const T* row = Kc + (off + t) * r;
    float x[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int c = lane + 32 * j;
      x[j] = c < r ? to_f32(row[c]) : 0.f;
    }
    for (int u = 0; u < U; ++u) {
      const float* qu = sq + u * r;
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int c = lane + 32 * j;
        if (c < r) acc = fmaf(x[j], qu[c], acc);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) scores[off * U + (int64_t)u * nb + t] = acc;
    }
  }
}

}  // namespace

cudaError_t launch_score(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)p.U * p.r;
  if (p.dtype == SALSC_BF16) {
    static int done[kMaxDevices] = {};
    auto k = score_simt_kernel<__nv_bfloat16>;
    cudaError_t e = ensure_smem(k, smem, done);
    if (e != cudaSuccess) return e;
    k<<<p.n_score_tiles, kThreads, smem, s>>>((const __nv_bfloat16*)a.Kc, a.qlat, a.seq_off,
                                              a.scores, p.B, p.U, p.r, p.score_tile);
  } else {
    static int done[kMaxDevices] = {};
    auto k = score_simt_kernel<float>;
    cudaError_t e = ensure_smem(k, smem, done);
    if (e != cudaSuccess) return e;
    k<<<p.n_score_tiles, kThreads, smem, s>>>((const float*)a.Kc, a.qlat, a.seq_off, a.scores,
                                              p.B, p.U, p.r, p.score_tile);
  }
  return cudaGetLastError();
}

}  // namespace salsc
