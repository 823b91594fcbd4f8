// shard.cu -- token-sharded decode: the candidate exchange's two kernels.
//
// With the tokens of every sequence split over several GPUs (shard s holds a
// contiguous slice), SALS's selection stays exact: a token among a unit's k
// best overall has fewer than k better tokens in its own slice, so it is in
// that slice's local top-k.  Every shard therefore publishes its local top-k
// per unit as candidates (score, global token index); after an all-gather,
// every shard selects the same k best of the N*k candidates (score descending,
// the lower global index first among equal scores, as the single-GPU top-k),
// keeps the ones in its own slice, attends over them, and the shards'
// partial softmax sums are merged (SALS technical framework, stages 2-4; the
// exchange is this library's, the pages run one GPU).
#include "common.cuh"

namespace salsc {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kSelThreads = 1024;
constexpr int kSelPer = kMaxShardCandidates / kSelThreads;  // candidates per thread

// Candidate (b, u, j): the score and the global token index of slot j of unit
// (b, u)'s local selection; an empty slot (-1) becomes (-inf, -1).
__global__ void __launch_bounds__(kGatherThreads)
shard_gather_kernel(const int32_t* __restrict__ idx, const float* __restrict__ scores,
                    const int64_t* __restrict__ seq_off, const int64_t* __restrict__ shard_off,
                    float* __restrict__ cand_score, int32_t* __restrict__ cand_idx, int U, int k) {
  const int bu = blockIdx.x, b = bu / U, u = bu % U;
  grid_dependency_wait();  // the selection comes from the top-k kernel
  allow_dependent_launch();
  const int64_t off = seq_off[b], nb = seq_off[b + 1] - off;
  const float* su = scores + off * U + (int64_t)u * nb;
  const int64_t base = shard_off[b];
  for (int j = threadIdx.x; j < k; j += kGatherThreads) {
    const int t = idx[(int64_t)bu * k + j];
    const bool ok = t >= 0 && t < nb;
    cand_score[(int64_t)bu * k + j] = ok ? su[t] : -INFINITY;
    cand_idx[(int64_t)bu * k + j] = ok ? (int32_t)(base + t) : -1;
  }
}

// Order key of a candidate: the score's order-preserving bits above the
// complement of the global index, so that a larger key is a better candidate
// and no two valid candidates tie; an empty candidate is 0, below all.
__device__ __forceinline__ uint64_t cand_key(float s, int32_t gi) {
  if (gi < 0) return 0ull;
  return ((uint64_t)order_key(s) << 32) | (uint64_t)(0xffffffffu - (uint32_t)gi);
}

// One CTA per unit (b, u): the k best of the N*k candidates by an exact radix
// select on the 64-bit keys (eight passes of 8 bits, histograms in shared
// memory), then this shard's share in candidate order as local token indices,
// -1 in the remaining slots.
__global__ void __launch_bounds__(kSelThreads)
shard_select_kernel(const float* __restrict__ cand_score, const int32_t* __restrict__ cand_idx,
                    int N, int B, int U, int k, const int64_t* __restrict__ local_off,
                    const int64_t* __restrict__ shard_off, int32_t* __restrict__ idx_local) {
  __shared__ uint32_t hist[256];
  __shared__ uint64_t s_prefix;
  __shared__ int s_need, s_valid;
  __shared__ int s_warp[kSelThreads / 32];
  const int bu = blockIdx.x, b = bu / U;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int n = N * k;
  // thread tid holds candidates tid*kSelPer .. +kSelPer-1 (candidate c = s*k + j)
  uint64_t key[kSelPer];
  int32_t gidx[kSelPer];
  int nv = 0;
#pragma unroll
  for (int e = 0; e < kSelPer; ++e) {
    const int c = tid * kSelPer + e;
    key[e] = 0ull;
    gidx[e] = -1;
    if (c < n) {
      const int s = c / k, j = c % k;
      const int64_t at = (((int64_t)s * B + b) * U + bu % U) * k + j;
      gidx[e] = cand_idx[at];
      key[e] = cand_key(cand_score[at], gidx[e]);
      nv += gidx[e] >= 0;
    }
  }
  if (tid == 0) {
    s_prefix = 0ull;
    s_valid = 0;
  }
  __syncthreads();
  atomicAdd(&s_valid, nv);
  __syncthreads();
  const int keff = min(k, s_valid);
  if (tid == 0) s_need = keff;
  uint64_t mask = 0ull;
  for (int shift = 56; shift >= 0 && keff > 0; shift -= 8) {
    for (int e = tid; e < 256; e += kSelThreads) hist[e] = 0u;
    __syncthreads();
    const uint64_t prefix = s_prefix;
#pragma unroll
    for (int e = 0; e < kSelPer; ++e)
      if (gidx[e] >= 0 && (key[e] & mask) == prefix)
        atomicAdd(&hist[(uint32_t)(key[e] >> shift) & 255u], 1u);
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255-8l .. 248-8l (descending); find the digit at
      // which the count of keys above reaches s_need
      uint32_t h[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        h[i] = hist[255 - 8 * lane - i];
        sum += h[i];
      }
      uint32_t incl = sum;  // inclusive prefix over lanes 0..lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - sum;
      const uint32_t need = (uint32_t)s_need;
      if (excl < need && incl >= need) {
        uint32_t above = excl;
        int dgt = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above + h[i] >= need) {
            dgt = 255 - 8 * lane - i;
            break;
          }
          above += h[i];
        }
        s_prefix = prefix | ((uint64_t)dgt << shift);
        s_need = (int)(need - above);
      }
    }
    mask |= 255ull << shift;
    __syncthreads();
  }
  const uint64_t thr = s_prefix;  // the key of the k_eff-th best candidate
  // this shard's tokens among the selected ones, compacted in candidate order
  const int64_t lo = shard_off[b], len = local_off[b + 1] - local_off[b];
  int mine = 0;
  bool sel[kSelPer];
#pragma unroll
  for (int e = 0; e < kSelPer; ++e) {
    sel[e] = keff > 0 && gidx[e] >= 0 && key[e] >= thr && gidx[e] >= lo && gidx[e] < lo + len;
    mine += sel[e];
  }
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += v;
    }
    s_warp[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int pos = incl - mine + (warp > 0 ? s_warp[warp - 1] : 0);
  const int total = s_warp[kSelThreads / 32 - 1];
  int32_t* out = idx_local + (int64_t)bu * k;
#pragma unroll
  for (int e = 0; e < kSelPer; ++e)
    if (sel[e]) out[pos++] = (int32_t)(gidx[e] - lo);
  for (int j = total + tid; j < k; j += kSelThreads) out[j] = -1;
}

}  // namespace

cudaError_t launch_shard_gather(const DecodePlan& p, const DecodeArgs& a, const int64_t* shard_off,
                                float* cand_score, int32_t* cand_idx, cudaStream_t s) {
  return launch_k(shard_gather_kernel, dim3((unsigned)(p.B * p.U)), dim3(kGatherThreads), 0, s,
                  true, (const int32_t*)a.idx, (const float*)a.scores, a.seq_off, shard_off,
                  cand_score, cand_idx, p.U, p.k);
}

cudaError_t launch_shard_select(const float* cand_score, const int32_t* cand_idx, int N, int B,
                                int U, int k, const int64_t* local_off, const int64_t* shard_off,
                                int32_t* idx_local, cudaStream_t s) {
  if ((int64_t)N * k > kMaxShardCandidates) return cudaErrorInvalidValue;
  shard_select_kernel<<<(unsigned)(B * U), kSelThreads, 0, s>>>(cand_score, cand_idx, N, B, U, k,
                                                                 local_off, shard_off, idx_local);
  return cudaGetLastError();
}

}  // namespace salsc
