// topk.cu -- exact per-unit top-k by cluster-wide radix select.
//
// SALS keeps only the most important tokens of each unit (page section "key
// designs": Top-K selection).  k_b = min(k, n_b) tokens with the largest
// score are kept; among equal scores the lower token index wins; slots
// k_b..k-1 are set to -1.
//
// Design: a thread-block cluster of C CTAs owns one unit.  Each CTA loads a
// contiguous slice of the unit's scores into shared memory once, as 32-bit
// keys whose unsigned order is the float order.  Four 8-bit radix passes find
// the exact k_b-th largest key T: each CTA histograms its slice, the C
// histograms are summed through distributed shared memory, and every CTA
// picks the same digit.  A final ordered compaction writes the keys > T and
// the lowest-index keys == T; slice ranks give a global index order, so the
// result is deterministic.  No full sort, no global-memory scratch.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace salsc {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

// Unsigned key with the same order as the float; -0 and +0 map to one key.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kThreads)
topk_cluster_kernel(const float* __restrict__ scores, const int64_t* __restrict__ seq_off,
                    int32_t* __restrict__ idx_out, int U, int k) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int unit = blockIdx.x / C;
  const int b = unit / U, u = unit % U;

  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[2][256];
  __shared__ uint32_t total[256];
  __shared__ uint32_t counts[2];  // this CTA's (#keys > T, #keys == T), read by the cluster
  __shared__ uint32_t wtot[kWarps][2];
  __shared__ uint32_t s_digit, s_above, s_base_gt, s_base_eq;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t off = seq_off[b];
  const int64_t nb = seq_off[b + 1] - off;
  const int64_t kb = nb < k ? nb : k;
  const float* s = scores + off * U + (int64_t)u * nb;
  const int64_t lo = nb * rank / C, hi = nb * (rank + 1) / C;
  const int n_loc = (int)(hi - lo);

  for (int i = tid; i < n_loc; i += kThreads) keys[i] = order_key(s[lo + i]);

  // Radix select: T = the kb-th largest key; `remaining` ends as the number
  // of keys equal to T that are kept.
  uint32_t prefix = 0u, mask = 0u, remaining = (uint32_t)kb;
  const bool take_all = kb == nb;
  if (take_all) {
    remaining = 0u;  // every finite score has key > 0
    __syncthreads();
  } else {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      uint32_t* h = hist[pass & 1];
      for (int i = tid; i < 256; i += kThreads) h[i] = 0u;
      __syncthreads();
      for (int i = tid; i < n_loc; i += kThreads) {
        const uint32_t key = keys[i];
        if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
      }
      cluster.sync();
      if (tid < 256) {
        uint32_t t = 0u;
        for (int q = 0; q < C; ++q) t += cluster.map_shared_rank(h, q)[tid];
        total[tid] = t;
      }
      __syncthreads();
      if (warp == 0) {
        // lane L covers bins 255-8L .. 248-8L, in descending order
        uint32_t v[8], sum = 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v[j] = total[255 - 8 * lane - j];
          sum += v[j];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        uint32_t run = incl - sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run < remaining && remaining <= run + v[j]) {
            s_digit = (uint32_t)(255 - 8 * lane - j);
            s_above = run;
          }
          run += v[j];
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= 255u << shift;
      remaining -= s_above;
    }
  }
  const uint32_t T = prefix;
  const uint32_t need_eq = remaining;
  const uint32_t n_gt_total = (uint32_t)kb - need_eq;

  // Local counts, then this CTA's offsets from the lower ranks.
  uint32_t my_gt = 0u, my_eq = 0u;
  for (int i = tid; i < n_loc; i += kThreads) {
    const uint32_t key = keys[i];
    my_gt += key > T;
    my_eq += key == T;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    my_gt += __shfl_xor_sync(0xffffffffu, my_gt, o);
    my_eq += __shfl_xor_sync(0xffffffffu, my_eq, o);
  }
  if (lane == 0) {
    wtot[warp][0] = my_gt;
    wtot[warp][1] = my_eq;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t g = 0u, e = 0u;
    for (int w = 0; w < kWarps; ++w) {
      g += wtot[w][0];
      e += wtot[w][1];
    }
    counts[0] = g;
    counts[1] = e;
  }
  cluster.sync();
  if (tid == 0) {
    uint32_t g = 0u, e = 0u;
    for (int q = 0; q < rank; ++q) {
      const uint32_t* rc = cluster.map_shared_rank(counts, q);
      g += rc[0];
      e += rc[1];
    }
    s_base_gt = g;
    s_base_eq = e;
  }
  __syncthreads();

  int32_t* out = idx_out + ((int64_t)b * U + u) * k;
  uint32_t run_gt = s_base_gt, run_eq = s_base_eq;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int c0 = 0; c0 < n_loc; c0 += kThreads) {
    const int i = c0 + tid;
    const bool valid = i < n_loc;
    const uint32_t key = valid ? keys[i] : 0u;
    const bool g = valid && key > T;
    const bool e = valid && key == T && need_eq > 0u;
    const uint32_t bg = __ballot_sync(0xffffffffu, g);
    const uint32_t be = __ballot_sync(0xffffffffu, e);
    if (lane == 0) {
      wtot[warp][0] = __popc(bg);
      wtot[warp][1] = __popc(be);
    }
    __syncthreads();
    uint32_t og = 0u, oe = 0u, tg = 0u, te = 0u;
    for (int w = 0; w < kWarps; ++w) {
      if (w < warp) {
        og += wtot[w][0];
        oe += wtot[w][1];
      }
      tg += wtot[w][0];
      te += wtot[w][1];
    }
    if (g) out[run_gt + og + __popc(bg & lt_mask)] = (int32_t)(lo + i);
    if (e) {
      const uint32_t er = run_eq + oe + __popc(be & lt_mask);
      if (er < need_eq) out[n_gt_total + er] = (int32_t)(lo + i);
    }
    run_gt += tg;
    run_eq += te;
    __syncthreads();
  }
  if (rank == 0)
    for (int64_t j = kb + tid; j < k; j += kThreads) out[j] = -1;
  cluster.sync();  // no CTA leaves while another may still read its counts
}

}  // namespace

cudaError_t launch_topk(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(uint32_t) * (size_t)p.topk_slice;
  static int done[kMaxDevices] = {};
  cudaError_t e = ensure_smem(topk_cluster_kernel, smem, done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.B * p.U * p.topk_cluster));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.topk_cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel, (const float*)a.scores, a.seq_off, a.idx,
                            p.U, p.k);
}

}  // namespace salsc
