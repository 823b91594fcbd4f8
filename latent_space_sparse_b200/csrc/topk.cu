// topk.cu -- exact per-unit top-k by radix select in shared memory.
//
// SALS keeps only the most important tokens of each unit (page section "key
// designs": Top-K selection).  k_b = min(k, n_b) tokens with the largest
// score are kept; among equal scores the lower token index wins; slots
// k_b..k-1 are set to -1.
//
// Design: C CTAs (a thread-block cluster when C > 1) own one unit.  Each CTA
// loads a contiguous slice of the unit's scores into shared memory once, as
// 32-bit keys whose unsigned order is the float order; the unit's score range
// [min, max] comes from the scoring kernel.  Each CTA histograms its slice
// into 1024 bins of equal width over that range (the bin is a monotone
// function of the score, and scores spread over many bins, so the
// shared-memory atomics barely contend) and adds it into every CTA's copy of
// the cluster histogram through distributed shared memory; every CTA then
// finds, with a block-wide scan, the bin that holds the k_b-th largest score.
// A second pass packs, per warp segment, the indices of the keys above that
// bin (all kept) and stores the (key, index) pairs inside it, which are few
// for any smooth score distribution, into every CTA's candidate list; each
// CTA ranks its own pairs (score descending, index ascending) against the
// whole list, and the pairs ranked below the number still needed are kept.
// The output holds the indices above the boundary bin first (in index order)
// and then the kept pairs in rank order, so the result is deterministic.
// Data crosses between the CTAs only as stores into the others' shared memory
// before a cluster barrier (no remote load waits for a reply).  When the
// boundary bin holds more pairs than one rank's part of the list (heavily
// repeated or extreme scores), a radix select on rel = key - kmin with 11-bit
// digits, starting at the top bit of the key range (at most three passes),
// finds the threshold instead, followed by a counting and a writing pass.  No
// full sort, no global-memory scratch.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace salsc {
namespace {

constexpr int kBatch = 8;  // keys a thread loads before converting them (the loop is unrolled: short code)
constexpr int kMaxCluster = 8;  // largest cluster of CTAs per unit

// Float whose order_key is `key` (-0 comes back as +0).
__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

constexpr int kBins = 2048;  // 11-bit digits of the radix fallback
constexpr int kDigit = 11;
constexpr int kLinBins = 1024;  // bins of the linear pass
constexpr int kCand = 1024;    // most candidates the boundary bin may hold for the fast path

// Bin of a key in the linear partition of [fmin, fmax] into kLinBins bins: a
// composition of monotone roundings, so a larger score never lands in a lower
// bin and equal scores share a bin.
__device__ __forceinline__ int linear_bin(uint32_t key, float fmin, float scale) {
  const float x = (key_float(key) - fmin) * scale;
  return min(kLinBins - 1, (int)x);
}

// Block-wide search for the digit that holds the target rank: cnt(i) is the
// count of bin i (ascending bins); bins are scanned from the top.  Thread t
// looks at the `per` bins nbins-1-t*per .. nbins-(t+1)*per (per = nbins /
// THREADS, at least 1).  Returns through s_digit / s_above / s_count (the
// digit's own count).
template <int THREADS, typename Cnt>
__device__ __forceinline__ void find_digit(Cnt cnt, uint32_t target, int nbins, uint32_t* wsum,
                                           uint32_t* s_digit, uint32_t* s_above,
                                           uint32_t* s_count) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = nbins / THREADS > 1 ? nbins / THREADS : 1;  // nbins / THREADS <= 8
  const int top = nbins - 1 - tid * per;
  uint32_t c[8];
  uint32_t mine = 0u;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = (j < per && top - j >= 0) ? cnt(top - j) : 0u;
    mine += c[j];
  }
  uint32_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = lane < THREADS / 32 ? wsum[lane] : 0u;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += t;
    }
    wsum[32 + lane] = x - v;  // exclusive prefix of the warps above
  }
  __syncthreads();
  uint32_t above = wsum[32 + warp] + incl - mine;  // keys in bins above this thread's
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < per && above < target && target <= above + c[j]) {
      *s_digit = (uint32_t)(top - j);
      *s_above = above;
      *s_count = c[j];
    }
    above += c[j];
  }
}

template <bool kCluster, int kThreads>
__device__ __forceinline__ void topk_body(const float* __restrict__ scores,
                                          const int64_t* __restrict__ seq_off,
                                          const uint32_t* __restrict__ krange,
                                          int32_t* __restrict__ idx_out, int U, int k,
                                          uint32_t kthr, int64_t uni_nb, uint64_t* trace) {
  constexpr int kWarps = kThreads / 32;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = kCluster ? (int)cluster.num_blocks() : 1;
  const int rank = kCluster ? (int)cluster.block_rank() : 0;
  const int unit = blockIdx.x / C;
  const int b = unit / U, u = unit % U;

  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[2][kBins];  // [0]: this CTA's histogram, [1]: the cluster's candidates
  __shared__ uint32_t total[kBins];    // the cluster histogram
  __shared__ uint32_t wsum[64];
  __shared__ uint32_t counts[2];       // fallback: this CTA's (#keys > T, #keys == T)
  __shared__ uint32_t wcnt[kWarps][2];
  __shared__ uint32_t wbase[kWarps][2];
  __shared__ uint32_t s_nq[kMaxCluster], s_gq[kMaxCluster];  // per rank: candidates, keys above
  __shared__ uint32_t s_digit, s_above, s_count, s_base_gt, s_base_eq, s_ncand, s_ngt;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) trace_stamp(trace, TRACE_START);
  // shared memory of cluster rank q (this CTA's own when not a cluster)
  auto remote = [&](uint32_t* ptr, int q) -> uint32_t* {
    return kCluster ? cluster.map_shared_rank(ptr, q) : ptr;
  };
  auto cluster_sync = [&]() {
    if (kCluster) cluster.sync(); else __syncthreads();
  };
  for (int i = tid; i < kLinBins; i += kThreads) {
    hist[0][i] = 0u;
    total[i] = 0u;
  }
  if (tid == 0) s_ncand = 0u;
  allow_dependent_launch();
  // equal lengths: the unit's scores are found without a load
  const int64_t off = uni_nb > 0 ? (int64_t)b * uni_nb : seq_off[b];
  const int64_t nb = uni_nb > 0 ? uni_nb : seq_off[b + 1] - off;
  const int64_t kb = nb < k ? nb : k;
  const float* s = scores + off * U + (int64_t)u * nb;
  const int64_t lo = nb * rank / C, hi = nb * (rank + 1) / C;
  const int n_loc = (int)(hi - lo);
  const int seg = (n_loc + kWarps - 1) / kWarps;  // warp w owns keys [w*seg, (w+1)*seg)
  const int s0 = warp * seg, s1 = min(s0 + seg, n_loc);
  const uint32_t lt_mask = (1u << lane) - 1u;
  int32_t* out = idx_out + ((int64_t)b * U + u) * k;
  // Threshold selection (kthr > 0): keys below kthr are not kept, so the
  // kept tokens are not all k_b; every slot starts at -1 and the kept ones are
  // written over it after a cluster barrier.
  const bool keep_all = kb == nb && kthr == 0u;
  // From here on the other CTAs of the cluster may add into this CTA's zeroed
  // cluster histogram (they wait for this arrival before they do).
  if (kCluster && !keep_all) cluster_arrive();
  grid_dependency_wait();  // the scores and their range come from the previous kernel
  if (tid == 0) trace_stamp(trace, TRACE_WAITED);
  if (keep_all) {
    // keep every token, in index order
    for (int i = tid; i < n_loc; i += kThreads) out[lo + i] = (int32_t)(lo + i);
    if (rank == 0)
      for (int64_t j = kb + tid; j < k; j += kThreads) out[j] = -1;
    if (tid == 0) trace_stamp(trace, TRACE_END);
    return;
  }
  // the slice's first batch of scores is requested together with the unit's
  // key range (reduced by the scoring kernel): one round trip, not two
  float v0[kBatch];
#pragma unroll
  for (int j = 0; j < kBatch; ++j) {
    const int i = j * kThreads + tid;
    v0[j] = i < n_loc ? s[lo + i] : 0.f;
  }
  uint32_t kmin = krange[2 * ((int64_t)b * U + u)], kmax = krange[2 * ((int64_t)b * U + u) + 1];
  const float fmin = key_float(kmin), fmax = key_float(kmax);
  const float frange = fmax - fmin;
  const float scale = (float)kLinBins / frange;
  const bool lin = isfinite(frange) && frange > 0.f && isfinite(scale);
  const int n_iter = (n_loc + kThreads - 1) / kThreads;
  __syncthreads();  // the zeroed histogram and counters

  // ---- pass 1: keys of the slice into shared memory, histogram of their bins
  for (int base = 0; base < n_loc; base += kThreads * kBatch) {
    float v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = base + j * kThreads + tid;
      v[j] = base == 0 ? v0[j] : (i < n_loc ? s[lo + i] : 0.f);
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = base + j * kThreads + tid;
      if (i < n_loc) {
        const uint32_t key = order_key(v[j]);
        keys[i] = key;
        if (lin) atomicAdd(&hist[0][linear_bin(key, fmin, scale)], 1u);
      }
    }
  }
  if (kthr != 0u) {
    const int64_t j0 = (int64_t)k * rank / C, j1 = (int64_t)k * (rank + 1) / C;
    for (int64_t j = j0 + tid; j < j1; j += kThreads) out[j] = -1;
  }
  if (kCluster) cluster_wait();  // every CTA's cluster histogram is zeroed
  bool fast = lin;
  int bstar = 0;
  uint32_t need = 0u, n_cand = 0u;
  if (fast) {
    // this CTA's histogram is added into every CTA's cluster histogram (pushed,
    // not read back: a remote load waits for its reply)
    __syncthreads();
    for (int i = tid; i < kLinBins; i += kThreads) {
      const uint32_t c = hist[0][i];
      if (!kCluster) {
        total[i] = c;
      } else if (c != 0u) {
        for (int q = 0; q < C; ++q) red_add_cluster(cluster_addr(&total[i], q), c);
      }
    }
    cluster_sync();
    find_digit<kThreads>([&](int i) { return total[i]; }, (uint32_t)kb, kLinBins, wsum, &s_digit,
                         &s_above, &s_count);
    __syncthreads();
    bstar = (int)s_digit;
    need = (uint32_t)kb - s_above;  // 1 <= need <= count of bin bstar
    n_cand = s_count;
    fast = n_cand <= (uint32_t)(kCand / C);  // every rank's candidates fit its part of the list
  }
  if (fast) {
    // ---- pass 2: classify.  The indices of the keys above the boundary bin
    //      (all kept) are packed, in index order, at the start of the warp's
    //      segment of `keys` (a write never passes the key being read); the
    //      boundary bin's (key, index) pairs are stored into every CTA's
    //      candidate list, in this rank's part of it.
    const uint32_t cap = (uint32_t)(kCand / C);
    uint32_t* ckey = hist[1];          // [kCand] keys, rank q's at [q*cap, (q+1)*cap)
    uint32_t* cidx = hist[1] + kCand;  // their token indices
    uint32_t ngt = 0u;
    for (int c0 = s0; c0 < s1; c0 += 32) {
      const int i = c0 + lane;
      const bool valid = i < s1;
      const uint32_t key = valid ? keys[i] : 0u;
      const int bin = linear_bin(key, fmin, scale);
      const bool gt = valid && bin > bstar && key >= kthr, cand = valid && bin == bstar;
      const uint32_t bg = __ballot_sync(0xffffffffu, gt);
      if (cand) {
        const uint32_t slot = (uint32_t)rank * cap + atomicAdd(&s_ncand, 1u);
        if (!kCluster) {
          ckey[slot] = key;
          cidx[slot] = (uint32_t)(lo + i);
        } else {
          for (int q = 0; q < C; ++q) {
            st_cluster(cluster_addr(&ckey[slot], q), key);
            st_cluster(cluster_addr(&cidx[slot], q), (uint32_t)(lo + i));
          }
        }
      }
      if (gt) keys[s0 + ngt + __popc(bg & lt_mask)] = (uint32_t)(lo + i);
      ngt += __popc(bg);
    }
    if (lane == 0) wcnt[warp][0] = ngt;
    __syncthreads();
    // this rank's counts into every CTA
    if (warp == 0) {
      uint32_t x = lane < kWarps ? wcnt[lane][0] : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (lane < C) {
        if (!kCluster) {
          s_nq[0] = s_ncand;
          s_gq[0] = x;
        } else {
          st_cluster(cluster_addr(&s_nq[rank], lane), s_ncand);
          st_cluster(cluster_addr(&s_gq[rank], lane), x);
        }
      }
    }
    cluster_sync();  // every CTA's candidates and counts have arrived
    // ---- output offsets: the keys above the boundary bin first (ranks, then
    //      warps, in index order), then the kept candidates best first
    if (warp == 0) {
      const uint32_t gq = lane < C ? s_gq[lane] : 0u;
      const uint32_t ngt_all = __reduce_add_sync(0xffffffffu, gq);
      const uint32_t before = __reduce_add_sync(0xffffffffu, lane < rank ? gq : 0u);
      const uint32_t mine = lane < kWarps ? wcnt[lane][0] : 0u;
      uint32_t x = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
      }
      if (lane < kWarps) wbase[lane][0] = before + x - mine;
      if (lane == 0) s_ngt = ngt_all;
    }
    __syncthreads();
    // ---- each of this CTA's candidates is ranked (score descending, index
    //      ascending) against the whole cluster's; it is kept when fewer than
    //      `need` pairs beat it, and that count is its place.  One warp per
    //      candidate.
    {
      const uint32_t ngt_all = s_ngt, n_own = s_nq[rank];
      for (uint32_t t = warp; t < n_own; t += kWarps) {
        const uint32_t kt = ckey[rank * cap + t], it_ = cidx[rank * cap + t];
        uint32_t better = 0u;
        for (int q = 0; q < C; ++q) {
          const uint32_t nq = s_nq[q];
          for (uint32_t j = lane; j < nq; j += 32) {
            const uint32_t kj = ckey[q * cap + j], ij = cidx[q * cap + j];
            better += (kj > kt) || (kj == kt && ij < it_);
          }
        }
        better = __reduce_add_sync(0xffffffffu, better);
        if (lane == 0 && better < need && kt >= kthr) out[ngt_all + better] = (int32_t)it_;
      }
    }
    // ---- pass 3: the packed indices of this warp's keys above the boundary bin
    {
      const uint32_t n_w = wcnt[warp][0], base = wbase[warp][0];
      for (uint32_t j = lane; j < n_w; j += 32) out[base + j] = (int32_t)keys[s0 + j];
    }
    if (rank == 0)
      for (int64_t j = kb + tid; j < k; j += kThreads) out[j] = -1;
    if (tid == 0) trace_stamp(trace, TRACE_END);
    // nothing reads or writes this CTA's shared memory from other CTAs any more
    return;
  }
  // ======== fallback: radix select over the keys' bits
  if (lin && kCluster) cluster.sync();  // the others are done reading this histogram
  uint64_t prefix = 0u;
  uint32_t remaining = (uint32_t)kb;
  uint32_t T = 0u;
  {
    const uint32_t range = kmax - kmin;
    int hi_bit = range == 0u ? 0 : 32 - __clz(range);  // bits of rel still to resolve: [0, hi_bit)
    int pass = 0;
    while (hi_bit > 0) {
      const int width = hi_bit < kDigit ? hi_bit : kDigit;
      const int lo_bit = hi_bit - width;
      uint32_t* h = hist[pass & 1];
      for (int i = tid; i < kBins; i += kThreads) h[i] = 0u;
      __syncthreads();
      for (int it = 0; it < n_iter; ++it) {
        const int i = it * kThreads + tid;
        if (i < n_loc) {
          const uint64_t rel = (uint64_t)(keys[i] - kmin);
          if ((rel >> hi_bit) == (prefix >> hi_bit))
            atomicAdd(&h[(uint32_t)(rel >> lo_bit) & ((1u << width) - 1u)], 1u);
        }
      }
      const uint32_t* cnt = h;
      if (kCluster) {
        cluster.sync();
        for (int i = tid; i < kBins; i += kThreads) {
          uint32_t t = 0u;
#pragma unroll
          for (int q = 0; q < kMaxCluster; ++q)
            if (q < C) t += remote(h, q)[i];
          total[i] = t;
        }
        cnt = total;
      }
      __syncthreads();
      find_digit<kThreads>([&](int i) { return cnt[i]; }, remaining, 1 << width, wsum, &s_digit,
                           &s_above, &s_count);
      __syncthreads();
      prefix |= (uint64_t)s_digit << lo_bit;
      remaining -= s_above;
      hi_bit = lo_bit;
      ++pass;
    }
    T = kmin + (uint32_t)prefix;
  }
  const uint32_t need_eq = remaining;
  const uint32_t n_gt_total = (uint32_t)kb - need_eq;

  // ---- compaction: warp w owns keys [w*seg, min((w+1)*seg, n_loc))
  uint32_t cgt = 0u, ceq = 0u;
  for (int i = s0 + lane; i < s1; i += 32) {
    const uint32_t key = keys[i];
    cgt += key > T && key >= kthr;
    ceq += key == T && key >= kthr;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cgt += __shfl_xor_sync(0xffffffffu, cgt, o);
    ceq += __shfl_xor_sync(0xffffffffu, ceq, o);
  }
  if (lane == 0) {
    wcnt[warp][0] = cgt;
    wcnt[warp][1] = ceq;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t g = lane < kWarps ? wcnt[lane][0] : 0u, e = lane < kWarps ? wcnt[lane][1] : 0u;
    uint32_t ig = g, ie = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t tg = __shfl_up_sync(0xffffffffu, ig, o);
      const uint32_t te = __shfl_up_sync(0xffffffffu, ie, o);
      if (lane >= o) {
        ig += tg;
        ie += te;
      }
    }
    if (lane < kWarps) {
      wbase[lane][0] = ig - g;
      wbase[lane][1] = ie - e;
    }
    if (lane == 31) {
      counts[0] = ig;
      counts[1] = ie;
    }
  }
  if (kCluster) {
    cluster.sync();
    if (tid == 0) {
      uint32_t g = 0u, e = 0u;
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        if (q < rank) {
          const uint32_t* rc = remote(counts, q);
          g += rc[0];
          e += rc[1];
        }
      }
      s_base_gt = g;
      s_base_eq = e;
    }
  } else if (tid == 0) {
    s_base_gt = 0u;
    s_base_eq = 0u;
  }
  __syncthreads();

  uint32_t run_gt = s_base_gt + wbase[warp][0], run_eq = s_base_eq + wbase[warp][1];
  for (int c0 = s0; c0 < s1; c0 += 32) {
    const int i = c0 + lane;
    const bool valid = i < s1;
    const uint32_t key = valid ? keys[i] : 0u;
    const bool g = valid && key > T && key >= kthr;
    const bool e = valid && key == T && key >= kthr && need_eq > 0u;
    const uint32_t bg = __ballot_sync(0xffffffffu, g);
    const uint32_t be = __ballot_sync(0xffffffffu, e);
    if (g) out[run_gt + __popc(bg & lt_mask)] = (int32_t)(lo + i);
    if (e) {
      const uint32_t er = run_eq + __popc(be & lt_mask);
      if (er < need_eq) out[n_gt_total + er] = (int32_t)(lo + i);
    }
    run_gt += __popc(bg);
    run_eq += __popc(be);
  }
  if (rank == 0)
    for (int64_t j = kb + tid; j < k; j += kThreads) out[j] = -1;
  if (kCluster) cluster.sync();  // no CTA leaves while another may still read its counts
  if (tid == 0) trace_stamp(trace, TRACE_END);
}

// 1024-thread CTAs, at most 48 registers a thread: a CTA (49K registers) then
// fits beside one scoring CTA (10.8K), so the top-k CTAs, launched early,
// take an SM as soon as one of its two scoring CTAs has finished, not both.
template <bool kCluster>
__global__ void __maxnreg__(48)
topk1024_kernel(const float* __restrict__ scores, const int64_t* __restrict__ seq_off,
                const uint32_t* __restrict__ krange, int32_t* __restrict__ idx_out, int U,
                int k, uint32_t kthr, int64_t uni_nb, uint64_t* trace) {
  topk_body<kCluster, 1024>(scores, seq_off, krange, idx_out, U, k, kthr, uni_nb, trace);
}

// 256-thread CTAs (many small units, several CTAs per SM)
template <bool kCluster>
__global__ void __launch_bounds__(256)
topk256_kernel(const float* __restrict__ scores, const int64_t* __restrict__ seq_off,
               const uint32_t* __restrict__ krange, int32_t* __restrict__ idx_out, int U, int k,
               uint32_t kthr, int64_t uni_nb, uint64_t* trace) {
  topk_body<kCluster, 256>(scores, seq_off, krange, idx_out, U, k, kthr, uni_nb, trace);
}

template <bool kCluster, int kThreads>
constexpr auto topk_kernel_of() {
  if constexpr (kThreads == 1024) return topk1024_kernel<kCluster>;
  else return topk256_kernel<kCluster>;
}

template <bool kCluster, int kThreads>
cudaError_t launch_tk(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(uint32_t) * (size_t)p.topk_slice;
  static int done[kMaxDevices] = {};
  cudaError_t e = ensure_smem(topk_kernel_of<kCluster, kThreads>(), smem, done);
  if (e != cudaSuccess) return e;
  e = prefer_max_shared((const void*)topk_kernel_of<kCluster, kThreads>());
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.B * p.U * p.topk_cluster));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)p.topk_cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kCluster ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, topk_kernel_of<kCluster, kThreads>(), (const float*)a.scores,
                            (const int64_t*)a.seq_off, (const uint32_t*)a.krange, a.idx, p.U, p.k,
                            p.topk_kthr, p.uni_nb, trace_of(a, 2));
}

}  // namespace

cudaError_t launch_topk(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  // 1024 threads when the CTAs fit one per SM, else 256 (small units: many
  // CTAs resident per SM)
  const bool small = p.topk_threads == 256;
  if (p.topk_cluster == 1) return small ? launch_tk<false, 256>(p, a, s) : launch_tk<false, 1024>(p, a, s);
  return small ? launch_tk<true, 256>(p, a, s) : launch_tk<true, 1024>(p, a, s);
}

}  // namespace salsc
