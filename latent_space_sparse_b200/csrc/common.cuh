// common.cuh -- internal definitions shared by the salsc CUDA sources.
//
// Nothing here is part of the public ABI (include/salsc.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>
#include <vector>

#include "salsc.h"

namespace salsc {

// Device-side anomaly flags (first word of the workspace).
enum : uint32_t {
  FLAG_BAD_INDEX = 1u << 0,  // a selected index fell outside its sequence
  FLAG_WAIT_TIMEOUT = 1u << 1,  // a bounded pipeline wait gave up
};

constexpr int kMaxRank = 512;

// Split partials: one row of part_row(r) floats per (sequence, query head,
// slot): m, l, two unused words, then acc[r] at kPartAcc, so that every row
// starts on a 16-byte boundary (rows are copied whole with cp.async.bulk).
constexpr int kPartAcc = 4;
__host__ __device__ constexpr int part_row(int r) { return r + kPartAcc; }

// Tile partition of the tensor-core attention: T tiles over g CTAs in
// contiguous ranges, CTA c from share_begin(c) to share_begin(c + 1).  The
// first T % g CTAs take one tile more: CTAs are dispatched in index order,
// so the longer ranges go to the CTAs that start first.
__host__ __device__ constexpr int64_t share_begin(int64_t c, int64_t T, int64_t g) {
  return c * (T / g) + (c < T % g ? c : T % g);
}
// The CTA whose range holds tile t (0 <= t < T).
__host__ __device__ constexpr int64_t share_of_tile(int64_t t, int64_t T, int64_t g) {
  return t < (T % g) * (T / g + 1) ? t / (T / g + 1)
                                   : T % g + (t - (T % g) * (T / g + 1)) / (T / g);
}
constexpr int kMaxHeadDim = 128;
constexpr int kMaxUnits = 256;  // KV heads per layer
constexpr size_t kWsAlign = 256;
constexpr int kMaxShardCandidates = 16384;  // token-sharded selection: shards x k per unit

// Host-side plan of one decode layer-step, derived from the descriptor only.
struct DecodePlan {
  int B, Hq, U, G, d, r, k;
  int npad;             // rows of the split latent query per sequence: 2U rounded up to 16
  salsc_dtype dtype;
  int64_t N, n_max;
  int n_score_tiles;    // sum_b ceil(n_b / score tile)
  int score_tile;       // tokens per scoring CTA
  int n_score_chunks;   // sum_b ceil(n_b / 32): the tensor-core scoring kernel's work items
  int64_t uni_nb;       // the common length when every sequence has it, else 0
  int topk_cluster;     // CTAs per selection unit in the top-k kernel
  int topk_slice;       // max keys per top-k CTA
  int topk_threads;     // threads per top-k CTA (1024, or 256 for many small units)
  uint32_t topk_kthr;   // threshold selection: order key of the threshold (0: plain top-k)
  int splits;           // partial-result slots per head (attention CTAs or tiles per unit)
  int chunk;            // kept tokens per slot
  bool attend_tc;       // tensor-core attention path (tiles of 128 kept tokens)
  int att_tiles;        // sum over units of ceil(k_b / 128) (tensor-core path)
  int att_cluster;      // > 0: the attention kernel merges each unit's partials and projects
                        // them itself, one cluster of att_cluster CTAs per unit (no merge kernel)
                        // (else a contiguous range of all tiles)
  float scale;
  double rope_base;
  // workspace layout (byte offsets)
  size_t off_flags, off_qlat, off_qsplit, off_scores, off_krange, off_idx, off_part, total;
};

// Raw pointers of one decode call, passed to the launchers.
struct DecodeArgs {
  const void* q;
  const void* Kc;
  const void* Vc;
  const void* Pk;
  const void* Pv;
  void* out;
  int32_t* idx;  // [B][U][k] (caller's or workspace)
  const int64_t* seq_off;
  const int64_t* seq_off_host = nullptr;  // the same offsets on the host (launch shapes)
  const int32_t* q_pos;
  uint32_t* flags;
  float* qlat;                 // [B][U][r]
  __nv_bfloat16* qsplit;       // [B][npad][r]: row 2u = hi(q_lat[u]), 2u+1 = lo, rest zero
  float* scores;               // packed per (b,u)
  uint32_t* krange;            // [B][U][2] (min, max) order key of each unit's scores
  float* part;                 // [B][Hq][splits][part_row(r)]
  const int64_t* pos_off = nullptr;  // [B] or null: added to a kept token's index for RoPE
  uint64_t* trace = nullptr;         // traced step: [kernel][cta][3] timestamps, or null
};

// Timeline of a traced step (salsc_decode_step_traced): kernel k of the step
// writes, for CTA c < SALSC_TRACE_MAX_CTAS (c = blockIdx.y * gridDim.x +
// blockIdx.x), the global nanosecond timer at three points into
// trace[(k * SALSC_TRACE_MAX_CTAS + c) * 3 + {0, 1, 2}]: its start, the
// return of its dependency wait, and its end.  Untraced steps pass null.
enum { TRACE_START = 0, TRACE_WAITED = 1, TRACE_END = 2 };
__device__ __forceinline__ void trace_stamp(uint64_t* kernel_trace, int which) {
  if (!kernel_trace) return;
  const unsigned c = blockIdx.y * gridDim.x + blockIdx.x;
  if (c >= (unsigned)SALSC_TRACE_MAX_CTAS) return;
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  kernel_trace[(size_t)c * 3 + which] = t;
}
// The trace rows of stage k (null when the step is not traced).
inline uint64_t* trace_of(const DecodeArgs& a, int k) {
  return a.trace ? a.trace + (size_t)k * SALSC_TRACE_MAX_CTAS * 3 : nullptr;
}

// Record a CUDA error for salsc_last_cuda_error() and return SALSC_ERR_CUDA.
salsc_status record_cuda_error(cudaError_t e);

// The checks salsc_decode_step makes on its descriptor and pointers (all but
// the workspace); host only, enqueues nothing.
salsc_status check_decode_step(const salsc_decode_desc* desc, const void* q, const void* Kc,
                               const void* Vc, const void* Pk, const void* Pv, const void* out,
                               const int32_t* idx_out);

// salsc_decode_step that first clears the workspace's anomaly word on the
// stream, after every argument has been checked (a rejected call enqueues
// nothing).
salsc_status decode_step_clearing_flags(const salsc_decode_desc* desc, const void* q,
                                        const void* Kc, const void* Vc, const void* Pk,
                                        const void* Pv, void* out, int32_t* idx_out, void* ws,
                                        size_t ws_bytes, salsc_stream stream);

// Launchers (each returns the cudaError_t of its launch).
cudaError_t launch_latent_q(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_score(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_topk(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_attend(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_combine(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s);
// Token-sharded decode (shard.cu, combine.cu): the local selection as
// candidates (score, global index); the global selection of this shard's
// tokens; the merged partial row of every head; the merge of the shards' rows.
cudaError_t launch_shard_gather(const DecodePlan& p, const DecodeArgs& a, const int64_t* shard_off,
                                float* cand_score, int32_t* cand_idx, cudaStream_t s);
cudaError_t launch_shard_select(const float* cand_score, const int32_t* cand_idx, int N, int B,
                                int U, int k, const int64_t* local_off, const int64_t* shard_off,
                                int32_t* idx_local, cudaStream_t s);
cudaError_t launch_combine_partial(const DecodePlan& p, const DecodeArgs& a, float* part_out,
                                   cudaStream_t s);
cudaError_t launch_shard_merge(const DecodePlan& p, const float* part_all, int n_shards,
                               const void* Pv, void* out, uint32_t* flags, cudaStream_t s);
bool attend_tc_supported(const DecodePlan& p);
int attend_merge_cluster(const DecodePlan& p);  // 0: merge kernel; else CTAs per unit
size_t fit_workspace_size(int64_t hidden, int64_t rank);
cudaError_t fit_projection(const void* X, int64_t n, int hidden, int rank, const float* omega,
                           int iters, void* P_out, salsc_dtype dt, void* ws, cudaStream_t s);
int attend_tc_grid(const DecodePlan& p);  // CTAs of the tensor-core attention (tile partition)
bool combine_supported(const DecodePlan& p);
cudaError_t launch_attend_tc(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_compress(const void* X, const void* P, void* Y, int64_t n, int hid, int r,
                            salsc_dtype dt, cudaStream_t s);
bool compress_tc_supported(int hid, int r, salsc_dtype dt);
// Decode-time append: Y[i][rows[b]] = X[i][b] . Pm[i] for the n_mats (1 or 2) matrices.
cudaError_t launch_append(const void* const X[2], const void* const Pm[2], void* const Y[2],
                          int n_mats, const int64_t* rows, int B, int hid, int r, salsc_dtype dt,
                          cudaStream_t s);
// Tensor-core compression of n_mats (1 or 2) matrices X[i] . Pm[i] -> Y[i] in one launch.
cudaError_t launch_compress_tc(const void* const X[2], const void* const Pm[2], void* const Y[2],
                               int n_mats, int64_t n, int hid, int r, cudaStream_t s);

// Raise a kernel's dynamic shared-memory limit once per device (not on every
// launch, so that launches inside CUDA-graph capture make no attribute calls).
constexpr int kMaxDevices = 64;
template <typename K>
cudaError_t ensure_smem(K* kernel, size_t bytes, int (&done)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if ((int)bytes <= done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done[dev] = (int)bytes;
  return e;
}

// Every decode kernel asks for the largest shared-memory carveout, so that an
// SM still running one kernel's CTAs can take the next kernel's CTAs (launched
// early by programmatic dependent launch) without first draining to change its
// L1 / shared-memory split.  Set once per kernel and device.
inline cudaError_t prefer_max_shared(const void* fn) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& d : done)
    if (d.first == fn && d.second == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done.emplace_back(fn, dev);
  return e;
}

// Launch `kernel` on `s`; with `pdl` the launch may begin while the previous
// kernel on the stream is still running (programmatic dependent launch): the
// kernel must execute grid_dependency_wait() before it reads anything the
// previous kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     bool pdl, Args&&... args) {
  const cudaError_t e = prefer_max_shared((const void*)kernel);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Wait until the kernels this one depends on have finished and their writes
// are visible (no-op when the kernel was launched without PDL).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Let the next kernel on the stream be scheduled now (it still waits, with
// grid_dependency_wait, for this kernel to finish before reading its output).
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- device helpers

// Shared-memory address of `p` in cluster CTA `rank` (thread-block clusters).
__device__ __forceinline__ uint32_t cluster_addr(const void* p, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"(rank));
  return r;
}
// Store and atomic add into the shared memory of another CTA of the cluster:
// no reply is awaited, and the next cluster barrier makes them visible.
__device__ __forceinline__ void st_cluster(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_cluster(uint32_t addr, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Load from the shared memory of a CTA of the cluster (waits for the reply).
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Split cluster barrier: arrive (releasing this thread's shared-memory reads
// and writes) and, later, wait for every thread of the cluster to arrive.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}


template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Unsigned key with the same order as the float; -0 and +0 map to one key.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Locate the tile `tile` of a ragged batch where sequence b has
// ceil(n_b / tile_len) tiles; returns b and the first token of the tile.
__device__ __forceinline__ void find_tile(const int64_t* __restrict__ seq_off, int B, int tile_len,
                                          int tile, int& b_out, int64_t& t0_out) {
  int acc = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t nb = seq_off[b + 1] - seq_off[b];
    const int nt = (int)((nb + tile_len - 1) / tile_len);
    if (tile < acc + nt) {
      b_out = b;
      t0_out = (int64_t)(tile - acc) * tile_len;
      return;
    }
    acc += nt;
  }
  b_out = -1;
  t0_out = 0;
}

// Walks consecutive fixed-length tiles of a ragged batch: each sequence has
// ceil(n_b / tile_len) tiles; sequence offsets are read only when the cursor
// enters a new sequence.
struct TileCursor {
  const int64_t* seq_off;
  int B, tile_len;
  int b;
  int64_t t0, off, nb;
  __device__ __forceinline__ void start(const int64_t* so, int B_, int len, int tile) {
    seq_off = so;
    B = B_;
    tile_len = len;
    find_tile(so, B_, len, tile, b, t0);
    load();
  }
  __device__ __forceinline__ void load() {
    if (b >= 0 && b < B) {
      off = seq_off[b];
      nb = seq_off[b + 1] - off;
    }
  }
  __device__ __forceinline__ void next() {
    t0 += tile_len;
    if (t0 >= nb) {
      ++b;
      t0 = 0;
      load();
    }
  }
};

}  // namespace salsc
