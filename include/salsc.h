/*
 * salsc.h -- C ABI of the SALS latent-space sparse attention library (B200, sm_100a).
 *
 * The method is "SALS: Sparse Attention in Latent Space for KV cache
 * Compression" (arXiv 2510.24273v1).  Its technical-framework section has four
 * stages: (1) project keys and values into a low-dimensional latent space
 * with a low-rank matrix, (2) select the important tokens in that space with
 * a RoPE-free query-key interaction, (3) reconstruct only the selected
 * tokens, (4) run standard attention on them; its abstract explains that
 * RoPE can only be applied after reconstruction.  The attention formula
 * softmax(Q K^T / sqrt(d)) is the one printed in the VL-Cache OpenReview
 * response to reviewer KiPr, "On Weakness 1".
 *
 * Conventions for every entry point
 *   - All tensors are row-major and contiguous; every data pointer is a CUDA
 *     device pointer owned by the caller, unless its name ends in _host.
 *   - Nothing allocates, frees or synchronises.  Work is enqueued on the
 *     given stream (NULL = legacy default stream) and is asynchronous.  The
 *     library keeps no state between calls; concurrent calls on different
 *     workspaces are safe.
 *   - Argument errors are reported synchronously by the return value before
 *     anything is enqueued.  SALSC_ERR_CUDA means a launch failed; the CUDA
 *     error string is available from salsc_last_cuda_error() on that thread.
 *   - No C++ exception crosses this boundary.
 *
 * Storage types: SALSC_F32 (IEEE binary32) or SALSC_BF16 (bfloat16).  All
 * arithmetic accumulates in fp32; outputs are rounded once to the storage
 * type, round-to-nearest-even.
 */
#ifndef SALSC_H
#define SALSC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SALSC_OK = 0,
  SALSC_ERR_INVALID_ARG = 1, /* a shape, pointer or option is invalid */
  SALSC_ERR_UNSUPPORTED = 2, /* valid but no kernel for this shape/dtype */
  SALSC_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small */
  SALSC_ERR_CUDA = 4         /* a CUDA launch or runtime call failed */
} salsc_status;

typedef enum { SALSC_F32 = 0, SALSC_BF16 = 1 } salsc_dtype;

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* salsc_stream;

/*
 * Stage 1, low-rank projection (prefill compression):
 *     Kc = K . Pk     Vc = V . Pv
 * SALS technical framework, stage 1 ("project K and V into a low-dimensional
 * latent space with a low-rank matrix"); keys are projected before RoPE
 * (abstract: the selection interaction is RoPE-free).
 *
 *   K, V     [n_tokens][hidden]   keys (pre-RoPE) and values; either may be
 *                                 NULL to skip that half (its Kc/Vc and P are
 *                                 then ignored)
 *   Pk, Pv   [hidden][rank]       projections (orthonormal columns expected,
 *                                 not checked)
 *   Kc, Vc   [n_tokens][rank]     outputs, storage dtype
 *   hidden = n_kv_heads * head_dim.
 * Requirements: n_tokens >= 0, hidden >= 16 and rank >= 16 multiples of 16
 * for SALSC_BF16 (multiples of 4 for SALSC_F32); 16-byte aligned pointers.
 * Errors: INVALID_ARG on bad sizes, null required pointers or misalignment;
 * CUDA on launch failure.  Accumulation is fp32; one rounding to the dtype.
 */
salsc_status salsc_compress(const void* K, const void* V, const void* Pk, const void* Pv,
                            void* Kc, void* Vc, int64_t n_tokens, int32_t hidden, int32_t rank,
                            salsc_dtype dtype, salsc_stream stream);

/*
 * Shapes of one decode layer-step.  B sequences share one layer's
 * projections; sequence b owns latent rows seq_offsets[b] .. seq_offsets[b+1]-1
 * of Kc/Vc (a packed ragged cache), so n_b = seq_offsets[b+1]-seq_offsets[b].
 * Cached token t of sequence b sits at RoPE position t.
 *
 * Query head h belongs to KV head (selection unit) u = h / (n_q_heads /
 * n_kv_heads); unit u uses rows u*head_dim .. u*head_dim+head_dim-1 of Pk and
 * Pv.  With n_q_heads == n_kv_heads (MHA) every head is its own unit.
 */
typedef struct {
  int32_t batch;      /* B >= 1 */
  int32_t n_q_heads;  /* Hq, a multiple of n_kv_heads */
  int32_t n_kv_heads; /* Hkv = U, selection units per sequence */
  int32_t head_dim;   /* d, even; 64 or 128 supported */
  int32_t rank;       /* r, latent width; multiple of 64 (bf16) or 4 (f32), r <= 512 */
  int32_t top_k;      /* k >= 1 tokens kept per unit (k_b = min(k, n_b)) */
  const int64_t* seq_offsets_host; /* [B+1] on the host, for planning; [0] == 0, strictly increasing */
  const int64_t* seq_offsets_dev;  /* [B+1] the same values in device memory */
  const int32_t* q_pos_dev;        /* [B] query positions in device memory, or NULL for n_b */
  double rope_base;                /* RoPE base (10000, 500000, ...) > 1 */
  float softmax_scale;             /* 0 -> 1/sqrt(head_dim) */
  salsc_dtype dtype;               /* storage type of q, Kc, Vc, Pk, Pv and out */
  int32_t select_mode;             /* 0: top-k; 1: threshold selection: of the top-k tokens,
                                      those whose unit score is below select_threshold are
                                      dropped (slots left over hold -1; a head with no token
                                      left outputs zeros) */
  float select_threshold;          /* the threshold of select_mode 1 (not NaN) */
} salsc_decode_desc;

/*
 * Bytes of device workspace salsc_decode_step needs for this shape (0 if the
 * descriptor is invalid).  It depends on the shapes and seq_offsets_host only.
 */
size_t salsc_decode_workspace_size(const salsc_decode_desc* desc);

/*
 * Initialise a workspace: clears its device-side status word.  Call once per
 * workspace before the first salsc_decode_step (stream-ordered, no sync).
 * Errors: INVALID_ARG (bad desc), WORKSPACE (NULL, not 256-byte aligned or
 * smaller than salsc_decode_workspace_size), CUDA.
 */
salsc_status salsc_decode_prepare(const salsc_decode_desc* desc, void* ws, size_t ws_bytes,
                                  salsc_stream stream);

/*
 * One decode layer-step, stages 2-4 of the SALS technical framework:
 *
 *   for every sequence b and unit u:
 *     s[t]  = sum_{h in u} (q[b,h] . Pk_u) . Kc_b[t]        (RoPE-free, all t < n_b)
 *     S     = the k_b tokens with the largest s (ties -> lower t)
 *     for every query head h of u:
 *       K_t   = RoPE(Kc_b[t] . Pk_u^T, t),  V_t = Vc_b[t] . Pv_u^T    (t in S only)
 *       l_t   = RoPE(q[b,h], q_pos[b]) . K_t * softmax_scale
 *       out[b,h] = sum_{t in S} softmax(l)_t V_t
 *
 * RoPE is the rotate-half form on pairs (i, i + d/2) with angle
 * pos * rope_base^(-2i/d).
 *
 *   q        [B][Hq][d]        current queries, before RoPE, storage dtype
 *   Kc, Vc   [N][r]            latent cache, N = seq_offsets[B]
 *   Pk, Pv   [Hkv*d][r]        projections
 *   out      [B][Hq][d]        attention output, storage dtype
 *   idx_out  [B][U][k] int32   selected token indices within each sequence,
 *                              unordered, -1 in slots >= k_b; may be NULL
 *   ws       workspace of at least salsc_decode_workspace_size bytes,
 *            prepared once with salsc_decode_prepare; 256-byte aligned
 * No allocation, no host synchronisation: safe to capture in a CUDA graph.
 * Stream order: the kernels are launched with programmatic dependent launch.
 * Until the work enqueued before the step has finished, the step reads only
 * Pk; after that its later kernels may start early and read the other inputs
 * (Kc, Vc, Pv, q, the sequence offsets), so no input may change until the
 * step has completed.
 * Errors: INVALID_ARG (desc or null pointer), UNSUPPORTED (shape without a
 * kernel), WORKSPACE, CUDA.
 */
salsc_status salsc_decode_step(const salsc_decode_desc* desc, const void* q, const void* Kc,
                               const void* Vc, const void* Pk, const void* Pv, void* out,
                               int32_t* idx_out, void* ws, size_t ws_bytes, salsc_stream stream);

/*
 * salsc_append followed by salsc_decode_step in one call: the new token's key
 * and value rows (K_new, V_new [batch][Hkv*d], either may be NULL) are
 * projected and written to Kc/Vc at rows_dev[b] (as salsc_append), then the
 * step runs over the updated caches; its first kernel starts its weight loads
 * while the rows are written.  The descriptor's sequence lengths and q_pos
 * are taken as given: with the new token already in the cache (row
 * seq_offsets[b] + n_b - 1) the usual decode query position is n_b - 1, to be
 * passed in q_pos_dev.  Arguments otherwise as salsc_append and
 * salsc_decode_step; every argument is checked before anything is enqueued.
 * Errors: as salsc_decode_step, INVALID_ARG (both rows NULL, rows_dev NULL),
 * UNSUPPORTED (Hkv*d > 8192).
 */
salsc_status salsc_decode_step_append(const salsc_decode_desc* desc, const void* K_new,
                                      const void* V_new, const int64_t* rows_dev, const void* q,
                                      void* Kc, void* Vc, const void* Pk, const void* Pv,
                                      void* out, int32_t* idx_out, void* ws, size_t ws_bytes,
                                      salsc_stream stream);

/*
 * Stages of one decode layer-step, in order: latent query, latent scoring,
 * top-k, attention over the kept tokens, split merge (with the deferred value
 * projection).  Each stage is one kernel, except that for some shapes the
 * attention kernel merges its own partials (one thread-block cluster per
 * selection unit) and the merge stage launches nothing.
 */
#define SALSC_DECODE_KERNELS 5

/*
 * Number of kernels salsc_decode_step launches for this descriptor:
 * SALSC_DECODE_KERNELS, or one fewer when the attention kernel merges its own
 * partials (the descriptor's units, each given a cluster of up to 8 CTAs,
 * occupy at least as many SMs as an even split of the attention tiles, with
 * the latent width r <= 256); -1 when the descriptor is invalid or
 * unsupported.
 */
int32_t salsc_decode_launch_count(const salsc_decode_desc* desc);

/*
 * salsc_decode_step with timing marks: the same work, plus
 * cudaEventRecord(events[i], stream) just before stage i and
 * events[SALSC_DECODE_KERNELS] after the last, so that
 * cudaEventElapsedTime(events[i], events[i+1]) is stage i's time on the
 * stream (about zero for a merge stage that launches nothing).  events: SALSC_DECODE_KERNELS + 1 cudaEvent_t handles created by
 * the caller (cast to void*); n_events must equal that count.
 * Errors: as salsc_decode_step; INVALID_ARG for a missing or short event list.
 */
salsc_status salsc_decode_step_timed(const salsc_decode_desc* desc, const void* q, const void* Kc,
                                     const void* Vc, const void* Pk, const void* Pv, void* out,
                                     int32_t* idx_out, void* ws, size_t ws_bytes,
                                     salsc_stream stream, void* const* events, int32_t n_events);

/*
 * salsc_decode_step with a timeline: the same work, and every kernel of the
 * step records, per CTA, the global nanosecond timer (%globaltimer) when the
 * CTA starts, when its dependency wait on the previous stage returns, and
 * when it ends:
 *   trace[((k * SALSC_TRACE_MAX_CTAS) + c) * 3 + {0, 1, 2}]
 * for stage k < SALSC_DECODE_KERNELS (latent query, scoring, top-k,
 * attention, merge) and CTA c = blockIdx.y * gridDim.x + blockIdx.x <
 * SALSC_TRACE_MAX_CTAS.  Entries of CTAs that do not exist, and of kernels
 * that do not record (the CUDA-core scoring and attention of fp32 storage, a
 * merge stage that launches nothing), are left as they were: clear the buffer
 * first.  trace: device memory of at least trace_bytes >= 3 * 8 *
 * SALSC_DECODE_KERNELS * SALSC_TRACE_MAX_CTAS bytes, 8-byte aligned.  The
 * kernels are the ones salsc_decode_step launches, with the same launch
 * shapes and programmatic dependent launches; each stamp is one store.
 * Errors: as salsc_decode_step; INVALID_ARG for a missing, misaligned or short
 * trace buffer.
 */
#define SALSC_TRACE_MAX_CTAS 8192
salsc_status salsc_decode_step_traced(const salsc_decode_desc* desc, const void* q,
                                      const void* Kc, const void* Vc, const void* Pk,
                                      const void* Pv, void* out, int32_t* idx_out, void* ws,
                                      size_t ws_bytes, uint64_t* trace, size_t trace_bytes,
                                      salsc_stream stream);

/*
 * Decode step whose scratch is a fixed array inside the library, for callers
 * that cannot allocate device memory (no counterpart in the SALS paper).
 *
 * Some callers cannot hand the library a workspace: a plugin inside a host
 * application whose memory manager owns every device allocation, or a
 * serving loop that must never call cudaMalloc.  This entry point computes
 * exactly what salsc_decode_step computes, with the same arguments minus the
 * workspace, and allocates nothing (no cudaMalloc/cudaFree, no allocating
 * library routine).  The caller still owns q, Kc, Vc, Pk, Pv, out and idx_out.
 *
 *   - Limit: the shape's salsc_decode_workspace_size(desc) must not exceed
 *     SALSC_STATIC_WORKSPACE_BYTES (16 MiB; enough for every full-size
 *     workload of the test-suite, e.g. 4 x 32768 tokens x 8 KV heads or
 *     245760 ragged tokens x 8 KV heads).  Larger shapes return
 *     SALSC_ERR_WORKSPACE and enqueue nothing.
 *   - Every GPU that loads this part of the library keeps the 16 MiB array
 *     until the process exits.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress,
 *     with the caller's device current).  The first call on a device also
 *     loads the array's module: make that first call before any stream
 *     capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents; each call clears the part that must start at zero, after all
 *     its arguments have been checked (a rejected call enqueues nothing).
 *     Calls that overlap on the GPU (different streams, or different host
 *     threads without ordering) race on the array: serialise them.
 *   - The anomaly flags of this variant are not readable by the caller.
 * Errors: as salsc_decode_step; WORKSPACE when the shape needs more scratch.
 */
#define SALSC_STATIC_WORKSPACE_BYTES (16u << 20)
salsc_status salsc_decode_step_static_ws(const salsc_decode_desc* desc, const void* q,
                                         const void* Kc, const void* Vc, const void* Pk,
                                         const void* Pv, void* out, int32_t* idx_out,
                                         salsc_stream stream);

/* SALSC_STATIC_WORKSPACE_BYTES as compiled into the library, so that bindings
 * need not copy the constant. */
size_t salsc_static_workspace_bytes(void);

/*
 * Decode-time append (SALS technical framework, stage 1 applied to the token
 * being decoded): for every sequence b < batch,
 *   Kc[rows_dev[b]] = K_new[b] . Pk   and   Vc[rows_dev[b]] = V_new[b] . Pv
 * with fp32 accumulation and one rounding to the storage dtype.  Together with
 * the decode step this keeps the latent cache up to date token by token.
 *
 *   K_new, V_new [batch][hidden]  the new token's key (before RoPE) and value
 *                                 rows; either may be NULL to skip that half
 *   Pk, Pv       [hidden][rank]   projections (the ones given to compress)
 *   Kc, Vc       [*][rank]        latent caches, written at the given rows only
 *   rows_dev     [batch] int64    device array: destination row of sequence b
 *                                 (the caller's packing, e.g. seq_offsets[b]+n_b
 *                                 with spare capacity); rows must be distinct
 *                                 and inside Kc/Vc (not checked)
 * Allocates nothing, stream-ordered, graph-capturable.
 * Errors: INVALID_ARG (dtype, negative batch, null required pointer),
 * UNSUPPORTED (hidden > 8192), CUDA.
 */
salsc_status salsc_append(const void* K_new, const void* V_new, const void* Pk, const void* Pv,
                          void* Kc, void* Vc, const int64_t* rows_dev, int32_t batch,
                          int32_t hidden, int32_t rank, salsc_dtype dtype, salsc_stream stream);

/*
 * Learned projection (SALS page, key designs: a low-rank projection from the
 * SVD / PCA of the keys): P [hidden][rank] with orthonormal columns spanning
 * the dominant rank-dimensional right-singular subspace of a calibration
 * matrix X [n][hidden] (keys for Pk, values for Pv; pre-RoPE keys).  The decode
 * path uses P only through P P^T, so any orthonormal basis of the subspace is
 * equivalent; this one is the result of subspace iteration on the Gram matrix
 * C = X^T X from the random start omega:
 *     V_0 = orth(omega),  V_{i+1} = orth(C V_i) for i < iters,  P = V_iters
 * (orth: Cholesky-QR twice; all arithmetic fp64).  The subspace error falls
 * as (sigma_{rank+1} / sigma_rank)^(2 iters) of X's singular values.
 *
 *   X       [n][hidden]      calibration rows, dtype; n >= rank
 *   omega   [hidden][rank]   fp32 device array: the random start (e.g.
 *                            standard normal entries, drawn by the caller)
 *   P_out   [hidden][rank]   output, dtype
 *   ws      >= salsc_fit_workspace_size(hidden, rank) bytes of device memory,
 *           256-byte aligned (about 8*hidden^2 bytes); word 0 holds flags,
 *           read with salsc_decode_read_flags: bit 2 set when a Cholesky pivot
 *           was not positive (rank-deficient X or omega; P is then unreliable)
 * Requirements: 1 <= rank <= min(hidden, 1024), iters >= 0.  Stream-ordered,
 * allocates nothing.  Errors: INVALID_ARG (shapes, null pointers, dtype),
 * UNSUPPORTED (rank > 1024), WORKSPACE, CUDA.
 */
size_t salsc_fit_workspace_size(int32_t hidden, int32_t rank);
salsc_status salsc_fit_projection(const void* X, int64_t n, int32_t hidden, int32_t rank,
                                  const float* omega, int32_t iters, void* P_out,
                                  salsc_dtype dtype, void* ws, size_t ws_bytes,
                                  salsc_stream stream);

/*
 * Token-sharded decode: the tokens of every sequence split over N GPUs, shard
 * s holding a contiguous slice (its own Kc/Vc rows; q, Pk, Pv replicated).
 * Selection stays exact: a token among a unit's k best overall has fewer than
 * k better tokens in its slice, so it is in that slice's local top-k (SALS
 * technical framework, stages 2-4; the pages run one GPU, the exchange is this
 * library's).  One layer-step on every shard, with the caller's all-gathers
 * (e.g. NCCL) between the calls:
 *   1. salsc_shard_candidates   local scoring + top-k -> (score, global index)
 *   2. all-gather the candidates of the N shards
 *   3. salsc_shard_select       the same global top-k on every shard; this
 *                               shard's tokens as local indices
 *   4. salsc_shard_attend       attention over them -> one partial row per head
 *   5. all-gather the partial rows
 *   6. salsc_shard_merge        merge the N rows of every head, apply Pv
 * The result equals salsc_decode_step on the whole sequences (up to rounding
 * order); ties in score go to the lower global token index.  The shard's
 * descriptor describes its slices (seq_offsets: local lengths).
 *
 * salsc_shard_candidates: stages 2 and top-k on this shard's slices.
 *   shard_off_dev [B] int64   global index of the slice's first token
 *   cand_score    [B][U][k]   fp32 score of each locally kept token (-inf in
 *                             empty slots)
 *   cand_idx      [B][U][k]   int32 global token index (-1 in empty slots)
 *   ws            workspace of salsc_decode_workspace_size(desc), prepared
 * With select_mode 1 the local top-k keeps only scores >= select_threshold
 * (dropped slots are empty candidates); the global selection of step 3 then
 * equals threshold selection on the whole sequences: a kept token is among
 * the k best overall with a score >= the threshold, so it is a candidate of
 * its slice, and every candidate clears the threshold.
 *
 * salsc_shard_select: per unit, the k best of the N*k gathered candidates
 * (score descending, lower global index first among equal scores; empty
 * candidates never selected), by an exact radix select.
 *   cand_score_all [N][B][U][k], cand_idx_all [N][B][U][k]  the gathered
 *                  candidates, shard-major (an all-gather's layout)
 *   local_offsets_dev [B+1] int64  this shard's slice offsets (its descriptor's
 *                  seq_offsets_dev); shard_off_dev [B] as above
 *   idx_local [B][U][k] int32  this shard's selected tokens as slice-local
 *                  indices, in candidate order, then -1
 * Requires N*k <= 16384, U <= 256 (UNSUPPORTED otherwise).
 *
 * salsc_shard_attend: stages 3-4 over idx_local, without the projection.
 *   desc->q_pos_dev is required (the query's global position); RoPE of a kept
 *   token uses shard_off_dev[b] + its local index.
 *   part_out [B][Hq][r+4] fp32, 16-byte aligned: per head (m, l, 0, 0,
 *   acc[r]): the maximum logit over this shard's kept tokens (-inf if none),
 *   the softmax normaliser relative to it, and the unnormalised latent value
 *   sum sum_t e^{l_t - m} Vc[t].
 *
 * salsc_shard_merge: out[b][h] = (sum_s w_s acc_s / sum_s w_s l_s) . Pv_u^T
 * with w_s = e^{m_s - max_s m_s}, over the N gathered rows part_all
 * [N][B][Hq][r+4] (16-byte aligned).  ws: any prepared decode workspace
 * (word 0 records wait timeouts).
 *
 * All four are stream-ordered and allocate nothing.  Their kernels use
 * programmatic dependent launch: in salsc_shard_attend and salsc_shard_merge,
 * Pk, Pv, q and the sequence and slice offsets may be read before the work
 * enqueued ahead of the call has finished (in salsc_shard_candidates only Pk,
 * as in salsc_decode_step), so the work before the call must not write them
 * while it runs; Kc, Vc, the candidates, idx_local and the partial rows are
 * read only after it.  Errors: INVALID_ARG
 * (null or misaligned pointers, shapes, missing q_pos), UNSUPPORTED,
 * WORKSPACE, CUDA.
 */
salsc_status salsc_shard_candidates(const salsc_decode_desc* desc, const void* q, const void* Kc,
                                    const void* Pk, const int64_t* shard_off_dev,
                                    float* cand_score, int32_t* cand_idx, void* ws,
                                    size_t ws_bytes, salsc_stream stream);
salsc_status salsc_shard_select(const float* cand_score_all, const int32_t* cand_idx_all,
                                int32_t n_shards, int32_t batch, int32_t n_units, int32_t top_k,
                                const int64_t* local_offsets_dev, const int64_t* shard_off_dev,
                                int32_t* idx_local, salsc_stream stream);
salsc_status salsc_shard_attend(const salsc_decode_desc* desc, const void* q, const void* Kc,
                                const void* Vc, const void* Pk, const int32_t* idx_local,
                                const int64_t* shard_off_dev, float* part_out, void* ws,
                                size_t ws_bytes, salsc_stream stream);
salsc_status salsc_shard_merge(const float* part_all, int32_t n_shards, int32_t batch,
                               int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                               int32_t rank, salsc_dtype dtype, const void* Pv, void* out,
                               void* ws, size_t ws_bytes, salsc_stream stream);

/*
 * Device-side anomaly flags recorded in a workspace since salsc_decode_prepare
 * (bit 0: a selected index fell outside its sequence; bit 1: a pipeline wait
 * gave up after its iteration limit).  Copies one word to *flags_host and
 * synchronises the stream.  Returns INVALID_ARG/WORKSPACE/CUDA on failure.
 */
salsc_status salsc_decode_read_flags(void* ws, size_t ws_bytes, uint32_t* flags_host,
                                     salsc_stream stream);

/*
 * Check of the device-side failure path (no counterpart in the SALS paper):
 * one kernel runs the bounded wait that every pipeline wait of the decode
 * kernels uses, on an mbarrier phase that nothing completes, with a limit of
 * limit_ns nanoseconds (1 .. 1e9) instead of the kernels' 2 s.  The wait gives
 * up, sets bit 1 (wait timeout) in the workspace's anomaly word and the kernel
 * returns; no copy is in flight meanwhile.  Read the word with
 * salsc_decode_read_flags; clear it with salsc_decode_prepare.
 *   ws   a decode workspace (or any 256-byte aligned device buffer of at
 *        least 16 bytes); only its anomaly word is written
 * Errors: INVALID_ARG (limit out of range), WORKSPACE, CUDA.
 */
salsc_status salsc_check_wait_timeout(uint64_t limit_ns, void* ws, size_t ws_bytes,
                                      salsc_stream stream);

/* Static description of a status code. */
const char* salsc_status_string(salsc_status status);

/* Text of the last CUDA error seen by this library on the calling thread. */
const char* salsc_last_cuda_error(void);

/* Library version string. */
const char* salsc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SALSC_H */
