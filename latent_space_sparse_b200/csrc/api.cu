// api.cu -- the extern "C" boundary of libsalsc: validation, planning,
// workspace layout and the launch sequence of one decode layer-step.
//
// Method: "SALS: Sparse Attention in Latent Space for KV cache Compression",
// technical framework, stages 1-4.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"

namespace {

thread_local char g_last_cuda_error[256] = "no error";

salsc_status cuda_fail(cudaError_t e) {
  snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", cudaGetErrorName(e),
           cudaGetErrorString(e));
  return SALSC_ERR_CUDA;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

constexpr int kScoreTile = 128;
constexpr int kFitMaxRank = 1024;  // learned projections: columns (one-CTA factorisations)
constexpr int kTopkTargetCtas = 148;    // top-k CTAs aimed at (one per SM)
constexpr int kTopkMinSlice = 4096;     // keys per CTA at which the cluster stops growing
constexpr int kTopkMaxSlice = 40960;    // keys per CTA in shared memory (160 KiB)
constexpr int kTopkMaxCluster = 8;
constexpr int kAttendTargetCtas = 2 * 148;

// Validate the descriptor and derive the plan.  Returns SALSC_OK or the error.
salsc_status make_plan(const salsc_decode_desc* D, salsc::DecodePlan* P) {
  if (!D || !D->seq_offsets_host) return SALSC_ERR_INVALID_ARG;
  if (D->batch < 1 || D->n_q_heads < 1 || D->n_kv_heads < 1 || D->head_dim < 2 || D->rank < 1 ||
      D->top_k < 1)
    return SALSC_ERR_INVALID_ARG;
  if (D->n_q_heads % D->n_kv_heads != 0 || D->head_dim % 2 != 0) return SALSC_ERR_INVALID_ARG;
  if (D->dtype != SALSC_F32 && D->dtype != SALSC_BF16) return SALSC_ERR_INVALID_ARG;
  if (!(D->rope_base > 1.0) || !isfinite(D->rope_base)) return SALSC_ERR_INVALID_ARG;
  if (!(D->softmax_scale >= 0.0f) || !isfinite(D->softmax_scale)) return SALSC_ERR_INVALID_ARG;
  if (D->seq_offsets_host[0] != 0) return SALSC_ERR_INVALID_ARG;
  int64_t n_max = 0;
  int n_tiles = 0, n_chunks = 0;
  for (int b = 0; b < D->batch; ++b) {
    const int64_t nb = D->seq_offsets_host[b + 1] - D->seq_offsets_host[b];
    if (nb < 1 || nb > (int64_t)INT32_MAX) return SALSC_ERR_INVALID_ARG;
    if (nb > n_max) n_max = nb;
    n_tiles += (int)((nb + kScoreTile - 1) / kScoreTile);
    n_chunks += (int)((nb + 31) / 32);
  }
  // shapes with kernels
  if (D->head_dim != 64 && D->head_dim != 128) return SALSC_ERR_UNSUPPORTED;
  if (D->rank > salsc::kMaxRank) return SALSC_ERR_UNSUPPORTED;
  if (D->n_kv_heads > salsc::kMaxUnits) return SALSC_ERR_UNSUPPORTED;
  if (D->dtype == SALSC_BF16 && D->rank % 64 != 0) return SALSC_ERR_UNSUPPORTED;
  if (D->dtype == SALSC_F32 && D->rank % 4 != 0) return SALSC_ERR_UNSUPPORTED;
  if (D->rank > D->n_kv_heads * D->head_dim) return SALSC_ERR_INVALID_ARG;

  salsc::DecodePlan p{};
  p.B = D->batch;
  p.Hq = D->n_q_heads;
  p.U = D->n_kv_heads;
  p.G = p.Hq / p.U;
  p.d = D->head_dim;
  p.r = D->rank;
  p.k = D->top_k;
  p.npad = (2 * p.U + 15) / 16 * 16;
  if (p.G > 8) return SALSC_ERR_UNSUPPORTED;  // the merge handles up to 8 query heads per unit
  p.dtype = D->dtype;
  p.N = D->seq_offsets_host[D->batch];
  p.n_max = n_max;
  p.score_tile = kScoreTile;
  p.n_score_tiles = n_tiles;
  p.n_score_chunks = n_chunks;
  p.uni_nb = D->seq_offsets_host[1];
  for (int b = 1; b < D->batch; ++b)
    if (D->seq_offsets_host[b + 1] - D->seq_offsets_host[b] != p.uni_nb) p.uni_nb = 0;
  // Top-k: C CTAs per unit, about one CTA per SM in all (up to 8 per unit, and
  // enough for a slice of the scores to fit shared memory); many small units
  // take 256-thread CTAs, several resident per SM.
  int c = 1;
  while (c < kTopkMaxCluster && (int64_t)p.B * p.U * c * 2 <= kTopkTargetCtas &&
         (n_max + c - 1) / c > kTopkMinSlice)
    c *= 2;
  while (c < kTopkMaxCluster && (n_max + c - 1) / c > kTopkMaxSlice) c *= 2;
  p.topk_cluster = c;
  p.topk_slice = (int)((n_max + c - 1) / c);
  if (p.topk_slice > kTopkMaxSlice) return SALSC_ERR_UNSUPPORTED;  // slice in smem
  p.topk_threads = (int64_t)p.B * p.U * c > kTopkTargetCtas ? 256 : 1024;
  // threshold selection: keys (order-preserving bit patterns of the fp32
  // scores) below the threshold's are dropped; 0 keeps every key
  if (D->select_mode != 0 && D->select_mode != 1) return SALSC_ERR_INVALID_ARG;
  p.topk_kthr = 0u;
  if (D->select_mode == 1) {
    if (isnan(D->select_threshold)) return SALSC_ERR_INVALID_ARG;
    float f = D->select_threshold;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (u == 0x80000000u) u = 0u;  // -0 is +0
    p.topk_kthr = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  }
  const int64_t k_eff = D->top_k < n_max ? D->top_k : n_max;
  p.attend_tc = salsc::attend_tc_supported(p);
  if (p.attend_tc) {
    // one partial slot per tile of 128 kept tokens
    p.chunk = 128;
    p.splits = (int)((k_eff + 127) / 128);
    int64_t tiles = 0;
    for (int b = 0; b < D->batch; ++b) {
      const int64_t nb = D->seq_offsets_host[b + 1] - D->seq_offsets_host[b];
      const int64_t kb = nb < D->top_k ? nb : D->top_k;
      tiles += (int64_t)p.U * ((kb + 127) / 128);
    }
    if (tiles > INT32_MAX) return SALSC_ERR_UNSUPPORTED;
    p.att_tiles = (int)tiles;
  } else {
    const int units = p.B * p.U;
    int splits = (kAttendTargetCtas + units - 1) / units;
    if (splits > 64) splits = 64;
    int chunk = (int)((k_eff + splits - 1) / splits);
    if (chunk < 64) chunk = 64;
    chunk = (chunk + 15) / 16 * 16;
    splits = (int)((k_eff + chunk - 1) / chunk);  // never more than before: chunk only grew
    if (splits < 1) splits = 1;
    p.splits = splits;
    p.chunk = chunk;
    p.att_tiles = 0;
  }
  p.att_cluster = p.attend_tc ? salsc::attend_merge_cluster(p) : 0;
  if (!salsc::combine_supported(p)) return SALSC_ERR_UNSUPPORTED;
  p.scale = D->softmax_scale != 0.0f ? D->softmax_scale : (float)(1.0 / sqrt((double)p.d));
  p.rope_base = D->rope_base;

  size_t off = 0;
  p.off_flags = off;
  off = align_up(off + 16, salsc::kWsAlign);
  p.off_qlat = off;
  off = align_up(off + sizeof(float) * (size_t)p.B * p.U * p.r, salsc::kWsAlign);
  p.off_qsplit = off;
  off = align_up(off + sizeof(__nv_bfloat16) * (size_t)p.B * p.npad * p.r, salsc::kWsAlign);
  p.off_scores = off;
  off = align_up(off + sizeof(float) * (size_t)p.N * p.U, salsc::kWsAlign);
  p.off_krange = off;
  off = align_up(off + sizeof(uint32_t) * 2 * (size_t)p.B * p.U, salsc::kWsAlign);
  p.off_idx = off;
  off = align_up(off + sizeof(int32_t) * (size_t)p.B * p.U * p.k, salsc::kWsAlign);
  p.off_part = off;
  off = align_up(off + sizeof(float) * (size_t)p.B * p.Hq * p.splits * salsc::part_row(p.r),
                 salsc::kWsAlign);
  p.total = off;
  *P = p;
  return SALSC_OK;
}

salsc_status check_ws(const salsc::DecodePlan& p, void* ws, size_t ws_bytes) {
  if (!ws || ((uintptr_t)ws % salsc::kWsAlign) != 0 || ws_bytes < p.total)
    return SALSC_ERR_WORKSPACE;
  return SALSC_OK;
}

}  // namespace

salsc_status salsc::record_cuda_error(cudaError_t e) { return cuda_fail(e); }

extern "C" {

const char* salsc_status_string(salsc_status st) {
  switch (st) {
    case SALSC_OK: return "ok";
    case SALSC_ERR_INVALID_ARG: return "invalid argument";
    case SALSC_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case SALSC_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SALSC_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* salsc_last_cuda_error(void) { return g_last_cuda_error; }

const char* salsc_version(void) { return "salsc 0.1 (sm_100a)"; }

int32_t salsc_decode_launch_count(const salsc_decode_desc* desc) {
  salsc::DecodePlan p;
  if (make_plan(desc, &p) != SALSC_OK) return -1;
  return p.att_cluster > 0 ? SALSC_DECODE_KERNELS - 1 : SALSC_DECODE_KERNELS;
}

size_t salsc_decode_workspace_size(const salsc_decode_desc* desc) {
  salsc::DecodePlan p;
  if (make_plan(desc, &p) != SALSC_OK) return 0;
  return p.total;
}

salsc_status salsc_decode_prepare(const salsc_decode_desc* desc, void* ws, size_t ws_bytes,
                                  salsc_stream stream) {
  salsc::DecodePlan p;
  salsc_status st = make_plan(desc, &p);
  if (st != SALSC_OK) return st;
  if ((st = check_ws(p, ws, ws_bytes)) != SALSC_OK) return st;
  cudaError_t e = cudaMemsetAsync((char*)ws + p.off_flags, 0, 16, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return SALSC_OK;
}

size_t salsc_fit_workspace_size(int32_t hidden, int32_t rank) {
  if (hidden < 1 || rank < 1 || rank > hidden || rank > kFitMaxRank) return 0;
  return salsc::fit_workspace_size(hidden, rank);
}

salsc_status salsc_fit_projection(const void* X, int64_t n, int32_t hidden, int32_t rank,
                                  const float* omega, int32_t iters, void* P_out,
                                  salsc_dtype dtype, void* ws, size_t ws_bytes,
                                  salsc_stream stream) {
  if (dtype != SALSC_F32 && dtype != SALSC_BF16) return SALSC_ERR_INVALID_ARG;
  if (!X || !omega || !P_out || hidden < 1 || rank < 1 || rank > hidden || n < rank ||
      n > INT32_MAX || iters < 0)
    return SALSC_ERR_INVALID_ARG;
  if (rank > kFitMaxRank) return SALSC_ERR_UNSUPPORTED;
  if (!ws || ((uintptr_t)ws % salsc::kWsAlign) != 0 ||
      ws_bytes < salsc::fit_workspace_size(hidden, rank))
    return SALSC_ERR_WORKSPACE;
  const cudaError_t e = salsc::fit_projection(X, n, hidden, rank, omega, iters, P_out, dtype, ws,
                                              (cudaStream_t)stream);
  return e == cudaSuccess ? SALSC_OK : cuda_fail(e);
}

salsc_status salsc_decode_read_flags(void* ws, size_t ws_bytes, uint32_t* flags_host,
                                     salsc_stream stream) {
  if (!flags_host) return SALSC_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws % salsc::kWsAlign) != 0 || ws_bytes < 16) return SALSC_ERR_WORKSPACE;
  cudaError_t e = cudaMemcpyAsync(flags_host, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost,
                                  (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return SALSC_OK;
}

salsc_status salsc_append(const void* K_new, const void* V_new, const void* Pk, const void* Pv,
                          void* Kc, void* Vc, const int64_t* rows_dev, int32_t batch,
                          int32_t hidden, int32_t rank, salsc_dtype dtype, salsc_stream stream) {
  if (dtype != SALSC_F32 && dtype != SALSC_BF16) return SALSC_ERR_INVALID_ARG;
  if (batch < 0 || hidden < 1 || rank < 1 || !rows_dev) return SALSC_ERR_INVALID_ARG;
  if (!K_new && !V_new) return SALSC_ERR_INVALID_ARG;
  if (K_new && (!Pk || !Kc)) return SALSC_ERR_INVALID_ARG;
  if (V_new && (!Pv || !Vc)) return SALSC_ERR_INVALID_ARG;
  if (hidden > 8 * 1024) return SALSC_ERR_UNSUPPORTED;
  if (batch == 0) return SALSC_OK;
  const void* X[2] = {K_new ? K_new : V_new, V_new};
  const void* Pm[2] = {K_new ? Pk : Pv, Pv};
  void* Y[2] = {K_new ? Kc : Vc, Vc};
  cudaError_t e = salsc::launch_append(X, Pm, Y, (K_new && V_new) ? 2 : 1, rows_dev, batch, hidden,
                                       rank, dtype, (cudaStream_t)stream);
  return e == cudaSuccess ? SALSC_OK : cuda_fail(e);
}

}  // extern "C"

namespace {

// The new token's rows, appended to the latent caches before the step reads
// them (salsc_decode_step_append).
struct AppendArgs {
  const void* K_new;
  const void* V_new;
  const int64_t* rows;
};

// Pointers of one call: the caller's arrays and the workspace's regions.
salsc::DecodeArgs make_args(const salsc::DecodePlan& p, const salsc_decode_desc* desc,
                            const void* q, const void* Kc, const void* Vc, const void* Pk,
                            const void* Pv, void* out, int32_t* idx_out, void* ws) {
  char* w = (char*)ws;
  salsc::DecodeArgs a;
  a.q = q;
  a.Kc = Kc;
  a.Vc = Vc;
  a.Pk = Pk;
  a.Pv = Pv;
  a.out = out;
  a.idx = idx_out ? idx_out : (int32_t*)(w + p.off_idx);
  a.seq_off = desc->seq_offsets_dev;
  a.seq_off_host = desc->seq_offsets_host;
  a.q_pos = desc->q_pos_dev;
  a.flags = (uint32_t*)(w + p.off_flags);
  a.qlat = (float*)(w + p.off_qlat);
  a.qsplit = (__nv_bfloat16*)(w + p.off_qsplit);
  a.scores = (float*)(w + p.off_scores);
  a.krange = (uint32_t*)(w + p.off_krange);
  a.part = (float*)(w + p.off_part);
  return a;
}

// The step's pointer arguments: present and aligned.
salsc_status check_step_pointers(const salsc_decode_desc* desc, const void* q, const void* Kc,
                                 const void* Vc, const void* Pk, const void* Pv, const void* out,
                                 const int32_t* idx_out) {
  if (!desc->seq_offsets_dev || !q || !Kc || !Vc || !Pk || !Pv || !out)
    return SALSC_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(Pk) || !aligned16(Pv) ||
      !aligned16(out) || ((uintptr_t)idx_out & 3u))
    return SALSC_ERR_INVALID_ARG;
  return SALSC_OK;
}

salsc_status decode_step_impl(const salsc_decode_desc* desc, const void* q, const void* Kc,
                              const void* Vc, const void* Pk, const void* Pv, void* out,
                              int32_t* idx_out, void* ws, size_t ws_bytes, salsc_stream stream,
                              void* const* events, int32_t n_events,
                              const AppendArgs* app = nullptr, bool clear_flags = false,
                              uint64_t* trace = nullptr) {
  salsc::DecodePlan p;
  salsc_status st = make_plan(desc, &p);
  if (st != SALSC_OK) return st;
  if (app) {
    if ((!app->K_new && !app->V_new) || !app->rows) return SALSC_ERR_INVALID_ARG;
    if (p.U * p.d > 8 * 1024) return SALSC_ERR_UNSUPPORTED;
  }
  if ((st = check_step_pointers(desc, q, Kc, Vc, Pk, Pv, out, idx_out)) != SALSC_OK) return st;
  if (events) {
    if (n_events != SALSC_DECODE_KERNELS + 1) return SALSC_ERR_INVALID_ARG;
    for (int i = 0; i < n_events; ++i)
      if (!events[i]) return SALSC_ERR_INVALID_ARG;
  }
  if ((st = check_ws(p, ws, ws_bytes)) != SALSC_OK) return st;

  salsc::DecodeArgs a = make_args(p, desc, q, Kc, Vc, Pk, Pv, out, idx_out, ws);
  a.trace = trace;

  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e0;
  // every argument has been checked: only now may anything be enqueued
  if (clear_flags && (e0 = cudaMemsetAsync((char*)ws + p.off_flags, 0, 16, s)) != cudaSuccess)
    return cuda_fail(e0);
  typedef cudaError_t (*launcher)(const salsc::DecodePlan&, const salsc::DecodeArgs&, cudaStream_t);
  const launcher seq[SALSC_DECODE_KERNELS] = {salsc::launch_latent_q, salsc::launch_score,
                                              salsc::launch_topk, salsc::launch_attend,
                                              salsc::launch_combine};
  // the tensor-core attention merges its own tiles (no separate merge kernel)
  cudaError_t e;
  if (app) {
    // the new rows first, in stream order (the step's kernels then wait for
    // them like for any earlier work); Kc and Vc are written, hence non-const
    const void* X[2] = {app->K_new ? app->K_new : app->V_new, app->V_new};
    const void* Pm[2] = {app->K_new ? Pk : Pv, Pv};
    void* Y[2] = {app->K_new ? (void*)Kc : (void*)Vc, (void*)Vc};
    if ((e = salsc::launch_append(X, Pm, Y, (app->K_new && app->V_new) ? 2 : 1, app->rows, p.B,
                                  p.U * p.d, p.r, p.dtype, s)) != cudaSuccess)
      return cuda_fail(e);
  }
  // Inside stream capture an event record must be an external node to
  // record at replay time.
  unsigned rec_flags = cudaEventRecordDefault;
  if (events) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if ((e = cudaStreamIsCapturing(s, &cs)) != cudaSuccess) return cuda_fail(e);
    if (cs == cudaStreamCaptureStatusActive) rec_flags = cudaEventRecordExternal;
  }
  for (int i = 0; i < SALSC_DECODE_KERNELS; ++i) {
    if (events &&
        (e = cudaEventRecordWithFlags((cudaEvent_t)events[i], s, rec_flags)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = seq[i](p, a, s)) != cudaSuccess) return cuda_fail(e);
  }
  if (events && (e = cudaEventRecordWithFlags((cudaEvent_t)events[SALSC_DECODE_KERNELS], s,
                                              rec_flags)) != cudaSuccess)
    return cuda_fail(e);
  return SALSC_OK;
}

}  // namespace

salsc_status salsc::check_decode_step(const salsc_decode_desc* desc, const void* q,
                                      const void* Kc, const void* Vc, const void* Pk,
                                      const void* Pv, const void* out, const int32_t* idx_out) {
  salsc::DecodePlan p;
  const salsc_status st = make_plan(desc, &p);
  if (st != SALSC_OK) return st;
  return check_step_pointers(desc, q, Kc, Vc, Pk, Pv, out, idx_out);
}

salsc_status salsc::decode_step_clearing_flags(const salsc_decode_desc* desc, const void* q,
                                               const void* Kc, const void* Vc, const void* Pk,
                                               const void* Pv, void* out, int32_t* idx_out,
                                               void* ws, size_t ws_bytes, salsc_stream stream) {
  return decode_step_impl(desc, q, Kc, Vc, Pk, Pv, out, idx_out, ws, ws_bytes, stream, nullptr, 0,
                          nullptr, true);
}

extern "C" {

salsc_status salsc_decode_step(const salsc_decode_desc* desc, const void* q, const void* Kc,
                               const void* Vc, const void* Pk, const void* Pv, void* out,
                               int32_t* idx_out, void* ws, size_t ws_bytes, salsc_stream stream) {
  return decode_step_impl(desc, q, Kc, Vc, Pk, Pv, out, idx_out, ws, ws_bytes, stream, nullptr, 0);
}

salsc_status salsc_decode_step_append(const salsc_decode_desc* desc, const void* K_new,
                                      const void* V_new, const int64_t* rows_dev, const void* q,
                                      void* Kc, void* Vc, const void* Pk, const void* Pv,
                                      void* out, int32_t* idx_out, void* ws, size_t ws_bytes,
                                      salsc_stream stream) {
  const AppendArgs app{K_new, V_new, rows_dev};
  return decode_step_impl(desc, q, Kc, Vc, Pk, Pv, out, idx_out, ws, ws_bytes, stream, nullptr, 0,
                          &app);
}

salsc_status salsc_decode_step_traced(const salsc_decode_desc* desc, const void* q,
                                      const void* Kc, const void* Vc, const void* Pk,
                                      const void* Pv, void* out, int32_t* idx_out, void* ws,
                                      size_t ws_bytes, uint64_t* trace, size_t trace_bytes,
                                      salsc_stream stream) {
  if (!trace || ((uintptr_t)trace & 7u) ||
      trace_bytes < sizeof(uint64_t) * 3 * (size_t)SALSC_DECODE_KERNELS * SALSC_TRACE_MAX_CTAS)
    return SALSC_ERR_INVALID_ARG;
  return decode_step_impl(desc, q, Kc, Vc, Pk, Pv, out, idx_out, ws, ws_bytes, stream, nullptr, 0,
                          nullptr, false, trace);
}

salsc_status salsc_decode_step_timed(const salsc_decode_desc* desc, const void* q, const void* Kc,
                                     const void* Vc, const void* Pk, const void* Pv, void* out,
                                     int32_t* idx_out, void* ws, size_t ws_bytes,
                                     salsc_stream stream, void* const* events, int32_t n_events) {
  if (!events) return SALSC_ERR_INVALID_ARG;
  return decode_step_impl(desc, q, Kc, Vc, Pk, Pv, out, idx_out, ws, ws_bytes, stream, events,
                          n_events);
}

salsc_status salsc_compress(const void* K, const void* V, const void* Pk, const void* Pv, void* Kc,
                            void* Vc, int64_t n_tokens, int32_t hidden, int32_t rank,
                            salsc_dtype dtype, salsc_stream stream) {
  if (dtype != SALSC_F32 && dtype != SALSC_BF16) return SALSC_ERR_INVALID_ARG;
  if (n_tokens < 0 || hidden < 1 || rank < 1) return SALSC_ERR_INVALID_ARG;
  const int q = dtype == SALSC_BF16 ? 16 : 4;
  if (hidden % q != 0 || rank % q != 0) return SALSC_ERR_INVALID_ARG;
  if (!K && !V) return SALSC_ERR_INVALID_ARG;
  if (K && (!Pk || !Kc || !aligned16(K) || !aligned16(Pk) || !aligned16(Kc)))
    return SALSC_ERR_INVALID_ARG;
  if (V && (!Pv || !Vc || !aligned16(V) || !aligned16(Pv) || !aligned16(Vc)))
    return SALSC_ERR_INVALID_ARG;
  if (n_tokens == 0) return SALSC_OK;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  if (salsc::compress_tc_supported(hidden, rank, dtype)) {
    // both halves in one tensor-core launch
    const void* X[2] = {K ? K : V, V};
    const void* Pm[2] = {K ? Pk : Pv, Pv};
    void* Y[2] = {K ? Kc : Vc, Vc};
    e = salsc::launch_compress_tc(X, Pm, Y, (K && V) ? 2 : 1, n_tokens, hidden, rank, s);
    return e == cudaSuccess ? SALSC_OK : cuda_fail(e);
  }
  if (K && (e = salsc::launch_compress(K, Pk, Kc, n_tokens, hidden, rank, dtype, s)) != cudaSuccess)
    return cuda_fail(e);
  if (V && (e = salsc::launch_compress(V, Pv, Vc, n_tokens, hidden, rank, dtype, s)) != cudaSuccess)
    return cuda_fail(e);
  return SALSC_OK;
}

salsc_status salsc_shard_candidates(const salsc_decode_desc* desc, const void* q, const void* Kc,
                                    const void* Pk, const int64_t* shard_off_dev,
                                    float* cand_score, int32_t* cand_idx, void* ws,
                                    size_t ws_bytes, salsc_stream stream) {
  salsc::DecodePlan p;
  salsc_status st = make_plan(desc, &p);
  if (st != SALSC_OK) return st;
  if (!desc->seq_offsets_dev || !q || !Kc || !Pk || !shard_off_dev || !cand_score || !cand_idx)
    return SALSC_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(Kc) || !aligned16(Pk) || ((uintptr_t)cand_score & 3u) ||
      ((uintptr_t)cand_idx & 3u) || ((uintptr_t)shard_off_dev & 7u))
    return SALSC_ERR_INVALID_ARG;
  if ((st = check_ws(p, ws, ws_bytes)) != SALSC_OK) return st;
  const salsc::DecodeArgs a = make_args(p, desc, q, Kc, nullptr, Pk, nullptr, nullptr, nullptr, ws);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  if ((e = salsc::launch_latent_q(p, a, s)) != cudaSuccess ||
      (e = salsc::launch_score(p, a, s)) != cudaSuccess ||
      (e = salsc::launch_topk(p, a, s)) != cudaSuccess ||
      (e = salsc::launch_shard_gather(p, a, shard_off_dev, cand_score, cand_idx, s)) !=
          cudaSuccess)
    return cuda_fail(e);
  return SALSC_OK;
}

salsc_status salsc_shard_select(const float* cand_score_all, const int32_t* cand_idx_all,
                                int32_t n_shards, int32_t batch, int32_t n_units, int32_t top_k,
                                const int64_t* local_offsets_dev, const int64_t* shard_off_dev,
                                int32_t* idx_local, salsc_stream stream) {
  if (!cand_score_all || !cand_idx_all || !local_offsets_dev || !shard_off_dev || !idx_local)
    return SALSC_ERR_INVALID_ARG;
  if (n_shards < 1 || batch < 1 || n_units < 1 || top_k < 1) return SALSC_ERR_INVALID_ARG;
  if (n_units > salsc::kMaxUnits || (int64_t)n_shards * top_k > salsc::kMaxShardCandidates)
    return SALSC_ERR_UNSUPPORTED;
  const cudaError_t e =
      salsc::launch_shard_select(cand_score_all, cand_idx_all, n_shards, batch, n_units, top_k,
                                 local_offsets_dev, shard_off_dev, idx_local, (cudaStream_t)stream);
  return e == cudaSuccess ? SALSC_OK : cuda_fail(e);
}

salsc_status salsc_shard_attend(const salsc_decode_desc* desc, const void* q, const void* Kc,
                                const void* Vc, const void* Pk, const int32_t* idx_local,
                                const int64_t* shard_off_dev, float* part_out, void* ws,
                                size_t ws_bytes, salsc_stream stream) {
  salsc::DecodePlan p;
  salsc_status st = make_plan(desc, &p);
  if (st != SALSC_OK) return st;
  // the shards' partials are merged after the exchange, so the attention
  // kernel does not merge (nor project) them itself
  p.att_cluster = 0;
  if (!desc->seq_offsets_dev || !desc->q_pos_dev || !q || !Kc || !Vc || !Pk || !idx_local ||
      !shard_off_dev || !part_out)
    return SALSC_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(Pk) ||
      ((uintptr_t)idx_local & 3u) || ((uintptr_t)part_out & 15u) || ((uintptr_t)shard_off_dev & 7u))
    return SALSC_ERR_INVALID_ARG;
  if ((st = check_ws(p, ws, ws_bytes)) != SALSC_OK) return st;
  salsc::DecodeArgs a =
      make_args(p, desc, q, Kc, Vc, Pk, nullptr, nullptr, const_cast<int32_t*>(idx_local), ws);
  a.pos_off = shard_off_dev;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  if ((e = salsc::launch_attend(p, a, s)) != cudaSuccess ||
      (e = salsc::launch_combine_partial(p, a, part_out, s)) != cudaSuccess)
    return cuda_fail(e);
  return SALSC_OK;
}

salsc_status salsc_shard_merge(const float* part_all, int32_t n_shards, int32_t batch,
                               int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                               int32_t rank, salsc_dtype dtype, const void* Pv, void* out,
                               void* ws, size_t ws_bytes, salsc_stream stream) {
  if (dtype != SALSC_F32 && dtype != SALSC_BF16) return SALSC_ERR_INVALID_ARG;
  if (!part_all || !Pv || !out || n_shards < 1 || batch < 1 || n_kv_heads < 1 || rank < 1 ||
      n_q_heads < n_kv_heads || n_q_heads % n_kv_heads != 0)
    return SALSC_ERR_INVALID_ARG;
  if (((uintptr_t)part_all & 15u) || !aligned16(Pv) || !aligned16(out)) return SALSC_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws % salsc::kWsAlign) != 0 || ws_bytes < 16) return SALSC_ERR_WORKSPACE;
  salsc::DecodePlan p{};
  p.B = batch;
  p.Hq = n_q_heads;
  p.U = n_kv_heads;
  p.G = n_q_heads / n_kv_heads;
  p.d = head_dim;
  p.r = rank;
  p.dtype = dtype;
  p.splits = n_shards;
  if ((head_dim != 64 && head_dim != 128) || rank > salsc::kMaxRank || p.G > 8 ||
      n_kv_heads > salsc::kMaxUnits || rank > n_kv_heads * head_dim ||
      !salsc::combine_supported(p))
    return SALSC_ERR_UNSUPPORTED;
  const cudaError_t e = salsc::launch_shard_merge(p, part_all, n_shards, Pv, out, (uint32_t*)ws,
                                                  (cudaStream_t)stream);
  return e == cudaSuccess ? SALSC_OK : cuda_fail(e);
}

}  // extern "C"
