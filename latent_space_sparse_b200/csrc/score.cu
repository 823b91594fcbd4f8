// score.cu -- RoPE-free latent scoring of every cached token.
//
// SALS technical framework, stage 2: s_u[t] = q_lat[b,u] . Kc_b[t] for every
// unit u and every cached token t < n_b.  Kc is read exactly once per step
// for all units of a sequence.
//
// Scores are written fp32, packed per (b,u): unit (b,u)'s n_b scores start at
// seq_off[b]*U + u*n_b.
#include "tc.cuh"

namespace salsc {
namespace {

constexpr int kThreads = 256;

// CUDA-core path: one warp per token row; each lane holds its slice of the
// row in registers and reduces U dot products across the warp.
template <typename T>
__global__ void __launch_bounds__(kThreads)
score_simt_kernel(const T* __restrict__ Kc, const float* __restrict__ qlat,
                  const int64_t* __restrict__ seq_off, float* __restrict__ scores,
                  uint32_t* __restrict__ krange, int B, int U, int r, int tile_len) {
  extern __shared__ float sq[];  // [U][r]
  __shared__ uint32_t s_kr[kMaxUnits][2];  // this CTA's (min, max) score key per unit
  int b;
  int64_t t0;
  find_tile(seq_off, B, tile_len, blockIdx.x, b, t0);
  if (b < 0) return;
  const int64_t off = seq_off[b];
  const int64_t nb = seq_off[b + 1] - off;
  allow_dependent_launch();
  grid_dependency_wait();  // q_lat comes from the previous kernel
  for (int e = threadIdx.x; e < U * r; e += kThreads) sq[e] = qlat[(size_t)b * U * r + e];
  for (int e = threadIdx.x; e < U; e += kThreads) {
    s_kr[e][0] = 0xffffffffu;
    s_kr[e][1] = 0u;
  }
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
      if (lane == 0) {
        scores[off * U + (int64_t)u * nb + t] = acc;
        atomicMin(&s_kr[u][0], order_key(acc));
        atomicMax(&s_kr[u][1], order_key(acc));
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < U; e += kThreads) {
    atomicMin(&krange[2 * ((int64_t)b * U + e)], s_kr[e][0]);
    atomicMax(&krange[2 * ((int64_t)b * U + e) + 1], s_kr[e][1]);
  }
}


// ---------------------------------------------------------------------------
// Tensor-core path (bf16 storage, r % 64 == 0, 2U <= 256).
//
// Per 128-token tile of one sequence: D[128 x npad] = Kc_tile[128 x r] .
// Qs[npad x r]^T on tcgen05, where Qs holds the hi and lo bf16 parts of each
// unit's fp32 latent query (rows 2u, 2u+1) so that hi + lo carries the query
// to ~16 bits and the score error stays far below the top-k tie band.  Kc is
// exact in bf16; the tensor core multiplies exactly and accumulates in fp32.
//
// Warp roles (192 threads): warp 0 lane 0 = TMA producer of 16 KiB Kc
// k-blocks [128 rows x 64] into a `stages`-deep ring (plus the sequence's Qs
// when the sequence changes); warp 1 = TMEM owner and (lane 0) MMA issuer,
// accumulating into one of two TMEM buffers; warps 2-5 = epilogue: TMEM ->
// registers, s_u = D[:, 2u] + D[:, 2u+1], coalesced fp32 stores.
// Each CTA owns a contiguous range of 32-row chunks (persistent, grid <= #SMs),
// taken as pieces of up to four chunks (one 128-row MMA tile) inside one
// sequence, so the CTAs' shares differ by at most one chunk and Qs is
// reloaded only at sequence boundaries.
constexpr int kTcThreads = 192;
constexpr int kRangeSeqs = 4;  // sequences per CTA whose score ranges are kept in shared memory
constexpr int kTileM = 128;
constexpr int kChunk = 32;                          // rows of a work item (one TMA box)
constexpr int kChunksPerTile = kTileM / kChunk;
constexpr uint32_t kStageBytes = kTileM * 64 * 2;  // one [128 x 64] bf16 k-block
constexpr uint32_t kChunkBytes = kChunk * 64 * 2;  // one [32 x 64] box of it

struct ScoreTcParams {
  const int64_t* seq_off;
  float* scores;
  uint32_t* krange;
  uint32_t* flags;
  int B, U, npad, r, n_chunks, stages, tmem_cols;
  int ng, ncol;  // unit groups, and the 2 * units-per-group query rows of one group
  uint64_t* trace;  // traced step: this kernel's rows, or null
};

// Item w's group, sequence and chunk, found by one warp: every lane reads the
// offsets of one sequence (32 at a time) and a warp scan of the chunks per
// sequence locates the item with one round trip of loads.  Lane 0 writes
// (g, b, q) to st[0..2] and (off, n_b) of sequence b to st64[0..1].
__device__ __forceinline__ void find_first_chunk(const int64_t* so, int B, int nq_all, int w,
                                                 int* st, int64_t* st64) {
  const int lane = threadIdx.x % 32;
  const int g = w / nq_all, c = w % nq_all;
  int64_t before = 0;
  bool found = false;
  for (int b0 = 0; b0 < B && !found; b0 += 32) {
    const int bb = b0 + lane;
    int64_t offb = 0, nbb = 0;
    if (bb < B) {
      offb = so[bb];
      nbb = so[bb + 1] - offb;
    }
    const int64_t x = (nbb + kChunk - 1) / kChunk;
    int64_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const int64_t excl = before + incl - x;
    const uint32_t m = __ballot_sync(0xffffffffu, bb < B && excl <= c && c < excl + x);
    if (m) {
      const int src = __ffs(m) - 1;
      if (lane == src) {
        st[0] = g;
        st[1] = bb;
        st[2] = (int)(c - excl);
        st64[0] = offb;
        st64[1] = nbb;
      }
      found = true;
    }
    before += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// Walks the work items of a CTA as pieces.  Item w is chunk w % nq_all of
// unit group w / nq_all (groups outermost, so the CTAs that read the same rows
// for different groups run at about the same time and share them through
// L2); sequence b has nq = ceil(n_b / 32) chunks.  A piece is up to four
// consecutive chunks of one sequence and group within the CTA's range.
struct PieceCursor {
  const int64_t* so;
  int B;
  int g, b, q, nq, len, left;  // group, sequence, first chunk, chunks of b, of the piece, left in the range
  int64_t off, nb;
  __device__ void load() {
    off = so[b];
    nb = so[b + 1] - off;
    nq = (int)((nb + kChunk - 1) / kChunk);
  }
  __device__ void fit() { len = min(min(kChunksPerTile, nq - q), left); }
  // first piece: chunk q of sequence b in group g (from find_first_chunk)
  __device__ void at(const int64_t* so_, int B_, int n, int g_, int b_, int q_, int64_t off_,
                     int64_t nb_) {
    so = so_;
    B = B_;
    left = n;
    len = 0;
    g = g_;
    b = b_;
    q = q_;
    off = off_;
    nb = nb_;
    nq = (int)((nb + kChunk - 1) / kChunk);
    if (left > 0) fit();
  }
  __device__ void next() {
    left -= len;
    q += len;
    if (left <= 0) return;
    while (q >= nq) {  // the range goes on in the next sequence (or group)
      q = 0;
      if (++b == B) {
        b = 0;
        ++g;
      }
      load();
    }
    fit();
  }
  __device__ bool done() const { return left <= 0; }
  __device__ int64_t row0() const { return off + (int64_t)q * kChunk; }
};

__global__ void __launch_bounds__(kTcThreads)
score_tc_kernel(const __grid_constant__ CUtensorMap tmap_kc,
                const __grid_constant__ CUtensorMap tmap_q, const ScoreTcParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int KB = P.r / 64;
  const int S = P.stages;
  const uint32_t b_kblock_bytes = (uint32_t)P.ncol * 128u;
  const int n_items = P.n_chunks * P.ng;
  uint8_t* a_ring = smem;
  uint8_t* b_buf = a_ring + (size_t)S * kStageBytes;
  uint64_t* bars = (uint64_t*)(b_buf + (size_t)KB * b_kblock_bytes);
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * S + 6);
  const uint32_t bar0 = tc::smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t bfull = bar0 + 8u * (2 * S), bempty = bar0 + 8u * (2 * S + 1);
  auto tfull = [&](int a) { return bar0 + 8u * (2 * S + 2 + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (2 * S + 4 + a); };

  // (min, max) score key per unit of the first kRangeSeqs sequences of this
  // CTA's tile range
  __shared__ uint32_t s_kr[kRangeSeqs][kMaxUnits][2];
  __shared__ int s_krb[kRangeSeqs], s_nkr;
  __shared__ int s_first[3];        // the CTA's first item: group, sequence, chunk
  __shared__ int64_t s_first64[2];  // and that sequence's (offset, length)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) trace_stamp(P.trace, TRACE_START);
  for (int e = threadIdx.x; e < kRangeSeqs * P.U; e += kTcThreads) {
    s_kr[e / P.U][e % P.U][0] = 0xffffffffu;
    s_kr[e / P.U][e % P.U][1] = 0u;
  }
  if (threadIdx.x == 0) s_nkr = 0;
  const int t_begin = (int)((int64_t)blockIdx.x * n_items / gridDim.x);
  const int t_end = (int)((int64_t)(blockIdx.x + 1) * n_items / gridDim.x);
  allow_dependent_launch();
  if (warp == 2 && t_end > t_begin)
    find_first_chunk(P.seq_off, P.B, P.n_chunks, t_begin, s_first, s_first64);
  auto first_piece = [&](PieceCursor& c) {
    c.at(P.seq_off, P.B, t_end - t_begin, s_first[0], s_first[1], s_first[2], s_first64[0],
         s_first64[1]);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), 1);
    }
    tc::mbar_init(bfull, 1);
    tc::mbar_init(bempty, 1);
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tfull(a), 1);
      tc::mbar_init(tempty(a), 128);
    }
    tc::mbar_fence_init();
    tc::tma_prefetch_desc(&tmap_kc);
    tc::tma_prefetch_desc(&tmap_q);
  }
  if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), (uint32_t)P.tmem_cols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    uint32_t it = 0, bpar = 0;
    int cur_bg = -1;
    bool ok = true;
    PieceCursor pc;
    first_piece(pc);
    // k-block kb of the piece: its chunks, one 32-row box each, into stage s
    auto load_kblock = [&](int s, int kb) {
      tc::mbar_expect_tx(full(s), (uint32_t)pc.len * kChunkBytes);
      for (int j = 0; j < pc.len; ++j)
        tc::tma_load_2d(tc::smem_u32(a_ring + (size_t)s * kStageBytes + (size_t)j * kChunkBytes),
                        &tmap_kc, kb * 64, (int)(pc.row0() + (int64_t)j * kChunk), full(s));
    };
    for (int i = 0; !pc.done() && ok; ++i, pc.next()) {
      const int b = pc.b;
      const int bg = b * P.ng + pc.g;
      if (bg != cur_bg) {
        if (cur_bg >= 0) {
          ok = tc::mbar_wait(bempty, bpar, P.flags);
          bpar ^= 1u;
          if (!ok) break;
        } else {
          // the latent cache streams in already; the split query comes from the
          // previous kernel
          if (i == 0)
            for (int kb = 0; kb < KB && kb < S; ++kb) load_kblock(kb, kb);
          grid_dependency_wait();
          trace_stamp(P.trace, TRACE_WAITED);
        }
        tc::mbar_expect_tx(bfull, (uint32_t)KB * b_kblock_bytes);
        for (int kb = 0; kb < KB; ++kb)
          tc::tma_load_2d(tc::smem_u32(b_buf + (size_t)kb * b_kblock_bytes), &tmap_q, kb * 64,
                          b * P.npad + pc.g * P.ncol, bfull);
        cur_bg = bg;
      }
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = (int)(it % (uint32_t)S);
        const uint32_t ph = (it / (uint32_t)S) & 1u;
        if (i == 0 && kb < S) continue;  // issued before the dependency wait
        if (!tc::mbar_wait(empty(s), ph ^ 1u, P.flags)) {
          ok = false;
          break;
        }
        load_kblock(s, kb);
      }
    }
    // every issued load has landed before the CTA may exit
    for (uint32_t j = it > (uint32_t)S ? it - (uint32_t)S : 0u; j < it; ++j)
      tc::mbar_wait(full((int)(j % (uint32_t)S)), (j / (uint32_t)S) & 1u, P.flags);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    const uint32_t idesc = tc::idesc_bf16_f32(kTileM, P.ncol);
    uint32_t it = 0, bpar = 0;
    int cur_bg = -1, nseq = 0, i = 0;
    bool ok = true;
    PieceCursor pc;
    first_piece(pc);
    for (; !pc.done() && ok; ++i) {
      const int bg = pc.b * P.ng + pc.g;
      if (bg != cur_bg) {
        if (!tc::mbar_wait(bfull, bpar, P.flags)) break;
        bpar ^= 1u;
        cur_bg = bg;
        ++nseq;
      }
      const int acc = i & 1;
      if (!tc::mbar_wait(tempty(acc), (((uint32_t)i >> 1) & 1u) ^ 1u, P.flags)) break;
      tc::fence_after_sync();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * P.ncol);
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = (int)(it % (uint32_t)S);
        const uint32_t ph = (it / (uint32_t)S) & 1u;
        if (!tc::mbar_wait(full(s), ph, P.flags)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t a_addr = tc::smem_u32(a_ring + (size_t)s * kStageBytes);
        const uint32_t b_addr = tc::smem_u32(b_buf + (size_t)kb * b_kblock_bytes);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_bf16(d_tmem, tc::sdesc_kmajor_sw128(a_addr + 32u * k),
                       tc::sdesc_kmajor_sw128(b_addr + 32u * k), idesc, (kb | k) != 0);
        tc::mma_commit(empty(s));
      }
      if (!ok) break;
      tc::mma_commit(tfull(acc));
      // last piece of this (sequence, group) in the CTA's range: its Qs is then free
      const int pb = pc.b, pg = pc.g;
      pc.next();
      if (pc.done() || pc.b != pb || pc.g != pg) tc::mma_commit(bempty);
    }
    // the last release of Qs lands before the CTA may exit
    if (ok && nseq > 0) tc::mbar_wait(bempty, (uint32_t)(nseq - 1) & 1u, P.flags);
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> scores, and each unit's score range
    //      (min and max order key, reduced per warp, kept per CTA and
    //      sequence in shared memory, added to the workspace at the end)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    int i = 0, eb = -1, so = -1;  // sequence and its ordinal in this CTA's range
    PieceCursor pc;
    first_piece(pc);
    for (; !pc.done(); ++i, pc.next()) {
      if (pc.b != eb) {
        eb = pc.b;
        ++so;
        if (so < kRangeSeqs && threadIdx.x == 64) {
          s_krb[so] = eb;
          s_nkr = so + 1;
        }
      }
      const int acc = i & 1;
      // warp-uniform wait: the TMEM loads below need a converged warp
      const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(tfull(acc), ((uint32_t)i >> 1) & 1u,
                                                            P.flags));
      if (!ok) break;
      tc::fence_after_sync();
      const int64_t off = pc.off;
      const int64_t nb = pc.nb;
      const int64_t t = (int64_t)pc.q * kChunk + row;
      // rows past the piece hold stale ring data: neither stored nor ranged
      const bool live = row < pc.len * kChunk && t < nb;
      float* sbase = P.scores + off * P.U + t;
      const int u0 = pc.g * (P.ncol / 2);  // first unit of the group
      for (int c0 = 0; c0 < P.ncol; c0 += 16) {
        uint32_t v[16];
        tc::tmem_ld16(lane_addr + (uint32_t)(acc * P.ncol + c0), v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int u = u0 + c0 / 2 + j;
          const float sv = __uint_as_float(v[2 * j]) + __uint_as_float(v[2 * j + 1]);
          const uint32_t key = order_key(sv);
          const uint32_t kmn = __reduce_min_sync(0xffffffffu, live ? key : 0xffffffffu);
          const uint32_t kmx = __reduce_max_sync(0xffffffffu, live ? key : 0u);
          if (u < P.U) {
            if (live) sbase[(int64_t)u * nb] = sv;
            if (lane == 0) {
              if (so < kRangeSeqs) {
                atomicMin(&s_kr[so][u][0], kmn);
                atomicMax(&s_kr[so][u][1], kmx);
              } else {  // more sequences than table rows: straight to the workspace
                atomicMin(&P.krange[2 * ((int64_t)eb * P.U + u)], kmn);
                atomicMax(&P.krange[2 * ((int64_t)eb * P.U + u) + 1], kmx);
              }
            }
          }
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(tempty(acc));
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) trace_stamp(P.trace, TRACE_END);
  for (int e = threadIdx.x; e < s_nkr * P.U; e += kTcThreads) {
    const int q = e / P.U, u = e % P.U;
    atomicMin(&P.krange[2 * ((int64_t)s_krb[q] * P.U + u)], s_kr[q][u][0]);
    atomicMax(&P.krange[2 * ((int64_t)s_krb[q] * P.U + u) + 1], s_kr[q][u][1]);
  }
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, (uint32_t)P.tmem_cols);
  }
}

int num_sms() {
  static int cached[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (!cached[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

cudaError_t launch_score_tc(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  const int KB = p.r / 64;
  // Unit groups: the units' query rows are split into ng groups of ncol rows
  // (ncol a multiple of 16) when there are too few tiles to give every SM two
  // work items, or when one group's query block is too large for two CTAs per
  // SM.  Each group re-reads the latent rows of its tiles (from L2 after the
  // first group).
  int ng = 1;
  auto qbytes = [&](int g) { return (size_t)KB * (2 * p.U / g) * 128; };
  while ((2 * p.U) % (16 * ng * 2) == 0 &&
         ((int64_t)p.n_score_tiles * ng < 2 * num_sms() || qbytes(ng) > 45 * 1024))
    ng *= 2;
  const int ncol = (2 * p.U) % 16 == 0 ? 2 * p.U / ng : p.npad;
  const size_t b_bytes = (size_t)KB * ncol * 128;
  // Small query blocks: two CTAs per SM with a 4-deep ring each; large ones one
  // CTA per SM with a deeper ring.
  int stages, ctas_per_sm;
  if (b_bytes <= 45 * 1024) {
    stages = 4;
    ctas_per_sm = 2;
  } else {
    stages = (int)((200u * 1024u - b_bytes) / kStageBytes);
    if (stages > 8) stages = 8;
    ctas_per_sm = 1;
  }
  if (stages < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = 1024 + (size_t)stages * kStageBytes + b_bytes + (2 * stages + 6) * 8 + 16;
  CUtensorMap tk, tq;
  if (!make_tmap_bf16_2d(&tk, a.Kc, (uint64_t)p.N, (uint64_t)p.r, kChunk, 64) ||
      !make_tmap_bf16_2d(&tq, a.qsplit, (uint64_t)p.B * p.npad, (uint64_t)p.r, ncol, 64))
    return cudaErrorInvalidValue;
  static int done[kMaxDevices] = {};
  cudaError_t e = ensure_smem(score_tc_kernel, smem, done);
  if (e != cudaSuccess) return e;
  ScoreTcParams P;
  P.seq_off = a.seq_off;
  P.scores = a.scores;
  P.krange = a.krange;
  P.flags = a.flags;
  P.trace = trace_of(a, 1);
  P.B = p.B;
  P.U = p.U;
  P.npad = p.npad;
  P.r = p.r;
  P.n_chunks = p.n_score_chunks;
  P.stages = stages;
  P.ng = ng;
  P.ncol = ncol;
  int cols = 32;
  while (cols < 2 * ncol) cols *= 2;
  P.tmem_cols = cols;
  // at most one CTA per 128 rows of work
  const int max_ctas = num_sms() * ctas_per_sm;
  const int64_t pieces = ((int64_t)p.n_score_chunks * ng + kChunksPerTile - 1) / kChunksPerTile;
  const int grid = pieces < max_ctas ? (int)pieces : max_ctas;
  return launch_k(score_tc_kernel, dim3(grid), dim3(kTcThreads), smem, s, true, tk, tq, P);
}

}  // namespace

cudaError_t launch_score(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  if (p.dtype == SALSC_BF16 && p.r % 64 == 0 && p.npad <= 256) return launch_score_tc(p, a, s);
  const size_t smem = sizeof(float) * (size_t)p.U * p.r;
  if (p.dtype == SALSC_BF16) {
    static int done[kMaxDevices] = {};
    auto k = score_simt_kernel<__nv_bfloat16>;
    cudaError_t e = ensure_smem(k, smem, done);
    if (e != cudaSuccess) return e;
    e = launch_k(k, dim3(p.n_score_tiles), dim3(kThreads), smem, s, true,
                 (const __nv_bfloat16*)a.Kc, (const float*)a.qlat, (const int64_t*)a.seq_off,
                 a.scores, a.krange, p.B, p.U, p.r, p.score_tile);
    if (e != cudaSuccess) return e;
  } else {
    static int done[kMaxDevices] = {};
    auto k = score_simt_kernel<float>;
    cudaError_t e = ensure_smem(k, smem, done);
    if (e != cudaSuccess) return e;
    e = launch_k(k, dim3(p.n_score_tiles), dim3(kThreads), smem, s, true, (const float*)a.Kc,
                 (const float*)a.qlat, (const int64_t*)a.seq_off, a.scores, a.krange, p.B, p.U,
                 p.r, p.score_tile);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace salsc
