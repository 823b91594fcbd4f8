// attend_tc.cu -- selective reconstruction, RoPE, softmax and the latent
// value sum over the kept tokens, on tcgen05 (bf16 storage, d in {64, 128},
// r <= 256, or r <= 512 in two latent halves, G in {1, 2, 4, 8}).
//
// SALS technical framework, stages 3-4, with RoPE applied after
// reconstruction (abstract).  Work unit: a tile of 128 kept tokens of one
// selection unit (b, u):
//   1. the gather warps copy the 128 latent key rows Kc_b[idx] into shared
//      memory by TMA gather4 (four rows of 64 latent columns per copy, into
//      the 128-byte swizzled K-major layout);
//   2. tcgen05: K_sel[128 x d] = Kc_tile . Pk_u^T into TMEM (fp32; Pk_u comes
//      by TMA once per unit and stays in shared memory);
//   3. the same rows of Vc are copied into the buffer the MMA has finished
//      with;
//   4. sixteen epilogue warps (one thread per token row and a quarter of the
//      RoPE pairs) read K_sel from TMEM, rotate pair (i, i+d/2) by the angle
//      t * base^(-2i/d) and dot it with every rotated query head of the unit;
//      the tile's softmax (max m, normaliser l) follows, one thread per
//      (head, token), and the weights p are written to shared memory as bf16
//      hi + lo parts;
//   5. tcgen05: acc^T[r x 2G] = Vc_tile^T . [p_hi p_lo] into TMEM (Vc_tile read
//      as an MN-major operand, so the latent value rows need no transpose);
//   6. the epilogue reads acc[c] = D[c][2g] + D[c][2g+1] and writes the
//      tile's (m, l, acc) per head;
//   7. consecutive tiles of one unit in a CTA are folded into a running
//      (m, l, acc) per head (online softmax rescaling); each CTA publishes one
//      partial per unit segment, at the slot of the segment's first tile.  A
//      segment starts at a unit's first tile and at every CTA's first tile,
//      so the combine kernel finds the used slots from the tile partition
//      alone; it merges the few segments of a unit and applies the deferred
//      Pv_u^T.
// Warp roles: warps 0-15 epilogue, warp 16 TMEM owner and MMA issuer, then
// the gather warps: r <= 256, a team of seven (768 threads, 24 warps, 80
// registers a thread) that issues every tile's copies together (a warp's
// lanes issue their TMA copies one after another, so a tile's issue time
// falls with the warps sharing it); r > 256, two groups of four, one per
// latent half (800 threads, 72 registers: 25 warps put seven on one
// scheduler, whose register file is a quarter of the SM's).  The epilogue is
// the busiest role (RoPE needs a sine and a cosine per pair and token), so it
// has four warps per scheduler.  Each CTA walks a contiguous range of tiles;
// the two tile buffers alternate (Kc(i) -> Vc(i) -> Kc(i+2)), so the
// reconstruction of tile i+1 runs during the epilogue of tile i.
//
// The RoPE angle uses an exact fixed-point phase: F_i = round(2^64 *
// theta_i / 2 pi), and the top 32 bits of t * F_i (mod 2^64) are t * theta_i
// modulo one turn, to 2^-32 of a turn, for any 32-bit position t.
#include "tc.cuh"

namespace salsc {
namespace {

constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kEpiParts = kEpiWarps / 4;  // threads per token row
constexpr int kMmaWarp = 16;
constexpr int kLoadWarp0 = 17;  // the gather warps follow the MMA warp
constexpr int kGatherWarps = 4;  // per latent half (W = 2)
constexpr int kGatherThreads = kGatherWarps * 32;
// Gather warps: one team of seven (W = 1), or four per latent half (W = 2).
// Seven keep the block at 24 warps, six per scheduler, which leaves 80
// registers a thread (25 warps put seven on one scheduler: 72 registers).
template <int W> constexpr int gather_warps() { return W == 1 ? 7 : 2 * kGatherWarps; }
template <int W> constexpr int block_threads() { return (kLoadWarp0 + gather_warps<W>()) * 32; }
constexpr int kTile = 128;
constexpr int kPRows = 16;  // rows of the p operand (2G <= 16)
constexpr uint32_t kEpiBar = 1;
constexpr double kTwoPi = 6.283185307179586476925286766559;

struct AttendTcParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* Kc;
  const __nv_bfloat16* Vc;
  const int32_t* idx;
  const int64_t* seq_off;
  const int32_t* q_pos;
  const int64_t* pos_off;  // [B] or null: added to a kept token's index for RoPE
  float* part;
  uint32_t* flags;
  const __nv_bfloat16* Pv;  // merged in the kernel: the value projection
  __nv_bfloat16* out;
  int B, Hq, U, r, k, n_slots, n_tiles;
  int64_t uni_nb;  // every sequence's length when they are equal, else 0
  int cluster;  // merged in the kernel: CTAs per unit (one thread-block cluster)
  uint64_t* trace;  // traced step: this kernel's rows, or null
  float scale;
  double base;
};

// Walks the tiles of a CTA.  Tiles are numbered in the order (sequence,
// unit, slot); unit (b, u) has tb = ceil(min(k, n_b) / 128) tiles.  A CTA's
// first tile is found once per CTA (find_first_tile) and set with at().
struct UnitTileCursor {
  const int64_t* so;
  int B, U, k;
  int b, u, slot, tb;
  int64_t off, nb, kb;
  __device__ void load() {
    off = so[b];
    nb = so[b + 1] - off;
    kb = nb < k ? nb : k;
    tb = (int)((kb + kTile - 1) / kTile);
  }
  __device__ void at(const int64_t* so_, int B_, int U_, int k_, int b_, int u_, int slot_,
                     int64_t off_, int64_t nb_) {
    so = so_;
    B = B_;
    U = U_;
    k = k_;
    b = b_;
    u = u_;
    slot = slot_;
    off = off_;
    nb = nb_;
    kb = nb < k ? nb : k;
    tb = (int)((kb + kTile - 1) / kTile);
  }
  __device__ void next() {
    if (++slot >= tb) {
      slot = 0;
      if (++u >= U) {
        u = 0;
        if (++b < B) load();
      }
    }
  }
};

// The CTA's tile range and its first tile, found by one warp: every lane reads
// the offsets of one sequence (32 at a time), and a warp scan of the tiles
// per sequence locates tile t_begin with one round trip of loads.  Merging
// CTAs (cluster > 0) take their rank's share of unit m_unit's tiles; the
// others take tiles [share_begin(c), share_begin(c + 1)).  Lane 0 writes (t_begin, n, b, u,
// slot) to st[0..4] and (off, nb) of sequence b to st64[0..1]; b = B when the
// range is empty.
__device__ __forceinline__ void find_first_tile(const int64_t* so, int B, int U, int k,
                                                int n_tiles, int cluster, int64_t uni_nb,
                                                int* st, int64_t* st64) {
  const int lane = threadIdx.x % 32;
  if (uni_nb > 0) {
    // every sequence has uni_nb tokens: the first tile is arithmetic, no loads
    const int tu = (int)(((uni_nb < k ? uni_nb : (int64_t)k) + kTile - 1) / kTile);
    int t_begin, n, fb, fu = 0, fslot = 0;
    if (cluster > 0) {
      const int m_unit = (int)(blockIdx.x / (unsigned)cluster);
      const int m_rank = (int)(blockIdx.x % (unsigned)cluster);
      const int l0 = tu * m_rank / cluster, h0 = tu * (m_rank + 1) / cluster;
      t_begin = m_unit * tu + l0;
      n = h0 - l0;
    } else {
      t_begin = (int)share_begin(blockIdx.x, n_tiles, gridDim.x);
      n = (int)share_begin(blockIdx.x + 1, n_tiles, gridDim.x) - t_begin;
    }
    fb = n > 0 && tu > 0 ? t_begin / (U * tu) : B;
    if (fb < B) {
      const int rem = t_begin - fb * U * tu;
      fu = rem / tu;
      fslot = rem % tu;
    }
    if (lane == 0) {
      st[0] = t_begin;
      st[1] = n;
      st[2] = fb;
      st[3] = fu;
      st[4] = fslot;
      st64[0] = (int64_t)fb * uni_nb;
      st64[1] = uni_nb;
    }
    return;
  }
  int t_begin = 0, n = 0, mb = -1;
  if (cluster > 0) {
    mb = (int)(blockIdx.x / (unsigned)cluster) / U;  // the unit's sequence
  } else {
    t_begin = (int)share_begin(blockIdx.x, n_tiles, gridDim.x);
    n = (int)share_begin(blockIdx.x + 1, n_tiles, gridDim.x) - t_begin;
  }
  int64_t before = 0;  // tiles of the sequences before this group of 32
  int fb = B, fu = 0, fslot = 0;
  int64_t foff = 0, fnb = 0;
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int bb = b0 + lane;
    int64_t offb = 0, nbb = 0;
    int tbb = 0;
    if (bb < B) {
      offb = so[bb];
      nbb = so[bb + 1] - offb;
      const int64_t kbb = nbb < k ? nbb : k;
      tbb = (int)((kbb + kTile - 1) / kTile);
    }
    const int64_t x = (int64_t)U * tbb;
    int64_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const int64_t excl = before + incl - x;
    if (cluster > 0) {
      // unit m_unit = (mb, u): the rank's share [lo, hi) of its tb tiles
      const uint32_t m = __ballot_sync(0xffffffffu, bb == mb);
      if (m) {
        const int src = __ffs(m) - 1;
        const int64_t e = __shfl_sync(0xffffffffu, excl, src);
        const int tu = __shfl_sync(0xffffffffu, tbb, src);
        const int64_t o2 = __shfl_sync(0xffffffffu, offb, src);
        const int64_t n2 = __shfl_sync(0xffffffffu, nbb, src);
        const int m_rank = (int)(blockIdx.x % (unsigned)cluster);
        const int u = (int)(blockIdx.x / (unsigned)cluster) % U;
        const int l0 = tu * m_rank / cluster, h0 = tu * (m_rank + 1) / cluster;
        t_begin = (int)(e + (int64_t)u * tu + l0);
        n = h0 - l0;
        if (n > 0) {
          fb = mb;
          fu = u;
          fslot = l0;
          foff = o2;
          fnb = n2;
        }
      }
    } else {
      const bool here = bb < B && tbb > 0 && excl <= t_begin && t_begin < excl + x;
      const uint32_t m = __ballot_sync(0xffffffffu, here);
      if (m && fb == B && n > 0) {
        const int src = __ffs(m) - 1;
        const int64_t e = __shfl_sync(0xffffffffu, excl, src);
        const int tu = __shfl_sync(0xffffffffu, tbb, src);
        fb = b0 + src;
        foff = __shfl_sync(0xffffffffu, offb, src);
        fnb = __shfl_sync(0xffffffffu, nbb, src);
        const int rem = (int)(t_begin - e);
        fu = rem / tu;
        fslot = rem % tu;
      }
    }
    before += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    st[0] = t_begin;
    st[1] = n;
    st[2] = fb;
    st[3] = fu;
    st[4] = fslot;
    st64[0] = foff;
    st64[1] = fnb;
  }
}

// Token of row `row` of the cursor's tile, or -1 past the unit's k_b kept
// tokens or on -1 (a slot threshold selection left empty); any other index
// outside [0, n_b) raises FLAG_BAD_INDEX and reads as -1.
__device__ __forceinline__ int row_token(const AttendTcParams& P, const UnitTileCursor& c,
                                         int row) {
  const int64_t jj = (int64_t)c.slot * kTile + row;
  int t = -1;
  if (jj < c.kb) {
    t = P.idx[((int64_t)c.b * P.U + c.u) * P.k + jj];
    if (t < -1 || t >= c.nb) {  // -1: no token (a slot threshold selection left empty)
      atomicOr(P.flags, FLAG_BAD_INDEX);
      t = -1;
    }
  }
  return t;
}

// The same in two steps, so that the load is not waited for until the token
// is used: the raw index of the row, and its check against n_b.
__device__ __forceinline__ int row_raw(const AttendTcParams& P, const UnitTileCursor& c, int row) {
  const int64_t jj = (int64_t)c.slot * kTile + row;
  return jj < c.kb ? P.idx[((int64_t)c.b * P.U + c.u) * P.k + jj] : -1;
}
__device__ __forceinline__ int row_checked(const AttendTcParams& P, int t, int64_t nb) {
  if (t < -1 || t >= nb) {
    atomicOr(P.flags, FLAG_BAD_INDEX);
    t = -1;
  }
  return t;
}

constexpr int kGatherRows = (kTile + kGatherThreads - 1) / kGatherThreads;  // token rows per gather thread

// Gather thread gt's share (of kW warps) of one tile's latent rows: items
// over 32 row groups x KB k-blocks; item e copies rows tk[4g .. 4g+3]
// (g = e % 32), latent columns (kb0 + kb)*64 .. +63 (kb = e / 32), by TMA
// gather4 into k-block kb of the buffer (128-byte swizzled [128 x 64] blocks,
// rows 4g .. 4g+3 at byte (g/2)*1024 + (g%2)*512).  A row without a token
// (-1) copies row `off`, which gets weight 0.
template <int kW>
__device__ __forceinline__ void gather_rows(const int* tk, int64_t off, uint32_t buf_s,
                                            const CUtensorMap* tmap, int kb0, int KB, int gt,
                                            uint32_t mbar) {
  // ops dealt round-robin over the warps: a warp's lanes issue their copies
  // one after another, so the issue time of a tile falls with the warps
  // that share it
  for (int e = (gt % 32) * kW + gt / 32; e < 32 * KB; e += kW * 32) {
    const int g4 = e & 31, kb = e >> 5;
    int rows[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tk[4 * g4 + j];
      rows[j] = (int)(off + (t < 0 ? 0 : t));
    }
    tc::tma_gather4(buf_s + (uint32_t)kb * 16384u + (uint32_t)(g4 >> 1) * 1024u +
                        (uint32_t)(g4 & 1) * 512u,
                    tmap, (kb0 + kb) * 64, rows[0], rows[1], rows[2], rows[3], mbar);
  }
}

// barrier indices
enum { B_PK = 0, B_KFULL = 1, B_VFULL = 3, B_KDONE = 5, B_PDONE = 7, B_PREADY = 9,
       B_TKFREE = 11, B_TOFREE = 13, B_PKDONE = 15, B_PV = 16, B_COUNT = 17 };

// W = 1: the latent width r <= 256 fits one tile buffer; two buffers hold two
// tiles, and tiles are pipelined.  W = 2 (256 < r <= 512): the two buffers hold
// the two latent halves of one tile, Pk_u is loaded half by half (the
// reconstruction accumulates over the halves), and tiles run one after the
// other.
template <int G, int D, int W, bool kMerge>
__global__ void __launch_bounds__(block_threads<W>(), 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tmap_pk,
                 const __grid_constant__ CUtensorMap tmap_kc,
                 const __grid_constant__ CUtensorMap tmap_vc, const AttendTcParams P) {
  constexpr int HALF = D / 2;
  constexpr int QP = HALF / kEpiParts;                     // RoPE pairs per epilogue thread
  constexpr int kPasses = (G * kTile + kEpiThreads - 1) / kEpiThreads;  // softmax items per thread
  constexpr int kSlots = (2 * W * G + kEpiParts - 1) / kEpiParts;  // (chunk, head) accumulators per epilogue thread
  static_assert(QP % 8 == 0, "TMEM loads of 8 columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int KB = P.r / 64 / W;              // k-blocks of 64 latent columns per buffer
  const int n_chunks = (P.r + 127) / 128;  // M = 128 slices of the latent width
  const uint32_t pk_bytes = (uint32_t)KB * D * 128;
  const uint32_t buf_bytes = (uint32_t)KB * 16384;
  // shared-memory layout (plain locals: nothing here may live in local memory)
  uint8_t* const s_pk = base;                                // Pk_u: KB x [D rows x 128 B]
  uint8_t* const s_buf0 = base + pk_bytes;                   // tile buffers: KB x [128 x 128 B]
  uint8_t* const s_buf1 = s_buf0 + buf_bytes;
  uint8_t* const s_pbuf0 = s_buf1 + buf_bytes;               // p operand: 2 x [16 x 128 B]
  uint8_t* const s_pbuf1 = s_pbuf0 + 4096;
  uint64_t* const s_fturn = (uint64_t*)(s_pbuf1 + 4096);    // [D/2] fixed-point turns
  double* const s_theta = (double*)(s_fturn + HALF);         // [D/2]
  float* const s_qr = (float*)(s_theta + HALF);              // [D/2][G] rotated (q_i, q_i+d/2)
  float* const s_pd = s_qr + G * D;                          // [parts][G][128] partial dots
  float* const s_wmax = s_pd + kEpiParts * G * kTile;        // [2][G][4] per-warp maxima
  float* const s_wsum = s_wmax + 8 * G;                      // [2][G][4] per-warp sums
  int* const s_tok = (int*)(s_wsum + 8 * G);                 // [2][128] token per row
  float* const s_run = (float*)(s_tok + 2 * kTile);          // [G][2] segment's running (m, l)
  float* const s_ab = s_run + 2 * G;                         // [G][2] rescale factors
  uint64_t* const s_bars = (uint64_t*)(((uintptr_t)(s_ab + 2 * G) + 7) & ~(uintptr_t)7);
  uint32_t* const s_tmem_slot = (uint32_t*)(s_bars + B_COUNT);
  int64_t* const s_start64 = (int64_t*)(s_bars + B_COUNT + 1);  // first tile's (off, n_b)
  int* const s_start = (int*)(s_start64 + 2);                    // t_begin, n, b, u, slot
  const uint32_t bar0 = tc::smem_u32(s_bars);
  auto bar = [bar0](int i) { return bar0 + 8u * (uint32_t)i; };

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (tid == 0) trace_stamp(P.trace, TRACE_START);
  allow_dependent_launch();
  const int m_rank = kMerge ? (int)(blockIdx.x % (unsigned)P.cluster) : 0;
  const int m_unit = kMerge ? (int)(blockIdx.x / (unsigned)P.cluster) : 0;
  // Tile range and first tile (set before the block-wide barrier below).
  if (warp == kLoadWarp0)
    find_first_tile(P.seq_off, P.B, P.U, P.k, P.n_tiles, kMerge ? P.cluster : 0, P.uni_nb,
                    s_start, s_start64);
  int n = 0;  // tiles of this CTA
  auto first_tile = [&](UnitTileCursor& c) {
    c.at(P.seq_off, P.B, P.U, P.k, s_start[2], s_start[3], s_start[4], s_start64[0],
         s_start64[1]);
  };
  // TMEM columns: K_sel [2][D], then acc [2][n_chunks * 16]
  const uint32_t o_col0 = 2 * D;
  const uint32_t o_cols = (uint32_t)n_chunks * 16;

  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) tc::mbar_init(bar(i), 1);
    tc::mbar_fence_init();
    tc::tma_prefetch_desc(&tmap_pk);
    tc::tma_prefetch_desc(&tmap_kc);
    tc::tma_prefetch_desc(&tmap_vc);
  }
  if (warp == kMmaWarp) tc::tmem_alloc(tc::smem_u32(s_tmem_slot), 512);
  // the p operand's unused rows (2G..15) stay zero
  for (int e = tid; e < 2 * 4096 / 4; e += block_threads<W>()) ((uint32_t*)s_pbuf0)[e] = 0u;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *s_tmem_slot;
  n = s_start[1];

  if (W == 2 && warp >= kLoadWarp0) {
    // ======================= gather warps, two latent halves =================
    // Warp h fills buffer h with latent half h of every tile: the key rows,
    // then, once the reconstruction is done, the value rows (gather_rows).
    // Thread gt looks up the token of row gt.
    const int h = (warp - kLoadWarp0) / kGatherWarps;
    const int gt = tid - (kLoadWarp0 + h * kGatherWarps) * 32;  // 0..127
    const uint32_t gbar = 2 + h;
    int* tk = s_tok + h * kTile;
    const uint32_t buf_s = tc::smem_u32(h ? s_buf1 : s_buf0);
    const uint32_t tile_bytes = (uint32_t)kTile * KB * 128;
    UnitTileCursor cur;
    first_tile(cur);
    grid_dependency_wait();  // the kept indices come from the previous kernel
    if (gt == 0 && h == 0) trace_stamp(P.trace, TRACE_WAITED);
    int t_next[kGatherRows];
#pragma unroll
    for (int j = 0; j < kGatherRows; ++j)
      t_next[j] = n > 0 && gt + j * kGatherThreads < kTile ? row_token(P, cur, gt + j * kGatherThreads) : -1;
    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      const int64_t off = cur.off;
      // the buffer is free once the value MMA of the previous tile is done
      if (i >= 1) ok = tc::mbar_wait(bar(B_PDONE + ((i - 1) & 1)), ((uint32_t)(i - 1) >> 1) & 1u, P.flags);
#pragma unroll
      for (int j = 0; j < kGatherRows; ++j)
        if (gt + j * kGatherThreads < kTile) tk[gt + j * kGatherThreads] = t_next[j];
      if (gt == 0) tc::mbar_expect_tx(bar(B_KFULL + h), tile_bytes);
      tc::named_sync(gbar, kGatherThreads);
      gather_rows<kGatherWarps>(tk, off, buf_s, &tmap_kc, h * KB, KB, gt, bar(B_KFULL + h));
      cur.next();
#pragma unroll
      for (int j = 0; j < kGatherRows; ++j)
        t_next[j] = i + 1 < n && gt + j * kGatherThreads < kTile
                        ? row_token(P, cur, gt + j * kGatherThreads) : -1;
      if (!tc::mbar_wait(bar(B_KDONE + (i & 1)), ((uint32_t)i >> 1) & 1u, P.flags)) break;
      if (gt == 0) tc::mbar_expect_tx(bar(B_VFULL + h), tile_bytes);
      tc::named_sync(gbar, kGatherThreads);
      gather_rows<kGatherWarps>(tk, off, buf_s, &tmap_vc, h * KB, KB, gt, bar(B_VFULL + h));
    }
  } else if (W == 2 && warp == kMmaWarp) {
    // ======================= MMA issuer, two latent halves ===================
    // Per tile: reconstruction over the latent half of Pk_u in the buffer ->
    // the other half of Pk_u -> reconstruction over it (accumulating) -> value
    // MMA over the four 128-column chunks of the latent width.  The next tile
    // of the same unit starts with the half left in the buffer; a new unit's
    // half 0 is loaded while the epilogue works on this tile.  The whole warp runs
    // the sequence (warp-uniform state and descriptors); one elected lane
    // issues each group of loads, MMAs and its commit.
    {
      const uint32_t idesc_k = tc::idesc_bf16_f32(kTile, D);
      const uint32_t idesc_v = tc::idesc_bf16_f32_amn(128, kPRows);
      const uint32_t pkb = tc::smem_u32(s_pk);
      UnitTileCursor cur;
      first_tile(cur);
      uint32_t pk_phase = 0, pkd_phase = 0;
      auto load_pk = [&](int u, int hh) {
        if (tc::elect_one()) {
          tc::mbar_expect_tx(bar(B_PK), pk_bytes);
          for (int kb = 0; kb < KB; ++kb)
            tc::tma_load_2d(pkb + (uint32_t)kb * D * 128, &tmap_pk, (hh * KB + kb) * 64, u * D,
                            bar(B_PK));
        }
        __syncwarp();
      };
      // reconstruction over one latent half, then a commit to `done`
      auto kmma = [&](uint32_t a0, uint32_t d_tmem, bool acc0, uint32_t done) {
        if (tc::elect_one()) {
          for (int kb = 0; kb < KB; ++kb)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc::mma_bf16(d_tmem, tc::sdesc_kmajor_sw128(a0 + kb * 16384 + 32 * k),
                           tc::sdesc_kmajor_sw128(pkb + kb * D * 128 + 32 * k), idesc_k,
                           (acc0 || kb || k) ? 1u : 0u);
          tc::mma_commit(done);
        }
        __syncwarp();
      };
      auto wait = [&](uint32_t b, uint32_t parity) {
        return __all_sync(0xffffffffu, tc::mbar_wait(b, parity, P.flags));
      };
      bool ok = true;
      // the Pk buffer holds latent half pk_h of Pk_{pk_u} (pk_u < 0: nothing
      // yet); a load into it is in flight while pk_pending
      int pk_u = -1, pk_h = 0;
      bool pk_pending = false;
      auto fetch_pk = [&](int u, int hh) {
        load_pk(u, hh);
        pk_u = u;
        pk_h = hh;
        pk_pending = true;
      };
      auto have_pk = [&]() -> bool {
        if (!pk_pending) return true;
        if (!wait(bar(B_PK), pk_phase)) return false;
        pk_phase ^= 1u;
        pk_pending = false;
        return true;
      };
      if (n > 0) fetch_pk(cur.u, 0);
      for (int i = 0; i < n && ok; ++i, cur.next()) {
        const int bi = i & 1;
        const uint32_t ph = ((uint32_t)i >> 1) & 1u;
        const uint32_t d_tmem = tmem_base + (uint32_t)bi * D;
        // The half of Pk_u already in the buffer goes first: consecutive tiles
        // of a unit take the halves in alternate order (the sum over halves
        // does not depend on it), so one load of Pk per tile, not two.
        const int h0 = pk_u == cur.u ? pk_h : 0, h1 = 1 - h0;
        if (pk_u != cur.u || pk_h != h0) {
          // not reached with the prefetch below; kept for any other order
          if (i > 0 && !(ok = wait(bar(B_KDONE + (bi ^ 1)), (((uint32_t)(i - 1)) >> 1) & 1u)))
            break;
          fetch_pk(cur.u, h0);
        }
        ok = have_pk() && wait(bar(B_KFULL + h0), (uint32_t)i & 1u) &&
             wait(bar(B_TKFREE + bi), ph ^ 1u);
        if (!ok) break;
        tc::fence_after_sync();
        kmma(tc::smem_u32(h0 ? s_buf1 : s_buf0), d_tmem, false, bar(B_PKDONE));
        if (!(ok = wait(bar(B_PKDONE), pkd_phase))) break;
        pkd_phase ^= 1u;
        fetch_pk(cur.u, h1);
        ok = have_pk() && wait(bar(B_KFULL + h1), (uint32_t)i & 1u);
        if (!ok) break;
        tc::fence_after_sync();
        kmma(tc::smem_u32(h1 ? s_buf1 : s_buf0), d_tmem, true, bar(B_KDONE + bi));
        if (i + 1 < n) {
          UnitTileCursor nx = cur;
          nx.next();
          if (nx.u != cur.u) {
            // half 0 of the next unit's Pk_u, once this reconstruction is done with Pk
            if (!(ok = wait(bar(B_KDONE + bi), ph))) break;
            fetch_pk(nx.u, 0);
          }
        }
        // value MMA: acc^T[r x 2G] = Vc_tile^T . p.  The two buffers are adjacent,
        // so latent k-block j of the tile is at s_buf0 + j * 16 KiB and chunk ch
        // (k-blocks 2ch, 2ch+1) may straddle them.
        ok = wait(bar(B_PREADY + bi), ph) && wait(bar(B_VFULL + 0), (uint32_t)i & 1u) &&
             wait(bar(B_VFULL + 1), (uint32_t)i & 1u) && wait(bar(B_TOFREE + bi), ph ^ 1u);
        if (!ok) break;
        tc::fence_after_sync();
        const uint32_t p0 = tc::smem_u32(bi ? s_pbuf1 : s_pbuf0);
        if (tc::elect_one()) {
          for (int ch = 0; ch < n_chunks; ++ch) {
            const uint32_t d_acc = tmem_base + o_col0 + (uint32_t)bi * o_cols + (uint32_t)ch * 16;
            const uint32_t v0 = tc::smem_u32(s_buf0) + (uint32_t)ch * 2 * 16384;
#pragma unroll
            for (int ks = 0; ks < kTile / 16; ++ks) {
              const uint64_t ad =
                  tc::sdesc_mnmajor_sw128(v0 + (uint32_t)(ks * 2) * 1024, 16384, 1024);
              const uint64_t bd = tc::sdesc_kmajor_sw128(p0 + (uint32_t)(ks >> 2) * 2048 +
                                                         (uint32_t)(ks & 3) * 32);
              tc::mma_bf16(d_acc, ad, bd, idesc_v, ks != 0);
            }
          }
          tc::mma_commit(bar(B_PDONE + bi));
        }
        __syncwarp();
      }
    }
  } else if (warp >= kLoadWarp0) {
    // ======================= gather warps =======================
    // The seven gather warps issue the copies of every tile together, in the
    // order K(i), K(i+1), V(i), V(i+1), K(i+2), ...: tile i goes to buffer
    // i % 2, its latent key rows Kc_b[idx] once the value MMA of tile i-2 is
    // done with the buffer, the same rows of Vc once the reconstruction of
    // tile i is done with the key rows (gather_rows).  A pair's 256 token
    // slots (slot s: row s % 128 of tile i + s / 128) are dealt to the team's
    // threads; the next pair's indices are loaded while this pair is in
    // flight, and checked when stored.  Every wait ends in a team-wide vote,
    // so the team leaves together when one gives up.
    constexpr int kTeamWarps = gather_warps<1>();
    constexpr int kTeam = kTeamWarps * 32;
    // token slots s = gt + j*kTeam < 256 of a pair: tile s / 128, row s % 128
    constexpr int kTokSlots = (2 * kTile + kTeam - 1) / kTeam;
    const int gt = tid - kLoadWarp0 * 32;
    constexpr uint32_t kTeamBar = 2;
    const uint32_t buf0 = tc::smem_u32(s_buf0), buf1 = tc::smem_u32(s_buf1);
    const uint32_t tile_bytes = (uint32_t)kTile * P.r * 2;
    UnitTileCursor ca, cb;  // tiles i and i+1
    first_tile(ca);
    cb = ca;
    cb.next();
    grid_dependency_wait();  // the kept indices come from the previous kernel
    if (gt == 0) trace_stamp(P.trace, TRACE_WAITED);
    int t_next[kTokSlots];
#pragma unroll
    for (int j = 0; j < kTokSlots; ++j) {
      const int sl = gt + j * kTeam;
      t_next[j] = sl < 2 * kTile && (sl >> 7) < n ? row_raw(P, (sl >> 7) ? cb : ca, sl & 127) : -1;
    }
    for (int i = 0; i < n; i += 2) {
      const bool two = i + 1 < n;
      const uint32_t ph = ((uint32_t)i >> 1) & 1u;
      const int64_t off0 = ca.off, off1 = cb.off;
      // K(i): buffer 0 is free once the value MMA of tile i-2 is done
      bool okl = i < 2 || tc::mbar_wait(bar(B_PDONE + 0), ph ^ 1u, P.flags);
#pragma unroll
      for (int j = 0; j < kTokSlots; ++j) {
        const int sl = gt + j * kTeam;
        if (okl && sl < kTile) s_tok[sl] = row_checked(P, t_next[j], ca.nb);
      }
      if (!tc::named_sync_and(kTeamBar, kTeam, okl)) break;
      if (gt == 0) tc::mbar_expect_tx(bar(B_KFULL + 0), tile_bytes);
      gather_rows<kTeamWarps>(s_tok, off0, buf0, &tmap_kc, 0, KB, gt, bar(B_KFULL + 0));
      // K(i+1) into buffer 1, free once the value MMA of tile i-1 is done
      if (two) {
        okl = i < 2 || tc::mbar_wait(bar(B_PDONE + 1), ph ^ 1u, P.flags);
#pragma unroll
        for (int j = 0; j < kTokSlots; ++j) {
          const int sl = gt + j * kTeam;
          if (okl && sl >= kTile && sl < 2 * kTile) s_tok[sl] = row_checked(P, t_next[j], cb.nb);
        }
        if (!tc::named_sync_and(kTeamBar, kTeam, okl)) break;
        if (gt == 0) tc::mbar_expect_tx(bar(B_KFULL + 1), tile_bytes);
        gather_rows<kTeamWarps>(s_tok + kTile, off1, buf1, &tmap_kc, 0, KB, gt,
                                bar(B_KFULL + 1));
      }
      // the next pair's indices: loaded now, used at its key gathers
      ca.next();
      ca.next();
      cb.next();
      cb.next();
#pragma unroll
      for (int j = 0; j < kTokSlots; ++j) {
        const int sl = gt + j * kTeam;
        t_next[j] = sl < 2 * kTile && i + 2 + (sl >> 7) < n
                        ? row_raw(P, (sl >> 7) ? cb : ca, sl & 127) : -1;
      }
      // V(i), V(i+1): the reconstruction is done with the key rows
      okl = tc::mbar_wait(bar(B_KDONE + 0), ph, P.flags);
      if (!tc::named_sync_and(kTeamBar, kTeam, okl)) break;
      if (gt == 0) tc::mbar_expect_tx(bar(B_VFULL + 0), tile_bytes);
      gather_rows<kTeamWarps>(s_tok, off0, buf0, &tmap_vc, 0, KB, gt, bar(B_VFULL + 0));
      if (two) {
        okl = tc::mbar_wait(bar(B_KDONE + 1), ph, P.flags);
        if (!tc::named_sync_and(kTeamBar, kTeam, okl)) break;
        if (gt == 0) tc::mbar_expect_tx(bar(B_VFULL + 1), tile_bytes);
        gather_rows<kTeamWarps>(s_tok + kTile, off1, buf1, &tmap_vc, 0, KB, gt,
                                bar(B_VFULL + 1));
      }
    }
  } else if (warp == kMmaWarp) {
    // ======================= MMA issuer =======================
    // An event loop: the reconstruction of tile nk (after its key rows have
    // landed and its TMEM buffer is free, with Pk_u reloaded at unit
    // boundaries) and the value MMA of tile np (after its weights and value
    // rows are ready) are each issued as soon as their own inputs are, so
    // neither waits behind the other.  At most two reconstructions run ahead
    // of the value MMAs (two tile buffers, two K_sel buffers in TMEM).  The
    // whole warp runs the loop, so its state and the descriptors are
    // warp-uniform; one elected lane issues each group of loads, MMAs and its
    // commit.
    {
      const uint32_t idesc_k = tc::idesc_bf16_f32(kTile, D);
      const uint32_t idesc_v = tc::idesc_bf16_f32_amn(128, kPRows);
      UnitTileCursor cur;
      first_tile(cur);
      int cur_u = -1;
      uint32_t pk_phase = 0;
      int pk_step = 0;  // 1: waiting to reload Pk, 2: Pk load in flight
      int nk = 0, np = 0;
      uint64_t idle_since = 0;
      const uint32_t pkb = tc::smem_u32(s_pk);
      auto ready = [](uint32_t b, uint32_t parity) {
        return __all_sync(0xffffffffu, tc::mbar_test_wait(b, parity));
      };
      while (np < n) {
        bool progress = false;
        if (nk < n && nk <= np + 2) {
          if (pk_step == 0 && cur.u != cur_u) pk_step = 1;  // Pk_u: the unit's rows of Pk
          // Pk_u of a new unit, once the previous reconstruction is done with Pk
          if (pk_step == 1 &&
              (nk == 0 || ready(bar(B_KDONE + ((nk - 1) & 1)), ((uint32_t)(nk - 1) >> 1) & 1u))) {
            if (tc::elect_one()) {
              tc::mbar_expect_tx(bar(B_PK), pk_bytes);
              for (int kb = 0; kb < KB; ++kb)
                tc::tma_load_2d(pkb + (uint32_t)kb * D * 128, &tmap_pk, kb * 64, cur.u * D,
                                bar(B_PK));
            }
            __syncwarp();
            pk_step = 2;
            progress = true;
          }
          if (pk_step == 2 && ready(bar(B_PK), pk_phase)) {
            pk_phase ^= 1u;
            cur_u = cur.u;
            pk_step = 0;
            progress = true;
          }
          const int bk = nk & 1;
          if (pk_step == 0 && ready(bar(B_KFULL + bk), ((uint32_t)nk >> 1) & 1u) &&
              ready(bar(B_TKFREE + bk), (((uint32_t)nk >> 1) & 1u) ^ 1u)) {
            tc::fence_after_sync();
            const uint32_t kb0 = tc::smem_u32(bk ? s_buf1 : s_buf0);
            const uint32_t d_tmem = tmem_base + (uint32_t)bk * D;
            if (tc::elect_one()) {
              for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  tc::mma_bf16(d_tmem, tc::sdesc_kmajor_sw128(kb0 + kb * 16384 + 32 * k),
                               tc::sdesc_kmajor_sw128(pkb + kb * D * 128 + 32 * k), idesc_k,
                               (kb | k) != 0);
              tc::mma_commit(bar(B_KDONE + bk));
            }
            __syncwarp();
            ++nk;
            cur.next();
            progress = true;
          }
        }
        const int bp = np & 1;
        if (np < nk && ready(bar(B_PREADY + bp), ((uint32_t)np >> 1) & 1u) &&
            ready(bar(B_VFULL + bp), ((uint32_t)np >> 1) & 1u) &&
            ready(bar(B_TOFREE + bp), (((uint32_t)np >> 1) & 1u) ^ 1u)) {
          tc::fence_after_sync();
          const uint32_t p0 = tc::smem_u32(bp ? s_pbuf1 : s_pbuf0);
          const uint32_t vb0 = tc::smem_u32(bp ? s_buf1 : s_buf0);
          if (tc::elect_one()) {
            for (int ch = 0; ch < n_chunks; ++ch) {
              const uint32_t d_tmem = tmem_base + o_col0 + (uint32_t)bp * o_cols + (uint32_t)ch * 16;
#pragma unroll
              for (int ks = 0; ks < kTile / 16; ++ks) {
                // A = Vc_tile^T: latent columns ch*128.. (MN), tokens ks*16.. (K)
                const uint64_t ad = tc::sdesc_mnmajor_sw128(
                    vb0 + (uint32_t)ch * 2 * 16384 + (uint32_t)(ks * 2) * 1024, 16384, 1024);
                // B = p rows (hi/lo per head), tokens ks*16..: K-major k-block ks/4
                const uint64_t bd = tc::sdesc_kmajor_sw128(p0 + (uint32_t)(ks >> 2) * 2048 +
                                                           (uint32_t)(ks & 3) * 32);
                tc::mma_bf16(d_tmem, ad, bd, idesc_v, ks != 0);
              }
            }
            tc::mma_commit(bar(B_PDONE + bp));
          }
          __syncwarp();
          ++np;
          progress = true;
        }
        if (progress) {
          idle_since = 0;
        } else {
          const uint64_t now = __shfl_sync(0xffffffffu, tc::globaltimer_ns(), 0);
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > tc::kWaitLimitNs) {
            if (lane == 0) atomicOr(P.flags, FLAG_WAIT_TIMEOUT);
            break;
          }
          __nanosleep(32);
        }
      }
      if constexpr (kMerge) {
        // this rank's rows of Pv_u for the value projection, into the Pk
        // buffer once the last reconstruction is done with it
        const bool okp =
            n == 0 || __all_sync(0xffffffffu, tc::mbar_wait(bar(B_KDONE + ((n - 1) & 1)),
                                                            ((uint32_t)(n - 1) >> 1) & 1u, P.flags));
        if (okp && tc::elect_one()) {
          const int dq = D / P.cluster;
          const uint32_t bytes = (uint32_t)dq * (uint32_t)P.r * 2u;
          tc::mbar_expect_tx(bar(B_PV), bytes);
          tc::bulk_load(tc::smem_u32(s_pk),
                        P.Pv + ((int64_t)(m_unit % P.U) * D + (int64_t)m_rank * dq) * P.r, bytes,
                        bar(B_PV));
        }
        __syncwarp();
      }
    }
  } else {
    // ======================= epilogue (warps 0-15) =======================
    // Warp w reads TMEM lanes 32*(w%4).. (its token rows) and takes the RoPE
    // pairs [part*QP, (part+1)*QP) of them, part = w/4; the parts' partial
    // logits meet in shared memory, where thread e takes head e/128 and token
    // e%128 for the tile's softmax.
    const int quarter = warp & 3, part = warp >> 2;
    const int m = quarter * 32 + lane;  // token row = TMEM lane
    // RoPE frequencies theta_i = base^(-2i/d) and their fixed-point turns
    // (here, not before the block-wide barrier: the gathers need neither)
    for (int i = tid; i < HALF; i += kEpiThreads) {
      const double th = pow(P.base, -2.0 * (double)i / (double)D);
      s_theta[i] = th;
      s_fturn[i] = __double2ull_rn(th / kTwoPi * 18446744073709551616.0);
    }
    tc::named_sync(kEpiBar, kEpiThreads);
    UnitTileCursor cur;
    first_tile(cur);
    int cur_b = -1, cur_u = -1;
    uint32_t pos_b = 0;  // position of the sequence's token 0 (token-sharded caches)
    // the segment's running sums: slot s = part + kEpiParts*j (j < kSlots) holds latent
    // column (s / G)*128 + quarter*32 + lane of head s % G
    const int n_used = n_chunks * G;
    float acc_run[kSlots];
#pragma unroll
    for (int j = 0; j < kSlots; ++j) acc_run[j] = 0.f;
    int seg_tiles = 0;
    if (tid < G) {
      s_run[2 * tid] = -INFINITY;
      s_run[2 * tid + 1] = 0.f;
    }
    // Fold tile j (the cursor fc is at it) into its unit segment's running
    // (m, l, acc) and publish the segment at its end.  Tile j is folded after
    // the weights of tile j+1 are computed, so that the value MMA of tile j
    // runs meanwhile.
    UnitTileCursor fc = cur;
    auto fold = [&](int j) {
      const int bj = j & 1;
      const uint32_t phj = ((uint32_t)j >> 1) & 1u;
      // the tile's (m, l) per head from the per-warp maxima and sums, and the
      // heads' scale factors
      if (tid < G) {
        const float* wm = s_wmax + (bj * G + tid) * 4;
        const float* ws = s_wsum + (bj * G + tid) * 4;
        const float mt = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
        const float lt = (ws[0] + ws[1]) + (ws[2] + ws[3]);
        const float mr = s_run[2 * tid], lr = s_run[2 * tid + 1];
        const float mx = fmaxf(mr, mt);
        float al = 0.f, be = 0.f;
        if (mx != -INFINITY) {
          al = mr == -INFINITY ? 0.f : expf(mr - mx);
          be = mt == -INFINITY ? 0.f : expf(mt - mx);
        }
        s_ab[2 * tid] = al;
        s_ab[2 * tid + 1] = be;
        s_run[2 * tid] = mx;
        s_run[2 * tid + 1] = lr * al + lt * be;
      }
      // the tile's acc from TMEM: columns (hi, lo) of head g in chunk c
      const bool ok2 = __all_sync(0xffffffffu, tc::mbar_wait(bar(B_PDONE + bj), phj, P.flags));
      tc::fence_after_sync();
      uint32_t v[kSlots][2];
#pragma unroll
      for (int jj = 0; jj < kSlots; ++jj) {
        const int sl = part + kEpiParts * jj;
        if (ok2 && sl < n_used)
          tc::tmem_ld2(tmem_base + ((uint32_t)(quarter * 32) << 16) + o_col0 + (uint32_t)bj * o_cols +
                           (uint32_t)(sl / G) * 16 + 2u * (uint32_t)(sl % G),
                       v[jj]);
      }
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      tc::named_sync(kEpiBar, kEpiThreads);
      if (tid == 0) tc::mbar_arrive(bar(B_TOFREE + bj));
#pragma unroll
      for (int jj = 0; jj < kSlots; ++jj) {
        const int sl = part + kEpiParts * jj;
        if (ok2 && sl < n_used) {
          const int g = sl % G;
          acc_run[jj] = acc_run[jj] * s_ab[2 * g] +
                        (__uint_as_float(v[jj][0]) + __uint_as_float(v[jj][1])) * s_ab[2 * g + 1];
        }
      }
      // end of this CTA's segment of the unit: publish it
      UnitTileCursor nx = fc;
      nx.next();
      const bool seg_end = j + 1 == n || nx.b != fc.b || nx.u != fc.u;
      ++seg_tiles;
      if (!kMerge && seg_end) {
        const int s0 = fc.slot + 1 - seg_tiles;  // first slot of the segment
        const int64_t row0 = ((int64_t)fc.b * P.Hq + fc.u * G) * P.n_slots + s0;
#pragma unroll
        for (int jj = 0; jj < kSlots; ++jj) {
          const int sl = part + kEpiParts * jj;
          const int c = (sl / G) * 128 + quarter * 32 + lane;
          if (sl < n_used && c < P.r)
            P.part[(row0 + (int64_t)(sl % G) * P.n_slots) * part_row(P.r) + kPartAcc + c] =
                acc_run[jj];
          acc_run[jj] = 0.f;
        }
        if (tid < G) {
          float* pp = P.part + (row0 + (int64_t)tid * P.n_slots) * part_row(P.r);
          pp[0] = s_run[2 * tid];
          pp[1] = s_run[2 * tid + 1];
          s_run[2 * tid] = -INFINITY;
          s_run[2 * tid + 1] = 0.f;
        }
        // a new segment starts with the next tile
        seg_tiles = 0;
      }
      fc = nx;
    };
    for (int i = 0; i < n; ++i, cur.next()) {
      const int bi = i & 1;
      const uint32_t ph = ((uint32_t)i >> 1) & 1u;
      if (cur.b != cur_b || cur.u != cur_u) {
        // rotated queries of the unit's heads (angles reduced in fp64), as
        // pairs (q_i, q_i+d/2) in the order [pair][head]
        const double qpos = P.q_pos ? (double)P.q_pos[cur.b] : (double)cur.nb;
        pos_b = P.pos_off ? (uint32_t)P.pos_off[cur.b] : 0u;
        for (int e = tid; e < G * HALF; e += kEpiThreads) {
          const int g = e / HALF, ii = e % HALF;
          const __nv_bfloat16* qh = P.q + ((int64_t)cur.b * P.Hq + cur.u * G + g) * D;
          const double a = qpos * s_theta[ii];
          const double nt = rint(a * (1.0 / kTwoPi));
          float s, c;
          sincosf((float)fma(-nt, kTwoPi, a), &s, &c);
          const float x0 = __bfloat162float(qh[ii]), x1 = __bfloat162float(qh[ii + HALF]);
          *(float2*)(s_qr + 2 * (ii * G + g)) = make_float2(x0 * c - x1 * s, x1 * c + x0 * s);
        }
        cur_b = cur.b;
        cur_u = cur.u;
        tc::named_sync(kEpiBar, kEpiThreads);
      }
      // ---- K_sel row m, pairs [part*QP, (part+1)*QP)
      const bool ok =
          __all_sync(0xffffffffu, tc::mbar_wait(bar(B_KDONE + bi), ph, P.flags));
      tc::fence_after_sync();
      // this row's token: written by the gather warp before it released the
      // Kc barrier of this tile, which is acquired here (its phase is complete)
      const int t = W == 1 ? (tc::mbar_wait(bar(B_KFULL + bi), ph, P.flags), s_tok[bi * kTile + m])
                           : (tc::mbar_wait(bar(B_KFULL), (uint32_t)i & 1u, P.flags), s_tok[m]);
      float dot[G];
#pragma unroll
      for (int g = 0; g < G; ++g) dot[g] = 0.f;
      if (ok) {
        const uint32_t row_addr =
            tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)bi * D + (uint32_t)(part * QP);
        const uint32_t tu = (uint32_t)(t < 0 ? 0 : t) + pos_b;
#pragma unroll 1
        for (int c8 = 0; c8 < QP; c8 += 8) {
          uint32_t v0[8], v1[8];
          tc::tmem_ld8(row_addr + c8, v0);
          tc::tmem_ld8(row_addr + HALF + c8, v1);
          tc::tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int ii = part * QP + c8 + jj;
            const uint64_t F = s_fturn[ii];
            const uint32_t turn = __umulhi(tu, (uint32_t)F) + tu * (uint32_t)(F >> 32);
            float s, c;
            __sincosf((float)(int32_t)turn * (float)(kTwoPi / 4294967296.0), &s, &c);
            const float x0 = __uint_as_float(v0[jj]), x1 = __uint_as_float(v1[jj]);
            const float k0 = x0 * c - x1 * s;
            const float k1 = x1 * c + x0 * s;
            const float* qp = s_qr + 2 * ii * G;
            if constexpr (G % 2 == 0) {
#pragma unroll
              for (int g = 0; g < G; g += 2) {
                const float4 qv = *(const float4*)(qp + 2 * g);
                dot[g] = fmaf(qv.x, k0, fmaf(qv.y, k1, dot[g]));
                dot[g + 1] = fmaf(qv.z, k0, fmaf(qv.w, k1, dot[g + 1]));
              }
            } else {
              const float2 qv = *(const float2*)qp;
              dot[0] = fmaf(qv.x, k0, fmaf(qv.y, k1, dot[0]));
            }
          }
        }
      }
      // a row without a token gets logit -inf through part 0's partial dot
#pragma unroll
      for (int g = 0; g < G; ++g)
        s_pd[(part * G + g) * kTile + m] = (part == 0 && t < 0) ? -INFINITY : dot[g];
      tc::fence_before_sync();
      tc::named_sync(kEpiBar, kEpiThreads);
      if (tid == 0) tc::mbar_arrive(bar(B_TKFREE + bi));  // K_sel[bi] may be overwritten
      // ---- logits and the tile's softmax: thread e takes head e / 128 and
      // token e % 128, so warp w covers 32 tokens of one head
      float lg[kPasses];
#pragma unroll
      for (int ps = 0; ps < kPasses; ++ps) {
        const int e = tid + ps * kEpiThreads;
        const int g = e >> 7, mm = e & (kTile - 1);
        float l = -INFINITY;
        if (e < G * kTile) {
          float sum = 0.f;
#pragma unroll
          for (int pt = 0; pt < kEpiParts; ++pt) sum += s_pd[(pt * G + g) * kTile + mm];
          l = sum * P.scale;
        }
        lg[ps] = l;
        float mx = l;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0 && e < G * kTile) s_wmax[(bi * G + g) * 4 + (mm >> 5)] = mx;
      }
      tc::named_sync(kEpiBar, kEpiThreads);
      // ---- weights p = exp(l - m) as bf16 hi/lo rows 2g, 2g+1 of the value
      // MMA's B operand (K-major, 128-byte swizzle)
      uint8_t* const pb = bi ? s_pbuf1 : s_pbuf0;
#pragma unroll
      for (int ps = 0; ps < kPasses; ++ps) {
        const int e = tid + ps * kEpiThreads;
        const int g = e >> 7, mm = e & (kTile - 1);
        if (e < G * kTile) {
          const float* wm = s_wmax + (bi * G + g) * 4;
          const float mt = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
          const float p = lg[ps] == -INFINITY ? 0.f : expf(lg[ps] - mt);
          float sum = p;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          if (lane == 0) s_wsum[(bi * G + g) * 4 + (mm >> 5)] = sum;
          const __nv_bfloat16 hi = __float2bfloat16_rn(p);
          const __nv_bfloat16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
          uint8_t* const pk = pb + (mm >> 6) * 2048;
          const int col = mm & 63, chunk = col >> 3, within = col & 7;
          const int r0 = 2 * g, r1 = 2 * g + 1;
          *(__nv_bfloat16*)(pk + (r0 >> 3) * 1024 + (r0 & 7) * 128 + ((chunk ^ (r0 & 7)) << 4) +
                            within * 2) = hi;
          *(__nv_bfloat16*)(pk + (r1 >> 3) * 1024 + (r1 & 7) * 128 + ((chunk ^ (r1 & 7)) << 4) +
                            within * 2) = lo;
        }
      }
      tc::fence_proxy_async_smem();
      tc::named_sync(kEpiBar, kEpiThreads);
      if (tid == 0) tc::mbar_arrive(bar(B_PREADY + bi));
      if (i > 0) fold(i - 1);
    }
    if (n > 0) {
      // the previous fold's readers of the scale factors are done
      tc::named_sync(kEpiBar, kEpiThreads);
      fold(n - 1);
    }
    if constexpr (kMerge) {
      // this CTA's partial of the unit, (m, l) and acc[r] per head, staged in
      // the first tile buffer (every MMA and copy into it has completed) for
      // the cluster's merge
      float* const st = (float*)s_buf0;
#pragma unroll
      for (int jj = 0; jj < kSlots; ++jj) {
        const int sl = part + kEpiParts * jj;
        const int c = (sl / G) * 128 + quarter * 32 + lane;
        if (sl < n_used && c < P.r) st[2 * G + (sl % G) * P.r + c] = acc_run[jj];
      }
      if (tid < G) {
        st[2 * tid] = s_run[2 * tid];
        st[2 * tid + 1] = s_run[2 * tid + 1];
      }
    }
  }
  if constexpr (kMerge) {
    // ---- the unit's partials, merged across the cluster (the same online-
    //      softmax combination as the merge kernel, over ranks in order), and
    //      the deferred value projection: rank q writes output dims
    //      q*d/C .. (q+1)*d/C - 1 of the unit's heads, out = acc . Pv_u^T
    cluster_arrive();
    cluster_wait();  // every CTA's partial is staged
    constexpr int kMaxCl = 8;
    const int C = P.cluster;
    float* const accm = (float*)s_buf1;  // merged acc [G][r]
    if (warp < kEpiWarps) {
      uint32_t rs[kMaxCl];  // each rank's staged partial
#pragma unroll
      for (int q = 0; q < kMaxCl; ++q) rs[q] = q < C ? cluster_addr(s_buf0, q) : 0u;
      for (int e = tid; e < G * P.r; e += kEpiThreads) {
        const int g = e / P.r, c = e % P.r;
        float mq[kMaxCl], lq[kMaxCl], aq[kMaxCl];
#pragma unroll
        for (int q = 0; q < kMaxCl; ++q) {
          if (q < C) {
            mq[q] = ld_cluster_f32(rs[q] + 4u * (uint32_t)(2 * g));
            lq[q] = ld_cluster_f32(rs[q] + 4u * (uint32_t)(2 * g + 1));
            aq[q] = ld_cluster_f32(rs[q] + 4u * (uint32_t)(2 * G + g * P.r + c));
          }
        }
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < kMaxCl; ++q)
          if (q < C) M = fmaxf(M, mq[q]);
        float L = 0.f, a = 0.f;
#pragma unroll
        for (int q = 0; q < kMaxCl; ++q) {
          if (q < C && mq[q] != -INFINITY) {
            const float w = expf(mq[q] - M);
            L += w * lq[q];
            a += w * aq[q];
          }
        }
        accm[e] = L > 0.f ? a / L : 0.f;
      }
    }
    cluster_arrive();  // done with the other CTAs' shared memory
    if (warp < kEpiWarps) {
      tc::named_sync(kEpiBar, kEpiThreads);  // the merged acc is complete
      const bool okv = __all_sync(0xffffffffu, tc::mbar_wait(bar(B_PV), 0u, P.flags));
      const int dq = D / C;
      const int u = m_unit % P.U, mb = m_unit / P.U;
      // four threads per output (G x dq outputs, dq a multiple of 8)
      for (int e = tid; e < G * dq * 4; e += kEpiThreads) {
        const int o = e >> 2, sub = e & 3;
        const int g = o / dq, dd = o % dq;
        const __nv_bfloat162* pvr = (const __nv_bfloat162*)(s_pk + (size_t)dd * P.r * 2);
        const float* ar = accm + g * P.r;
        float acc = 0.f;
        if (okv)
          for (int c = 2 * sub; c < P.r; c += 8) {
            const float2 pv = __bfloat1622float2(pvr[c >> 1]);
            acc = fmaf(ar[c], pv.x, fmaf(ar[c + 1], pv.y, acc));
          }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (sub == 0)
          P.out[((int64_t)mb * P.Hq + u * G + g) * D + m_rank * dq + dd] = __float2bfloat16_rn(acc);
      }
    }
    cluster_wait();
  }
  tc::fence_before_sync();
  __syncthreads();
  if (tid == 0) trace_stamp(P.trace, TRACE_END);
  if (warp == kMmaWarp) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, 512);
  }
}

int num_sms_att() {
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

template <int G, int D, int W>
size_t smem_bytes(int r) {
  const int KB = r / 64 / W;
  return 1024 + (size_t)KB * D * 128 + 2 * (size_t)KB * 16384 + 2 * 4096 + 8 * (D / 2) * 2 +
         4 * (G * D + kEpiParts * G * kTile + 16 * G + 2 * kTile + 4 * G) + 8 +
         8 * B_COUNT + 16 + 16 + 24;
}

template <int G, int D, int W, bool kMerge>
cudaError_t launch_g_d(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = smem_bytes<G, D, W>(p.r);
  CUtensorMap tpk, tkc, tvc;
  if (!make_tmap_bf16_2d(&tpk, a.Pk, (uint64_t)p.U * D, (uint64_t)p.r, D, 64) ||
      !make_tmap_bf16_2d(&tkc, a.Kc, (uint64_t)p.N, (uint64_t)p.r, 1, 64) ||
      !make_tmap_bf16_2d(&tvc, a.Vc, (uint64_t)p.N, (uint64_t)p.r, 1, 64))
    return cudaErrorInvalidValue;
  static int done[kMaxDevices] = {};
  cudaError_t e = ensure_smem(attend_tc_kernel<G, D, W, kMerge>, smem, done);
  if (e != cudaSuccess) return e;
  AttendTcParams P;
  P.q = (const __nv_bfloat16*)a.q;
  P.Kc = (const __nv_bfloat16*)a.Kc;
  P.Vc = (const __nv_bfloat16*)a.Vc;
  P.idx = a.idx;
  P.seq_off = a.seq_off;
  P.q_pos = a.q_pos;
  P.pos_off = a.pos_off;
  P.part = a.part;
  P.flags = a.flags;
  P.Pv = (const __nv_bfloat16*)a.Pv;
  P.out = (__nv_bfloat16*)a.out;
  P.B = p.B;
  P.Hq = p.Hq;
  P.U = p.U;
  P.r = p.r;
  P.k = p.k;
  P.n_slots = p.splits;
  P.n_tiles = p.att_tiles;
  P.uni_nb = p.uni_nb;
  P.cluster = kMerge ? p.att_cluster : 1;
  P.trace = trace_of(a, 3);
  P.scale = p.scale;
  P.base = p.rope_base;
  if constexpr (!kMerge) {
    return launch_k(attend_tc_kernel<G, D, W, false>, dim3(attend_tc_grid(p)),
                    dim3(block_threads<W>()),
                    smem, s, true, tpk, tkc, tvc, P);
  } else {
    // one cluster of att_cluster CTAs per unit
    e = prefer_max_shared((const void*)attend_tc_kernel<G, D, W, true>);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.B * p.U * p.att_cluster));
    cfg.blockDim = dim3(block_threads<W>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)p.att_cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, attend_tc_kernel<G, D, W, true>, tpk, tkc, tvc, P);
  }
}

template <int W, bool kMerge>
cudaError_t launch_w(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  if (p.d == 128) {
    switch (p.G) {
      case 1: return launch_g_d<1, 128, W, kMerge>(p, a, s);
      case 2: return launch_g_d<2, 128, W, kMerge>(p, a, s);
      case 4: return launch_g_d<4, 128, W, kMerge>(p, a, s);
      case 8: return launch_g_d<8, 128, W, kMerge>(p, a, s);
    }
  } else {
    switch (p.G) {
      case 1: return launch_g_d<1, 64, W, kMerge>(p, a, s);
      case 2: return launch_g_d<2, 64, W, kMerge>(p, a, s);
      case 4: return launch_g_d<4, 64, W, kMerge>(p, a, s);
      case 8: return launch_g_d<8, 64, W, kMerge>(p, a, s);
    }
  }
  return cudaErrorInvalidConfiguration;
}

}  // namespace

int attend_tc_grid(const DecodePlan& p) {
  return p.att_tiles < num_sms_att() ? p.att_tiles : num_sms_att();
}

bool attend_tc_supported(const DecodePlan& p) {
  const int64_t k_eff = p.k < p.n_max ? p.k : p.n_max;
  // r <= 256: one tile per buffer; 256 < r <= 512 with r % 128 == 0: two latent halves
  const bool width_ok = (p.r % 64 == 0 && p.r <= 256) || (p.r % 128 == 0 && p.r <= 512);
  return p.dtype == SALSC_BF16 && width_ok && (p.d == 64 || p.d == 128) &&
         (p.G == 1 || p.G == 2 || p.G == 4 || p.G == 8) && p.N <= INT32_MAX &&
         (k_eff + kTile - 1) / kTile <= kTile;  // the merge takes <= 128 slots per unit
}

int attend_merge_cluster(const DecodePlan& p) {
  // r <= 256 (one tile buffer per tile), and every unit's cluster resident at
  // once: the largest power of two C <= 8 with B*U*C <= #SMs (d/C >= 8 output
  // dims per rank).  The tile phase is bound by the row gathers of all SMs
  // together, so the clusters are used only when they take at least as many
  // SMs as the even split of the tiles, and no CTA gets more tiles than there.
  if (!attend_tc_supported(p) || p.r > 256 || p.att_tiles <= 0) return 0;
  const int64_t sms = num_sms_att();
  const int64_t units = (int64_t)p.B * p.U;
  int c = 0;
  for (int cc = 1; cc <= 8; cc *= 2)
    if (units * cc <= sms && p.d / cc >= 8) c = cc;
  if (c == 0) return 0;
  const int64_t grid_split = p.att_tiles < sms ? p.att_tiles : sms;
  const int64_t k_eff = p.k < p.n_max ? p.k : p.n_max;
  const int64_t tu_max = (k_eff + kTile - 1) / kTile;
  if (units * c < grid_split ||
      (tu_max + c - 1) / c > (p.att_tiles + grid_split - 1) / grid_split)
    return 0;
  return c;
}

cudaError_t launch_attend_tc(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  if (p.r > 256) return launch_w<2, false>(p, a, s);
  return p.att_cluster > 0 ? launch_w<1, true>(p, a, s) : launch_w<1, false>(p, a, s);
}

}  // namespace salsc
