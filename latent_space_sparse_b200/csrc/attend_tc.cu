// attend_tc.cu -- selective reconstruction, RoPE, softmax and the latent
// value sum over the kept tokens, on tcgen05 (bf16 storage, d in {64, 128},
// r <= 256, G in {1, 2, 4, 8}).
//
// SALS technical framework, stages 3-4, with RoPE applied after
// reconstruction (abstract).  Work unit: a tile of 128 kept tokens of one
// selection unit (b, u):
//   1. TMA gather4 brings the 128 latent key rows Kc_b[idx] into shared memory
//      (128-byte swizzled, K-major);
//   2. tcgen05: K_sel[128 x d] = Kc_tile . Pk_u^T into TMEM (fp32; Pk_u comes
//      by TMA once per unit and stays in shared memory);
//   3. the same rows of Vc are gathered into the buffer the MMA has finished
//      with;
//   4. eight epilogue warps (one thread per token row and half of the RoPE
//      pairs) read K_sel from TMEM, rotate pair (i, i+d/2) by the angle
//      t * base^(-2i/d) and dot it with every rotated query head of the unit;
//      the tile's softmax (max m, normaliser l) follows, and the weights p are
//      written to shared memory as bf16 hi + lo parts;
//   5. tcgen05: acc^T[r x 2G] = Vc_tile^T . [p_hi p_lo] into TMEM (Vc_tile read
//      as an MN-major operand, so the latent value rows need no transpose);
//   6. the epilogue reads acc[c] = D[c][2g] + D[c][2g+1] and writes the
//      tile's (m, l, acc) per head; the combine kernel merges tiles.
// Warp roles (320 threads): warps 0-7 epilogue, warp 8 TMEM owner and MMA
// issuer, warp 9 gather issuer.  Each CTA walks a contiguous range of tiles;
// the two tile buffers alternate (Kc(i) -> Vc(i) -> Kc(i+2)), so the
// reconstruction of tile i+1 runs during the epilogue of tile i.
//
// The RoPE angle uses an exact fixed-point phase: F_i = round(2^64 *
// theta_i / 2 pi), and the top 32 bits of t * F_i (mod 2^64) are t * theta_i
// modulo one turn, to 2^-32 of a turn, for any 32-bit position t.
#include "tc.cuh"

namespace salsc {
namespace {

constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kThreads = 320;
constexpr int kTile = 128;
constexpr int kPRows = 16;  // rows of the p operand (2G <= 16)
constexpr uint32_t kEpiBar = 1;
constexpr double kTwoPi = 6.283185307179586476925286766559;

struct AttendTcParams {
  const __nv_bfloat16* q;
  const int32_t* idx;
  const int64_t* seq_off;
  const int32_t* q_pos;
  float* part;
  uint32_t* flags;
  int B, Hq, U, r, k, n_slots, n_tiles;
  float scale;
  double base;
};

// Walks the tiles of all units in order (sequence, unit, slot); unit (b, u)
// has ceil(min(k, n_b) / 128) tiles.
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
  __device__ void start(const int64_t* so_, int B_, int U_, int k_, int tile) {
    so = so_;
    B = B_;
    U = U_;
    k = k_;
    int acc = 0;
    for (b = 0; b < B; ++b) {
      load();
      if (tile < acc + U * tb) {
        const int rem = tile - acc;
        u = rem / tb;
        slot = rem % tb;
        return;
      }
      acc += U * tb;
    }
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

struct Smem {
  uint8_t* pk;       // Pk_u: KB k-blocks of [D rows x 128 B]
  uint8_t* buf[2];   // tile buffers: KB k-blocks of [128 rows x 128 B]
  uint8_t* pbuf[2];  // p operand: 2 k-blocks of [16 rows x 128 B]
  uint64_t* fturn;   // [D/2] fixed-point turns per token position
  double* theta;     // [D/2]
  float* qr;         // [G][D] rotated queries
  float* pd;         // [2][G][128] partial dot products of the two pair halves
  float* lg;         // [G][128] logits, then softmax weights
  float* stat;       // [G][2] (m, l)
  int* tok;          // [2][128] token index per row (-1: no token), gather warp only
  uint64_t* bars;
  uint32_t* tmem_slot;
};

// barrier indices
enum { B_PK = 0, B_KFULL = 1, B_VFULL = 3, B_KDONE = 5, B_PDONE = 7, B_PREADY = 9,
       B_TKFREE = 11, B_TOFREE = 13, B_COUNT = 15 };

template <int G, int D>
__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tmap_pk,
                 const __grid_constant__ CUtensorMap tmap_kc,
                 const __grid_constant__ CUtensorMap tmap_vc, const AttendTcParams P) {
  constexpr int HALF = D / 2;
  constexpr int QPAIRS = HALF / 2;  // RoPE pairs per epilogue thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int KB = P.r / 64;
  const int n_chunks = (P.r + 127) / 128;  // M = 128 slices of the latent width
  const uint32_t pk_bytes = (uint32_t)KB * D * 128;
  const uint32_t buf_bytes = (uint32_t)KB * 16384;
  Smem S;
  S.pk = base;
  S.buf[0] = base + pk_bytes;
  S.buf[1] = S.buf[0] + buf_bytes;
  S.pbuf[0] = S.buf[1] + buf_bytes;
  S.pbuf[1] = S.pbuf[0] + 4096;
  S.fturn = (uint64_t*)(S.pbuf[1] + 4096);
  S.theta = (double*)(S.fturn + HALF);
  S.qr = (float*)(S.theta + HALF);
  S.pd = S.qr + G * D;
  S.lg = S.pd + 2 * G * kTile;
  S.stat = S.lg + G * kTile;
  S.tok = (int*)(S.stat + 2 * G);
  S.bars = (uint64_t*)(((uintptr_t)(S.tok + 2 * kTile) + 7) & ~(uintptr_t)7);
  S.tmem_slot = (uint32_t*)(S.bars + B_COUNT);
  const uint32_t bar0 = tc::smem_u32(S.bars);
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int t_begin = (int)((int64_t)blockIdx.x * P.n_tiles / gridDim.x);
  const int t_end = (int)((int64_t)(blockIdx.x + 1) * P.n_tiles / gridDim.x);
  const int n = t_end - t_begin;
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
  if (warp == kMmaWarp) tc::tmem_alloc(tc::smem_u32(S.tmem_slot), 512);
  for (int i = tid; i < HALF; i += kThreads) {
    const double th = pow(P.base, -2.0 * (double)i / (double)D);
    S.theta[i] = th;
    S.fturn[i] = __double2ull_rn(th / kTwoPi * 18446744073709551616.0);
  }
  // the p operand's unused rows (2G..15) stay zero
  for (int e = tid; e < 2 * 4096 / 4; e += kThreads) ((uint32_t*)S.pbuf[0])[e] = 0u;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *S.tmem_slot;

  if (warp == kLoadWarp) {
    // ======================= gather issuer (all 32 lanes) ======================
    // Lane l owns rows 4l..4l+3 of every tile: it resolves their token indices
    // and issues the gather4 copies of those rows for every k-block.
    UnitTileCursor cur;
    cur.start(P.seq_off, P.B, P.U, P.k, t_begin);
    UnitTileCursor ahead = cur;  // tile i+2 when loading Kc(i+2)
    auto issue = [&](const UnitTileCursor& c, int bi, const CUtensorMap* map, int b_full,
                     bool resolve) {
      int rows[4];
      int* tk = S.tok + bi * kTile;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int m = 4 * lane + j;
        int t;
        if (resolve) {
          const int64_t jj = (int64_t)c.slot * kTile + m;
          t = -1;
          if (jj < c.kb) {
            t = P.idx[((int64_t)c.b * P.U + c.u) * P.k + jj];
            if (t < 0 || t >= c.nb) {
              atomicOr(P.flags, FLAG_BAD_INDEX);
              t = -1;
            }
          }
          tk[m] = t;
        } else {
          t = tk[m];
        }
        // rows without a token read the sequence's first row; their weight is 0
        rows[j] = (int)(c.off + (t < 0 ? 0 : t));
      }
      if (lane == 0) tc::mbar_expect_tx(bar(b_full + bi), (uint32_t)kTile * P.r * 2);
      __syncwarp();
      const uint32_t dst0 = tc::smem_u32(S.buf[bi]) + (uint32_t)(lane >> 1) * 1024u +
                            (uint32_t)(lane & 1) * 512u;
      for (int kb = 0; kb < KB; ++kb)
        tc::tma_gather4(dst0 + kb * 16384u, map, kb * 64, rows[0], rows[1], rows[2], rows[3],
                        bar(b_full + bi));
    };
    for (int i = 0; i < 2 && i < n; ++i) {
      issue(ahead, i, &tmap_kc, B_KFULL, true);
      ahead.next();
    }
    bool ok = true;
    for (int i = 0; i < n && ok; ++i, cur.next()) {
      const int bi = i & 1;
      const uint32_t ph = ((uint32_t)i >> 1) & 1u;
      // the reconstruction is done with Kc(i): bring Vc(i) into the same buffer
      ok = __all_sync(0xffffffffu, tc::mbar_wait(bar(B_KDONE + bi), ph, P.flags));
      if (!ok) break;
      issue(cur, bi, &tmap_vc, B_VFULL, false);
      if (i + 2 < n) {
        // the value MMA is done with Vc(i): bring Kc(i+2)
        ok = __all_sync(0xffffffffu, tc::mbar_wait(bar(B_PDONE + bi), ph, P.flags));
        if (!ok) break;
        issue(ahead, bi, &tmap_kc, B_KFULL, true);
        ahead.next();
      }
    }
  } else if (warp == kMmaWarp) {
    // ======================= MMA issuer (lane 0) =======================
    if (lane == 0) {
      const uint32_t idesc_k = tc::idesc_bf16_f32(kTile, D);
      const uint32_t idesc_v = tc::idesc_bf16_f32_amn(128, kPRows);
      UnitTileCursor cur;
      cur.start(P.seq_off, P.B, P.U, P.k, t_begin);
      int cur_b = -1, cur_u = -1;
      uint32_t pk_phase = 0;
      bool ok = true;
      auto issue_pv = [&](int j) -> bool {
        const int bj = j & 1;
        const uint32_t ph = ((uint32_t)j >> 1) & 1u;
        if (!tc::mbar_wait(bar(B_PREADY + bj), ph, P.flags)) return false;
        if (!tc::mbar_wait(bar(B_VFULL + bj), ph, P.flags)) return false;
        if (!tc::mbar_wait(bar(B_TOFREE + bj), ph ^ 1u, P.flags)) return false;
        tc::fence_after_sync();
        const uint32_t v0 = tc::smem_u32(S.buf[bj]), p0 = tc::smem_u32(S.pbuf[bj]);
        for (int ch = 0; ch < n_chunks; ++ch) {
          const uint32_t d_tmem = tmem_base + o_col0 + (uint32_t)bj * o_cols + (uint32_t)ch * 16;
#pragma unroll
          for (int ks = 0; ks < kTile / 16; ++ks) {
            // A = Vc_tile^T: latent columns ch*128.. (MN), tokens ks*16.. (K)
            const uint64_t ad = tc::sdesc_mnmajor_sw128(
                v0 + (uint32_t)ch * 2 * 16384 + (uint32_t)(ks * 2) * 1024, 16384, 1024);
            // B = p rows (hi/lo per head), tokens ks*16..: K-major k-block ks/4
            const uint64_t bd =
                tc::sdesc_kmajor_sw128(p0 + (uint32_t)(ks >> 2) * 2048 + (uint32_t)(ks & 3) * 32);
            tc::mma_bf16(d_tmem, ad, bd, idesc_v, ks != 0);
          }
        }
        tc::mma_commit(bar(B_PDONE + bj));
        return true;
      };
      for (int i = 0; i < n && ok; ++i, cur.next()) {
        const int bi = i & 1;
        const uint32_t ph = ((uint32_t)i >> 1) & 1u;
        if (cur.b != cur_b || cur.u != cur_u) {
          // Pk_u of the new unit; the previous reconstruction must be done with Pk
          if (i > 0 &&
              !tc::mbar_wait(bar(B_KDONE + ((i - 1) & 1)), ((uint32_t)(i - 1) >> 1) & 1u,
                             P.flags)) {
            ok = false;
            break;
          }
          tc::mbar_expect_tx(bar(B_PK), pk_bytes);
          for (int kb = 0; kb < KB; ++kb)
            tc::tma_load_2d(tc::smem_u32(S.pk + (size_t)kb * D * 128), &tmap_pk, kb * 64,
                            cur.u * D, bar(B_PK));
          if (!tc::mbar_wait(bar(B_PK), pk_phase, P.flags)) {
            ok = false;
            break;
          }
          pk_phase ^= 1u;
          cur_b = cur.b;
          cur_u = cur.u;
        }
        if (!tc::mbar_wait(bar(B_KFULL + bi), ph, P.flags) ||
            !tc::mbar_wait(bar(B_TKFREE + bi), ph ^ 1u, P.flags)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t a0 = tc::smem_u32(S.buf[bi]), b0 = tc::smem_u32(S.pk);
        const uint32_t d_tmem = tmem_base + (uint32_t)bi * D;
        for (int kb = 0; kb < KB; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16(d_tmem, tc::sdesc_kmajor_sw128(a0 + kb * 16384 + 32 * k),
                         tc::sdesc_kmajor_sw128(b0 + kb * D * 128 + 32 * k), idesc_k,
                         (kb | k) != 0);
        tc::mma_commit(bar(B_KDONE + bi));
        if (i > 0 && !issue_pv(i - 1)) ok = false;
      }
      if (ok && n > 0) issue_pv(n - 1);
    }
  } else {
    // ======================= epilogue (warps 0-7) =======================
    const int quarter = warp & 3, half = warp >> 2;
    const int m = quarter * 32 + lane;  // token row = TMEM lane
    UnitTileCursor cur;
    cur.start(P.seq_off, P.B, P.U, P.k, t_begin);
    int cur_b = -1, cur_u = -1;
    for (int i = 0; i < n; ++i, cur.next()) {
      const int bi = i & 1;
      const uint32_t ph = ((uint32_t)i >> 1) & 1u;
      if (cur.b != cur_b || cur.u != cur_u) {
        // rotated queries of the unit's heads (angles reduced in fp64)
        const double qpos = P.q_pos ? (double)P.q_pos[cur.b] : (double)cur.nb;
        for (int e = tid; e < G * HALF; e += kEpiThreads) {
          const int g = e / HALF, ii = e % HALF;
          const __nv_bfloat16* qh = P.q + ((int64_t)cur.b * P.Hq + cur.u * G + g) * D;
          const double a = qpos * S.theta[ii];
          const double nt = rint(a * (1.0 / kTwoPi));
          float s, c;
          sincosf((float)fma(-nt, kTwoPi, a), &s, &c);
          const float x0 = __bfloat162float(qh[ii]), x1 = __bfloat162float(qh[ii + HALF]);
          S.qr[g * D + ii] = x0 * c - x1 * s;
          S.qr[g * D + ii + HALF] = x1 * c + x0 * s;
        }
        cur_b = cur.b;
        cur_u = cur.u;
        tc::named_sync(kEpiBar, kEpiThreads);
      }
      // ---- K_sel row m, pairs [half*QPAIRS, (half+1)*QPAIRS)
      const bool ok =
          __all_sync(0xffffffffu, tc::mbar_wait(bar(B_KDONE + bi), ph, P.flags));
      tc::fence_after_sync();
      // this row's token (resolved again here rather than read from the
      // gather warp's table, so no cross-warp ordering is needed)
      int t = -1;
      {
        const int64_t jj = (int64_t)cur.slot * kTile + m;
        if (jj < cur.kb) {
          t = P.idx[((int64_t)cur.b * P.U + cur.u) * P.k + jj];
          if (t < 0 || t >= cur.nb) t = -1;
        }
      }
      float dot[G];
#pragma unroll
      for (int g = 0; g < G; ++g) dot[g] = 0.f;
      if (ok) {
        const uint32_t row_addr =
            tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)bi * D;
        const uint32_t tu = (uint32_t)(t < 0 ? 0 : t);
#pragma unroll 1
        for (int i0 = half * QPAIRS; i0 < (half + 1) * QPAIRS; i0 += 16) {
          uint32_t v0[16], v1[16];
          tc::tmem_ld16(row_addr + i0, v0);
          tc::tmem_ld16(row_addr + HALF + i0, v1);
          tc::tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int ii = i0 + jj;
            const uint64_t F = S.fturn[ii];
            const uint32_t turn = __umulhi(tu, (uint32_t)F) + tu * (uint32_t)(F >> 32);
            float s, c;
            __sincosf((float)(int32_t)turn * (float)(kTwoPi / 4294967296.0), &s, &c);
            const float x0 = __uint_as_float(v0[jj]), x1 = __uint_as_float(v1[jj]);
            const float k0 = x0 * c - x1 * s;
            const float k1 = x1 * c + x0 * s;
#pragma unroll
            for (int g = 0; g < G; ++g)
              dot[g] = fmaf(S.qr[g * D + ii], k0, fmaf(S.qr[g * D + ii + HALF], k1, dot[g]));
          }
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) S.pd[(half * G + g) * kTile + m] = dot[g];
      tc::fence_before_sync();
      tc::named_sync(kEpiBar, kEpiThreads);
      if (tid == 0) tc::mbar_arrive(bar(B_TKFREE + bi));  // K_sel[bi] may be overwritten
      if (tid < kTile) {  // half 0: m == tid
#pragma unroll
        for (int g = 0; g < G; ++g)
          S.lg[g * kTile + tid] =
              t >= 0 ? (S.pd[g * kTile + tid] + S.pd[(G + g) * kTile + tid]) * P.scale : -INFINITY;
      }
      tc::named_sync(kEpiBar, kEpiThreads);
      // ---- softmax inside the tile: warp w takes head w
      if (warp < G) {
        const int g = warp;
        float v[4], mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          v[q] = S.lg[g * kTile + lane + 32 * q];
          mx = fmaxf(mx, v[q]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float p = v[q] == -INFINITY ? 0.f : expf(v[q] - mx);
          S.lg[g * kTile + lane + 32 * q] = p;
          sum += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
          S.stat[2 * g] = mx;
          S.stat[2 * g + 1] = sum;
        }
      }
      tc::named_sync(kEpiBar, kEpiThreads);
      // ---- p as bf16 hi/lo rows 2g, 2g+1 of the value MMA's B operand
      if (tid < kTile) {
        const int mm = tid;
        uint8_t* pb = S.pbuf[bi] + (mm >> 6) * 2048;
        const int col = mm & 63, chunk = col >> 3, within = col & 7;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float p = S.lg[g * kTile + mm];
          const __nv_bfloat16 hi = __float2bfloat16_rn(p);
          const __nv_bfloat16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
          const int r0 = 2 * g, r1 = 2 * g + 1;
          *(__nv_bfloat16*)(pb + (r0 >> 3) * 1024 + (r0 & 7) * 128 + ((chunk ^ (r0 & 7)) << 4) +
                            within * 2) = hi;
          *(__nv_bfloat16*)(pb + (r1 >> 3) * 1024 + (r1 & 7) * 128 + ((chunk ^ (r1 & 7)) << 4) +
                            within * 2) = lo;
        }
      }
      tc::fence_proxy_async_smem();
      tc::named_sync(kEpiBar, kEpiThreads);
      if (tid == 0) tc::mbar_arrive(bar(B_PREADY + bi));
      // ---- acc from TMEM: warp (quarter, half) reads latent columns half*128 + quarter*32 + lane
      const bool ok2 = __all_sync(0xffffffffu, tc::mbar_wait(bar(B_PDONE + bi), ph, P.flags));
      tc::fence_after_sync();
      if (ok2 && half < n_chunks) {
        uint32_t v[16];
        tc::tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + o_col0 +
                          (uint32_t)bi * o_cols + (uint32_t)half * 16,
                      v);
        tc::tmem_ld_wait();
        const int c = half * 128 + quarter * 32 + lane;
        if (c < P.r) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float* pp = P.part +
                        (((int64_t)cur.b * P.Hq + cur.u * G + g) * P.n_slots + cur.slot) *
                            (P.r + 2);
            pp[2 + c] = __uint_as_float(v[2 * g]) + __uint_as_float(v[2 * g + 1]);
          }
        }
      }
      if (tid < G) {
        float* pp = P.part +
                    (((int64_t)cur.b * P.Hq + cur.u * G + tid) * P.n_slots + cur.slot) * (P.r + 2);
        pp[0] = S.stat[2 * tid];
        pp[1] = S.stat[2 * tid + 1];
      }
      tc::fence_before_sync();
      tc::named_sync(kEpiBar, kEpiThreads);
      if (tid == 0) tc::mbar_arrive(bar(B_TOFREE + bi));
    }
  }
  tc::fence_before_sync();
  __syncthreads();
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

template <int G, int D>
size_t smem_bytes(int r) {
  const int KB = r / 64;
  return 1024 + (size_t)KB * D * 128 + 2 * (size_t)KB * 16384 + 2 * 4096 + 8 * (D / 2) * 2 +
         4 * (G * D + 2 * G * kTile + G * kTile + 2 * G + 2 * kTile) + 8 + 8 * B_COUNT + 16;
}

template <int G, int D>
cudaError_t launch_g_d(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = smem_bytes<G, D>(p.r);
  CUtensorMap tpk, tkc, tvc;
  if (!make_tmap_bf16_2d(&tpk, a.Pk, (uint64_t)p.U * D, (uint64_t)p.r, D, 64) ||
      !make_tmap_bf16_2d(&tkc, a.Kc, (uint64_t)p.N, (uint64_t)p.r, 1, 64) ||
      !make_tmap_bf16_2d(&tvc, a.Vc, (uint64_t)p.N, (uint64_t)p.r, 1, 64))
    return cudaErrorInvalidValue;
  static int done[kMaxDevices] = {};
  cudaError_t e = ensure_smem(attend_tc_kernel<G, D>, smem, done);
  if (e != cudaSuccess) return e;
  AttendTcParams P;
  P.q = (const __nv_bfloat16*)a.q;
  P.idx = a.idx;
  P.seq_off = a.seq_off;
  P.q_pos = a.q_pos;
  P.part = a.part;
  P.flags = a.flags;
  P.B = p.B;
  P.Hq = p.Hq;
  P.U = p.U;
  P.r = p.r;
  P.k = p.k;
  P.n_slots = p.splits;
  P.n_tiles = p.att_tiles;
  P.scale = p.scale;
  P.base = p.rope_base;
  const int grid = p.att_tiles < num_sms_att() ? p.att_tiles : num_sms_att();
  attend_tc_kernel<G, D><<<grid, kThreads, smem, s>>>(tpk, tkc, tvc, P);
  return cudaGetLastError();
}

}  // namespace

bool attend_tc_supported(const DecodePlan& p) {
  return p.dtype == SALSC_BF16 && p.r % 64 == 0 && p.r <= 256 && (p.d == 64 || p.d == 128) &&
         (p.G == 1 || p.G == 2 || p.G == 4 || p.G == 8) && p.N <= INT32_MAX;
}

cudaError_t launch_attend_tc(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  if (p.d == 128) {
    switch (p.G) {
      case 1: return launch_g_d<1, 128>(p, a, s);
      case 2: return launch_g_d<2, 128>(p, a, s);
      case 4: return launch_g_d<4, 128>(p, a, s);
      case 8: return launch_g_d<8, 128>(p, a, s);
    }
  } else {
    switch (p.G) {
      case 1: return launch_g_d<1, 64>(p, a, s);
      case 2: return launch_g_d<2, 64>(p, a, s);
      case 4: return launch_g_d<4, 64>(p, a, s);
      case 8: return launch_g_d<8, 64>(p, a, s);
    }
  }
  return cudaErrorInvalidConfiguration;
}

}  // namespace salsc
