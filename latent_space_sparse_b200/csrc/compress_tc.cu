// compress_tc.cu -- prefill low-rank projection on the tensor cores.
//
// SALS technical framework, stage 1: the keys (before RoPE) and values of the
// prompt are projected once into the latent space, Kc = K . Pk and
// Vc = V . Pv (n x hidden times hidden x r), accumulated in fp32 and rounded
// once to bf16.  At prefill sizes (65536 x 4096 x 512, twice) this is a dense
// contraction that is bound by tensor throughput, so it runs as a persistent,
// warp-specialised tcgen05 GEMM:
//
//   warp 0      TMA producer: per stage, MT boxes of X (128 rows x 64 K,
//               K-major, 128-byte swizzle) and BN/64 boxes of P (64 K-rows x
//               64 latent columns, MN-major, 128-byte swizzle) into a ring of
//               shared-memory stages;
//   warp 1      MMA issuer (one thread): tcgen05.mma kind::f16, M = 128 per
//               sub-tile, N = BN, K = 16, accumulating in TMEM; each stage is
//               released with tcgen05.commit when its MMAs are done;
//   warps 2-5   epilogue: TMEM -> registers (tcgen05.ld), one RNE rounding to
//               bf16, 16-byte stores of each output row.
//
// Tiles are (matrix, 128*MT rows, BN latent columns), with the latent
// column tile fastest so that the CTAs running at the same time share their
// rows of X through L2; each CTA walks tiles with a stride of the grid.  When
// TMEM holds two accumulators (MT*BN <= 256) the epilogue of one tile
// overlaps the main loop of the next.
//
// When r is a multiple of 256 the kernel runs on CTA pairs instead
// (compress_pair_kernel, a cluster of two): one tcgen05 MMA of M = 256 rows
// and N = 256 latent columns spans both CTAs (cta_group::2).  Each CTA loads
// its own 128 rows of X and its own 128 of the tile's 256 columns of P, so a
// CTA's stage is 32 KiB for 128 x 256 x 64 of MMA work (the one-CTA 256 x 256
// tile moves 64 KiB of stages for twice that work, and its shared-memory
// traffic, TMA writes plus MMA reads, is above what the SM serves), and its
// accumulator is 128 x 256: two fit in TMEM, so the epilogue of one tile
// overlaps the main loop of the next.  The first CTA of the pair issues the
// MMAs; both CTAs' copies complete on its stage barriers, and its commits
// arrive on the barriers of both.
#include "tc.cuh"

namespace salsc {
namespace {

constexpr int kBK = 64;           // K elements per stage: one 128-byte swizzle row
constexpr int kThreads = 192;     // 6 warps
constexpr int kEpiWarp0 = 2;
constexpr uint32_t kASub = 128u * 128u;  // one 128-row box of X: 16 KiB
constexpr uint32_t kBBox = 64u * 128u;   // one 64-row box of P: 8 KiB

struct CompressTcParams {
  __nv_bfloat16* Y[2];  // outputs of matrix 0 and 1, [n][r]
  int64_t n;            // rows of X
  int hid, r;
  int m_tiles, n_tiles;
  int64_t tiles;        // n_mats * m_tiles * n_tiles
};

template <int MT, int BN>
struct Cfg {
  static constexpr uint32_t kStage = MT * kASub + (BN / 64) * kBBox;
  static constexpr int kStages = (int)((200u * 1024u) / kStage) < 8 ? (int)((200u * 1024u) / kStage) : 8;
  static constexpr int kAcc = MT * BN;                   // TMEM columns of one tile
  static constexpr int kBufs = 2 * kAcc <= 512 ? 2 : 1;  // accumulators in TMEM
  static constexpr uint32_t kTmemCols = kBufs * kAcc <= 256 ? 256u : 512u;
  static constexpr size_t kSmem = (size_t)kStages * kStage + 1024;  // + alignment slack
  static_assert(kStages >= 2, "at least two stages");
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "N of one MMA");
  static_assert(kBufs * kAcc <= 512, "TMEM has 512 columns");
};

template <int MT, int BN>
__global__ void __launch_bounds__(kThreads, 1)
compress_tc_kernel(const __grid_constant__ CUtensorMap tx0, const __grid_constant__ CUtensorMap tp0,
                   const __grid_constant__ CUtensorMap tx1, const __grid_constant__ CUtensorMap tp1,
                   const CompressTcParams P) {
  using C = Cfg<MT, BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t s_bar[2 * S + 4];
  __shared__ uint32_t s_tmem;
  const uint32_t ring = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
  auto full = [&](int s) { return tc::smem_u32(&s_bar[s]); };
  auto empty = [&](int s) { return tc::smem_u32(&s_bar[S + s]); };
  auto tfull = [&](int a) { return tc::smem_u32(&s_bar[2 * S + a]); };
  auto tempty = [&](int a) { return tc::smem_u32(&s_bar[2 * S + 2 + a]); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int KB = (P.hid + kBK - 1) / kBK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tfull(a), 1);
      tc::mbar_init(tempty(a), 32 * (kThreads / 32 - kEpiWarp0));
    }
    tc::mbar_fence_init();
    tc::tma_prefetch_desc(&tx0);
    tc::tma_prefetch_desc(&tp0);
    tc::tma_prefetch_desc(&tx1);
    tc::tma_prefetch_desc(&tp1);
  }
  if (warp == 1) tc::tmem_alloc(tc::smem_u32(&s_tmem), C::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = s_tmem;

  // tile t -> (matrix, row block, latent column block), column block fastest
  auto decode = [&](int64_t t, int& mat, int64_t& m0, int& n0) {
    n0 = (int)(t % P.n_tiles) * BN;
    const int64_t rest = t / P.n_tiles;
    m0 = (rest % P.m_tiles) * (int64_t)(128 * MT);
    mat = (int)(rest / P.m_tiles);
  };

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < P.tiles && ok; t += gridDim.x) {
        int mat, n0;
        int64_t m0;
        decode(t, mat, m0, n0);
        const CUtensorMap* mx = mat ? &tx1 : &tx0;
        const CUtensorMap* mp = mat ? &tp1 : &tp0;
        for (int kb = 0; kb < KB; ++kb) {
          if (!tc::mbar_wait(empty(s), ph ^ 1u, nullptr)) {
            ok = false;
            break;
          }
          const uint32_t st = ring + (uint32_t)s * C::kStage;
          tc::mbar_expect_tx(full(s), C::kStage);
#pragma unroll
          for (int j = 0; j < MT; ++j)
            tc::tma_load_2d(st + (uint32_t)j * kASub, mx, kb * kBK, (int)(m0 + 128 * j), full(s));
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tc::tma_load_2d(st + MT * kASub + (uint32_t)j * kBBox, mp, n0 + 64 * j, kb * kBK,
                            full(s));
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32_bmn(128, BN);
      int s = 0;
      uint32_t ph = 0;
      int lt = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < P.tiles && ok; t += gridDim.x, ++lt) {
        const int a = C::kBufs == 2 ? (lt & 1) : 0;
        const uint32_t aph = (uint32_t)(C::kBufs == 2 ? (lt >> 1) : lt) & 1u;
        if (!tc::mbar_wait(tempty(a), aph ^ 1u, nullptr)) break;
        tc::fence_after_sync();
        const uint32_t d0 = tmem_base + (uint32_t)(a * C::kAcc);
        for (int kb = 0; kb < KB; ++kb) {
          if (!tc::mbar_wait(full(s), ph, nullptr)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t st = ring + (uint32_t)s * C::kStage;
          const uint32_t bst = st + MT * kASub;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // B: 16 K-rows of P starting at row 16k, BN latent columns in
            // 64-column boxes kBBox apart
            const uint64_t bd = tc::sdesc_mnmajor_sw128(bst + (uint32_t)k * 2048u, kBBox, 1024u);
#pragma unroll
            for (int j = 0; j < MT; ++j)
              tc::mma_bf16(d0 + (uint32_t)(j * BN),
                           tc::sdesc_kmajor_sw128(st + (uint32_t)j * kASub + 32u * k), bd, idesc,
                           (kb | k) != 0);
          }
          tc::mma_commit(empty(s));  // the stage is free once these MMAs are done
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) tc::mma_commit(tfull(a));
      }
    }
  } else {
    // ======================= epilogue (warps 2-5) =======================
    const int quarter = warp & 3;  // TMEM lanes 32*quarter.. are this warp's
    int lt = 0;
    for (int64_t t = blockIdx.x; t < P.tiles; t += gridDim.x, ++lt) {
      const int a = C::kBufs == 2 ? (lt & 1) : 0;
      const uint32_t aph = (uint32_t)(C::kBufs == 2 ? (lt >> 1) : lt) & 1u;
      if (!tc::mbar_wait(tfull(a), aph, nullptr)) break;
      tc::fence_after_sync();
      int mat, n0;
      int64_t m0;
      decode(t, mat, m0, n0);
      __nv_bfloat16* Y = P.Y[mat];
#pragma unroll 1
      for (int j = 0; j < MT; ++j) {
        const int64_t row = m0 + 128 * j + 32 * quarter + lane;
        const uint32_t tbase =
            tmem_base + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(a * C::kAcc + j * BN);
        __nv_bfloat16* yrow = Y + row * P.r + n0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v0[16], v1[16];
          tc::tmem_ld16(tbase + (uint32_t)c, v0);
          tc::tmem_ld16(tbase + (uint32_t)c + 16u, v1);
          tc::tmem_ld_wait();
          if (row < P.n) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const __nv_bfloat162 h0 =
                  __floats2bfloat162_rn(__uint_as_float(v0[2 * e]), __uint_as_float(v0[2 * e + 1]));
              const __nv_bfloat162 h1 =
                  __floats2bfloat162_rn(__uint_as_float(v1[2 * e]), __uint_as_float(v1[2 * e + 1]));
              w[e] = *reinterpret_cast<const uint32_t*>(&h0);
              w[8 + e] = *reinterpret_cast<const uint32_t*>(&h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(yrow + c);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
          }
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(tempty(a));
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int MT, int BN>
cudaError_t launch_tc(const CUtensorMap (&tx)[2], const CUtensorMap (&tp)[2],
                      const CompressTcParams& P, cudaStream_t s) {
  using C = Cfg<MT, BN>;
  static int done[kMaxDevices] = {};
  cudaError_t e = ensure_smem(compress_tc_kernel<MT, BN>, C::kSmem, done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int64_t grid = P.tiles < sms ? P.tiles : sms;
  compress_tc_kernel<MT, BN><<<(unsigned)grid, kThreads, C::kSmem, s>>>(tx[0], tp[0], tx[1], tp[1],
                                                                        P);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- CTA pairs

constexpr int kPairBN = 256;                       // latent columns of a pair's tile
constexpr uint32_t kPairStage = kASub + 2 * kBBox;  // 128 rows of X + 128 columns of P: 32 KiB
constexpr int kPairStages = 6;
constexpr uint32_t kPairCols = 2 * kPairBN;        // two 128 x 256 fp32 accumulators
constexpr size_t kPairSmem = (size_t)kPairStages * kPairStage + 1024;
constexpr int kEpiWarps = kThreads / 32 - kEpiWarp0;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
compress_pair_kernel(const __grid_constant__ CUtensorMap tx0,
                     const __grid_constant__ CUtensorMap tp0,
                     const __grid_constant__ CUtensorMap tx1,
                     const __grid_constant__ CUtensorMap tp1, const CompressTcParams P) {
  constexpr int S = kPairStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t s_bar[2 * S + 4];
  __shared__ uint32_t s_tmem;
  const uint32_t ring = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
  auto full = [&](int s) { return tc::smem_u32(&s_bar[s]); };
  auto empty = [&](int s) { return tc::smem_u32(&s_bar[S + s]); };
  auto tfull = [&](int a) { return tc::smem_u32(&s_bar[2 * S + a]); };
  auto tempty = [&](int a) { return tc::smem_u32(&s_bar[2 * S + 2 + a]); };
  // the same barrier in the pair's first CTA (cluster rank 0)
  auto lead = [&](uint32_t bar) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(bar));
    return r;
  };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const int64_t pair = blockIdx.x / 2, n_pairs = gridDim.x / 2;
  const int KB = (P.hid + kBK - 1) / kBK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tfull(a), 1);
      tc::mbar_init(tempty(a), 2 * kEpiWarps);  // one arrival per epilogue warp of each CTA
    }
    tc::mbar_fence_init();
    tc::tma_prefetch_desc(&tx0);
    tc::tma_prefetch_desc(&tp0);
    tc::tma_prefetch_desc(&tx1);
    tc::tma_prefetch_desc(&tp1);
  }
  if (warp == 1) tc::tmem_alloc_pair(tc::smem_u32(&s_tmem), kPairCols);
  tc::fence_before_sync();
  __syncthreads();
  // both CTAs' barriers are initialised and their TMEM allocated before
  // either CTA's copies, MMAs or arrivals reach the other
  cluster_arrive();
  cluster_wait();
  tc::fence_after_sync();
  const uint32_t tmem_base = s_tmem;

  // tile t -> (matrix, 256-row block, 256-column block), column block fastest
  auto decode = [&](int64_t t, int& mat, int64_t& m0, int& n0) {
    n0 = (int)(t % P.n_tiles) * kPairBN;
    const int64_t rest = t / P.n_tiles;
    m0 = (rest % P.m_tiles) * 256;
    mat = (int)(rest / P.m_tiles);
  };

  if (warp == 0) {
    // ============ TMA producer (both CTAs): this CTA's half of every stage
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int64_t t = pair; t < P.tiles && ok; t += n_pairs) {
        int mat, n0;
        int64_t m0;
        decode(t, mat, m0, n0);
        const CUtensorMap* mx = mat ? &tx1 : &tx0;
        const CUtensorMap* mp = mat ? &tp1 : &tp0;
        for (int kb = 0; kb < KB; ++kb) {
          if (!tc::mbar_wait(empty(s), ph ^ 1u, nullptr)) {
            ok = false;
            break;
          }
          // the first CTA's stage barrier counts the bytes of both halves
          if (rank == 0) tc::mbar_expect_tx(full(s), 2 * kPairStage);
          const uint32_t st = ring + (uint32_t)s * kPairStage;
          const uint32_t fb = lead(full(s));
          tc::tma_load_2d_pair(st, mx, kb * kBK, (int)(m0 + 128 * rank), fb);
#pragma unroll
          for (int j = 0; j < 2; ++j)
            tc::tma_load_2d_pair(st + kASub + (uint32_t)j * kBBox, mp,
                                 n0 + 128 * (int)rank + 64 * j, kb * kBK, fb);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ============ MMA issuer (first CTA, one thread)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32_bmn(256, kPairBN);
      int s = 0;
      uint32_t ph = 0;
      int lt = 0;
      bool ok = true;
      for (int64_t t = pair; t < P.tiles && ok; t += n_pairs, ++lt) {
        const int a = lt & 1;
        const uint32_t aph = (uint32_t)(lt >> 1) & 1u;
        // both CTAs' epilogues are done with accumulator a
        if (!tc::mbar_wait_cluster(tempty(a), aph ^ 1u, nullptr)) break;
        tc::fence_after_sync();
        const uint32_t d0 = tmem_base + (uint32_t)(a * kPairBN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!tc::mbar_wait(full(s), ph, nullptr)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t st = ring + (uint32_t)s * kPairStage;
          const uint32_t bst = st + kASub;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            tc::mma_bf16_pair(d0, tc::sdesc_kmajor_sw128(st + 32u * k),
                              tc::sdesc_mnmajor_sw128(bst + (uint32_t)k * 2048u, kBBox, 1024u),
                              idesc, (kb | k) != 0);
          tc::mma_commit_pair(empty(s), 0x3);  // the stage is free in both CTAs
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) tc::mma_commit_pair(tfull(a), 0x3);
      }
    }
  } else {
    // ============ epilogue (warps 2-5 of both CTAs): this CTA's 128 rows
    const int quarter = warp & 3;  // TMEM lanes 32*quarter.. are this warp's
    int lt = 0;
    for (int64_t t = pair; t < P.tiles; t += n_pairs, ++lt) {
      const int a = lt & 1;
      const uint32_t aph = (uint32_t)(lt >> 1) & 1u;
      if (!tc::mbar_wait(tfull(a), aph, nullptr)) break;
      tc::fence_after_sync();
      int mat, n0;
      int64_t m0;
      decode(t, mat, m0, n0);
      __nv_bfloat16* Y = P.Y[mat];
      const int64_t row = m0 + 128 * rank + 32 * quarter + lane;
      const uint32_t tbase =
          tmem_base + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(a * kPairBN);
      __nv_bfloat16* yrow = Y + row * P.r + n0;
#pragma unroll 1
      for (int c = 0; c < kPairBN; c += 32) {
        uint32_t v0[16], v1[16];
        tc::tmem_ld16(tbase + (uint32_t)c, v0);
        tc::tmem_ld16(tbase + (uint32_t)c + 16u, v1);
        tc::tmem_ld_wait();
        if (row < P.n) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const __nv_bfloat162 h0 =
                __floats2bfloat162_rn(__uint_as_float(v0[2 * e]), __uint_as_float(v0[2 * e + 1]));
            const __nv_bfloat162 h1 =
                __floats2bfloat162_rn(__uint_as_float(v1[2 * e]), __uint_as_float(v1[2 * e + 1]));
            w[e] = *reinterpret_cast<const uint32_t*>(&h0);
            w[8 + e] = *reinterpret_cast<const uint32_t*>(&h1);
          }
          uint4* dst = reinterpret_cast<uint4*>(yrow + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          tc::mbar_arrive(tempty(a));
        else
          tc::mbar_arrive_remote(lead(tempty(a)));
      }
    }
  }
  // every MMA into this CTA's TMEM has completed (its epilogue saw the last
  // tile's commit) and the other CTA is done with its arrivals
  tc::fence_before_sync();
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_relinquish_pair();
    tc::tmem_dealloc_pair(tmem_base, kPairCols);
  }
}

cudaError_t launch_pair(const CUtensorMap (&tx)[2], const CUtensorMap (&tp)[2],
                        const CompressTcParams& P, cudaStream_t s) {
  static int done[kMaxDevices] = {};
  cudaError_t e = ensure_smem(compress_pair_kernel, kPairSmem, done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  // as many pairs as can run at once (an SM pairs only within its GPC)
  static int max_pairs[kMaxDevices] = {};
  if (dev < kMaxDevices && !max_pairs[dev]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sms / 2 * 2));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kPairSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&n, compress_pair_kernel, &cfg)) != cudaSuccess) return e;
    max_pairs[dev] = n > 0 ? n : 1;
  }
  const int64_t cap = dev < kMaxDevices ? max_pairs[dev] : sms / 2;
  const int64_t pairs = P.tiles < cap ? P.tiles : cap;
  compress_pair_kernel<<<(unsigned)(2 * pairs), kThreads, kPairSmem, s>>>(tx[0], tp[0], tx[1],
                                                                         tp[1], P);
  return cudaGetLastError();
}

}  // namespace

bool compress_tc_supported(int hid, int r, salsc_dtype dt) {
  // TMA row strides must be multiples of 16 bytes; latent tiles of 64 columns
  return dt == SALSC_BF16 && hid % 8 == 0 && r % 64 == 0;
}

cudaError_t launch_compress_tc(const void* const X[2], const void* const Pm[2], void* const Y[2],
                               int n_mats, int64_t n, int hid, int r, cudaStream_t s) {
  CUtensorMap tx[2], tp[2];
  CompressTcParams P = {};
  const int BN = r % 256 == 0 ? 256 : (r % 128 == 0 ? 128 : 64);
  for (int i = 0; i < 2; ++i) {
    const int src = i < n_mats ? i : 0;  // unused slot: a copy of slot 0
    if (!make_tmap_bf16_2d(&tx[i], X[src], (uint64_t)n, (uint64_t)hid, 128, 64) ||
        !make_tmap_bf16_2d(&tp[i], Pm[src], (uint64_t)hid, (uint64_t)r, 64, 64))
      return cudaErrorInvalidValue;
    P.Y[i] = (__nv_bfloat16*)Y[src];
  }
  P.n = n;
  P.hid = hid;
  P.r = r;
  P.n_tiles = r / BN;
  if (BN == 256) {
    P.m_tiles = (int)((n + 255) / 256);
    P.tiles = (int64_t)n_mats * P.m_tiles * P.n_tiles;
    return launch_pair(tx, tp, P, s);
  }
  P.m_tiles = (int)((n + 127) / 128);
  P.tiles = (int64_t)n_mats * P.m_tiles * P.n_tiles;
  return BN == 128 ? launch_tc<1, 128>(tx, tp, P, s) : launch_tc<1, 64>(tx, tp, P, s);
}

}  // namespace salsc
