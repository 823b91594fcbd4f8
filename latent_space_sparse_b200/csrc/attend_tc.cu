// attend_tc.cu -- selective reconstruction on tcgen05, RoPE, softmax and the
// latent value sum over the kept tokens (bf16 storage, d in {64, 128},
// r <= 256, G in {1, 2, 4, 8}).
//
// SALS technical framework, stages 3-4, with RoPE after reconstruction
// (abstract).  Work unit: a tile of 128 kept tokens of one selection unit
// (b, u).  For each tile:
//   1. gather the 128 latent key rows Kc_b[idx] into shared memory in the
//      128-byte-swizzled K-major layout (cp.async, 16 B per copy);
//   2. K_sel[128 x d] = Kc_tile . Pk_u^T on tcgen05 into TMEM (fp32; Pk_u is
//      loaded once per unit by TMA and stays in shared memory);
//   3. one thread per token row reads its K_sel row from TMEM, rotates each
//      pair (i, i+d/2) by t * base^(-2i/d) (angle reduced modulo 2 pi in fp64)
//      and dots it with each rotated query head of the unit;
//   4. softmax inside the tile (max m and normaliser l per head);
//   5. the tile's latent value rows Vc_b[idx] are gathered into the buffer the
//      MMA has finished with, and acc[r] = sum_t p_t Vc_b[t] is formed on the
//      CUDA cores in fp32.
// Each tile writes its own (m, l, acc) per head; the combine kernel merges
// the tiles of a unit and applies Pv_u^T.  The Kc gather of the next tile
// and the Vc gather of the current one overlap steps 3-4.
#include "tc.cuh"

namespace salsc {
namespace {

constexpr int kThreads = 128;
constexpr int kTile = 128;
constexpr double kTwoPi = 6.283185307179586476925286766559;

struct AttendTcParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* Kc;
  const __nv_bfloat16* Vc;
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte offset of element column c of row m in a [128 x r] tile stored as
// r/64 k-blocks of [128 rows x 128 B] with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz_offset(int m, int c) {
  const int kb = c >> 6, chunk = (c >> 3) & 7;
  return (uint32_t)(kb * 16384 + (m >> 3) * 1024 + (m & 7) * 128 + ((chunk ^ (m & 7)) << 4) +
                    (c & 7) * 2);
}

// Copy the rows tok[0..127] of `src` ([N][r] bf16, rows relative to `off`)
// into `buf`; rows with tok < 0 are zero-filled.  Thread e copies 16-byte
// chunks e, e+128, ...: consecutive threads cover consecutive bytes of a row.
__device__ __forceinline__ void gather_rows(uint8_t* buf, const __nv_bfloat16* src, int64_t off,
                                            const int* tok, int r) {
  const int cpr = r / 8;  // 16-byte chunks per row
  const uint32_t base = tc::smem_u32(buf);
  for (int e = threadIdx.x; e < kTile * cpr; e += kThreads) {
    const int m = e / cpr, cc = e % cpr;
    const int t = tok[m];
    const __nv_bfloat16* s = t >= 0 ? src + (off + t) * r + cc * 8 : src;
    cp_async16(base + swz_offset(m, cc * 8), s, t >= 0 ? 16u : 0u);
  }
  cp_async_commit();
}

template <int G, int D>
__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tmap_pk, const AttendTcParams P) {
  constexpr int HALF = D / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int KB = P.r / 64;
  const uint32_t pk_bytes = (uint32_t)KB * D * 128;
  const uint32_t buf_bytes = (uint32_t)KB * 16384;
  uint8_t* pk = smem;
  uint8_t* bufs[2] = {pk + pk_bytes, pk + pk_bytes + buf_bytes};
  double* theta = (double*)(pk + pk_bytes + 2 * buf_bytes);
  float* qr = (float*)(theta + HALF);     // [G][D]
  float* lg = qr + G * D;                 // [G][128]
  float* stat = lg + G * kTile;           // [G][2]
  int* tok = (int*)(stat + 2 * G);        // [2][128]
  uint64_t* bars = (uint64_t*)(((uintptr_t)(tok + 2 * kTile) + 7) & ~(uintptr_t)7);
  uint32_t* tmem_slot = (uint32_t*)(bars + 2);
  const uint32_t pk_full = tc::smem_u32(bars), mma_done = pk_full + 8;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int t_begin = (int)((int64_t)blockIdx.x * P.n_tiles / gridDim.x);
  const int t_end = (int)((int64_t)(blockIdx.x + 1) * P.n_tiles / gridDim.x);

  if (tid == 0) {
    tc::mbar_init(pk_full, 1);
    tc::mbar_init(mma_done, 1);
    tc::mbar_fence_init();
    tc::tma_prefetch_desc(&tmap_pk);
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(tmem_slot), 2 * D);
  for (int i = tid; i < HALF; i += kThreads) theta[i] = pow(P.base, -2.0 * (double)i / (double)D);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t idesc = tc::idesc_bf16_f32(kTile, D);

  // token index of every row of a tile (thread m = row m), then the gather
  auto prepare_tok = [&](const UnitTileCursor& c, int* tk) {
    const int64_t j = (int64_t)c.slot * kTile + tid;
    int t = -1;
    if (j < c.kb) {
      t = P.idx[((int64_t)c.b * P.U + c.u) * P.k + j];
      if (t < 0 || t >= c.nb) {
        atomicOr(P.flags, FLAG_BAD_INDEX);
        t = -1;
      }
    }
    tk[tid] = t;
    __syncthreads();
  };

  UnitTileCursor cur, nxt;
  cur.start(P.seq_off, P.B, P.U, P.k, t_begin);
  nxt = cur;
  if (t_begin < t_end) {
    prepare_tok(cur, tok);
    gather_rows(bufs[0], P.Kc, cur.off, tok, P.r);
  }
  int cur_b = -1, cur_u = -1;
  uint32_t pk_phase = 0, mma_phase = 0;
  bool ok = true;
  for (int i = 0; t_begin + i < t_end && ok; ++i, cur.next()) {
    const int bi = i & 1;
    int* tk = tok + bi * kTile;
    // ---- new unit: Pk_u by TMA, rotated queries of the unit's heads
    const bool new_unit = cur.b != cur_b || cur.u != cur_u;
    if (new_unit) {
      if (tid == 0) {
        tc::mbar_expect_tx(pk_full, pk_bytes);
        for (int kb = 0; kb < KB; ++kb)
          tc::tma_load_2d(tc::smem_u32(pk + (size_t)kb * D * 128), &tmap_pk, kb * 64, cur.u * D,
                          pk_full);
      }
      const double qpos = P.q_pos ? (double)P.q_pos[cur.b] : (double)cur.nb;
      for (int e = tid; e < G * HALF; e += kThreads) {
        const int g = e / HALF, ii = e % HALF;
        const __nv_bfloat16* qh = P.q + ((int64_t)cur.b * P.Hq + cur.u * G + g) * D;
        const double a = qpos * theta[ii];
        const double n = rint(a * (1.0 / kTwoPi));
        float s, c;
        sincosf((float)fma(-n, kTwoPi, a), &s, &c);
        const float x0 = __bfloat162float(qh[ii]), x1 = __bfloat162float(qh[ii + HALF]);
        qr[g * D + ii] = x0 * c - x1 * s;
        qr[g * D + ii + HALF] = x1 * c + x0 * s;
      }
      cur_b = cur.b;
      cur_u = cur.u;
    }
    // ---- Kc tile of this step has landed
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncthreads();
    // ---- K_sel = Kc_tile . Pk_u^T on the tensor cores
    if (tid == 0) {
      bool ready = true;
      if (new_unit) {
        ready = tc::mbar_wait(pk_full, pk_phase, P.flags);
        pk_phase ^= 1u;
      }
      if (ready) {
        tc::fence_after_sync();
        const uint32_t a0 = tc::smem_u32(bufs[bi]), b0 = tc::smem_u32(pk);
        const uint32_t d_tmem = tmem_base + (uint32_t)(bi * D);
        for (int kb = 0; kb < KB; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16(d_tmem, tc::sdesc_kmajor_sw128(a0 + kb * 16384 + 32 * k),
                         tc::sdesc_kmajor_sw128(b0 + kb * D * 128 + 32 * k), idesc,
                         (kb | k) != 0);
        tc::mma_commit(mma_done);
      } else {
        tc::mbar_arrive(mma_done);  // release the waiters; the flag reports the failure
      }
    }
    ok = __syncthreads_and(tc::mbar_wait(mma_done, mma_phase, P.flags));
    mma_phase ^= 1u;
    if (!ok) break;
    tc::fence_after_sync();
    // ---- the MMA is done with the Kc tile: gather the same rows of Vc into it,
    //      and the next tile's Kc rows into the other buffer
    gather_rows(bufs[bi], P.Vc, cur.off, tk, P.r);
    const bool has_next = t_begin + i + 1 < t_end;
    if (has_next) {
      nxt = cur;
      nxt.next();
      prepare_tok(nxt, tok + (bi ^ 1) * kTile);
      gather_rows(bufs[bi ^ 1], P.Kc, nxt.off, tok + (bi ^ 1) * kTile, P.r);
    }
    // ---- logits: one thread per kept token (TMEM lane = row)
    {
      const int t = tk[tid];
      float dot[G];
#pragma unroll
      for (int g = 0; g < G; ++g) dot[g] = 0.f;
      const uint32_t row_addr = tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(bi * D);
      const double pos = (double)(t < 0 ? 0 : t);
#pragma unroll 1
      for (int i0 = 0; i0 < HALF; i0 += 16) {
        uint32_t v0[16], v1[16];
        tc::tmem_ld16(row_addr + i0, v0);
        tc::tmem_ld16(row_addr + HALF + i0, v1);
        tc::tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int ii = i0 + jj;
          const double a = pos * theta[ii];
          const double n = rint(a * (1.0 / kTwoPi));
          float s, c;
          __sincosf((float)fma(-n, kTwoPi, a), &s, &c);
          const float x0 = __uint_as_float(v0[jj]), x1 = __uint_as_float(v1[jj]);
          const float k0 = x0 * c - x1 * s;
          const float k1 = x1 * c + x0 * s;
#pragma unroll
          for (int g = 0; g < G; ++g)
            dot[g] = fmaf(qr[g * D + ii], k0, fmaf(qr[g * D + ii + HALF], k1, dot[g]));
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) lg[g * kTile + tid] = t >= 0 ? dot[g] * P.scale : -INFINITY;
    }
    tc::fence_before_sync();
    __syncthreads();
    // ---- softmax inside the tile: warp w takes heads w, w+4, ...
    for (int g = warp; g < G; g += kThreads / 32) {
      float v[4], mx = -INFINITY;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[q] = lg[g * kTile + lane + 32 * q];
        mx = fmaxf(mx, v[q]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float p = v[q] == -INFINITY ? 0.f : expf(v[q] - mx);
        lg[g * kTile + lane + 32 * q] = p;
        sum += p;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        stat[2 * g] = mx;
        stat[2 * g + 1] = sum;
      }
    }
    // ---- the Vc rows have landed (the next tile's Kc group may still be in flight)
    if (has_next)
      cp_async_wait<1>();
    else
      cp_async_wait<0>();
    __syncthreads();
    // ---- acc[g][c] = sum_m p[g][m] * Vc_tile[m][c]; thread owns column pairs
    const uint8_t* vb = bufs[bi];
    for (int cp = tid; cp < P.r / 2; cp += kThreads) {
      const int c = 2 * cp;
      float acc0[G], acc1[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc0[g] = acc1[g] = 0.f;
#pragma unroll 4
      for (int m = 0; m < kTile; ++m) {
        const __nv_bfloat162 v = *(const __nv_bfloat162*)(vb + swz_offset(m, c));
        const float2 f = __bfloat1622float2(v);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float p = lg[g * kTile + m];
          acc0[g] = fmaf(p, f.x, acc0[g]);
          acc1[g] = fmaf(p, f.y, acc1[g]);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float* pp = P.part +
                    (((int64_t)cur.b * P.Hq + cur.u * G + g) * P.n_slots + cur.slot) * (P.r + 2);
        *(float2*)(pp + 2 + c) = make_float2(acc0[g], acc1[g]);
      }
    }
    if (tid < G) {
      float* pp = P.part +
                  (((int64_t)cur.b * P.Hq + cur.u * G + tid) * P.n_slots + cur.slot) * (P.r + 2);
      pp[0] = stat[2 * tid];
      pp[1] = stat[2 * tid + 1];
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, 2 * D);
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
cudaError_t launch_g_d(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  const int KB = p.r / 64;
  const size_t smem = 1024 + (size_t)KB * D * 128 + 2 * (size_t)KB * 16384 + 8 * (D / 2) +
                      4 * (G * D + G * kTile + 2 * G + 2 * kTile) + 64;
  CUtensorMap tpk;
  if (!make_tmap_bf16_2d(&tpk, a.Pk, (uint64_t)p.U * D, (uint64_t)p.r, D, 64))
    return cudaErrorInvalidValue;
  static int done[kMaxDevices] = {};
  cudaError_t e = ensure_smem(attend_tc_kernel<G, D>, smem, done);
  if (e != cudaSuccess) return e;
  AttendTcParams P;
  P.q = (const __nv_bfloat16*)a.q;
  P.Kc = (const __nv_bfloat16*)a.Kc;
  P.Vc = (const __nv_bfloat16*)a.Vc;
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
  attend_tc_kernel<G, D><<<grid, kThreads, smem, s>>>(tpk, P);
  return cudaGetLastError();
}

}  // namespace

bool attend_tc_supported(const DecodePlan& p) {
  return p.dtype == SALSC_BF16 && p.r % 64 == 0 && p.r <= 256 && (p.d == 64 || p.d == 128) &&
         (p.G == 1 || p.G == 2 || p.G == 4 || p.G == 8);
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
