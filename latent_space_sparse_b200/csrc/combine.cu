// combine.cu -- merge of a unit's split partials and the deferred value
// projection.
//
// The attention kernels split the kept tokens of a selection unit (b, u)
// over several slots; slot s of query head h holds (m, l, acc[r]): the
// running maximum logit, the softmax normaliser and the unnormalised latent
// value sum of its tokens.  The merge is the exact online-softmax combination
//   M = max_s m_s,  w_s = e^{m_s - M},  L = sum_s w_s l_s,
//   acc = sum_s w_s acc_s / L,
// and the output is out_h = acc . Pv_u^T (SALS technical framework, stage 4:
// the value projection is applied once, after the weighted sum of latent
// rows, which is exact by associativity).
//
// Two kernels compute it.  combine_head_kernel (several query heads per unit,
// or a grid of several CTAs per SM): one warp per (sequence, head, 16 output
// rows), merging in registers with no block barrier after the dependency
// wait.  combine_kernel (otherwise, and for the shard merge below): CTA
// (b, u, slice) produces output rows slice*16 .. slice*16+15 of the G heads
// of unit u.  Its loads are whole-row bulk copies into shared memory, so that
// they are in flight together while the code stays short (the kernel runs
// once per SM and layer-step; every instruction it executes once is a cold
// instruction fetch).  In both, the 16 rows of Pv_u are loaded before the
// dependency wait (Pv is a weight, not an output of the attention kernel),
// the used partial rows after it.  Used slots: with the tensor-core
// attention, a slot holds a partial when a CTA's contiguous range of tiles
// starts there or the unit starts there, which follows from the tile
// partition; with the CUDA-core attention every slot of the unit is used.
// The sums run over slots in slot order, so the result is deterministic.
//
// Two more uses for token-sharded decode, both by combine_kernel: with
// part_out set, it stops after the merge and writes the merged (M, L, acc) of
// every head as one partial row (one CTA per unit, no projection); with the
// row strides set to (1, B*Hq), it merges one such row per shard (every slot
// used) and projects.
#include "tc.cuh"

namespace salsc {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 16;                      // output rows per CTA
constexpr int kTpr = kThreads / kRows;         // threads per output row
constexpr int kColsPer = kMaxRank / kThreads;  // latent columns per thread (r <= 512)
constexpr uint32_t kRowBuf = 72u * 1024u;      // most bytes of partial rows per batch
constexpr size_t kPairSmem = 100u * 1024u;     // dynamic shared memory that fits two CTAs per SM
constexpr int kMaxSegs = kMaxShardCandidates / 64 > 128 ? kMaxShardCandidates / 64 : 128;

struct CombineParams {
  const float* part;
  const void* Pv;
  void* out;
  const int64_t* seq_off;
  uint32_t* flags;
  int B, Hq, U, d, r, k, n_slots, chunk;
  int seg_grid, seg_tiles;  // tensor-core tile partition (seg_grid = 0: every slot used)
  int64_t bh_stride, slot_stride;  // partial row of (b, h, slot): (b*Hq + h)*bh_stride + slot*slot_stride
  float* part_out;  // non-null: write the merged partial row of every head, no projection
  int fixed_slots;  // > 0: every unit has this many slots (no tile count from the lengths)
  uint64_t* trace;  // traced step: this kernel's rows, or null
  uint32_t rowbuf;  // bytes of partial rows per batch (a multiple of one row per head)
};

// Used slots of unit (b, u), in slot order, into seg[]; by one whole warp,
// every lane returns the count.  Slots follow from the sequence lengths and
// the tile partition alone (inputs of the step, not outputs of the attention
// kernel), so they are found before the dependency wait.
__device__ __forceinline__ int used_slots(const CombineParams& P, int b, int u, int* seg) {
  const int lane = threadIdx.x % 32;
  // slots of unit (b, u) and, with the tile partition, the unit's first tile:
  // every lane reads one sequence's offsets, a warp scan sums the tiles
  int64_t before = 0;  // tiles of the sequences before b
  int tb = P.fixed_slots;
  for (int b0 = 0; b0 <= b && P.fixed_slots == 0; b0 += 32) {
    const int bb = b0 + lane;
    int64_t t = 0;
    if (bb <= b && bb < P.B) {
      const int64_t n2 = P.seq_off[bb + 1] - P.seq_off[bb];
      const int64_t k2 = n2 < P.k ? n2 : P.k;
      t = (k2 + P.chunk - 1) / P.chunk;
      if (bb == b) tb = (int)t;
    }
    int64_t x = bb < b ? t : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    before += x;
  }
  if (P.fixed_slots == 0) tb = __reduce_max_sync(0xffffffffu, tb);  // set by the lane of sequence b only
  const int64_t unit_tile0 = before * P.U + (int64_t)u * tb;
  int cnt = 0;
  for (int s0 = 0; s0 < tb; s0 += 32) {
    const int sl = s0 + lane;
    bool used = sl < tb;
    if (used && sl > 0 && P.seg_grid > 0) {
      // tile t starts the range of the CTA that holds it
      const int64_t t = unit_tile0 + sl, T = P.seg_tiles, gc = P.seg_grid;
      used = share_begin(share_of_tile(t, T, gc), T, gc) == t;
    }
    const uint32_t mk = __ballot_sync(0xffffffffu, used);
    if (used) seg[cnt + __popc(mk & ((1u << lane) - 1u))] = sl;
    cnt += __popc(mk);
  }
  return cnt;
}

template <typename T, int G>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const CombineParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int rowf = part_row(P.r);  // floats per partial row
  T* const pv_s = (T*)smem;                                                 // [16][r]
  float* const rows_s = (float*)(smem + (size_t)kRows * P.r * sizeof(T));  // batch of rows
  float* const acc_s = rows_s + P.rowbuf / 4;                               // [G][r]
  float* const w_s = acc_s + G * P.r;                                       // [G][32]
  __shared__ int s_seg[kMaxSegs];
  __shared__ int s_nseg, s_ok;
  __shared__ float s_scale[G], s_L[G], s_M[G];
  __shared__ __align__(8) uint64_t s_bar[2];
  const uint32_t bar_pv = tc::smem_u32(&s_bar[0]), bar_rows = tc::smem_u32(&s_bar[1]);

  const int n_slices = P.part_out ? 1 : P.d / kRows;
  const int slice = blockIdx.x % n_slices;
  const int bu = blockIdx.x / n_slices;
  const int b = bu / P.U, u = bu % P.U;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const uint32_t pv_bytes = (uint32_t)(kRows * P.r * sizeof(T));
  if (tid == 0) trace_stamp(P.trace, TRACE_START);
  if (tid == 0) {
    tc::mbar_init(bar_pv, 1);
    tc::mbar_init(bar_rows, 1);
    tc::mbar_fence_init();
    // the 16 rows of Pv_u: a weight, copied before the dependency wait
    if (!P.part_out) {
      tc::mbar_expect_tx(bar_pv, pv_bytes);
      tc::bulk_load(tc::smem_u32(pv_s),
                    (const T*)P.Pv + ((int64_t)u * P.d + (int64_t)slice * kRows) * P.r, pv_bytes,
                    bar_pv);
    }
  }
  allow_dependent_launch();
  // The used slots follow from the sequence lengths and the tile partition
  // alone (inputs of the step, not outputs of the attention kernel), so they
  // are found before the dependency wait.
  if (warp == 0) {
    const int cnt = used_slots(P, b, u, s_seg);
    if (lane == 0) s_nseg = cnt;
    if (lane < G) {
      s_M[lane] = -INFINITY;
      s_L[lane] = 0.f;
    }
  }
  grid_dependency_wait();  // the partials come from the attention kernel
  if (tid == 0) trace_stamp(P.trace, TRACE_WAITED);
  __syncthreads();
  const int nseg = s_nseg;
  // this thread's latent columns tid, tid + 256 for every head
  float acc[G][kColsPer];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int j = 0; j < kColsPer; ++j) acc[g][j] = 0.f;
  int bs = (int)(P.rowbuf / (uint32_t)(rowf * 4)) / G;  // slots per batch
  if (bs > 32) bs = 32;  // one weight per lane of a head's warp
  const float* part_u = P.part + ((int64_t)b * P.Hq + (int64_t)u * G) * P.bh_stride * rowf;
  uint32_t phase = 0;
  bool ok = true;
  for (int q0 = 0; q0 < nseg; q0 += bs, phase ^= 1u) {
    const int nq = nseg - q0 < bs ? nseg - q0 : bs;
    if (warp == 0) {
      // lanes copy rows e = (head e / nq, slot q0 + e % nq); one warp waits
      if (lane == 0) tc::mbar_expect_tx(bar_rows, (uint32_t)(G * nq * rowf * 4));
      __syncwarp();
      for (int e = lane; e < G * nq; e += 32) {
        const int g = e / nq, j = e % nq;
        tc::bulk_load(tc::smem_u32(rows_s + (size_t)e * rowf),
                      part_u + ((int64_t)g * P.bh_stride + s_seg[q0 + j] * P.slot_stride) * rowf,
                      (uint32_t)(rowf * 4), bar_rows);
      }
      ok = tc::mbar_wait(bar_rows, phase, P.flags) && ok;
    }
    __syncthreads();
    // weights of this batch: warp g, lane j
    if (warp < G) {
      const int g = warp;
      const float m = lane < nq ? rows_s[(size_t)(g * nq + lane) * rowf] : -INFINITY;
      const float l = lane < nq ? rows_s[(size_t)(g * nq + lane) * rowf + 1] : 0.f;
      float mb = m;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
      const float Mo = s_M[g], Mn = fmaxf(Mo, mb);
      const float sc = Mo == -INFINITY ? 0.f : expf(Mo - Mn);
      const float w = m == -INFINITY ? 0.f : expf(m - Mn);
      float wl = w * l;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) wl += __shfl_xor_sync(0xffffffffu, wl, o);
      if (lane < nq) w_s[g * 32 + lane] = w;
      __syncwarp();
      if (lane == 0) {
        s_scale[g] = sc;
        s_L[g] = s_L[g] * sc + wl;
        s_M[g] = Mn;
      }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kColsPer; ++j) {
      const int c = tid + j * kThreads;
      if (c < P.r) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float a = acc[g][j] * s_scale[g];
          for (int q = 0; q < nq; ++q)
            a = fmaf(w_s[g * 32 + q], rows_s[(size_t)(g * nq + q) * rowf + kPartAcc + c], a);
          acc[g][j] = a;
        }
      }
    }
    __syncthreads();  // the row buffer is refilled by the next batch
  }
  if (P.part_out) {
    // the merged partial of every head: (M, L) and the unnormalised sum
    float* po = P.part_out + ((int64_t)b * P.Hq + (int64_t)u * G) * rowf;
#pragma unroll
    for (int j = 0; j < kColsPer; ++j) {
      const int c = tid + j * kThreads;
      if (c < P.r) {
#pragma unroll
        for (int g = 0; g < G; ++g) po[(int64_t)g * rowf + kPartAcc + c] = acc[g][j];
      }
    }
    if (tid < G) {
      po[(int64_t)tid * rowf] = s_M[tid];
      po[(int64_t)tid * rowf + 1] = s_L[tid];
      po[(int64_t)tid * rowf + 2] = 0.f;
      po[(int64_t)tid * rowf + 3] = 0.f;
    }
    if (tid == 0) trace_stamp(P.trace, TRACE_END);
    return;
  }
#pragma unroll
  for (int j = 0; j < kColsPer; ++j) {
    const int c = tid + j * kThreads;
    if (c < P.r) {
#pragma unroll
      for (int g = 0; g < G; ++g) acc_s[g * P.r + c] = s_L[g] > 0.f ? acc[g][j] / s_L[g] : 0.f;
    }
  }
  if (warp == 0) {
    ok = tc::mbar_wait(bar_pv, 0, P.flags) && ok;
    if (lane == 0) s_ok = ok;
  }
  __syncthreads();
  // out row i = slice*16 + tid/16: the row's 16 threads take interleaved
  // groups of 4 latent columns, then add up with shuffles
  const int i = tid / kTpr, part = tid % kTpr;
  float o[G];
#pragma unroll
  for (int g = 0; g < G; ++g) o[g] = 0.f;
  const T* pvr = pv_s + (size_t)i * P.r;
#pragma unroll 2
  for (int c = part * 4; c < P.r; c += 4 * kTpr) {
    float f[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) f[e] = to_f32(pvr[c + e]);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 a4 = *(const float4*)(acc_s + g * P.r + c);
      o[g] = fmaf(a4.x, f[0], fmaf(a4.y, f[1], fmaf(a4.z, f[2], fmaf(a4.w, f[3], o[g]))));
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int off = kTpr / 2; off > 0; off >>= 1) o[g] += __shfl_xor_sync(0xffffffffu, o[g], off);
  if (part == 0 && s_ok) {
    T* out = (T*)P.out + ((int64_t)b * P.Hq + (int64_t)u * G) * P.d + slice * kRows + i;
#pragma unroll
    for (int g = 0; g < G; ++g) out[(int64_t)g * P.d] = from_f32<T>(o[g]);
  }
  if (tid == 0) trace_stamp(P.trace, TRACE_END);
}

// Low-latency merge: one warp per (sequence, query head, 16 output rows), eight
// such heads per CTA, all of one unit and one slice so that they share the
// CTA's 16 rows of Pv_u.  Everything that does not depend on the attention
// kernel (the Pv rows, the used slots) is done before the dependency wait;
// after it a warp runs alone, with no block barrier: it loads the rows of NB
// of its head's used slots at once (lane j holds latent columns 2j + 64i,
// +1), merges them in registers, then projects: each lane forms its columns'
// share of the 16 output dots, and a shuffle reduce-scatter leaves the sum of
// row i on lanes 2i, 2i+1.  Same merge as above, NB slots at a time in slot
// order.  NB > 1 takes the slot loads' latency once for several slots (few
// CTAs, each warp's chain is the kernel's time); NB = 1 keeps the registers,
// and so the CTAs resident per SM, for grids of several CTAs per SM.
constexpr int kSeqWarps = 8;
__device__ __forceinline__ float2 pv2_f32(const __nv_bfloat16* p) {
  return __bfloat1622float2(*(const __nv_bfloat162*)p);
}
__device__ __forceinline__ float2 pv2_f32(const float* p) { return *(const float2*)p; }
template <typename T, int G, int R64, int NB>  // R64 = r / 64, NB slots a batch
__global__ void __launch_bounds__(kSeqWarps * 32)
combine_head_kernel(const CombineParams P) {
  extern __shared__ __align__(16) uint8_t smem_pv[];
  T* const pv_s = (T*)smem_pv;  // [16][r]
  __shared__ int s_seg[kSeqWarps][kMaxSegs];
  const int n_slices = P.d / kRows;
  const int slice = blockIdx.x % n_slices;
  const int rest = blockIdx.x / n_slices;
  const int u = rest % P.U, hgroup = rest / P.U;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int head = hgroup * kSeqWarps + warp;  // (sequence, head of the unit)
  const int b = head / G, g = head % G;
  const int r = R64 * 64;
  if (tid == 0) trace_stamp(P.trace, TRACE_START);
  allow_dependent_launch();
  // the 16 rows of Pv_u (a weight) and the used slots, before the wait
  {
    const uint4* src = (const uint4*)((const T*)P.Pv + ((int64_t)u * P.d + (int64_t)slice * kRows) * r);
    uint4* dst = (uint4*)pv_s;
    const int n16 = kRows * r * (int)sizeof(T) / 16;
    for (int e = tid; e < n16; e += kSeqWarps * 32) dst[e] = src[e];
  }
  const int nseg = b < P.B ? used_slots(P, b, u, s_seg[warp]) : 0;
  __syncthreads();  // the Pv rows
  grid_dependency_wait();  // the partials come from the attention kernel
  if (tid == 0) trace_stamp(P.trace, TRACE_WAITED);
  if (b < P.B) {
    const int rowf = part_row(r);
    const float* part_h =
        P.part + ((int64_t)b * P.Hq + (int64_t)u * G + g) * P.bh_stride * rowf;
    float acc[2 * R64];
    float M = -INFINITY, L = 0.f;
#pragma unroll
    for (int j = 0; j < 2 * R64; ++j) acc[j] = 0.f;
    for (int q0 = 0; q0 < nseg; q0 += NB) {
      float m[NB], l[NB];
      float2 v[NB][R64];
#pragma unroll
      for (int q = 0; q < NB; ++q) {
        m[q] = -INFINITY;
        l[q] = 0.f;
#pragma unroll
        for (int i = 0; i < R64; ++i) v[q][i] = make_float2(0.f, 0.f);
        if (q0 + q < nseg) {
          const float* row = part_h + (int64_t)s_seg[warp][q0 + q] * P.slot_stride * rowf;
          m[q] = row[0];
          l[q] = row[1];
#pragma unroll
          for (int i = 0; i < R64; ++i) v[q][i] = *(const float2*)(row + kPartAcc + 2 * lane + 64 * i);
        }
      }
      float Mn = M;
#pragma unroll
      for (int q = 0; q < NB; ++q) Mn = fmaxf(Mn, m[q]);
      const float sc = M == -INFINITY ? 0.f : expf(M - Mn);
      L *= sc;
#pragma unroll
      for (int j = 0; j < 2 * R64; ++j) acc[j] *= sc;
#pragma unroll
      for (int q = 0; q < NB; ++q) {
        if (q0 + q >= nseg) break;  // the same for the whole warp
        const float w = m[q] == -INFINITY ? 0.f : expf(m[q] - Mn);
        L = fmaf(w, l[q], L);
#pragma unroll
        for (int i = 0; i < R64; ++i) {
          acc[2 * i] = fmaf(w, v[q][i].x, acc[2 * i]);
          acc[2 * i + 1] = fmaf(w, v[q][i].y, acc[2 * i + 1]);
        }
      }
      M = Mn;
    }
    // projection: o[i] = sum over this lane's columns of Pv row i . acc / L
    const float inv = L > 0.f ? 1.f / L : 0.f;
    float o[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) o[i] = 0.f;
#pragma unroll
    for (int c = 0; c < R64; ++c) {
      const float a0 = acc[2 * c] * inv, a1 = acc[2 * c + 1] * inv;
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const float2 pv = pv2_f32(pv_s + (size_t)i * r + 2 * lane + 64 * c);
        o[i] = fmaf(pv.x, a0, fmaf(pv.y, a1, o[i]));
      }
    }
    // reduce-scatter over the 32 lanes: after the step with offset 16 >> s,
    // a lane keeps the rows whose bit (3 - s) matches its lane bit (4 - s)
#pragma unroll
    for (int half = 8, off = 16; half >= 1; half >>= 1, off >>= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? o[i] : o[i + half];
        const float keep = upper ? o[i + half] : o[i];
        o[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
    // lanes 2i, 2i+1 hold row i's sums over lanes of equal bit 0: add the pair
    const float tot = o[0] + __shfl_xor_sync(0xffffffffu, o[0], 1);
    const int i = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                  ((lane >> 1) & 1);
    if ((lane & 1) == 0)
      ((T*)P.out)[((int64_t)b * P.Hq + (int64_t)u * G + g) * P.d + slice * kRows + i] =
          from_f32<T>(tot);
  }
  if (tid == 0) trace_stamp(P.trace, TRACE_END);
}

size_t combine_smem(const DecodePlan& p, uint32_t rowbuf) {
  const size_t elem = p.dtype == SALSC_BF16 ? 2 : 4;
  return (size_t)kRows * p.r * elem + rowbuf + sizeof(float) * (size_t)p.G * (p.r + 32);
}

// Most used slots of any unit: the CTAs of the tensor-core partition that meet
// the unit's tiles, or every slot.
int max_used_slots(const DecodePlan& p, const int64_t* seq_off_host, int seg_grid, int fixed) {
  if (fixed > 0) return fixed;
  if (seg_grid <= 0 || !seq_off_host || p.att_tiles <= 0) return p.splits;
  int most = 1;
  int64_t tile = 0;
  for (int b = 0; b < p.B; ++b) {
    const int64_t nb = seq_off_host[b + 1] - seq_off_host[b];
    const int64_t kb = nb < p.k ? nb : p.k;
    const int64_t tb = (kb + p.chunk - 1) / p.chunk;
    for (int u = 0; u < p.U; ++u, tile += tb) {
      // the unit's tiles meet the CTAs from its first tile's to its last
      // tile's (share_of_tile: the contiguous partition of the T tiles over
      // gc CTAs)
      const int64_t gc = seg_grid, T = p.att_tiles, t0 = tile;
      if (tb == 0) continue;
      int64_t n = share_of_tile(t0 + tb - 1, T, gc) - share_of_tile(t0, T, gc) + 1;
      if (n > tb) n = tb;  // a segment holds one tile at least
      if (n > most) most = (int)n;
    }
  }
  return most < p.splits ? most : p.splits;
}

// Bytes of partial rows per batch: every used slot of a unit at once, within
// kRowBuf.
uint32_t rowbuf_bytes(const DecodePlan& p, int maxseg) {
  const uint64_t row = (uint64_t)p.G * part_row(p.r) * 4;
  uint64_t want = row * (uint64_t)maxseg;
  if (want > kRowBuf) want = kRowBuf / row * row;
  if (want < row) want = row;
  return (uint32_t)want;
}

int num_sms_cb() {
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

template <typename T, int G, int R64>
cudaError_t launch_head(const CombineParams& P, const DecodePlan& p, cudaStream_t s) {
  // one head a unit: the grid is several CTAs per SM (the rule below), one
  // slot at a time; several heads: a few CTAs per SM at most, a batch of slots
  constexpr int NB = G == 1 ? 1 : 32 / R64;
  static int done[kMaxDevices] = {};
  const size_t smem = (size_t)kRows * p.r * sizeof(T);
  cudaError_t e = ensure_smem(combine_head_kernel<T, G, R64, NB>, smem, done);
  if (e != cudaSuccess) return e;
  const int64_t groups = ((int64_t)p.B * G + kSeqWarps - 1) / kSeqWarps;
  const dim3 grid((unsigned)((p.d / kRows) * p.U * groups));
  return launch_k(combine_head_kernel<T, G, R64, NB>, grid, dim3(kSeqWarps * 32), smem, s, true,
                  P);
}

template <typename T, int G>
cudaError_t launch_tg(const CombineParams& P, const DecodePlan& p, cudaStream_t s) {
  static int done[kMaxDevices] = {};
  // a warp per (sequence, head, slice): with several heads per unit always,
  // with one head per unit when the grid above would exceed two CTAs per SM
  if (!P.part_out && P.fixed_slots == 0 &&
      (G > 1 || (int64_t)p.B * p.U * (p.d / kRows) > 2 * (int64_t)num_sms_cb())) {
    if (p.r == 512) return launch_head<T, G, 8>(P, p, s);
    if (p.r == 256) return launch_head<T, G, 4>(P, p, s);
  }
  size_t smem = combine_smem(p, P.rowbuf);
  // A grid of at most two CTAs per SM asks for enough shared memory that no
  // more than two fit on an SM: the CTAs launched early, while the attention
  // kernel still holds most SMs, would otherwise pile up on the few free SMs
  // and run their share one after another.
  const int64_t ctas = (int64_t)p.B * p.U * (P.part_out ? 1 : p.d / kRows);
  if (ctas <= 2 * (int64_t)num_sms_cb() && smem < kPairSmem) smem = kPairSmem;
  cudaError_t e = ensure_smem(combine_kernel<T, G>, smem, done);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)(p.B * p.U * (P.part_out ? 1 : p.d / kRows)));
  return launch_k(combine_kernel<T, G>, grid, dim3(kThreads), smem, s, true, P);
}

template <typename T>
cudaError_t launch_t(const CombineParams& P, const DecodePlan& p, cudaStream_t s) {
  switch (p.G) {
    case 1: return launch_tg<T, 1>(P, p, s);
    case 2: return launch_tg<T, 2>(P, p, s);
    case 4: return launch_tg<T, 4>(P, p, s);
    case 8: return launch_tg<T, 8>(P, p, s);
  }
  return cudaErrorInvalidConfiguration;
}

}  // namespace

bool combine_supported(const DecodePlan& p) {
  // one row of partials per head fits the row buffer; the used slots of a unit
  // fit the segment list
  return (p.G == 1 || p.G == 2 || p.G == 4 || p.G == 8) && p.r <= kMaxRank && p.d % kRows == 0 &&
         (uint32_t)(p.G * part_row(p.r) * 4) <= kRowBuf && p.splits <= kMaxSegs;
}

namespace {

CombineParams base_params(const DecodePlan& p, const DecodeArgs& a) {
  CombineParams P;
  P.part = a.part;
  P.Pv = a.Pv;
  P.out = a.out;
  P.seq_off = a.seq_off;
  P.flags = a.flags;
  P.B = p.B;
  P.Hq = p.Hq;
  P.U = p.U;
  P.d = p.d;
  P.r = p.r;
  P.k = p.k;
  P.n_slots = p.splits;
  P.chunk = p.chunk;
  P.seg_grid = p.attend_tc ? attend_tc_grid(p) : 0;
  P.seg_tiles = p.att_tiles;
  P.bh_stride = p.splits;
  P.slot_stride = 1;
  P.part_out = nullptr;
  P.fixed_slots = 0;
  P.trace = trace_of(a, 4);
  return P;
}

cudaError_t launch_params(CombineParams P, const DecodePlan& p, const int64_t* seq_off_host,
                          cudaStream_t s) {
  P.rowbuf = rowbuf_bytes(p, max_used_slots(p, seq_off_host, P.seg_grid, P.fixed_slots));
  return p.dtype == SALSC_BF16 ? launch_t<__nv_bfloat16>(P, p, s) : launch_t<float>(P, p, s);
}

}  // namespace

cudaError_t launch_combine(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  if (p.att_cluster > 0) return cudaSuccess;  // the attention kernel merged the partials
  if (!combine_supported(p)) return cudaErrorInvalidConfiguration;
  return launch_params(base_params(p, a), p, a.seq_off_host, s);
}

cudaError_t launch_combine_partial(const DecodePlan& p, const DecodeArgs& a, float* part_out,
                                   cudaStream_t s) {
  if (p.att_cluster > 0 || !combine_supported(p)) return cudaErrorInvalidConfiguration;
  CombineParams P = base_params(p, a);
  P.part_out = part_out;
  return launch_params(P, p, a.seq_off_host, s);
}

cudaError_t launch_shard_merge(const DecodePlan& p, const float* part_all, int n_shards,
                               const void* Pv, void* out, uint32_t* flags, cudaStream_t s) {
  if (n_shards < 1 || n_shards > kMaxSegs) return cudaErrorInvalidValue;
  DecodeArgs a{};
  a.part = (float*)part_all;
  a.Pv = Pv;
  a.out = out;
  a.flags = flags;
  CombineParams P = base_params(p, a);
  // slot s of head (b, h) is shard s's merged row: part_all[s][b][h]
  P.n_slots = n_shards;
  P.seg_grid = 0;  // every slot used
  P.fixed_slots = n_shards;
  P.bh_stride = 1;
  P.slot_stride = (int64_t)p.B * p.Hq;
  return launch_params(P, p, nullptr, s);
}

}  // namespace salsc
