// attend.cu -- selective reconstruction, RoPE and attention over the kept tokens.
//
// SALS technical framework, stages 3-4, and the abstract's point that RoPE
// is applied only after reconstruction:
//   K_t = RoPE(Kc_b[t] . Pk_u^T, t)          for the kept tokens t only
//   l_t = RoPE(q_h, q_pos) . K_t * scale,    p = softmax(l)
//   out_h = sum_t p_t (Vc_b[t] . Pv_u^T) = (sum_t p_t Vc_b[t]) . Pv_u^T
// The value projection is deferred to the combine kernel (exact in real
// arithmetic by associativity), so only latent rows of Vc are gathered.
//
// The kept tokens of one unit are split over `splits` CTAs; each writes the
// running maximum m, the normaliser l and the unnormalised latent
// accumulator acc[r] of every head of the unit; combine merges the splits
// and applies Pv_u^T.
#include "common.cuh"

namespace salsc {
namespace {

constexpr int kThreads = 256;
constexpr int kTok = 8;        // kept tokens per iteration
constexpr int kAccPer = 8;     // latent accumulator slots per thread (G*r <= 2048)
constexpr double kTwoPi = 6.283185307179586476925286766559;

// cos/sin of pos*theta with the angle formed and reduced modulo 2pi in fp64.
__device__ __forceinline__ void rope_cs(double pos, double theta, float& c, float& s) {
  const double a = pos * theta;
  const double n = rint(a * (1.0 / kTwoPi));
  const float rf = (float)fma(-n, kTwoPi, a);
  sincosf(rf, &s, &c);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
attend_simt_kernel(const T* __restrict__ q, const T* __restrict__ Kc, const T* __restrict__ Vc,
                   const T* __restrict__ Pk, const int32_t* __restrict__ idx,
                   const int64_t* __restrict__ seq_off, const int32_t* __restrict__ q_pos,
                   const int64_t* __restrict__ pos_off, float* __restrict__ part,
                   uint32_t* __restrict__ flags, int Hq, int U, int G,
                   int d, int r, int k, int chunk, int splits, float scale, double base) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int split = blockIdx.x;
  const int unit = blockIdx.y;
  const int b = unit / U, u = unit % U;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int half = d / 2;

  // shared layout
  double* theta = (double*)smem_raw;                      // [d/2]
  float* kc = (float*)(theta + kMaxHeadDim / 2);          // [kTok][r]
  float* vc = kc + kTok * r;                              // [kTok][r]
  float* ks = vc + kTok * r;                              // [kTok][d]
  float* qr = ks + kTok * kMaxHeadDim;                    // [G][d]
  float* lg = qr + G * d;                                 // [G][kTok]
  float* m_s = lg + G * kTok;                             // [G]
  float* l_s = m_s + G;                                   // [G]
  float* al_s = l_s + G;                                  // [G]
  int* tok = (int*)(al_s + G);                            // [kTok]
  T* pk = (T*)(((uintptr_t)(tok + kTok) + 15) & ~(uintptr_t)15);  // [d][r] = Pk_u

  const int64_t off = seq_off[b];
  const int64_t nb = seq_off[b + 1] - off;
  const int64_t kb = nb < k ? nb : k;
  const double qpos = q_pos ? (double)q_pos[b] : (double)nb;
  const double pos0 = pos_off ? (double)pos_off[b] : 0.0;  // position of the sequence's token 0
  allow_dependent_launch();
  grid_dependency_wait();  // the kept indices come from the previous kernel

  for (int i = tid; i < half; i += kThreads) theta[i] = pow(base, -2.0 * (double)i / (double)d);
  for (int e = tid; e < d * r; e += kThreads) pk[e] = Pk[(size_t)u * d * r + e];
  if (tid < G) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }
  __syncthreads();
  // rotated queries of the unit's heads
  for (int e = tid; e < G * half; e += kThreads) {
    const int g = e / half, i = e % half;
    const T* qh = q + ((size_t)b * Hq + u * G + g) * d;
    float c, s;
    rope_cs(qpos, theta[i], c, s);
    const float x0 = to_f32(qh[i]), x1 = to_f32(qh[i + half]);
    qr[g * d + i] = x0 * c - x1 * s;
    qr[g * d + i + half] = x1 * c + x0 * s;
  }
  float acc[kAccPer];
#pragma unroll
  for (int j = 0; j < kAccPer; ++j) acc[j] = 0.f;

  const int64_t j0 = (int64_t)split * chunk;
  const int64_t j1 = min(j0 + chunk, kb);
  const int32_t* uidx = idx + ((int64_t)b * U + u) * k;
  for (int64_t jt = j0; jt < j1; jt += kTok) {
    __syncthreads();
    if (tid < kTok) {
      int t = -1;
      if (jt + tid < j1) {
        t = uidx[jt + tid];
        if (t < -1 || t >= nb) {  // -1: no token (a slot threshold selection left empty)
          atomicOr(flags, FLAG_BAD_INDEX);
          t = -1;
        }
      }
      tok[tid] = t;
    }
    __syncthreads();
    for (int e = tid; e < kTok * r; e += kThreads) {
      const int j = e / r, c = e % r;
      const int t = tok[j];
      kc[e] = t >= 0 ? to_f32(Kc[(off + t) * r + c]) : 0.f;
      vc[e] = t >= 0 ? to_f32(Vc[(off + t) * r + c]) : 0.f;
    }
    __syncthreads();
    // reconstruct: ks[j][i] = sum_c kc[j][c] * Pk_u[i][c]; one warp per row i
    for (int i = warp; i < d; i += kThreads / 32) {
      float a[kTok];
#pragma unroll
      for (int j = 0; j < kTok; ++j) a[j] = 0.f;
      const T* prow = pk + (size_t)i * r;
      for (int c = lane; c < r; c += 32) {
        const float w = to_f32(prow[c]);
#pragma unroll
        for (int j = 0; j < kTok; ++j) a[j] = fmaf(kc[j * r + c], w, a[j]);
      }
#pragma unroll
      for (int j = 0; j < kTok; ++j) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a[j] += __shfl_xor_sync(0xffffffffu, a[j], o);
      }
      if (lane < kTok) {
        float v = a[0];
#pragma unroll
        for (int j = 1; j < kTok; ++j) v = lane == j ? a[j] : v;
        ks[lane * kMaxHeadDim + i] = v;
      }
    }
    __syncthreads();
    // RoPE at the token's own position
    for (int e = tid; e < kTok * half; e += kThreads) {
      const int j = e / half, i = e % half;
      const int t = tok[j];
      if (t < 0) continue;
      float c, s;
      rope_cs((double)t + pos0, theta[i], c, s);
      float* kr = ks + j * kMaxHeadDim;
      const float x0 = kr[i], x1 = kr[i + half];
      kr[i] = x0 * c - x1 * s;
      kr[i + half] = x1 * c + x0 * s;
    }
    __syncthreads();
    // logits
    for (int pidx = warp; pidx < G * kTok; pidx += kThreads / 32) {
      const int g = pidx / kTok, j = pidx % kTok;
      float a = 0.f;
      for (int i = lane; i < d; i += 32) a = fmaf(qr[g * d + i], ks[j * kMaxHeadDim + i], a);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) lg[g * kTok + j] = tok[j] >= 0 ? a * scale : -INFINITY;
    }
    __syncthreads();
    // online softmax
    if (tid < G) {
      const int g = tid;
      float mx = m_s[g];
      for (int j = 0; j < kTok; ++j) mx = fmaxf(mx, lg[g * kTok + j]);
      float alpha = 1.f, sum = 0.f;
      if (mx != -INFINITY) {
        alpha = m_s[g] == -INFINITY ? 0.f : expf(m_s[g] - mx);
        for (int j = 0; j < kTok; ++j) {
          const float l = lg[g * kTok + j];
          const float pj = l == -INFINITY ? 0.f : expf(l - mx);
          lg[g * kTok + j] = pj;
          sum += pj;
        }
      } else {
        for (int j = 0; j < kTok; ++j) lg[g * kTok + j] = 0.f;
      }
      l_s[g] = l_s[g] * alpha + sum;
      m_s[g] = mx;
      al_s[g] = alpha;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kAccPer; ++j) {
      const int e = tid + j * kThreads;
      if (e < G * r) {
        const int g = e / r, c = e % r;
        float a = acc[j] * al_s[g];
        for (int t = 0; t < kTok; ++t) a = fmaf(lg[g * kTok + t], vc[t * r + c], a);
        acc[j] = a;
      }
    }
  }
  __syncthreads();
  // partial results of this split
#pragma unroll
  for (int j = 0; j < kAccPer; ++j) {
    const int e = tid + j * kThreads;
    if (e < G * r) {
      const int g = e / r, c = e % r;
      float* pp = part + (((size_t)b * Hq + u * G + g) * splits + split) * part_row(r);
      pp[kPartAcc + c] = acc[j];
    }
  }
  if (tid < G) {
    float* pp = part + (((size_t)b * Hq + u * G + tid) * splits + split) * part_row(r);
    pp[0] = m_s[tid];
    pp[1] = l_s[tid];
  }
}

size_t attend_smem(const DecodePlan& p, size_t elem) {
  size_t sz = sizeof(double) * (kMaxHeadDim / 2) + sizeof(float) * (2 * kTok * p.r +
               kTok * kMaxHeadDim + p.G * p.d + p.G * kTok + 3 * p.G) + sizeof(int) * kTok;
  sz = (sz + 15) / 16 * 16 + elem * (size_t)p.r * p.d;
  return sz;
}

}  // namespace

cudaError_t launch_attend(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  if (p.attend_tc) return launch_attend_tc(p, a, s);
  if (p.G * p.r > kAccPer * kThreads) return cudaErrorInvalidConfiguration;
  dim3 grid(p.splits, p.B * p.U);
  if (p.dtype == SALSC_BF16) {
    static int done[kMaxDevices] = {};
    auto kern = attend_simt_kernel<__nv_bfloat16>;
    const size_t smem = attend_smem(p, 2);
    cudaError_t e = ensure_smem(kern, smem, done);
    if (e != cudaSuccess) return e;
    e = launch_k(kern, grid, dim3(kThreads), smem, s, true, (const __nv_bfloat16*)a.q,
                 (const __nv_bfloat16*)a.Kc, (const __nv_bfloat16*)a.Vc,
                 (const __nv_bfloat16*)a.Pk, (const int32_t*)a.idx, (const int64_t*)a.seq_off,
                 (const int32_t*)a.q_pos, a.pos_off, a.part, a.flags, p.Hq, p.U, p.G, p.d, p.r, p.k, p.chunk,
                 p.splits, p.scale, p.rope_base);
    if (e != cudaSuccess) return e;
  } else {
    static int done[kMaxDevices] = {};
    auto kern = attend_simt_kernel<float>;
    const size_t smem = attend_smem(p, 4);
    cudaError_t e = ensure_smem(kern, smem, done);
    if (e != cudaSuccess) return e;
    e = launch_k(kern, grid, dim3(kThreads), smem, s, true, (const float*)a.q,
                 (const float*)a.Kc, (const float*)a.Vc, (const float*)a.Pk, (const int32_t*)a.idx,
                 (const int64_t*)a.seq_off, (const int32_t*)a.q_pos, a.pos_off, a.part, a.flags, p.Hq, p.U,
                 p.G, p.d, p.r, p.k, p.chunk, p.splits, p.scale, p.rope_base);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace salsc
