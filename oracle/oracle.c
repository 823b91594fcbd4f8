/*
 * oracle.c -- plain fp64 CPU oracle for SALS latent-space sparse decode.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * statement of what the decode path computes.  Only the test-suite, the
 * package smoke check and the benchmark's CPU-baseline leg may load it; the
 * CUDA library never links, includes or calls anything here, and nothing
 * here is shared with it (no header, table or helper).
 *
 * Source of the method: "SALS: Sparse Attention in Latent Space for KV cache
 * Compression" (arXiv 2510.24273v1), page section "technical framework"
 * (four stages: low-rank projection, sparse token selection in latent space
 * with RoPE-free query-key interaction, reconstruction of only the selected
 * tokens, standard attention on them) and the English abstract (RoPE must be
 * applied after reconstruction; selection is RoPE-free).  The attention
 * formula softmax(Q K^T / sqrt(d)) is as printed in the VL-Cache OpenReview
 * response to reviewer KiPr, "On Weakness 1".
 *
 * Readings of points the pages leave open (each one is listed again in the
 * design notes):
 *   - one projection per layer, Pk and Pv of shape hidden x r; KV head u
 *     uses rows u*d .. u*d+d-1 of it;
 *   - K is projected before RoPE; scoring uses the unrotated query;
 *   - under GQA the selection unit is the KV head; its score is the plain
 *     sum of the raw latent scores of its G query heads;
 *   - top-k keeps k_b = min(k, n_b) tokens; ties go to the lower index;
 *     unused slots hold -1;
 *   - threshold selection (select_mode 1, the alternative to Top-K the
 *     page's key designs name): of those k_b tokens, the ones whose unit
 *     score is below the threshold are dropped (a threshold alone is the
 *     case k >= n_b); a head with no token left outputs zeros;
 *   - RoPE is the rotate-half pairing (i, i + d/2), theta_i = base^(-2i/d),
 *     cached token t sits at position t, the query at q_pos[b] (default n_b);
 *   - softmax scale 1/sqrt(head_dim) unless given.
 *
 * Everything is computed literally in the order the method states it:
 * per-head latent query, per-head scores, group sum, exhaustive sort, full
 * reconstruction of each selected row with Pk and Pv, RoPE, softmax, sum.
 * No reassociation, no blocking, no deferral.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

typedef struct {
  int32_t batch;       /* B */
  int32_t n_q_heads;   /* Hq */
  int32_t n_kv_heads;  /* Hkv = number of selection units per sequence */
  int32_t head_dim;    /* d (even) */
  int32_t rank;        /* r, latent width */
  int32_t top_k;       /* k */
  const int64_t* seq_offsets; /* B+1 row offsets of each sequence in Kc/Vc */
  const int32_t* q_pos;       /* B query positions, or NULL for n_b */
  double rope_base;
  double softmax_scale;       /* 0 -> 1/sqrt(head_dim) */
  int32_t n_threads;          /* <= 0 -> 1 */
  int32_t select_mode;        /* 0: top-k; 1: top-k, then unit score >= select_threshold */
  double select_threshold;
} oracle_desc;

/* ---------------------------------------------------------------------- */
/* Rounding to the storage type: round-to-nearest, ties to even.          */
/* ---------------------------------------------------------------------- */

/* bfloat16 keeps 8 significant bits.  frexp gives x = m * 2^e with
 * 0.5 <= |m| < 1, so m * 2^8 is in [128, 256) and nearbyint (default mode:
 * nearest, ties to even) rounds it to the 8-bit significand. */
double oracle_round_bf16(double x) {
  if (x == 0.0 || isnan(x) || isinf(x)) return x;
  int e;
  double m = frexp(x, &e);
  if (e - 1 < -126) {
    /* subnormal range of bf16: fixed quantum 2^-133 */
    return ldexp(nearbyint(ldexp(x, 133)), -133);
  }
  double y = ldexp(nearbyint(ldexp(m, 8)), e - 8);
  if (fabs(y) > 3.3895313892515355e38) return copysign(INFINITY, x);
  return y;
}

void oracle_round_array(const double* x, double* y, int64_t n, int32_t to_bf16) {
  for (int64_t i = 0; i < n; ++i)
    y[i] = to_bf16 ? oracle_round_bf16(x[i]) : (double)(float)x[i];
}

/* ---------------------------------------------------------------------- */
/* Stage 1: low-rank projection  Y = X . P   (X: n x hid, P: hid x r)     */
/* ---------------------------------------------------------------------- */

typedef struct {
  const double* X;
  const double* P;
  double* Y;
  int64_t n;
  int32_t hid, r;
  int64_t row0, row1;
} compress_job;

static void* compress_worker(void* arg) {
  compress_job* j = (compress_job*)arg;
  for (int64_t i = j->row0; i < j->row1; ++i) {
    const double* x = j->X + i * j->hid;
    double* y = j->Y + i * j->r;
    for (int32_t c = 0; c < j->r; ++c) {
      double acc = 0.0;
      for (int32_t h = 0; h < j->hid; ++h) acc += x[h] * j->P[(int64_t)h * j->r + c];
      y[c] = acc;
    }
  }
  return NULL;
}

int oracle_compress(const double* X, const double* P, int64_t n, int32_t hid, int32_t r,
                    double* Y, int32_t n_threads) {
  if (!X || !P || !Y || n < 0 || hid < 1 || r < 1) return ORACLE_ERR_ARG;
  if (n_threads < 1) n_threads = 1;
  if (n_threads > n && n > 0) n_threads = (int32_t)n;
  compress_job* jobs = (compress_job*)calloc((size_t)n_threads, sizeof(compress_job));
  pthread_t* th = (pthread_t*)calloc((size_t)n_threads, sizeof(pthread_t));
  if (!jobs || !th) { free(jobs); free(th); return ORACLE_ERR_NOMEM; }
  for (int32_t w = 0; w < n_threads; ++w) {
    jobs[w] = (compress_job){X, P, Y, n, hid, r, n * w / n_threads, n * (w + 1) / n_threads};
    pthread_create(&th[w], NULL, compress_worker, &jobs[w]);
  }
  for (int32_t w = 0; w < n_threads; ++w) pthread_join(th[w], NULL);
  free(jobs);
  free(th);
  return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* RoPE, rotate-half pairing.  For i < d/2, with a = pos * base^(-2i/d):   */
/*   y_i       = x_i cos a - x_{i+d/2} sin a                               */
/*   y_{i+d/2} = x_{i+d/2} cos a + x_i sin a                               */
/* ---------------------------------------------------------------------- */

void oracle_rope(const double* x, int32_t d, double pos, double base, double* y) {
  int32_t half = d / 2;
  for (int32_t i = 0; i < half; ++i) {
    double theta = pow(base, -2.0 * (double)i / (double)d);
    double a = pos * theta;
    double c = cos(a), s = sin(a);
    double x0 = x[i], x1 = x[i + half];
    y[i] = x0 * c - x1 * s;
    y[i + half] = x1 * c + x0 * s;
  }
}

/* ---------------------------------------------------------------------- */
/* Decode                                                                  */
/* ---------------------------------------------------------------------- */

typedef struct {
  double s;
  int64_t t;
} scored_token;

/* Order: score descending, then token index ascending (ties -> lower t). */
static int cmp_scored(const void* a, const void* b) {
  const scored_token* x = (const scored_token*)a;
  const scored_token* y = (const scored_token*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  if (x->t < y->t) return -1;
  if (x->t > y->t) return 1;
  return 0;
}

typedef struct {
  const oracle_desc* D;
  const double *q, *Kc, *Vc, *Pk, *Pv;
  const int32_t* idx_in; /* non-NULL: attend over these (stages 3-4 only) */
  int32_t* idx_out;
  double* scores_out;
  double* probs_out;
  double* out;
  int64_t next_task; /* shared counter */
  pthread_mutex_t lock;
  int status;
} decode_ctx;

static int64_t take_task(decode_ctx* C) {
  pthread_mutex_lock(&C->lock);
  int64_t t = C->next_task++;
  pthread_mutex_unlock(&C->lock);
  return t;
}

static void set_status(decode_ctx* C, int st) {
  pthread_mutex_lock(&C->lock);
  if (C->status == ORACLE_OK) C->status = st;
  pthread_mutex_unlock(&C->lock);
}

/* One selection unit (sequence b, KV head u). */
static int decode_unit(decode_ctx* C, int32_t b, int32_t u) {
  const oracle_desc* D = C->D;
  const int32_t Hq = D->n_q_heads, U = D->n_kv_heads, d = D->head_dim, r = D->rank;
  const int32_t G = Hq / U, k = D->top_k;
  const int64_t off = D->seq_offsets[b];
  const int64_t nb = D->seq_offsets[b + 1] - off;
  const int64_t kb = nb < k ? nb : k;
  const double* Kc_b = C->Kc + off * r;
  const double* Vc_b = C->Vc + off * r;
  const double* Pk_u = C->Pk + (int64_t)u * d * r; /* d x r block of rows */
  const double* Pv_u = C->Pv + (int64_t)u * d * r;
  const double qpos = D->q_pos ? (double)D->q_pos[b] : (double)nb;
  const double scale = D->softmax_scale != 0.0 ? D->softmax_scale : 1.0 / sqrt((double)d);

  int64_t* sel = (int64_t*)malloc(sizeof(int64_t) * (size_t)(kb > 0 ? kb : 1));
  if (!sel) return ORACLE_ERR_NOMEM;
  int64_t n_sel = 0;

  if (!C->idx_in) {
    /* Stage 2: RoPE-free scoring in latent space, every cached token. */
    double* s_u = (double*)calloc((size_t)nb, sizeof(double));
    double* qlat = (double*)malloc(sizeof(double) * (size_t)r);
    scored_token* order = (scored_token*)malloc(sizeof(scored_token) * (size_t)nb);
    if (!s_u || !qlat || !order) {
      free(s_u); free(qlat); free(order); free(sel);
      return ORACLE_ERR_NOMEM;
    }
    for (int32_t g = 0; g < G; ++g) {
      const int32_t h = u * G + g; /* query head h belongs to unit h / G */
      const double* qh = C->q + ((int64_t)b * Hq + h) * d;
      /* latent query of head h: q_h . Pk_u  (1 x d times d x r) */
      for (int32_t c = 0; c < r; ++c) {
        double acc = 0.0;
        for (int32_t i = 0; i < d; ++i) acc += qh[i] * Pk_u[(int64_t)i * r + c];
        qlat[c] = acc;
      }
      /* s_h[t] = qlat . Kc_b[t]; the unit's score is the sum over its heads */
      for (int64_t t = 0; t < nb; ++t) {
        double acc = 0.0;
        for (int32_t c = 0; c < r; ++c) acc += qlat[c] * Kc_b[t * r + c];
        s_u[t] += acc;
      }
    }
    if (C->scores_out) {
      double* dst = C->scores_out + off * U + (int64_t)u * nb;
      memcpy(dst, s_u, sizeof(double) * (size_t)nb);
    }
    /* Top-k by exhaustive sort; with a threshold, the sorted prefix whose
     * scores reach it. */
    for (int64_t t = 0; t < nb; ++t) order[t] = (scored_token){s_u[t], t};
    qsort(order, (size_t)nb, sizeof(scored_token), cmp_scored);
    for (int64_t j = 0; j < kb; ++j) {
      if (D->select_mode == 1 && !(order[j].s >= D->select_threshold)) break;
      sel[n_sel++] = order[j].t;
    }
    int32_t* io = C->idx_out + ((int64_t)b * U + u) * k;
    for (int64_t j = 0; j < k; ++j) io[j] = j < n_sel ? (int32_t)sel[j] : -1;
    free(s_u);
    free(qlat);
    free(order);
  } else {
    const int32_t* ii = C->idx_in + ((int64_t)b * U + u) * k;
    for (int64_t j = 0; j < k; ++j) {
      if (ii[j] < 0) continue;
      if (ii[j] >= nb || n_sel >= kb) { free(sel); return ORACLE_ERR_ARG; }
      sel[n_sel++] = ii[j];
    }
  }

  /* Stage 3: reconstruct only the selected rows:
   *   K_sel[j] = Kc_b[t_j] . Pk_u^T,   V_sel[j] = Vc_b[t_j] . Pv_u^T       */
  double* Ksel = (double*)malloc(sizeof(double) * (size_t)(n_sel > 0 ? n_sel : 1) * d);
  double* Vsel = (double*)malloc(sizeof(double) * (size_t)(n_sel > 0 ? n_sel : 1) * d);
  double* Krot = (double*)malloc(sizeof(double) * (size_t)d);
  double* qrot = (double*)malloc(sizeof(double) * (size_t)d);
  double* logit = (double*)malloc(sizeof(double) * (size_t)(n_sel > 0 ? n_sel : 1));
  if (!Ksel || !Vsel || !Krot || !qrot || !logit) {
    free(Ksel); free(Vsel); free(Krot); free(qrot); free(logit); free(sel);
    return ORACLE_ERR_NOMEM;
  }
  for (int64_t j = 0; j < n_sel; ++j) {
    const double* kc = Kc_b + sel[j] * r;
    const double* vc = Vc_b + sel[j] * r;
    for (int32_t i = 0; i < d; ++i) {
      double ak = 0.0, av = 0.0;
      for (int32_t c = 0; c < r; ++c) {
        ak += kc[c] * Pk_u[(int64_t)i * r + c];
        av += vc[c] * Pv_u[(int64_t)i * r + c];
      }
      Ksel[j * d + i] = ak;
      Vsel[j * d + i] = av;
    }
    /* RoPE after reconstruction, at the token's own position. */
    oracle_rope(Ksel + j * d, d, (double)sel[j], D->rope_base, Krot);
    memcpy(Ksel + j * d, Krot, sizeof(double) * (size_t)d);
  }

  /* Stage 4: standard attention of each query head of the unit. */
  for (int32_t g = 0; g < G; ++g) {
    const int32_t h = u * G + g;
    const double* qh = C->q + ((int64_t)b * Hq + h) * d;
    oracle_rope(qh, d, qpos, D->rope_base, qrot);
    double mx = -INFINITY;
    for (int64_t j = 0; j < n_sel; ++j) {
      double acc = 0.0;
      for (int32_t i = 0; i < d; ++i) acc += qrot[i] * Ksel[j * d + i];
      logit[j] = acc * scale;
      if (logit[j] > mx) mx = logit[j];
    }
    double den = 0.0;
    for (int64_t j = 0; j < n_sel; ++j) {
      logit[j] = exp(logit[j] - mx);
      den += logit[j];
    }
    double* o = C->out + ((int64_t)b * Hq + h) * d;
    for (int32_t i = 0; i < d; ++i) o[i] = 0.0;
    for (int64_t j = 0; j < n_sel; ++j) {
      double p = logit[j] / den;
      for (int32_t i = 0; i < d; ++i) o[i] += p * Vsel[j * d + i];
      if (C->probs_out) C->probs_out[((int64_t)b * Hq + h) * k + j] = p;
    }
    if (C->probs_out)
      for (int64_t j = n_sel; j < k; ++j) C->probs_out[((int64_t)b * Hq + h) * k + j] = 0.0;
  }
  free(Ksel); free(Vsel); free(Krot); free(qrot); free(logit); free(sel);
  return ORACLE_OK;
}

static void* decode_worker(void* arg) {
  decode_ctx* C = (decode_ctx*)arg;
  const int64_t n_tasks = (int64_t)C->D->batch * C->D->n_kv_heads;
  for (;;) {
    int64_t task = take_task(C);
    if (task >= n_tasks) break;
    int st = decode_unit(C, (int32_t)(task / C->D->n_kv_heads), (int32_t)(task % C->D->n_kv_heads));
    if (st != ORACLE_OK) set_status(C, st);
  }
  return NULL;
}

static int check_desc(const oracle_desc* D) {
  if (!D || !D->seq_offsets) return ORACLE_ERR_ARG;
  if (D->batch < 1 || D->n_q_heads < 1 || D->n_kv_heads < 1 || D->head_dim < 2 ||
      D->rank < 1 || D->top_k < 1 || D->select_mode < 0 || D->select_mode > 1)
    return ORACLE_ERR_ARG;
  if (D->head_dim % 2 || D->n_q_heads % D->n_kv_heads) return ORACLE_ERR_ARG;
  if (D->seq_offsets[0] != 0) return ORACLE_ERR_ARG;
  for (int32_t b = 0; b < D->batch; ++b)
    if (D->seq_offsets[b + 1] <= D->seq_offsets[b]) return ORACLE_ERR_ARG;
  return ORACLE_OK;
}

static int run_decode(decode_ctx* C) {
  int32_t nt = C->D->n_threads < 1 ? 1 : C->D->n_threads;
  pthread_t* th = (pthread_t*)calloc((size_t)nt, sizeof(pthread_t));
  if (!th) return ORACLE_ERR_NOMEM;
  pthread_mutex_init(&C->lock, NULL);
  for (int32_t w = 0; w < nt; ++w) pthread_create(&th[w], NULL, decode_worker, C);
  for (int32_t w = 0; w < nt; ++w) pthread_join(th[w], NULL);
  pthread_mutex_destroy(&C->lock);
  free(th);
  return C->status;
}

/* Full decode: scores (optional, packed per (b,u): offset seq_offsets[b]*U
 * + u*n_b), top-k indices [B][U][k], probabilities over the selected tokens
 * in selection order (optional, [B][Hq][k]) and the output [B][Hq][d]. */
int oracle_decode(const oracle_desc* D, const double* q, const double* Kc, const double* Vc,
                  const double* Pk, const double* Pv, int32_t* idx_out, double* scores_out,
                  double* probs_out, double* out) {
  int st = check_desc(D);
  if (st) return st;
  if (!q || !Kc || !Vc || !Pk || !Pv || !idx_out || !out) return ORACLE_ERR_ARG;
  decode_ctx C;
  memset(&C, 0, sizeof C);
  C.D = D; C.q = q; C.Kc = Kc; C.Vc = Vc; C.Pk = Pk; C.Pv = Pv;
  C.idx_out = idx_out; C.scores_out = scores_out; C.probs_out = probs_out; C.out = out;
  return run_decode(&C);
}

/* Stages 3-4 only, over a supplied index set [B][U][k] (-1 = unused slot). */
int oracle_attend_given_idx(const oracle_desc* D, const double* q, const double* Kc,
                            const double* Vc, const double* Pk, const double* Pv,
                            const int32_t* idx, double* probs_out, double* out) {
  int st = check_desc(D);
  if (st) return st;
  if (!q || !Kc || !Vc || !Pk || !Pv || !idx || !out) return ORACLE_ERR_ARG;
  decode_ctx C;
  memset(&C, 0, sizeof C);
  C.D = D; C.q = q; C.Kc = Kc; C.Vc = Vc; C.Pk = Pk; C.Pv = Pv;
  C.idx_in = idx; C.probs_out = probs_out; C.out = out;
  return run_decode(&C);
}
