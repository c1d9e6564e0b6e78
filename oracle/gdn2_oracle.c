/*
 * gdn2_oracle.c -- fp64 CPU oracle for the Gated DeltaNet-2 forward operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA path and must never be used
 * as a fallback for it.
 *
 * What it computes (the plain definition; no blocking, fusion or reordering):
 *
 *   Gated Delta Rule-2, per (sequence, head), one token at a time.
 *   Source: page "Gated DeltaNet-2：将擦除与写入分开" (iplexlaw blog),
 *   section "在两个维度上独立控制": the erase gate b acts on the key channels and
 *   the write gate w on the value channels, giving e = b (.) k and z = w (.) v;
 *   the state is first decayed channel-wise, Sbar = D S_prev with
 *   D = diag(alpha_t) on the key axis, then read with the erase vector,
 *   r = Sbar^T e, then updated as S = Sbar + k (z - r)^T, and the query reads
 *   the UPDATED state.  The output scale is an explicit argument
 *   (o_t = scale * S_t^T q_t).
 *
 *   The decay is passed as its logarithm, lambda_t = log(alpha_t) <= 0, per
 *   (token, head, key channel); alpha_t = exp(lambda_t).
 *
 * Scalar-gate oracles, written separately from the generic one (page
 * "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention",
 * cere-bro blog, sections "TL;DR" and "The mechanism"; page 5 section
 * "在两个维度上独立控制"; the method reduces to KDA when both gates are the
 * same scalar and to Gated DeltaNet when the decay is a scalar as well):
 *
 *   KDA:       S = (I - beta k k^T) diag(alpha) S + beta k v^T
 *   GDN:       S = alpha (I - beta k k^T) S + beta k v^T
 *   DeltaNet:  S = (I - k k^T) S + k v^T           (beta = 1, alpha = 1)
 *
 * Layouts (all row-major, fp64):
 *   q, k, la, b : [T_total, H, dk]      v, w : [T_total, H, dv]
 *   o           : [T_total, H, dv]
 *   h0, hT      : [N, H, dk, dv]        (row = key channel, column = value channel)
 *   cu_seqlens  : [N + 1] int32, sequence n covers tokens [cu[n], cu[n+1]).
 * h0 may be NULL (zero initial state); hT may be NULL (not stored).
 *
 * Work is split over (sequence, head) pairs with POSIX threads; each pair is
 * computed by exactly one thread in the same sequential order, so results do
 * not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { MODE_GDN2 = 0, MODE_KDA = 1, MODE_GDN = 2, MODE_DELTANET = 3 };

typedef struct {
  int mode;
  int N, H, dk, dv;
  const int32_t* cu;
  const double *q, *k, *v, *la, *b, *w;
  /* scalar-gate inputs: beta [T_total, H]; alpha_s [T_total, H] (GDN) */
  const double *beta, *la_s;
  double scale;
  const double* h0;
  double* o;
  double* hT;
  int next; /* work counter (atomic) */
} job_t;

/* One (sequence, head) pair of the generic Gated Delta Rule-2 recurrence. */
static void gdn2_pair(const job_t* J, int n, int h, double* S, double* e, double* z, double* r) {
  const int H = J->H, dk = J->dk, dv = J->dv;
  const size_t SS = (size_t)dk * dv;
  if (J->h0)
    memcpy(S, J->h0 + ((size_t)n * H + h) * SS, SS * sizeof(double));
  else
    memset(S, 0, SS * sizeof(double));
  for (int t = J->cu[n]; t < J->cu[n + 1]; ++t) {
    const double* qt = J->q + ((size_t)t * H + h) * dk;
    const double* kt = J->k + ((size_t)t * H + h) * dk;
    const double* lat = J->la + ((size_t)t * H + h) * dk;
    const double* bt = J->b + ((size_t)t * H + h) * dk;
    const double* vt = J->v + ((size_t)t * H + h) * dv;
    const double* wt = J->w + ((size_t)t * H + h) * dv;
    /* erase vector on the key side, write vector on the value side */
    for (int c = 0; c < dk; ++c) e[c] = bt[c] * kt[c];
    for (int j = 0; j < dv; ++j) z[j] = wt[j] * vt[j];
    /* Sbar = diag(alpha_t) S : decay acts on rows (key channels) */
    for (int c = 0; c < dk; ++c) {
      const double a = exp(lat[c]);
      double* row = S + (size_t)c * dv;
      for (int j = 0; j < dv; ++j) row[j] *= a;
    }
    /* r = Sbar^T e */
    for (int j = 0; j < dv; ++j) r[j] = 0.0;
    for (int c = 0; c < dk; ++c) {
      const double ec = e[c];
      const double* row = S + (size_t)c * dv;
      for (int j = 0; j < dv; ++j) r[j] += row[j] * ec;
    }
    /* S = Sbar + k (z - r)^T */
    for (int c = 0; c < dk; ++c) {
      const double kc = kt[c];
      double* row = S + (size_t)c * dv;
      for (int j = 0; j < dv; ++j) row[j] += kc * (z[j] - r[j]);
    }
    /* o_t = scale * S_t^T q_t  (the query reads the updated state) */
    double* ot = J->o + ((size_t)t * H + h) * dv;
    for (int j = 0; j < dv; ++j) ot[j] = 0.0;
    for (int c = 0; c < dk; ++c) {
      const double qc = qt[c];
      const double* row = S + (size_t)c * dv;
      for (int j = 0; j < dv; ++j) ot[j] += row[j] * qc;
    }
    for (int j = 0; j < dv; ++j) ot[j] *= J->scale;
  }
  if (J->hT) memcpy(J->hT + ((size_t)n * H + h) * SS, S, SS * sizeof(double));
}

/* One (sequence, head) pair of a scalar-gate recurrence (KDA, GDN, DeltaNet).
 * Written from the scalar formulas directly: p = S^T k is the current read
 * along k, and the rank-1 correction beta k (v - p)^T replaces it. */
static void scalar_pair(const job_t* J, int n, int h, double* S, double* p) {
  const int H = J->H, dk = J->dk, dv = J->dv;
  const size_t SS = (size_t)dk * dv;
  if (J->h0)
    memcpy(S, J->h0 + ((size_t)n * H + h) * SS, SS * sizeof(double));
  else
    memset(S, 0, SS * sizeof(double));
  for (int t = J->cu[n]; t < J->cu[n + 1]; ++t) {
    const double* qt = J->q + ((size_t)t * H + h) * dk;
    const double* kt = J->k + ((size_t)t * H + h) * dk;
    const double* vt = J->v + ((size_t)t * H + h) * dv;
    double beta = 1.0;
    if (J->mode == MODE_KDA) {
      /* channel-wise decay first: diag(alpha) S */
      beta = J->beta[(size_t)t * H + h];
      const double* lat = J->la + ((size_t)t * H + h) * dk;
      for (int c = 0; c < dk; ++c) {
        const double a = exp(lat[c]);
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a;
      }
    } else if (J->mode == MODE_GDN) {
      /* one scalar decay for the whole state */
      beta = J->beta[(size_t)t * H + h];
      const double a = exp(J->la_s[(size_t)t * H + h]);
      for (size_t i = 0; i < SS; ++i) S[i] *= a;
    }
    /* p = S^T k ; S += beta k (v - p)^T  ==  (I - beta k k^T) S + beta k v^T */
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * kt[c];
      p[j] = acc;
    }
    for (int c = 0; c < dk; ++c)
      for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] += beta * kt[c] * (vt[j] - p[j]);
    double* ot = J->o + ((size_t)t * H + h) * dv;
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * qt[c];
      ot[j] = J->scale * acc;
    }
  }
  if (J->hT) memcpy(J->hT + ((size_t)n * H + h) * SS, S, SS * sizeof(double));
}

static void* worker(void* arg) {
  job_t* J = (job_t*)arg;
  const int dk = J->dk, dv = J->dv;
  double* S = (double*)malloc(sizeof(double) * ((size_t)dk * dv + 2 * (size_t)dk + 2 * (size_t)dv));
  if (!S) return (void*)1;
  double* e = S + (size_t)dk * dv;
  double* z = e + dk;
  double* r = z + dv;
  const int total = J->N * J->H;
  for (;;) {
    const int idx = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
    if (idx >= total) break;
    const int n = idx / J->H, h = idx % J->H;
    if (J->mode == MODE_GDN2)
      gdn2_pair(J, n, h, S, e, z, r);
    else
      scalar_pair(J, n, h, S, r);
  }
  free(S);
  return NULL;
}

static int run(job_t* J, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 1024) nthreads = 1024;
  J->next = 0;
  if (nthreads == 1) return worker(J) == NULL ? 0 : -1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
  if (!th) return -1;
  int launched = 0, rc = 0;
  for (int i = 0; i < nthreads; ++i) {
    if (pthread_create(&th[i], NULL, worker, J) != 0) break;
    ++launched;
  }
  if (launched == 0) rc = worker(J) == NULL ? 0 : -1;
  for (int i = 0; i < launched; ++i) {
    void* ret = NULL;
    pthread_join(th[i], &ret);
    if (ret != NULL) rc = -1;
  }
  free(th);
  return rc;
}

/* Generic Gated Delta Rule-2 recurrence.  Returns 0 on success. */
int oracle_gdn2_recurrent_f64(int N, int H, int dk, int dv, const int32_t* cu_seqlens,
                              const double* q, const double* k, const double* v,
                              const double* log_alpha, const double* b, const double* w,
                              double scale, const double* h0, double* o, double* hT,
                              int nthreads) {
  job_t J;
  memset(&J, 0, sizeof(J));
  J.mode = MODE_GDN2;
  J.N = N; J.H = H; J.dk = dk; J.dv = dv; J.cu = cu_seqlens;
  J.q = q; J.k = k; J.v = v; J.la = log_alpha; J.b = b; J.w = w;
  J.scale = scale; J.h0 = h0; J.o = o; J.hT = hT;
  return run(&J, nthreads);
}

/* KDA: scalar beta [T_total, H], channel-wise log-decay [T_total, H, dk]. */
int oracle_kda_f64(int N, int H, int dk, int dv, const int32_t* cu_seqlens,
                   const double* q, const double* k, const double* v,
                   const double* log_alpha, const double* beta, double scale,
                   const double* h0, double* o, double* hT, int nthreads) {
  job_t J;
  memset(&J, 0, sizeof(J));
  J.mode = MODE_KDA;
  J.N = N; J.H = H; J.dk = dk; J.dv = dv; J.cu = cu_seqlens;
  J.q = q; J.k = k; J.v = v; J.la = log_alpha; J.beta = beta;
  J.scale = scale; J.h0 = h0; J.o = o; J.hT = hT;
  return run(&J, nthreads);
}

/* Gated DeltaNet: scalar beta [T_total, H], scalar log-decay [T_total, H]. */
int oracle_gdn_f64(int N, int H, int dk, int dv, const int32_t* cu_seqlens,
                   const double* q, const double* k, const double* v,
                   const double* log_alpha_scalar, const double* beta, double scale,
                   const double* h0, double* o, double* hT, int nthreads) {
  job_t J;
  memset(&J, 0, sizeof(J));
  J.mode = MODE_GDN;
  J.N = N; J.H = H; J.dk = dk; J.dv = dv; J.cu = cu_seqlens;
  J.q = q; J.k = k; J.v = v; J.la_s = log_alpha_scalar; J.beta = beta;
  J.scale = scale; J.h0 = h0; J.o = o; J.hT = hT;
  return run(&J, nthreads);
}

/* Plain DeltaNet (beta = 1, no decay). */
int oracle_deltanet_f64(int N, int H, int dk, int dv, const int32_t* cu_seqlens,
                        const double* q, const double* k, const double* v, double scale,
                        const double* h0, double* o, double* hT, int nthreads) {
  job_t J;
  memset(&J, 0, sizeof(J));
  J.mode = MODE_DELTANET;
  J.N = N; J.H = H; J.dk = dk; J.dv = dv; J.cu = cu_seqlens;
  J.q = q; J.k = k; J.v = v;
  J.scale = scale; J.h0 = h0; J.o = o; J.hT = hT;
  return run(&J, nthreads);
}
