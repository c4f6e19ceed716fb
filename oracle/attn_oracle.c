/*
 * CPU ORACLE for block-diagonal (varlen) non-causal attention -- TEST
 * INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this file; the product path never does.
 *
 * What it computes (the plain definition, nothing faster):
 * for every segment s = [cu[s], cu[s+1]), head h, query row i in s, column d
 *
 *     a_ij     = scale * sum_e Q[i,h,e] K[j,h,e]           for j in s
 *     m_i      = max_j a_ij
 *     O[i,h,d] = sum_j exp(a_ij - m_i) V[j,h,d] / sum_j exp(a_ij - m_i)
 *
 * i.e. softmax(Q_s K_s^T * scale) V_s run independently per segment.  Source of
 * the method: issue #1545 (vllm.cpp) "Why this one is bad" (non-causal, H=16,
 * head_dim=96) and "The fix" (the block-diagonal mask is a set of per-segment
 * row slices mapped 1:1 onto the kernel); PR #1579 "Numerics, both halves"
 * (the flash rung is the same attention under a running softmax, differing
 * only in f32 partial-sum grouping).
 *
 * Arithmetic: every input element (bf16 bits, f32 or f64) is widened exactly
 * to double; all sums, the max, exp and the division are done in double; the
 * softmax is the two-pass form (max first, then sum), not an online one.
 * Packed layout [T, H, D]: element (t, h, d) at (t*H + h)*D + d.
 *
 * Shares no code with the CUDA path.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_BF16 = 0, OR_F32 = 1, OR_F64 = 2 };

static double widen(const void* p, int dtype, size_t i) {
  if (dtype == OR_BF16) {
    uint32_t b = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &b, 4);
    return (double)f;
  }
  if (dtype == OR_F32) return (double)((const float*)p)[i];
  return ((const double*)p)[i];
}

/* 0 when cu is a valid segmentation of T tokens into n segments. */
int oracle_check_seqlens(const int32_t* cu, int32_t n, int32_t T) {
  if (n < 0 || T < 0) return -1;
  if (n == 0) return T == 0 ? 0 : -1;
  if (cu[0] != 0 || cu[n] != T) return -1;
  for (int32_t s = 0; s < n; ++s)
    if (cu[s + 1] < cu[s]) return -1;
  return 0;
}

typedef struct {
  const void *q, *k, *v;
  int dtype;
  const int32_t* cu;
  int32_t n, T, H, D;
  double scale;
} problem_t;

/* One output row O[i, h, :] of the segment [a, b); logits/weights scratch has b-a doubles. */
static void one_row(const problem_t* P, int32_t a, int32_t b, int32_t i, int32_t h, double* w,
                    double* out_row) {
  const int32_t H = P->H, D = P->D;
  /* logits */
  double m = -INFINITY;
  for (int32_t j = a; j < b; ++j) {
    double dot = 0.0;
    for (int32_t e = 0; e < D; ++e)
      dot += widen(P->q, P->dtype, ((size_t)i * H + h) * D + e) *
             widen(P->k, P->dtype, ((size_t)j * H + h) * D + e);
    w[j - a] = P->scale * dot;
    if (w[j - a] > m) m = w[j - a];
  }
  /* weights and normaliser */
  double z = 0.0;
  for (int32_t j = a; j < b; ++j) {
    w[j - a] = exp(w[j - a] - m);
    z += w[j - a];
  }
  /* weighted sum of values */
  for (int32_t d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int32_t j = a; j < b; ++j) acc += w[j - a] * widen(P->v, P->dtype, ((size_t)j * H + h) * D + d);
    out_row[d] = acc / z;
  }
}

typedef struct {
  const problem_t* P;
  double* out;
  int64_t* next; /* shared work counter over (segment, head) pairs */
  int32_t max_len;
} full_job_t;

static void* full_worker(void* arg) {
  full_job_t* J = (full_job_t*)arg;
  const problem_t* P = J->P;
  double* w = (double*)malloc(sizeof(double) * (size_t)(J->max_len > 0 ? J->max_len : 1));
  if (!w) return (void*)1;
  const int64_t total = (int64_t)P->n * P->H;
  for (;;) {
    int64_t item = __sync_fetch_and_add(J->next, 1);
    if (item >= total) break;
    int32_t s = (int32_t)(item / P->H), h = (int32_t)(item % P->H);
    int32_t a = P->cu[s], b = P->cu[s + 1];
    for (int32_t i = a; i < b; ++i)
      one_row(P, a, b, i, h, w, J->out + ((size_t)i * P->H + h) * P->D);
  }
  free(w);
  return 0;
}

static int run_threads(void* (*fn)(void*), void* jobs, size_t job_size, int nthreads) {
  pthread_t th[512];
  int created[512];
  int rc = 0;
  for (int t = 1; t < nthreads; ++t)
    created[t] = pthread_create(&th[t], 0, fn, (char*)jobs + t * job_size) == 0;
  if (fn((char*)jobs) != 0) rc = -2;
  for (int t = 1; t < nthreads; ++t) {
    if (created[t]) {
      void* r = 0;
      pthread_join(th[t], &r);
      if (r) rc = -2;
    } else if (fn((char*)jobs + t * job_size) != 0) {
      rc = -2;
    }
  }
  return rc;
}

/* Full forward: out[T, H, D] (double).  Returns 0, or -1 on invalid arguments. */
int oracle_attn_fwd(const void* q, const void* k, const void* v, int dtype, double* out,
                    const int32_t* cu, int32_t n, int32_t T, int32_t H, int32_t D, double scale,
                    int nthreads) {
  if (oracle_check_seqlens(cu, n, T) != 0 || H < 1 || D < 1 || dtype < 0 || dtype > 2) return -1;
  if (T == 0) return 0;
  problem_t P = {q, k, v, dtype, cu, n, T, H, D, scale};
  int32_t max_len = 0;
  for (int32_t s = 0; s < n; ++s)
    if (cu[s + 1] - cu[s] > max_len) max_len = cu[s + 1] - cu[s];
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  int64_t next = 0;
  full_job_t jobs[512];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].P = &P;
    jobs[t].out = out;
    jobs[t].next = &next;
    jobs[t].max_len = max_len;
  }
  return run_threads(full_worker, jobs, sizeof(full_job_t), nthreads);
}

typedef struct {
  const problem_t* P;
  const int32_t *tok, *head;
  int32_t nrows;
  double* out;
  int64_t* next;
  int32_t max_len;
} rows_job_t;

static int32_t segment_of(const int32_t* cu, int32_t n, int32_t t) {
  /* largest s with cu[s] <= t and cu[s+1] > t */
  int32_t lo = 0, hi = n - 1;
  while (lo < hi) {
    int32_t mid = (lo + hi + 1) / 2;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  while (lo < n - 1 && cu[lo + 1] <= t) ++lo; /* skip empty segments */
  return lo;
}

static void* rows_worker(void* arg) {
  rows_job_t* J = (rows_job_t*)arg;
  const problem_t* P = J->P;
  double* w = (double*)malloc(sizeof(double) * (size_t)(J->max_len > 0 ? J->max_len : 1));
  if (!w) return (void*)1;
  for (;;) {
    int64_t r = __sync_fetch_and_add(J->next, 1);
    if (r >= J->nrows) break;
    int32_t t = J->tok[r], h = J->head[r];
    int32_t s = segment_of(P->cu, P->n, t);
    one_row(P, P->cu[s], P->cu[s + 1], t, h, w, J->out + (size_t)r * P->D);
  }
  free(w);
  return 0;
}

/* Selected output rows: out[r, :] = O[tok[r], head[r], :] for r < nrows. */
int oracle_attn_rows(const void* q, const void* k, const void* v, int dtype, const int32_t* tok,
                     const int32_t* head, int32_t nrows, double* out, const int32_t* cu, int32_t n,
                     int32_t T, int32_t H, int32_t D, double scale, int nthreads) {
  if (oracle_check_seqlens(cu, n, T) != 0 || H < 1 || D < 1 || dtype < 0 || dtype > 2) return -1;
  for (int32_t r = 0; r < nrows; ++r)
    if (tok[r] < 0 || tok[r] >= T || head[r] < 0 || head[r] >= H) return -1;
  problem_t P = {q, k, v, dtype, cu, n, T, H, D, scale};
  int32_t max_len = 0;
  for (int32_t s = 0; s < n; ++s)
    if (cu[s + 1] - cu[s] > max_len) max_len = cu[s + 1] - cu[s];
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  int64_t next = 0;
  rows_job_t jobs[512];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].P = &P;
    jobs[t].tok = tok;
    jobs[t].head = head;
    jobs[t].nrows = nrows;
    jobs[t].out = out;
    jobs[t].next = &next;
    jobs[t].max_len = max_len;
  }
  return run_threads(rows_worker, jobs, sizeof(rows_job_t), nthreads);
}

/* Attention probabilities of one (segment, head): probs[L, L], row i = softmax of query cu[s]+i. */
int oracle_attn_probs(const void* q, const void* k, int dtype, const int32_t* cu, int32_t n,
                      int32_t T, int32_t H, int32_t D, double scale, int32_t seg, int32_t h,
                      double* probs) {
  if (oracle_check_seqlens(cu, n, T) != 0 || seg < 0 || seg >= n || h < 0 || h >= H) return -1;
  int32_t a = cu[seg], b = cu[seg + 1], L = b - a;
  for (int32_t i = a; i < b; ++i) {
    double* w = probs + (size_t)(i - a) * L;
    double m = -INFINITY;
    for (int32_t j = a; j < b; ++j) {
      double dot = 0.0;
      for (int32_t e = 0; e < D; ++e)
        dot += widen(q, dtype, ((size_t)i * H + h) * D + e) * widen(k, dtype, ((size_t)j * H + h) * D + e);
      w[j - a] = scale * dot;
      if (w[j - a] > m) m = w[j - a];
    }
    double z = 0.0;
    for (int32_t j = 0; j < L; ++j) {
      w[j] = exp(w[j] - m);
      z += w[j];
    }
    for (int32_t j = 0; j < L; ++j) w[j] /= z;
  }
  return 0;
}
