/*
 * R-SWA CPU oracle, FP64.  TEST INFRASTRUCTURE ONLY.
 *
 * This file is the slow, plain, obviously-correct statement of what the
 * Reference Sliding Window Attention (R-SWA) decode path computes.  Only the
 * test-suite, the smoke check and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header, table or helper with the CUDA library and neither
 * side includes the other.
 *
 * Source of the method (cited by page title and section):
 *   [P5] "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" (gtnt.cn),
 *        §2.1 环形滑窗注意力 (ring sliding-window attention) and
 *        §2.3 反循环采样 (anti-loop n-gram sampling).
 *   [P1] "Kimi K3 et Unlimited OCR en tête des classements mondiaux ..." -- the
 *        one-paragraph statement of the R-SWA idea (attend to the whole source
 *        document, keep only the most recent generated tokens as working memory).
 *
 * Readings taken where the extracted text is garbled or silent (the HTML
 * extraction dropped '+', '=' and ',' in formulas):
 *   - cache size "prefill_len W"       is read as prefill_len + W;
 *   - "slot prefill_len ring_pos"       is read as slot = prefill_len + ring_pos;
 *   - "ring_pos (ring_pos 1) % W"       is read as ring_pos = (ring_pos + 1) % W;
 *   - ring_pos is 0 when steady state begins, so the first overwrite hits the
 *     oldest generated entry (the only start consistent with "keep the most
 *     recent generated tokens");
 *   - the new token's K/V is written before the attention, so it attends to
 *     itself (P5 §2.1 orders the overwrite before the attention pass);
 *   - prefill attention is causal (decoder LM) with no window;
 *   - n-gram bans count only n-grams lying fully inside the history window.
 *
 * Precision: every arithmetic step is double.  exp() is called, never rebuilt.
 *
 * Parity pins live in tests/ (float64 SDPA from torch, closed forms, brute
 * force over the union key set, the HF no-repeat-ngram processor).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENOMEM 2
#define ORC_ESTATE 4
#define ORC_EDATA 6

/* ------------------------------------------------------------------------ */
/* Softmax attention of one query over n keys.                               */
/*                                                                           */
/*   z_j = scale * <q, k_j>,  m = max_j z_j,                                 */
/*   out = sum_j exp(z_j - m) v_j / sum_j exp(z_j - m)                        */
/*                                                                           */
/* k and v rows are `stride` doubles apart.  The max shift changes nothing    */
/* mathematically; it only keeps exp() in range.                              */
/* ------------------------------------------------------------------------ */
int oracle_attend(const double *q, const double *k, const double *v, int64_t n,
                  int64_t stride, int d, double scale, double *out) {
  if (n < 1 || d < 1 || !q || !k || !v || !out) return ORC_EINVAL;
  double *z = (double *)malloc(sizeof(double) * (size_t)n);
  if (!z) return ORC_ENOMEM;
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) {
    double s = 0.0;
    for (int e = 0; e < d; ++e) s += q[e] * k[j * stride + e];
    z[j] = scale * s;
    if (z[j] > m) m = z[j];
  }
  double den = 0.0;
  for (int e = 0; e < d; ++e) out[e] = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    double p = exp(z[j] - m);
    den += p;
    for (int e = 0; e < d; ++e) out[e] += p * v[j * stride + e];
  }
  for (int e = 0; e < d; ++e) out[e] /= den;
  free(z);
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Prefill: full causal attention over the prompt of one sequence.           */
/* [P5 §2.1: the prefill segment keeps full attention; no token is dropped]  */
/*                                                                           */
/* q, k, v, out: [P][H][d] token-major.  Rows [row_lo, row_hi) are computed   */
/* for every head; query i attends keys 0..i.                                */
/* ------------------------------------------------------------------------ */
int oracle_prefill(const double *q, const double *k, const double *v,
                   int64_t P, int H, int d, double scale, int64_t row_lo,
                   int64_t row_hi, double *out) {
  if (P < 1 || H < 1 || d < 1 || row_lo < 0 || row_hi > P || row_lo > row_hi)
    return ORC_EINVAL;
  int64_t stride = (int64_t)H * d;
  int err = ORC_OK;
  int64_t nrow = row_hi - row_lo;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t it = 0; it < nrow * H; ++it) {
    int64_t i = row_lo + it / H;
    int h = (int)(it % H);
    int rc = oracle_attend(q + i * stride + (int64_t)h * d, k + (int64_t)h * d,
                           v + (int64_t)h * d, i + 1, stride, d, scale,
                           out + i * stride + (int64_t)h * d);
    if (rc != ORC_OK) err = rc;
  }
  return err;
}

/* ------------------------------------------------------------------------ */
/* The R-SWA cache of one (layer, sequence), simulated the way P5 §2.1        */
/* describes it, in three phases:                                            */
/*   1. prefill: every prompt token's K/V is kept (slots 0..P-1);            */
/*   2. warm-up: each generated token's K/V is appended while the cache      */
/*      holds fewer than P + W entries;                                      */
/*   3. steady state: each generated token overwrites slot P + ring_pos,     */
/*      then ring_pos advances by one modulo W.                              */
/* After the write the token attends to every entry the cache holds.         */
/* ------------------------------------------------------------------------ */
typedef struct oracle_ring {
  int64_t prefill_len; /* P */
  int64_t window;      /* W */
  int heads, head_dim;
  int64_t len;      /* entries currently held */
  int64_t ring_pos; /* next ring slot to overwrite once the cache is full */
  int64_t steps;    /* generated tokens written so far */
  int prefilled;
  double *k, *v; /* [P + W][H][d] */
} oracle_ring;

oracle_ring *oracle_ring_create(int64_t prefill_len, int64_t window, int heads,
                                int head_dim) {
  if (prefill_len < 0 || window < 1 || heads < 1 || head_dim < 1) return NULL;
  oracle_ring *r = (oracle_ring *)calloc(1, sizeof(oracle_ring));
  if (!r) return NULL;
  size_t n = (size_t)(prefill_len + window) * (size_t)heads * (size_t)head_dim;
  r->k = (double *)calloc(n, sizeof(double));
  r->v = (double *)calloc(n, sizeof(double));
  if (!r->k || !r->v) {
    free(r->k);
    free(r->v);
    free(r);
    return NULL;
  }
  r->prefill_len = prefill_len;
  r->window = window;
  r->heads = heads;
  r->head_dim = head_dim;
  return r;
}

void oracle_ring_destroy(oracle_ring *r) {
  if (!r) return;
  free(r->k);
  free(r->v);
  free(r);
}

/* Phase 1: keep the whole prompt.  k, v: [P][H][d]. */
int oracle_ring_prefill(oracle_ring *r, const double *k, const double *v) {
  if (!r || (r->prefill_len > 0 && (!k || !v))) return ORC_EINVAL;
  size_t n = (size_t)r->prefill_len * (size_t)r->heads * (size_t)r->head_dim;
  if (n) {
    memcpy(r->k, k, n * sizeof(double));
    memcpy(r->v, v, n * sizeof(double));
  }
  r->len = r->prefill_len;
  r->ring_pos = 0;
  r->steps = 0;
  r->prefilled = 1;
  return ORC_OK;
}

/* Phases 2 and 3 for one generated token, then attention over the cache.
 * q, k_new, v_new, out: [H][d].  slot_out / len_out (optional) receive the
 * slot written and the number of entries attended. */
int oracle_ring_step(oracle_ring *r, const double *q, const double *k_new,
                     const double *v_new, double scale, double *out,
                     int64_t *slot_out, int64_t *len_out) {
  if (!r || !q || !k_new || !v_new || !out) return ORC_EINVAL;
  if (!r->prefilled) return ORC_ESTATE;
  int64_t slot;
  if (r->len < r->prefill_len + r->window) {
    slot = r->len; /* warm-up: append */
    r->len += 1;
  } else {
    slot = r->prefill_len + r->ring_pos; /* steady state: overwrite */
    r->ring_pos = (r->ring_pos + 1) % r->window;
  }
  int64_t row = (int64_t)r->heads * r->head_dim;
  memcpy(r->k + slot * row, k_new, (size_t)row * sizeof(double));
  memcpy(r->v + slot * row, v_new, (size_t)row * sizeof(double));
  r->steps += 1;
  int err = ORC_OK;
#pragma omp parallel for schedule(static, 1)
  for (int h = 0; h < r->heads; ++h) {
    int64_t o = (int64_t)h * r->head_dim;
    int rc = oracle_attend(q + o, r->k + o, r->v + o, r->len, row, r->head_dim,
                           scale, out + o);
    if (rc != ORC_OK) err = rc;
  }
  if (slot_out) *slot_out = slot;
  if (len_out) *len_out = r->len;
  return err;
}

/* Copy of the cache as it stands: k_out, v_out [P + W][H][d]; entries past
 * `len` are zero until first written.  Returns the number of entries held. */
int64_t oracle_ring_snapshot(const oracle_ring *r, double *k_out,
                             double *v_out) {
  if (!r) return -1;
  size_t n = (size_t)(r->prefill_len + r->window) * (size_t)r->heads *
             (size_t)r->head_dim;
  if (k_out) memcpy(k_out, r->k, n * sizeof(double));
  if (v_out) memcpy(v_out, r->v, n * sizeof(double));
  return r->len;
}

int64_t oracle_ring_ring_pos(const oracle_ring *r) { return r ? r->ring_pos : -1; }
int64_t oracle_ring_len(const oracle_ring *r) { return r ? r->len : -1; }

/* ------------------------------------------------------------------------ */
/* No-repeat n-gram ban inside a sliding window.                             */
/* [P5 §2.3: only the window is checked; every token that would complete an  */
/*  n-gram already present in the window gets score -inf; defaults           */
/*  no_repeat_ngram_size 35, ngram_window 128]                               */
/*                                                                           */
/* Row r's history is history[r*hist_stride + 0 .. h-1], oldest first, with  */
/* h = hist_len[r] (or `window` when hist_len is NULL), h <= window.         */
/* The next token would form the n-gram (hist[h-n+1..h-1], x).  Every start  */
/* i in [0, h-n] whose (n-1)-gram hist[i..i+n-2] equals that prefix bans its */
/* follower x = hist[i+n-1].  With h < n nothing is banned.                  */
/*                                                                           */
/* A row whose length is outside [0, window] or whose history holds a token  */
/* outside [0, vocab) is left untouched and counted in the return value      */
/* (negated), so callers can tell "bad data" apart from success (0).         */
/* ------------------------------------------------------------------------ */
int oracle_ngram_ban(float *logits, int64_t ld, const int32_t *history,
                     int64_t hist_stride, const int32_t *hist_len, int rows,
                     int vocab, int n, int window) {
  if (rows < 0 || vocab < 1 || n < 1 || window < 0 || ld < vocab ||
      (rows > 0 && (!logits || !history)) || hist_stride < window)
    return ORC_EINVAL;
  int bad_rows = 0;
  for (int r = 0; r < rows; ++r) {
    const int32_t *hist = history + (int64_t)r * hist_stride;
    int h = hist_len ? hist_len[r] : window;
    if (h < 0 || h > window) {
      ++bad_rows;
      continue;
    }
    int ok = 1;
    for (int i = 0; i < h; ++i)
      if (hist[i] < 0 || hist[i] >= vocab) ok = 0;
    if (!ok) {
      ++bad_rows;
      continue;
    }
    if (h < n) continue;
    const int32_t *prefix = hist + (h - n + 1);
    for (int i = 0; i + n <= h; ++i) {
      int match = 1;
      for (int j = 0; j < n - 1; ++j)
        if (hist[i + j] != prefix[j]) {
          match = 0;
          break;
        }
      if (match) logits[(int64_t)r * ld + hist[i + n - 1]] = -INFINITY;
    }
  }
  return bad_rows ? -bad_rows : ORC_OK;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
