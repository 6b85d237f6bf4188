/*
 * oracle.c -- plain fp64 CPU oracle for exact scaled dot-product attention
 * forward.  TEST INFRASTRUCTURE ONLY (see oracle.h): nothing in the product
 * library links or calls this file.
 *
 * The code follows the definition step by step, without blocking, fusion or
 * reordering beyond what each cited passage states.  Threads split the list
 * of query rows; each row is computed independently in double precision.
 */
#include "oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* bf16 bit pattern -> double, exact (bf16 is the top half of an fp32). */
static double bf16_bits_to_double(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* double -> nearest bf16 value (via fp32, then round-to-nearest-even on the
 * upper 16 bits), returned as a double.  Models a bf16 store. */
static double round_to_bf16(double x) {
  float f = (float)x;
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ---- softmax / logsumexp ([CIA] 3.1) ---------------------------------- */

void oracle_softmax(const double* x, int64_t n, double* out) {
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) if (x[j] > m) m = x[j];
  double l = 0.0;
  for (int64_t j = 0; j < n; ++j) { out[j] = exp(x[j] - m); l += out[j]; }
  for (int64_t j = 0; j < n; ++j) out[j] /= l;
}

double oracle_logsumexp(const double* x, int64_t n) {
  if (n <= 0) return -INFINITY;
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) if (x[j] > m) m = x[j];
  if (m == -INFINITY) return -INFINITY;
  double l = 0.0;
  for (int64_t j = 0; j < n; ++j) l += exp(x[j] - m);
  return m + log(l);
}

/* ---- RoPE ([TAB] 3.1 rotation matrix; [CIA] 3.5 frequencies/pairing) --- */

/* Rotate one row of length d in place at position pos. */
static void rope_row(double* row, int64_t d, int64_t pos, double base,
                     int pairing) {
  const int64_t half = d / 2;
  for (int64_t i = 0; i < half; ++i) {
    const double theta = pow(base, -2.0 * (double)i / (double)d);
    const double ang = (double)pos * theta;
    const double c = cos(ang), s = sin(ang);
    const int64_t ia = pairing ? 2 * i : i;
    const int64_t ib = pairing ? 2 * i + 1 : i + half;
    const double a = row[ia], b = row[ib];
    row[ia] = a * c - b * s;
    row[ib] = a * s + b * c;
  }
}

void oracle_rope(const uint16_t* x, double* out, int64_t B, int64_t H,
                 int64_t N, int64_t d, double base, int64_t pos_offset,
                 int pairing) {
  for (int64_t bh = 0; bh < B * H; ++bh)
    for (int64_t t = 0; t < N; ++t) {
      const uint16_t* src = x + (bh * N + t) * d;
      double* dst = out + (bh * N + t) * d;
      for (int64_t c = 0; c < d; ++c) dst[c] = bf16_bits_to_double(src[c]);
      rope_row(dst, d, pos_offset + t, base, pairing);
    }
}

/* ---- masks ([AME] 5 causal; [CIA] 3.2 padding, self-test 5 alignment) -- */

int64_t oracle_visible_prefix(int64_t i, int64_t Nq, int64_t Nk, int causal,
                              int64_t key_len) {
  int64_t L = key_len < 0 ? 0 : (key_len > Nk ? Nk : key_len);
  if (causal) {
    const int64_t c = i + (Nk - Nq) + 1; /* keys j <= i + (Nk - Nq) */
    if (c < L) L = c;
  }
  return L < 0 ? 0 : L;
}

/* Key position of query row i.  align 0: the Nq rows are the last Nq
 * positions of the Nk keys, p = i + (Nk - Nq).  align 1: they are the last
 * Nq positions of the sequence's own L = key_len keys, p = i + (L - Nq)
 * ([CIA] self-test 5: t new tokens after a cache of `len` keys see the
 * cache and a lower triangle among themselves, per sequence). */
int64_t oracle_query_position(int64_t i, int64_t Nq, int64_t Nk,
                              int64_t key_len, int align) {
  const int64_t L = key_len < 0 ? 0 : (key_len > Nk ? Nk : key_len);
  return i + ((align ? L : Nk) - Nq);
}

/* [AME] 11: with a window w > 0, key j is legal only if |p - j| < w, where
 * p is the query's key position; causal adds j <= p; key_len adds j < L. */
void oracle_visible_range_ex(int64_t i, int64_t Nq, int64_t Nk, int causal,
                             int64_t key_len, int64_t window, int align,
                             int64_t* lo, int64_t* hi) {
  const int64_t L = key_len < 0 ? 0 : (key_len > Nk ? Nk : key_len);
  const int64_t p = oracle_query_position(i, Nq, Nk, key_len, align);
  int64_t h = L, l = 0;
  if (causal && p + 1 < h) h = p + 1;
  if (window > 0) {
    if (p - window + 1 > l) l = p - window + 1;
    if (p + window < h) h = p + window;
  }
  if (h < l) h = l;
  *lo = l;
  *hi = h;
}

void oracle_visible_range(int64_t i, int64_t Nq, int64_t Nk, int causal,
                          int64_t key_len, int64_t window, int64_t* lo,
                          int64_t* hi) {
  oracle_visible_range_ex(i, Nq, Nk, causal, key_len, window, 0, lo, hi);
}

void oracle_kv_tiles(int64_t Nq, int64_t Nk, int causal, int64_t key_len,
                     int64_t Br, int64_t Bc, int64_t qt, int64_t* first,
                     int64_t* last, int64_t* count) {
  oracle_kv_tiles_ex(Nq, Nk, causal, key_len, 0, 0, Br, Bc, qt, first, last,
                     count);
}

void oracle_kv_tiles_window(int64_t Nq, int64_t Nk, int causal,
                            int64_t key_len, int64_t window, int64_t Br,
                            int64_t Bc, int64_t qt, int64_t* first,
                            int64_t* last, int64_t* count) {
  oracle_kv_tiles_ex(Nq, Nk, causal, key_len, window, 0, Br, Bc, qt, first,
                     last, count);
}

void oracle_kv_tiles_ex(int64_t Nq, int64_t Nk, int causal, int64_t key_len,
                        int64_t window, int align, int64_t Br, int64_t Bc,
                        int64_t qt, int64_t* first, int64_t* last,
                        int64_t* count) {
  *first = -1; *last = -1; *count = 0;
  const int64_t i0 = qt * Br, i1 = (qt + 1) * Br < Nq ? (qt + 1) * Br : Nq;
  const int64_t ntiles = (Nk + Bc - 1) / Bc;
  for (int64_t jt = 0; jt < ntiles; ++jt) {
    const int64_t j0 = jt * Bc, j1 = (jt + 1) * Bc < Nk ? (jt + 1) * Bc : Nk;
    int touched = 0;
    for (int64_t i = i0; i < i1 && !touched; ++i) {
      int64_t lo, hi;
      oracle_visible_range_ex(i, Nq, Nk, causal, key_len, window, align, &lo,
                              &hi);
      for (int64_t j = j0; j < j1; ++j)
        if (j >= lo && j < hi) { touched = 1; break; }
    }
    if (touched) {
      if (*first < 0) *first = jt;
      *last = jt;
      ++*count;
    }
  }
}

/* ---- paged KV cache ([TIN] PagedAttention; [AME] 20) -------------------- */

/* Logical key j of kv head h of sequence b lives in physical block
 * block_table[b][j / page_size] at offset j % page_size: cache layout
 * [num_pages, Hkv, page_size, d], as the pages write a token's K/V into
 * kv_cache[phys, :, offset, :].  Copies keys [0, key_lens[b]) of every
 * (b, h) into out [B, Hkv, Nk, d] and zero-fills keys [key_lens[b], Nk).
 * Returns -1 (and writes nothing further) if a needed table entry lies
 * outside [0, num_pages). */
int oracle_gather_paged(const uint16_t* cache, int64_t num_pages, int64_t Hkv,
                        int64_t page_size, int64_t d,
                        const int32_t* block_table, int64_t max_pages,
                        const int32_t* key_lens, int64_t B, int64_t Nk,
                        uint16_t* out) {
  if (page_size <= 0 || max_pages * page_size < Nk) return -1;
  for (int64_t b = 0; b < B; ++b) {
    int64_t L = key_lens[b];
    if (L < 0) L = 0;
    if (L > Nk) L = Nk;
    for (int64_t h = 0; h < Hkv; ++h) {
      uint16_t* dst = out + (b * Hkv + h) * Nk * d;
      for (int64_t j = 0; j < Nk; ++j) {
        if (j >= L) {
          memset(dst + j * d, 0, sizeof(uint16_t) * d);
          continue;
        }
        const int64_t page = block_table[b * max_pages + j / page_size];
        if (page < 0 || page >= num_pages) return -1;
        const uint16_t* src =
            cache + ((page * Hkv + h) * page_size + j % page_size) * d;
        memcpy(dst + j * d, src, sizeof(uint16_t) * d);
      }
    }
  }
  return 0;
}

/* ---- attention rows ---------------------------------------------------- */

typedef struct {
  const uint16_t *q, *k, *v;
  int64_t B, Hq, Hkv, Nq, Nk, d;
  int causal;
  int64_t window; /* > 0: sliding window ([AME] 11) */
  int align;      /* query positions: 0 end of Nk, 1 end of key_lens[b] */
  double scale;
  const int32_t* key_lens;
  int rope;
  double rope_base;
  int rope_pairing;
  int rope_round; /* round rotated q/k rows to bf16 (composed-pipeline check) */
  int64_t q_pos_offset, k_pos_offset;
  int64_t block; /* > 0: online recurrence with this block size */
  const int64_t* rows;
  int64_t nrows;
  double *o, *lse;
  int64_t row_begin, row_end; /* this thread's share of the row list */
  int status;
  /* per-thread cache of one rotated kv head (RoPE only): values are the
   * same as rotating each key row on access, computed once per head */
  double* kcache;
  int64_t kcache_bg;
} job_t;

/* Key row j of kv head (b, g) as doubles, rotated when RoPE is on. */
static void load_key(job_t* J, const uint16_t* base_ptr, int64_t b,
                     int64_t g, int64_t j, int rotate, double* dst) {
  const int64_t d = J->d;
  if (rotate && J->kcache) {
    const int64_t bg = b * J->Hkv + g;
    if (J->kcache_bg != bg) {
      for (int64_t jj = 0; jj < J->Nk; ++jj) {
        const uint16_t* src = base_ptr + (bg * J->Nk + jj) * d;
        double* row = J->kcache + jj * d;
        for (int64_t c = 0; c < d; ++c) row[c] = bf16_bits_to_double(src[c]);
        rope_row(row, d, J->k_pos_offset + jj, J->rope_base, J->rope_pairing);
        if (J->rope_round)
          for (int64_t c = 0; c < d; ++c) row[c] = round_to_bf16(row[c]);
      }
      J->kcache_bg = bg;
    }
    memcpy(dst, J->kcache + j * d, sizeof(double) * d);
    return;
  }
  const uint16_t* src = base_ptr + ((b * J->Hkv + g) * J->Nk + j) * d;
  for (int64_t c = 0; c < d; ++c) dst[c] = bf16_bits_to_double(src[c]);
  if (rotate) {
    rope_row(dst, d, J->k_pos_offset + j, J->rope_base, J->rope_pairing);
    if (J->rope_round)
      for (int64_t c = 0; c < d; ++c) dst[c] = round_to_bf16(dst[c]);
  }
}

/* One output row, naive definition: all visible scores, stable softmax,
 * weighted sum of values, lse = m + log l. */
static void row_naive(job_t* J, int64_t r, double* qrow, double* krow,
                      double* s, double* p, double* out, double* lse_out) {
  const int64_t d = J->d;
  const int64_t i = r % J->Nq, h = (r / J->Nq) % J->Hq, b = r / (J->Nq * J->Hq);
  const int64_t g = h / (J->Hq / J->Hkv); /* query head -> kv head ([AME] 9) */
  const int64_t key_len = J->key_lens ? J->key_lens[b] : J->Nk;
  int64_t lo, hi;
  oracle_visible_range_ex(i, J->Nq, J->Nk, J->causal, key_len, J->window,
                          J->align, &lo, &hi);
  const int64_t n = hi - lo;
  for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
  if (n == 0) { *lse_out = -INFINITY; return; }

  const uint16_t* qsrc = J->q + r * d;
  for (int64_t c = 0; c < d; ++c) qrow[c] = bf16_bits_to_double(qsrc[c]);
  if (J->rope) {
    rope_row(qrow, d, J->q_pos_offset + i, J->rope_base, J->rope_pairing);
    if (J->rope_round)
      for (int64_t c = 0; c < d; ++c) qrow[c] = round_to_bf16(qrow[c]);
  }

  for (int64_t j = lo; j < hi; ++j) {
    load_key(J, J->k, b, g, j, J->rope, krow);
    double dot = 0.0;
    for (int64_t c = 0; c < d; ++c) dot += qrow[c] * krow[c];
    s[j - lo] = J->scale * dot;
  }
  /* stable softmax: p = exp(s - m) / l */
  oracle_softmax(s, n, p);
  for (int64_t j = lo; j < hi; ++j) {
    load_key(J, J->v, b, g, j, 0, krow);
    for (int64_t c = 0; c < d; ++c) out[c] += p[j - lo] * krow[c];
  }
  *lse_out = oracle_logsumexp(s, n);
}

/* One output row through the online recurrence over blocks of keys. */
static void row_online(job_t* J, int64_t r, double* qrow, double* krow,
                       double* s, double* acc, double* out, double* lse_out) {
  const int64_t d = J->d;
  const int64_t i = r % J->Nq, h = (r / J->Nq) % J->Hq, b = r / (J->Nq * J->Hq);
  const int64_t g = h / (J->Hq / J->Hkv);
  const int64_t key_len = J->key_lens ? J->key_lens[b] : J->Nk;
  int64_t lo, hi;
  oracle_visible_range_ex(i, J->Nq, J->Nk, J->causal, key_len, J->window,
                          J->align, &lo, &hi);
  const int64_t n = hi - lo;
  const uint16_t* qsrc = J->q + r * d;
  for (int64_t c = 0; c < d; ++c) qrow[c] = bf16_bits_to_double(qsrc[c]);

  double m = -INFINITY, l = 0.0;
  for (int64_t c = 0; c < d; ++c) acc[c] = 0.0;
  for (int64_t start = lo; start < hi; start += J->block) {
    const int64_t stop = start + J->block < hi ? start + J->block : hi;
    double bmax = -INFINITY;
    for (int64_t j = start; j < stop; ++j) {
      load_key(J, J->k, b, g, j, 0, krow);
      double dot = 0.0;
      for (int64_t c = 0; c < d; ++c) dot += qrow[c] * krow[c];
      s[j - start] = J->scale * dot;
      if (s[j - start] > bmax) bmax = s[j - start];
    }
    const double m_new = m > bmax ? m : bmax;
    /* rescale of the old state; the first block has nothing to rescale */
    const double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
    l *= alpha;
    for (int64_t c = 0; c < d; ++c) acc[c] *= alpha;
    for (int64_t j = start; j < stop; ++j) {
      const double pj = exp(s[j - start] - m_new);
      l += pj;
      load_key(J, J->v, b, g, j, 0, krow);
      for (int64_t c = 0; c < d; ++c) acc[c] += pj * krow[c];
    }
    m = m_new;
  }
  if (n == 0) {
    for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
    *lse_out = -INFINITY;
    return;
  }
  for (int64_t c = 0; c < d; ++c) out[c] = acc[c] / l;
  *lse_out = m + log(l);
}

static void* worker(void* arg) {
  job_t* J = (job_t*)arg;
  const int64_t d = J->d;
  const int64_t scratch = J->block > 0 ? J->block : J->Nk;
  double* qrow = (double*)malloc(sizeof(double) * d);
  double* krow = (double*)malloc(sizeof(double) * d);
  double* acc = (double*)malloc(sizeof(double) * d);
  double* s = (double*)malloc(sizeof(double) * (scratch > 0 ? scratch : 1));
  double* p = (double*)malloc(sizeof(double) * (J->Nk > 0 ? J->Nk : 1));
  J->kcache = NULL;
  J->kcache_bg = -1;
  if (J->rope && J->Nk > 0)
    J->kcache = (double*)malloc(sizeof(double) * J->Nk * d);
  if (!qrow || !krow || !acc || !s || !p) {
    J->status = -1;
  } else {
    for (int64_t t = J->row_begin; t < J->row_end; ++t) {
      const int64_t r = J->rows ? J->rows[t] : t;
      double lse_v;
      if (J->block > 0)
        row_online(J, r, qrow, krow, s, acc, J->o + t * d, &lse_v);
      else
        row_naive(J, r, qrow, krow, s, p, J->o + t * d, &lse_v);
      if (J->lse) J->lse[t] = lse_v;
    }
  }
  free(qrow); free(krow); free(acc); free(s); free(p); free(J->kcache);
  J->kcache = NULL;
  return NULL;
}

static int run_rows(job_t* proto, int nthreads) {
  const job_t* J = proto;
  if (!J->q || !J->k || !J->v || !J->o) return -1;
  if (J->B < 0 || J->Hq <= 0 || J->Hkv <= 0 || J->Nq < 0 || J->Nk < 0 ||
      J->d <= 0 || J->Hq % J->Hkv != 0 || (J->rope && J->d % 2 != 0))
    return -1;
  const int64_t total = J->B * J->Hq * J->Nq;
  if (J->nrows < 0) return -1;
  for (int64_t t = 0; J->rows && t < J->nrows; ++t)
    if (J->rows[t] < 0 || J->rows[t] >= total) return -1;
  if (!J->rows && J->nrows != total) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (J->nrows < nthreads) nthreads = J->nrows > 0 ? (int)J->nrows : 1;

  job_t jobs[256];
  pthread_t tid[256];
  int started[256];
  const int64_t per = (J->nrows + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = *J;
    jobs[t].row_begin = t * per < J->nrows ? t * per : J->nrows;
    jobs[t].row_end = (t + 1) * per < J->nrows ? (t + 1) * per : J->nrows;
    jobs[t].status = 0;
    started[t] = pthread_create(&tid[t], NULL, worker, &jobs[t]) == 0;
    if (!started[t]) worker(&jobs[t]);
  }
  int status = 0;
  for (int t = 0; t < nthreads; ++t) {
    if (started[t]) pthread_join(tid[t], NULL);
    if (jobs[t].status) status = jobs[t].status;
  }
  return status;
}

int oracle_attn_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                     int64_t Nk, int64_t d, int causal, int64_t window,
                     int align, double scale,
                     const int32_t* key_lens, int rope, double rope_base,
                     int rope_pairing, int rope_round, int64_t q_pos_offset,
                     int64_t k_pos_offset, const int64_t* rows, int64_t nrows,
                     double* o, double* lse, int nthreads) {
  job_t J;
  memset(&J, 0, sizeof J);
  J.q = q; J.k = k; J.v = v;
  J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Nq = Nq; J.Nk = Nk; J.d = d;
  J.causal = causal; J.window = window; J.align = align; J.scale = scale;
  J.key_lens = key_lens;
  J.rope = rope; J.rope_base = rope_base; J.rope_pairing = rope_pairing;
  J.rope_round = rope_round;
  J.q_pos_offset = q_pos_offset; J.k_pos_offset = k_pos_offset;
  J.block = 0; J.rows = rows; J.nrows = nrows; J.o = o; J.lse = lse;
  return run_rows(&J, nthreads);
}

int oracle_attn_online_rows(const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, int64_t B, int64_t Hq,
                            int64_t Hkv, int64_t Nq, int64_t Nk, int64_t d,
                            int causal, int64_t window, int align,
                            double scale, const int32_t* key_lens,
                            int64_t block, const int64_t* rows, int64_t nrows,
                            double* o, double* lse, int nthreads) {
  if (block <= 0) return -1;
  job_t J;
  memset(&J, 0, sizeof J);
  J.q = q; J.k = k; J.v = v;
  J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Nq = Nq; J.Nk = Nk; J.d = d;
  J.causal = causal; J.window = window; J.align = align; J.scale = scale;
  J.key_lens = key_lens;
  J.block = block; J.rows = rows; J.nrows = nrows; J.o = o; J.lse = lse;
  return run_rows(&J, nthreads);
}
