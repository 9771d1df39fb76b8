/*
 * fp8idx_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, float64 CPU restatement of the sparse-attention indexer:
 * fp8 multi-query logits followed by a per-row top-k.  Only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg may load this code;
 * the product path never does.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * What it computes (the definition the indexer pages give: the
 * `fp8_mqa_logits(q, (kv, kv_scales), weights, ks, ke)` call of the
 * "bench_mqa_logits_chunking.py" page, module docstring and `_run_chunked`,
 * with H = 32 index heads and D = 128):
 *
 *     logits[i,j] = s[j] * sum_h w[i,h] * max(0, sum_d q[i,h,d] * k[j,d])
 *                   for max(ks[i],0) <= j < min(ke[i],n), and -inf otherwise;
 *     out[i,:]    = indices of the k largest logits of row i, ties broken
 *                   by the lower index, padded with -1 when fewer than k
 *                   keys are valid.
 *
 * Every fp8 byte is decoded exactly to float64.  Each head dot product is
 * then exact in float64: a product of two e4m3 values is an integer
 * multiple of 2^-18 below 2^18 in magnitude, and a 128-term sum of those
 * stays far below 2^53 units of 2^-18.  The head-weighted sum and the key
 * scale are applied in float64 in ascending head order.
 *
 * It also restates the producer of the paged keys (the key quantisation
 * into the fp8 pool, at the end of this file).
 *
 * Parity pins (tests/test_oracle.py): the codec against torch's e4m3fn
 * cast and the rounding ties printed on the "Serve GLM-5.3-Flash on SM80"
 * page (unit-test commit notes); the dot against an int64 evaluation;
 * hand-computed tiny logits (tests/golden/); torch float64 einsum on small
 * shapes; brute-force top-k over all subsets; mask invariants; the paged
 * form against the prefill form on a gathered key array; the key
 * quantisation against the codec, its scale floor, torch's fp32 arithmetic
 * with torch's e4m3fn cast, and the e4m3 error bound.
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* e4m3fn codec (OCP FP8 E4M3, the format torch names float8_e4m3fn):  */
/* sign bit 7, exponent bits 6..3 with bias 7, mantissa bits 2..0;     */
/* exponent 0 is subnormal, 0x7F / 0xFF are NaN, no infinities.        */
/* ------------------------------------------------------------------ */

double oracle_e4m3_decode(uint8_t b) {
  int sign = (b >> 7) & 1;
  int e = (b >> 3) & 0xF;
  int mant = b & 7;
  double v;
  if (e == 15 && mant == 7) return sign ? -NAN : NAN;
  if (e == 0)
    v = ldexp((double)mant, -9);           /* subnormal: mant * 2^-9   */
  else
    v = ldexp((double)(8 + mant), e - 10); /* (1 + mant/8) * 2^(e-7)   */
  return sign ? -v : v;
}

/* Round to nearest, ties to even mantissa; magnitudes beyond the largest
 * finite value saturate to +-448; NaN maps to 0x7F with the input's sign.
 * Written as a search over the 127 non-negative finite codes: the codes
 * are monotone in value, so "even mantissa" on a tie is "even code". */
uint8_t oracle_e4m3_encode(double x) {
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  if (isnan(x)) return (uint8_t)(sign | 0x7F);
  double a = fabs(x);
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double err = fabs(oracle_e4m3_decode((uint8_t)c) - a);
    if (err < best_err || (err == best_err && (c & 1) == 0)) {
      best = c;
      best_err = err;
    }
  }
  return (uint8_t)(sign | best);
}

void oracle_e4m3_decode_array(const uint8_t* in, int64_t count, double* out) {
  for (int64_t i = 0; i < count; ++i) out[i] = oracle_e4m3_decode(in[i]);
}

void oracle_e4m3_encode_array(const double* in, int64_t count, uint8_t* out) {
  for (int64_t i = 0; i < count; ++i) out[i] = oracle_e4m3_encode(in[i]);
}

/* ------------------------------------------------------------------ */
/* Logits                                                             */
/* ------------------------------------------------------------------ */

/* The valid key range of one row: [max(ks,0), min(ke,n)), empty if the
 * clamped start is not below the clamped end. */
static void row_range(int32_t ks, int32_t ke, int64_t n, int64_t* lo, int64_t* hi) {
  int64_t a = ks < 0 ? 0 : ks;
  int64_t b = ke > n ? n : ke;
  if (b < a) b = a;
  *lo = a;
  *hi = b;
}

/* One logit from already decoded operands: qd is row i's [H, D] block,
 * kd is key j's [D] vector. */
static double one_logit(const double* qd, const double* kd, double sj,
                        const float* wi, int H, int D) {
  double sum = 0.0;
  for (int h = 0; h < H; ++h) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += qd[(int64_t)h * D + d] * kd[d];
    double relu = dot > 0.0 ? dot : 0.0;
    sum += (double)wi[h] * relu;
  }
  return sj * sum;
}

typedef struct {
  /* inputs */
  const uint8_t* q;
  const double* kdec; /* decoded keys [n, D] */
  const float* s;
  const float* w;
  const int32_t* ks;
  const int32_t* ke;
  int64_t n;
  int H, D;
  const int64_t* rows;
  int64_t nrows;
  /* output */
  double* out; /* [nrows, n] */
  /* work split */
  int64_t r0, r1;
} logits_job;

static void* logits_worker(void* arg) {
  logits_job* jb = (logits_job*)arg;
  int H = jb->H, D = jb->D;
  double* qd = (double*)malloc(sizeof(double) * (size_t)H * D);
  for (int64_t r = jb->r0; r < jb->r1; ++r) {
    int64_t i = jb->rows[r];
    oracle_e4m3_decode_array(jb->q + i * H * D, (int64_t)H * D, qd);
    int64_t lo, hi;
    row_range(jb->ks[i], jb->ke[i], jb->n, &lo, &hi);
    double* orow = jb->out + r * jb->n;
    for (int64_t j = 0; j < jb->n; ++j) {
      if (j < lo || j >= hi) {
        orow[j] = -INFINITY;
      } else {
        orow[j] = one_logit(qd, jb->kdec + j * D, (double)jb->s[j], jb->w + i * H, H, D);
      }
    }
  }
  free(qd);
  return NULL;
}

static void run_jobs(void* (*fn)(void*), void* jobs, size_t job_size, int nthreads) {
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, fn, (char*)jobs + job_size * (size_t)t);
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
}

/* Full logit rows for the listed query rows: out[r, j] for r < nrows. */
void oracle_mqa_logits_rows(const uint8_t* q, const uint8_t* k, const float* s, const float* w,
                            const int32_t* ks, const int32_t* ke, int64_t m, int64_t n, int H,
                            int D, const int64_t* rows, int64_t nrows, double* out,
                            int nthreads) {
  (void)m;
  if (nrows <= 0) return;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nrows) nthreads = (int)nrows;
  double* kdec = (double*)malloc(sizeof(double) * (size_t)(n * D > 0 ? n * D : 1));
  oracle_e4m3_decode_array(k, n * D, kdec);
  logits_job* jobs = (logits_job*)calloc((size_t)nthreads, sizeof(logits_job));
  for (int t = 0; t < nthreads; ++t) {
    logits_job* jb = &jobs[t];
    jb->q = q; jb->kdec = kdec; jb->s = s; jb->w = w; jb->ks = ks; jb->ke = ke;
    jb->n = n; jb->H = H; jb->D = D; jb->rows = rows; jb->nrows = nrows; jb->out = out;
    jb->r0 = nrows * t / nthreads;
    jb->r1 = nrows * (t + 1) / nthreads;
  }
  run_jobs(logits_worker, jobs, sizeof(logits_job), nthreads);
  free(jobs);
  free(kdec);
}

/* ------------------------------------------------------------------ */
/* Top-k: full sort of the valid entries by (logit desc, index asc).  */
/* ------------------------------------------------------------------ */

typedef struct {
  double v;
  int64_t j;
} vj_pair;

static int cmp_desc_then_index(const void* a, const void* b) {
  const vj_pair* x = (const vj_pair*)a;
  const vj_pair* y = (const vj_pair*)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->j < y->j) ? -1 : (x->j > y->j);
}

/* Top-k of one row of logits restricted to [lo, hi).  Writes k indices
 * (padded with -1) and their logits (padded with -inf); returns the number
 * of valid keys. */
static int64_t topk_one_row(const double* row, int64_t lo, int64_t hi, int k, int32_t* out_idx,
                            double* out_val) {
  int64_t cnt = hi - lo;
  vj_pair* v = (vj_pair*)malloc(sizeof(vj_pair) * (size_t)(cnt > 0 ? cnt : 1));
  for (int64_t j = lo; j < hi; ++j) {
    v[j - lo].v = row[j];
    v[j - lo].j = j;
  }
  qsort(v, (size_t)cnt, sizeof(vj_pair), cmp_desc_then_index);
  for (int t = 0; t < k; ++t) {
    if (t < cnt) {
      out_idx[t] = (int32_t)v[t].j;
      if (out_val) out_val[t] = v[t].v;
    } else {
      out_idx[t] = -1;
      if (out_val) out_val[t] = -INFINITY;
    }
  }
  free(v);
  return cnt;
}

/* Top-k over logit rows already computed (rows[r] names the query row whose
 * ks/ke apply to logits row r). */
void oracle_topk_rows(const double* logits, int64_t n, const int32_t* ks, const int32_t* ke,
                      const int64_t* rows, int64_t nrows, int k, int32_t* out_idx,
                      double* out_val) {
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t lo, hi;
    int64_t i = rows[r];
    row_range(ks[i], ke[i], n, &lo, &hi);
    topk_one_row(logits + r * n, lo, hi, k, out_idx + r * k, out_val ? out_val + r * k : NULL);
  }
}

/* ------------------------------------------------------------------ */
/* Paged form: key j of request b is slot j % P of physical page       */
/* block_table[b][j / P]; row t of request b (R rows per request)     */
/* sees keys [0, L_b - R + t + 1), clamped to [0, L_b].                */
/* ------------------------------------------------------------------ */

typedef struct {
  const uint8_t* q;
  const uint8_t* k_pages;
  const float* s_pages;
  const float* w;
  const int32_t* block_table;
  const int32_t* seq_lens;
  int R, max_blocks, page_size, H, D;
  const int64_t* rows;
  int64_t nrows;
  int64_t lmax; /* row stride of out */
  double* out;
  int64_t r0, r1;
} paged_job;

static void* paged_worker(void* arg) {
  paged_job* jb = (paged_job*)arg;
  int H = jb->H, D = jb->D, P = jb->page_size;
  double* qd = (double*)malloc(sizeof(double) * (size_t)H * D);
  double* kd = (double*)malloc(sizeof(double) * (size_t)D);
  for (int64_t r = jb->r0; r < jb->r1; ++r) {
    int64_t row = jb->rows[r];
    int64_t b = row / jb->R;
    int64_t t = row % jb->R;
    int64_t L = jb->seq_lens[b];
    int64_t ke = L - jb->R + t + 1;
    if (ke < 0) ke = 0;
    if (ke > L) ke = L;
    oracle_e4m3_decode_array(jb->q + row * H * D, (int64_t)H * D, qd);
    double* orow = jb->out + r * jb->lmax;
    for (int64_t j = 0; j < jb->lmax; ++j) {
      if (j >= ke) {
        orow[j] = -INFINITY;
        continue;
      }
      int64_t page = jb->block_table[b * jb->max_blocks + j / P];
      int64_t slot = j % P;
      oracle_e4m3_decode_array(jb->k_pages + (page * P + slot) * D, D, kd);
      double sj = (double)jb->s_pages[page * P + slot];
      orow[j] = one_logit(qd, kd, sj, jb->w + row * H, H, D);
    }
  }
  free(kd);
  free(qd);
  return NULL;
}

/* Logit rows of the paged form for the listed global rows (row = b*R + t);
 * out is [nrows, lmax] with -inf beyond each row's range. */
void oracle_paged_logits_rows(const uint8_t* q, const uint8_t* k_pages, const float* s_pages,
                              const float* w, const int32_t* block_table, const int32_t* seq_lens,
                              int B, int R, int max_blocks, int page_size, int H, int D,
                              const int64_t* rows, int64_t nrows, int64_t lmax, double* out,
                              int nthreads) {
  (void)B;
  if (nrows <= 0) return;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nrows) nthreads = (int)nrows;
  paged_job* jobs = (paged_job*)calloc((size_t)nthreads, sizeof(paged_job));
  for (int t = 0; t < nthreads; ++t) {
    paged_job* jb = &jobs[t];
    jb->q = q; jb->k_pages = k_pages; jb->s_pages = s_pages; jb->w = w;
    jb->block_table = block_table; jb->seq_lens = seq_lens;
    jb->R = R; jb->max_blocks = max_blocks; jb->page_size = page_size; jb->H = H; jb->D = D;
    jb->rows = rows; jb->nrows = nrows; jb->lmax = lmax; jb->out = out;
    jb->r0 = nrows * t / nthreads;
    jb->r1 = nrows * (t + 1) / nthreads;
  }
  run_jobs(paged_worker, jobs, sizeof(paged_job), nthreads);
  free(jobs);
}

/* Top-k over paged logit rows: row r's valid range is [0, ke) with the
 * paged rule above. */
void oracle_paged_topk_rows(const double* logits, int64_t lmax, const int32_t* seq_lens, int R,
                            const int64_t* rows, int64_t nrows, int k, int32_t* out_idx,
                            double* out_val) {
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t row = rows[r];
    int64_t b = row / R, t = row % R;
    int64_t L = seq_lens[b];
    int64_t ke = L - R + t + 1;
    if (ke < 0) ke = 0;
    if (ke > L) ke = L;
    if (ke > lmax) ke = lmax;
    topk_one_row(logits + r * lmax, 0, ke, k, out_idx + r * k, out_val ? out_val + r * k : NULL);
  }
}

/* ------------------------------------------------------------------ */
/* Key quantisation into the paged key pool                           */
/* ------------------------------------------------------------------ */

/* The producer side of the paged keys: the `act_quant` step and the fp8
 * k-pool stores that the "Serve GLM-5.3-Flash on SM80" page names (commit
 * notes: the k-pool write kernels, stored through an e4m3fn codec).  The
 * pages do not print the scale rule; the reading taken is one fp32 scale per
 * token,
 *     s_t = max(amax_t, 1e-4) / 448,   amax_t = max_d |x[t,d]|,
 * and codes e4m3(x[t,d] / s_t) rounded to nearest even and saturated.  The
 * scale and the quotient decide integer codes, so they are taken in fp32,
 * the precision the library computes them in; the rounding of the fp32
 * quotient to e4m3 is the codec above.  Token t is written to pool slot
 * slot[t] (page slot[t] / 64, row slot[t] % 64); a slot outside
 * [0, num_slots) means "do not store" and leaves the pool untouched. */
static float bf16_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

void oracle_act_quant_store(const uint16_t* x, int64_t T, int D, const int64_t* slot,
                            int64_t num_slots, uint8_t* k_pool, float* s_pool) {
  for (int64_t t = 0; t < T; ++t) {
    const int64_t sl = slot[t];
    if (sl < 0 || sl >= num_slots) continue;
    const uint16_t* row = x + t * D;
    float amax = 0.0f;
    for (int d = 0; d < D; ++d) {
      const float a = fabsf(bf16_to_float(row[d]));
      if (a > amax) amax = a;
    }
    const float sc = (amax > 1e-4f ? amax : 1e-4f) / 448.0f;
    for (int d = 0; d < D; ++d) {
      const float v = bf16_to_float(row[d]) / sc;
      k_pool[sl * D + d] = oracle_e4m3_encode((double)v);
    }
    s_pool[sl] = sc;
  }
}
