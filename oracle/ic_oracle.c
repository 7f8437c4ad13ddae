/*
 * ic_oracle.c -- plain, slow, fp64 CPU oracle for the IndexCache / DeepSeek
 * Sparse Attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load
 * this file; only tests/, __graft_entry__.smoke() and the cpu_baseline leg of
 * bench.py use it.  It shares no code, header, table or constant with the CUDA
 * library: every definition below is written out from the pages.
 *
 * Sources (page title, then the passage):
 *  [P1] "IndexCache: Wie DeepSeek O(NL^2)-Kosten in Sparse Attention um 75%
 *       reduziert" (itoverdose.com):
 *         - intro paragraph: k = 2048 positions per query, attention cost O(Lk);
 *         - second paragraph: the indexer scores *all previous tokens*;
 *         - the F/S list and "the first layer is always F";
 *         - the routing loop in "Einfache Implementierung";
 *         - "Wie der Indexer funktioniert": score, then ReLU, then top-k;
 *         - the MLA paragraph (latent KV shared by all heads).
 *  [P2] parapluman.nl article, "Aandacht cachen met IndexCache": S layers reuse
 *       the indices of the nearest preceding F layer.
 *  The exact indexer formula I[t,s] = sum_h w[t,h] * ReLU(q[t,h] . k[s]) and the
 *  tie rule (lower index wins) are the project's stated reading of the garbled
 *  "score s_i, g_i = max(0, s_i), top-k" passage of [P1]; the e4m3 format is the
 *  OCP 8-bit floating point specification (E4M3, bias 7, no infinities,
 *  S.1111.111 = NaN, largest finite 448).
 *
 * Pinned by tests/test_oracle_pins.py (brute force, closed forms, library
 * special cases, hand-worked golden fixtures under tests/golden/).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Threading: rows are independent; split them over nthreads workers.        */
/* ------------------------------------------------------------------------- */
typedef void (*row_fn)(void* ctx, long row);
typedef struct { row_fn fn; void* ctx; long first, step, end; } span_t;

static void* run_span(void* p) {
  span_t* s = (span_t*)p;
  for (long r = s->first; r < s->end; r += s->step) s->fn(s->ctx, r);
  return NULL;
}

static void parallel_rows(row_fn fn, void* ctx, long nrows, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (nthreads == 1 || nrows < 2) {
    for (long r = 0; r < nrows; ++r) fn(ctx, r);
    return;
  }
  pthread_t th[256];
  span_t sp[256];
  int started[256];
  /* interleave rows over workers so that causal rows of unequal length balance */
  for (int i = 0; i < nthreads; ++i) {
    started[i] = 0;
    if (i >= nrows) continue;
    sp[i].fn = fn; sp[i].ctx = ctx; sp[i].first = i; sp[i].step = nthreads; sp[i].end = nrows;
    if (pthread_create(&th[i], NULL, run_span, &sp[i]) == 0) started[i] = 1;
    else run_span(&sp[i]);
  }
  for (int i = 0; i < nthreads; ++i)
    if (started[i]) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------------------- */
/* OCP E4M3: sign bit, 4 exponent bits (bias 7), 3 mantissa bits.            */
/*   e == 0:  (-1)^s * 2^-6 * (m / 8)          (subnormals, incl. +-0)         */
/*   e  > 0:  (-1)^s * 2^(e-7) * (1 + m / 8)   except e == 15 && m == 7: NaN  */
/* ------------------------------------------------------------------------- */
double ico_e4m3_decode(uint8_t code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return s ? -mag : mag;
}

/* Round-to-nearest-even onto the E4M3 grid, saturating at +-448 (the largest
 * finite value).  Done by scanning the 127 non-negative finite codes, which is
 * slow but follows the definition directly: the representable value nearest
 * to |x|; on an exact midpoint, the code with an even mantissa (the even
 * significand).  NaN input is not supported by the method (finite inputs). */
uint8_t ico_e4m3_encode(double x) {
  int neg = signbit(x) ? 1 : 0;
  double a = fabs(x);
  if (a >= 448.0) return (uint8_t)((neg << 7) | 0x7E);
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double v = ico_e4m3_decode((uint8_t)c);
    double err = fabs(v - a);
    if (err < best_err) { best_err = err; best = c; }
    else if (err == best_err) {
      /* tie: exact midpoint between two neighbours; keep the even one */
      if ((c & 1) == 0) best = c;
    }
  }
  return (uint8_t)((neg << 7) | best);
}

/* Per-row scaling to e4m3 (one fp32 scale per token): each row of n values gets
 * scale = amax / 448 (1 when the row is all zero); code = E4M3(x / scale).
 * The scale and the division are fp32 operations (IEEE round-to-nearest), the
 * precision the quantised code is decided in. */
void ico_quant_rows_e4m3(const float* x, long rows, int n, uint8_t* codes, float* scales) {
  for (long r = 0; r < rows; ++r) {
    const float* xr = x + r * (long)n;
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) { float a = fabsf(xr[i]); if (a > amax) amax = a; }
    volatile float scale = (amax > 0.0f) ? amax / 448.0f : 1.0f;
    scales[r] = scale;
    for (int i = 0; i < n; ++i) {
      volatile float v = xr[i] / scale;
      codes[r * (long)n + i] = ico_e4m3_encode((double)v);
    }
  }
}

/* ------------------------------------------------------------------------- */
/* Lightning indexer score ([P1] "Wie der Indexer funktioniert"):           */
/*   I[b,r,s] = sum_h w[b,r,h] * max(0, sum_d q[b,r,h,d] * k[b,s,d])          */
/* for keys s <= pos0 + r (causal: all previous tokens and the token itself); */
/* keys s > pos0 + r are not candidates and get -inf.                          */
/* Layouts (row-major): q [B, rows, H, D]; k [B, Lk, D]; w [B, rows, H];       */
/* out [B, nsel, Lk] for the selected rows sel[0..nsel) (or all rows).         */
/* ------------------------------------------------------------------------- */
typedef struct {
  const double *q, *k, *w;
  int B, rows, H, D, Lk;
  long pos0;
  const int* sel; int nsel;
  double* out;
} idx_ctx;

static void idx_row(void* p, long job) {
  idx_ctx* c = (idx_ctx*)p;
  long b = job / c->nsel, j = job % c->nsel;
  long r = c->sel ? c->sel[j] : j;
  const double* qr = c->q + ((b * c->rows + r) * (long)c->H) * c->D;
  const double* wr = c->w + (b * c->rows + r) * (long)c->H;
  const double* kb = c->k + b * (long)c->Lk * c->D;
  double* o = c->out + (b * c->nsel + j) * (long)c->Lk;
  long pos = c->pos0 + r;
  for (long s = 0; s < c->Lk; ++s) {
    if (s > pos) { o[s] = -INFINITY; continue; }
    const double* ks = kb + s * c->D;
    double acc = 0.0;
    for (int h = 0; h < c->H; ++h) {
      const double* qh = qr + (long)h * c->D;
      double dot = 0.0;
      for (int d = 0; d < c->D; ++d) dot += qh[d] * ks[d];
      double g = dot > 0.0 ? dot : 0.0;   /* ReLU gate */
      acc += wr[h] * g;
    }
    o[s] = acc;
  }
}

void ico_indexer_scores(const double* q, const double* k, const double* w, int B, int rows,
                        int H, int D, int Lk, long pos0, const int* sel, int nsel,
                        double* out, int nthreads) {
  idx_ctx c = {q, k, w, B, rows, H, D, Lk, pos0, sel, sel ? nsel : rows, out};
  parallel_rows(idx_row, &c, (long)B * c.nsel, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Top-k ([P1] intro: k positions per query; routing loop T <- top-k(I)):     */
/* the min(k, valid) candidate indices s < valid with the largest scores;     */
/* ties go to the lower index; scores compare as IEEE values (-0 == +0).      */
/* Brute force: sort all candidates, keep the first m, emit them in            */
/* ascending index order, pad the rest of the row with -1.                     */
/* ------------------------------------------------------------------------- */
typedef struct { float v; int i; } cand_t;

static int cand_cmp(const void* a, const void* b) {
  const cand_t* x = (const cand_t*)a;
  const cand_t* y = (const cand_t*)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->i < y->i) ? -1 : (x->i > y->i);
}
static int int_cmp(const void* a, const void* b) {
  int x = *(const int*)a, y = *(const int*)b;
  return (x > y) - (x < y);
}

typedef struct {
  const float* scores; long ld; int n; const int* valid; int k; int* idx;
} topk_ctx;

static void topk_row(void* p, long r) {
  topk_ctx* c = (topk_ctx*)p;
  int nv = c->valid ? c->valid[r] : c->n;
  if (nv > c->n) nv = c->n;
  if (nv < 0) nv = 0;
  const float* row = c->scores + r * c->ld;
  cand_t* cs = (cand_t*)malloc(sizeof(cand_t) * (size_t)(nv > 0 ? nv : 1));
  for (int s = 0; s < nv; ++s) { cs[s].v = row[s]; cs[s].i = s; }
  qsort(cs, (size_t)nv, sizeof(cand_t), cand_cmp);
  int m = nv < c->k ? nv : c->k;
  int* out = c->idx + r * (long)c->k;
  for (int j = 0; j < m; ++j) out[j] = cs[j].i;
  qsort(out, (size_t)m, sizeof(int), int_cmp);
  for (int j = m; j < c->k; ++j) out[j] = -1;
  free(cs);
}

void ico_topk(const float* scores, long rows, int n, long ld, const int* valid, int k, int* idx,
              int nthreads) {
  topk_ctx c = {scores, ld, n, valid, k, idx};
  parallel_rows(topk_row, &c, rows, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Sparse attention over the index set ([P1] routing loop X <- SparseAttn(X,T); */
/* MLA paragraph).  For query row r, head h, with J = {idx[r][j] >= 0}:       */
/*   z_j = scale * q[r,h,:] . kv[j,:Dk]                                        */
/*   p_j = exp(z_j - max z) / sum exp(z - max z)                               */
/*   out[r,h,:] = sum_j p_j * v[j,:Dv];  lse[r,h] = max z + log sum exp(...)   */
/* MLA in absorbed form: v is the first Dv columns of the shared latent kv     */
/* (pass v = NULL); MQA: separate v rows.                                      */
/* Layouts: q [B, rows, Hq, Dk]; kv [B, Lkv, ld_kv]; v [B, Lkv, ld_v];         */
/* idx [B, rows, k]; out [B, rows, Hq, Dv]; lse [B, rows, Hq].                 */
/* An index set with no valid entry gives out = 0 and lse = -inf.             */
/* ------------------------------------------------------------------------- */
typedef struct {
  const double *q, *kv, *v; const int* idx;
  int B, rows, Hq, Dk, Dv, k, Lkv; long ld_kv, ld_v; double scale;
  double *out, *lse;
} attn_ctx;

static void attn_row(void* p, long job) {
  attn_ctx* c = (attn_ctx*)p;
  long b = job / c->rows, r = job % c->rows;
  const int* ir = c->idx + (b * c->rows + r) * (long)c->k;
  const double* kvb = c->kv + b * (long)c->Lkv * c->ld_kv;
  const double* vb = c->v ? c->v + b * (long)c->Lkv * c->ld_v : kvb;
  long ldv = c->v ? c->ld_v : c->ld_kv;
  double* z = (double*)malloc(sizeof(double) * (size_t)c->k);
  for (int h = 0; h < c->Hq; ++h) {
    const double* qh = c->q + ((b * c->rows + r) * (long)c->Hq + h) * c->Dk;
    double* o = c->out + ((b * c->rows + r) * (long)c->Hq + h) * c->Dv;
    double zmax = -INFINITY;
    for (int j = 0; j < c->k; ++j) {
      int s = ir[j];
      if (s < 0) continue;
      const double* kr = kvb + (long)s * c->ld_kv;
      double dot = 0.0;
      for (int d = 0; d < c->Dk; ++d) dot += qh[d] * kr[d];
      z[j] = dot * c->scale;
      if (z[j] > zmax) zmax = z[j];
    }
    for (int d = 0; d < c->Dv; ++d) o[d] = 0.0;
    if (zmax == -INFINITY) {
      if (c->lse) c->lse[(b * c->rows + r) * (long)c->Hq + h] = -INFINITY;
      continue;
    }
    double den = 0.0;
    for (int j = 0; j < c->k; ++j) {
      int s = ir[j];
      if (s < 0) continue;
      double e = exp(z[j] - zmax);
      den += e;
      const double* vr = vb + (long)s * ldv;
      for (int d = 0; d < c->Dv; ++d) o[d] += e * vr[d];
    }
    for (int d = 0; d < c->Dv; ++d) o[d] /= den;
    if (c->lse) c->lse[(b * c->rows + r) * (long)c->Hq + h] = zmax + log(den);
  }
  free(z);
}

void ico_sparse_attn(const double* q, const double* kv, long ld_kv, const double* v, long ld_v,
                     const int* idx, int B, int rows, int Hq, int Dk, int Dv, int k, int Lkv,
                     double scale, double* out, double* lse, int nthreads) {
  attn_ctx c = {q, kv, v, idx, B, rows, Hq, Dk, Dv, k, Lkv, ld_kv, ld_v, scale, out, lse};
  parallel_rows(attn_row, &c, (long)B * rows, nthreads);
}
