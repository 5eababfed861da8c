/*
 * sdl_oracle -- plain fp64 CPU oracle for block-sparse attention in
 * diffusion-LLM denoising steps.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The GPU library shares
 * no code with it, and nothing on the GPU path may call it.
 *
 * What it computes follows the Step-dLLM abstract ("Step-dLLM: Adaptive
 * Step-aware Sparse Attention for Efficient Diffusion LLM Inference",
 * mlinfo.pages.dev, abstract): a block-sparse mask is rebuilt at anchor steps
 * under one head-adaptive global budget and reused in between, and attention
 * is evaluated only on the blocks the mask keeps.  The abstract leaves the
 * block score and the selection rule open; this oracle writes out the reading
 * used throughout the library:
 *
 *   pool:    Qbar[b,h,i,:] = mean of Q[b,t,h,:] over the tokens t of block i
 *            (likewise Kbar over KV heads)
 *   score:   Z[b,h,i,j] = scale * Qbar[b,h,i,:] . Kbar[b,h/g,j,:]
 *            P[b,h,i,:] = softmax over j of Z[b,h,i,:]
 *   budget:  per batch element, floor((1 - sparsity) * H * nb^2 + 0.5)
 *   select:  every diagonal block (i, i) is kept; the remaining budget goes
 *            to the largest off-diagonal P of all heads of the batch element
 *            together, ties broken by the lower flat index ((b*H+h)*nb+i)*nb+j
 *   attend:  for token t of block i, softmax(scale * q_t . k_u) over the
 *            tokens u of the kept blocks of row i, times v_u  (non-causal)
 *
 * Everything is fp64 on inputs widened exactly from bf16 or fp32.  There is
 * no blocking, fusion or reordering beyond these definitions.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* --------------------------------------------------------------- inputs */

static double load_elem(const void* x, int dtype, int64_t idx) {
  if (dtype == 1) return (double)((const float*)x)[idx];
  uint32_t bits = (uint32_t)((const uint16_t*)x)[idx] << 16;
  float f;
  memcpy(&f, &bits, sizeof(f));
  return (double)f;
}

/* strides (in elements) for the (b, t, h) axes; the head dim is contiguous */
static int64_t offs(const int64_t* s, int b, int t, int h) {
  return (int64_t)b * s[0] + (int64_t)t * s[1] + (int64_t)h * s[2];
}

/* --------------------------------------------------------------- budget */

/* Number of blocks kept for ONE batch element: floor((1 - s) * H * nb^2 + 0.5),
 * or -1 when sparsity is outside [0, 1) or the budget is below the H * nb
 * diagonal blocks that are always kept. */
int64_t oracle_budget(int H, int nb, double sparsity) {
  if (!(sparsity >= 0.0 && sparsity < 1.0) || H <= 0 || nb <= 0) return -1;
  double total = (double)H * (double)nb * (double)nb;
  int64_t k = (int64_t)floor((1.0 - sparsity) * total + 0.5);
  if (k < (int64_t)H * nb) return -1;
  return k;
}

/* ------------------------------------------------------------------ pool */

/* out[b, h, i, c] = (1/bs) * sum over t in [i*bs, (i+1)*bs) of x[b, t, h, c] */
int oracle_pool(const void* x, int dtype, int B, int L, int Hx, int d, int bs,
                const int64_t* strides, double* out) {
  if (!x || !out || bs <= 0 || L % bs) return -1;
  int nb = L / bs;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hx; ++h)
      for (int i = 0; i < nb; ++i)
        for (int c = 0; c < d; ++c) {
          double s = 0.0;
          for (int t = i * bs; t < (i + 1) * bs; ++t) s += load_elem(x, dtype, offs(strides, b, t, h) + c);
          out[(((int64_t)b * Hx + h) * nb + i) * d + c] = s / (double)bs;
        }
  return 0;
}

/* --------------------------------------------------------- block scores */

/* P[b, h, i, j] = softmax_j(scale * Qbar[b,h,i,:] . Kbar[b,h/g,j,:]) */
int oracle_block_scores(const void* q, const void* k, int dtype, int B, int H, int Hkv, int L,
                        int d, int bs, const int64_t* qs, const int64_t* ks, double scale,
                        double* P) {
  if (!q || !k || !P || Hkv <= 0 || H % Hkv || bs <= 0 || L % bs) return -1;
  int nb = L / bs, g = H / Hkv;
  double* qb = (double*)malloc(sizeof(double) * (size_t)B * H * nb * d);
  double* kb = (double*)malloc(sizeof(double) * (size_t)B * Hkv * nb * d);
  double* z = (double*)malloc(sizeof(double) * (size_t)nb);
  if (!qb || !kb || !z) {
    free(qb);
    free(kb);
    free(z);
    return -2;
  }
  oracle_pool(q, dtype, B, L, H, d, bs, qs, qb);
  oracle_pool(k, dtype, B, L, Hkv, d, bs, ks, kb);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      int kh = h / g;
      for (int i = 0; i < nb; ++i) {
        const double* qi = qb + (((int64_t)b * H + h) * nb + i) * d;
        double m = -INFINITY;
        for (int j = 0; j < nb; ++j) {
          const double* kj = kb + (((int64_t)b * Hkv + kh) * nb + j) * d;
          double s = 0.0;
          for (int c = 0; c < d; ++c) s += qi[c] * kj[c];
          z[j] = scale * s;
          if (z[j] > m) m = z[j];
        }
        double sum = 0.0;
        for (int j = 0; j < nb; ++j) {
          z[j] = exp(z[j] - m);
          sum += z[j];
        }
        double* row = P + (((int64_t)b * H + h) * nb + i) * nb;
        for (int j = 0; j < nb; ++j) row[j] = z[j] / sum;
      }
    }
  free(qb);
  free(kb);
  free(z);
  return 0;
}

/* ------------------------------------------------------------- selection */

typedef struct {
  double p;
  int64_t idx;
} cand;

/* Total order: larger P first, then smaller flat index. */
static int cand_cmp(const void* a, const void* b) {
  const cand* x = (const cand*)a;
  const cand* y = (const cand*)b;
  if (x->p > y->p) return -1;
  if (x->p < y->p) return 1;
  return (x->idx > y->idx) - (x->idx < y->idx);
}

/* mask[b,h,i,j] = 1 for kept blocks.  tau[b] = P of the last off-diagonal
 * block taken in batch element b (+inf when none is taken).  Returns the
 * number of kept blocks over all batch elements, or -1 on a bad budget. */
int64_t oracle_select(const double* P, int B, int H, int nb, double sparsity, uint8_t* mask,
                      double* tau) {
  int64_t kb = oracle_budget(H, nb, sparsity);
  if (kb < 0 || !P || !mask) return -1;
  int64_t per = (int64_t)H * nb * nb;
  int64_t nfree = (int64_t)H * nb * (nb - 1);
  int64_t k = kb - (int64_t)H * nb;
  cand* c = (cand*)malloc(sizeof(cand) * (size_t)(nfree > 0 ? nfree : 1));
  if (!c) return -2;
  memset(mask, 0, (size_t)(B * per));
  int64_t kept = 0;
  for (int b = 0; b < B; ++b) {
    int64_t n = 0;
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < nb; ++i)
        for (int j = 0; j < nb; ++j) {
          int64_t flat = (((int64_t)b * H + h) * nb + i) * nb + j;
          if (i == j) {
            mask[flat] = 1;
            ++kept;
          } else {
            c[n].p = P[flat];
            c[n].idx = flat;
            ++n;
          }
        }
    qsort(c, (size_t)n, sizeof(cand), cand_cmp);
    for (int64_t r = 0; r < k; ++r) mask[c[r].idx] = 1;
    kept += k;
    if (tau) tau[b] = k > 0 ? c[k - 1].p : INFINITY;
  }
  free(c);
  return kept;
}

/* ------------------------------------------------------------- attention */

typedef struct {
  const void *q, *k, *v;
  int dtype, B, H, Hkv, L, d, bs;
  const int64_t *qs, *ks, *vs;
  const uint8_t* mask;
  double scale;
  const int64_t* rows;
  int64_t r0, r1;
  double *O, *lse;
  int err;
} attn_job;

static void* attn_worker(void* arg) {
  attn_job* j = (attn_job*)arg;
  int nb = j->L / j->bs, g = j->H / j->Hkv, d = j->d;
  double* x = (double*)malloc(sizeof(double) * (size_t)j->L);
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  double* acc = (double*)malloc(sizeof(double) * (size_t)d);
  if (!x || !qv || !acc) {
    j->err = -2;
    free(x);
    free(qv);
    free(acc);
    return NULL;
  }
  for (int64_t r = j->r0; r < j->r1; ++r) {
    int b, h, t;
    if (j->rows) {
      b = (int)j->rows[3 * r];
      h = (int)j->rows[3 * r + 1];
      t = (int)j->rows[3 * r + 2];
    } else {
      b = (int)(r / ((int64_t)j->H * j->L));
      h = (int)((r / j->L) % j->H);
      t = (int)(r % j->L);
    }
    int kh = h / g, i = t / j->bs;
    for (int c = 0; c < d; ++c) qv[c] = load_elem(j->q, j->dtype, offs(j->qs, b, t, h) + c);
    /* logits over the tokens of every kept block of row i */
    double m = -INFINITY;
    int n = 0;
    for (int jb = 0; jb < nb; ++jb) {
      if (j->mask && !j->mask[(((int64_t)b * j->H + h) * nb + i) * nb + jb]) continue;
      for (int u = jb * j->bs; u < (jb + 1) * j->bs; ++u) {
        double s = 0.0;
        int64_t ko = offs(j->ks, b, u, kh);
        for (int c = 0; c < d; ++c) s += qv[c] * load_elem(j->k, j->dtype, ko + c);
        x[u] = j->scale * s;
        if (x[u] > m) m = x[u];
        ++n;
      }
    }
    double l = 0.0;
    for (int c = 0; c < d; ++c) acc[c] = 0.0;
    for (int jb = 0; jb < nb; ++jb) {
      if (j->mask && !j->mask[(((int64_t)b * j->H + h) * nb + i) * nb + jb]) continue;
      for (int u = jb * j->bs; u < (jb + 1) * j->bs; ++u) {
        double p = exp(x[u] - m);
        l += p;
        int64_t vo = offs(j->vs, b, u, kh);
        for (int c = 0; c < d; ++c) acc[c] += p * load_elem(j->v, j->dtype, vo + c);
      }
    }
    for (int c = 0; c < d; ++c) j->O[r * d + c] = n ? acc[c] / l : 0.0;
    if (j->lse) j->lse[r] = n ? m + log(l) : -INFINITY;
  }
  free(x);
  free(qv);
  free(acc);
  return NULL;
}

/* O[r, :] and lse[r] for each requested row r = (b, h, t): rows is n_rows
 * triples, or NULL for every (b, h, t) in that order.  mask is the block mask
 * [B, H, nb, nb] (NULL = every block, i.e. dense attention).  lse may be NULL. */
int oracle_attention(const void* q, const void* k, const void* v, int dtype, int B, int H,
                     int Hkv, int L, int d, int bs, const int64_t* qs, const int64_t* ks,
                     const int64_t* vs, const uint8_t* mask, double scale, const int64_t* rows,
                     int64_t n_rows, double* O, double* lse, int nthreads) {
  if (!q || !k || !v || !O || Hkv <= 0 || H % Hkv || bs <= 0 || L % bs) return -1;
  if (!rows) n_rows = (int64_t)B * H * L;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (nthreads > n_rows) nthreads = (int)(n_rows > 0 ? n_rows : 1);
  pthread_t th[256];
  attn_job jobs[256];
  for (int i = 0; i < nthreads; ++i) {
    attn_job jb = {q, k, v, dtype, B, H, Hkv, L, d, bs, qs, ks, vs, mask, scale, rows,
                   n_rows * i / nthreads, n_rows * (i + 1) / nthreads, O, lse, 0};
    jobs[i] = jb;
    pthread_create(&th[i], NULL, attn_worker, &jobs[i]);
  }
  int err = 0;
  for (int i = 0; i < nthreads; ++i) {
    pthread_join(th[i], NULL);
    if (jobs[i].err) err = jobs[i].err;
  }
  return err;
}

/* ---------------------------------------------- column-sparse attention */
/*
 * The PulseCol abstract ("PulseCol: periodically refreshed column-sparse
 * attention for diffusion language models", same site, abstract): instead of
 * blocks, a column-sparse pattern -- the key tokens (columns of the attention
 * matrix) a query head keeps for all of its query rows -- found at an early
 * denoising step and refreshed at a few later ones.  The abstract gives no
 * estimator or budget; the reading written out here:
 *
 *   score:   S[b,h,u] = (1/nb) * sum over query blocks i of
 *            softmax over u of (scale * Qbar[b,h,i,:] . k[b,u,h/g,:])
 *            (block-mean queries against every key token)
 *   budget:  Lc = 64 * floor((1 - s) * L / 64 + 0.5) columns per head, at
 *            least 64 (whole 64-key tiles)
 *   select:  the Lc largest S[b,h,u] of each head, ties by the lower u,
 *            listed in ascending u
 *   attend:  for every query token t of head h, softmax over the selected
 *            keys only of (scale * q_t . k_u), times v_u (non-causal)
 */

int64_t oracle_col_budget(int L, double sparsity) {
  if (!(sparsity >= 0.0 && sparsity < 1.0) || L <= 0 || L % 64) return -1;
  int64_t c = 64 * (int64_t)floor((1.0 - sparsity) * (double)L / 64.0 + 0.5);
  if (c < 64) c = 64;
  return c;
}

int oracle_col_scores(const void* q, const void* k, int dtype, int B, int H, int Hkv, int L,
                      int d, int bs, const int64_t* qs, const int64_t* ks, double scale,
                      double* S) {
  if (!q || !k || !S || Hkv <= 0 || H % Hkv || bs <= 0 || L % bs) return -1;
  int nb = L / bs, g = H / Hkv;
  double* qb = (double*)malloc(sizeof(double) * (size_t)B * H * nb * d);
  double* z = (double*)malloc(sizeof(double) * (size_t)L);
  if (!qb || !z) {
    free(qb);
    free(z);
    return -2;
  }
  oracle_pool(q, dtype, B, L, H, d, bs, qs, qb);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      int kh = h / g;
      double* row = S + ((int64_t)b * H + h) * L;
      for (int u = 0; u < L; ++u) row[u] = 0.0;
      for (int i = 0; i < nb; ++i) {
        const double* qi = qb + (((int64_t)b * H + h) * nb + i) * d;
        double m = -INFINITY;
        for (int u = 0; u < L; ++u) {
          double s = 0.0;
          int64_t ko = offs(ks, b, u, kh);
          for (int c = 0; c < d; ++c) s += qi[c] * load_elem(k, dtype, ko + c);
          z[u] = scale * s;
          if (z[u] > m) m = z[u];
        }
        double sum = 0.0;
        for (int u = 0; u < L; ++u) {
          z[u] = exp(z[u] - m);
          sum += z[u];
        }
        for (int u = 0; u < L; ++u) row[u] += z[u] / sum / (double)nb;
      }
    }
  free(qb);
  free(z);
  return 0;
}

typedef struct {
  double s;
  int u;
} colcand;

/* larger score first, then the lower column */
static int colcand_cmp(const void* a, const void* b) {
  const colcand* x = (const colcand*)a;
  const colcand* y = (const colcand*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->u > y->u) - (x->u < y->u);
}

static int int_cmp(const void* a, const void* b) {
  int x = *(const int*)a, y = *(const int*)b;
  return (x > y) - (x < y);
}

/* cols[b, h, 0 .. Lc) ascending; returns Lc or -1 */
int64_t oracle_col_select(const double* S, int B, int H, int L, double sparsity, int32_t* cols) {
  int64_t Lc = oracle_col_budget(L, sparsity);
  if (Lc < 0 || !S || !cols || Lc > L) return -1;
  colcand* c = (colcand*)malloc(sizeof(colcand) * (size_t)L);
  int* pick = (int*)malloc(sizeof(int) * (size_t)Lc);
  if (!c || !pick) {
    free(c);
    free(pick);
    return -1;
  }
  for (int64_t r = 0; r < (int64_t)B * H; ++r) {
    for (int u = 0; u < L; ++u) {
      c[u].s = S[r * L + u];
      c[u].u = u;
    }
    qsort(c, (size_t)L, sizeof(colcand), colcand_cmp);
    for (int64_t x = 0; x < Lc; ++x) pick[x] = c[x].u;
    qsort(pick, (size_t)Lc, sizeof(int), int_cmp);
    for (int64_t x = 0; x < Lc; ++x) cols[r * Lc + x] = pick[x];
  }
  free(c);
  free(pick);
  return Lc;
}

typedef struct {
  const void *q, *k, *v;
  int dtype, B, H, Hkv, L, d;
  const int64_t *qs, *ks, *vs;
  const int32_t* cols;
  int Lc;
  double scale;
  const int64_t* rows;
  int64_t r0, r1;
  double *O, *lse;
  int err;
} colattn_job;

static void* colattn_worker(void* arg) {
  colattn_job* j = (colattn_job*)arg;
  int g = j->H / j->Hkv, d = j->d;
  double* x = (double*)malloc(sizeof(double) * (size_t)j->Lc);
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  double* acc = (double*)malloc(sizeof(double) * (size_t)d);
  if (!x || !qv || !acc) {
    j->err = -2;
    free(x);
    free(qv);
    free(acc);
    return NULL;
  }
  for (int64_t r = j->r0; r < j->r1; ++r) {
    int b, h, t;
    if (j->rows) {
      b = (int)j->rows[3 * r];
      h = (int)j->rows[3 * r + 1];
      t = (int)j->rows[3 * r + 2];
    } else {
      b = (int)(r / ((int64_t)j->H * j->L));
      h = (int)((r / j->L) % j->H);
      t = (int)(r % j->L);
    }
    int kh = h / g;
    const int32_t* cl = j->cols + ((int64_t)b * j->H + h) * j->Lc;
    for (int c = 0; c < d; ++c) qv[c] = load_elem(j->q, j->dtype, offs(j->qs, b, t, h) + c);
    double m = -INFINITY;
    for (int x_ = 0; x_ < j->Lc; ++x_) {
      double s = 0.0;
      int64_t ko = offs(j->ks, b, cl[x_], kh);
      for (int c = 0; c < d; ++c) s += qv[c] * load_elem(j->k, j->dtype, ko + c);
      x[x_] = j->scale * s;
      if (x[x_] > m) m = x[x_];
    }
    double l = 0.0;
    for (int c = 0; c < d; ++c) acc[c] = 0.0;
    for (int x_ = 0; x_ < j->Lc; ++x_) {
      double p = exp(x[x_] - m);
      l += p;
      int64_t vo = offs(j->vs, b, cl[x_], kh);
      for (int c = 0; c < d; ++c) acc[c] += p * load_elem(j->v, j->dtype, vo + c);
    }
    for (int c = 0; c < d; ++c) j->O[r * d + c] = acc[c] / l;
    if (j->lse) j->lse[r] = m + log(l);
  }
  free(x);
  free(qv);
  free(acc);
  return NULL;
}

/* O[r, :] and lse[r] for each requested row r = (b, h, t) (NULL: all, in
 * (b, h, t) order), attending to the Lc columns cols[b, h, :] of each head. */
int oracle_col_attention(const void* q, const void* k, const void* v, int dtype, int B, int H,
                         int Hkv, int L, int d, const int64_t* qs, const int64_t* ks,
                         const int64_t* vs, const int32_t* cols, int Lc, double scale,
                         const int64_t* rows, int64_t n_rows, double* O, double* lse,
                         int nthreads) {
  if (!q || !k || !v || !O || !cols || Lc <= 0 || Hkv <= 0 || H % Hkv) return -1;
  if (!rows) n_rows = (int64_t)B * H * L;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (nthreads > n_rows) nthreads = (int)(n_rows > 0 ? n_rows : 1);
  pthread_t th[256];
  colattn_job jobs[256];
  for (int i = 0; i < nthreads; ++i) {
    colattn_job jb = {q, k, v, dtype, B, H, Hkv, L, d, qs, ks, vs, cols, Lc, scale, rows,
                      n_rows * i / nthreads, n_rows * (i + 1) / nthreads, O, lse, 0};
    jobs[i] = jb;
    pthread_create(&th[i], NULL, colattn_worker, &jobs[i]);
  }
  int err = 0;
  for (int i = 0; i < nthreads; ++i) {
    pthread_join(th[i], NULL);
    if (jobs[i].err) err = jobs[i].err;
  }
  return err;
}
