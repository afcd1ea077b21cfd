/*
 * fp64 CPU oracle for SegPagedAttention prefill.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA path.
 *
 * What it computes (RedKnot pages: README excerpt "Head Classification",
 * "Offline KV Reuse + RoPE Relocation", "SegPagedAttention Runtime"; paooo
 * page "technical principles" and "how to use" sections for the global /
 * local split and the mask-free paged layout):
 *
 *   - RoPE (rotate-half convention, a reading: the pages fix none):
 *       pair m = (m, m + D/2), inv_freq_m = theta^(-2m/D),
 *       R(p) x:  x'_m       = x_m cos(p f_m) - x_{m+D/2} sin(p f_m)
 *                x'_{m+D/2} = x_m sin(p f_m) + x_{m+D/2} cos(p f_m)
 *     Relocation of a cached key stored at position s to logical position
 *     s + delta is R(delta) applied to the stored (already rotated) key.
 *   - Visibility of key j to row i of one (request, layer, kv_head) table:
 *       global / dense : rows = every position; j <= i
 *       local (W)      : rows = uncached positions; i - W < j <= i
 *       retrieval (S)  : rows = uncached positions;
 *                        j <= i and (j uncached or page(j) in S, cached)
 *   - Attention: s_j = scale <q_i, K'_j> over visible j, softmax in fp64,
 *     o_i = sum_j p_j v_j, lse_i = max + ln(sum exp(s - max)).
 *   - Page table of a table: every page of the request holding at least one
 *     key visible to at least one row, ascending logical position, as
 *     (phys_page, logical_pos, delta, n_valid); row set as merged half-open
 *     ranges.  Both are derived by brute force over (row, key) pairs.
 *
 *   - Retrieval page scoring (ora_score_pages, a reading stated there).
 *   - Token importance for the sparse FFN (ora_importance, a reading stated
 *     there): the prefill's softmax weights summed per token over q heads
 *     and computed rows.
 *   - The token-selective FFN itself (ora_sparse_ffn, a reading stated
 *     there): the gated SiLU MLP on the listed rows, residual elsewhere.
 *
 * parity pins: see tests/test_oracle_pins.py (RoPE closed form and
 * composition, causal and windowed SDPA special cases, perturbation
 * invariance, sharing, brute-force vs closed-form page tables, pair counts),
 * tests/test_oracle_scoring.py and tests/test_oracle_importance.py (dense
 * restatement, unit row sums, harmonic closed form, selection brute force),
 * tests/test_oracle_ffn.py (hand-computed values, silu's odd-part identity,
 * zero-gate and scaled-down-projection special cases).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORA_GLOBAL = 0, ORA_LOCAL = 1, ORA_RETRIEVAL = 2, ORA_DENSE = 3 };

typedef struct {
  int32_t n_req, n_layers, hq, hkv, d, p;
  int32_t n_seg;
  const int32_t* seg;        /* [n_seg][5]: req, logical_start, len, stored_pos_base, cached */
  const int32_t* page_base;  /* [n_seg][n_layers*hkv] */
  const int32_t* cu_seqlens; /* [n_req+1] */
  const int8_t* class_map;   /* [n_layers*hkv] */
  const int32_t* class_window; /* [4] */
  const int32_t* retr_indptr;  /* [n_tables+1] */
  const int32_t* retr_pages;
} ora_problem;

/* ---------------------------------------------------------------- helpers */

static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static int req_len(const ora_problem* pr, int r) {
  return pr->cu_seqlens[r + 1] - pr->cu_seqlens[r];
}

/* index of the segment of request r that holds position j, or -1 */
static int seg_at(const ora_problem* pr, int r, int j) {
  for (int s = 0; s < pr->n_seg; ++s) {
    const int32_t* sg = pr->seg + 5 * s;
    if (sg[0] == r && j >= sg[1] && j < sg[1] + sg[2]) return s;
  }
  return -1;
}

/* Per-table view with the request's per-position facts precomputed, so the
 * visibility predicate below is a plain function of (i, j). */
typedef struct {
  const ora_problem* pr;
  int r, layer, kvh, cls, window, L;
  int8_t* uncached;  /* [L] */
  int8_t* in_s;      /* [n_pages_req]: page listed for retrieval and cached */
  int32_t* seg_of;   /* [L] */
} ora_table;

static void table_open(ora_table* t, const ora_problem* pr, int r, int layer, int kvh) {
  t->pr = pr;
  t->r = r;
  t->layer = layer;
  t->kvh = kvh;
  t->cls = pr->class_map[layer * pr->hkv + kvh];
  t->window = pr->class_window[ORA_LOCAL];
  t->L = req_len(pr, r);
  int L = t->L, P = pr->p;
  int npg = (L + P - 1) / P;
  t->uncached = (int8_t*)calloc((size_t)L + 1, 1);
  t->seg_of = (int32_t*)calloc((size_t)L + 1, sizeof(int32_t));
  t->in_s = (int8_t*)calloc((size_t)npg + 1, 1);
  for (int j = 0; j < L; ++j) {
    int s = seg_at(pr, r, j);
    t->seg_of[j] = s;
    t->uncached[j] = (s >= 0 && pr->seg[5 * s + 4] == 0);
  }
  int tid = (r * pr->n_layers + layer) * pr->hkv + kvh;
  if (pr->retr_indptr) {
    for (int k = pr->retr_indptr[tid]; k < pr->retr_indptr[tid + 1]; ++k) {
      int pg = pr->retr_pages[k];
      if (pg >= 0 && pg < npg && !t->uncached[pg * P]) t->in_s[pg] = 1;
    }
  }
}

static void table_close(ora_table* t) {
  free(t->uncached);
  free(t->seg_of);
  free(t->in_s);
}

/* Is position i a computed row of this table? */
static int is_row(const ora_table* t, int i) {
  if (i < 0 || i >= t->L) return 0;
  if (t->cls == ORA_GLOBAL || t->cls == ORA_DENSE) return 1;
  return t->uncached[i];
}

/* Is key j visible to row i? (the definition; no closed forms) */
static int visible(const ora_table* t, int i, int j) {
  if (!is_row(t, i) || j < 0 || j >= t->L || j > i) return 0;
  switch (t->cls) {
    case ORA_GLOBAL:
    case ORA_DENSE:
      return 1;
    case ORA_LOCAL:
      return j > i - t->window;
    case ORA_RETRIEVAL:
      return t->uncached[j] || t->in_s[j / t->pr->p];
  }
  return 0;
}

/* RoPE rotation of a D-vector by position pos, fp64. */
void ora_rope_rotate(const double* x, int d, double theta, double pos, double* y) {
  int h = d / 2;
  for (int m = 0; m < h; ++m) {
    double f = pow(theta, -2.0 * (double)m / (double)d);
    double a = pos * f;
    double c = cos(a), s = sin(a);
    double x0 = x[m], x1 = x[m + h];
    y[m] = x0 * c - x1 * s;
    y[m + h] = x0 * s + x1 * c;
  }
}

/* ------------------------------------------------------- page tables */

/* Brute-force page table and row ranges of one table.
 * entries_out: [cap][4] (phys_page, logical_pos, delta, n_valid);
 * ranges_out: [rcap][2].  Returns 0, or -1 when a capacity is too small. */
int ora_page_table(const ora_problem* pr, int r, int layer, int kvh,
                   int32_t* entries_out, int cap, int* n_entries,
                   int32_t* ranges_out, int rcap, int* n_ranges) {
  ora_table t;
  table_open(&t, pr, r, layer, kvh);
  int L = t.L, P = pr->p, lh = layer * pr->hkv + kvh;
  int ne = 0, nr = 0, rc = 0;
  /* rows of the table, in order */
  int* rows = (int*)malloc(sizeof(int) * ((size_t)L + 1));
  int nrows = 0;
  for (int i = 0; i < L; ++i)
    if (is_row(&t, i)) rows[nrows++] = i;
  for (int k = 0; k * P < L; ++k) {
    int any = 0;
    for (int j = k * P; j < (k + 1) * P && j < L && !any; ++j)
      for (int a = 0; a < nrows && !any; ++a) any = visible(&t, rows[a], j);
    if (!any) continue;
    if (ne >= cap) { rc = -1; break; }
    int s = t.seg_of[k * P];
    const int32_t* sg = pr->seg + 5 * s;
    int page_in_seg = (k * P - sg[1]) / P;
    int stored_pos = sg[3] + page_in_seg * P;
    int nv = L - k * P < P ? L - k * P : P;
    int32_t* e = entries_out + 4 * ne;
    e[0] = pr->page_base[(size_t)s * pr->n_layers * pr->hkv + lh] + page_in_seg;
    e[1] = k * P;
    e[2] = k * P - stored_pos;
    e[3] = nv;
    ++ne;
  }
  for (int i = 0; i < L && rc == 0; ++i) {
    if (!is_row(&t, i)) continue;
    if (nr > 0 && ranges_out[2 * (nr - 1) + 1] == i) {
      ranges_out[2 * (nr - 1) + 1] = i + 1;
    } else {
      if (nr >= rcap) { rc = -1; break; }
      ranges_out[2 * nr] = i;
      ranges_out[2 * nr + 1] = i + 1;
      ++nr;
    }
  }
  free(rows);
  table_close(&t);
  *n_entries = ne;
  *n_ranges = nr;
  return rc;
}

/* ---------------------------------------------------- visible pair count */

/* Number of (row, key) pairs with key visible to row, over rows
 * [row_begin, row_end) of one table (one q head). */
int64_t ora_count_pairs(const ora_problem* pr, int r, int layer, int kvh,
                        int row_begin, int row_end) {
  ora_table t;
  table_open(&t, pr, r, layer, kvh);
  int64_t c = 0;
  if (row_end > t.L) row_end = t.L;
  for (int i = row_begin; i < row_end; ++i) {
    if (!is_row(&t, i)) continue;
    /* visible() is zero for every j > i, so the scan stops at i */
    for (int j = 0; j <= i; ++j) c += visible(&t, i, j);
  }
  table_close(&t);
  return c;
}

/* --------------------------------------------------------- relocation */

/* out[job][row][d] = R(delta) K_stored[src][row][:] in fp64.
 * jobs: [n][3] (src_page, dst_page, delta). */
void ora_relocate(const uint16_t* k_pool, const int32_t* jobs, int n_jobs, int p, int d,
                  double theta, double* out) {
  double* x = (double*)malloc(sizeof(double) * d);
  for (int jb = 0; jb < n_jobs; ++jb) {
    const uint16_t* src = k_pool + (size_t)jobs[3 * jb] * p * d;
    for (int row = 0; row < p; ++row) {
      for (int c = 0; c < d; ++c) x[c] = bf16_to_double(src[(size_t)row * d + c]);
      ora_rope_rotate(x, d, theta, (double)jobs[3 * jb + 2], out + ((size_t)jb * p + row) * d);
    }
  }
  free(x);
}

/* ---------------------------------------------------------- attention */

/* Requested outputs: rows[n][3] = (layer, q_head, token) with token an index
 * into the packed [T] axis; q_rows: bf16 [n][d], the query of each requested
 * row (already rotated to its absolute position); pools: bf16
 * [n_pages][p][d].  o_out: [n][d]; lse_out: [n]; computed_out: [n] = 1 if
 * the row belongs to its table's row set (outputs are 0 / -inf otherwise).
 * The requests are grouped by table here, and each table's relocated keys are
 * built once in fp64. */
typedef struct {
  const ora_problem* pr;
  const uint16_t *q, *kp, *vp;
  double theta, scale;
  const int32_t* rows;
  const int32_t* order; /* request indices sorted by table */
  int n;
  double *o, *lse;
  int32_t* computed;
  /* current table */
  ora_table* tab;
  double *kr, *vr;
  int begin, end, next;
  pthread_mutex_t mu;
} attn_job;

static void attend_row(attn_job* aj, int idx) {
  const ora_problem* pr = aj->pr;
  const ora_table* t = aj->tab;
  int d = pr->d;
  int layer = aj->rows[3 * idx], h = aj->rows[3 * idx + 1], tok = aj->rows[3 * idx + 2];
  int i = tok - pr->cu_seqlens[t->r];
  double* o = aj->o + (size_t)idx * d;
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  if (!is_row(t, i)) {
    aj->lse[idx] = -INFINITY;
    aj->computed[idx] = 0;
    return;
  }
  aj->computed[idx] = 1;
  (void)layer;
  (void)h;
  const uint16_t* qrow = aj->q + (size_t)idx * d;
  double* qd = (double*)malloc(sizeof(double) * d);
  for (int c = 0; c < d; ++c) qd[c] = bf16_to_double(qrow[c]);
  int L = t->L;
  double* s = (double*)malloc(sizeof(double) * ((size_t)L + 1));
  double mx = -INFINITY;
  for (int j = 0; j < L; ++j) {
    if (!visible(t, i, j)) { s[j] = -INFINITY; continue; }
    double acc = 0.0;
    const double* kj = aj->kr + (size_t)j * d;
    for (int c = 0; c < d; ++c) acc += qd[c] * kj[c];
    s[j] = acc * aj->scale;
    if (s[j] > mx) mx = s[j];
  }
  double sum = 0.0;
  if (mx > -INFINITY) {
    for (int j = 0; j < L; ++j) {
      if (s[j] == -INFINITY) continue;
      double w = exp(s[j] - mx);
      sum += w;
      const double* vj = aj->vr + (size_t)j * d;
      for (int c = 0; c < d; ++c) o[c] += w * vj[c];
    }
    for (int c = 0; c < d; ++c) o[c] /= sum;
    aj->lse[idx] = mx + log(sum);
  } else {
    aj->lse[idx] = -INFINITY;
  }
  free(s);
  free(qd);
}

static void* attn_worker(void* arg) {
  attn_job* aj = (attn_job*)arg;
  for (;;) {
    pthread_mutex_lock(&aj->mu);
    int k = aj->next++;
    pthread_mutex_unlock(&aj->mu);
    if (k >= aj->end) break;
    attend_row(aj, aj->order[k]);
  }
  return NULL;
}

static int table_of_request(const ora_problem* pr, const int32_t* row, int* r_out) {
  int tok = row[2], r = 0;
  while (r < pr->n_req && tok >= pr->cu_seqlens[r + 1]) ++r;
  *r_out = r;
  int g = pr->hq / pr->hkv;
  return (r * pr->n_layers + row[0]) * pr->hkv + row[1] / g;
}

static const int32_t* g_sort_keys;
static int cmp_by_key(const void* a, const void* b) {
  int x = *(const int*)a, y = *(const int*)b;
  if (g_sort_keys[x] != g_sort_keys[y]) return g_sort_keys[x] < g_sort_keys[y] ? -1 : 1;
  return x < y ? -1 : (x > y);
}

int ora_attention(const ora_problem* pr, const uint16_t* q_rows, const uint16_t* k_pool,
                  const uint16_t* v_pool, double theta, double scale,
                  const int32_t* rows, int n, double* o_out, double* lse_out,
                  int32_t* computed_out, int n_threads) {
  if (n_threads < 1) n_threads = 1;
  int32_t* key = (int32_t*)malloc(sizeof(int32_t) * (n + 1));
  int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (n + 1));
  for (int k = 0; k < n; ++k) {
    int r;
    key[k] = table_of_request(pr, rows + 3 * k, &r);
    order[k] = k;
  }
  g_sort_keys = key;
  qsort(order, n, sizeof(int32_t), cmp_by_key);
  attn_job aj;
  memset(&aj, 0, sizeof aj);
  aj.pr = pr;
  aj.q = q_rows;
  aj.kp = k_pool;
  aj.vp = v_pool;
  aj.theta = theta;
  aj.scale = scale;
  aj.rows = rows;
  aj.order = order;
  aj.n = n;
  aj.o = o_out;
  aj.lse = lse_out;
  aj.computed = computed_out;
  pthread_mutex_init(&aj.mu, NULL);
  int d = pr->d, P = pr->p;
  int begin = 0;
  while (begin < n) {
    int tid = key[order[begin]];
    int end = begin;
    while (end < n && key[order[end]] == tid) ++end;
    int kvh = tid % pr->hkv, layer = (tid / pr->hkv) % pr->n_layers;
    int r = tid / (pr->hkv * pr->n_layers);
    ora_table t;
    table_open(&t, pr, r, layer, kvh);
    int L = t.L, lh = layer * pr->hkv + kvh;
    /* relocated keys K'_j = R(delta_j) K_stored_j and values, fp64 */
    double* kr = (double*)malloc(sizeof(double) * ((size_t)L * d + 1));
    double* vr = (double*)malloc(sizeof(double) * ((size_t)L * d + 1));
    /* every key of a segment moves by the same delta: R(delta) is formed
     * once per segment (cos / sin of delta * theta^(-2m/D), fp64) */
    int h = d / 2;
    double* cs = (double*)malloc(sizeof(double) * d);
    int cur_seg = -1;
    for (int j = 0; j < L; ++j) {
      int s = t.seg_of[j];
      const int32_t* sg = pr->seg + 5 * s;
      int off = j - sg[1];
      int page = pr->page_base[(size_t)s * pr->n_layers * pr->hkv + lh] + off / P;
      int delta = sg[1] - sg[3];
      if (s != cur_seg) {
        for (int m = 0; m < h; ++m) {
          double a = (double)delta * pow(theta, -2.0 * (double)m / (double)d);
          cs[m] = cos(a);
          cs[h + m] = sin(a);
        }
        cur_seg = s;
      }
      const uint16_t* ks = k_pool + ((size_t)page * P + off % P) * d;
      const uint16_t* vs = v_pool + ((size_t)page * P + off % P) * d;
      double* kj = kr + (size_t)j * d;
      for (int m = 0; m < h; ++m) {
        double x0 = bf16_to_double(ks[m]), x1 = bf16_to_double(ks[m + h]);
        kj[m] = x0 * cs[m] - x1 * cs[h + m];
        kj[m + h] = x0 * cs[h + m] + x1 * cs[m];
      }
      for (int c = 0; c < d; ++c) vr[(size_t)j * d + c] = bf16_to_double(vs[c]);
    }
    free(cs);
    aj.tab = &t;
    aj.kr = kr;
    aj.vr = vr;
    aj.begin = begin;
    aj.end = end;
    aj.next = begin;
    int nt = n_threads < end - begin ? n_threads : end - begin;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (nt + 1));
    for (int k = 0; k < nt; ++k) pthread_create(&th[k], NULL, attn_worker, &aj);
    for (int k = 0; k < nt; ++k) pthread_join(th[k], NULL);
    free(th);
    free(kr);
    free(vr);
    table_close(&t);
    begin = end;
  }
  pthread_mutex_destroy(&aj.mu);
  free(key);
  free(order);
  return 0;
}

/* ------------------------------------------------ retrieval page scoring */

/* Retrieval heads attend the uncached tail plus a list of cached pages that
 * the RedKnot pages say is chosen "by query semantics" (paooo page, "how to
 * use" section, SELECTVISIBLESTATE) without giving a rule.  The reading
 * implemented here, for one retrieval table (r, layer, kvh):
 *   rows     = the table's computed rows (the uncached positions of r);
 *   u        = sum over the G q heads h of kvh of the mean over the rows i of
 *              q[layer][cu[r] + i][h] (queries are given post-RoPE);
 *   cand     = pages pg of r whose keys are cached and whose first position
 *              is at most the last row;
 *   kbar_pg  = mean over the page's n_valid keys of the relocated key
 *              R(delta) K_stored;
 *   score_pg = <u, kbar_pg>;
 *   pick     = the top_k candidates by score (ties to the lower page index),
 *              all candidates when there are at most top_k, in ascending
 *              page order.
 * q: bf16 [n_layers][T][hq][d]; k_pool: bf16 [n_pages][p][d].  pages_out
 * gets the picks; scores_out[pg] (length = pages of the request) gets each
 * candidate's score and NaN elsewhere.  Returns the number of picks (0 for a
 * table of another class or without rows). */
int ora_score_pages(const ora_problem* pr, const uint16_t* q, const uint16_t* k_pool,
                    double theta, int top_k, int r, int layer, int kvh, int32_t* pages_out,
                    double* scores_out) {
  ora_table t;
  table_open(&t, pr, r, layer, kvh);
  int L = t.L, P = pr->p, d = pr->d, h = d / 2;
  int npg = (L + P - 1) / P;
  int T = pr->cu_seqlens[pr->n_req];
  for (int pg = 0; pg < npg; ++pg) scores_out[pg] = NAN;
  int n_out = 0;
  int last_row = -1, n_rows = 0;
  for (int i = 0; i < L; ++i)
    if (is_row(&t, i)) {
      last_row = i;
      ++n_rows;
    }
  if (t.cls != ORA_RETRIEVAL || n_rows == 0) {
    table_close(&t);
    return 0;
  }
  int g = pr->hq / pr->hkv;
  double* u = (double*)calloc((size_t)d, sizeof(double));
  for (int hh = kvh * g; hh < kvh * g + g; ++hh) {
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int i = 0; i < L; ++i) {
        if (!is_row(&t, i)) continue;
        size_t off = (((size_t)layer * T + pr->cu_seqlens[r] + i) * pr->hq + hh) * d + c;
        acc += bf16_to_double(q[off]);
      }
      u[c] += acc / n_rows;
    }
  }
  int lh = layer * pr->hkv + kvh;
  double* kbar = (double*)malloc(sizeof(double) * d);
  double* kr = (double*)malloc(sizeof(double) * d);
  double* x = (double*)malloc(sizeof(double) * d);
  int* cand = (int*)malloc(sizeof(int) * ((size_t)npg + 1));
  int n_cand = 0;
  for (int pg = 0; pg < npg; ++pg) {
    int j0 = pg * P;
    if (t.uncached[j0] || j0 > last_row) continue;
    int s = t.seg_of[j0];
    const int32_t* sg = pr->seg + 5 * s;
    const int shift = sg[1] - sg[3]; /* the page's relocation delta */
    int nv = L - j0 < P ? L - j0 : P;
    for (int c = 0; c < d; ++c) kbar[c] = 0.0;
    for (int rr = 0; rr < nv; ++rr) {
      int off = j0 + rr - sg[1];
      int page = pr->page_base[(size_t)s * pr->n_layers * pr->hkv + lh] + off / P;
      const uint16_t* ks = k_pool + ((size_t)page * P + off % P) * d;
      for (int c = 0; c < d; ++c) x[c] = bf16_to_double(ks[c]);
      ora_rope_rotate(x, d, theta, (double)shift, kr);
      for (int c = 0; c < d; ++c) kbar[c] += kr[c];
    }
    double sc = 0.0;
    for (int c = 0; c < d; ++c) sc += u[c] * (kbar[c] / nv);
    scores_out[pg] = sc;
    cand[n_cand++] = pg;
  }
  (void)h;
  /* top_k by repeated selection of the best remaining candidate */
  int8_t* taken = (int8_t*)calloc((size_t)npg + 1, 1);
  int n_pick = n_cand < top_k ? n_cand : top_k;
  for (int k = 0; k < n_pick; ++k) {
    int best = -1;
    for (int a = 0; a < n_cand; ++a) {
      int pg = cand[a];
      if (taken[pg]) continue;
      if (best < 0 || scores_out[pg] > scores_out[best]) best = pg;
    }
    taken[best] = 1;
  }
  for (int pg = 0; pg < npg; ++pg)
    if (taken[pg]) pages_out[n_out++] = pg;
  free(taken);
  free(cand);
  free(x);
  free(kr);
  free(kbar);
  free(u);
  table_close(&t);
  return n_out;
}

/* ------------------------------------------------- attention importance */

/* Token importance for the sparse FFN.  The RedKnot pages send the tokens with
 * the highest attention scores through the dense FFN and the rest along the
 * residual path (README "About", Elastic Sparsity / Sparse FFN; paooo page,
 * "main functions" and "core advantages"), without a formula.  The reading
 * implemented here, for request r and one layer:
 *   I(j) = sum over the layer's q heads h, and over the rows i that the
 *          table of h's kv head computes, of the softmax weight
 *          P_h(i, j) = exp(scale * q_h(i) . K'_j - lse_h(i)),
 *          zero where j is not visible to i,
 * with K'_j = R(delta_j) K_stored_j the relocated key and lse_h(i) the
 * row's log-sum-exp over its visible keys: the weight the prefill's own
 * attention gives key j at row i, summed.  Each row's weights sum to 1, so
 * the I(j) add up to the number of computed (q head, row) pairs.
 * q: bf16 [n_layers][T][hq][d]; k_pool: bf16 [n_pages][p][d]; imp_out [L].
 * fp64 throughout; each row's softmax by definition (max-subtracted). */
int ora_importance(const ora_problem* pr, const uint16_t* q, const uint16_t* k_pool,
                   double theta, double scale, int r, int layer, double* imp_out) {
  int L = req_len(pr, r), d = pr->d, P = pr->p, hh = d / 2;
  int g = pr->hq / pr->hkv, T = pr->cu_seqlens[pr->n_req];
  for (int j = 0; j < L; ++j) imp_out[j] = 0.0;
  double* kr = (double*)malloc(sizeof(double) * ((size_t)L * d + 1));
  double* s = (double*)malloc(sizeof(double) * ((size_t)L + 1));
  double* qd = (double*)malloc(sizeof(double) * d);
  for (int kvh = 0; kvh < pr->hkv; ++kvh) {
    ora_table t;
    table_open(&t, pr, r, layer, kvh);
    int lh = layer * pr->hkv + kvh;
    /* relocated keys of the whole request for this kv head */
    for (int j = 0; j < L; ++j) {
      int sgi = t.seg_of[j];
      const int32_t* sg = pr->seg + 5 * sgi;
      int off = j - sg[1];
      int page = pr->page_base[(size_t)sgi * pr->n_layers * pr->hkv + lh] + off / P;
      int dpos = sg[1] - sg[3];
      const uint16_t* ks = k_pool + ((size_t)page * P + off % P) * d;
      double* kj = kr + (size_t)j * d;
      for (int m = 0; m < hh; ++m) {
        double a = (double)dpos * pow(theta, -2.0 * (double)m / (double)d);
        double x0 = bf16_to_double(ks[m]), x1 = bf16_to_double(ks[m + hh]);
        kj[m] = x0 * cos(a) - x1 * sin(a);
        kj[m + hh] = x0 * sin(a) + x1 * cos(a);
      }
    }
    for (int hg = 0; hg < g; ++hg) {
      int h = kvh * g + hg;
      for (int i = 0; i < L; ++i) {
        if (!is_row(&t, i)) continue;
        const uint16_t* qrow = q + (((size_t)layer * T + pr->cu_seqlens[r] + i) * pr->hq + h) * d;
        for (int c = 0; c < d; ++c) qd[c] = bf16_to_double(qrow[c]);
        double mx = -INFINITY;
        for (int j = 0; j < L; ++j) {
          if (!visible(&t, i, j)) { s[j] = -INFINITY; continue; }
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += qd[c] * kr[(size_t)j * d + c];
          s[j] = acc * scale;
          if (s[j] > mx) mx = s[j];
        }
        if (mx == -INFINITY) continue;
        double sum = 0.0;
        for (int j = 0; j < L; ++j)
          if (s[j] > -INFINITY) sum += exp(s[j] - mx);
        double lse = mx + log(sum);
        for (int j = 0; j < L; ++j)
          if (s[j] > -INFINITY) imp_out[j] += exp(s[j] - lse);
      }
    }
    table_close(&t);
  }
  free(kr);
  free(s);
  free(qd);
  return 0;
}

/* ------------------------------------------------------------ sparse FFN */

/* Token-selective FFN (README "About", Elastic Sparsity / Sparse FFN; paooo
 * page, "main functions": the tokens with the highest attention scores run
 * the dense FFN, the others take the residual path).  The pages name the
 * Mistral-7B and Qwen3 families, whose FFN is the gated SiLU MLP; the
 * reading implemented here, for every listed row i of the hidden state x:
 *   g_f = sum_c x_ic Wg_fc,   u_f = sum_c x_ic Wu_fc        (f < d_ff)
 *   h_f = silu(g_f) u_f,      silu(z) = z / (1 + exp(-z))
 *   y_in = x_in + sum_f h_f Wd_nf                           (n < d_model)
 * and y_i = x_i for every other row (the residual path, not computed here).
 * x: bf16 [.][d_model]; Wg, Wu: bf16 [d_ff][d_model]; Wd: bf16
 * [d_model][d_ff] (rows are output features, as in a linear layer's
 * weight); rows: the listed row indices; y_out: fp64 [n_rows][d_model].
 * fp64 throughout, no intermediate rounding. */
typedef struct {
  const uint16_t *x, *wg, *wu, *wd;
  const int32_t* rows;
  int n_rows, d_model, d_ff;
  double* y;
  int next;
  pthread_mutex_t mu;
} ffn_job;

static void ffn_row(ffn_job* j, int k) {
  int dm = j->d_model, df = j->d_ff;
  const uint16_t* xr = j->x + (size_t)j->rows[k] * dm;
  double* xd = (double*)malloc(sizeof(double) * dm);
  double* h = (double*)malloc(sizeof(double) * df);
  for (int c = 0; c < dm; ++c) xd[c] = bf16_to_double(xr[c]);
  for (int f = 0; f < df; ++f) {
    const uint16_t* wgr = j->wg + (size_t)f * dm;
    const uint16_t* wur = j->wu + (size_t)f * dm;
    double g = 0.0, u = 0.0;
    for (int c = 0; c < dm; ++c) {
      g += xd[c] * bf16_to_double(wgr[c]);
      u += xd[c] * bf16_to_double(wur[c]);
    }
    h[f] = g / (1.0 + exp(-g)) * u;
  }
  double* y = j->y + (size_t)k * dm;
  for (int n = 0; n < dm; ++n) {
    const uint16_t* wdr = j->wd + (size_t)n * df;
    double acc = 0.0;
    for (int f = 0; f < df; ++f) acc += h[f] * bf16_to_double(wdr[f]);
    y[n] = xd[n] + acc;
  }
  free(xd);
  free(h);
}

static void* ffn_worker(void* arg) {
  ffn_job* j = (ffn_job*)arg;
  for (;;) {
    pthread_mutex_lock(&j->mu);
    int k = j->next++;
    pthread_mutex_unlock(&j->mu);
    if (k >= j->n_rows) return NULL;
    ffn_row(j, k);
  }
}

int ora_sparse_ffn(const uint16_t* x, int d_model, const int32_t* rows, int n_rows,
                   const uint16_t* wg, const uint16_t* wu, const uint16_t* wd, int d_ff,
                   double* y_out, int n_threads) {
  ffn_job j;
  j.x = x;
  j.wg = wg;
  j.wu = wu;
  j.wd = wd;
  j.rows = rows;
  j.n_rows = n_rows;
  j.d_model = d_model;
  j.d_ff = d_ff;
  j.y = y_out;
  j.next = 0;
  pthread_mutex_init(&j.mu, NULL);
  if (n_threads < 1) n_threads = 1;
  if (n_threads > n_rows) n_threads = n_rows > 0 ? n_rows : 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * n_threads);
  for (int k = 0; k < n_threads; ++k) pthread_create(&th[k], NULL, ffn_worker, &j);
  for (int k = 0; k < n_threads; ++k) pthread_join(th[k], NULL);
  free(th);
  pthread_mutex_destroy(&j.mu);
  return 0;
}
