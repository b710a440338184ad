/*
 * nsa_oracle.c -- plain, slow, fp64 CPU oracle for the forward pass of Native Sparse
 * Attention (NSA) over video tokens, as adapted by VideoNSA.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU
 * baseline may load this library. It shares no code, header, table or helper with the
 * CUDA path in sparse_attention_long_fwd_b200/, and it never calls it.
 *
 * What it computes, row by row (one query token t, all heads), in fp64:
 *   - three branches -- compression, selection and sliding window -- combined per
 *     token and head by gates ("VideoNSA" news article at top168.com, section
 *     "一、革命性的三重注意机制"; CSDN blog "VideoNSA：重新定义视频理解的稀疏注意力机制",
 *     section 2.2 "VideoNSA的三分支创新架构");
 *   - dense causal attention for text tokens, NSA for video tokens (shd-paper.top page
 *     "VideoNSA: Native Sparse Attention Scales Video Understanding", abstract);
 *   - the selection branch scores blocks of video tokens and keeps the most important
 *     ones (top168.com article, section 一, the selection-branch paragraph).
 * The pages fix none of the constants or formulas below; where they are silent the
 * plainest reading is taken (each one is named at the function that uses it):
 *   compression   Kc[i] = bf16_rne(mean_{u<l} K[i*s+u]), complete blocks only; the
 *                 learnable form weights the l positions per head instead of averaging;
 *   cmp branch    block i visible to t iff i*s + l - 1 <= t; softmax over visible blocks;
 *   block scores  score[j] = sum_{h in group} sum_i P_h[i] * |tokens(i) & tokens(j)| / l;
 *   selection     blocks 0, j_t and j_t-1 always kept (j_t = t / l'); the remaining
 *                 top_n - |forced| by (score desc, index asc); result ascending, -1 padded;
 *   sel branch    softmax over tokens tau <= t of the selected blocks;
 *   win branch    softmax over tokens max(0, t-w+1) .. t;
 *   combine       out = g_cmp*o_cmp + g_sel*o_sel + g_win*o_win (gates used as given);
 *   text rows     t >= n_video: dense causal softmax over 0..t.
 * The GQA group of query head h is h / (hq / hkv).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int n_tokens;   /* N: keys available (prefill) / cache capacity (decode) */
  int n_video;    /* N_v: leading tokens handled by NSA; rows >= N_v are text */
  int hq, hkv, d; /* query heads, key/value heads, head dim */
  int cmp_len;    /* l  : compression block length */
  int cmp_stride; /* s  : compression stride */
  int sel_len;    /* l' : selection block length */
  int top_n;      /* n  : selected blocks per (token, group), forced ones included */
  int window;     /* w  : sliding-window length, t itself included */
  double scale;   /* softmax scale applied to q.k */
} oracle_cfg;

/* ------------------------------------------------------------ bf16 <-> fp64 */

double oracle_bf16_to_double(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round a double straight to the nearest bfloat16 (8-bit exponent, 7 stored mantissa
 * bits), ties to even, with one rounding (no detour through float). */
uint16_t oracle_double_to_bf16(double x) {
  const uint16_t sign = signbit(x) ? 0x8000u : 0u;
  if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
  if (isinf(x)) return (uint16_t)(sign | 0x7F80u);
  const double a = fabs(x);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);       /* a = m * 2^e, m in [0.5, 1): floor(log2 a) = e - 1 */
  int ex = e - 1;
  if (ex < -126) ex = -126; /* subnormal bf16 values are spaced 2^-133 apart */
  const double ulp = ldexp(1.0, ex - 7);
  const double r = nearbyint(a / ulp) * ulp; /* a / ulp is exact; default mode = ties to even */
  if (r > 3.3895313892515355e38) return (uint16_t)(sign | 0x7F80u); /* beyond the largest bf16 */
  const float f = (float)r; /* exact: every bf16 value is a float */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(sign | ((u >> 16) & 0x7FFFu));
}

/* Element-wise oracle_double_to_bf16 over an array (used by the tests). */
void oracle_round_bf16_array(const double* x, uint16_t* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = oracle_double_to_bf16(x[i]);
}

/* ------------------------------------------------------------ block counts */

/* Number of complete compression blocks among the first T tokens. */
int oracle_num_cmp(int T, int l, int s) { return T >= l ? (T - l) / s + 1 : 0; }

/* Number of selection blocks covering the first T tokens. */
int oracle_num_sel(int T, int lsel) { return (T + lsel - 1) / lsel; }

/* ------------------------------------------------------------ compression */

/* Compression branch: every complete block of l tokens, taken at stride s, is
 * summarised by the mean of its keys (values), rounded once to bf16. The pages only say
 * that consecutive content is merged into representative summaries (top168.com article,
 * section 一, the compression-branch paragraph); a plain mean with no learned weights
 * is the reading taken here.
 * k: [T][h][d] bf16 bits; kc: [Ncmp(T)][h][d] bf16 bits. */
void oracle_compress(const uint16_t* k, int T, int h, int d, int l, int s, uint16_t* kc) {
  const int nc = oracle_num_cmp(T, l, s);
  for (int i = 0; i < nc; ++i)
    for (int g = 0; g < h; ++g)
      for (int c = 0; c < d; ++c) {
        double sum = 0.0;
        for (int u = 0; u < l; ++u) sum += oracle_bf16_to_double(k[((size_t)(i * s + u) * h + g) * d + c]);
        kc[((size_t)i * h + g) * d + c] = oracle_double_to_bf16(sum / (double)l);
      }
}

/* Learnable compression: the sparse pattern is steered by learned parameters
 * (shd-paper.top page "VideoNSA: Native Sparse Attention Scales Video Understanding",
 * section "方法详解", key design (1)). The page gives no form for them; the reading here
 * is the plainest learnable version of the mean above: a per-head linear map over the l
 * positions of a block, Kc[i][g] = bf16_rne(sum_u w[g][u] * K[i*s+u][g]), with w = 1/l
 * giving the mean. Each product of an fp32 weight and a bf16 key is exact in fp64 and the
 * sum runs in token order, rounded once.
 * k: [T][h][d] bf16 bits; w: [h][l] fp32; kc: [Ncmp(T)][h][d] bf16 bits. */
void oracle_compress_weighted(const uint16_t* k, const float* w, int T, int h, int d, int l, int s, uint16_t* kc) {
  const int nc = oracle_num_cmp(T, l, s);
  for (int i = 0; i < nc; ++i)
    for (int g = 0; g < h; ++g)
      for (int c = 0; c < d; ++c) {
        double sum = 0.0;
        for (int u = 0; u < l; ++u)
          sum += (double)w[(size_t)g * l + u] * oracle_bf16_to_double(k[((size_t)(i * s + u) * h + g) * d + c]);
        kc[((size_t)i * h + g) * d + c] = oracle_double_to_bf16(sum);
      }
}

/* ------------------------------------------------------------ attention */

/* Softmax attention of one query row (already converted to double) over an explicit list
 * of key positions. K, V: bf16 rows with `stride` elements between positions; the head's
 * slice starts at offset `col0`. Writes o[d], returns the log-sum-exp of the scaled
 * scores (natural log); optionally stores the normalised probabilities in prob[]. */
static double attend_list(const double* q, const uint16_t* K, const uint16_t* V, size_t stride, size_t col0,
                          int d, double scale, const int* keys, int nkeys, double* z, double* prob, double* o) {
  double m = -INFINITY;
  for (int a = 0; a < nkeys; ++a) {
    const uint16_t* kr = K + (size_t)keys[a] * stride + col0;
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += q[c] * oracle_bf16_to_double(kr[c]);
    z[a] = scale * dot;
    if (z[a] > m) m = z[a];
  }
  double sum = 0.0;
  for (int a = 0; a < nkeys; ++a) {
    z[a] = exp(z[a] - m);
    sum += z[a];
  }
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  for (int a = 0; a < nkeys; ++a) {
    const double p = z[a] / sum;
    if (prob) prob[a] = p;
    const uint16_t* vr = V + (size_t)keys[a] * stride + col0;
    for (int c = 0; c < d; ++c) o[c] += p * oracle_bf16_to_double(vr[c]);
  }
  return m + log(sum);
}

typedef struct {
  int* keys;      /* key positions of one branch */
  double* z;      /* scores / exp scratch */
  double* prob;   /* cmp-branch probabilities */
  double* qd;     /* query row in double */
  double* bins;   /* block scores of one group */
  int* cand;      /* candidate blocks */
  double* ocmp;   /* per-head branch outputs [hq][d] */
  double* osel;
  double* owin;
} scratch_t;

typedef struct {
  double score;
  int idx;
} cand_t;

/* Selection order: higher score first, lower block index first among equal scores. */
static int cmp_cand(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->idx > b->idx) - (a->idx < b->idx);
}

static int cmp_int(const void* pa, const void* pb) {
  const int a = *(const int*)pa, b = *(const int*)pb;
  return (a > b) - (a < b);
}

/* Outputs of one row; every pointer may be NULL except out. */
typedef struct {
  double* out;     /* [hq][d] */
  int* sel;        /* [hkv][top_n] */
  double* scores;  /* [hkv][nsel_w] */
  int nsel_w;
  double* o_cmp;   /* [hq][d] */
  double* lse;     /* [hq] cmp-branch log-sum-exp */
  double* o_sel;   /* [hq][d] */
  double* o_win;   /* [hq][d] */
  double* tie_gap; /* [hkv] */
  double* lse_sel; /* [hq] selected-branch log-sum-exp */
  double* lse_win; /* [hq] window-branch log-sum-exp */
} row_out_t;

/* One NSA (video) row at position t. K, V: [*][hkv][d] token rows of the sequence;
 * KC, VC: [*][hkv][d] compressed rows. sel_override: NULL or [hkv][top_n] block lists
 * (ascending, -1 padded) to use instead of the row's own selection (replay). */
static void video_row(const oracle_cfg* c, int t, const uint16_t* qrow, const uint16_t* K, const uint16_t* V,
                      const uint16_t* KC, const uint16_t* VC, const float* grow, const int* sel_override,
                      const row_out_t* ro, scratch_t* w) {
  const int d = c->d, hkv = c->hkv, G = c->hq / c->hkv;
  const int l = c->cmp_len, s = c->cmp_stride, ls = c->sel_len;
  const size_t stride = (size_t)hkv * d;
  const int nc = oracle_num_cmp(t + 1, l, s); /* block i visible iff i*s + l - 1 <= t */
  const int jt = t / ls;                       /* selection block holding t */
  for (int g = 0; g < hkv; ++g) {
    /* ---- compression branch, and block scores from its probabilities */
    for (int j = 0; j <= jt; ++j) w->bins[j] = 0.0;
    for (int a = 0; a < nc; ++a) w->keys[a] = a;
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      double* ocmp = w->ocmp + (size_t)h * d;
      for (int e = 0; e < d; ++e) w->qd[e] = oracle_bf16_to_double(qrow[(size_t)h * d + e]);
      double lse = -INFINITY;
      if (nc > 0) {
        lse = attend_list(w->qd, KC, VC, stride, (size_t)g * d, d, c->scale, w->keys, nc, w->z, w->prob, ocmp);
        /* token-overlap weighting of compression block i onto selection block j */
        for (int i = 0; i < nc; ++i) {
          const int b0 = i * s, b1 = i * s + l; /* tokens [b0, b1) */
          for (int j = b0 / ls; j <= (b1 - 1) / ls; ++j) {
            const int lo = b0 > j * ls ? b0 : j * ls;
            const int hi = b1 < (j + 1) * ls ? b1 : (j + 1) * ls;
            if (hi > lo) w->bins[j] += w->prob[i] * (double)(hi - lo) / (double)l;
          }
        }
      } else {
        for (int e = 0; e < d; ++e) ocmp[e] = 0.0;
      }
      if (ro->lse) ro->lse[h] = lse;
    }
    if (ro->scores) {
      for (int j = 0; j < ro->nsel_w; ++j) ro->scores[(size_t)g * ro->nsel_w + j] = (j <= jt) ? w->bins[j] : 0.0;
    }
    /* ---- selection: forced {0, jt, jt-1}, then the best of the rest */
    int chosen[512];
    int nchosen = 0;
    double gap = INFINITY;
    if (sel_override) {
      for (int a = 0; a < c->top_n; ++a)
        if (sel_override[g * c->top_n + a] >= 0) chosen[nchosen++] = sel_override[g * c->top_n + a];
    } else {
      int forced[3], nf = 0;
      forced[nf++] = 0;
      if (jt > 0) forced[nf++] = jt;
      if (jt - 1 > 0) forced[nf++] = jt - 1;
      cand_t* cand = (cand_t*)w->cand;
      int ncand = 0;
      for (int j = 0; j <= jt; ++j) {
        int is_forced = 0;
        for (int a = 0; a < nf; ++a) is_forced |= (forced[a] == j);
        if (!is_forced) {
          cand[ncand].score = w->bins[j];
          cand[ncand].idx = j;
          ++ncand;
        }
      }
      qsort(cand, (size_t)ncand, sizeof(cand_t), cmp_cand);
      int k = c->top_n - nf;
      if (k < 0) k = 0;
      if (k > ncand) k = ncand;
      for (int a = 0; a < nf; ++a) chosen[nchosen++] = forced[a];
      for (int a = 0; a < k; ++a) chosen[nchosen++] = cand[a].idx;
      if (k > 0 && k < ncand) {
        const double hi = cand[k - 1].score, lo = cand[k].score;
        gap = hi > 0.0 ? (hi - lo) / hi : 0.0;
      }
    }
    qsort(chosen, (size_t)nchosen, sizeof(int), cmp_int);
    if (ro->sel) {
      for (int a = 0; a < c->top_n; ++a) ro->sel[g * c->top_n + a] = a < nchosen ? chosen[a] : -1;
    }
    if (ro->tie_gap) ro->tie_gap[g] = gap;
    /* ---- selection-branch and window-branch key sets */
    int nsk = 0;
    for (int a = 0; a < nchosen; ++a)
      for (int tau = chosen[a] * ls; tau < (chosen[a] + 1) * ls && tau <= t; ++tau) w->keys[nsk++] = tau;
    int* wkeys = w->keys + nsk;
    int nwk = 0;
    for (int tau = (t - c->window + 1 > 0 ? t - c->window + 1 : 0); tau <= t; ++tau) wkeys[nwk++] = tau;
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      for (int e = 0; e < d; ++e) w->qd[e] = oracle_bf16_to_double(qrow[(size_t)h * d + e]);
      double* osel = w->osel + (size_t)h * d;
      double* owin = w->owin + (size_t)h * d;
      const double lsel = attend_list(w->qd, K, V, stride, (size_t)g * d, d, c->scale, w->keys, nsk, w->z, NULL, osel);
      const double lwin = attend_list(w->qd, K, V, stride, (size_t)g * d, d, c->scale, wkeys, nwk, w->z, NULL, owin);
      if (ro->lse_sel) ro->lse_sel[h] = lsel;
      if (ro->lse_win) ro->lse_win[h] = lwin;
      /* gated combine, gates ordered (cmp, sel, win), used as given */
      const double g0 = grow[h * 3 + 0], g1 = grow[h * 3 + 1], g2 = grow[h * 3 + 2];
      const double* ocmp = w->ocmp + (size_t)h * d;
      for (int e = 0; e < d; ++e) ro->out[(size_t)h * d + e] = g0 * ocmp[e] + g1 * osel[e] + g2 * owin[e];
    }
  }
  if (ro->o_cmp) memcpy(ro->o_cmp, w->ocmp, sizeof(double) * (size_t)c->hq * d);
  if (ro->o_sel) memcpy(ro->o_sel, w->osel, sizeof(double) * (size_t)c->hq * d);
  if (ro->o_win) memcpy(ro->o_win, w->owin, sizeof(double) * (size_t)c->hq * d);
}

/* Text row at position t (hybrid scheme): dense causal attention over tokens 0..t. */
static void text_row(const oracle_cfg* c, int t, const uint16_t* qrow, const uint16_t* K, const uint16_t* V,
                     const row_out_t* ro, scratch_t* w) {
  const int d = c->d, G = c->hq / c->hkv;
  const size_t stride = (size_t)c->hkv * d;
  for (int tau = 0; tau <= t; ++tau) w->keys[tau] = tau;
  for (int h = 0; h < c->hq; ++h) {
    for (int e = 0; e < d; ++e) w->qd[e] = oracle_bf16_to_double(qrow[(size_t)h * d + e]);
    attend_list(w->qd, K, V, stride, (size_t)(h / G) * d, d, c->scale, w->keys, t + 1, w->z, NULL,
                ro->out + (size_t)h * d);
  }
}

static int cfg_ok(const oracle_cfg* c) {
  if (!c) return 0;
  if (c->n_tokens < 1 || c->n_video < 0 || c->n_video > c->n_tokens) return 0;
  if (c->hq < 1 || c->hkv < 1 || c->hq % c->hkv != 0 || c->d < 1) return 0;
  if (c->cmp_len < 1 || c->cmp_stride < 1 || c->sel_len < 1 || c->window < 1) return 0;
  if (c->top_n < 1 || c->top_n > 500) return 0;
  return 1;
}

static int alloc_scratch(scratch_t* w, const oracle_cfg* c) {
  const size_t nmax = (size_t)c->n_tokens + 2 * (size_t)c->sel_len + (size_t)c->window + 8;
  const size_t nsel = (size_t)oracle_num_sel(c->n_tokens, c->sel_len) + 8;
  w->keys = (int*)malloc(sizeof(int) * 2 * nmax);
  w->z = (double*)malloc(sizeof(double) * nmax);
  w->prob = (double*)malloc(sizeof(double) * nmax);
  w->qd = (double*)malloc(sizeof(double) * (size_t)c->d);
  w->bins = (double*)malloc(sizeof(double) * nsel);
  w->cand = (int*)malloc(sizeof(cand_t) * nsel);
  w->ocmp = (double*)malloc(sizeof(double) * (size_t)c->hq * c->d);
  w->osel = (double*)malloc(sizeof(double) * (size_t)c->hq * c->d);
  w->owin = (double*)malloc(sizeof(double) * (size_t)c->hq * c->d);
  return w->keys && w->z && w->prob && w->qd && w->bins && w->cand && w->ocmp && w->osel && w->owin;
}

static void free_scratch(scratch_t* w) {
  free(w->keys); free(w->z); free(w->prob); free(w->qd); free(w->bins);
  free(w->cand); free(w->ocmp); free(w->osel); free(w->owin);
}

/* Prefill rows. q: [N][hq][d], k, v: [N][hkv][d], gates: [N][hq][3] (cmp, sel, win),
 * kc, vc: [Ncmp(N_v)][hkv][d] from oracle_compress over the video prefix.
 * rows: nrows token positions. Per-row outputs are indexed by the position in rows[]:
 * out [nrows][hq][d]; sel [nrows][hkv][top_n]; scores [nrows][hkv][nsel_w];
 * o_cmp/o_sel/o_win [nrows][hq][d]; lse (compressed branch), lse_sel, lse_win [nrows][hq];
 * tie_gap [nrows][hkv]. For text rows only out is written. Returns 0, or -1 on invalid
 * arguments. */
int oracle_prefill_rows(const oracle_cfg* c, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const float* gates, const uint16_t* kc, const uint16_t* vc, int nrows, const int* rows,
                        const int* sel_override, double* out, int* sel, double* scores, int nsel_w, double* o_cmp,
                        double* lse, double* o_sel, double* o_win, double* tie_gap, double* lse_sel,
                        double* lse_win, int nthreads) {
  if (!cfg_ok(c) || !q || !k || !v || !gates || !out || nrows < 0 || (nrows > 0 && !rows)) return -1;
  for (int r = 0; r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= c->n_tokens) return -1;
  const int hq = c->hq, hkv = c->hkv, d = c->d, n = c->top_n;
  int bad = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel reduction(| : bad)
#endif
  {
    scratch_t w;
    if (!alloc_scratch(&w, c)) {
      bad = 1;
    } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int r = 0; r < nrows; ++r) {
        const int t = rows[r];
        row_out_t ro;
        ro.out = out + (size_t)r * hq * d;
        ro.sel = sel ? sel + (size_t)r * hkv * n : NULL;
        ro.scores = scores ? scores + (size_t)r * hkv * nsel_w : NULL;
        ro.nsel_w = nsel_w;
        ro.o_cmp = o_cmp ? o_cmp + (size_t)r * hq * d : NULL;
        ro.lse = lse ? lse + (size_t)r * hq : NULL;
        ro.o_sel = o_sel ? o_sel + (size_t)r * hq * d : NULL;
        ro.o_win = o_win ? o_win + (size_t)r * hq * d : NULL;
        ro.tie_gap = tie_gap ? tie_gap + (size_t)r * hkv : NULL;
        ro.lse_sel = lse_sel ? lse_sel + (size_t)r * hq : NULL;
        ro.lse_win = lse_win ? lse_win + (size_t)r * hq : NULL;
        const uint16_t* qrow = q + (size_t)t * hq * d;
        if (t < c->n_video) {
          video_row(c, t, qrow, k, v, kc, vc, gates + (size_t)t * hq * 3,
                    sel_override ? sel_override + (size_t)r * hkv * n : NULL, &ro, &w);
        } else {
          text_row(c, t, qrow, k, v, &ro, &w);
        }
      }
      free_scratch(&w);
    }
  }
  return bad ? -1 : 0;
}

/* Single-query decode: sequence b holds seq_lens[b] = L tokens in kcache/vcache
 * ([B][Lmax][hkv][d]); its query (position L-1, already in the cache) is q[b] ([B][hq][d]);
 * kcmp/vcmp ([B][Ncmp(Lmax)][hkv][d]) are the caller's compressed caches, used as given.
 * cfg.n_tokens = Lmax. seqs: the nseq sequences to evaluate; per-sequence outputs are
 * laid out like oracle_prefill_rows' per-row outputs. Returns 0, or -1 on bad arguments. */
int oracle_decode(const oracle_cfg* c, const uint16_t* q, const uint16_t* kcache, const uint16_t* vcache,
                  const uint16_t* kcmp, const uint16_t* vcmp, const int* seq_lens, const float* gates, int nseq,
                  const int* seqs, const int* sel_override, double* out, int* sel, double* scores, int nsel_w,
                  double* o_cmp, double* lse, double* o_sel, double* o_win, double* tie_gap, int nthreads) {
  if (!cfg_ok(c) || !q || !kcache || !vcache || !kcmp || !vcmp || !seq_lens || !gates || !out || nseq < 0 ||
      (nseq > 0 && !seqs))
    return -1;
  const int hq = c->hq, hkv = c->hkv, d = c->d, n = c->top_n, Lmax = c->n_tokens;
  const int ncmax = oracle_num_cmp(Lmax, c->cmp_len, c->cmp_stride);
  for (int r = 0; r < nseq; ++r)
    if (seq_lens[seqs[r]] < 1 || seq_lens[seqs[r]] > Lmax) return -1;
  int bad = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel reduction(| : bad)
#endif
  {
    scratch_t w;
    if (!alloc_scratch(&w, c)) {
      bad = 1;
    } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int r = 0; r < nseq; ++r) {
        const int b = seqs[r];
        const int L = seq_lens[b];
        row_out_t ro;
        ro.out = out + (size_t)r * hq * d;
        ro.sel = sel ? sel + (size_t)r * hkv * n : NULL;
        ro.scores = scores ? scores + (size_t)r * hkv * nsel_w : NULL;
        ro.nsel_w = nsel_w;
        ro.o_cmp = o_cmp ? o_cmp + (size_t)r * hq * d : NULL;
        ro.lse = lse ? lse + (size_t)r * hq : NULL;
        ro.o_sel = o_sel ? o_sel + (size_t)r * hq * d : NULL;
        ro.o_win = o_win ? o_win + (size_t)r * hq * d : NULL;
        ro.tie_gap = tie_gap ? tie_gap + (size_t)r * hkv : NULL;
        ro.lse_sel = NULL;
        ro.lse_win = NULL;
        const size_t seq_off = (size_t)b * Lmax * hkv * d;
        const size_t cmp_off = (size_t)b * ncmax * hkv * d;
        video_row(c, L - 1, q + (size_t)b * hq * d, kcache + seq_off, vcache + seq_off, kcmp + cmp_off,
                  vcmp + cmp_off, gates + (size_t)b * hq * 3, sel_override ? sel_override + (size_t)r * hkv * n : NULL,
                  &ro, &w);
      }
      free_scratch(&w);
    }
  }
  return bad ? -1 : 0;
}

/* Threads the parallel loops above will use (for reporting the baseline's core count). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
