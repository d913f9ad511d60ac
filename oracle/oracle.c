/*
 * oracle.c — plain, slow CPU reference of one EdgeRock-4B SWA∥RMA layer and
 * of the RMA anchor-bank commit.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code with the CUDA path (the only common code is the synthetic input
 * generator in synth/, which holds none of the layer's arithmetic).
 *
 * Precision: every sum, norm, angle and softmax is taken in float64; values
 * that the layer stores in BF16 (projections, normed/rotated q/k, the
 * attention output fed to o_proj, the layer output) are rounded once from
 * float64 to BF16 (round to nearest even); scores are rounded once to
 * float32.  Loops are the definitions written out, in the order the pages
 * describe the steps; no blocking, fusion or reordering.
 *
 * Sources (page title, section):
 *  [F-arch]   fluxbbs.com "EdgeRock-4B 开源：72 MiB 固定 KV，AIME 82.9 分",
 *             §架构：递归、局部窗口与记忆锚点三件套  — 16 q heads over 4 KV groups,
 *             head dim 256, learned RMS-norm on q and k, partial RoPE on 64 of
 *             256 dims with base 1e7, v neither rotated nor normed; bias-free
 *             FP32 score chain 2560→256→4, one score per group; groups pick
 *             their top records independently and may share source positions;
 *             candidates gather in a 256-record block, the bank keeps 1024.
 *  [F-mem]    same page, §72 MiB 是怎么算出来的 — 2×8×4×1024×256×2 B = 32 MiB
 *             committed, 8 MiB pending, 32 MiB window, 72 MiB in total.
 *  [N-rma]    neodrop.ai "内存还会跌吗？KV Cache砍掉99%…", §三段记忆，只记值得记的 —
 *             one candidate record per token; every 256 candidates are merged
 *             with the bank and the top 1024 by score are kept, per KV group;
 *             kept anchors never change; 1,024-token local window.
 *  [spec]     readings fixed for this build where the pages are silent: SiLU
 *             between the two score matmuls; the RMA read is its own softmax
 *             over committed+pending records with its own q/k/v projections,
 *             summed with the SWA output before one shared o_proj; top-k
 *             ties broken by lower source position.
 * Readings of open points (listed in the design notes): window of positions
 * [t-1023, t] including the current token; every token is appended to
 * pending as it is produced; within a step: project, score, write window,
 * append, read, o_proj, commit if the block is full; −0 ranks as +0 and NaN
 * ranks below −inf; evicted bank slots (ascending) take the pending winners
 * (ascending pending index); attention scale 1/16; head h reads group h/4;
 * rotate-half RoPE pairing (i, i+32) with inv_freq_i = 1e7^(−2i/64);
 * RMS-norm eps 1e-6 with the gain applied directly.
 *
 * parity: pinned (closed forms, invariants, brute force — tests/test_oracle_pins.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OD 256                       /* head dim */
#define OHID 2560                    /* hidden */
#define ONH 16                       /* q heads */
#define ONG 4                        /* KV groups */
#define OWIN 1024                    /* window slots */
#define OBANK 1024                   /* committed anchors per group */
#define OPEND 256                    /* pending block */
#define OROPE 64                     /* rotated dims */
#define OSH 256                      /* score hidden width */
#define OQKV (2 * (ONH * OD + 2 * ONG * OD)) /* 12288 projection rows */
#define OTHETA 1.0e7
#define OEPS 1.0e-6

/* ---------------------------------------------------------------- scalars */

static double bf(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* float64 -> BF16, one rounding to nearest (ties to even), normal range. */
static uint16_t to_bf(double x) {
  if (x != x) return 0x7FC0;
  if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
  if (isinf(x)) return x > 0 ? 0x7F80 : 0xFF80;
  int e;
  double m = frexp(x, &e);                 /* x = m * 2^e, 0.5 <= |m| < 1 */
  double r = nearbyint(ldexp(m, 8));       /* keep 8 significant bits */
  float f = (float)ldexp(r, e - 8);        /* exact (or overflows to inf) */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

double orc_bf16_to_f64(uint16_t h) { return bf(h); }
uint16_t orc_f64_to_bf16(double x) { return to_bf(x); }

/* ------------------------------------------------------------------ state */

typedef struct {
  int32_t s_max, n_layers;
  uint16_t *win_k, *win_v;     /* [s][l][g][1024][256] */
  uint16_t *bank_k, *bank_v;   /* [s][l][g][1024][256] */
  uint16_t *pend_k, *pend_v;   /* [s][l][g][256][256] */
  float *bank_score, *pend_score;   /* [s][l][g][slots] */
  int32_t *bank_pos, *pend_pos;     /* [s][l][g][slots] */
  int32_t *meta;                    /* [s][4]: pos, pend_count, bank_count, 0 */
} orc_state;

typedef struct {
  const uint16_t* w_qkv;  /* [12288][2560]: q_swa 4096 | k_swa 1024 | v_swa 1024 |
                             q_rma 4096 | k_rma 1024 | v_rma 1024 */
  const uint16_t* w_o;    /* [2560][4096] */
  const uint16_t *g_q_swa, *g_k_swa, *g_q_rma, *g_k_rma; /* [256] */
  const float* w1;        /* [256][2560] */
  const float* w2;        /* [4][256] */
} orc_weights;

static size_t gidx(const orc_state* st, int s, int l, int g) {
  return ((size_t)s * st->n_layers + l) * ONG + g;
}
static uint16_t* win_k_row(const orc_state* st, int s, int l, int g, int slot) {
  return st->win_k + (gidx(st, s, l, g) * OWIN + slot) * OD;
}
static uint16_t* win_v_row(const orc_state* st, int s, int l, int g, int slot) {
  return st->win_v + (gidx(st, s, l, g) * OWIN + slot) * OD;
}
static uint16_t* bank_k_row(const orc_state* st, int s, int l, int g, int slot) {
  return st->bank_k + (gidx(st, s, l, g) * OBANK + slot) * OD;
}
static uint16_t* bank_v_row(const orc_state* st, int s, int l, int g, int slot) {
  return st->bank_v + (gidx(st, s, l, g) * OBANK + slot) * OD;
}
static uint16_t* pend_k_row(const orc_state* st, int s, int l, int g, int slot) {
  return st->pend_k + (gidx(st, s, l, g) * OPEND + slot) * OD;
}
static uint16_t* pend_v_row(const orc_state* st, int s, int l, int g, int slot) {
  return st->pend_v + (gidx(st, s, l, g) * OPEND + slot) * OD;
}

/* Bytes of one sequence's K/V state ([F-mem]): window + bank + pending, K and V. */
int64_t orc_kv_bytes_per_seq(int n_layers) {
  return (int64_t)2 * n_layers * ONG * (OWIN + OBANK + OPEND) * OD * 2;
}

/* ------------------------------------------------------- a2: norm + RoPE */

/* RMS-norm with a learned gain, then rotary embedding on the first 64 of 256
 * dims at position `pos` with base 1e7 ([F-arch]); rows of 256 BF16 values. */
void orc_norm_rope(const uint16_t* x, const uint16_t* gain, const int32_t* pos, int64_t n_rows,
                   uint16_t* out) {
  for (int64_t r = 0; r < n_rows; ++r) {
    const uint16_t* xr = x + r * OD;
    double v[OD];
    double ss = 0.0;
    for (int i = 0; i < OD; ++i) {
      v[i] = bf(xr[i]);
      ss += v[i] * v[i];
    }
    double inv_rms = 1.0 / sqrt(ss / OD + OEPS);
    for (int i = 0; i < OD; ++i) v[i] = v[i] * inv_rms * bf(gain[i]);
    for (int i = 0; i < OROPE / 2; ++i) {
      double inv_freq = pow(OTHETA, -2.0 * i / OROPE);
      double ang = (double)pos[r] * inv_freq;
      double c = cos(ang), s = sin(ang);
      double a = v[i], b = v[i + OROPE / 2];
      v[i] = a * c - b * s;
      v[i + OROPE / 2] = b * c + a * s;
    }
    for (int i = 0; i < OD; ++i) out[r * OD + i] = to_bf(v[i]);
  }
}

/* ------------------------------------------------------- a1 / a6: linear */

/* y[o] = bf16( sum_i W[o][i] * x[i] ), W BF16 row-major [out][in]. */
void orc_linear_bf16(const uint16_t* W, int out_dim, int in_dim, const uint16_t* x,
                     uint16_t* y) {
  for (int o = 0; o < out_dim; ++o) {
    const uint16_t* w = W + (size_t)o * in_dim;
    double acc = 0.0;
    for (int i = 0; i < in_dim; ++i) acc += bf(w[i]) * bf(x[i]);
    y[o] = to_bf(acc);
  }
}

/* ------------------------------------------------------- a3: score chain */

/* s = W2 · SiLU(W1 · x), bias-free, 2560 → 256 → 4, one score per KV group
 * ([F-arch], [N-rma]; SiLU from [spec]).  Rounded once to float32. */
void orc_score(const float* w1, const float* w2, const uint16_t* x, int n, float* s) {
  for (int t = 0; t < n; ++t) {
    const uint16_t* xt = x + (size_t)t * OHID;
    double a[OSH];
    for (int j = 0; j < OSH; ++j) {
      double h = 0.0;
      for (int i = 0; i < OHID; ++i) h += (double)w1[(size_t)j * OHID + i] * bf(xt[i]);
      a[j] = h / (1.0 + exp(-h));
    }
    for (int g = 0; g < ONG; ++g) {
      double acc = 0.0;
      for (int j = 0; j < OSH; ++j) acc += (double)w2[g * OSH + j] * a[j];
      s[t * ONG + g] = (float)acc;
    }
  }
}

/* ---------------------------------------------------- a5: one softmax read */

/* o = softmax(q·kᵢ / 16) · vᵢ over the n listed rows; o = 0 when n = 0. */
static void attend(const uint16_t* q, const uint16_t* const* krows, const uint16_t* const* vrows,
                   int n, double* o) {
  for (int d = 0; d < OD; ++d) o[d] = 0.0;
  if (n == 0) return;
  double* logit = (double*)malloc(sizeof(double) * n);
  double m = -INFINITY;
  for (int i = 0; i < n; ++i) {
    double acc = 0.0;
    for (int d = 0; d < OD; ++d) acc += bf(q[d]) * bf(krows[i][d]);
    logit[i] = acc / 16.0;
    if (logit[i] > m) m = logit[i];
  }
  double denom = 0.0;
  for (int i = 0; i < n; ++i) {
    double w = exp(logit[i] - m);
    denom += w;
    for (int d = 0; d < OD; ++d) o[d] += w * bf(vrows[i][d]);
  }
  for (int d = 0; d < OD; ++d) o[d] /= denom;
  free(logit);
}

/* Contiguous-row form, exported for the special-case pins. */
void orc_attend_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, int n, double* o) {
  const uint16_t** kr = (const uint16_t**)malloc(sizeof(void*) * (n > 0 ? n : 1));
  const uint16_t** vr = (const uint16_t**)malloc(sizeof(void*) * (n > 0 ? n : 1));
  for (int i = 0; i < n; ++i) {
    kr[i] = k + (size_t)i * OD;
    vr[i] = v + (size_t)i * OD;
  }
  attend(q, kr, vr, n, o);
  free(kr);
  free(vr);
}

/* ------------------------------------------------------------ a7: commit */

typedef struct {
  float score;
  int32_t pos;
  int32_t src; /* bank slot i -> i, pending index j -> 1024 + j */
} orc_rec;

/* Order: score descending, then source position ascending ([F-arch], [spec]).
 * −0 compares equal to +0 (plain ==); NaN ranks below every number. */
static int rec_cmp(const void* pa, const void* pb) {
  const orc_rec* a = (const orc_rec*)pa;
  const orc_rec* b = (const orc_rec*)pb;
  int na = isnan(a->score), nb = isnan(b->score);
  if (!na && !nb) {
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
  } else if (na != nb) {
    return na ? 1 : -1;
  }
  if (a->pos < b->pos) return -1;
  if (a->pos > b->pos) return 1;
  return 0;
}

/* One group's merge: the c committed records and p pending records compete;
 * the top min(1024, c+p) stay.  Evicted bank slots, ascending, then the free
 * slots c, c+1, … receive the pending winners in ascending pending index.
 * kept (optional, 1024 entries): source indices in rank order, -1 padded. */
static void commit_group(orc_state* st, int s, int l, int g, int c, int p, int32_t* kept) {
  orc_rec recs[OBANK + OPEND];
  size_t gi = gidx(st, s, l, g);
  int n = 0;
  for (int i = 0; i < c; ++i) {
    recs[n].score = st->bank_score[gi * OBANK + i];
    recs[n].pos = st->bank_pos[gi * OBANK + i];
    recs[n].src = i;
    ++n;
  }
  for (int j = 0; j < p; ++j) {
    recs[n].score = st->pend_score[gi * OPEND + j];
    recs[n].pos = st->pend_pos[gi * OPEND + j];
    recs[n].src = OBANK + j;
    ++n;
  }
  qsort(recs, n, sizeof(orc_rec), rec_cmp);
  int keep = n < OBANK ? n : OBANK;

  int bank_kept[OBANK], pend_won[OPEND];
  memset(bank_kept, 0, sizeof bank_kept);
  memset(pend_won, 0, sizeof pend_won);
  for (int r = 0; r < keep; ++r) {
    if (recs[r].src < OBANK) bank_kept[recs[r].src] = 1;
    else pend_won[recs[r].src - OBANK] = 1;
  }
  if (kept) {
    for (int r = 0; r < OBANK; ++r) kept[r] = r < keep ? recs[r].src : -1;
  }
  /* target slots: evicted bank slots ascending, then c, c+1, ... */
  int targets[OBANK];
  int nt = 0;
  for (int i = 0; i < c; ++i)
    if (!bank_kept[i]) targets[nt++] = i;
  for (int i = c; i < OBANK; ++i) targets[nt++] = i;
  int t = 0;
  for (int j = 0; j < p; ++j) {
    if (!pend_won[j]) continue;
    int slot = targets[t++];
    if (st->bank_k) { /* a state built without K/V rows ranks and places records only */
      memcpy(bank_k_row(st, s, l, g, slot), pend_k_row(st, s, l, g, j), OD * 2);
      memcpy(bank_v_row(st, s, l, g, slot), pend_v_row(st, s, l, g, j), OD * 2);
    }
    st->bank_score[gi * OBANK + slot] = st->pend_score[gi * OPEND + j];
    st->bank_pos[gi * OBANK + slot] = st->pend_pos[gi * OPEND + j];
  }
}

/* Commit one layer (layer >= 0: state metadata untouched) or every layer
 * (layer == -1: then pend_count := 0 and bank_count := min(1024, c + p)).
 * kept: optional [n_layers or 1][4][1024]. */
void orc_commit(orc_state* st, int layer, int seq, int32_t* kept) {
  int32_t* meta = st->meta + (size_t)seq * 4;
  int c = meta[2], p = meta[1];
  int l0 = layer < 0 ? 0 : layer, l1 = layer < 0 ? st->n_layers : layer + 1;
  for (int l = l0; l < l1; ++l)
    for (int g = 0; g < ONG; ++g)
      commit_group(st, seq, l, g, c, p, kept ? kept + ((size_t)(l - l0) * ONG + g) * OBANK : NULL);
  if (layer < 0) {
    meta[2] = c + p < OBANK ? c + p : OBANK;
    meta[1] = 0;
  }
}

/* End of a step of T tokens (after every layer): position and pending count
 * advance; a full block has been committed by each layer, so it empties.
 * With the RMA switched off (the pages' ablation) only the position moves. */
void orc_advance(orc_state* st, int seq, int T, int rma_off) {
  int32_t* meta = st->meta + (size_t)seq * 4;
  meta[0] += T;
  if (rma_off) return;
  meta[1] += T;
  if (meta[1] >= OPEND) {
    meta[1] = 0;
    meta[2] = meta[2] + OPEND < OBANK ? meta[2] + OPEND : OBANK;
  }
}

/* ------------------------------------------------- token-level helpers */

typedef struct {
  uint16_t q_swa[ONH][OD], k_swa[ONG][OD], v_swa[ONG][OD];
  uint16_t q_rma[ONH][OD], k_rma[ONG][OD], v_rma[ONG][OD];
  float s[ONG];
} orc_tok;

/* a1 + a2 + a3 for one token at position t. */
static void project_token(const orc_weights* w, const uint16_t* x, int32_t t, orc_tok* tk) {
  uint16_t* proj = (uint16_t*)malloc(sizeof(uint16_t) * OQKV);
  orc_linear_bf16(w->w_qkv, OQKV, OHID, x, proj);
  const uint16_t* p = proj;
  orc_norm_rope(p, w->g_q_swa, (int32_t[]){t, t, t, t, t, t, t, t, t, t, t, t, t, t, t, t}, ONH,
                &tk->q_swa[0][0]);
  p += ONH * OD;
  orc_norm_rope(p, w->g_k_swa, (int32_t[]){t, t, t, t}, ONG, &tk->k_swa[0][0]);
  p += ONG * OD;
  memcpy(tk->v_swa, p, sizeof tk->v_swa);
  p += ONG * OD;
  orc_norm_rope(p, w->g_q_rma, (int32_t[]){t, t, t, t, t, t, t, t, t, t, t, t, t, t, t, t}, ONH,
                &tk->q_rma[0][0]);
  p += ONH * OD;
  orc_norm_rope(p, w->g_k_rma, (int32_t[]){t, t, t, t}, ONG, &tk->k_rma[0][0]);
  p += ONG * OD;
  memcpy(tk->v_rma, p, sizeof tk->v_rma);
  free(proj);
  orc_score(w->w1, w->w2, x, 1, tk->s);
}

/* a6: o = bf16(o_swa + o_rma) per head, out = bf16(W_o · o). */
static void output_token(const orc_weights* w, double o_swa[ONH][OD], double o_rma[ONH][OD],
                         uint16_t* out) {
  uint16_t o[ONH * OD];
  for (int h = 0; h < ONH; ++h)
    for (int d = 0; d < OD; ++d) o[h * OD + d] = to_bf(o_swa[h][d] + o_rma[h][d]);
  orc_linear_bf16(w->w_o, OHID, ONH * OD, o, out);
}

/* ------------------------------------------------------- decode (a1–a7) */

/* One decode step of one layer for one sequence.  Optional o_swa / o_rma
 * ([16][256] float64) receive the two branch outputs before o_proj.  With
 * rma_off (the pages' ablation of the RMA modules) the RMA output is 0, the
 * token is not appended to pending and nothing commits. */
void orc_decode_layer(const orc_weights* w, orc_state* st, int layer, int seq, const uint16_t* x,
                      uint16_t* out, double* o_swa_out, double* o_rma_out, int rma_off) {
  int32_t* meta = st->meta + (size_t)seq * 4;
  int32_t t = meta[0];
  int p = meta[1], c = meta[2];
  orc_tok* tk = (orc_tok*)malloc(sizeof(orc_tok));
  project_token(w, x, t, tk);

  /* a4: window slot t mod 1024, pending slot p */
  size_t gi0 = gidx(st, seq, layer, 0);
  for (int g = 0; g < ONG; ++g) {
    memcpy(win_k_row(st, seq, layer, g, t % OWIN), tk->k_swa[g], OD * 2);
    memcpy(win_v_row(st, seq, layer, g, t % OWIN), tk->v_swa[g], OD * 2);
    if (rma_off) continue;
    memcpy(pend_k_row(st, seq, layer, g, p), tk->k_rma[g], OD * 2);
    memcpy(pend_v_row(st, seq, layer, g, p), tk->v_rma[g], OD * 2);
    st->pend_score[(gi0 + g) * OPEND + p] = tk->s[g];
    st->pend_pos[(gi0 + g) * OPEND + p] = t;
  }

  /* a5: SWA over positions [max(0,t-1023), t]; RMA over bank 0..c-1 and pending 0..p */
  double(*o_swa)[OD] = (double(*)[OD])malloc(sizeof(double) * ONH * OD);
  double(*o_rma)[OD] = (double(*)[OD])malloc(sizeof(double) * ONH * OD);
  const uint16_t* kr[OWIN + OBANK + OPEND];
  const uint16_t* vr[OWIN + OBANK + OPEND];
  for (int h = 0; h < ONH; ++h) {
    int g = h / (ONH / ONG);
    int n = 0;
    for (int32_t pos = t - (OWIN - 1) < 0 ? 0 : t - (OWIN - 1); pos <= t; ++pos) {
      kr[n] = win_k_row(st, seq, layer, g, pos % OWIN);
      vr[n] = win_v_row(st, seq, layer, g, pos % OWIN);
      ++n;
    }
    attend(tk->q_swa[h], kr, vr, n, o_swa[h]);
    if (rma_off) {
      for (int d = 0; d < OD; ++d) o_rma[h][d] = 0.0;
      continue;
    }
    n = 0;
    for (int i = 0; i < c; ++i) {
      kr[n] = bank_k_row(st, seq, layer, g, i);
      vr[n] = bank_v_row(st, seq, layer, g, i);
      ++n;
    }
    for (int j = 0; j <= p; ++j) {
      kr[n] = pend_k_row(st, seq, layer, g, j);
      vr[n] = pend_v_row(st, seq, layer, g, j);
      ++n;
    }
    attend(tk->q_rma[h], kr, vr, n, o_rma[h]);
  }
  if (o_swa_out) memcpy(o_swa_out, o_swa, sizeof(double) * ONH * OD);
  if (o_rma_out) memcpy(o_rma_out, o_rma, sizeof(double) * ONH * OD);
  output_token(w, o_swa, o_rma, out);

  /* a7: the token that fills the block is read with all 1280 records, then
   * this layer commits; metadata moves on in orc_advance. */
  if (!rma_off && p + 1 == OPEND) {
    meta[1] = OPEND;
    orc_commit(st, layer, seq, NULL);
    meta[1] = p;
  }
  free(o_swa);
  free(o_rma);
  free(tk);
}

/* -------------------------------------------------- prefill chunk (a8) */

/* T tokens at positions t0..t0+T-1 (t0 = pos, requires pend + T <= 256).
 * Causal: token i reads window positions [t-1023, t] (old ring entries below
 * t0, the chunk's own tokens from t0) and the bank plus pending 0..p0+i.  The
 * chunk enters the ring after every token has been read. */
int orc_prefill_chunk(const orc_weights* w, orc_state* st, int layer, int seq,
                      const uint16_t* x, int T, uint16_t* out, int rma_off) {
  int32_t* meta = st->meta + (size_t)seq * 4;
  int32_t t0 = meta[0];
  int p0 = meta[1], c = meta[2];
  if (T < 1 || p0 + T > OPEND) return -1;
  orc_tok* tk = (orc_tok*)malloc(sizeof(orc_tok) * (size_t)T);
  for (int i = 0; i < T; ++i) project_token(w, x + (size_t)i * OHID, t0 + i, &tk[i]);
  size_t gi0 = gidx(st, seq, layer, 0);
  for (int i = 0; i < T && !rma_off; ++i)
    for (int g = 0; g < ONG; ++g) {
      memcpy(pend_k_row(st, seq, layer, g, p0 + i), tk[i].k_rma[g], OD * 2);
      memcpy(pend_v_row(st, seq, layer, g, p0 + i), tk[i].v_rma[g], OD * 2);
      st->pend_score[(gi0 + g) * OPEND + p0 + i] = tk[i].s[g];
      st->pend_pos[(gi0 + g) * OPEND + p0 + i] = t0 + i;
    }
  double(*o_swa)[OD] = (double(*)[OD])malloc(sizeof(double) * ONH * OD);
  double(*o_rma)[OD] = (double(*)[OD])malloc(sizeof(double) * ONH * OD);
  const uint16_t* kr[OWIN + OBANK + OPEND];
  const uint16_t* vr[OWIN + OBANK + OPEND];
  for (int i = 0; i < T; ++i) {
    int32_t t = t0 + i;
    for (int h = 0; h < ONH; ++h) {
      int g = h / (ONH / ONG);
      int n = 0;
      for (int32_t pos = t - (OWIN - 1) < 0 ? 0 : t - (OWIN - 1); pos <= t; ++pos) {
        if (pos < t0) {
          kr[n] = win_k_row(st, seq, layer, g, pos % OWIN);
          vr[n] = win_v_row(st, seq, layer, g, pos % OWIN);
        } else {
          kr[n] = tk[pos - t0].k_swa[g];
          vr[n] = tk[pos - t0].v_swa[g];
        }
        ++n;
      }
      attend(tk[i].q_swa[h], kr, vr, n, o_swa[h]);
      if (rma_off) {
        for (int d = 0; d < OD; ++d) o_rma[h][d] = 0.0;
        continue;
      }
      n = 0;
      for (int b = 0; b < c; ++b) {
        kr[n] = bank_k_row(st, seq, layer, g, b);
        vr[n] = bank_v_row(st, seq, layer, g, b);
        ++n;
      }
      for (int j = 0; j <= p0 + i; ++j) {
        kr[n] = pend_k_row(st, seq, layer, g, j);
        vr[n] = pend_v_row(st, seq, layer, g, j);
        ++n;
      }
      attend(tk[i].q_rma[h], kr, vr, n, o_rma[h]);
    }
    output_token(w, o_swa, o_rma, out + (size_t)i * OHID);
  }
  for (int i = 0; i < T; ++i)
    for (int g = 0; g < ONG; ++g) {
      memcpy(win_k_row(st, seq, layer, g, (t0 + i) % OWIN), tk[i].k_swa[g], OD * 2);
      memcpy(win_v_row(st, seq, layer, g, (t0 + i) % OWIN), tk[i].v_swa[g], OD * 2);
    }
  if (!rma_off && p0 + T == OPEND) {
    meta[1] = OPEND;
    orc_commit(st, layer, seq, NULL);
    meta[1] = p0;
  }
  free(o_swa);
  free(o_rma);
  free(tk);
  return 0;
}

/* Appends (k, v, s, pos) for n sequences at their pending_count, one layer
 * (metadata untouched, as in a decode step). */
void orc_append_pending(orc_state* st, int layer, const int32_t* seqs, int n, const uint16_t* k,
                        const uint16_t* v, const float* s, const int32_t* pos) {
  for (int b = 0; b < n; ++b) {
    int seq = seqs[b];
    int p = st->meta[(size_t)seq * 4 + 1];
    size_t gi0 = gidx(st, seq, layer, 0);
    for (int g = 0; g < ONG; ++g) {
      memcpy(pend_k_row(st, seq, layer, g, p), k + ((size_t)b * ONG + g) * OD, OD * 2);
      memcpy(pend_v_row(st, seq, layer, g, p), v + ((size_t)b * ONG + g) * OD, OD * 2);
      st->pend_score[(gi0 + g) * OPEND + p] = s[b * ONG + g];
      st->pend_pos[(gi0 + g) * OPEND + p] = pos[b];
    }
  }
}
