/*
 * RLT CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the bench's CPU-baseline leg may load
 * this library. The CUDA product path never calls it and shares no code,
 * header, table or helper with it.
 *
 * A plain, slow, obviously correct statement of what the Recurrent Looped
 * Transformer (RLT) computes, in one floating-point type `real` chosen at
 * compile time (double for parity, float for the timed CPU baseline). Loops
 * are written in the order the method states them: no blocking, fusion or
 * reordering. Parallelism is only across independent sequences (OpenMP).
 *
 * Citation key (page title, site):
 *   [RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No Resets"
 *            (aimastery.page)
 *   [RLT-TC] "Recurrent Looped Transformer (RLT): prompts in parallel, depth in
 *            sequence" (thakicloud.com)
 *   [RLT-FT] "Recurrent Looped Transformer debunked" (flowtivity.ai)
 *   [RLT-PV] "Per-token recurrence, no quality gain" (news.promtvault.app)
 *
 * The pages print no equations; where they are silent the oracle takes the
 * plainest reading and states it at the function that uses it:
 *   gate      g = sigmoid(W_g [e_t ; s_{t-1}] + b_g),  x_t = e_t + alpha g*s_{t-1}
 *   norm      pre-RMSNorm, y = x / sqrt(mean(x^2) + eps) * gamma, no bias
 *   position  RoPE (theta 1e4, rotate-half pairs (i, i + dh/2)) on q and k of
 *             the encoder's causal attention and the decoder's SWA, at the
 *             absolute position t (first token t = 0); none on cross-attention
 *   attention scale 1/sqrt(dh), softmax with max subtraction, no biases
 *   FFN       W_2 GELU_erf(W_1 u)  or  W_2 (SiLU(W_a u) * (W_b u))
 *   s_t       RMSNorm_f of the residual stream after the last decoder block
 *   memory    K^g_j = W_mk^g e_j, V^g_j = W_mv^g e_j; the decoder at t reads
 *             positions 0..t (inclusive)
 *   window    SWA at t attends positions max(0, t-W+1) .. t
 * Matrices are row-major [out][in] (y_j = sum_i W[j][i] x_i). The q/k/v
 * projection stacks rows q | k | v; head h owns entries h*dh .. h*dh+dh-1.
 *
 * Pins: every piece, the ring window, the gate at alpha = 0, causality, the
 * carried-state split, the G and tying plumbing are checked against closed
 * forms, brute force and textbook routines by the CPU tests. The whole
 * model's outputs are parity unpinned against the pages: they print no
 * values for any configuration.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORC_REAL
#define ORC_REAL double
#endif
typedef ORC_REAL real;

#define ORC_MAX_LAYERS 64
#define ORC_GELU 0
#define ORC_SWIGLU 1

typedef struct {
  int d, n_heads, head_dim, n_enc, n_dec, ffn_dim, ffn_kind, vocab, window,
      mem_groups;
  double alpha, rms_eps, rope_theta;
} orc_cfg;

typedef struct {
  const real *embed;                                   /* [V][d] */
  const real *enc_ln1[ORC_MAX_LAYERS], *enc_wqkv[ORC_MAX_LAYERS],
      *enc_wo[ORC_MAX_LAYERS], *enc_ln2[ORC_MAX_LAYERS],
      *enc_w1[ORC_MAX_LAYERS], *enc_wb[ORC_MAX_LAYERS], *enc_w2[ORC_MAX_LAYERS];
  const real *enc_lnf;                                 /* [d] */
  const real *mem_wk[ORC_MAX_LAYERS], *mem_wv[ORC_MAX_LAYERS]; /* [d][d] */
  const real *gate_w, *gate_b, *sstar;                 /* [d][2d], [d], [d] */
  const real *dec_ln1[ORC_MAX_LAYERS], *dec_wqkv[ORC_MAX_LAYERS],
      *dec_wo[ORC_MAX_LAYERS], *dec_ln2[ORC_MAX_LAYERS],
      *dec_wqx[ORC_MAX_LAYERS], *dec_wox[ORC_MAX_LAYERS],
      *dec_ln3[ORC_MAX_LAYERS], *dec_w1[ORC_MAX_LAYERS],
      *dec_wb[ORC_MAX_LAYERS], *dec_w2[ORC_MAX_LAYERS];
  const real *dec_lnf;
} orc_weights;

int orc_real_bytes(void) { return (int)sizeof(real); }

/* ------------------------------------------------------------------ pieces */

/* Pre-norm of every sublayer (reading of the pages' silence on the norm). */
void orc_rmsnorm(const real *x, const real *gamma, int n, double eps, real *y) {
  real ss = 0;
  for (int i = 0; i < n; i++) ss += x[i] * x[i];
  real r = (real)(1.0 / sqrt((double)(ss / n) + eps));
  for (int i = 0; i < n; i++) y[i] = x[i] * r * gamma[i];
}

/* y = W x with W row-major [n_out][n_in]. */
void orc_linear(const real *W, const real *x, int n_out, int n_in, real *y) {
  for (int j = 0; j < n_out; j++) {
    real acc = 0;
    const real *row = W + (size_t)j * n_in;
    for (int i = 0; i < n_in; i++) acc += row[i] * x[i];
    y[j] = acc;
  }
}

real orc_gelu(real x) { return (real)(0.5 * x * (1.0 + erf(x / sqrt(2.0)))); }
real orc_silu(real x) { return (real)(x / (1.0 + exp(-(double)x))); }
real orc_sigmoid(real x) { return (real)(1.0 / (1.0 + exp(-(double)x))); }

/* Rotary position encoding of one head vector at absolute position pos. */
void orc_rope(real *v, int dh, long pos, double theta) {
  int half = dh / 2;
  for (int i = 0; i < half; i++) {
    double freq = pow(theta, -2.0 * i / dh);
    double ang = (double)pos * freq;
    real c = (real)cos(ang), s = (real)sin(ang);
    real a = v[i], b = v[i + half];
    v[i] = a * c - b * s;
    v[i + half] = b * c + a * s;
  }
}

/* One query against n keys given as row pointers: softmax(q.k/sqrt(dh)) v.
 * `score` is caller scratch of n entries. */
void orc_attend(const real *q, const real *const *k, const real *const *v,
                int n, int dh, real *score, real *out) {
  real scale = (real)(1.0 / sqrt((double)dh));
  real mx = -INFINITY;
  for (int j = 0; j < n; j++) {
    real dot = 0;
    for (int i = 0; i < dh; i++) dot += q[i] * k[j][i];
    score[j] = dot * scale;
    if (score[j] > mx) mx = score[j];
  }
  real den = 0;
  for (int j = 0; j < n; j++) {
    score[j] = (real)exp((double)(score[j] - mx));
    den += score[j];
  }
  for (int i = 0; i < dh; i++) out[i] = 0;
  for (int j = 0; j < n; j++)
    for (int i = 0; i < dh; i++) out[i] += score[j] * v[j][i];
  for (int i = 0; i < dh; i++) out[i] /= den;
}

/* Dense form for tests: K, V row-major [n][dh]. */
void orc_attend_dense(const real *q, const real *K, const real *V, int n,
                      int dh, real *out) {
  const real **kp = malloc(sizeof(real *) * (size_t)(n > 0 ? n : 1));
  const real **vp = malloc(sizeof(real *) * (size_t)(n > 0 ? n : 1));
  real *sc = malloc(sizeof(real) * (size_t)(n > 0 ? n : 1));
  for (int j = 0; j < n; j++) {
    kp[j] = K + (size_t)j * dh;
    vp[j] = V + (size_t)j * dh;
  }
  orc_attend(q, kp, vp, n, dh, sc, out);
  free(kp);
  free(vp);
  free(sc);
}

/* Position-wise feed-forward of one block ([RLT-96] "Architecture"). */
static void ffn(const orc_cfg *c, const real *w1, const real *wb,
                const real *w2, const real *u, real *out, real *tmp_a,
                real *tmp_b) {
  int d = c->d, F = c->ffn_dim;
  orc_linear(w1, u, F, d, tmp_a);
  if (c->ffn_kind == ORC_SWIGLU) {
    orc_linear(wb, u, F, d, tmp_b);
    for (int i = 0; i < F; i++) tmp_a[i] = orc_silu(tmp_a[i]) * tmp_b[i];
  } else {
    for (int i = 0; i < F; i++) tmp_a[i] = orc_gelu(tmp_a[i]);
  }
  orc_linear(w2, tmp_a, d, F, out);
}

/* -------------------------------------------------------------- encoder */

/* Causal token-parallel encoder of one sequence and its memory projection.
 * [RLT-96] "Architecture: encoder memory meets recurrent decoder": the encoder
 * processes tokens in parallel under a causal mask, producing e_t, from which
 * the key-value memory M<=t is projected, shared (G = 1) or per decoder layer
 * (G = L_D). [RLT-TC] "What is this technology": prefix-restricted memory.
 * e_out [T][d]; mem_out [G][mem_cap][2][d] (K row then V row per position). */
int orc_encode(const orc_cfg *c, const orc_weights *w, const int *tok, int T,
               real *e_out, real *mem_out, int mem_cap) {
  int d = c->d, H = c->n_heads, dh = c->head_dim, F = c->ffn_dim;
  if (T > mem_cap || T < 0) return -1;
  real *h = calloc((size_t)T * d, sizeof(real));
  real *qkv = calloc((size_t)T * 3 * d, sizeof(real));
  real *a = calloc((size_t)T * d, sizeof(real));
  real *u = calloc((size_t)d, sizeof(real));
  real *o = calloc((size_t)d, sizeof(real));
  real *ta = calloc((size_t)F, sizeof(real));
  real *tb = calloc((size_t)F, sizeof(real));
  real *sc = calloc((size_t)(T > 0 ? T : 1), sizeof(real));
  const real **kp = calloc((size_t)(T > 0 ? T : 1), sizeof(real *));
  const real **vp = calloc((size_t)(T > 0 ? T : 1), sizeof(real *));
  for (int t = 0; t < T; t++)
    memcpy(h + (size_t)t * d, w->embed + (size_t)tok[t] * d, sizeof(real) * d);
  for (int l = 0; l < c->n_enc; l++) {
    /* causal self-attention sublayer */
    for (int t = 0; t < T; t++) {
      orc_rmsnorm(h + (size_t)t * d, w->enc_ln1[l], d, c->rms_eps, u);
      orc_linear(w->enc_wqkv[l], u, 3 * d, d, qkv + (size_t)t * 3 * d);
      for (int hd = 0; hd < H; hd++) {
        orc_rope(qkv + (size_t)t * 3 * d + hd * dh, dh, t, c->rope_theta);
        orc_rope(qkv + (size_t)t * 3 * d + d + hd * dh, dh, t, c->rope_theta);
      }
    }
    for (int t = 0; t < T; t++) {
      for (int hd = 0; hd < H; hd++) {
        for (int j = 0; j <= t; j++) {
          kp[j] = qkv + (size_t)j * 3 * d + d + hd * dh;
          vp[j] = qkv + (size_t)j * 3 * d + 2 * d + hd * dh;
        }
        orc_attend(qkv + (size_t)t * 3 * d + hd * dh, kp, vp, t + 1, dh, sc,
                   a + (size_t)t * d + hd * dh);
      }
    }
    for (int t = 0; t < T; t++) {
      orc_linear(w->enc_wo[l], a + (size_t)t * d, d, d, o);
      for (int i = 0; i < d; i++) h[(size_t)t * d + i] += o[i];
    }
    /* FFN sublayer */
    for (int t = 0; t < T; t++) {
      orc_rmsnorm(h + (size_t)t * d, w->enc_ln2[l], d, c->rms_eps, u);
      ffn(c, w->enc_w1[l], w->enc_wb[l], w->enc_w2[l], u, o, ta, tb);
      for (int i = 0; i < d; i++) h[(size_t)t * d + i] += o[i];
    }
  }
  for (int t = 0; t < T; t++)
    orc_rmsnorm(h + (size_t)t * d, w->enc_lnf, d, c->rms_eps, e_out + (size_t)t * d);
  for (int g = 0; g < c->mem_groups; g++)
    for (int t = 0; t < T; t++) {
      real *row = mem_out + (((size_t)g * mem_cap + t) * 2) * d;
      orc_linear(w->mem_wk[g], e_out + (size_t)t * d, d, d, row);
      orc_linear(w->mem_wv[g], e_out + (size_t)t * d, d, d, row + d);
    }
  free(h); free(qkv); free(a); free(u); free(o); free(ta); free(tb); free(sc);
  free(kp); free(vp);
  return 0;
}

/* ------------------------------------------------------- decoder pieces */

/* Gated merge with feedback scale alpha. [RLT-96] "Architecture": a gated
 * merge combines e_t with the previous output s_{t-1}; [RLT-FT] "Key
 * Takeaways": the final decoder output feeds the next token's input through a
 * gated merge; [RLT-PV] body: alpha = 0 strips out the recurrent path. */
static void gated_merge(const orc_cfg *c, const orc_weights *w, const real *e_t,
                        const real *s_prev, real *x, real *cat, real *gpre) {
  int d = c->d;
  for (int i = 0; i < d; i++) {
    cat[i] = e_t[i];
    cat[d + i] = s_prev[i];
  }
  orc_linear(w->gate_w, cat, d, 2 * d, gpre);
  for (int i = 0; i < d; i++) {
    real g = orc_sigmoid(gpre[i] + w->gate_b[i]);
    x[i] = e_t[i] + (real)c->alpha * g * s_prev[i];
  }
}

/* Cross-attention sublayer of decoder layer l at position t over the
 * prefix-restricted memory rows 0..t of group g(l) (g = 0 when G = 1, else l).
 * [RLT-96] "Architecture"; [RLT-FT] "What is the RLT?". h is updated. */
typedef struct {
  real *u, *q, *a, *o, *ta, *tb, *sc, *cat, *gpre, *kcur, *vcur;
  const real **kp, **vp;
} scratch;

static int scratch_init(scratch *s, const orc_cfg *c, int n_keys) {
  int d = c->d, F = c->ffn_dim;
  int nk = n_keys > 1 ? n_keys : 1;
  s->u = calloc((size_t)d, sizeof(real));
  s->q = calloc((size_t)3 * d, sizeof(real));
  s->a = calloc((size_t)d, sizeof(real));
  s->o = calloc((size_t)d, sizeof(real));
  s->ta = calloc((size_t)F, sizeof(real));
  s->tb = calloc((size_t)F, sizeof(real));
  s->sc = calloc((size_t)nk, sizeof(real));
  s->cat = calloc((size_t)2 * d, sizeof(real));
  s->gpre = calloc((size_t)d, sizeof(real));
  s->kcur = calloc((size_t)d, sizeof(real));
  s->vcur = calloc((size_t)d, sizeof(real));
  s->kp = calloc((size_t)nk, sizeof(real *));
  s->vp = calloc((size_t)nk, sizeof(real *));
  return 0;
}

static void scratch_free(scratch *s) {
  free(s->u); free(s->q); free(s->a); free(s->o); free(s->ta); free(s->tb);
  free(s->sc); free(s->cat); free(s->gpre); free(s->kcur); free(s->vcur);
  free(s->kp); free(s->vp);
}

static void cross_attn_sublayer(const orc_cfg *c, const orc_weights *w, int l,
                                const real *mem, int mem_cap, long t, real *h,
                                scratch *s) {
  int d = c->d, H = c->n_heads, dh = c->head_dim;
  int g = (c->mem_groups == 1) ? 0 : l;
  const real *mg = mem + (size_t)g * mem_cap * 2 * d;
  orc_rmsnorm(h, w->dec_ln2[l], d, c->rms_eps, s->u);
  orc_linear(w->dec_wqx[l], s->u, d, d, s->q);
  for (int hd = 0; hd < H; hd++) {
    for (long j = 0; j <= t; j++) {
      s->kp[j] = mg + (size_t)j * 2 * d + hd * dh;
      s->vp[j] = mg + (size_t)j * 2 * d + d + hd * dh;
    }
    orc_attend(s->q + hd * dh, s->kp, s->vp, (int)t + 1, dh, s->sc, s->a + hd * dh);
  }
  orc_linear(w->dec_wox[l], s->a, d, d, s->o);
  for (int i = 0; i < d; i++) h[i] += s->o[i];
}

static void ffn_sublayer(const orc_cfg *c, const orc_weights *w, int l, real *h,
                         scratch *s) {
  int d = c->d;
  orc_rmsnorm(h, w->dec_ln3[l], d, c->rms_eps, s->u);
  ffn(c, w->dec_w1[l], w->dec_wb[l], w->dec_w2[l], s->u, s->o, s->ta, s->tb);
  for (int i = 0; i < d; i++) h[i] += s->o[i];
}

/* q, k, v of the SWA sublayer at position t, RoPE applied to q and k.
 * Writes q into s->q[0..d), k into s->kcur, v into s->vcur. */
static void swa_project(const orc_cfg *c, const orc_weights *w, int l,
                        const real *h, long t, scratch *s) {
  int d = c->d, H = c->n_heads, dh = c->head_dim;
  orc_rmsnorm(h, w->dec_ln1[l], d, c->rms_eps, s->u);
  orc_linear(w->dec_wqkv[l], s->u, 3 * d, d, s->q);
  for (int hd = 0; hd < H; hd++) {
    orc_rope(s->q + hd * dh, dh, t, c->rope_theta);
    orc_rope(s->q + d + hd * dh, dh, t, c->rope_theta);
  }
  memcpy(s->kcur, s->q + d, sizeof(real) * d);
  memcpy(s->vcur, s->q + 2 * d, sizeof(real) * d);
}

/* -------------------------------------------------- decoder transition */

/* One recurrent decoder transition H_{t-1} -> H_t for one sequence.
 * [RLT-96] "Architecture": H_t = (s_t, C_t^D); per token a gated merge of e_t
 * with s_{t-1}, then each decoder block runs causal SWA over decoder
 * activations, cross-attention to encoder memory and an FFN; the window W
 * includes the current token, so at most W-1 historical entries per layer are
 * retained. [RLT-TC] "What is this technology": no reset at the prompt /
 * response boundary (this function has no notion of that boundary).
 *
 * State (in/out): s [d]; win [L_D][2][W-1][d] holding the post-RoPE K and the V
 * of positions t-(W-1) .. t-1, oldest first, right-aligned (slot W-2 is the
 * newest); slots of positions < 0 are zero and never read.
 * e_t [d]; mem [G][mem_cap][2][d] with rows 0..t valid. */
static void step_with(const orc_cfg *c, const orc_weights *w, const real *e_t,
                      const real *mem, int mem_cap, long t, real *s, real *win,
                      real *h, scratch *sc) {
  int d = c->d, H = c->n_heads, dh = c->head_dim, Wm1 = c->window - 1;
  long nh = t < Wm1 ? t : Wm1; /* retained history entries */
  gated_merge(c, w, e_t, s, h, sc->cat, sc->gpre);
  for (int l = 0; l < c->n_dec; l++) {
    real *wk = win + ((size_t)l * 2 + 0) * Wm1 * d;
    real *wv = win + ((size_t)l * 2 + 1) * Wm1 * d;
    /* sliding-window self-attention: history (oldest first) then current */
    swa_project(c, w, l, h, t, sc);
    for (int hd = 0; hd < H; hd++) {
      int n = 0;
      for (long j = Wm1 - nh; j < Wm1; j++, n++) {
        sc->kp[n] = wk + (size_t)j * d + hd * dh;
        sc->vp[n] = wv + (size_t)j * d + hd * dh;
      }
      sc->kp[n] = sc->kcur + hd * dh;
      sc->vp[n] = sc->vcur + hd * dh;
      n++;
      orc_attend(sc->q + hd * dh, sc->kp, sc->vp, n, dh, sc->sc, sc->a + hd * dh);
    }
    orc_linear(w->dec_wo[l], sc->a, d, d, sc->o);
    for (int i = 0; i < d; i++) h[i] += sc->o[i];
    /* retain the current entry: drop the oldest slot, append at the right */
    if (Wm1 > 0) {
      memmove(wk, wk + d, sizeof(real) * (size_t)(Wm1 - 1) * d);
      memmove(wv, wv + d, sizeof(real) * (size_t)(Wm1 - 1) * d);
      memcpy(wk + (size_t)(Wm1 - 1) * d, sc->kcur, sizeof(real) * d);
      memcpy(wv + (size_t)(Wm1 - 1) * d, sc->vcur, sizeof(real) * d);
    }
    cross_attn_sublayer(c, w, l, mem, mem_cap, t, h, sc);
    ffn_sublayer(c, w, l, h, sc);
  }
  /* s_t: the final decoder output vector, read by the next-token head */
  orc_rmsnorm(h, w->dec_lnf, d, c->rms_eps, s);
}

void orc_step(const orc_cfg *c, const orc_weights *w, const real *e_t,
              const real *mem, int mem_cap, long t, real *s, real *win) {
  scratch sc;
  int n_keys = (int)(t + 1 > c->window ? t + 1 : c->window);
  scratch_init(&sc, c, n_keys);
  real *h = calloc((size_t)c->d, sizeof(real));
  step_with(c, w, e_t, mem, mem_cap, t, s, win, h, &sc);
  free(h);
  scratch_free(&sc);
}

/* Steps t0 .. t1-1 in order (the decoder runs over every prompt and response
 * token: [RLT-FT] "How slow is per-token recurrence to train?"). s_out, if
 * not NULL, receives s_t for each step, [t1-t0][d]. e [mem_cap][d]. */
void orc_decode(const orc_cfg *c, const orc_weights *w, const real *e,
                const real *mem, int mem_cap, long t0, long t1, real *s,
                real *win, real *s_out) {
  scratch sc;
  scratch_init(&sc, c, (int)(t1 > c->window ? t1 : c->window));
  real *h = calloc((size_t)c->d, sizeof(real));
  for (long t = t0; t < t1; t++) {
    step_with(c, w, e + (size_t)t * c->d, mem, mem_cap, t, s, win, h, &sc);
    if (s_out) memcpy(s_out + (size_t)(t - t0) * c->d, s, sizeof(real) * c->d);
  }
  free(h);
  scratch_free(&sc);
}

/* Initial state: the learned start state s* and an empty cache, set once
 * before the first token ([RLT-96] "Architecture"). */
void orc_init_state(const orc_cfg *c, const orc_weights *w, real *s, real *win) {
  memcpy(s, w->sstar, sizeof(real) * c->d);
  size_t n = (size_t)c->n_dec * 2 * (c->window - 1) * c->d;
  if (n) memset(win, 0, sizeof(real) * n);
}

/* Encoder then every decoder step of one sequence from the initial state. */
int orc_run(const orc_cfg *c, const orc_weights *w, const int *tok, int T,
            real *s_out, real *s, real *win) {
  real *e = calloc((size_t)(T > 0 ? T : 1) * c->d, sizeof(real));
  real *mem = calloc((size_t)c->mem_groups * (T > 0 ? T : 1) * 2 * c->d, sizeof(real));
  int rc = orc_encode(c, w, tok, T, e, mem, T > 0 ? T : 1);
  orc_init_state(c, w, s, win);
  if (rc == 0) orc_decode(c, w, e, mem, T > 0 ? T : 1, 0, T, s, win, s_out);
  free(e);
  free(mem);
  return rc;
}

/* Independent formulation of the window: keep the full K/V history of every
 * decoder layer and mask explicitly, keeping position j for query t iff
 * t - W < j <= t. Same other sublayers. s_out [T][d]. */
void orc_decode_bruteforce(const orc_cfg *c, const orc_weights *w, const real *e,
                           const real *mem, int mem_cap, int T, real *s_out) {
  int d = c->d, H = c->n_heads, dh = c->head_dim;
  scratch sc;
  scratch_init(&sc, c, T > c->window ? T : c->window);
  real *hist = calloc((size_t)c->n_dec * (T > 0 ? T : 1) * 2 * d, sizeof(real));
  real *h = calloc((size_t)d, sizeof(real));
  real *s = calloc((size_t)d, sizeof(real));
  memcpy(s, w->sstar, sizeof(real) * d);
  for (int t = 0; t < T; t++) {
    gated_merge(c, w, e + (size_t)t * d, s, h, sc.cat, sc.gpre);
    for (int l = 0; l < c->n_dec; l++) {
      real *hl = hist + (size_t)l * T * 2 * d;
      swa_project(c, w, l, h, t, &sc);
      memcpy(hl + ((size_t)t * 2 + 0) * d, sc.kcur, sizeof(real) * d);
      memcpy(hl + ((size_t)t * 2 + 1) * d, sc.vcur, sizeof(real) * d);
      for (int hd = 0; hd < H; hd++) {
        int n = 0;
        for (int j = 0; j <= t; j++) {
          if (!(t - c->window < j)) continue; /* explicit window mask */
          sc.kp[n] = hl + ((size_t)j * 2 + 0) * d + hd * dh;
          sc.vp[n] = hl + ((size_t)j * 2 + 1) * d + hd * dh;
          n++;
        }
        orc_attend(sc.q + hd * dh, sc.kp, sc.vp, n, dh, sc.sc, sc.a + hd * dh);
      }
      orc_linear(w->dec_wo[l], sc.a, d, d, sc.o);
      for (int i = 0; i < d; i++) h[i] += sc.o[i];
      cross_attn_sublayer(c, w, l, mem, mem_cap, t, h, &sc);
      ffn_sublayer(c, w, l, h, &sc);
    }
    orc_rmsnorm(h, w->dec_lnf, d, c->rms_eps, s);
    memcpy(s_out + (size_t)t * d, s, sizeof(real) * d);
  }
  free(hist); free(h); free(s);
  scratch_free(&sc);
}

/* A standard token-parallel decoder pass with window masks and no feedback:
 * every position's input is e_t, layer by layer over all positions at once.
 * [RLT-96] "Three design principles": such a pass is not equivalent to the
 * recurrence in general; with alpha = 0 ([RLT-PV] body, the feedback-off
 * control) the recurrence reduces to it. s_out [T][d]. */
void orc_decode_parallel_nofeedback(const orc_cfg *c, const orc_weights *w,
                                    const real *e, const real *mem, int mem_cap,
                                    int T, real *s_out) {
  int d = c->d, H = c->n_heads, dh = c->head_dim, Wn = c->window;
  scratch sc;
  scratch_init(&sc, c, T > Wn ? T : Wn);
  size_t Tn = (size_t)(T > 0 ? T : 1);
  real *h = calloc(Tn * d, sizeof(real));
  real *qkv = calloc(Tn * 3 * d, sizeof(real));
  real *a = calloc(Tn * d, sizeof(real));
  memcpy(h, e, sizeof(real) * (size_t)T * d);
  for (int l = 0; l < c->n_dec; l++) {
    for (int t = 0; t < T; t++) {
      swa_project(c, w, l, h + (size_t)t * d, t, &sc);
      memcpy(qkv + (size_t)t * 3 * d, sc.q, sizeof(real) * 3 * d);
    }
    for (int t = 0; t < T; t++) {
      int j0 = t - Wn + 1 > 0 ? t - Wn + 1 : 0;
      for (int hd = 0; hd < H; hd++) {
        int n = 0;
        for (int j = j0; j <= t; j++, n++) {
          sc.kp[n] = qkv + (size_t)j * 3 * d + d + hd * dh;
          sc.vp[n] = qkv + (size_t)j * 3 * d + 2 * d + hd * dh;
        }
        orc_attend(qkv + (size_t)t * 3 * d + hd * dh, sc.kp, sc.vp, n, dh,
                   sc.sc, a + (size_t)t * d + hd * dh);
      }
    }
    for (int t = 0; t < T; t++) {
      real *ht = h + (size_t)t * d;
      orc_linear(w->dec_wo[l], a + (size_t)t * d, d, d, sc.o);
      for (int i = 0; i < d; i++) ht[i] += sc.o[i];
      cross_attn_sublayer(c, w, l, mem, mem_cap, t, ht, &sc);
      ffn_sublayer(c, w, l, ht, &sc);
    }
  }
  for (int t = 0; t < T; t++)
    orc_rmsnorm(h + (size_t)t * d, w->dec_lnf, d, c->rms_eps, s_out + (size_t)t * d);
  free(h); free(qkv); free(a);
  scratch_free(&sc);
}

/* -------------------------------------------------------- serving loop */

/* Next-token logits read from the decoder output s_t ([RLT-96]
 * "Architecture": the next-token distribution is read from s_t), with the
 * embedding matrix as the output head (reading: tied input and output
 * embeddings; the pages name no separate head). logits [V]. */
void orc_lm_head(const orc_cfg *c, const orc_weights *w, const real *s,
                 real *logits) {
  orc_linear(w->embed, s, c->vocab, c->d, logits);
}

/* One token from logits (reading: the pages leave decoding open).
 * tau = 0: the first index of the largest logit. tau > 0: inverse-CDF
 * sampling of softmax(logits / tau) at u in [0, 1): the smallest v whose
 * cumulative weight exceeds u times the total, with weights
 * exp((logit_v - max) / tau). */
int orc_sample(const real *logits, int V, double tau, double u) {
  int arg = 0;
  for (int v = 1; v < V; v++)
    if (logits[v] > logits[arg]) arg = v;
  if (!(tau > 0)) return arg;
  double Z = 0;
  for (int v = 0; v < V; v++) Z += exp(((double)logits[v] - (double)logits[arg]) / tau);
  double target = u * Z, cum = 0;
  int last = arg;
  for (int v = 0; v < V; v++) {
    double p = exp(((double)logits[v] - (double)logits[arg]) / tau);
    cum += p;
    if (p > 0) last = v;
    if (cum > target) return v;
  }
  return last;
}

/* Independent sequences in parallel (OpenMP over sequences only): full
 * encoder + decoder run of each; s_final [B][d] gets each sequence's last s.
 * tok [B][tok_stride]. Returns the number of threads used. */
int orc_run_batch(const orc_cfg *c, const orc_weights *w, const int *tok,
                  int tok_stride, const int *lengths, int B, int n_threads,
                  real *s_final) {
  int used = 1;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
  {
#pragma omp single
    used = omp_get_num_threads();
  }
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int b = 0; b < B; b++) {
    size_t wn = (size_t)c->n_dec * 2 * (c->window - 1) * c->d;
    real *win = calloc(wn > 0 ? wn : 1, sizeof(real));
    orc_run(c, w, tok + (size_t)b * tok_stride, lengths[b], NULL,
            s_final + (size_t)b * c->d, win);
    free(win);
  }
  return used;
}
