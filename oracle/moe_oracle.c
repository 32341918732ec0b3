/*
 * Oracle for the routed mixture-of-experts layer -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow CPU restatement of what the layer computes, in fp64, written
 * from the pages' description and sharing no code with the CUDA library.  Only
 * the tests, the package smoke check and the benchmark's CPU-baseline leg may
 * load it.  Every quantity is converted exactly to double (bf16 -> its value,
 * int8 -> q*s, int4 -> q*s) and accumulated in fp64 in index order; there is no
 * blocking, fusion or reordering beyond the definition.
 *
 * The layer, per token t (sources named per step below):
 *   1. logits   l_e = sum_h W_r[e,h] x[t,h]                   for every expert e
 *   2. keys     sigmoid router: s_e = 1/(1+exp(-l_e)), key_e = s_e + b_e
 *               softmax router: key_e = exp(l_e - m) / sum_{a active} exp(l_a - m)
 *      Kimi-Linear: top 8 on sigmoid score plus correction bias, the chosen
 *       scores renormalised and scaled by 2.446 -- Kimi-Linear LiteRT-LM
 *       details page, Conversion notes, mixture-of-experts bullet; the CMF code
 *       specialist page (How it was made, step 1) names the same sigmoid router
 *       and selection bias.  Qwen3: softmax, top 8 and renormalisation as
 *       plain ops -- Qwen3-30B-A3B LiteRT-LM card, Conversion Notes.
 *   3. top-k    sort the ACTIVE experts by (key descending, index ascending) and
 *               keep the first k; masked experts are never selectable (the CMF
 *               page's Defrag step equates the sliced file with a runtime mask).
 *   4. weights  w_j = r_j / sum_{selected} r * scale, with r = s (sigmoid scores,
 *               WITHOUT the bias, which only selects) or r = p (softmax).
 *   5. experts  for each selected e: g = W_gate[e] x, u = W_up[e] x,
 *               a = act(g) * u  (gated), o = W_down[e] a; act = SiLU,
 *               g * sigmoid(g), or GELU in its tanh form.
 *               a token runs only through its 8 routed experts --
 *               Qwen3 card, Conversion Notes; activation 'silu' -- same card and
 *               the Kimi details page (moe op with SiLU); the moe op's other
 *               activation, 'gelu_tanh', is named by the same two passages (the
 *               runtime's error messages); its formula is the paper's, cited at
 *               act_value below.
 *   6. combine  y[t] = sum_j w_j o_j in slot order; no residual add (the add
 *               sits outside the moe op -- Qwen3 card, Conversion Notes,
 *               moe_fusion_guard bullet).
 *
 * Stored formats read here (rows are output channels, columns the reduction):
 *   W_gate, W_up [E, I, H]; W_down [E, H, I]
 *   f32 / bf16 (raw 16-bit patterns) / int8 with s[E, rows] (one scale per
 *   output row and expert -- Kimi details page, quantization bullet) / int4
 *   packed two per byte, low nibble = even column, two's complement, with
 *   s[E, rows, cols/32] (block 32, fp32 scales -- Qwen3 card, Artifacts table),
 *   or the same nibbles with s[E, rows, cols/128] (128-wide expert blocks --
 *   Qwen3 card, the int4 notes comparing 128-wide with 32-wide blocks).
 */
#include <math.h>
#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_INT8 = 2, ORC_INT4 = 3, ORC_INT4_B128 = 4 };
enum { ORC_SILU = 0, ORC_GELU_TANH = 1 };
enum { ORC_SIGMOID = 0, ORC_SOFTMAX = 1 };
enum { ORC_GATE = 0, ORC_UP = 1, ORC_DOWN = 2 };

typedef struct {
  int32_t H, I, E, k;
  int32_t router; /* ORC_SIGMOID or ORC_SOFTMAX */
  int32_t wfmt;   /* expert storage format */
  int32_t xfmt;   /* ORC_F32 or ORC_BF16 */
  int32_t act;    /* ORC_SILU or ORC_GELU_TANH */
  double scale;   /* 2.446 (Kimi) or 1 (Qwen3) */
  const float* W_r;      /* [E, H] */
  const float* b;        /* [E] or NULL (= zero bias) */
  const uint8_t* mask;   /* [E] 1 = active, or NULL (all active) */
  const void* W_gate;
  const void* W_up;
  const void* W_down;
  const float* s_gate;
  const float* s_up;
  const float* s_down;
} oracle_layer;

/* ---------------------------------------------------------------- decoding */

static double bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static double x_value(const oracle_layer* L, const void* x, int64_t t, int64_t h) {
  if (L->xfmt == ORC_BF16) return bf16_value(((const uint16_t*)x)[t * L->H + h]);
  return (double)((const float*)x)[t * L->H + h];
}

/* value of expert weight (row, col) of matrix `which` of expert e */
double oracle_weight(const oracle_layer* L, int which, int64_t e, int64_t row, int64_t col) {
  const int64_t R = (which == ORC_DOWN) ? L->H : L->I;
  const int64_t C = (which == ORC_DOWN) ? L->I : L->H;
  const void* W = which == ORC_GATE ? L->W_gate : which == ORC_UP ? L->W_up : L->W_down;
  const float* S = which == ORC_GATE ? L->s_gate : which == ORC_UP ? L->s_up : L->s_down;
  const int64_t r = e * R + row;
  switch (L->wfmt) {
    case ORC_F32:
      return (double)((const float*)W)[r * C + col];
    case ORC_BF16:
      return bf16_value(((const uint16_t*)W)[r * C + col]);
    case ORC_INT8:
      return (double)((const int8_t*)W)[r * C + col] * (double)S[r];
    case ORC_INT4:
    case ORC_INT4_B128: {
      const int64_t B = L->wfmt == ORC_INT4 ? 32 : 128;
      const uint8_t byte = ((const uint8_t*)W)[r * (C / 2) + col / 2];
      int nib = (col & 1) ? (byte >> 4) : (byte & 0xF);
      if (nib >= 8) nib -= 16;
      return (double)nib * (double)S[r * (C / B) + col / B];
    }
  }
  return NAN;
}

static int is_active(const oracle_layer* L, int e) { return L->mask == NULL || L->mask[e] != 0; }

static int count_active(const oracle_layer* L) {
  int n = 0;
  for (int e = 0; e < L->E; ++e) n += is_active(L, e);
  return n;
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* the gate's activation: SiLU g*sigmoid(g), or the tanh form of GELU,
   g/2 * (1 + tanh(sqrt(2/pi) * (g + 0.044715 g^3))) (Hendrycks and Gimpel,
   "Gaussian Error Linear Units", section 2) */
static double act_value(const oracle_layer* L, double g) {
  if (L->act == ORC_GELU_TANH) {
    const double c = sqrt(2.0 / M_PI);
    return 0.5 * g * (1.0 + tanh(c * (g + 0.044715 * g * g * g)));
  }
  return g * sigmoid(g);
}

/* ------------------------------------------------------------------ router */

/* logits[(t - t0) * E + e] for tokens [t0, t1), all experts (masking is a selection rule) */
int oracle_router_logits(const oracle_layer* L, const void* x, int64_t t0, int64_t t1, double* logits) {
  if (!L || !x || !logits || t1 < t0) return -1;
  for (int64_t t = t0; t < t1; ++t)
    for (int64_t e = 0; e < L->E; ++e) {
      double acc = 0.0;
      for (int64_t h = 0; h < L->H; ++h) acc += (double)L->W_r[e * L->H + h] * x_value(L, x, t, h);
      logits[(t - t0) * L->E + e] = acc;
    }
  return 0;
}

typedef struct {
  double key;
  int e;
} ranked;

/* key descending, then expert index ascending */
static int by_key_then_index(const void* pa, const void* pb) {
  const ranked* a = (const ranked*)pa;
  const ranked* b = (const ranked*)pb;
  if (a->key > b->key) return -1;
  if (a->key < b->key) return 1;
  return a->e < b->e ? -1 : (a->e > b->e ? 1 : 0);
}

/* selection keys of every expert for one token (masked experts get -inf) */
int oracle_keys(const oracle_layer* L, const double* logits, double* keys) {
  if (!L || !logits || !keys) return -1;
  if (L->router == ORC_SIGMOID) {
    for (int e = 0; e < L->E; ++e)
      keys[e] = is_active(L, e) ? sigmoid(logits[e]) + (L->b ? (double)L->b[e] : 0.0) : -INFINITY;
    return 0;
  }
  if (L->router == ORC_SOFTMAX) {
    double m = -INFINITY, z = 0.0;
    for (int e = 0; e < L->E; ++e)
      if (is_active(L, e) && logits[e] > m) m = logits[e];
    for (int e = 0; e < L->E; ++e)
      if (is_active(L, e)) z += exp(logits[e] - m);
    for (int e = 0; e < L->E; ++e) keys[e] = is_active(L, e) ? exp(logits[e] - m) / z : -INFINITY;
    return 0;
  }
  return -1;
}

/*
 * Route one token from its logits: idx[k], w[k] in descending key order, and
 * margin = key of the k-th selected minus key of the best unselected active
 * expert (+inf when every active expert is selected).
 */
int oracle_select(const oracle_layer* L, const double* logits, int32_t* idx, double* w, double* margin) {
  const int E = L->E, k = L->k;
  const int n_act = count_active(L);
  if (k < 1 || k > n_act) return -1;
  double* keys = (double*)malloc(sizeof(double) * E);
  ranked* order = (ranked*)malloc(sizeof(ranked) * n_act);
  if (!keys || !order || oracle_keys(L, logits, keys) != 0) {
    free(keys);
    free(order);
    return -1;
  }
  int n = 0;
  for (int e = 0; e < E; ++e)
    if (is_active(L, e)) {
      order[n].key = keys[e];
      order[n].e = e;
      ++n;
    }
  qsort(order, n, sizeof(ranked), by_key_then_index);
  double total = 0.0;
  for (int j = 0; j < k; ++j) {
    const int e = order[j].e;
    const double r = (L->router == ORC_SIGMOID) ? sigmoid(logits[e]) : keys[e];
    idx[j] = e;
    w[j] = r;
    total += r;
  }
  for (int j = 0; j < k; ++j) w[j] = w[j] / total * L->scale;
  if (margin) *margin = (k < n) ? order[k - 1].key - order[k].key : INFINITY;
  free(keys);
  free(order);
  return 0;
}

/* route tokens [t0, t1): idx/w/margin are indexed by (t - t0) */
int oracle_route(const oracle_layer* L, const void* x, int64_t t0, int64_t t1, int32_t* idx, double* w,
                 double* margin) {
  if (!L || !x || !idx || !w || t1 < t0) return -1;
  double* logits = (double*)malloc(sizeof(double) * L->E);
  if (!logits) return -1;
  int rc = 0;
  for (int64_t t = t0; t < t1 && rc == 0; ++t) {
    rc = oracle_router_logits(L, x, t, t + 1, logits);
    if (rc == 0)
      rc = oracle_select(L, logits, idx + (t - t0) * L->k, w + (t - t0) * L->k, margin ? margin + (t - t0) : NULL);
  }
  free(logits);
  return rc;
}

/* ----------------------------------------------------------------- experts */

/* o[H] = W_down[e] (SiLU(W_gate[e] xt) * (W_up[e] xt)) for one token vector xt[H] */
int oracle_expert(const oracle_layer* L, int64_t e, const double* xt, double* o) {
  if (!L || !xt || !o || e < 0 || e >= L->E) return -1;
  const int64_t H = L->H, I = L->I;
  double* a = (double*)malloc(sizeof(double) * I);
  if (!a) return -1;
  for (int64_t i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    for (int64_t h = 0; h < H; ++h) {
      g += oracle_weight(L, ORC_GATE, e, i, h) * xt[h];
      u += oracle_weight(L, ORC_UP, e, i, h) * xt[h];
    }
    a[i] = act_value(L, g) * u;
  }
  for (int64_t r = 0; r < H; ++r) {
    double acc = 0.0;
    for (int64_t i = 0; i < I; ++i) acc += oracle_weight(L, ORC_DOWN, e, r, i) * a[i];
    o[r] = acc;
  }
  free(a);
  return 0;
}

/*
 * y for tokens [t0, t1) under a GIVEN routing: y[(t - t0) * H + h] =
 * sum_j w[j] o_{idx[j]}[h] in slot order.  idx/w are indexed by (t - t0).
 */
int oracle_combine(const oracle_layer* L, const void* x, int64_t t0, int64_t t1, const int32_t* idx,
                   const double* w, double* y) {
  if (!L || !x || !idx || !w || !y || t1 < t0) return -1;
  const int64_t H = L->H;
  double* xt = (double*)malloc(sizeof(double) * H);
  double* o = (double*)malloc(sizeof(double) * H);
  if (!xt || !o) {
    free(xt);
    free(o);
    return -1;
  }
  int rc = 0;
  for (int64_t t = t0; t < t1 && rc == 0; ++t) {
    for (int64_t h = 0; h < H; ++h) xt[h] = x_value(L, x, t, h);
    double* yt = y + (t - t0) * H;
    for (int64_t h = 0; h < H; ++h) yt[h] = 0.0;
    for (int j = 0; j < L->k && rc == 0; ++j) {
      rc = oracle_expert(L, idx[(t - t0) * L->k + j], xt, o);
      for (int64_t h = 0; h < H; ++h) yt[h] += w[(t - t0) * L->k + j] * o[h];
    }
  }
  free(xt);
  free(o);
  return rc;
}

/* the whole layer for tokens [t0, t1): route, then combine under that routing */
int oracle_forward(const oracle_layer* L, const void* x, int64_t t0, int64_t t1, int32_t* idx, double* w,
                   double* margin, double* y) {
  int rc = oracle_route(L, x, t0, t1, idx, w, margin);
  if (rc == 0) rc = oracle_combine(L, x, t0, t1, idx, w, y);
  return rc;
}

/* ------------------------------------------------- shared expert + residual */
/*
 * The whole MoE block for tokens [t0, t1) under a given routing:
 *   y[t] = sum_j w_j o_{idx_j}(x_t)  +  shared(x_t)  +  residual[t]
 * The routed sum is oracle_combine's; shared(x) is one more gated FFN with
 * weight 1 over every token (256 routed experts plus one shared one -- Kimi-Linear
 * APEX quantization page, intro; the shared expert runs beside the moe op --
 * Kimi-Linear LiteRT-LM details page, Conversion notes, mixture-of-experts
 * bullet), described by S as a one-expert layer (S->E == 1, same H and
 * activation); the residual add is the block's own, outside the moe op (Qwen3
 * card, Conversion Notes, moe_fusion_guard bullet).  S and residual may be
 * NULL; residual is in x's format.
 */
int oracle_block(const oracle_layer* L, const oracle_layer* S, const void* x, const void* residual, int64_t t0,
                 int64_t t1, const int32_t* idx, const double* w, double* y) {
  if (S && (S->E != 1 || S->H != L->H)) return -1;
  int rc = oracle_combine(L, x, t0, t1, idx, w, y);
  if (rc != 0) return rc;
  const int64_t H = L->H;
  double* xt = (double*)malloc(sizeof(double) * H);
  double* o = (double*)malloc(sizeof(double) * H);
  if (!xt || !o) {
    free(xt);
    free(o);
    return -1;
  }
  for (int64_t t = t0; t < t1 && rc == 0; ++t) {
    double* yt = y + (t - t0) * H;
    if (S) {
      for (int64_t h = 0; h < H; ++h) xt[h] = x_value(L, x, t, h);
      rc = oracle_expert(S, 0, xt, o);
      for (int64_t h = 0; h < H; ++h) yt[h] += o[h];
    }
    if (residual)
      for (int64_t h = 0; h < H; ++h) yt[h] += x_value(L, residual, t, h);
  }
  free(xt);
  free(o);
  return rc;
}

/* ------------------------------------------------------- routing statistics */
/*
 * Per-expert routing frequencies and the covering expert set (CMF code
 * specialist page, How it was made: the Calibrate step records per-layer expert
 * routing frequencies over a corpus; the Defrag step keeps, per layer, the
 * smallest expert set that covers a given share (0.95) of that routing mass,
 * renumbers the kept experts into a dense prefix and slices router rows and
 * selection bias to match).
 */

/* counts[e] += number of (token, slot) entries equal to e; entries outside
   [0, E) are not counted */
int oracle_expert_counts(const int32_t* idx, int64_t n, int32_t E, uint64_t* counts) {
  if ((!idx && n) || !counts || E < 1 || n < 0) return -1;
  for (int64_t i = 0; i < n; ++i)
    if (idx[i] >= 0 && idx[i] < E) counts[idx[i]] += 1;
  return 0;
}

/*
 * Smallest set of experts whose counts reach cover * (sum of counts): experts
 * are taken by count descending (ties: lower index first) until the running
 * sum, as a double, is >= cover * total.  keep[e] = 1 for kept experts;
 * new_index[e] = position of e among the kept experts in ascending index order
 * (the dense prefix), or -1.  cover must lie in (0, 1].
 */
int oracle_cover_set(const uint64_t* counts, int32_t E, double cover, uint8_t* keep, int32_t* new_index,
                     int32_t* n_keep) {
  if (!counts || !keep || !new_index || !n_keep || E < 1 || !(cover > 0.0 && cover <= 1.0)) return -1;
  uint64_t total = 0;
  for (int e = 0; e < E; ++e) total += counts[e];
  const double target = cover * (double)total;
  for (int e = 0; e < E; ++e) keep[e] = 0;
  uint64_t cum = 0;
  int taken = 0;
  while ((double)cum < target && taken < E) {
    int best = -1; /* the largest count not yet kept, lowest index on ties */
    for (int e = 0; e < E; ++e)
      if (!keep[e] && (best < 0 || counts[e] > counts[best])) best = e;
    keep[best] = 1;
    cum += counts[best];
    ++taken;
  }
  int next = 0;
  for (int e = 0; e < E; ++e) new_index[e] = keep[e] ? next++ : -1;
  *n_keep = taken;
  return 0;
}
