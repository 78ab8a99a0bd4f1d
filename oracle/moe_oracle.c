/*
 * moe_oracle.c -- plain, slow, CPU reference of the top-k routed MoE FFN forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU
 * baseline may load this file's library.  It shares no code, header, table or
 * constant with the CUDA path, and it never calls it.
 *
 * Every value is decoded to double by this file's own decoders (bf16, e2m1,
 * e8m0) and every sum is a serial double loop in index order; only the routing
 * key of an unbiased softmax stays the exact fp32 value it is.
 *
 * Sources (the five pages on the MoE FFN, cited by title and item):
 *   [MoE]     "MoE" (ClikaRT Python nn/MoE): __init__ options, forward, set_weights.
 *   [QMoE]    "ClikaRT::nn::QMoEWoQ": forward(x, router_logits, shared_output),
 *             weight-only quantized experts decoded block by block.
 *   [MoeSpec] "Struct MoeSpec" (logicaffeine tensor_recognize::qwen): field docs
 *             router_bias, biases, renormalize, act, score, weigh_inputs,
 *             selection_bias, groups, scale, and method sum_can_clamp.
 *   [Op]      "MoE" graph-op page (graiphic): input layouts fc1/fc2 and the
 *             attributes activation_alpha/beta, k, normalize_routing_weights,
 *             swiglu_fusion, swiglu_limit.
 *   [Moe]     "Struct Moe" (logicaffeine model::spec): shared_experts, shared_dff,
 *             shared_gate, biases, groups.
 *
 * Readings where the pages are silent (each one also listed in the design notes):
 *   - ties between experts (and between groups) go to the lower index;
 *   - an unbiased softmax ranks by the biased logit l' (monotone in the score);
 *     every other key is formed in double: sigma(l') or softmax(l'), plus the
 *     selection bias;
 *   - a NaN key ranks below every number;
 *   - a group's score is the sum of its two largest keys; groups are contiguous;
 *   - the renormalizing sum is clamped from below: w / max(sum, 2^-14);
 *   - the routed scale multiplies every kept weight, after renormalization;
 *   - gated activation h = act(g) * (u + beta); for SiLU act(g) = g*sigmoid(alpha*g);
 *     limit L > 0 clamps g <- min(g, L) and u <- clamp(u, -L, L) first (SiLU only);
 *   - gate is the first half of the fused stack (concat) or the even rows
 *     (interleaved);
 *   - the shared expert is one more expert of the same kind (same activation and
 *     layout, dff = Fs, no biases), weighed 1 or sigmoid(x . g_s);
 *   - MXFP4: blocks of 32 along K, e2m1 code (sign bit 3, exponent bits 2..1,
 *     mantissa bit 0), low nibble = even k, e8m0 scale 2^(s-127) per (row, block).
 *     Parity unpinned against any real checkpoint's packing.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- enums (values chosen by the binding; independent of the CUDA library) ---- */
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_MXFP4 = 2 };
enum { ORC_SOFTMAX = 0, ORC_SIGMOID = 1 };
enum { ORC_SILU = 0, ORC_GELU_ERF = 1, ORC_GELU_TANH = 2, ORC_RELU = 3, ORC_IDENTITY = 4 };
enum { ORC_CONCAT = 0, ORC_INTERLEAVED = 1, ORC_UNFUSED = 2 };
enum { ORC_GATED = 0, ORC_PLAIN = 1 };

typedef struct {
  int64_t T, d, F, E, k, Fs;
  int32_t act_dtype;    /* x, biases, shared weights, shared_output: F32 or BF16 */
  int32_t w_dtype;      /* routed expert stacks: F32, BF16 or MXFP4 */
  int32_t logit_dtype;  /* router_logits and router_bias: F32 or BF16 */
  int32_t score, renormalize;
  double routed_scale;
  int32_t n_group, topk_group, weigh_inputs, act;
  double alpha, beta, limit;
  int32_t gu_layout, shared_gate;
  int32_t ffn;          /* ORC_GATED: act(gate) * (up + beta); ORC_PLAIN: act(fc1) alone */
  /* host pointers; NULL = absent */
  const void *x, *logits, *router_bias;
  const float *selection_bias;
  const void *gate_up, *gate_up_scales, *gate_up_bias;
  const void *down, *down_scales, *down_bias;
  const void *shared_gate_up, *shared_down, *shared_gate_vec, *shared_output;
  /* unfused layout: the gate stack [E, F, d] (w_dtype; MXFP4 scales [E, F, d/32])
     and its bias [E, F]; gate_up then holds the up rows [E, F, d] and their bias */
  const void *gate, *gate_scales, *gate_bias;
  /* router weight Wr [d, E] (act dtype): logits = x Wr when logits is NULL */
  const void *router_weight;
} orc_problem;

/* ---------------- decoders ---------------- */

/* bf16 is the upper half of an IEEE binary32. */
double orc_bf16(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* OCP MX e2m1: 1 sign, 2 exponent (bias 1), 1 mantissa; exponent 0 is subnormal. */
double orc_e2m1(int code) {
  int sign = (code >> 3) & 1, ex = (code >> 1) & 3, m = code & 1;
  double mag = ex == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, ex - 1);
  return sign ? -mag : mag;
}

/* OCP MX e8m0: 2^(s-127); 255 is NaN. */
double orc_e8m0(int s) {
  if (s == 255) return NAN;
  return ldexp(1.0, s - 127);
}

static double load(const void *p, int32_t dtype, int64_t i) {
  if (dtype == ORC_BF16) return orc_bf16(((const uint16_t *)p)[i]);
  return (double)((const float *)p)[i];
}

/* fp32 value of a logit-typed element (bf16 -> fp32 is exact). */
static float load_f32(const void *p, int32_t dtype, int64_t i) {
  return (float)load(p, dtype, i);
}

/* Element (r, c) of one expert's [rows, K] weight matrix, K contiguous. */
static double weight(const void *w, const void *scales, int32_t dtype, int64_t e, int64_t rows,
                     int64_t K, int64_t r, int64_t c) {
  if (dtype == ORC_MXFP4) {
    const uint8_t *q = (const uint8_t *)w;
    const uint8_t *s = (const uint8_t *)scales;
    int64_t row = e * rows + r;
    uint8_t byte = q[row * (K / 2) + c / 2];
    int code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return orc_e2m1(code) * orc_e8m0(s[row * (K / 32) + c / 32]);
  }
  return load(w, dtype, (e * rows + r) * K + c);
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* ---------------- routing ([MoeSpec] fields; [Op] k, normalize_routing_weights) ---------------- */

/* a outranks b: larger key first, NaN below every number, then the lower index. */
static int outranks(double ka, int64_t ia, double kb, int64_t ib) {
  int na = isnan(ka), nb = isnan(kb);
  if (na || nb) {
    if (na && nb) return ia < ib;
    return nb;
  }
  if (ka != kb) return ka > kb;
  return ia < ib;
}

/*
 * Route token t.  Writes the k chosen experts (best first), their weights, and
 * optionally every expert's key and score.  Returns 0, or -1 on a bad argument.
 */
int orc_route(const orc_problem *p, int64_t t, int32_t *idx, double *w, double *keys_out,
              double *scores_out) {
  const int64_t E = p->E, k = p->k;
  if (k < 1 || k > E) return -1;
  if (p->n_group > 0 && (E % p->n_group != 0 || p->topk_group < 1 || p->topk_group > p->n_group ||
                         p->topk_group * (E / p->n_group) < k))
    return -1;
  float *lp = (float *)malloc(sizeof(float) * E);
  double *s = (double *)malloc(sizeof(double) * E);
  double *key = (double *)malloc(sizeof(double) * E);
  char *eligible = (char *)malloc(E);
  char *taken = (char *)malloc(E);

  /* l' = l + Br, an fp32 add ([MoeSpec] router_bias: added to each logit before scoring).
     Without caller logits, l = x_t Wr ([MoeSpec] wr, indexed wr[(i-1)E + e]: Wr is [d, E]),
     summed in double over i and rounded once to fp32. */
  for (int64_t e = 0; e < E; e++) {
    float l;
    if (p->logits) {
      l = load_f32(p->logits, p->logit_dtype, t * E + e);
    } else {
      double acc = 0.0;
      for (int64_t i = 0; i < p->d; i++)
        acc += load(p->x, p->act_dtype, t * p->d + i) * load(p->router_weight, p->act_dtype, i * E + e);
      l = (float)acc;
    }
    if (p->router_bias) l = l + load_f32(p->router_bias, p->logit_dtype, e);
    lp[e] = l;
  }

  /* scores ([MoeSpec] score: softmax over every logit, or each logit's own sigmoid) */
  if (p->score == ORC_SOFTMAX) {
    double m = -INFINITY;
    for (int64_t e = 0; e < E; e++)
      if (lp[e] > m) m = lp[e];
    double den = 0.0;
    for (int64_t e = 0; e < E; e++) den += exp((double)lp[e] - m);
    for (int64_t e = 0; e < E; e++) s[e] = exp((double)lp[e] - m) / den;
  } else {
    for (int64_t e = 0; e < E; e++) s[e] = sigmoid((double)lp[e]);
  }

  /* selection key ([MoeSpec] selection_bias: chosen by score + B[e], weighed by score alone) */
  for (int64_t e = 0; e < E; e++) {
    if (p->score == ORC_SOFTMAX && !p->selection_bias)
      key[e] = (double)lp[e];
    else
      key[e] = s[e] + (p->selection_bias ? (double)p->selection_bias[e] : 0.0);
  }

  /* group limit ([MoeSpec] groups; [Moe] groups: scored by the two best experts) */
  for (int64_t e = 0; e < E; e++) eligible[e] = 1;
  if (p->n_group > 0) {
    const int64_t G = p->n_group, per = E / G;
    double *gscore = (double *)malloc(sizeof(double) * G);
    char *gtaken = (char *)malloc(G);
    for (int64_t g = 0; g < G; g++) {
      int64_t b1 = -1, b2 = -1;
      for (int64_t e = g * per; e < (g + 1) * per; e++) {
        if (b1 < 0 || outranks(key[e], e, key[b1], b1)) {
          b2 = b1;
          b1 = e;
        } else if (b2 < 0 || outranks(key[e], e, key[b2], b2)) {
          b2 = e;
        }
      }
      gscore[g] = per >= 2 ? key[b1] + key[b2] : key[b1];
      gtaken[g] = 0;
    }
    for (int64_t e = 0; e < E; e++) eligible[e] = 0;
    for (int64_t r = 0; r < p->topk_group; r++) {
      int64_t best = -1;
      for (int64_t g = 0; g < G; g++)
        if (!gtaken[g] && (best < 0 || outranks(gscore[g], g, gscore[best], best))) best = g;
      gtaken[best] = 1;
      for (int64_t e = best * per; e < (best + 1) * per; e++) eligible[e] = 1;
    }
    free(gscore);
    free(gtaken);
  }

  /* top-k by repeated selection of the best remaining eligible expert */
  for (int64_t e = 0; e < E; e++) taken[e] = 0;
  for (int64_t j = 0; j < k; j++) {
    int64_t best = -1;
    for (int64_t e = 0; e < E; e++)
      if (eligible[e] && !taken[e] && (best < 0 || outranks(key[e], e, key[best], best))) best = e;
    taken[best] = 1;
    idx[j] = (int32_t)best;
  }

  /* weights: the unbiased score; renormalize with the 2^-14 clamp; then the routed scale */
  double sum = 0.0;
  for (int64_t j = 0; j < k; j++) {
    w[j] = s[idx[j]];
    sum += w[j];
  }
  if (p->renormalize) {
    double den = sum > 0x1p-14 ? sum : 0x1p-14;
    for (int64_t j = 0; j < k; j++) w[j] = w[j] / den;
  }
  for (int64_t j = 0; j < k; j++) w[j] = w[j] * p->routed_scale;

  if (keys_out)
    for (int64_t e = 0; e < E; e++) keys_out[e] = key[e];
  if (scores_out)
    for (int64_t e = 0; e < E; e++) scores_out[e] = s[e];
  free(lp);
  free(s);
  free(key);
  free(eligible);
  free(taken);
  return 0;
}

/* ---------------- expert FFN ([Op] fc1/fc2 layouts, activation attributes) ---------------- */

static double gated(const orc_problem *p, double g, double u) {
  double a;
  switch (p->act) {
  case ORC_SILU:
    if (p->limit > 0.0) {
      g = g < p->limit ? g : p->limit;
      u = u < p->limit ? (u > -p->limit ? u : -p->limit) : p->limit;
    }
    a = g * sigmoid(p->alpha * g);
    break;
  case ORC_GELU_ERF: a = 0.5 * g * (1.0 + erf(g / sqrt(2.0))); break;
  case ORC_GELU_TANH:
    a = 0.5 * g * (1.0 + tanh(sqrt(2.0 / acos(-1.0)) * (g + 0.044715 * g * g * g)));
    break;
  case ORC_RELU: a = g > 0.0 ? g : 0.0; break;
  default: a = g; break; /* identity */
  }
  return a * (u + p->beta);
}

/* The non-gated expert's activation of fc1's output ([Op] activation_type relu, gelu,
   silu or identity with fusion_size 1): the same functions without an up value,
   alpha for SiLU only, no limit and no beta. */
static double plain(const orc_problem *p, double g) {
  switch (p->act) {
  case ORC_SILU: return g * sigmoid(p->alpha * g);
  case ORC_GELU_ERF: return 0.5 * g * (1.0 + erf(g / sqrt(2.0)));
  case ORC_GELU_TANH: return 0.5 * g * (1.0 + tanh(sqrt(2.0 / acos(-1.0)) * (g + 0.044715 * g * g * g)));
  case ORC_RELU: return g > 0.0 ? g : 0.0;
  default: return g; /* identity */
  }
}

/*
 * One expert on input z[d]: out[d] = W_down[e] h + b_down[e], with
 *   gated: h_f = gated(W_gate[e] z + b_gate[e], W_up[e] z + b_up[e]);
 *   plain: h_f = plain(W_1[e] z + b_1[e])  ([Op] fc1 with fusion_size 1).
 * Gate and up rows come from the fused stack (concat or interleaved) or, unfused,
 * from the separate gate stack and the up stack ([MoE] set_weights gate_experts,
 * gate_bias; [Op] fc3_experts_weights).
 * e == E selects the shared expert (act dtype weights, dff = Fs, no biases; its
 * stack is [2Fs, d] gate rows first when the routed experts are unfused, [Fs, d]
 * for a plain FFN).
 */
int orc_expert(const orc_problem *p, int64_t e, const double *z, double *out) {
  const int64_t d = p->d;
  const int shared = (e == p->E);
  if (e < 0 || e > p->E || (shared && p->Fs <= 0)) return -1;
  const int64_t F = shared ? p->Fs : p->F;
  const void *gu = shared ? p->shared_gate_up : p->gate_up;
  const void *gus = shared ? NULL : p->gate_up_scales;
  const void *dn = shared ? p->shared_down : p->down;
  const void *dns = shared ? NULL : p->down_scales;
  const int32_t wdt = shared ? p->act_dtype : p->w_dtype;
  const int64_t ee = shared ? 0 : e;
  const void *bgu = shared ? NULL : p->gate_up_bias;
  const void *bd = shared ? NULL : p->down_bias;
  double *h = (double *)malloc(sizeof(double) * F);
  if (p->ffn == ORC_PLAIN) {
    for (int64_t f = 0; f < F; f++) {
      double g = 0.0;
      for (int64_t i = 0; i < d; i++) g += weight(gu, gus, wdt, ee, F, d, f, i) * z[i];
      if (bgu) g += load(bgu, p->act_dtype, ee * F + f);
      h[f] = plain(p, g);
    }
  } else if (p->gu_layout == ORC_UNFUSED && !shared) {
    for (int64_t f = 0; f < F; f++) {
      double g = 0.0, u = 0.0;
      for (int64_t i = 0; i < d; i++) g += weight(p->gate, p->gate_scales, wdt, ee, F, d, f, i) * z[i];
      for (int64_t i = 0; i < d; i++) u += weight(gu, gus, wdt, ee, F, d, f, i) * z[i];
      if (p->gate_bias) g += load(p->gate_bias, p->act_dtype, ee * F + f);
      if (bgu) u += load(bgu, p->act_dtype, ee * F + f);
      h[f] = gated(p, g, u);
    }
  } else {
    for (int64_t f = 0; f < F; f++) {
      int64_t rg = p->gu_layout == ORC_INTERLEAVED ? 2 * f : f;
      int64_t ru = p->gu_layout == ORC_INTERLEAVED ? 2 * f + 1 : F + f;
      double g = 0.0, u = 0.0;
      for (int64_t i = 0; i < d; i++) g += weight(gu, gus, wdt, ee, 2 * F, d, rg, i) * z[i];
      for (int64_t i = 0; i < d; i++) u += weight(gu, gus, wdt, ee, 2 * F, d, ru, i) * z[i];
      if (bgu) {
        g += load(bgu, p->act_dtype, ee * 2 * F + rg);
        u += load(bgu, p->act_dtype, ee * 2 * F + ru);
      }
      h[f] = gated(p, g, u);
    }
  }
  for (int64_t o = 0; o < d; o++) {
    double acc = 0.0;
    for (int64_t f = 0; f < F; f++) acc += weight(dn, dns, wdt, ee, d, F, o, f) * h[f];
    if (bd) acc += load(bd, p->act_dtype, ee * d + o);
    out[o] = acc;
  }
  free(h);
  return 0;
}

/* ---------------- one token ([QMoE] forward; [MoeSpec] weigh_inputs; [Moe] shared) ---------------- */

int orc_token(const orc_problem *p, int64_t t, double *y) {
  const int64_t d = p->d, k = p->k;
  int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * k);
  double *w = (double *)malloc(sizeof(double) * k);
  double *x = (double *)malloc(sizeof(double) * d);
  double *z = (double *)malloc(sizeof(double) * d);
  double *o = (double *)malloc(sizeof(double) * d);
  int rc = orc_route(p, t, idx, w, NULL, NULL);
  if (rc == 0) {
    for (int64_t i = 0; i < d; i++) x[i] = load(p->x, p->act_dtype, t * d + i);
    for (int64_t i = 0; i < d; i++) y[i] = 0.0;
    for (int64_t j = 0; j < k; j++) {
      /* weigh-inputs: the weight scales the expert's input, its output joins unweighted */
      double zin = p->weigh_inputs ? w[j] : 1.0;
      double wout = p->weigh_inputs ? 1.0 : w[j];
      for (int64_t i = 0; i < d; i++) z[i] = zin * x[i];
      orc_expert(p, idx[j], z, o);
      for (int64_t i = 0; i < d; i++) y[i] += wout * o[i];
    }
    if (p->Fs > 0) {
      orc_expert(p, p->E, x, o);
      double gate = 1.0;
      if (p->shared_gate) {
        double dot = 0.0;
        for (int64_t i = 0; i < d; i++) dot += x[i] * load(p->shared_gate_vec, p->act_dtype, i);
        gate = sigmoid(dot);
      }
      for (int64_t i = 0; i < d; i++) y[i] += gate * o[i];
    }
    if (p->shared_output)
      for (int64_t i = 0; i < d; i++) y[i] += load(p->shared_output, p->act_dtype, t * d + i);
  }
  free(idx);
  free(w);
  free(x);
  free(z);
  free(o);
  return rc;
}

/*
 * Tokens tokens[0..n) -> y[n, d] (double).  Tokens are independent; the
 * threads split them, each token's arithmetic stays serial, so the result does
 * not depend on the thread count.  Returns 0, or the first failing status.
 */
int orc_forward(const orc_problem *p, const int64_t *tokens, int64_t n, double *y, int nthreads) {
  int rc = 0;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : rc)
#endif
  for (int64_t i = 0; i < n; i++) rc |= orc_token(p, tokens[i], y + i * p->d);
  (void)nthreads;
  return rc;
}

/* Threads orc_forward would use for nthreads <= 0. */
int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
