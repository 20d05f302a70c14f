/*
 * Oracle for the Mixture-of-Experts FFN forward layer -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, CPU implementation in fp64 of what the layer computes, written from the
 * pages' definitions. Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * may call it; the product path never does. It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * Sources (page -- section):
 *   [G5]  Grok-1 book ch.5 "MoE routing & experts" -- 5.2 Router (fp32 logits x.W_r, softmax,
 *         TopK), 5.2.3 softmax-then-top-k without renormalisation, 5.3.5 GeGLU expert and the
 *         gate-weighted sum over k, 5.3.5.1 exact-erf vs tanh GELU.
 *   [L12] LLMs-from-scratch ch.12 "MoE" -- 12.1 top-k softmax over the selected set and the
 *         gated expert f_e(x) = [SiLU(x W1) (.) (x W2)] W3, 12.2 N*k dispatch records and
 *         accumulate-not-overwrite.
 *   [GS]  MoE series (GShard/Mixtral/Switch) -- 2.2 overflow: a dropped slot contributes 0.
 *   [W]   MoE formula-to-code walkthrough -- 1.1 max-subtracted softmax, 1.2 top-k ordered by
 *         descending score + renormalisation, 1.3 expert load, 2.1 balance loss, 3.1 capacity
 *         ceil(CF*N*K/E), 3.2 dispatch with dropped mask, 3.3 drop rate.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - top-k ties: lower expert index first; selection is made on the fp32 logits (softmax is
 *     strictly increasing, so the set equals the set selected on probabilities);
 *   - capacity slots are assigned slot-major by default: every rank-0 record in token order,
 *     then every rank-1 record, ... (the walkthrough's loop with its two loops swapped);
 *     token-major order (the walkthrough's own loop, [W] 3.2) is the other policy;
 *   - a dropped record contributes zero; by default the other slots keep their gates
 *     unchanged; the other policy ([GS] 2.2 case A, (w1, w2) -> (1, 0) when one of the two
 *     experts overflows) renormalises the gates of a token's kept slots to sum 1 whenever at
 *     least one slot was dropped and one was kept;
 *   - capacity = max(ceil(CF*N*K/E), min_capacity) ([GS] 2.1), min_capacity = 0 by default;
 *   - balance loss f_i = load_i / (N*k), P_i = mean full-softmax probability.
 *
 * Every floating-point step accumulates in double in the order the definition states.
 * Inputs: X / W1 / W2 / W3 are fp32 (dtype 0) or bf16 bit patterns (dtype 1), widened
 * exactly to double; W_r and bias are fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F32 0
#define OR_BF16 1

#define OR_SILU 0
#define OR_GELU_ERF 1
#define OR_GELU_TANH 2

/* ---------------------------------------------------------------- element access */

static double bf16_bits_to_double(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Widen n consecutive elements starting at element index `first` into `out`. */
static void widen(const void* base, int dtype, int64_t first, int64_t n, double* out) {
  if (dtype == OR_BF16) {
    const uint16_t* p = (const uint16_t*)base + first;
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_bits_to_double(p[i]);
  } else {
    const float* p = (const float*)base + first;
    for (int64_t i = 0; i < n; ++i) out[i] = (double)p[i];
  }
}

static int all_finite_f32(const float* v, int64_t n) {
  for (int64_t i = 0; i < n; ++i)
    if (!isfinite(v[i])) return 0;
  return 1;
}

/* ---------------------------------------------------------------- capacity  [W] 3.1 */

/* Capacity = ceil(CF * N * K / E), evaluated in double left to right. CF <= 0 means "no
 * capacity": every record fits, i.e. N*k. */
int64_t oracle_capacity(int64_t N, int32_t k, int32_t E, double cf) {
  if (cf <= 0.0) return N * (int64_t)k;
  return (int64_t)ceil(cf * (double)N * (double)k / (double)E);
}

/* GShard's form ([GS] 2.1): capacity = max(S/E * K * capacity_factor, min_capacity), the first
 * term rounded up as above. With CF <= 0 there is no capacity and min_capacity is unused. */
int64_t oracle_capacity_min(int64_t N, int32_t k, int32_t E, double cf, int64_t min_capacity) {
  const int64_t c = oracle_capacity(N, k, E, cf);
  if (cf <= 0.0) return c;
  return c > min_capacity ? c : min_capacity;
}

/* ---------------------------------------------------------------- router  [G5] 5.2 */

/* logits[t,e] = sum_d x[t,d] * W_r[d,e]  (+ bias[e]), in double, d ascending.
 * logits32 (optional) receives the fp32 rounding of each value: the router works in fp32
 * ([G5] 5.2.1), and top-k selection is decided on these fp32 values. */
void oracle_router_logits(int64_t N, int64_t D, int32_t E, const void* X, int32_t x_dtype,
                          const float* W_r, const float* bias, double* logits64,
                          float* logits32) {
#pragma omp parallel
  {
    double* x = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
      widen(X, x_dtype, t * D, D, x);
      for (int32_t e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += x[d] * (double)W_r[d * E + e];
        if (bias) acc += (double)bias[e];
        if (logits64) logits64[t * E + e] = acc;
        if (logits32) logits32[t * E + e] = (float)acc;
      }
    }
    free(x);
  }
}

/* p_i = exp(z_i - max z) / sum_j exp(z_j - max z)  over all E experts ([W] 1.1). */
static void softmax_row(const float* z, int32_t E, double* p) {
  double m = (double)z[0];
  for (int32_t e = 1; e < E; ++e)
    if ((double)z[e] > m) m = (double)z[e];
  double s = 0.0;
  for (int32_t e = 0; e < E; ++e) {
    p[e] = exp((double)z[e] - m);
    s += p[e];
  }
  for (int32_t e = 0; e < E; ++e) p[e] /= s;
}

/* Experts ordered by descending score; among equal scores the lower index comes first.
 * A stable insertion sort that only moves an element past a strictly smaller one. */
static void order_desc_f32(const float* z, int32_t E, int32_t* order) {
  for (int32_t e = 0; e < E; ++e) order[e] = e;
  for (int32_t i = 1; i < E; ++i) {
    int32_t cur = order[i];
    int32_t j = i - 1;
    while (j >= 0 && z[cur] > z[order[j]]) {
      order[j + 1] = order[j];
      --j;
    }
    order[j + 1] = cur;
  }
}

/* Routing from fp32 logits ([G5] 5.2, 5.2.3; [W] 1.1-1.3; [L12] 12.1):
 *   probs      = softmax over all E experts (fp64, max-subtracted);
 *   idx[t,0..k-1] = the k experts with the largest logits, rank 0 = largest;
 *   gate       = probs[idx]                      (renorm = 0: Grok-1, gates sum < 1)
 *              = probs[idx] / sum_{sel} probs    (renorm = 1: Mixtral / walkthrough).
 * probs [N,E] and prob_colsum [E] (= sum_t probs[t,e]) are optional outputs.
 * Returns 0, or -1 if a logit is not finite. */
int oracle_route(int64_t N, int32_t E, int32_t k, int32_t renorm, const float* logits32,
                 int32_t* idx, double* gate, double* probs, double* prob_colsum) {
  if (!all_finite_f32(logits32, N * E)) return -1;
  double* P = probs ? probs : (double*)malloc(sizeof(double) * (size_t)(N * E + 1));
#pragma omp parallel
  {
    int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
      const float* z = logits32 + t * E;
      double* p = P + t * E;
      softmax_row(z, E, p);
      order_desc_f32(z, E, order);
      double sel = 0.0;
      for (int32_t j = 0; j < k; ++j) sel += p[order[j]];
      for (int32_t j = 0; j < k; ++j) {
        idx[t * k + j] = order[j];
        gate[t * k + j] = renorm ? p[order[j]] / sel : p[order[j]];
      }
    }
    free(order);
  }
  if (prob_colsum) {
    for (int32_t e = 0; e < E; ++e) prob_colsum[e] = 0.0;
    for (int64_t t = 0; t < N; ++t)
      for (int32_t e = 0; e < E; ++e) prob_colsum[e] += P[t * E + e];
  }
  if (!probs) free(P);
  return 0;
}

/* Training-time routing variants ([G5] 5.2.2, [GS] 3) and the z-loss ([G5] 5.2.2).
 *   mode 0: plain top-k (oracle_route).
 *   mode 1, noisy top-k (Switch): z' = z + noise, formed in fp32 (the precision the kernel adds
 *           in, so both sides decide on the same values); top-k of z' and gates from
 *           softmax(z') (renormalised over the selected set when renorm).
 *   mode 2, GShard random routing: the first expert is the largest unperturbed logit; every
 *           later one is the largest z' = z + noise (fp32) among the experts not yet chosen;
 *           gates from the unperturbed softmax(z) (renormalised over the selected set when
 *           renorm: w_i = P_i / (P_0 + P_1) for top-2, [GS] 3).
 * Ties keep the lower expert index. probs / prob_colsum report the softmax the gates come
 * from. zloss (optional): mean over tokens of (log sum_e exp z_e)^2 on the unperturbed logits
 * (the penalty alpha * (log Z)^2 of [G5] 5.2.2 without alpha). noise may be NULL for mode 0. */
static int32_t argmax_excluding(const float* v, int32_t E, const uint8_t* taken) {
  int32_t best = -1;
  for (int32_t e = 0; e < E; ++e) {
    if (taken[e]) continue;
    if (best < 0 || v[e] > v[best]) best = e;
  }
  return best;
}

int oracle_route_ex(int64_t N, int32_t E, int32_t k, int32_t renorm, int32_t mode,
                    const float* logits32, const float* noise32, int32_t* idx, double* gate,
                    double* probs, double* prob_colsum, double* zloss) {
  if (mode == 0) {
    if (oracle_route(N, E, k, renorm, logits32, idx, gate, probs, prob_colsum) != 0) return -1;
  } else {
    if (!all_finite_f32(logits32, N * E) || noise32 == NULL || !all_finite_f32(noise32, N * E))
      return -1;
    double* P = probs ? probs : (double*)malloc(sizeof(double) * (size_t)(N * E + 1));
#pragma omp parallel
    {
      float* zn = (float*)malloc(sizeof(float) * (size_t)E);
      uint8_t* taken = (uint8_t*)malloc((size_t)E);
#pragma omp for schedule(static)
      for (int64_t t = 0; t < N; ++t) {
        const float* z = logits32 + t * E;
        for (int32_t e = 0; e < E; ++e) {
          volatile float sum = z[e] + noise32[t * E + e]; /* one fp32 rounding */
          zn[e] = sum;
          taken[e] = 0;
        }
        double* p = P + t * E;
        softmax_row(mode == 1 ? zn : z, E, p);
        for (int32_t j = 0; j < k; ++j) {
          const int32_t c = argmax_excluding((mode == 2 && j == 0) ? z : zn, E, taken);
          taken[c] = 1;
          idx[t * k + j] = c;
        }
        double sel = 0.0;
        for (int32_t j = 0; j < k; ++j) sel += p[idx[t * k + j]];
        for (int32_t j = 0; j < k; ++j)
          gate[t * k + j] = renorm ? p[idx[t * k + j]] / sel : p[idx[t * k + j]];
      }
      free(zn);
      free(taken);
    }
    if (prob_colsum) {
      for (int32_t e = 0; e < E; ++e) prob_colsum[e] = 0.0;
      for (int64_t t = 0; t < N; ++t)
        for (int32_t e = 0; e < E; ++e) prob_colsum[e] += P[t * E + e];
    }
    if (!probs) free(P);
  }
  if (zloss) {
    double acc = 0.0;
    for (int64_t t = 0; t < N; ++t) {
      const float* z = logits32 + t * E;
      double m = (double)z[0];
      for (int32_t e = 1; e < E; ++e)
        if ((double)z[e] > m) m = (double)z[e];
      double sum = 0.0;
      for (int32_t e = 0; e < E; ++e) sum += exp((double)z[e] - m);
      const double lz = m + log(sum);
      acc += lz * lz;
    }
    *zloss = N > 0 ? acc / (double)N : 0.0;
  }
  return 0;
}

/* Near-tie margin of each token: with the fp64 logits sorted descending s_0 >= s_1 >= ...,
 * margin = min over the gaps that decide the selected set and its order:
 * s_i - s_{i+1} for i = 0 .. min(k, E-1) - 1. (+inf when E == 1.) */
void oracle_topk_margin(int64_t N, int32_t E, int32_t k, const double* logits64,
                        double* margin) {
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)E);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
      for (int32_t e = 0; e < E; ++e) s[e] = logits64[t * E + e];
      for (int32_t i = 1; i < E; ++i) { /* insertion sort, descending */
        double v = s[i];
        int32_t j = i - 1;
        while (j >= 0 && v > s[j]) {
          s[j + 1] = s[j];
          --j;
        }
        s[j + 1] = v;
      }
      double m = INFINITY;
      int32_t last = k < E - 1 ? k : E - 1;
      for (int32_t i = 0; i < last; ++i)
        if (s[i] - s[i + 1] < m) m = s[i] - s[i + 1];
      margin[t] = m;
    }
    free(s);
  }
}

/* ---------------------------------------------------------------- dispatch  [W] 1.3, 3.2 */

/* Literal sequential capacity check, slot-major then token order:
 *   for j in 0..k-1: for t in 0..N-1:
 *       e = idx[t,j]; pos[t,j] = count[e]++; dropped[t,j] = pos[t,j] >= C
 * load[e]    = number of records routed to e (before capacity)      ([W] 1.3)
 * offsets    = exclusive prefix sum of kept_e = min(load_e, C); offsets[E] = kept records
 * row_token[offsets[e] + pos] = t for every kept record (expert-contiguous order). */
/* One routing record (t, j): its position is the number of records routed to the same expert
 * before it in the visiting order; it is dropped when that position reaches C. */
static void visit_record(int64_t t, int32_t j, int32_t k, int64_t C, const int32_t* idx,
                         int64_t* count, int32_t* pos, uint8_t* dropped) {
  int32_t e = idx[t * k + j];
  int64_t p = count[e]++;
  pos[t * k + j] = (int32_t)p;
  dropped[t * k + j] = (uint8_t)(p >= C);
}

/* order 0 (slot-major): all rank-0 records in token order, then rank 1, ...
 * order 1 (token-major, the walkthrough's loop [W] 3.2): token by token, its slots in rank
 * order. */
void oracle_dispatch_order(int64_t N, int32_t k, int32_t E, int64_t C, int32_t order,
                           const int32_t* idx, int32_t* load, int32_t* offsets, int32_t* pos,
                           uint8_t* dropped, int32_t* row_token) {
  int64_t* count = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  if (order == 1) {
    for (int64_t t = 0; t < N; ++t)
      for (int32_t j = 0; j < k; ++j) visit_record(t, j, k, C, idx, count, pos, dropped);
  } else {
    for (int32_t j = 0; j < k; ++j)
      for (int64_t t = 0; t < N; ++t) visit_record(t, j, k, C, idx, count, pos, dropped);
  }
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) {
    load[e] = (int32_t)count[e];
    int64_t kept = count[e] < C ? count[e] : C;
    offsets[e + 1] = offsets[e] + (int32_t)kept;
  }
  if (row_token)
    for (int64_t t = 0; t < N; ++t)
      for (int32_t j = 0; j < k; ++j)
        if (!dropped[t * k + j]) row_token[offsets[idx[t * k + j]] + pos[t * k + j]] = (int32_t)t;
  free(count);
}

void oracle_dispatch(int64_t N, int32_t k, int32_t E, int64_t C, const int32_t* idx,
                     int32_t* load, int32_t* offsets, int32_t* pos, uint8_t* dropped,
                     int32_t* row_token) {
  oracle_dispatch_order(N, k, E, C, 0, idx, load, offsets, pos, dropped, row_token);
}

/* ---------------------------------------------------------------- expert FFN  [L12] 12.1 */

static double activation(double a, int32_t act) {
  switch (act) {
    case OR_SILU: /* SiLU(a) = a * sigmoid(a)  ([G5] 5.3.5.1) */
      return a / (1.0 + exp(-a));
    case OR_GELU_ERF: /* GELU(a) = a * Phi(a), Phi the standard normal CDF ([G5] 5.3.5) */
      return 0.5 * a * (1.0 + erf(a / sqrt(2.0)));
    case OR_GELU_TANH: /* tanh approximation ([G5] 5.3.5.1) */
      return 0.5 * a * (1.0 + tanh(sqrt(2.0 / M_PI) * (a + 0.044715 * a * a * a)));
    default:
      return NAN;
  }
}

/* Where an expert weight matrix comes from: plain fp32/bf16 values (W, dtype), or 8-bit
 * weights with one scale per expert and output column (Q, S), dequantized as q * s before the
 * matmul ([G5] 5.3.3, "weight = weight * scales"; the scales broadcast over the reduction
 * dimension, the reading that makes the 8-bit copy smaller than the bf16 one). */
typedef struct {
  const void* W;
  int32_t dtype;
  const int8_t* Q;
  const float* S;
} wsrc;

/* Row `row` of expert e's [rows, n] matrix, widened (or dequantized, exactly) to double. */
static void weight_row(const wsrc* w, int64_t e, int64_t rows, int64_t row, int64_t n,
                       double* out) {
  const int64_t first = (e * rows + row) * n;
  if (w->Q) {
    const int8_t* q = w->Q + first;
    const float* sc = w->S + e * n;
    for (int64_t i = 0; i < n; ++i) out[i] = (double)q[i] * (double)sc[i];
  } else {
    widen(w->W, w->dtype, first, n, out);
  }
}

/* Gated expert of record r (token t = rec_token[r], expert e = rec_expert[r]):
 *   a = x W1_e, b = x W2_e  (sum over d ascending),  h = act(a) (.) b,
 *   y = h W3_e              (sum over f ascending).
 * W1 (activated branch, Grok "linear"), W2 (linear branch, Grok "linear_v"): [E,D,F];
 * W3 (Grok "linear_1"): [E,F,D]. Y: [n_rec, D] doubles. */
static void expert_ffn_core(int64_t n_rec, const int32_t* rec_token, const int32_t* rec_expert,
                            int64_t D, int64_t F, const void* X, int32_t x_dtype,
                            const wsrc* W1, const wsrc* W2, const wsrc* W3, int32_t act,
                            double* Y) {
#pragma omp parallel
  {
    double* x = (double*)malloc(sizeof(double) * (size_t)D);
    double* a = (double*)malloc(sizeof(double) * (size_t)F);
    double* b = (double*)malloc(sizeof(double) * (size_t)F);
    double* w = (double*)malloc(sizeof(double) * (size_t)(F > D ? F : D));
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rec; ++r) {
      const int64_t t = rec_token[r], e = rec_expert[r];
      widen(X, x_dtype, t * D, D, x);
      for (int64_t f = 0; f < F; ++f) a[f] = b[f] = 0.0;
      for (int64_t d = 0; d < D; ++d) {
        weight_row(W1, e, D, d, F, w);
        for (int64_t f = 0; f < F; ++f) a[f] += x[d] * w[f];
        weight_row(W2, e, D, d, F, w);
        for (int64_t f = 0; f < F; ++f) b[f] += x[d] * w[f];
      }
      for (int64_t f = 0; f < F; ++f) a[f] = activation(a[f], act) * b[f]; /* h */
      double* y = Y + r * D;
      for (int64_t d = 0; d < D; ++d) y[d] = 0.0;
      for (int64_t f = 0; f < F; ++f) {
        weight_row(W3, e, F, f, D, w);
        for (int64_t d = 0; d < D; ++d) y[d] += a[f] * w[d];
      }
    }
    free(x);
    free(a);
    free(b);
    free(w);
  }
}

void oracle_expert_ffn(int64_t n_rec, const int32_t* rec_token, const int32_t* rec_expert,
                       int64_t D, int64_t F, const void* X, const void* W1, const void* W2,
                       const void* W3, int32_t dtype, int32_t act, double* Y) {
  const wsrc w1 = {W1, dtype, NULL, NULL}, w2 = {W2, dtype, NULL, NULL}, w3 = {W3, dtype, NULL, NULL};
  expert_ffn_core(n_rec, rec_token, rec_expert, D, F, X, dtype, &w1, &w2, &w3, act, Y);
}

/* The same expert with 8-bit weights: W1q, W2q [E,D,F] and W3q [E,F,D] int8, S1, S2 [E,F] and
 * S3 [E,D] fp32; X is bf16 (dtype 1) or fp32 (dtype 0). */
void oracle_expert_ffn_w8(int64_t n_rec, const int32_t* rec_token, const int32_t* rec_expert,
                          int64_t D, int64_t F, const void* X, int32_t x_dtype,
                          const int8_t* W1q, const float* S1, const int8_t* W2q, const float* S2,
                          const int8_t* W3q, const float* S3, int32_t act, double* Y) {
  const wsrc w1 = {NULL, 0, W1q, S1}, w2 = {NULL, 0, W2q, S2}, w3 = {NULL, 0, W3q, S3};
  expert_ffn_core(n_rec, rec_token, rec_expert, D, F, X, x_dtype, &w1, &w2, &w3, act, Y);
}

/* ---------------------------------------------------------------- combine  [G5] 5.3.5 */

/* out[t] = sum_{j=0}^{k-1} [not dropped(t,j)] * gate[t,j] * y(t,j)   (j ascending; a token
 * accumulates its k contributions, [L12] 12.2; a dropped slot adds nothing, [GS] 2.2).
 * Yrec holds one row per record in record order (t*k + j). */
/* out[t] = sum over kept slots j of g'[t,j] * Y[t,j]. policy 0: g' = g. policy 1 ([GS] 2.2
 * case A): when a token has both dropped and kept slots, g'[t,j] = g[t,j] / (sum of the kept
 * slots' gates), so that the kept gates sum to 1 ((w1, w2) -> (1, 0) for top-2). */
void oracle_combine_policy(int64_t N, int32_t k, int64_t D, const double* gate,
                           const uint8_t* dropped, int32_t policy, const double* Yrec,
                           double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < N; ++t) {
    double* o = out + t * D;
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    double kept_sum = 0.0;
    int32_t kept = 0;
    for (int32_t j = 0; j < k; ++j)
      if (!(dropped && dropped[t * k + j])) {
        kept_sum += gate[t * k + j];
        ++kept;
      }
    const int reweight = policy == 1 && kept > 0 && kept < k;
    for (int32_t j = 0; j < k; ++j) {
      const int64_t r = t * k + j;
      if (dropped && dropped[r]) continue;
      const double g = reweight ? gate[r] / kept_sum : gate[r];
      const double* y = Yrec + r * D;
      for (int64_t d = 0; d < D; ++d) o[d] += g * y[d];
    }
  }
}

void oracle_combine(int64_t N, int32_t k, int64_t D, const double* gate,
                    const uint8_t* dropped, const double* Yrec, double* out) {
  oracle_combine_policy(N, k, D, gate, dropped, 0, Yrec, out);
}

/* ---------------------------------------------------------------- diagnostics  [W] 2, 3.3 */

/* L_balance = E * sum_i f_i * P_i with f_i = load_i / denom, P_i = colsum_i / N.
 * denom = N*k (the reading under which perfectly uniform routing gives exactly 1 for any k)
 * when nk_denominator != 0, else N (the walkthrough's code, which gives k at uniform). */
double oracle_balance_loss(int64_t N, int32_t k, int32_t E, const int32_t* load,
                           const double* prob_colsum, int32_t nk_denominator) {
  const double denom = nk_denominator ? (double)N * (double)k : (double)N;
  double s = 0.0;
  for (int32_t i = 0; i < E; ++i) s += ((double)load[i] / denom) * (prob_colsum[i] / (double)N);
  return (double)E * s;
}

/* Drop rate = N_drop / (N*K), over routing slots ([W] 3.3). */
double oracle_drop_rate(int64_t N, int32_t k, const uint8_t* dropped) {
  if (N * k == 0) return 0.0;
  int64_t n = 0;
  for (int64_t r = 0; r < N * k; ++r) n += dropped[r] ? 1 : 0;
  return (double)n / ((double)N * (double)k);
}

/* ---------------------------------------------------------------- whole layer */

/* The full forward in the pages' order: logits -> softmax -> top-k (+renorm) -> load ->
 * capacity (with min_capacity) -> dispatch in the given order -> gated expert FFN per kept
 * record -> gate-weighted combine under the drop policy. out [N,D] doubles (before any
 * rounding to the output dtype). Every other output pointer is optional. Returns 0, or -1 on
 * a non-finite logit. */
static int forward_core(int64_t N, int64_t D, int64_t F, int32_t E, int32_t k, double cf,
                        int64_t min_capacity, int32_t order, int32_t drop_policy,
                        int32_t renorm, int32_t act, int32_t dtype, const void* X,
                        const float* W_r, const float* bias, const wsrc* W1, const wsrc* W2,
                        const wsrc* W3, double* out, float* logits32_out, int32_t* idx_out,
                        double* gate_out, int32_t* load_out, int32_t* offsets_out,
                        int32_t* pos_out, uint8_t* dropped_out, double* prob_colsum_out) {
  const int64_t R = N * k;
  float* l32 = logits32_out ? logits32_out : (float*)malloc(sizeof(float) * (size_t)(N * E + 1));
  int32_t* idx = idx_out ? idx_out : (int32_t*)malloc(sizeof(int32_t) * (size_t)(R + 1));
  double* gate = gate_out ? gate_out : (double*)malloc(sizeof(double) * (size_t)(R + 1));
  int32_t* load = load_out ? load_out : (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  int32_t* offs = offsets_out ? offsets_out : (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
  int32_t* pos = pos_out ? pos_out : (int32_t*)malloc(sizeof(int32_t) * (size_t)(R + 1));
  uint8_t* drp = dropped_out ? dropped_out : (uint8_t*)malloc((size_t)(R + 1));
  int rc = 0;

  oracle_router_logits(N, D, E, X, dtype, W_r, bias, NULL, l32);
  if (oracle_route(N, E, k, renorm, l32, idx, gate, NULL, prob_colsum_out) != 0) {
    rc = -1;
  } else {
    const int64_t C = oracle_capacity_min(N, k, E, cf, min_capacity);
    oracle_dispatch_order(N, k, E, C, order, idx, load, offs, pos, drp, NULL);
    /* expert outputs of the kept records, one row per record (dropped rows stay zero) */
    int64_t nk = 0;
    for (int64_t r = 0; r < R; ++r) nk += drp[r] ? 0 : 1;
    int32_t* rt = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nk + 1));
    int32_t* re = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nk + 1));
    int64_t q = 0;
    for (int64_t r = 0; r < R; ++r) {
      if (drp[r]) continue;
      rt[q] = (int32_t)(r / k);
      re[q] = idx[r];
      ++q;
    }
    double* Yk = (double*)malloc(sizeof(double) * (size_t)(nk * D + 1));
    expert_ffn_core(nk, rt, re, D, F, X, dtype, W1, W2, W3, act, Yk);
    double* Yrec = (double*)calloc((size_t)(R * D + 1), sizeof(double));
    q = 0;
    for (int64_t r = 0; r < R; ++r) {
      if (drp[r]) continue;
      memcpy(Yrec + r * D, Yk + q * D, sizeof(double) * (size_t)D);
      ++q;
    }
    oracle_combine_policy(N, k, D, gate, drp, drop_policy, Yrec, out);
    free(rt);
    free(re);
    free(Yk);
    free(Yrec);
  }
  if (!logits32_out) free(l32);
  if (!idx_out) free(idx);
  if (!gate_out) free(gate);
  if (!load_out) free(load);
  if (!offsets_out) free(offs);
  if (!pos_out) free(pos);
  if (!dropped_out) free(drp);
  return rc;
}

int oracle_forward(int64_t N, int64_t D, int64_t F, int32_t E, int32_t k, double cf,
                   int64_t min_capacity, int32_t order, int32_t drop_policy,
                   int32_t renorm, int32_t act, int32_t dtype, const void* X, const float* W_r,
                   const float* bias, const void* W1, const void* W2, const void* W3,
                   double* out, float* logits32_out, int32_t* idx_out, double* gate_out,
                   int32_t* load_out, int32_t* offsets_out, int32_t* pos_out,
                   uint8_t* dropped_out, double* prob_colsum_out) {
  const wsrc w1 = {W1, dtype, NULL, NULL}, w2 = {W2, dtype, NULL, NULL}, w3 = {W3, dtype, NULL, NULL};
  return forward_core(N, D, F, E, k, cf, min_capacity, order, drop_policy, renorm, act, dtype, X,
                      W_r, bias, &w1, &w2, &w3, out, logits32_out, idx_out, gate_out, load_out,
                      offsets_out, pos_out, dropped_out, prob_colsum_out);
}

/* The forward with 8-bit expert weights (see oracle_expert_ffn_w8). */
int oracle_forward_w8(int64_t N, int64_t D, int64_t F, int32_t E, int32_t k, double cf,
                      int64_t min_capacity, int32_t order, int32_t drop_policy,
                      int32_t renorm, int32_t act, int32_t dtype, const void* X,
                      const float* W_r, const float* bias, const int8_t* W1q, const float* S1,
                      const int8_t* W2q, const float* S2, const int8_t* W3q, const float* S3,
                      double* out, float* logits32_out, int32_t* idx_out, double* gate_out,
                      int32_t* load_out, int32_t* offsets_out, int32_t* pos_out,
                      uint8_t* dropped_out, double* prob_colsum_out) {
  const wsrc w1 = {NULL, 0, W1q, S1}, w2 = {NULL, 0, W2q, S2}, w3 = {NULL, 0, W3q, S3};
  return forward_core(N, D, F, E, k, cf, min_capacity, order, drop_policy, renorm, act, dtype, X,
                      W_r, bias, &w1, &w2, &w3, out, logits32_out, idx_out, gate_out, load_out,
                      offsets_out, pos_out, dropped_out, prob_colsum_out);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
