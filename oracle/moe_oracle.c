/*
 * moe_oracle.c -- plain, slow CPU oracle for one fine-grained sparse-MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this
 * file.  Only the test suite, the smoke check and the CPU-baseline leg of the benchmark
 * use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition, no blocking, no fusion, no reordering):
 *
 *   Sources (page title, then the passage):
 *   [P2 2.2]   "Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active Parameters",
 *              section 2.2 (sparse-MoE backbone): each MoE layer has 288 routed experts and
 *              one shared expert; every token activates its top-k = 8 experts.
 *   [P2 2.2.2] same page, section 2.2.2 (expert-parallel load balancing): loss-free load
 *              balancing; S_t is the top-K expert set of token t, s_{t,e} = 1[e in S_t],
 *              p_{t,e} the routing probability.
 *   [P3 MoE]   "Step 3.5 Flash 技术论文深度解读：196B MoE 如何做到 11B 激活打 37B",
 *              architecture item 1 (fine-grained MoE, 288 experts top-8): parameter table
 *              (288 routed + 1 shared, top-8, routed-expert hidden size 1280) and the note
 *              under it: balancing by bias adjustment, not an auxiliary loss.
 *   [P3 stab]  same page, training stability, "local activation explosion", root cause 3:
 *              the experts are SwiGLU with gate and up projection branches.
 *   [P2 4.1.2] first page above, section 4.1.2 (expert collapse): aggregation of the
 *              routed experts needs an explicit scale (value not given: routed_scale).
 *   [P2 3.2.4] first page above, section 3.2.4 (GPU kernel optimisation): fused MoE
 *              gather/scatter with grouped GEMM -- the expert-sorted permutation below.
 *
 *   Readings where the pages are silent (each is listed in the design notes):
 *   - router score: logits l[t,e] = x_t . W_r[e]; the bias b_e is added for SELECTION only
 *     (s = fl32(l + b)); the gates are a softmax over the k selected UNBIASED logits,
 *     i.e. the full softmax renormalised over S_t.
 *   - ties in top-k: larger fp32 score first; equal scores -> lower expert id first;
 *     -0.0 == +0.0 (float compare); NaN ranks below every number (NaNs by id).
 *   - the slots of a token are ordered by that same ranking (descending biased score).
 *   - the shared expert is always on with weight 1; out = shared + routed_scale*sum g*y.
 *   - expert-sorted order: group e holds its (t, j) pairs in ascending t.
 *
 * Arithmetic: inputs are decoded exactly to double (bf16 -> float is exact), every dot
 * product is accumulated in double; logits are rounded ONCE to fp32 (they are an fp32
 * output of the router); s = l + b is an fp32 add (the selection is decided in the same
 * precision as the GPU's); gates are computed in double and rounded once to fp32; the
 * expert FFNs and the combine stay in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1

/* exact bf16 (stored as its 16 high bits) -> double */
static double orc_bf16_to_double(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* element i of a row-major matrix stored either as fp32 or as bf16 bits */
static double orc_elem(const void *base, int dtype, size_t i) {
  if (dtype == ORC_BF16) return orc_bf16_to_double(((const uint16_t *)base)[i]);
  return (double)((const float *)base)[i];
}

/* silu(z) = z * sigmoid(z) = z / (1 + exp(-z))   [P3 stab: SwiGLU experts] */
static double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* ranking used for top-k: returns 1 if (sa, ea) ranks strictly before (sb, eb) */
static int orc_ranks_before(float sa, int ea, float sb, int eb) {
  int na = isnan(sa), nb = isnan(sb);
  if (na != nb) return nb;          /* a number ranks before a NaN */
  if (!na && sa != sb) return sa > sb;
  return ea < eb;                   /* equal scores (or both NaN): lower id first */
}

/* ------------------------------------------------------------------------------------ */
/* Router logits: l[t,e] = sum_i x[t,i] * W_r[e,i], double accumulation, one fp32 round. */
/* [P2 2.2.2]: p_{t,e} is a distribution over experts computed from these logits.        */
void oracle_router_logits(const void *x, const void *w_r, int dtype, int T, int d, int E,
                          float *logits) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i)
        acc += orc_elem(x, dtype, (size_t)t * d + i) * orc_elem(w_r, dtype, (size_t)e * d + i);
      logits[(size_t)t * E + e] = (float)acc;
    }
  }
}

/* ------------------------------------------------------------------------------------ */
/* Gates of one token for a given selection sel[0..k): softmax over the k selected         */
/* UNBIASED logits, max-shifted, in double, each rounded once to fp32.  [P2 2.2.2] p_{t,e} */
/* renormalised over S_t; [P3 MoE] the bias takes no part in the gates.                    */
static void orc_gates_of_selection(const float *l, const int *sel, int k, float *gates) {
  double m = -INFINITY;
  for (int j = 0; j < k; ++j) {
    double v = (double)l[sel[j]];
    if (v > m) m = v;
  }
  double z = 0.0;
  for (int j = 0; j < k; ++j) z += exp((double)l[sel[j]] - m);
  for (int j = 0; j < k; ++j) gates[j] = (float)(exp((double)l[sel[j]] - m) / z);
}

/* ------------------------------------------------------------------------------------ */
/* Selection and gates for one token.                                                     */
/* [P3 MoE] bias for selection only; [P2 2.2.2] S_t = top-K set; gates renormalised.       */
static void orc_route_token(const float *l, const float *bias, int E, int k, int *idx,
                            float *gates) {
  /* s = fl32(l + b): the fp32 add decides the selection */
  float *s = (float *)malloc(sizeof(float) * (size_t)E);
  int *order = (int *)malloc(sizeof(int) * (size_t)E);
  for (int e = 0; e < E; ++e) {
    s[e] = l[e] + (bias ? bias[e] : 0.0f);
    order[e] = e;
  }
  /* full insertion sort of all E experts by the ranking, then take the first k */
  for (int a = 1; a < E; ++a) {
    int cur = order[a];
    int b = a - 1;
    while (b >= 0 && orc_ranks_before(s[cur], cur, s[order[b]], order[b])) {
      order[b + 1] = order[b];
      --b;
    }
    order[b + 1] = cur;
  }
  for (int j = 0; j < k; ++j) idx[j] = order[j];
  orc_gates_of_selection(l, idx, k, gates);
  free(s);
  free(order);
}

void oracle_route(const float *logits, const float *bias, int T, int E, int k, int *idx,
                  float *gates) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t)
    orc_route_token(logits + (size_t)t * E, bias, E, k, idx + (size_t)t * k,
                    gates + (size_t)t * k);
}

/* Gates for a selection made elsewhere (e.g. the GPU's idx), from these logits: the same */
/* softmax as oracle_route applies to its own selection.                                   */
void oracle_gates(const float *logits, const int *idx, int T, int E, int k, float *gates) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t)
    orc_gates_of_selection(logits + (size_t)t * E, idx + (size_t)t * k, k,
                           gates + (size_t)t * k);
}

/* ------------------------------------------------------------------------------------ */
/* Expert-sorted permutation by counting sort.  [P2 3.2.4] gather/scatter grouping.        */
/* counts[e] = |{t : e in S_t}|; offsets = exclusive prefix sum (offsets[E] = T*k);        */
/* perm[offsets[e] + r] = t*k + j for the r-th token (ascending t) that chose e in slot j; */
/* slot_row[t*k + j] = that position.                                                      */
void oracle_permute(const int *idx, int T, int E, int k, int *counts, int *offsets,
                    int *perm, int *slot_row) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int q = 0; q < T * k; ++q) counts[idx[q]] += 1;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int *fill = (int *)calloc((size_t)E, sizeof(int));
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      int q = t * k + j;
      int e = idx[q];
      int p = offsets[e] + fill[e];
      fill[e] += 1;
      perm[p] = q;
      slot_row[q] = p;
    }
  }
  free(fill);
}

/* ------------------------------------------------------------------------------------ */
/* One SwiGLU expert on one token, double:  [P3 stab]                                     */
/*   g_r = x . W_g[r],  u_r = x . W_u[r],  h_r = silu(g_r) * u_r,  y_c = sum_r h_r W_d[c,r] */
/* W_g, W_u are [f, d] row-major (d contiguous); W_d is [d, f] row-major (f contiguous).    */
void oracle_expert_ffn(const void *x_row, const void *wg, const void *wu, const void *wd,
                       int dtype, int d, int f, double *y) {
  double *h = (double *)malloc(sizeof(double) * (size_t)f);
  for (int r = 0; r < f; ++r) {
    double g = 0.0, u = 0.0;
    for (int i = 0; i < d; ++i) {
      double xi = orc_elem(x_row, dtype, (size_t)i);
      g += xi * orc_elem(wg, dtype, (size_t)r * d + i);
      u += xi * orc_elem(wu, dtype, (size_t)r * d + i);
    }
    h[r] = orc_silu(g) * u;
  }
  for (int c = 0; c < d; ++c) {
    double acc = 0.0;
    for (int r = 0; r < f; ++r) acc += h[r] * orc_elem(wd, dtype, (size_t)c * f + r);
    y[c] = acc;
  }
  free(h);
}

/* ------------------------------------------------------------------------------------ */
/* The whole layer for a list of tokens (all of them, or a sample).                        */
/*   out[i,:] = shared(x_t) + routed_scale * sum_j g[t,j] * expert_{idx[t,j]}(x_t)          */
/* [P2 2.2] shared expert always on; [P2 4.1.2] explicit routed scale.                     */
/* Expert e's weights start at element e*f*d of w_gate / w_up and e*d*f of w_down; the     */
/* shared expert (if n_shared == 1) is expert index E in the same arrays.                  */
/* If `logits_in` is non-null the router logits of the listed tokens are taken from it     */
/* ([n_list, E]); otherwise they are computed by oracle_router_logits' definition.         */
/* idx_out / gates_out / logits_out ([n_list, k] / [n_list, k] / [n_list, E]) may be null.  */
void oracle_moe_forward(const void *x, const void *w_r, const float *bias, const void *w_gate,
                        const void *w_up, const void *w_down, int dtype, int d, int E, int k,
                        int f, int n_shared, double routed_scale, const int *tokens, int n_list,
                        const float *logits_in, double *out, int *idx_out, float *gates_out,
                        float *logits_out) {
  const size_t esz = (dtype == ORC_BF16) ? 2 : 4;
  const size_t wsz = (size_t)f * (size_t)d; /* elements per expert matrix */
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n_list; ++i) {
    const int t = tokens[i];
    const char *xr = (const char *)x + (size_t)t * d * esz;
    float *l = (float *)malloc(sizeof(float) * (size_t)E);
    if (logits_in) {
      memcpy(l, logits_in + (size_t)i * E, sizeof(float) * (size_t)E);
    } else {
      for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
          acc += orc_elem(xr, dtype, (size_t)c) * orc_elem(w_r, dtype, (size_t)e * d + c);
        l[e] = (float)acc;
      }
    }
    int *idx = (int *)malloc(sizeof(int) * (size_t)k);
    float *g = (float *)malloc(sizeof(float) * (size_t)k);
    orc_route_token(l, bias, E, k, idx, g);
    double *o = out + (size_t)i * d;
    double *y = (double *)malloc(sizeof(double) * (size_t)d);
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int j = 0; j < k; ++j) {
      const int e = idx[j];
      oracle_expert_ffn(xr, (const char *)w_gate + (size_t)e * wsz * esz,
                        (const char *)w_up + (size_t)e * wsz * esz,
                        (const char *)w_down + (size_t)e * wsz * esz, dtype, d, f, y);
      for (int c = 0; c < d; ++c) o[c] += routed_scale * (double)g[j] * y[c];
    }
    if (n_shared) {
      oracle_expert_ffn(xr, (const char *)w_gate + (size_t)E * wsz * esz,
                        (const char *)w_up + (size_t)E * wsz * esz,
                        (const char *)w_down + (size_t)E * wsz * esz, dtype, d, f, y);
      for (int c = 0; c < d; ++c) o[c] += y[c];
    }
    if (idx_out) memcpy(idx_out + (size_t)i * k, idx, sizeof(int) * (size_t)k);
    if (gates_out) memcpy(gates_out + (size_t)i * k, g, sizeof(float) * (size_t)k);
    if (logits_out) memcpy(logits_out + (size_t)i * E, l, sizeof(float) * (size_t)E);
    free(y);
    free(g);
    free(idx);
    free(l);
  }
}

/* number of OpenMP threads the oracle runs with (1 when built without OpenMP); the setter
 * overrides OMP_NUM_THREADS (a launcher may have set it to 1 for every process) */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
void oracle_set_num_threads(int n) {
  if (n > 0) omp_set_num_threads(n);
}
#else
int oracle_num_threads(void) { return 1; }
void oracle_set_num_threads(int n) { (void)n; }
#endif

/* ------------------------------------------------------------------------------------ */
/* Router statistics, [P2 2.2.2] (EP-group balance loss) and [P2 5.2.3] (routing          */
/* confidence, called Sigma_k there):                                                      */
/*   p[t,e]   = softmax over all E unbiased logits of token t (the routing probability)    */
/*   p_e      = (1/T) sum_t p[t,e]            f_e = (1/(T k)) sum_t s[t,e]                 */
/*   p_g, f_g = sums over the experts of group g (G contiguous groups of E/G experts)      */
/*   L_EP     = G sum_g f_g p_g                                                            */
/*   conf     = (1/T) sum_t sum_{e in S_t} p[t,e]                                          */
/* Everything in double, rounded once to fp32 at the end.                                  */
void oracle_router_stats(const float *logits, const int *idx, int T, int E, int k, int G,
                         float *p_mean, float *f_sel, float *l_ep, float *conf) {
  double *pm = (double *)calloc((size_t)E, sizeof(double));
  double *fs = (double *)calloc((size_t)E, sizeof(double));
  double *p = (double *)malloc(sizeof(double) * (size_t)E);
  double cf = 0.0;
  for (int t = 0; t < T; ++t) {
    const float *l = logits + (size_t)t * E;
    double m = -INFINITY;
    for (int e = 0; e < E; ++e)
      if ((double)l[e] > m) m = (double)l[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = exp((double)l[e] - m);
      z += p[e];
    }
    for (int e = 0; e < E; ++e) {
      p[e] /= z;
      pm[e] += p[e];
    }
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      fs[e] += 1.0;
      cf += p[e];
    }
  }
  const int per = E / G;
  double loss = 0.0;
  for (int g = 0; g < G; ++g) {
    double pg = 0.0, fg = 0.0;
    for (int e = g * per; e < (g + 1) * per; ++e) {
      pg += pm[e] / T;
      fg += fs[e] / ((double)T * k);
    }
    loss += fg * pg;
  }
  for (int e = 0; e < E; ++e) {
    p_mean[e] = (float)(pm[e] / T);
    f_sel[e] = (float)(fs[e] / ((double)T * k));
  }
  *l_ep = (float)(G * loss);
  *conf = (float)(cf / T);
  free(p);
  free(fs);
  free(pm);
}

/* Loss-free balancing bias step ([P3 MoE] note: balance by adjusting a per-expert bias, no
 * auxiliary loss).  The pages give no update rule; this library's reading is the plain sign
 * step toward the mean load:  b_e <- b_e + gamma * sign(T k / E - counts[e])  (sign(0) = 0),
 * computed in fp32 like the bias itself.  PARITY UNPINNED against the pages (no rule there);
 * pinned only by the closed forms in the tests. */
void oracle_bias_update(const int *counts, int E, int Tk, float gamma, float *bias) {
  const float mean = (float)Tk / (float)E;
  for (int e = 0; e < E; ++e) {
    const float gap = mean - (float)counts[e];
    const float s = (gap > 0.f) ? 1.f : ((gap < 0.f) ? -1.f : 0.f);
    bias[e] = bias[e] + gamma * s;
  }
}

/* ------------------------------------------------------------------------------------ */
/* Expert health signals.  [P2 4.1.2]: expert collapse shows as vanishing expert          */
/* activations and stalling parameter norms, so per-expert activation norms and parameter */
/* norms are to be monitored; [P3], training stability, "expert collapse": the per-expert  */
/* activation RMS norm and the min-to-median ratio of the parameter Frobenius norms.       */
/* Readings: the activation is the SwiGLU output h = silu(x W_g^T) * (x W_u^T) of expert g */
/* over the tokens routed to it (all tokens for a shared expert), RMS over tokens and the f */
/* features (0 for an expert no token chose); the parameter norm of expert g is the        */
/* Frobenius norm of its three matrices together.  Double throughout.                      */
void oracle_expert_act_rms(const void *x, const void *w_gate, const void *w_up, int dtype,
                           int T, int d, int f, int E, int n_shared, const int *idx, int k,
                           double *rms) {
  const int G = E + n_shared;
  for (int g = 0; g < G; ++g) {
    double ss = 0.0;
    long long rows = 0;
    for (int t = 0; t < T; ++t) {
      int chosen = g >= E;
      for (int j = 0; j < k && !chosen; ++j) chosen = idx[(size_t)t * k + j] == g;
      if (!chosen) continue;
      ++rows;
      for (int n = 0; n < f; ++n) {
        double a = 0.0, b = 0.0;
        for (int i = 0; i < d; ++i) {
          const double xv = orc_elem(x, dtype, (size_t)t * d + i);
          a += xv * orc_elem(w_gate, dtype, ((size_t)g * f + n) * d + i);
          b += xv * orc_elem(w_up, dtype, ((size_t)g * f + n) * d + i);
        }
        const double h = orc_silu(a) * b;
        ss += h * h;
      }
    }
    rms[g] = rows ? sqrt(ss / ((double)rows * f)) : 0.0;
  }
}

void oracle_expert_param_norms(const void *w_gate, const void *w_up, const void *w_down,
                               int dtype, int d, int f, int G, double *norm) {
  const size_t per = (size_t)f * d;
  for (int g = 0; g < G; ++g) {
    double ss = 0.0;
    for (size_t i = 0; i < per; ++i) {
      const double a = orc_elem(w_gate, dtype, (size_t)g * per + i);
      const double b = orc_elem(w_up, dtype, (size_t)g * per + i);
      const double c = orc_elem(w_down, dtype, (size_t)g * per + i);
      ss += a * a + b * b + c * c;
    }
    norm[g] = sqrt(ss);
  }
}

/* ------------------------------------------------------------------------------------ */
/* Backward of the layer: the chain rule through oracle_moe_forward's definition, for a     */
/* given selection (idx) and gates -- the selection itself carries no gradient ([P3 MoE]:   */
/* the bias only selects).  Double throughout; tokens one after another (the weight         */
/* gradients accumulate over tokens).                                                      */
/*   for token t and each contribution (expert e, scale s = routed_scale * g_j, or 1 for   */
/*   the shared expert):                                                                    */
/*     a = W_g[e] x_t,  b = W_u[e] x_t,  h = silu(a) * b,  yhat = W_d[e] h                 */
/*     dy = s * dout_t;   dW_d[e] += dy h^T;   dh = W_d[e]^T dy                             */
/*     da = dh * b * silu'(a),  db = dh * silu(a),  silu'(a) = sig(a) (1 + a (1 - sig(a)))  */
/*     dW_g[e] += da x_t^T;  dW_u[e] += db x_t^T;  dx_t += W_g[e]^T da + W_u[e]^T db         */
/*     routed: dgate_j = routed_scale * (dout_t . yhat)                                     */
/*   router: the gates are the softmax of the selected unbiased logits, so                  */
/*     dl[e_j] = g_j (dgate_j - sum_i g_i dgate_i), 0 for unselected experts;               */
/*     dW_r[e] += dl[e] x_t;  dx_t += sum_e dl[e] W_r[e]                                    */
/* Outputs: dx [T,d], dw_router [E,d], dw_gate / dw_up [G,f,d], dw_down [G,d,f] (G = E +   */
/* n_shared), overwritten.                                                                 */
void oracle_moe_backward(const void *x, const void *dout, const void *w_r, const void *w_gate,
                         const void *w_up, const void *w_down, int dtype, int T, int d, int E,
                         int k, int f, int n_shared, double routed_scale, const int *idx,
                         const float *gates, double *dx, double *dw_router, double *dw_gate,
                         double *dw_up, double *dw_down) {
  const int G = E + n_shared;
  const size_t wsz = (size_t)f * (size_t)d;
  memset(dx, 0, sizeof(double) * (size_t)T * d);
  memset(dw_router, 0, sizeof(double) * (size_t)E * d);
  memset(dw_gate, 0, sizeof(double) * (size_t)G * wsz);
  memset(dw_up, 0, sizeof(double) * (size_t)G * wsz);
  memset(dw_down, 0, sizeof(double) * (size_t)G * wsz);
  double *xt = (double *)malloc(sizeof(double) * (size_t)d);
  double *ot = (double *)malloc(sizeof(double) * (size_t)d);
  double *a = (double *)malloc(sizeof(double) * (size_t)f);
  double *b = (double *)malloc(sizeof(double) * (size_t)f);
  double *h = (double *)malloc(sizeof(double) * (size_t)f);
  double *dh = (double *)malloc(sizeof(double) * (size_t)f);
  double *dy = (double *)malloc(sizeof(double) * (size_t)d);
  double *dgate = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  for (int t = 0; t < T; ++t) {
    for (int i = 0; i < d; ++i) {
      xt[i] = orc_elem(x, dtype, (size_t)t * d + i);
      ot[i] = orc_elem(dout, dtype, (size_t)t * d + i);
    }
    for (int c = 0; c < k + n_shared; ++c) {
      const int routed = c < k;
      const int e = routed ? idx[(size_t)t * k + c] : E;
      const double s = routed ? routed_scale * (double)gates[(size_t)t * k + c] : 1.0;
      for (int n = 0; n < f; ++n) {
        double av = 0.0, bv = 0.0;
        for (int i = 0; i < d; ++i) {
          av += xt[i] * orc_elem(w_gate, dtype, (size_t)e * wsz + (size_t)n * d + i);
          bv += xt[i] * orc_elem(w_up, dtype, (size_t)e * wsz + (size_t)n * d + i);
        }
        a[n] = av;
        b[n] = bv;
        h[n] = orc_silu(av) * bv;
      }
      double dot = 0.0;  /* dout_t . yhat */
      for (int i = 0; i < d; ++i) {
        double yh = 0.0;
        for (int n = 0; n < f; ++n)
          yh += orc_elem(w_down, dtype, (size_t)e * wsz + (size_t)i * f + n) * h[n];
        dot += ot[i] * yh;
        dy[i] = s * ot[i];
      }
      if (routed) dgate[c] = routed_scale * dot;
      for (int n = 0; n < f; ++n) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) {
          acc += orc_elem(w_down, dtype, (size_t)e * wsz + (size_t)i * f + n) * dy[i];
          dw_down[(size_t)e * wsz + (size_t)i * f + n] += dy[i] * h[n];
        }
        dh[n] = acc;
      }
      for (int n = 0; n < f; ++n) {
        const double sg = 1.0 / (1.0 + exp(-a[n]));
        const double da = dh[n] * b[n] * sg * (1.0 + a[n] * (1.0 - sg));
        const double db = dh[n] * a[n] * sg;
        for (int i = 0; i < d; ++i) {
          const size_t wi = (size_t)e * wsz + (size_t)n * d + i;
          dw_gate[wi] += da * xt[i];
          dw_up[wi] += db * xt[i];
          dx[(size_t)t * d + i] +=
              orc_elem(w_gate, dtype, wi) * da + orc_elem(w_up, dtype, wi) * db;
        }
      }
    }
    double sgd = 0.0;
    for (int j = 0; j < k; ++j) sgd += (double)gates[(size_t)t * k + j] * dgate[j];
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      const double dl = (double)gates[(size_t)t * k + j] * (dgate[j] - sgd);
      for (int i = 0; i < d; ++i) {
        dw_router[(size_t)e * d + i] += dl * xt[i];
        dx[(size_t)t * d + i] += dl * orc_elem(w_r, dtype, (size_t)e * d + i);
      }
    }
  }
  free(dgate);
  free(dy);
  free(dh);
  free(h);
  free(b);
  free(a);
  free(ot);
  free(xt);
}

/* ------------------------------------------------------------------------------------ */
/* Sampled backward for layer sizes whose full weight gradients do not fit in memory: the  */
/* same chain rule as oracle_moe_backward, restricted to                                    */
/*   dx of the tokens toks[0..n_tok)                        -> dx_s  [n_tok, d]             */
/*   dW_gate, dW_up, dW_down of the experts exps[0..n_exp)  -> dwg_s, dwu_s [n_exp, f, d],  */
/*                                                             dwd_s [n_exp, d, f]          */
/*   dW_router rows of the routed experts rexps[0..n_rexp)  -> dwr_s [n_rexp, d]            */
/* A contribution (token t, expert e) is evaluated when e is in exps or the token's dx or   */
/* router terms are needed (t in toks, or one of its routed experts in rexps: those need    */
/* dgate of all of its slots).  Tokens in increasing order, as in oracle_moe_backward.      */
static int orc_in(const int *list, int n, int v) {
  for (int i = 0; i < n; ++i)
    if (list[i] == v) return i;
  return -1;
}

void oracle_moe_backward_sampled(const void *x, const void *dout, const void *w_r,
                                 const void *w_gate, const void *w_up, const void *w_down,
                                 int dtype, int T, int d, int E, int k, int f, int n_shared,
                                 double routed_scale, const int *idx, const float *gates,
                                 int n_tok, const int *toks, double *dx_s, int n_exp,
                                 const int *exps, double *dwg_s, double *dwu_s, double *dwd_s,
                                 int n_rexp, const int *rexps, double *dwr_s) {
  const size_t wsz = (size_t)f * (size_t)d;
  memset(dx_s, 0, sizeof(double) * (size_t)n_tok * d);
  memset(dwg_s, 0, sizeof(double) * (size_t)n_exp * wsz);
  memset(dwu_s, 0, sizeof(double) * (size_t)n_exp * wsz);
  memset(dwd_s, 0, sizeof(double) * (size_t)n_exp * wsz);
  memset(dwr_s, 0, sizeof(double) * (size_t)n_rexp * d);
  double *xt = (double *)malloc(sizeof(double) * (size_t)d);
  double *ot = (double *)malloc(sizeof(double) * (size_t)d);
  double *a = (double *)malloc(sizeof(double) * (size_t)f);
  double *b = (double *)malloc(sizeof(double) * (size_t)f);
  double *h = (double *)malloc(sizeof(double) * (size_t)f);
  double *dh = (double *)malloc(sizeof(double) * (size_t)f);
  double *dy = (double *)malloc(sizeof(double) * (size_t)d);
  double *dgate = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  for (int t = 0; t < T; ++t) {
    const int ti = orc_in(toks, n_tok, t);
    int whole = ti >= 0;  /* every contribution of the token is needed */
    for (int j = 0; j < k; ++j)
      if (orc_in(rexps, n_rexp, idx[(size_t)t * k + j]) >= 0) whole = 1;
    int any = whole;
    for (int c = 0; c < k + n_shared && !any; ++c) {
      const int e = c < k ? idx[(size_t)t * k + c] : E;
      if (orc_in(exps, n_exp, e) >= 0) any = 1;
    }
    if (!any) continue;
    for (int i = 0; i < d; ++i) {
      xt[i] = orc_elem(x, dtype, (size_t)t * d + i);
      ot[i] = orc_elem(dout, dtype, (size_t)t * d + i);
    }
    for (int c = 0; c < k + n_shared; ++c) {
      const int routed = c < k;
      const int e = routed ? idx[(size_t)t * k + c] : E;
      const int ei = orc_in(exps, n_exp, e);
      if (!whole && ei < 0) continue;
      const double s = routed ? routed_scale * (double)gates[(size_t)t * k + c] : 1.0;
      for (int n = 0; n < f; ++n) {
        double av = 0.0, bv = 0.0;
        for (int i = 0; i < d; ++i) {
          av += xt[i] * orc_elem(w_gate, dtype, (size_t)e * wsz + (size_t)n * d + i);
          bv += xt[i] * orc_elem(w_up, dtype, (size_t)e * wsz + (size_t)n * d + i);
        }
        a[n] = av;
        b[n] = bv;
        h[n] = orc_silu(av) * bv;
      }
      double dot = 0.0;  /* dout_t . yhat */
      for (int i = 0; i < d; ++i) {
        double yh = 0.0;
        for (int n = 0; n < f; ++n)
          yh += orc_elem(w_down, dtype, (size_t)e * wsz + (size_t)i * f + n) * h[n];
        dot += ot[i] * yh;
        dy[i] = s * ot[i];
      }
      if (routed) dgate[c] = routed_scale * dot;
      for (int n = 0; n < f; ++n) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) {
          acc += orc_elem(w_down, dtype, (size_t)e * wsz + (size_t)i * f + n) * dy[i];
          if (ei >= 0) dwd_s[(size_t)ei * wsz + (size_t)i * f + n] += dy[i] * h[n];
        }
        dh[n] = acc;
      }
      for (int n = 0; n < f; ++n) {
        const double sg = 1.0 / (1.0 + exp(-a[n]));
        const double da = dh[n] * b[n] * sg * (1.0 + a[n] * (1.0 - sg));
        const double db = dh[n] * a[n] * sg;
        for (int i = 0; i < d; ++i) {
          const size_t wi = (size_t)e * wsz + (size_t)n * d + i;
          if (ei >= 0) {
            dwg_s[(size_t)ei * wsz + (size_t)n * d + i] += da * xt[i];
            dwu_s[(size_t)ei * wsz + (size_t)n * d + i] += db * xt[i];
          }
          if (ti >= 0)
            dx_s[(size_t)ti * d + i] +=
                orc_elem(w_gate, dtype, wi) * da + orc_elem(w_up, dtype, wi) * db;
        }
      }
    }
    if (!whole) continue;
    double sgd = 0.0;
    for (int j = 0; j < k; ++j) sgd += (double)gates[(size_t)t * k + j] * dgate[j];
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      const double dl = (double)gates[(size_t)t * k + j] * (dgate[j] - sgd);
      const int ri = orc_in(rexps, n_rexp, e);
      for (int i = 0; i < d; ++i) {
        if (ri >= 0) dwr_s[(size_t)ri * d + i] += dl * xt[i];
        if (ti >= 0) dx_s[(size_t)ti * d + i] += dl * orc_elem(w_r, dtype, (size_t)e * d + i);
      }
    }
  }
  free(dgate);
  free(dy);
  free(dh);
  free(h);
  free(b);
  free(a);
  free(ot);
  free(xt);
}
