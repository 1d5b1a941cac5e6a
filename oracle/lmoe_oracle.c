/*
 * lmoe_oracle.c -- plain fp64 CPU oracle of the LatentMoE layer forward and
 * of its backward (the gradient for an output cotangent, after the forward).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is what the CUDA library is checked
 * against; it is never part of the product path.  Only tests/, the smoke
 * check in __graft_entry__.py and the CPU-baseline leg of bench.py may load
 * it.  It shares no code, header, table or helper with the CUDA library.
 *
 * Sources (web pages, cited by title and section):
 *   [Explained]  "LatentMoE: NVIDIA's Latent Mixture of Experts Explained
 *                Through Equations, Architecture, Code and..." (Towards AI):
 *                Figure 3 (router), Figure 8 (the latent layer with shapes),
 *                Figure 9 (the latent expert), the MoE and LatentMoE code
 *                modules, and the paragraph after Figure 1 (SwiGLU has a
 *                third matrix beside W1).
 *   [README]     "Latent-MoE" GitHub README, sections Usage and the two
 *                variants (eff / acc).
 *   [Shaping]    "Shaping Latent Mixture-of-Experts" summary page, Table 9
 *                (expert matrices W_g, W_u, W_o).
 *
 * What it computes, per token x (width d), in the order the LatentMoE code
 * module of [Explained] takes the steps:
 *   1. s_e = sum_i x_i W_r[e][i] (+ b_e)                  router on x, not z
 *   2. p   = softmax(s) over all N' experts
 *   3. the K' experts with the largest s, ordered by (s desc, e asc)
 *   4. g_k = p_{id_k} / sum_k' p_{id_k'}                   gates sum to 1
 *   5. z   = W_down x                                      d -> l, no bias
 *   6. u   = sum_{k=0..K'-1} g_k E_{id_k}(z),  E(v) = W_o (silu(W_g v) * (W_u v))
 *   7. y   = W_up u + sum_{j=0..n_s-1} S_j(x)              S_j: SwiGLU at width d
 * With activation = squared ReLU (the Expert class of the [Explained] code:
 * two matrices, the up-projection's output passed through relu and squared),
 * E(v) = W_o (relu(W_u v))^2 and the shared experts likewise; W_g is unused.
 * Readings where the pages are silent:
 *   - experts are SwiGLU with three matrices (the pages' code shows squared
 *     ReLU with two; the article says SwiGLU carries over with a third
 *     matrix, and [Shaping] Table 9 names W_g, W_u, W_o); silu(a)=a/(1+e^-a);
 *   - top-K' ties go to the lower expert index; selection is made on s
 *     (the same set as on p, and immune to exp rounding in fp64);
 *   - the optional router bias is added to the logits before the softmax;
 *   - slot order k = 0..K'-1 is the summation order of the combine, then
 *     W_up, then the shared experts in index order.
 * Arithmetic is fp64 throughout; inputs are widened exactly from f32 or
 * bf16 (a bf16 value is the top 16 bits of an IEEE f32).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ODT_F32 = 0, ODT_BF16 = 1, ODT_F64 = 2 };

enum { OACT_SWIGLU = 0, OACT_RELU2 = 1 };
enum { OQ_NONE = 0, OQ_E4M3 = 1, OQ_NVFP4 = 2, OQ_MODE = 3, OQ_BF16_ROWS = 16 };

typedef struct {
  int32_t d, l, m, n_routed, k_active, n_shared, m_shared;
  int32_t dtype;             /* element type of x and every weight below */
  int32_t activation;        /* OACT_SWIGLU or OACT_RELU2 */
  const void *w_router;      /* [N'][d] */
  const double *b_router;    /* [N'] or NULL */
  const void *w_down;        /* [l][d] */
  const void *w_up;          /* [d][l] */
  const void *w_gate;        /* [N'][m][l] */
  const void *w_upx;         /* [N'][m][l] */
  const void *w_out;         /* [N'][l][m] */
  const void *s_gate;        /* [n_s][m_s][d] */
  const void *s_up;          /* [n_s][m_s][d] */
  const void *s_out;         /* [n_s][d][m_s] */
  int32_t act_quant;         /* routed experts' activations: OQ_NONE, OQ_E4M3 (q_vec_e4m3)
                                or OQ_NVFP4 (q_vec_nvfp4), plus OQ_BF16_ROWS: the rows
                                are rounded to bf16 first (see q_act) */
} oracle_layer;

/* Exact widening of one stored element to double. */
static double elem(const void *base, int dt, size_t i) {
  if (dt == ODT_F32) return (double)((const float *)base)[i];
  if (dt == ODT_BF16) {
    uint32_t u = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  return ((const double *)base)[i];
}

/* out[r] = sum_c W[off + r*cols + c] * v[c], for r < rows. */
static void matvec(const void *W, int dt, size_t off, int rows, int cols,
                   const double *v, double *out) {
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    size_t base = off + (size_t)r * (size_t)cols;
    for (int c = 0; c < cols; ++c) acc += elem(W, dt, base + (size_t)c) * v[c];
    out[r] = acc;
  }
}

static double silu(double a) { return a / (1.0 + exp(-a)); }
static double relu2(double a) { return a > 0.0 ? a * a : 0.0; }

/* One expert feed-forward at the layer's activation.
 * SwiGLU: out = W_o (silu(W_g v) * (W_u v))  ([Explained], paragraph after
 * Figure 1: a gated activation adds a third matrix; Figure 9: the hidden
 * width is m on both sides).
 * Squared ReLU: out = W_o (relu(W_u v))^2  ([Explained], the Expert class:
 * up, relu, square, down).
 * W_g, W_u: [hid][in_w] at element offset off_in; W_o: [out_w][hid] at off_out. */
static void q_act(const oracle_layer *L, int mode, double *v, int n);

/* quant_hidden: the hidden vector is replaced by its row quantisation in
 * that mode (OQ_E4M3 or OQ_NVFP4) before the down-projection (the routed
 * experts when act_quant is set). */
static void swiglu_ffn(const oracle_layer *L, const void *Wg, const void *Wu,
                       const void *Wo, size_t off_in, size_t off_out, int in_w,
                       int hid, int out_w, const double *v, double *out,
                       double *scratch /* 2*hid */, int quant_hidden) {
  double *a = scratch, *b = scratch + hid;
  if (L->activation == OACT_RELU2) {
    matvec(Wu, L->dtype, off_in, hid, in_w, v, b);
    for (int j = 0; j < hid; ++j) a[j] = relu2(b[j]);
  } else {
    matvec(Wg, L->dtype, off_in, hid, in_w, v, a);
    matvec(Wu, L->dtype, off_in, hid, in_w, v, b);
    for (int j = 0; j < hid; ++j) a[j] = silu(a[j]) * b[j];
  }
  if (quant_hidden) q_act(L, quant_hidden, a, hid);
  matvec(Wo, L->dtype, off_out, out_w, hid, a, out);
}

/* ---- step 1: router logits, [Explained] Figure 3 and "routes in FULL d" */
static void router_row(const oracle_layer *L, const void *x, int xdt,
                       int64_t t, double *s) {
  const int d = L->d, N = L->n_routed;
  for (int e = 0; e < N; ++e) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i)
      acc += elem(x, xdt, (size_t)t * d + i) *
             elem(L->w_router, L->dtype, (size_t)e * d + i);
    s[e] = acc + (L->b_router ? L->b_router[e] : 0.0);
  }
}

void oracle_router_logits(const oracle_layer *L, const void *x, int64_t T,
                          double *s /* [T][N'] */) {
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t t = 0; t < T; ++t) router_row(L, x, L->dtype, t, s + t * L->n_routed);
}

/* ---- steps 2-4 for one token: softmax, top-K', renormalised gates.
 * [Explained] LatentMoE code module: the top-K' of the softmax of the
 * scores, then the selected weights divided by their sum. */
static void select_row(const double *s, int N, int K, int32_t *ids,
                       double *gates, unsigned char *taken) {
  double smax = s[0];
  for (int e = 1; e < N; ++e) if (s[e] > smax) smax = s[e];
  double denom = 0.0;
  for (int e = 0; e < N; ++e) denom += exp(s[e] - smax);
  memset(taken, 0, (size_t)N);
  for (int k = 0; k < K; ++k) {
    int best = -1;
    for (int e = 0; e < N; ++e) {
      if (taken[e]) continue;
      if (best < 0 || s[e] > s[best]) best = e; /* strict: ties keep lower e */
    }
    taken[best] = 1;
    ids[k] = best;
  }
  double psum = 0.0;
  for (int k = 0; k < K; ++k) {
    gates[k] = exp(s[ids[k]] - smax) / denom; /* p_{id_k} */
    psum += gates[k];
  }
  for (int k = 0; k < K; ++k) gates[k] /= psum;
}

int oracle_select(const double *s, int64_t T, int N, int K, int32_t *ids,
                  double *gates) {
  if (K < 1 || K > N) return -1;
#pragma omp parallel
  {
    unsigned char *taken = (unsigned char *)malloc((size_t)N);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t)
      select_row(s + t * N, N, K, ids + t * K, gates + t * K, taken);
    free(taken);
  }
  return 0;
}

/* Gates for caller-given ids: p_{id_k} / sum p over the given set. */
static void gates_for_ids(const double *s, int N, int K, const int32_t *ids,
                          double *gates) {
  double smax = s[0];
  for (int e = 1; e < N; ++e) if (s[e] > smax) smax = s[e];
  double denom = 0.0;
  for (int e = 0; e < N; ++e) denom += exp(s[e] - smax);
  double psum = 0.0;
  for (int k = 0; k < K; ++k) {
    gates[k] = exp(s[ids[k]] - smax) / denom;
    psum += gates[k];
  }
  for (int k = 0; k < K; ++k) gates[k] /= psum;
}

/* Gates of caller-given selections, row by row: step 4's rule (softmax at
 * the selected ids, renormalised over them) applied to any K'-subset, e.g.
 * a selection that differs from ours only on a near-tie. */
int oracle_gates(const double *s, int64_t T, int N, int K, const int32_t *ids,
                 double *gates) {
  if (K < 1 || K > N) return -1;
  for (int64_t i = 0; i < T * K; ++i)
    if (ids[i] < 0 || ids[i] >= N) return -2;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    gates_for_ids(s + t * N, N, K, ids + t * K, gates + t * K);
  return 0;
}

/* ---- components, exposed so tests can recompose the layer another way */

/* z = W_down x_t   ([Explained] Figure 6 upper half, "the only d-wide op") */
void oracle_down(const oracle_layer *L, const void *x, int64_t t, double *z) {
  double *xv = (double *)malloc(sizeof(double) * (size_t)L->d);
  for (int i = 0; i < L->d; ++i) xv[i] = elem(x, L->dtype, (size_t)t * L->d + i);
  matvec(L->w_down, L->dtype, 0, L->l, L->d, xv, z);
  free(xv);
}

/* out = E_e(z), one routed latent expert l -> m -> l ([Explained] Figure 9) */
void oracle_expert(const oracle_layer *L, int e, const double *z, double *out) {
  double *scratch = (double *)malloc(sizeof(double) * 2 * (size_t)L->m);
  swiglu_ffn(L, L->w_gate, L->w_upx, L->w_out, (size_t)e * L->m * L->l,
             (size_t)e * L->l * L->m, L->l, L->m, L->l, z, out, scratch, L->act_quant);
  free(scratch);
}

/* out = W_up u   ([Explained] Figure 6 lower half) */
void oracle_up(const oracle_layer *L, const double *u, double *out) {
  matvec(L->w_up, L->dtype, 0, L->d, L->l, u, out);
}

/* out = sum_j S_j(x_t), the shared experts at width d, in index order */
void oracle_shared(const oracle_layer *L, const void *x, int64_t t, double *out) {
  const int d = L->d, ms = L->m_shared;
  double *xv = (double *)malloc(sizeof(double) * (size_t)d);
  double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
  double *scratch = (double *)malloc(sizeof(double) * 2 * (size_t)(ms > 0 ? ms : 1));
  for (int i = 0; i < d; ++i) { xv[i] = elem(x, L->dtype, (size_t)t * d + i); out[i] = 0.0; }
  for (int j = 0; j < L->n_shared; ++j) {
    swiglu_ffn(L, L->s_gate, L->s_up, L->s_out, (size_t)j * ms * d,
               (size_t)j * d * ms, d, ms, d, xv, tmp, scratch, 0);
    for (int i = 0; i < d; ++i) out[i] += tmp[i];
  }
  free(xv); free(tmp); free(scratch);
}

/* ---- the whole layer for a list of tokens.
 * ids_in == NULL: route each token (steps 1-4).  Otherwise use ids_in[t][k]
 * as the selection (gates renormalised over that set) -- used when a token's
 * K'-th and (K'+1)-th logits are too close for the selection to be unique.
 * y[n][d] for n < n_tok is the output of token tokens[n]. */
int oracle_forward(const oracle_layer *L, const void *x, int64_t T,
                   const int64_t *tokens, int64_t n_tok, const int32_t *ids_in,
                   double *y, int32_t *ids_out, double *gates_out) {
  const int d = L->d, l = L->l, m = L->m, N = L->n_routed, K = L->k_active;
  if (K < 1 || K > N || l < 1 || d < 1 || m < 1) return -1;
  if (L->act_quant & ~(OQ_MODE | OQ_BF16_ROWS) || (L->act_quant & OQ_MODE) == OQ_MODE) return -1;
  if ((L->act_quant & OQ_MODE) == OQ_NVFP4 && (l % 16 || m % 16)) return -1;  /* 16-blocks */
  int err = 0;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *xv = (double *)malloc(sizeof(double) * (size_t)d);
    double *z = (double *)malloc(sizeof(double) * (size_t)l);
    double *u = (double *)malloc(sizeof(double) * (size_t)l);
    double *eo = (double *)malloc(sizeof(double) * (size_t)l);
    double *sh = (double *)malloc(sizeof(double) * (size_t)d);
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    double *g = (double *)malloc(sizeof(double) * (size_t)K);
    unsigned char *taken = (unsigned char *)malloc((size_t)N);
    int ms = L->m_shared > 0 ? L->m_shared : 1;
    double *scratch = (double *)malloc(sizeof(double) * 2 * (size_t)(m > ms ? m : ms));
#pragma omp for schedule(dynamic, 1)
    for (int64_t n = 0; n < n_tok; ++n) {
      const int64_t t = tokens ? tokens[n] : n;
      if (t < 0 || t >= T) { err = -2; continue; }
      router_row(L, x, L->dtype, t, s);
      if (ids_in) {
        memcpy(ids, ids_in + t * K, sizeof(int32_t) * (size_t)K);
        gates_for_ids(s, N, K, ids, g);
      } else {
        select_row(s, N, K, ids, g, taken);
      }
      for (int i = 0; i < d; ++i) xv[i] = elem(x, L->dtype, (size_t)t * d + i);
      matvec(L->w_down, L->dtype, 0, l, d, xv, z);
      if (L->act_quant) q_act(L, L->act_quant, z, l);  /* the experts read z quantised */
      for (int i = 0; i < l; ++i) u[i] = 0.0;
      for (int k = 0; k < K; ++k) { /* slot loop, in slot order */
        const int e = ids[k];
        swiglu_ffn(L, L->w_gate, L->w_upx, L->w_out, (size_t)e * m * l,
                   (size_t)e * l * m, l, m, l, z, eo, scratch, L->act_quant);
        for (int i = 0; i < l; ++i) u[i] += g[k] * eo[i];
      }
      double *yr = y + n * d;
      matvec(L->w_up, L->dtype, 0, d, l, u, yr);
      for (int j = 0; j < L->n_shared; ++j) {
        swiglu_ffn(L, L->s_gate, L->s_up, L->s_out, (size_t)j * L->m_shared * d,
                   (size_t)j * d * L->m_shared, d, L->m_shared, d, xv, sh, scratch, 0);
        for (int i = 0; i < d; ++i) yr[i] += sh[i];
      }
      if (ids_out) memcpy(ids_out + n * K, ids, sizeof(int32_t) * (size_t)K);
      if (gates_out) memcpy(gates_out + n * K, g, sizeof(double) * (size_t)K);
    }
    free(s); free(xv); free(z); free(u); free(eo); free(sh); free(ids); free(g);
    free(taken); free(scratch);
  }
  return err;
}

/* ---- dispatch: group the (token, slot) pairs by expert.
 * [Explained] LatentMoE code module: its slot loop visits each distinct
 * expert once and takes, through a boolean mask, the tokens that chose it,
 * in token order.  Written out plainly:
 * offsets[e] = number of pairs with expert < e (exclusive prefix count);
 * perm lists, expert by expert, the flat pair index t*K+k with t ascending;
 * pos is the inverse of perm. */
int oracle_dispatch(const int32_t *ids, int64_t T, int K, int N,
                    int32_t *offsets, int32_t *perm, int32_t *pos) {
  int64_t cursor = 0;
  for (int e = 0; e < N; ++e) {
    offsets[e] = (int32_t)cursor;
    for (int64_t t = 0; t < T; ++t)
      for (int k = 0; k < K; ++k)
        if (ids[t * K + k] == e) {
          perm[cursor] = (int32_t)(t * K + k);
          pos[t * K + k] = (int32_t)cursor;
          ++cursor;
        }
  }
  offsets[N] = (int32_t)cursor;
  return cursor == T * (int64_t)K ? 0 : -1; /* -1: an id outside [0, N) */
}

/* ---- backward: the gradient of the layer output with respect to x and to
 * every weight, for a given output cotangent dy (what loss.backward() of the
 * [README] Usage example computes for this layer).  The pages state no
 * formulas for it; it is the chain rule through steps 1-7 above, written
 * out per token:
 *   du   = W_up^T dy                         dW_up   += dy u^T
 *   per slot k (expert e, gate g_k, hidden h_k, output o_k):
 *     dg_k = du . o_k,  do_k = g_k du        dW_o[e] += do_k h_k^T
 *     dh   = W_o[e]^T do_k
 *     SwiGLU (a = W_g z, b = W_u z, h = silu(a) b):
 *       da = dh * b * silu'(a),  db = dh * silu(a)
 *     squared ReLU (b = W_u z, h = relu(b)^2):  db = dh * 2 relu(b)
 *     dz  += W_g[e]^T da + W_u[e]^T db       dW_g[e] += da z^T, dW_u[e] += db z^T
 *   gates g_k = p_{id_k} / sum p over the selected set = exp(s_{id_k}) /
 *   sum_j exp(s_{id_j}); the selection itself is piecewise constant, so
 *     ds_{id_k} = g_k (dg_k - sum_j g_j dg_j), ds_e = 0 for unselected e
 *                                           dW_r += ds x^T, db_r += ds
 *   dx = W_r^T ds + W_down^T dz + sum_j (S_g[j]^T da_j + S_u[j]^T db_j)
 *                                           dW_down += dz x^T
 *   shared expert j (input x, output added to y): dh_j = S_o[j]^T dy,
 *     da_j, db_j as above                   dS_o[j] += dy h_j^T,
 *                                           dS_g[j] += da_j x^T, dS_u[j] += db_j x^T
 * silu'(a) = sigma(a) (1 + a (1 - sigma(a))), sigma(a) = 1 / (1 + e^-a).
 * Weight gradients sum the listed tokens' contributions in token order. */
typedef struct {
  double *dx;        /* [n_tok][d], row n for token tokens[n] */
  double *w_router;  /* [N'][d]      (each array may be NULL: not computed) */
  double *b_router;  /* [N'] */
  double *w_down;    /* [l][d] */
  double *w_up;      /* [d][l] */
  double *w_gate;    /* [N'][m][l] */
  double *w_upx;     /* [N'][m][l] */
  double *w_out;     /* [N'][l][m] */
  double *s_gate;    /* [n_s][m_s][d] */
  double *s_up;      /* [n_s][m_s][d] */
  double *s_out;     /* [n_s][d][m_s] */
} oracle_grads;

static double dsilu(double a) {
  const double sg = 1.0 / (1.0 + exp(-a));
  return sg * (1.0 + a * (1.0 - sg));
}

/* Backward of one feed-forward (SwiGLU or squared ReLU) for input v, given
 * dout: writes the hidden h and the pre-activation gradients da, db (da is
 * zero for squared ReLU), and ADDS W_g^T da + W_u^T db to dv. */
static void ffn_backward(const oracle_layer *L, const void *Wg, const void *Wu,
                         const void *Wo, size_t off_in, size_t off_out, int in_w,
                         int hid, int out_w, const double *v, const double *dout,
                         double *h, double *da, double *db, double *dv,
                         double *scratch /* 2*hid */) {
  double *a = scratch, *b = scratch + hid;
  const int dt = L->dtype;
  matvec(Wu, dt, off_in, hid, in_w, v, b);
  if (L->activation == OACT_RELU2) {
    for (int c = 0; c < hid; ++c) h[c] = relu2(b[c]);
  } else {
    matvec(Wg, dt, off_in, hid, in_w, v, a);
    for (int c = 0; c < hid; ++c) h[c] = silu(a[c]) * b[c];
  }
  for (int c = 0; c < hid; ++c) { /* dh[c] = sum_j W_o[j][c] dout[j] */
    double dh = 0.0;
    for (int j = 0; j < out_w; ++j)
      dh += elem(Wo, dt, off_out + (size_t)j * hid + c) * dout[j];
    if (L->activation == OACT_RELU2) {
      da[c] = 0.0;
      db[c] = dh * 2.0 * (b[c] > 0.0 ? b[c] : 0.0);
    } else {
      da[c] = dh * b[c] * dsilu(a[c]);
      db[c] = dh * silu(a[c]);
    }
  }
  for (int i = 0; i < in_w; ++i) {
    double acc = 0.0;
    for (int c = 0; c < hid; ++c) {
      const size_t wi = off_in + (size_t)c * in_w + i;
      if (L->activation != OACT_RELU2) acc += elem(Wg, dt, wi) * da[c];
      acc += elem(Wu, dt, wi) * db[c];
    }
    dv[i] += acc;
  }
}

int oracle_backward(const oracle_layer *L, const void *x, int64_t T,
                    const int64_t *tokens, int64_t n_tok, const int32_t *ids_in,
                    const double *dy, const oracle_grads *G) {
  const int d = L->d, l = L->l, m = L->m, N = L->n_routed, K = L->k_active;
  const int ns = L->n_shared, ms = L->m_shared > 0 ? L->m_shared : 1;
  const int relu = L->activation == OACT_RELU2;
  if (K < 1 || K > N || l < 1 || d < 1 || m < 1) return -1;
  if (L->act_quant) return -3;  /* no gradient through the activation quantiser */
  /* per-token and per-slot records for the weight-gradient sums */
  double *X = (double *)malloc(sizeof(double) * (size_t)n_tok * d);
  double *Z = (double *)malloc(sizeof(double) * (size_t)n_tok * l);
  double *U = (double *)malloc(sizeof(double) * (size_t)n_tok * l);
  double *DZ = (double *)malloc(sizeof(double) * (size_t)n_tok * l);
  double *DS = (double *)malloc(sizeof(double) * (size_t)n_tok * K);
  int32_t *ID = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_tok * K);
  double *DO = (double *)malloc(sizeof(double) * (size_t)n_tok * K * l);
  double *H = (double *)malloc(sizeof(double) * (size_t)n_tok * K * m);
  double *DA = (double *)malloc(sizeof(double) * (size_t)n_tok * K * m);
  double *DB = (double *)malloc(sizeof(double) * (size_t)n_tok * K * m);
  double *HS = (double *)malloc(sizeof(double) * (size_t)n_tok * ns * ms + 1);
  double *DAS = (double *)malloc(sizeof(double) * (size_t)n_tok * ns * ms + 1);
  double *DBS = (double *)malloc(sizeof(double) * (size_t)n_tok * ns * ms + 1);
  if (!X || !Z || !U || !DZ || !DS || !ID || !DO || !H || !DA || !DB || !HS || !DAS || !DBS) {
    free(X); free(Z); free(U); free(DZ); free(DS); free(ID); free(DO); free(H);
    free(DA); free(DB); free(HS); free(DAS); free(DBS);
    return -3;
  }
  int err = 0;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *g = (double *)malloc(sizeof(double) * (size_t)K);
    double *dg = (double *)malloc(sizeof(double) * (size_t)K);
    double *du = (double *)malloc(sizeof(double) * (size_t)l);
    double *eo = (double *)malloc(sizeof(double) * (size_t)l);
    double *dxs = (double *)malloc(sizeof(double) * (size_t)d);
    unsigned char *taken = (unsigned char *)malloc((size_t)N);
    double *scratch = (double *)malloc(sizeof(double) * 2 * (size_t)(m > ms ? m : ms));
#pragma omp for schedule(dynamic, 1)
    for (int64_t n = 0; n < n_tok; ++n) {
      const int64_t t = tokens ? tokens[n] : n;
      if (t < 0 || t >= T) { err = -2; continue; }
      double *xv = X + n * d, *z = Z + n * l, *u = U + n * l, *dz = DZ + n * l;
      int32_t *ids = ID + n * K;
      const double *dyr = dy + n * d;
      router_row(L, x, L->dtype, t, s);
      if (ids_in) {
        memcpy(ids, ids_in + t * K, sizeof(int32_t) * (size_t)K);
        gates_for_ids(s, N, K, ids, g);
      } else {
        select_row(s, N, K, ids, g, taken);
      }
      for (int i = 0; i < d; ++i) xv[i] = elem(x, L->dtype, (size_t)t * d + i);
      matvec(L->w_down, L->dtype, 0, l, d, xv, z);
      /* forward of the slots (o_k is recomputed by ffn_backward's h; keep u) */
      for (int i = 0; i < l; ++i) u[i] = 0.0;
      for (int k = 0; k < K; ++k) {
        const int e = ids[k];
        swiglu_ffn(L, L->w_gate, L->w_upx, L->w_out, (size_t)e * m * l,
                   (size_t)e * l * m, l, m, l, z, eo, scratch, 0);
        for (int i = 0; i < l; ++i) u[i] += g[k] * eo[i];
        /* dg_k = du . o_k needs du first: o_k kept in DO for now */
        memcpy(DO + (n * K + k) * l, eo, sizeof(double) * (size_t)l);
      }
      /* du = W_up^T dy */
      for (int j = 0; j < l; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += elem(L->w_up, L->dtype, (size_t)i * l + j) * dyr[i];
        du[j] = acc;
      }
      double gdg = 0.0;
      for (int k = 0; k < K; ++k) {
        double acc = 0.0;
        const double *ok = DO + (n * K + k) * l;
        for (int j = 0; j < l; ++j) acc += du[j] * ok[j];
        dg[k] = acc;
        gdg += g[k] * acc;
      }
      for (int i = 0; i < l; ++i) dz[i] = 0.0;
      for (int k = 0; k < K; ++k) {
        const int e = ids[k];
        double *dok = DO + (n * K + k) * l;
        for (int j = 0; j < l; ++j) dok[j] = g[k] * du[j];
        ffn_backward(L, L->w_gate, L->w_upx, L->w_out, (size_t)e * m * l, (size_t)e * l * m,
                     l, m, l, z, dok, H + (n * K + k) * m, DA + (n * K + k) * m,
                     DB + (n * K + k) * m, dz, scratch);
        DS[n * K + k] = g[k] * (dg[k] - gdg);
      }
      /* dx = W_r^T ds + W_down^T dz + shared */
      for (int i = 0; i < d; ++i) dxs[i] = 0.0;
      for (int k = 0; k < K; ++k)
        for (int i = 0; i < d; ++i)
          dxs[i] += elem(L->w_router, L->dtype, (size_t)ids[k] * d + i) * DS[n * K + k];
      for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < l; ++j) acc += elem(L->w_down, L->dtype, (size_t)j * d + i) * dz[j];
        dxs[i] += acc;
      }
      for (int j = 0; j < ns; ++j)
        ffn_backward(L, L->s_gate, L->s_up, L->s_out, (size_t)j * L->m_shared * d,
                     (size_t)j * d * L->m_shared, d, L->m_shared, d, xv, dyr,
                     HS + (n * ns + j) * ms, DAS + (n * ns + j) * ms, DBS + (n * ns + j) * ms,
                     dxs, scratch);
      if (G->dx) memcpy(G->dx + n * d, dxs, sizeof(double) * (size_t)d);
    }
    free(s); free(g); free(dg); free(du); free(eo); free(dxs); free(taken); free(scratch);
  }
  if (err) goto done;
  /* weight gradients: each output element sums its tokens in token order */
  if (G->w_up) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < l; ++j) {
        double acc = 0.0;
        for (int64_t n = 0; n < n_tok; ++n) acc += dy[n * d + i] * U[n * l + j];
        G->w_up[(size_t)i * l + j] = acc;
      }
  }
  if (G->w_down) {
#pragma omp parallel for schedule(static)
    for (int j = 0; j < l; ++j)
      for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t n = 0; n < n_tok; ++n) acc += DZ[n * l + j] * X[n * d + i];
        G->w_down[(size_t)j * d + i] = acc;
      }
  }
  if (G->w_router || G->b_router) {
#pragma omp parallel for schedule(static)
    for (int e = 0; e < N; ++e) {
      double bacc = 0.0;
      double *row = G->w_router ? G->w_router + (size_t)e * d : NULL;
      if (row) for (int i = 0; i < d; ++i) row[i] = 0.0;
      for (int64_t n = 0; n < n_tok; ++n)
        for (int k = 0; k < K; ++k)
          if (ID[n * K + k] == e) {
            const double dsv = DS[n * K + k];
            bacc += dsv;
            if (row) for (int i = 0; i < d; ++i) row[i] += dsv * X[n * d + i];
          }
      if (G->b_router) G->b_router[e] = bacc;
    }
  }
  if (G->w_out || G->w_gate || G->w_upx) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int e = 0; e < N; ++e) {
      double *wo = G->w_out ? G->w_out + (size_t)e * l * m : NULL;
      double *wg = G->w_gate ? G->w_gate + (size_t)e * m * l : NULL;
      double *wu = G->w_upx ? G->w_upx + (size_t)e * m * l : NULL;
      if (wo) memset(wo, 0, sizeof(double) * (size_t)l * m);
      if (wg) memset(wg, 0, sizeof(double) * (size_t)m * l);
      if (wu) memset(wu, 0, sizeof(double) * (size_t)m * l);
      for (int64_t n = 0; n < n_tok; ++n)
        for (int k = 0; k < K; ++k) {
          if (ID[n * K + k] != e) continue;
          const double *dok = DO + (n * K + k) * l, *hk = H + (n * K + k) * m;
          const double *dak = DA + (n * K + k) * m, *dbk = DB + (n * K + k) * m;
          const double *z = Z + n * l;
          if (wo)
            for (int j = 0; j < l; ++j)
              for (int c = 0; c < m; ++c) wo[(size_t)j * m + c] += dok[j] * hk[c];
          for (int c = 0; c < m; ++c)
            for (int j = 0; j < l; ++j) {
              if (wg && !relu) wg[(size_t)c * l + j] += dak[c] * z[j];
              if (wu) wu[(size_t)c * l + j] += dbk[c] * z[j];
            }
        }
    }
  }
  if (ns > 0 && (G->s_out || G->s_gate || G->s_up)) {
    const int msr = L->m_shared;
#pragma omp parallel for schedule(static)
    for (int j = 0; j < ns; ++j) {
      double *so = G->s_out ? G->s_out + (size_t)j * d * msr : NULL;
      double *sg = G->s_gate ? G->s_gate + (size_t)j * msr * d : NULL;
      double *su = G->s_up ? G->s_up + (size_t)j * msr * d : NULL;
      if (so) memset(so, 0, sizeof(double) * (size_t)d * msr);
      if (sg) memset(sg, 0, sizeof(double) * (size_t)msr * d);
      if (su) memset(su, 0, sizeof(double) * (size_t)msr * d);
      for (int64_t n = 0; n < n_tok; ++n) {
        const double *hs = HS + (n * ns + j) * ms, *das = DAS + (n * ns + j) * ms;
        const double *dbs = DBS + (n * ns + j) * ms, *xv = X + n * d, *dyr = dy + n * d;
        if (so)
          for (int i = 0; i < d; ++i)
            for (int c = 0; c < msr; ++c) so[(size_t)i * msr + c] += dyr[i] * hs[c];
        for (int c = 0; c < msr; ++c)
          for (int i = 0; i < d; ++i) {
            if (sg && !relu) sg[(size_t)c * d + i] += das[c] * xv[i];
            if (su) su[(size_t)c * d + i] += dbs[c] * xv[i];
          }
      }
    }
  }
done:
  free(X); free(Z); free(U); free(DZ); free(DS); free(ID); free(DO); free(H);
  free(DA); free(DB); free(HS); free(DAS); free(DBS);
  return err;
}

/* ---- FP8 expert weights (the "LatentMoE Explained" remark that an expert
 * is 22 MB in FP8, and the models' NVFP4 pretraining; the pages give no
 * scaling recipe, so this one is chosen and stated): every weight row r of
 * an expert matrix gets a power-of-two scale s_r = 2^e_r, the smallest with
 * max_c |W[r][c]| <= 448 s_r (448 = the largest finite E4M3 value), and each
 * element is stored as q = E4M3(W[r][c] / s_r); the layer then uses
 * W'[r][c] = q * s_r.  E4M3 (the OCP 8-bit floating point format, E4M3
 * variant): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; normal values 2^(E-7) (1 + M/8) for E in 1..15 (E = 15, M = 7
 * is NaN, so the largest is 2^8 * 1.75 = 448); subnormals 2^-6 * M/8 (spacing
 * 2^-9).  Rounding is to nearest, ties to even mantissa, and out-of-range
 * magnitudes saturate to 448.  A row of zeros gets s = 1. */
static double e4m3_round(double v) {
  const double a = fabs(v);
  if (a == 0.0) return 0.0 * v;
  double r;
  if (a >= 448.0) {
    r = 448.0;
  } else {
    int e;
    frexp(a, &e);               /* a = f * 2^e, f in [0.5, 1): a in [2^(e-1), 2^e) */
    int ex = e - 1;             /* a in [2^ex, 2^(ex+1)) */
    if (ex < -6) ex = -6;       /* below the normal range: subnormal spacing */
    const double q = ldexp(1.0, ex - 3);  /* spacing of 3 mantissa bits */
    const double n = a / q;     /* exact: q is a power of two */
    double k = floor(n);
    const double frac = n - k;
    if (frac > 0.5 || (frac == 0.5 && fmod(k, 2.0) != 0.0)) k += 1.0;
    r = k * q;
    if (r > 448.0) r = 448.0;
  }
  return v < 0.0 ? -r : r;
}

/* The row scale: the smallest power of two s with amax <= 448 s (1 for a
 * row of zeros). */
static double e4m3_row_scale(double amax) {
  int e = 0;
  if (amax > 0.0) {
    e = (int)ceil(log2(amax / 448.0));
    while (ldexp(448.0, e) < amax) ++e;
    while (e > -200 && ldexp(448.0, e - 1) >= amax) --e;
  }
  return ldexp(1.0, e);
}

/* W [rows][cols] (any element type) -> W' (double) and the row scales. */
void oracle_fp8_rows(const void *W, int dt, int64_t rows, int cols, double *Wq,
                     double *scales) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    double amax = 0.0;
    for (int c = 0; c < cols; ++c) {
      const double v = fabs(elem(W, dt, (size_t)r * cols + c));
      if (v > amax) amax = v;
    }
    const double s = e4m3_row_scale(amax);
    scales[r] = s;
    for (int c = 0; c < cols; ++c)
      Wq[(size_t)r * cols + c] = e4m3_round(elem(W, dt, (size_t)r * cols + c) / s) * s;
  }
}

/* ---- E4M3 activations (act_quant = OQ_E4M3; a reading chosen here, the pages give no
 * FP8 activation recipe): the same rule as the weight rows, applied to each
 * activation vector the routed experts multiply -- a token's z (its row of
 * the expert GEMMs' first operand) and each expert's hidden h (its row of the
 * down-projection's first operand): v <- E4M3(v / s) * s with s the row
 * scale of v.  The router, W_down, the combine, W_up and the shared experts
 * stay as they are. */
static void q_vec_e4m3(double *v, int n) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i)
    if (fabs(v[i]) > amax) amax = fabs(v[i]);
  const double s = e4m3_row_scale(amax);
  for (int i = 0; i < n; ++i) v[i] = e4m3_round(v[i] / s) * s;
}

/* ---- NVFP4 (a reading chosen here: the pages say only that the models were
 * pretrained in NVFP4; the format is NVIDIA's published 4-bit floating
 * point).  Elements are E2M1 -- 1 sign bit, 2 exponent bits with bias 1, 1
 * mantissa bit, magnitudes 0, 0.5, 1, 1.5 (subnormal 0.5 and normals
 * 2^(E-1) (1 + M/2) for E = 1..3) up to 6 -- and every run of 16 consecutive
 * elements of a row (along the reduction dimension of the GEMM that reads
 * the row) shares one E4M3 block scale.  The second-level scale is taken per
 * row: s_r, the smallest power of two with amax_r <= 6 * 448 * s_r, so that
 * every block scale falls in E4M3's range.  Block j of the row gets
 *   b_j = E4M3(amax_j / (6 s_r)),
 * each of its elements the code q = E2M1(x * rcp_j) with rcp_j = 1 / (b_j
 * s_r) rounded once (0 for the whole block when b_j = 0): the element is
 * scaled by the reciprocal of its decoded block scale, as scaling to a
 * low-precision format is done in practice; the value the layer uses is
 * q b_j s_r.  The division, the reciprocal and the product decide codes, so
 * they are taken in IEEE single precision (round to nearest) on the
 * elements' single-precision values: the precision the GPU's quantisers
 * take them in.  (b_j s_r is exact in single precision: a 4-significant-bit
 * value times a power of two.)  E2M1 rounding is to nearest, ties to the
 * even mantissa, and magnitudes above 6 saturate. */
static double e2m1_round(double v) {
  const double a = fabs(v);
  double r;
  if (a >= 6.0) {
    r = 6.0;
  } else {
    /* grid spacing: 0.5 below 2 (0, 0.5, 1, 1.5), 1 in [2, 4), 2 in [4, 6] */
    const double q = a < 2.0 ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
    const double n = a / q;   /* exact */
    double k = floor(n);
    const double frac = n - k;
    /* an even k is an even mantissa on every segment of the grid */
    if (frac > 0.5 || (frac == 0.5 && fmod(k, 2.0) != 0.0)) k += 1.0;
    r = k * q;
  }
  return v < 0.0 ? -r : r;
}

/* The second-level row scale: the smallest power of two s with
 * amax <= 2688 s (2688 = 6 * 448), 1 for a row of zeros. */
static double nvfp4_row_scale(double amax) {
  int e = 0;
  if (amax > 0.0) {
    e = (int)ceil(log2(amax / 2688.0));
    while (ldexp(2688.0, e) < amax) ++e;
    while (e > -200 && ldexp(2688.0, e - 1) >= amax) --e;
  }
  return ldexp(1.0, e);
}

/* One row of n (a multiple of 16) single-precision values -> the values the
 * layer uses (out), the row scale and the n/16 block scales. */
static void nvfp4_row(const float *x, int n, double *out, double *row_scale,
                      double *block_scales) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i)
    if (fabs((double)x[i]) > amax) amax = fabs((double)x[i]);
  const double sr = nvfp4_row_scale(amax);
  *row_scale = sr;
  const float six_sr = (float)(6.0 * sr);
  for (int j = 0; j < n / 16; ++j) {
    float am = 0.0f;
    for (int i = 16 * j; i < 16 * j + 16; ++i)
      if (fabsf(x[i]) > am) am = fabsf(x[i]);
    const float t = am / six_sr;                         /* single precision */
    const double b = e4m3_round((double)t);
    if (block_scales) block_scales[j] = b;
    const float den = (float)(b * sr);                   /* exact */
    const float rcp = b == 0.0 ? 0.0f : 1.0f / den;      /* single precision */
    for (int i = 16 * j; i < 16 * j + 16; ++i) {
      if (b == 0.0) { out[i] = 0.0; continue; }
      const float y = x[i] * rcp;                        /* single precision */
      out[i] = e2m1_round((double)y) * b * sr;
    }
  }
}

/* W [rows][cols] (any element type, cols a multiple of 16) -> W' (double),
 * the row scales [rows] and the block scales [rows][cols/16].  -1 when cols
 * is not a multiple of 16. */
int oracle_nvfp4_rows(const void *W, int dt, int64_t rows, int cols, double *Wq,
                      double *row_scales, double *block_scales) {
  if (cols <= 0 || cols % 16) return -1;
#pragma omp parallel
  {
    float *xf = (float *)malloc(sizeof(float) * (size_t)cols);
#pragma omp for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
      for (int c = 0; c < cols; ++c) xf[c] = (float)elem(W, dt, (size_t)r * cols + c);
      nvfp4_row(xf, cols, Wq + (size_t)r * cols, row_scales + r,
                block_scales ? block_scales + (size_t)r * (cols / 16) : NULL);
    }
    free(xf);
  }
  return 0;
}

/* NVFP4 activations (act_quant = OQ_NVFP4): z and h quantised with the row
 * rule above, on their single-precision values. */
static void q_vec_nvfp4(double *v, int n) {
  float *xf = (float *)malloc(sizeof(float) * (size_t)n);
  for (int i = 0; i < n; ++i) xf[i] = (float)v[i];
  double sr;
  nvfp4_row(xf, n, v, &sr, NULL);
  free(xf);
}

/* v rounded to the nearest bf16 value (through single precision, ties to
 * even): the precision in which a bf16 layer holds z and h. */
static double round_bf16(double v) {
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7F800000u) != 0x7F800000u) u += 0x7FFFu + ((u >> 16) & 1u);
  u &= 0xFFFF0000u;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* The quantisation of an expert's activation row.  A code is an integer that
 * floating point decides, so it is decided on the values in the precision
 * the layer holds them in: for a bf16 layer (or with OQ_BF16_ROWS, a layer
 * whose other weights stand for bf16 ones) the row is first rounded to bf16
 * (z and h are bf16 vectors there). */
static void q_act(const oracle_layer *L, int mode, double *v, int n) {
  if (L->dtype == ODT_BF16 || (L->act_quant & OQ_BF16_ROWS))
    for (int i = 0; i < n; ++i) v[i] = round_bf16(v[i]);
  mode &= OQ_MODE;
  if (mode == OQ_E4M3) q_vec_e4m3(v, n);
  else if (mode == OQ_NVFP4) q_vec_nvfp4(v, n);
}

int oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
