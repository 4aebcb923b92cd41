/*
 * oracle.c -- plain fp64 reference of the Particle Transformer pair-bias block.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library. The CUDA product path
 * never links, imports or calls it, and it shares no code, header or table
 * with that path.
 *
 * What it computes, step by step (sources are the pages on the subject):
 *   1. Per particle, from the energy-first four-momentum (E, px, py, pz)
 *      [lloca.backbone.transformer_v2.Transformer, forward(): p_ref is
 *      energy-first]: pT = sqrt(px^2+py^2), rapidity y = 1/2 ln((E+pz)/(E-pz)),
 *      azimuth phi = atan2(py, px).
 *   2. Per ordered valid pair (a, b), the four Lorentz-invariant features named
 *      in "Event Classification with Masked Transformer Autoencoders",
 *      section "Fusion 2 -- Pairwise Features + Conv1d MLP -> FusedPairMLP",
 *      in the order (ln kT, ln z, ln dR, ln m^2), with the benchmark workload's
 *      definitions: dy = y_a - y_b, dphi wrapped to (-pi, pi],
 *      dR = sqrt(dy^2 + dphi^2), kT = min(pT)*dR, z = min(pT)/(pT_a + pT_b),
 *      m^2 = (E_a+E_b)^2 - |p_a+p_b|^2, each feature ln(max(x, 1e-8)).
 *   3. The pair-embedding MLP 4 -> 64 -> 64 -> 64 -> 8 of the same section,
 *      UNFOLDED: input affine x = a0*f + c0; three times
 *      h = GELU(a_k*(W_k h + b_k) + c_k) with the exact erf GELU; then
 *      U = W4 h + b4 with no activation. (The batch-norm layers appear as the
 *      per-channel affines a_k, c_k; the product folds them, this file does
 *      not, so agreement also checks the folding.)
 *   4. Masked multi-head attention with the additive pair bias, section
 *      "Fusion 3 -- Self-Attention + Additive Bias -> Fused Triton Attention":
 *      o_i = sum_j softmax_j(q_i.k_j / sqrt(D) + U[h,i,j]) v_j over valid
 *      keys j; masked keys are excluded (score -inf); masked query rows are 0.
 *
 *   5. (variant) int8 inputs of the hidden layers, the data-type quantisation
 *      of "Economical Jet Taggers -- Equivariant, Slim and Quantised",
 *      section "Kwantiseringsstrategieen": the inputs of linear layers are
 *      int8 with zero-point quantisation, the weights binary or ternary.
 *      Reading (orc_*_i8): layer 1 keeps its float input (the features);
 *      for layers 2, 3 and 4 the input row x (64 activations of one pair)
 *      is quantised on its own: lo = min(0, min x), hi = max(0, max x),
 *      s = (hi - lo) / 255 (s = 1 when hi == lo), z = -128 - round(lo / s),
 *      q = clamp(round(x / s) + z, -128, 127), rounding half to even; the
 *      layer's folded weights W' (rows a_k * W_k, bias a_k b_k + c_k; W4 and
 *      b4 as they are) are quantised per output row, alpha = max|W'_row| /
 *      127, T = round(W' / alpha); then y_o = alpha_o s sum_i T_oi (q_i - z)
 *      + b'_o, evaluated exactly (the integer sum in int64).
 *
 * Readings where the pages are silent: diagonal pairs (a == b) are included
 * and use the same formulas; pairs with a masked end are never evaluated and
 * their feature / bias entries are 0; Q/K/V are bf16 bit patterns widened
 * exactly to double.
 *
 * Layouts. Padded: momenta and mask [N*P], Q/K/V/out [N,H,P,D]. Packed
 * (mask == NULL, ptr != NULL): jet n owns tokens ptr[n] .. ptr[n+1]-1, its
 * local slot t is token ptr[n]+t, Q/K/V/out are [tokens,H,D]. Feature and
 * bias outputs are always padded per jet: feat [N,P,P,4], U [N,8,P,P].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_HID 64
#define ORC_NF 4
#define ORC_NH 8
#define ORC_PI 3.14159265358979323846

typedef struct {
  const float *a0, *c0;
  const float *W1, *b1, *a1, *c1;
  const float *W2, *b2, *a2, *c2;
  const float *W3, *b3, *a3, *c3;
  const float *W4, *b4;
} orc_params;

typedef struct {
  const float *E, *px, *py, *pz;
  const uint8_t *mask;   /* padded layout, 1 = valid */
  const int32_t *ptr;    /* packed layout, length N+1 */
  int32_t N, P;
} orc_jets;

static int g_threads = 0;

void orc_set_threads(int n) { g_threads = n; }

int orc_get_threads(void) {
#ifdef _OPENMP
  return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---------------------------------------------------------------- step 2 */

/* Neumaier's compensated sum: the running error of each addition is kept. */
static double compensated_sum(const double *x, int n) {
  double s = 0.0, c = 0.0;
  for (int i = 0; i < n; ++i) {
    double t = s + x[i];
    if (fabs(s) >= fabs(x[i])) c += (s - t) + x[i];
    else c += (x[i] - t) + s;
    s = t;
  }
  return s + c;
}

/* Product x*y as the unevaluated exact sum terms[0] + terms[1]. */
static void exact_product(double x, double y, double scale, double *terms) {
  double p = x * y;
  double e = fma(x, y, -p);
  terms[0] = scale * p;
  terms[1] = scale * e;
}

/* Invariant mass squared of a+b from its definition (E_a+E_b)^2 - |p_a+p_b|^2,
 * expanded into its twelve products; each product is split exactly and the
 * 24 terms are summed with compensation, so that the cancellation between
 * energy and momentum for near-collinear pairs loses no digits. */
static double pair_mass2(const double a[4], const double b[4]) {
  double t[24];
  int k = 0;
  for (int c = 0; c < 4; ++c) {
    double sign = (c == 0) ? 1.0 : -1.0;   /* metric (+,-,-,-) */
    exact_product(a[c], a[c], sign, t + k); k += 2;
    exact_product(b[c], b[c], sign, t + k); k += 2;
    exact_product(a[c], b[c], 2.0 * sign, t + k); k += 2;
  }
  return compensated_sum(t, 24);
}

static void particle(const double p[4], double *pt, double *y, double *phi) {
  *pt = sqrt(p[1] * p[1] + p[2] * p[2]);
  *y = 0.5 * log((p[0] + p[3]) / (p[0] - p[3]));
  *phi = atan2(p[2], p[1]);
}

static double log_clamped(double x) { return log(x > 1e-8 ? x : 1e-8); }

/* The four pair features (ln kT, ln z, ln dR, ln m^2) of particles a, b,
 * each given as (E, px, py, pz). */
void orc_pair_features(const double a[4], const double b[4], double out[4]) {
  double pta, ya, phia, ptb, yb, phib;
  particle(a, &pta, &ya, &phia);
  particle(b, &ptb, &yb, &phib);
  double dy = ya - yb;
  double dphi = phia - phib;
  if (dphi > ORC_PI) dphi -= 2.0 * ORC_PI;
  else if (dphi <= -ORC_PI) dphi += 2.0 * ORC_PI;
  double dr = sqrt(dy * dy + dphi * dphi);
  double ptmin = pta < ptb ? pta : ptb;
  double kt = ptmin * dr;
  double z = ptmin / (pta + ptb);
  double m2 = pair_mass2(a, b);
  out[0] = log_clamped(kt);
  out[1] = log_clamped(z);
  out[2] = log_clamped(dr);
  out[3] = log_clamped(m2);
}

/* ---------------------------------------------------------------- step 3 */

double orc_gelu(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }

/* One hidden layer: out = GELU(a * (W in + b) + c), W is [64][nin] row-major. */
static void hidden_layer(const double *in, int nin, const float *W, const float *b,
                         const float *a, const float *c, double *out) {
  for (int o = 0; o < ORC_HID; ++o) {
    double acc = 0.0;
    for (int i = 0; i < nin; ++i) acc += (double)W[o * nin + i] * in[i];
    double lin = acc + (double)b[o];
    out[o] = orc_gelu((double)a[o] * lin + (double)c[o]);
  }
}

/* Unfolded MLP for one pair row: features f[4] -> bias u[8]. */
void orc_mlp_row(const double f[4], const orc_params *w, double u[8]) {
  double x[ORC_NF], h1[ORC_HID], h2[ORC_HID], h3[ORC_HID];
  for (int i = 0; i < ORC_NF; ++i) x[i] = (double)w->a0[i] * f[i] + (double)w->c0[i];
  hidden_layer(x, ORC_NF, w->W1, w->b1, w->a1, w->c1, h1);
  hidden_layer(h1, ORC_HID, w->W2, w->b2, w->a2, w->c2, h2);
  hidden_layer(h2, ORC_HID, w->W3, w->b3, w->a3, w->c3, h3);
  for (int h = 0; h < ORC_NH; ++h) {
    double acc = 0.0;
    for (int i = 0; i < ORC_HID; ++i) acc += (double)w->W4[h * ORC_HID + i] * h3[i];
    u[h] = acc + (double)w->b4[h];
  }
}

/* ------------------------------------------------ int8 hidden-layer inputs */

/* Round half to even (the rounding of the quantiser). */
static double round_even(double x) { return nearbyint(x); }

/* Zero-point quantisation of one input row x[n] (see 5. above). */
void orc_quantize_act(const double *x, int n, int8_t *q, double *s_out, int *z_out) {
  double lo = 0.0, hi = 0.0;
  for (int i = 0; i < n; ++i) {
    if (x[i] < lo) lo = x[i];
    if (x[i] > hi) hi = x[i];
  }
  double s = hi > lo ? (hi - lo) / 255.0 : 1.0;
  int z = -128 - (int)round_even(lo / s);
  for (int i = 0; i < n; ++i) {
    double c = round_even(x[i] / s) + z;
    q[i] = (int8_t)(c < -128.0 ? -128 : (c > 127.0 ? 127 : c));
  }
  *s_out = s;
  *z_out = z;
}

/* Symmetric per-row weight codes: alpha = max|W_row| / 127 (1 for a zero
 * row), T = round(W / alpha). W is [rows][cols] row-major. */
void orc_quantize_weights(const double *W, int rows, int cols, int8_t *T, double *alpha) {
  for (int r = 0; r < rows; ++r) {
    double mx = 0.0;
    for (int c = 0; c < cols; ++c) mx = fmax(mx, fabs(W[r * cols + c]));
    double a = mx > 0.0 ? mx / 127.0 : 1.0;
    for (int c = 0; c < cols; ++c) T[r * cols + c] = (int8_t)round_even(W[r * cols + c] / a);
    alpha[r] = a;
  }
}

/* One linear layer with int8 input and weight codes:
 * y_o = alpha_o s sum_i T_oi (q_i - z) + b_o. */
static void int8_layer(const int8_t *q, double s, int z, const int8_t *T, const double *alpha,
                       const double *b, int nin, int nout, double *y) {
  for (int o = 0; o < nout; ++o) {
    int64_t acc = 0;
    for (int i = 0; i < nin; ++i) acc += (int64_t)T[o * nin + i] * ((int64_t)q[i] - z);
    y[o] = alpha[o] * s * (double)acc + b[o];
  }
}

/* The whole quantised linear map of one row, from float input and float
 * weights: both are quantised as above, then int8_layer. */
void orc_int8_linear(const double *x, int nin, const double *W, const double *b, int nout, double *y) {
  int8_t *q = malloc((size_t)nin), *T = malloc((size_t)nin * nout);
  double *alpha = malloc(sizeof(double) * nout), s;
  int z;
  orc_quantize_act(x, nin, q, &s, &z);
  orc_quantize_weights(W, nout, nin, T, alpha);
  int8_layer(q, s, z, T, alpha, b, nin, nout, y);
  free(q); free(T); free(alpha);
}

/* Folded and quantised layers 2..4 of one parameter set. */
typedef struct {
  int8_t T2[ORC_HID * ORC_HID], T3[ORC_HID * ORC_HID], T4[ORC_NH * ORC_HID];
  double al2[ORC_HID], al3[ORC_HID], al4[ORC_NH];
  double b2[ORC_HID], b3[ORC_HID], b4[ORC_NH];
} orc_i8;

static void fold_quantize_layer(const float *W, const float *b, const float *a, const float *c, int nout,
                                int8_t *T, double *alpha, double *bf) {
  double *Wf = malloc(sizeof(double) * nout * ORC_HID);
  for (int o = 0; o < nout; ++o) {
    double ao = a ? (double)a[o] : 1.0;
    for (int i = 0; i < ORC_HID; ++i) Wf[o * ORC_HID + i] = ao * (double)W[o * ORC_HID + i];
    bf[o] = ao * (double)b[o] + (c ? (double)c[o] : 0.0);
  }
  orc_quantize_weights(Wf, nout, ORC_HID, T, alpha);
  free(Wf);
}

static void prepare_i8(const orc_params *w, orc_i8 *qw) {
  fold_quantize_layer(w->W2, w->b2, w->a2, w->c2, ORC_HID, qw->T2, qw->al2, qw->b2);
  fold_quantize_layer(w->W3, w->b3, w->a3, w->c3, ORC_HID, qw->T3, qw->al3, qw->b3);
  fold_quantize_layer(w->W4, w->b4, NULL, NULL, ORC_NH, qw->T4, qw->al4, qw->b4);
}

/* MLP row with int8 inputs to layers 2..4: f[4] -> u[8]. */
static void mlp_row_i8(const double f[4], const orc_params *w, const orc_i8 *qw, double u[8]) {
  double x[ORC_NF], h[ORC_HID], y[ORC_HID], s;
  int8_t q[ORC_HID];
  int z;
  for (int i = 0; i < ORC_NF; ++i) x[i] = (double)w->a0[i] * f[i] + (double)w->c0[i];
  hidden_layer(x, ORC_NF, w->W1, w->b1, w->a1, w->c1, h);
  orc_quantize_act(h, ORC_HID, q, &s, &z);
  int8_layer(q, s, z, qw->T2, qw->al2, qw->b2, ORC_HID, ORC_HID, y);
  for (int i = 0; i < ORC_HID; ++i) h[i] = orc_gelu(y[i]);
  orc_quantize_act(h, ORC_HID, q, &s, &z);
  int8_layer(q, s, z, qw->T3, qw->al3, qw->b3, ORC_HID, ORC_HID, y);
  for (int i = 0; i < ORC_HID; ++i) h[i] = orc_gelu(y[i]);
  orc_quantize_act(h, ORC_HID, q, &s, &z);
  int8_layer(q, s, z, qw->T4, qw->al4, qw->b4, ORC_HID, ORC_NH, u);
}

/* One pair row of the int8 variant (for tests). */
void orc_mlp_row_i8(const double f[4], const orc_params *w, double u[8]) {
  orc_i8 *qw = malloc(sizeof(orc_i8));
  prepare_i8(w, qw);
  mlp_row_i8(f, w, qw, u);
  free(qw);
}

/* ------------------------------------------------------------ jet access */

/* Valid local slots of jet n and their element indices into the momentum
 * arrays. Returns the count, or -1 if the jet's description is invalid. */
static int jet_slots(const orc_jets *j, int n, int *slot, int64_t *elem) {
  int m = 0;
  if (j->mask) {
    for (int s = 0; s < j->P; ++s)
      if (j->mask[(int64_t)n * j->P + s]) { slot[m] = s; elem[m] = (int64_t)n * j->P + s; ++m; }
    return m;
  }
  int cnt = j->ptr[n + 1] - j->ptr[n];
  if (cnt < 0 || cnt > j->P) return -1;
  for (int t = 0; t < cnt; ++t) { slot[t] = t; elem[t] = (int64_t)j->ptr[n] + t; }
  return cnt;
}

static void momentum(const orc_jets *j, int64_t e, double p[4]) {
  p[0] = j->E[e]; p[1] = j->px[e]; p[2] = j->py[e]; p[3] = j->pz[e];
}

/* Element index of (jet n, head h, local slot s, dim 0) in Q/K/V/out. */
static int64_t qkv_index(const orc_jets *j, int n, int h, int s, int D) {
  if (j->mask) return (((int64_t)n * ORC_NH + h) * j->P + s) * D;
  return (((int64_t)j->ptr[n] + s) * ORC_NH + h) * D;
}

static double bf16_to_double(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ------------------------------------------------------------ batch APIs */

/* feat [N,P,P,4]: features of every valid ordered pair, 0 elsewhere. */
int orc_features(const orc_jets *j, double *feat) {
  int bad = 0;
  memset(feat, 0, sizeof(double) * (size_t)j->N * j->P * j->P * 4);
#pragma omp parallel for schedule(dynamic) num_threads(orc_get_threads()) reduction(| : bad)
  for (int n = 0; n < j->N; ++n) {
    int *slot = malloc(sizeof(int) * j->P);
    int64_t *elem = malloc(sizeof(int64_t) * j->P);
    int m = jet_slots(j, n, slot, elem);
    if (m < 0) { bad = 1; free(slot); free(elem); continue; }
    for (int ia = 0; ia < m; ++ia)
      for (int ib = 0; ib < m; ++ib) {
        double pa[4], pb[4];
        momentum(j, elem[ia], pa);
        momentum(j, elem[ib], pb);
        double *o = feat + ((((int64_t)n * j->P + slot[ia]) * j->P) + slot[ib]) * 4;
        orc_pair_features(pa, pb, o);
      }
    free(slot); free(elem);
  }
  return bad ? -1 : 0;
}

/* Bias of one jet over its valid ordered pairs: u[(h*m + ia)*m + ib]; with
 * qw, the int8 variant of the MLP. */
static void jet_bias(const orc_jets *j, const orc_params *w, const orc_i8 *qw, int m, const int64_t *elem,
                     double *u) {
  for (int ia = 0; ia < m; ++ia)
    for (int ib = 0; ib < m; ++ib) {
      double pa[4], pb[4], f[4], row[8];
      momentum(j, elem[ia], pa);
      momentum(j, elem[ib], pb);
      orc_pair_features(pa, pb, f);
      if (qw) mlp_row_i8(f, w, qw, row);
      else orc_mlp_row(f, w, row);
      for (int h = 0; h < ORC_NH; ++h) u[((int64_t)h * m + ia) * m + ib] = row[h];
    }
}

/* U [N,8,P,P]: bias of every valid ordered pair, 0 elsewhere; with qw the
 * int8 variant. */
static int pair_bias(const orc_jets *j, const orc_params *w, const orc_i8 *qw, double *U) {
  int bad = 0;
  memset(U, 0, sizeof(double) * (size_t)j->N * ORC_NH * j->P * j->P);
#pragma omp parallel for schedule(dynamic) num_threads(orc_get_threads()) reduction(| : bad)
  for (int n = 0; n < j->N; ++n) {
    int *slot = malloc(sizeof(int) * j->P);
    int64_t *elem = malloc(sizeof(int64_t) * j->P);
    int m = jet_slots(j, n, slot, elem);
    if (m < 0) { bad = 1; free(slot); free(elem); continue; }
    double *u = malloc(sizeof(double) * (size_t)ORC_NH * (m ? m : 1) * (m ? m : 1));
    jet_bias(j, w, qw, m, elem, u);
    for (int h = 0; h < ORC_NH; ++h)
      for (int ia = 0; ia < m; ++ia)
        for (int ib = 0; ib < m; ++ib)
          U[(((int64_t)n * ORC_NH + h) * j->P + slot[ia]) * j->P + slot[ib]] =
              u[((int64_t)h * m + ia) * m + ib];
    free(u); free(slot); free(elem);
  }
  return bad ? -1 : 0;
}

int orc_pair_bias(const orc_jets *j, const orc_params *w, double *U) { return pair_bias(j, w, NULL, U); }

int orc_pair_bias_i8(const orc_jets *j, const orc_params *w, double *U) {
  orc_i8 *qw = malloc(sizeof(orc_i8));
  prepare_i8(w, qw);
  int r = pair_bias(j, w, qw, U);
  free(qw);
  return r;
}

/* Attention of one jet. bias(h, ia, ib) is read from u_local (m x m per head)
 * when given, else from the padded U array of the batch. */
static void jet_attention(const orc_jets *j, int n, int m, const int *slot, const double *u_local,
                          const double *U, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          int D, double *out) {
  double scale = 1.0 / sqrt((double)D);
  double *s = malloc(sizeof(double) * (m ? m : 1));
  for (int h = 0; h < ORC_NH; ++h)
    for (int ia = 0; ia < m; ++ia) {
      int64_t qi = qkv_index(j, n, h, slot[ia], D);
      double smax = -INFINITY;
      for (int ib = 0; ib < m; ++ib) {
        int64_t ki = qkv_index(j, n, h, slot[ib], D);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf16_to_double(q[qi + d]) * bf16_to_double(k[ki + d]);
        double bias = u_local ? u_local[((int64_t)h * m + ia) * m + ib]
                              : U[(((int64_t)n * ORC_NH + h) * j->P + slot[ia]) * j->P + slot[ib]];
        s[ib] = dot * scale + bias;
        if (s[ib] > smax) smax = s[ib];
      }
      double denom = 0.0;
      for (int ib = 0; ib < m; ++ib) { s[ib] = exp(s[ib] - smax); denom += s[ib]; }
      for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int ib = 0; ib < m; ++ib)
          acc += s[ib] * bf16_to_double(v[qkv_index(j, n, h, slot[ib], D) + d]);
        out[qi + d] = acc / denom;
      }
    }
  free(s);
}

static int64_t qkv_elems(const orc_jets *j, int D) {
  if (j->mask) return (int64_t)j->N * ORC_NH * j->P * D;
  return (int64_t)j->ptr[j->N] * ORC_NH * D;
}

/* out (layout of q): attention with the given padded bias U [N,8,P,P]. */
int orc_attention(const orc_jets *j, const double *U, const uint16_t *q, const uint16_t *k,
                  const uint16_t *v, int D, double *out) {
  int bad = 0;
  memset(out, 0, sizeof(double) * (size_t)qkv_elems(j, D));
#pragma omp parallel for schedule(dynamic) num_threads(orc_get_threads()) reduction(| : bad)
  for (int n = 0; n < j->N; ++n) {
    int *slot = malloc(sizeof(int) * j->P);
    int64_t *elem = malloc(sizeof(int64_t) * j->P);
    int m = jet_slots(j, n, slot, elem);
    if (m < 0) bad = 1;
    else jet_attention(j, n, m, slot, NULL, U, q, k, v, D, out);
    free(slot); free(elem);
  }
  return bad ? -1 : 0;
}

/* out (layout of q): the whole block -- features, MLP bias and attention --
 * with each jet's bias kept local to the jet; with qw the int8 MLP. */
static int forward(const orc_jets *j, const orc_params *w, const orc_i8 *qw, const uint16_t *q,
                   const uint16_t *k, const uint16_t *v, int D, double *out) {
  int bad = 0;
  memset(out, 0, sizeof(double) * (size_t)qkv_elems(j, D));
#pragma omp parallel for schedule(dynamic) num_threads(orc_get_threads()) reduction(| : bad)
  for (int n = 0; n < j->N; ++n) {
    int *slot = malloc(sizeof(int) * j->P);
    int64_t *elem = malloc(sizeof(int64_t) * j->P);
    int m = jet_slots(j, n, slot, elem);
    if (m < 0) { bad = 1; free(slot); free(elem); continue; }
    double *u = malloc(sizeof(double) * (size_t)ORC_NH * (m ? m : 1) * (m ? m : 1));
    jet_bias(j, w, qw, m, elem, u);
    jet_attention(j, n, m, slot, u, NULL, q, k, v, D, out);
    free(u); free(slot); free(elem);
  }
  return bad ? -1 : 0;
}

int orc_forward(const orc_jets *j, const orc_params *w, const uint16_t *q, const uint16_t *k,
                const uint16_t *v, int D, double *out) {
  return forward(j, w, NULL, q, k, v, D, out);
}

int orc_forward_i8(const orc_jets *j, const orc_params *w, const uint16_t *q, const uint16_t *k,
                   const uint16_t *v, int D, double *out) {
  orc_i8 *qw = malloc(sizeof(orc_i8));
  prepare_i8(w, qw);
  int r = forward(j, w, qw, q, k, v, D, out);
  free(qw);
  return r;
}
