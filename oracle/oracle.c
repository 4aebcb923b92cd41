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

/* Bias of one jet over its valid ordered pairs: u[(h*m + ia)*m + ib]. */
static void jet_bias(const orc_jets *j, const orc_params *w, int m, const int64_t *elem, double *u) {
  for (int ia = 0; ia < m; ++ia)
    for (int ib = 0; ib < m; ++ib) {
      double pa[4], pb[4], f[4], row[8];
      momentum(j, elem[ia], pa);
      momentum(j, elem[ib], pb);
      orc_pair_features(pa, pb, f);
      orc_mlp_row(f, w, row);
      for (int h = 0; h < ORC_NH; ++h) u[((int64_t)h * m + ia) * m + ib] = row[h];
    }
}

/* U [N,8,P,P]: bias of every valid ordered pair, 0 elsewhere. */
int orc_pair_bias(const orc_jets *j, const orc_params *w, double *U) {
  int bad = 0;
  memset(U, 0, sizeof(double) * (size_t)j->N * ORC_NH * j->P * j->P);
#pragma omp parallel for schedule(dynamic) num_threads(orc_get_threads()) reduction(| : bad)
  for (int n = 0; n < j->N; ++n) {
    int *slot = malloc(sizeof(int) * j->P);
    int64_t *elem = malloc(sizeof(int64_t) * j->P);
    int m = jet_slots(j, n, slot, elem);
    if (m < 0) { bad = 1; free(slot); free(elem); continue; }
    double *u = malloc(sizeof(double) * (size_t)ORC_NH * (m ? m : 1) * (m ? m : 1));
    jet_bias(j, w, m, elem, u);
    for (int h = 0; h < ORC_NH; ++h)
      for (int ia = 0; ia < m; ++ia)
        for (int ib = 0; ib < m; ++ib)
          U[(((int64_t)n * ORC_NH + h) * j->P + slot[ia]) * j->P + slot[ib]] =
              u[((int64_t)h * m + ia) * m + ib];
    free(u); free(slot); free(elem);
  }
  return bad ? -1 : 0;
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
 * with each jet's bias kept local to the jet. */
int orc_forward(const orc_jets *j, const orc_params *w, const uint16_t *q, const uint16_t *k,
                const uint16_t *v, int D, double *out) {
  int bad = 0;
  memset(out, 0, sizeof(double) * (size_t)qkv_elems(j, D));
#pragma omp parallel for schedule(dynamic) num_threads(orc_get_threads()) reduction(| : bad)
  for (int n = 0; n < j->N; ++n) {
    int *slot = malloc(sizeof(int) * j->P);
    int64_t *elem = malloc(sizeof(int64_t) * j->P);
    int m = jet_slots(j, n, slot, elem);
    if (m < 0) { bad = 1; free(slot); free(elem); continue; }
    double *u = malloc(sizeof(double) * (size_t)ORC_NH * (m ? m : 1) * (m ? m : 1));
    jet_bias(j, w, m, elem, u);
    jet_attention(j, n, m, slot, u, NULL, q, k, v, D, out);
    free(u); free(slot); free(elem);
  }
  return bad ? -1 : 0;
}
