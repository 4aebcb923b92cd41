// pb_backward.cuh -- gradients of the fused pair-bias attention for sm_100a.
//
// pair_attention_backward launches, in order (per chunk of at most 8192 jets):
//   k_fused_grid<PM, true>  the bias of every unordered pair, 8 f16 in one
//                  16-byte record (the forward's balanced MLP phase over all
//                  SMs, the same values as the forward's fused paths), and
//                  the tile prefix T of the jets
//   k_attn_bwd     per jet: softmax statistics, dQ, dK, dV on m16n8k16 tensor
//                  cores; dL/dU[h,i,j] + dL/dU[h,j,i] accumulated into one
//                  fp32 record per unordered pair
//   k_mlp_bwd      the pairs' 128-row tiles split evenly over the CTAs: the
//                  MLP recomputed on tcgen05 (GELU' kept in TMEM), the
//                  backward through it on tcgen05, the weight gradients on
//                  m16n8k16 tensor cores in registers that persist over all
//                  the CTA's tiles (and chunks)
// then, once, k_grad_reduce: the per-CTA partials summed in CTA order.
//
// Source: "Event Classification with Masked Transformer Autoencoders",
// section "Fusion 3 -- Self-Attention + Additive Bias -> Fused Triton
// Attention" (forward and backward kernels of the biased attention), with the
// pair-MLP bias of "Fusion 2 -- Pairwise Features + Conv1d MLP ->
// FusedPairMLP".
#pragma once

#include "pb_kernels.cuh"

namespace pb {

// Records of jet n's unordered pair p = b(b+1)/2 + a (a <= b) sit at row
// T[n] * 128 + p of the record arrays (rows of a jet's last tile past its
// pairs are unused).
struct BwdArgs {
  const uint16_t *q, *k, *v, *dout;  // bf16, layout of the jets (padded [N,H,P,D], packed [tokens,H,D])
  uint16_t *dq, *dk, *dv;
  const uint4* urec;                 // bias: 8 f16 per pair
  float* grec;                       // upstream gradient of the pair's bias row: 8 fp32 per pair
  const int* T;                      // tile prefix [N + 1]
};

// ============================================== attention backward (k_attn_bwd)
//
// Per (jet, head), over the jet's m valid particles, with s = q.k/4 + U in
// log2 units (x log2 e) and 16-particle tiles I, J:
//   statistics (warp = tile I as queries): the row maximum and sum of exp2
//     give lse_i; O_i = sum_j p_ij v_j (p split into two bf16 terms so that O
//     is accurate to ~2^-17) gives D_i = dO_i . O_i;
//   gradients (warp = tile I, both as queries and as keys), for every tile J:
//     as queries  p_ij = exp2(s_ij - lse_i), dS_ij = p_ij (dO_i.v_j - D_i),
//                 dQ_i += 1/4 dS_ij k_j;
//     as keys     p_ji, dS_ji from the transposed tiles K_I Q_J^T, V_I dO_J^T
//                 (the bias U_ji = U_ij is the same element), dV_i += p_ji dO_j,
//                 dK_i += 1/4 dS_ji q_j;
//     both dS_ij and dS_ji then sit at the same fragment position, and the
//     pair's bias row gets g = dS_ij + dS_ji (dS_ii on the diagonal), written
//     once, by the tile of its smaller particle index, to the pair's fp32
//     record: no atomics and no zero-fill.
// Every statistics item finishes before any gradient item reads lse and D.
//
// Each staged head holds Q, K, V and dO of its rows as bf16 [m16][kKStride]
// (zero rows past m), then lse and D as fp32 [m16]. Every operand fragment
// comes from these row-major tiles through ldmatrix (.trans for the
// operands whose K dimension runs along the rows).

__host__ __device__ constexpr int bwd_tensor_bytes(int m) { return round16(m) * kKStride * 2; }
__host__ __device__ constexpr int bwd_head_bytes(int m) { return 4 * bwd_tensor_bytes(m) + 8 * round16(m); }

template <int PM>
__device__ void stage_bwd(const Particles<PM>& S, const JetArgs& J, const BwdArgs& X, int n, int h0, int hr,
                          unsigned char* buf) {
  const int m = S.m, m16 = round16(m), hb = bwd_head_bytes(m), tb = bwd_tensor_bytes(m);
  const int total = hr * m16 * 8, nthr = blockDim.x;
  for (int base = threadIdx.x; base < total; base += 4 * nthr) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * nthr;
      const int part = idx & 7, j = (idx >> 3) % m16, hh = (idx >> 3) / m16;
      v[u] = make_uint4(0, 0, 0, 0);
      if (idx < total && j < m) {
        const uint16_t* src = part < 2 ? X.q : (part < 4 ? X.k : (part < 6 ? X.v : X.dout));
        v[u] = *reinterpret_cast<const uint4*>(src + qkv_off<PM>(S, J, n, h0 + hh, j) + (part & 1) * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * nthr;
      if (idx >= total) break;
      const int part = idx & 7, j = (idx >> 3) % m16, hh = (idx >> 3) / m16;
      *reinterpret_cast<uint4*>(buf + hh * hb + (part >> 1) * tb + j * kKStride * 2 + (part & 1) * 16) = v[u];
    }
  }
  // lse and D of rows m .. m16-1 (read, masked, by the key pass) are 0
  for (int idx = threadIdx.x; idx < hr * 2 * m16; idx += nthr) {
    const int hh = idx / (2 * m16), r = idx % (2 * m16);
    reinterpret_cast<float*>(buf + hh * hb + 4 * tb)[r] = 0.f;
  }
}

// p (fp32) as the A fragment of a k16 step, split into hi + lo bf16 terms.
__device__ __forceinline__ void split_bf16_frag(const float* p, uint32_t* hi, uint32_t* lo) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    hi[i] = cvt_bf16x2(p[2 * i], p[2 * i + 1]);
    lo[i] = cvt_bf16x2(p[2 * i] - bf16lo(hi[i]), p[2 * i + 1] - bf16hi(hi[i]));
  }
}

__device__ __forceinline__ void pack_bf16_frag(const float* p, uint32_t* a) {
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = cvt_bf16x2(p[2 * i], p[2 * i + 1]);
}

// Scores of one 16 x 16 block in log2 units: s = acc / 4 + u, -inf where the
// column index (cols(e)) is >= m.
template <class Col>
__device__ __forceinline__ void bwd_scores(float* s, const float* u, int m, const Col& col) {
  const float qs = 0.25f * kLog2e;
#pragma unroll
  for (int e = 0; e < 8; ++e) s[e] = col(e) < m ? fmaf(s[e], qs, u[e] * kLog2e) : -INFINITY;
}

// Statistics of the queries [i0, i0 + 16) of one staged head at shared
// address hs: lse (log2 units) and D of its valid rows. Warp-wide.
template <class UBlock>
__device__ void bwd_stats_tile(uint32_t hs, int m, int i0, const UBlock& ub, float* lse, float* dd) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint32_t pitch = kKStride * 2, tb = (uint32_t)bwd_tensor_bytes(m);
  const uint32_t Qs = hs, Ks = hs + tb, Vs = hs + 2 * tb, Os = hs + 3 * tb;
  const int nrows = min(16, m - i0);
  const bool va = g < nrows, vb = g + 8 < nrows;
  const int ia = i0 + (va ? g : 0), ib = i0 + (vb ? g + 8 : 0);  // rows past the block alias row i0
  const uint32_t fa = frag_a_off(lane), fbn = frag_bn_off(lane), fbt = frag_bt_off(lane);
  uint32_t aq[4], ado[4];
  ldsm_x4(Qs + i0 * pitch + fa, aq);
  ldsm_x4(Os + i0 * pitch + fa, ado);
  float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float mxa = -INFINITY, mxb = -INFINITY, la = 0.f, lb = 0.f;
  for (int n0 = 0; n0 < m; n0 += 16) {
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    uint32_t bk[4];
    ldsm_x4(Ks + n0 * pitch + fbn, bk);
    mma_16816(s, aq, bk[0], bk[1]);
    mma_16816(s + 4, aq, bk[2], bk[3]);
    float u[8];
    ub(n0, i0, ia, ib, t, m, u);
    bwd_scores(s, u, m, [&](int e) { return n0 + (e & 4 ? 8 : 0) + 2 * t + (e & 1); });
    float bma = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[4], s[5]));
    float bmb = fmaxf(fmaxf(s[2], s[3]), fmaxf(s[6], s[7]));
    bma = fmaxf(bma, __shfl_xor_sync(0xffffffffu, bma, 1));
    bma = fmaxf(bma, __shfl_xor_sync(0xffffffffu, bma, 2));
    bmb = fmaxf(bmb, __shfl_xor_sync(0xffffffffu, bmb, 1));
    bmb = fmaxf(bmb, __shfl_xor_sync(0xffffffffu, bmb, 2));
    const float nma = fmaxf(mxa, bma), nmb = fmaxf(mxb, bmb);  // finite: key n0 < m is valid
    const float ca = ex2(mxa - nma), cb = ex2(mxb - nmb);
    mxa = nma;
    mxb = nmb;
    float p[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) p[e] = ex2(s[e] - (e & 2 ? nmb : nma));
    la = la * ca + ((p[0] + p[1]) + (p[4] + p[5]));
    lb = lb * cb + ((p[2] + p[3]) + (p[6] + p[7]));
    o[0] *= ca; o[1] *= ca; o[4] *= ca; o[5] *= ca;
    o[2] *= cb; o[3] *= cb; o[6] *= cb; o[7] *= cb;
    uint32_t ph[4], pl[4], bv[4];
    split_bf16_frag(p, ph, pl);
    ldsm_x4_t(Vs + n0 * pitch + fbt, bv);
    mma_16816(o, ph, bv[0], bv[1]);
    mma_16816(o + 4, ph, bv[2], bv[3]);
    mma_16816(o, pl, bv[0], bv[1]);
    mma_16816(o + 4, pl, bv[2], bv[3]);
  }
  la += __shfl_xor_sync(0xffffffffu, la, 1);
  la += __shfl_xor_sync(0xffffffffu, la, 2);
  lb += __shfl_xor_sync(0xffffffffu, lb, 1);
  lb += __shfl_xor_sync(0xffffffffu, lb, 2);
  // D = dO . O: the lane's O elements sit at the positions of its dO fragment
  float da = bf16lo(ado[0]) * o[0] + bf16hi(ado[0]) * o[1] + bf16lo(ado[2]) * o[4] + bf16hi(ado[2]) * o[5];
  float db = bf16lo(ado[1]) * o[2] + bf16hi(ado[1]) * o[3] + bf16lo(ado[3]) * o[6] + bf16hi(ado[3]) * o[7];
  da += __shfl_xor_sync(0xffffffffu, da, 1);
  da += __shfl_xor_sync(0xffffffffu, da, 2);
  db += __shfl_xor_sync(0xffffffffu, db, 1);
  db += __shfl_xor_sync(0xffffffffu, db, 2);
  if (t == 0) {
    if (va) {
      lse[ia] = mxa + __log2f(la);
      dd[ia] = da / la;
    }
    if (vb) {
      lse[ib] = mxb + __log2f(lb);
      dd[ib] = db / lb;
    }
  }
}

// Gradients of tile [i0, i0 + 16) of one staged head: dQ (its particles as
// queries), dK and dV (as keys) through dqrow / dkrow / dvrow, and the
// pairs' bias-row gradients g into gh[8 r] (gh = the jet's first record at
// head h, r = j(j+1)/2 + i for i <= j). Warp-wide.
template <class UBlock, class QRow, class KRow, class VRow>
__device__ void bwd_pair_tile(uint32_t hs, int m, int i0, const UBlock& ub, const float* lse, const float* dd,
                              float* gh, const QRow& dqrow, const KRow& dkrow, const VRow& dvrow) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint32_t pitch = kKStride * 2, tb = (uint32_t)bwd_tensor_bytes(m);
  const uint32_t Qs = hs, Ks = hs + tb, Vs = hs + 2 * tb, Os = hs + 3 * tb;
  const int nrows = min(16, m - i0);
  const bool va = g < nrows, vb = g + 8 < nrows;
  const int ia = i0 + (va ? g : 0), ib = i0 + (vb ? g + 8 : 0);
  const uint32_t fa = frag_a_off(lane), fbn = frag_bn_off(lane), fbt = frag_bt_off(lane);
  uint32_t aq[4], ado[4], ak[4], av[4];
  ldsm_x4(Qs + i0 * pitch + fa, aq);
  ldsm_x4(Os + i0 * pitch + fa, ado);
  ldsm_x4(Ks + i0 * pitch + fa, ak);
  ldsm_x4(Vs + i0 * pitch + fa, av);
  const float lse_a = lse[ia], lse_b = lse[ib], d_a = dd[ia], d_b = dd[ib];
  float dq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float dk[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float dv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int n0 = 0; n0 < m; n0 += 16) {
    auto col = [&](int e) { return n0 + (e & 4 ? 8 : 0) + 2 * t + (e & 1); };
    float u[8];
    ub(n0, i0, ia, ib, t, m, u);  // U_ij = U_ji
    uint32_t bk[4], bq[4], bv[4], bo[4];
    ldsm_x4(Ks + n0 * pitch + fbn, bk);
    ldsm_x4(Qs + n0 * pitch + fbn, bq);
    ldsm_x4(Vs + n0 * pitch + fbn, bv);
    ldsm_x4(Os + n0 * pitch + fbn, bo);
    // rows of the tile as queries: S = Q_I K_J^T, dP = dO_I V_J^T
    float sq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, dpq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    mma_16816(sq, aq, bk[0], bk[1]);
    mma_16816(sq + 4, aq, bk[2], bk[3]);
    mma_16816(dpq, ado, bv[0], bv[1]);
    mma_16816(dpq + 4, ado, bv[2], bv[3]);
    // as keys: S^T = K_I Q_J^T, dP^T = V_I dO_J^T
    float sk[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, dpk[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    mma_16816(sk, ak, bq[0], bq[1]);
    mma_16816(sk + 4, ak, bq[2], bq[3]);
    mma_16816(dpk, av, bo[0], bo[1]);
    mma_16816(dpk + 4, av, bo[2], bo[3]);
    bwd_scores(sq, u, m, col);
    bwd_scores(sk, u, m, col);
    const float2 l0 = *reinterpret_cast<const float2*>(lse + n0 + 2 * t);
    const float2 l1 = *reinterpret_cast<const float2*>(lse + n0 + 8 + 2 * t);
    const float2 d0 = *reinterpret_cast<const float2*>(dd + n0 + 2 * t);
    const float2 d1 = *reinterpret_cast<const float2*>(dd + n0 + 8 + 2 * t);
    const float lcol[4] = {l0.x, l0.y, l1.x, l1.y}, dcol[4] = {d0.x, d0.y, d1.x, d1.y};
    float dsq[8], pk[8], dsk[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int cidx = (e & 1) + ((e >> 1) & 2);  // column slot of element e: 2t + (e & 1) + 8 (e >> 2)
      const float pq = ex2(sq[e] - (e & 2 ? lse_b : lse_a));
      dsq[e] = pq * (dpq[e] - (e & 2 ? d_b : d_a));
      pk[e] = ex2(sk[e] - lcol[cidx]);
      dsk[e] = pk[e] * (dpk[e] - dcol[cidx]);
    }
    uint32_t pa[4], bkt[4], bot[4], bqt[4];
    pack_bf16_frag(dsq, pa);
    ldsm_x4_t(Ks + n0 * pitch + fbt, bkt);
    mma_16816(dq, pa, bkt[0], bkt[1]);
    mma_16816(dq + 4, pa, bkt[2], bkt[3]);
    pack_bf16_frag(pk, pa);
    ldsm_x4_t(Os + n0 * pitch + fbt, bot);
    mma_16816(dv, pa, bot[0], bot[1]);
    mma_16816(dv + 4, pa, bot[2], bot[3]);
    pack_bf16_frag(dsk, pa);
    ldsm_x4_t(Qs + n0 * pitch + fbt, bqt);
    mma_16816(dk, pa, bqt[0], bqt[1]);
    mma_16816(dk + 4, pa, bqt[2], bqt[3]);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = e & 2 ? ib : ia, j = col(e);
      const bool row_ok = e & 2 ? vb : va;
      if (row_ok && j < m && i <= j) gh[8 * (j * (j + 1) / 2 + i)] = i == j ? dsq[e] : dsq[e] + dsk[e];
    }
  }
  auto put = [&](uint16_t* row, const float* x, int o, float sc) {
    *reinterpret_cast<uint32_t*>(row + 2 * t) = cvt_bf16x2(sc * x[o], sc * x[o + 1]);
    *reinterpret_cast<uint32_t*>(row + 8 + 2 * t) = cvt_bf16x2(sc * x[o + 4], sc * x[o + 5]);
  };
  if (va) {
    put(dqrow(ia), dq, 0, 0.25f);
    put(dkrow(ia), dk, 0, 0.25f);
    put(dvrow(ia), dv, 0, 1.f);
  }
  if (vb) {
    put(dqrow(ib), dq, 2, 0.25f);
    put(dkrow(ib), dk, 2, 0.25f);
    put(dvrow(ib), dv, 2, 1.f);
  }
}

constexpr int kBwdStageBytes = 96 * 1024;  // staged heads of the attention backward (two CTAs per SM)
constexpr int kBwdHeadGroups = 2;          // CTA items: (jet, half of the heads)

template <int PM>
struct AttnBwdSmem {
  unsigned char stage[kBwdStageBytes];
  Particles<PM> part;
};

template <int PM>
__global__ void __launch_bounds__(256, 2) k_attn_bwd(JetArgs J, BwdArgs X) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  AttnBwdSmem<PM>& S = *reinterpret_cast<AttnBwdSmem<PM>*>(smem_raw);
  const int warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  constexpr int kHG = kH / kBwdHeadGroups;
  for (int item = blockIdx.x; item < J.N * kBwdHeadGroups; item += gridDim.x) {
    const int n = item / kBwdHeadGroups, hg = item % kBwdHeadGroups;
    stage_jet<PM, false>(S.part, J, n);
    const int m = S.part.m;
    const size_t rowbase = (size_t)X.T[n] * kTileM;
    if (m > 0) {
      const int hb = bwd_head_bytes(m), tb = bwd_tensor_bytes(m), m16 = round16(m);
      const int HR = max(1, min(kHG, kBwdStageBytes / hb));
      const int tiles = (m + 15) >> 4;
      const RecordUBias ub{reinterpret_cast<const __half*>(X.urec + rowbase)};
      if (in_bounds(hb <= kBwdStageBytes)) {
        for (int h0 = hg * kHG; h0 < (hg + 1) * kHG; h0 += HR) {
          const int hr = min(HR, (hg + 1) * kHG - h0);
          stage_bwd<PM>(S.part, J, X, n, h0, hr, S.stage);
          __syncthreads();
          for (int it = warp; it < hr * tiles; it += nwarp) {
            const int hh = it / tiles, h = h0 + hh;
            unsigned char* hbuf = S.stage + hh * hb;
            float* lse = reinterpret_cast<float*>(hbuf + 4 * tb);
            bwd_stats_tile(smem_u32(hbuf), m, (it % tiles) * 16, ub.head(h), lse, lse + m16);
          }
          __syncthreads();
          for (int it = warp; it < hr * tiles; it += nwarp) {
            const int hh = it / tiles, h = h0 + hh;
            unsigned char* hbuf = S.stage + hh * hb;
            const float* lse = reinterpret_cast<const float*>(hbuf + 4 * tb);
            bwd_pair_tile(smem_u32(hbuf), m, (it % tiles) * 16, ub.head(h), lse, lse + m16, X.grec + rowbase * 8 + h,
                          [&](int i) { return X.dq + qkv_off<PM>(S.part, J, n, h, i); },
                          [&](int i) { return X.dk + qkv_off<PM>(S.part, J, n, h, i); },
                          [&](int i) { return X.dv + qkv_off<PM>(S.part, J, n, h, i); });
          }
          __syncthreads();
        }
      }
    }
    if (hg == 0) {  // masked rows of every head
      zero_masked_rows<PM>(S.part, J, X.dq, n);
      zero_masked_rows<PM>(S.part, J, X.dk, n);
      zero_masked_rows<PM>(S.part, J, X.dv, n);
    }
    __syncthreads();
  }
}

// ==================================================== MLP backward (k_mlp_bwd)
//
// For the unordered pair (a, b) of a jet, the bias row u = MLP(f(a, b)) feeds
// both U[h, a, b] and U[h, b, a], so its upstream gradient is
// g_h = dS_h[a, b] + dS_h[b, a] (a != b) or dS_h[a, a], the record that the
// attention backward accumulated. Per tile of 128 such rows (one CTA, 512
// threads; thread (row r, quarter c) owns TMEM lane r and columns 16c ..
// 16c + 15 of each 64-wide accumulator):
//   z1 = W1' f + b1', h1 = GELU(z1), z2 = W2' h1 + b2', ... h3   (tcgen05)
//   e3 = g W4 (issued with z1), d3 = e3 * GELU'(z3), e2 = d3 W3', d2, e1 = d2 W2', d1
//   dW4 += g^T h3, dWk' += dk^T h(k-1) (h0 = f), dbk' += column sums of dk
// with bf16 operands and fp32 accumulation; f, g and the folded layer-1
// weights enter as bf16 hi + lo terms. GELU is the tanh form the forward
// kernels use (tanh.approx); GELU'(z) is computed with h and parked in TMEM
// over z until the backward step needs it. The weight gradients are 31
// (layer, 16-row block, up to three 8-column blocks) parts spread over the
// 16 warps as m16n8k16 MMAs whose A operand (d^T) and B operand (h) come
// from the row-major tiles through ldmatrix.trans; a column block of ones
// gives the bias gradients.

constexpr int kBwdMaxCtas = 256;     // partial-gradient slots in the workspace
constexpr int kFoldedFloats = 9160;  // W1 b1 W2 b2 W3 b3 W4 b4, as pb_fold_affine lays them out
constexpr int kOffW1 = 0, kOffB1 = 256, kOffW2 = 320, kOffB2 = 4416, kOffW3 = 4480, kOffB3 = 8576,
              kOffW4 = 8640, kOffB4 = 9152;

struct GradArgs {
  float *W1, *b1, *W2, *b2, *W3, *b3, *W4, *b4;
};

template <int PM>
struct MlpBwdSmem {
  __nv_bfloat16 A0[kTileM * 16];     // [hi(f) | lo(f) | hi(f) | 0]
  __nv_bfloat16 G4[kTileM * 16];     // [hi(g) | lo(g)] (8 heads each)
  __half Hf[2][kTileM * 64];         // h1, h2 in f16: operands of z2, z3
  __nv_bfloat16 Hs[3][kTileM * 64];  // h1, h2, h3 in bf16: operands of the weight gradients
  __nv_bfloat16 Ds[3][kTileM * 64];  // d1, d2, d3 = dL/dz
  __nv_bfloat16 W1f[64 * 16];        // [hi(W1') | hi(W1') | lo(W1') | 0] per output row
  __half Wf[2][2][64 * 64];          // W2', W3' as [out][in], f16: hi, lo
  __nv_bfloat16 Wt[2][2][64 * 64];   // W2'^T, W3'^T as [in][out]: hi, lo
  __nv_bfloat16 W4t[2][64 * 16];     // [W4^T | W4^T] as [in][out]: hi, lo
  float bias[3][64];                 // b1', b2', b3'
  uint64_t mbar;
  uint32_t tmem_base;
  Particles<PM> part;
};

// Weights in the canonical K-major layouts of their MMA roles.
template <int PM>
__device__ void bwd_load_weights(MlpBwdSmem<PM>& S, const MlpArgs& W) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  for (int e = tid; e < 64 * 64; e += nthr) {
    const int o = e >> 6, i = e & 63;
    const float w[2] = {W.W2[e], W.W3[e]};
#pragma unroll
    for (int L = 0; L < 2; ++L) {
      const __half fh = __float2half_rn(w[L]), fl = __float2half_rn(w[L] - __half2float(fh));
      S.Wf[L][0][cofs(o, i, 64)] = fh;
      S.Wf[L][1][cofs(o, i, 64)] = fl;
      const __nv_bfloat16 hi = __float2bfloat16_rn(w[L]), lo = __float2bfloat16_rn(w[L] - __bfloat162float(hi));
      S.Wt[L][0][cofs(i, o, 64)] = hi;
      S.Wt[L][1][cofs(i, o, 64)] = lo;
    }
  }
  for (int e = tid; e < 64 * 16; e += nthr) {
    const int r = e >> 4, k = e & 15;  // W1f row = output r, W4t row = input r
    const float w1 = k < 12 ? W.W1[r * 4 + (k & 3)] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w1);
    S.W1f[cofs(r, k, 16)] = (k >= 8 && k < 12) ? __float2bfloat16_rn(w1 - __bfloat162float(hi)) : hi;
    const float w4 = W.W4[(k & 7) * 64 + r];
    const __nv_bfloat16 h4 = __float2bfloat16_rn(w4);
    S.W4t[0][cofs(r, k, 16)] = h4;
    S.W4t[1][cofs(r, k, 16)] = __float2bfloat16_rn(w4 - __bfloat162float(h4));
  }
  for (int e = tid; e < 3 * 64; e += nthr) S.bias[e >> 6][e & 63] = (e < 64 ? W.b1 : (e < 128 ? W.b2 : W.b3))[e & 63];
}

// GELU(z) = z/2 (1 + tanh(u)), u = sqrt(2/pi) (z + 0.044715 z^3), and its
// derivative Phi + z/2 sech^2(u) sqrt(2/pi) (1 + 3 0.044715 z^2), where
// Phi = (1 + tanh u) / 2. Both come from w = exp(-2|u|): Phi = 1 / (1 + w)
// (u >= 0) or w / (1 + w), sech^2 u = 4 w / (1 + w)^2, which stay accurate
// where tanh saturates (1 - tanh^2 from an approximate tanh would not, and
// its error there is the same for every pair with large |u|).
__device__ __forceinline__ void gelu_tanh_and_grad(float z, float& h, float& dh) {
  constexpr float kC0 = 0.7978845608028654f, kC1 = 0.044715f;
  const float z2 = z * z, c0z = kC0 * z;
  const float u = c0z * fmaf(kC1, z2, 1.f);
  const float w = ex2(-2.f * kLog2e * fabsf(u));
  const float r = __fdividef(1.f, 1.f + w);
  const float phi = u >= 0.f ? r : w * r;
  h = z * phi;
  const float sech2 = 4.f * w * r * r;
  dh = fmaf(0.5f * sech2, c0z * fmaf(3.f * kC1, z2, 1.f), phi);
}

// TMEM <- registers, 32 lanes x 16 columns (thread t of the warp writes lane
// quadrant base + t), then wait for the stores.
__device__ __forceinline__ void tmem_st16_wait(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}

// One weight-gradient part: layer L (1..4), 16-row block mb of dW, column
// blocks nb0 .. nb0 + nc - 1 (the last block index of a layer is the ones
// column: 8 for L = 2..4, 1 for L = 1).
struct GradPart {
  int L, mb, nb0, nc;
};

__device__ __forceinline__ GradPart grad_part(int q) {
  if (q < 3) return GradPart{4, 0, 3 * q, 3};
  if (q < 15) return GradPart{3, (q - 3) / 3, 3 * ((q - 3) % 3), 3};
  if (q < 27) return GradPart{2, (q - 15) / 3, 3 * ((q - 15) % 3), 3};
  return GradPart{1, q - 27, 0, 2};
}
constexpr int kGradParts = 31;

template <int PM>
__device__ __forceinline__ void grad_tiles(const MlpBwdSmem<PM>& S, const GradPart& gp, const __nv_bfloat16*& Dt,
                                           int& Kd, const __nv_bfloat16*& Bt, int& Kb, int& ones) {
  Dt = gp.L == 4 ? S.G4 : S.Ds[gp.L - 1];
  Kd = gp.L == 4 ? 16 : 64;
  Bt = gp.L == 1 ? S.A0 : S.Hs[gp.L - 2];
  Kb = gp.L == 1 ? 16 : 64;
  ones = gp.L == 1 ? 1 : 8;
}

// acc[j] += d^T h over the tile's 128 rows for the part's column blocks.
// Lane addresses are formed once; each 16-row step moves both operands by
// two 8-row core groups.
template <int PM>
__device__ __forceinline__ void grad_mma(const MlpBwdSmem<PM>& S, const GradPart& gp, float (*acc)[4]) {
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16 *Dt, *Bt;
  int Kd, Kb, ones;
  grad_tiles(S, gp, Dt, Kd, Bt, Kb, ones);
  const int mi = lane >> 3;
  const uint32_t a_addr = smem_u32(Dt) + 2u * cofs((lane & 7) + (mi >> 1) * 8, gp.mb * 16 + (mi & 1) * 8, Kd);
  const uint32_t b_row = smem_u32(Bt) + 2u * cofs((lane & 7) + ((lane >> 3) & 1) * 8, 0, Kb);
  const uint32_t a_step = (uint32_t)Kd * 32u, b_step = (uint32_t)Kb * 32u;  // 16 rows
  uint32_t b_addr[3];
  bool is_one[3];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int nb = gp.nb0 + j;
    is_one[j] = nb == ones;
    b_addr[j] = b_row + 128u * (uint32_t)(is_one[j] ? 0 : nb);
  }
#pragma unroll 2
  for (int k = 0; k < kTileM / 16; ++k) {
    uint32_t a[4];
    ldsm_x4_t(a_addr + a_step * k, a);
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      if (j >= gp.nc) break;
      uint32_t b[2];
      if (is_one[j]) {
        b[0] = b[1] = 0x3F803F80u;  // bf16 1.0 in both halves
      } else {
        ldsm_x2_t(b_addr[j] + b_step * k, b);
      }
      mma_16816(acc[j], a, b[0], b[1]);
    }
  }
}

// The part's accumulators into the CTA's partial (folded layout), added to
// what the slot holds when `accumulate`.
__device__ void grad_store(const GradPart& gp, float (*acc)[4], float* part, bool accumulate) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int oa = gp.mb * 16 + g, ob = oa + 8;
  auto put = [&](int idx, float v) { part[idx] = accumulate ? part[idx] + v : v; };
  for (int j = 0; j < gp.nc; ++j) {
    const int nb = gp.nb0 + j;
    const float* c = acc[j];
    if (gp.L == 1) {
      // columns 0..3 hold sum d hi(f), 4..7 sum d lo(f)
      const float p0 = __shfl_down_sync(0xffffffffu, c[0], 2), p1 = __shfl_down_sync(0xffffffffu, c[1], 2);
      const float p2 = __shfl_down_sync(0xffffffffu, c[2], 2), p3 = __shfl_down_sync(0xffffffffu, c[3], 2);
      if (nb == 0) {
        if (t < 2) {
          put(kOffW1 + oa * 4 + 2 * t, c[0] + p0);
          put(kOffW1 + oa * 4 + 2 * t + 1, c[1] + p1);
          put(kOffW1 + ob * 4 + 2 * t, c[2] + p2);
          put(kOffW1 + ob * 4 + 2 * t + 1, c[3] + p3);
        }
      } else if (t == 0) {
        put(kOffB1 + oa, c[0]);
        put(kOffB1 + ob, c[2]);
      }
    } else if (gp.L == 4) {  // rows g: sum hi(g) h3, rows g + 8: sum lo(g) h3
      if (nb < 8) {
        put(kOffW4 + g * 64 + nb * 8 + 2 * t, c[0] + c[2]);
        put(kOffW4 + g * 64 + nb * 8 + 2 * t + 1, c[1] + c[3]);
      } else if (t == 0) {
        put(kOffB4 + g, c[0] + c[2]);
      }
    } else {
      const int offW = gp.L == 2 ? kOffW2 : kOffW3, offB = gp.L == 2 ? kOffB2 : kOffB3;
      if (nb < 8) {
        put(offW + oa * 64 + nb * 8 + 2 * t, c[0]);
        put(offW + oa * 64 + nb * 8 + 2 * t + 1, c[1]);
        put(offW + ob * 64 + nb * 8 + 2 * t, c[2]);
        put(offW + ob * 64 + nb * 8 + 2 * t + 1, c[3]);
      } else if (t == 0) {
        put(offB + oa, c[0]);
        put(offB + ob, c[2]);
      }
    }
  }
}

// The T[N] tiles are split evenly over the CTAs (a CTA's range may start and
// end inside a jet); the CTA's weight-gradient partial goes to slot
// blockIdx.x, added to it when `accumulate` (later chunks of a batch).
template <int PM>
__global__ void __launch_bounds__(512, 1) k_mlp_bwd(JetArgs J, MlpArgs W, BwdArgs X, float* __restrict__ partials,
                                                    int accumulate) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  MlpBwdSmem<PM>& S = *reinterpret_cast<MlpBwdSmem<PM>*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int r = tid & 127, c = tid >> 7;  // tile row (TMEM lane) and column quarter
  bwd_load_weights<PM>(S, W);
  if (tid == 0) {
    mbar_init(&S.mbar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, 256);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // TMEM columns: z1 [0, 64), z2 [64, 128), z3 [128, 192) (then GELU'), e3 / e2 / e1 [192, 256)
  const uint32_t tm = S.tmem_base, lane_off = (uint32_t)((warp & 3) * 32) << 16;
  constexpr uint32_t kId = idesc_bf16_m128(64);
  const uint32_t a0 = smem_u32(S.A0), g4 = smem_u32(S.G4), w1f = smem_u32(S.W1f);
  const uint32_t w4t_hi = smem_u32(S.W4t[0]), w4t_lo = smem_u32(S.W4t[1]);
  uint32_t phase = 0u;
  bool ok = true, aborted = false;

  const GradPart gp0 = grad_part(warp), gp1 = grad_part(min(warp + 16, kGradParts - 1));
  const bool has1 = warp + 16 < kGradParts;
  float acc0[3][4], acc1[3][4];
#pragma unroll
  for (int j = 0; j < 3; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc0[j][e] = acc1[j][e] = 0.f;

  // operand writes published, then thread 0 issues `body` and commits
  auto issue = [&](auto&& body) -> bool {
    fence_proxy_async_smem();
    tc_fence_before();
    if (__syncthreads_or(!ok)) return false;
    if (tid == 0) {
      tc_fence_after();
      body();
      mma_commit(&S.mbar);
    }
    return true;
  };
  auto wait = [&]() {
    const bool done = mbar_wait(&S.mbar, phase);
    phase ^= 1u;
    ok = ok && done;
    tc_fence_after();
  };
  // D = A (W_hi + W_lo): the weights' rounding error is the same for every
  // pair row and would not average out of the gradient sums, so they enter as
  // two terms. The recompute's products (A = h, f16) use kind::f16 with f16
  // operands, the backward's (A = d, bf16) bf16 operands.
  auto gemm64 = [&](uint32_t d, uint32_t aa, uint32_t b_hi, uint32_t b_lo, uint32_t id) {
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const uint32_t bb = part ? b_lo : b_hi;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_f16(d, smem_desc(aa + 256u * k, 128, 1024), smem_desc(bb + 256u * k, 128, 1024), id,
                (part | k) != 0 ? 1u : 0u);
    }
  };
  constexpr uint32_t kIdF16 = idesc_f16_m128(64);
  auto store16 = [&](void* T, const float* v, bool f16) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = f16 ? cvt_f16x2(v[2 * i], v[2 * i + 1]) : cvt_bf16x2(v[2 * i], v[2 * i + 1]);
    uint16_t* T16 = static_cast<uint16_t*>(T);
    *reinterpret_cast<uint4*>(T16 + cofs(r, 16 * c, 64)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(T16 + cofs(r, 16 * c + 8, 64)) = make_uint4(w[4], w[5], w[6], w[7]);
  };
  // h_k = GELU(z_k + b_k) to the operand tile, GELU'(z_k + b_k) back over z_k in TMEM
  auto hidden = [&](int k) {
    float z[16], h[16];
    const uint32_t ta = tm + lane_off + 64u * k + 16u * c;
    tmem_ld16_wait(ta, z);
    const float4* bq = reinterpret_cast<const float4*>(&S.bias[k][16 * c]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 bb = bq[i];
      z[4 * i] += bb.x;
      z[4 * i + 1] += bb.y;
      z[4 * i + 2] += bb.z;
      z[4 * i + 3] += bb.w;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) gelu_tanh_and_grad(z[i], h[i], z[i]);
    if (k < 2) store16(S.Hf[k], h, true);  // the next layer's operand
    store16(S.Hs[k], h, false);
    tmem_st16_wait(ta, z);
  };
  // d_k = e * GELU'(z_k + b_k)
  auto delta = [&](int k) {
    float gp[16], e[16];
    tmem_ld16_wait(tm + lane_off + 64u * k + 16u * c, gp);
    tmem_ld16_wait(tm + lane_off + 192u + 16u * c, e);
#pragma unroll
    for (int i = 0; i < 16; ++i) e[i] *= gp[i];
    store16(S.Ds[k], e, false);
  };

  const long long Ttot = X.T[J.N];
  const long long lo = Ttot * blockIdx.x / gridDim.x, hi = Ttot * (blockIdx.x + 1) / gridDim.x;
  int n = 0;
  {
    int l = 0, rr = J.N;  // first jet whose tiles reach past lo
    while (l < rr) {
      const int mid = (l + rr) >> 1;
      if (X.T[mid + 1] > lo) rr = mid; else l = mid + 1;
    }
    n = l;
  }
  for (; n < J.N && X.T[n] < hi && !aborted; ++n) {
    const long long tj0 = X.T[n], tj1 = X.T[n + 1];
    if (tj1 <= tj0) continue;  // no pairs
    stage_jet<PM>(S.part, J, n);
    const int m = S.part.m;
    const int npairs = m * (m + 1) / 2;
    const float* gjet = X.grec + (size_t)tj0 * kTileM * 8;
    const int t_first = (int)(max(lo, tj0) - tj0), t_last = (int)(min(hi, tj1) - tj0);
    for (int t = t_first; t < t_last; ++t) {
      // row r: the unordered pair p = b(b+1)/2 + a; features (c = 0) and g (c = 1)
      const int p = t * kTileM + r;
      int a = 0, b = 0;
      bool valid = p < npairs;
      if (valid && c == 0) {
        TriPairs{}.map(p, a, b);
        valid = in_bounds(a >= 0 && a <= b && b < m);
      }
      if (c == 0) {
        float f[4] = {0.f, 0.f, 0.f, 0.f};
        if (valid) pair_feat<PM, true>(S.part, a, b, f);  // the forward MLP's features
        const uint32_t h01 = cvt_bf16x2(f[0], f[1]), h23 = cvt_bf16x2(f[2], f[3]);
        const uint32_t l01 = cvt_bf16x2(f[0] - bf16lo(h01), f[1] - bf16hi(h01));
        const uint32_t l23 = cvt_bf16x2(f[2] - bf16lo(h23), f[3] - bf16hi(h23));
        *reinterpret_cast<uint4*>(S.A0 + cofs(r, 0, 16)) = make_uint4(h01, h23, l01, l23);
        *reinterpret_cast<uint4*>(S.A0 + cofs(r, 8, 16)) = make_uint4(h01, h23, 0u, 0u);
      } else if (c == 1) {
        float gv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (valid) {
          const float4 u0 = *reinterpret_cast<const float4*>(gjet + (size_t)p * 8);
          const float4 u1 = *reinterpret_cast<const float4*>(gjet + (size_t)p * 8 + 4);
          gv[0] = u0.x; gv[1] = u0.y; gv[2] = u0.z; gv[3] = u0.w;
          gv[4] = u1.x; gv[5] = u1.y; gv[6] = u1.z; gv[7] = u1.w;
        }
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          hw[i] = cvt_bf16x2(gv[2 * i], gv[2 * i + 1]);
          lw[i] = cvt_bf16x2(gv[2 * i] - bf16lo(hw[i]), gv[2 * i + 1] - bf16hi(hw[i]));
        }
        *reinterpret_cast<uint4*>(S.G4 + cofs(r, 0, 16)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(S.G4 + cofs(r, 8, 16)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      // forward: z1 (and e3 = g W4, which needs nothing else), z2, z3
      if (!issue([&] {
            mma_f16(tm, smem_desc(a0, 128, 256), smem_desc(w1f, 128, 256), kId, 0u);
            mma_f16(tm + 192u, smem_desc(g4, 128, 256), smem_desc(w4t_hi, 128, 256), kId, 0u);
            mma_f16(tm + 192u, smem_desc(g4, 128, 256), smem_desc(w4t_lo, 128, 256), kId, 1u);
          })) {
        aborted = true;
        break;
      }
      wait();
      hidden(0);
      if (!issue([&] { gemm64(tm + 64u, smem_u32(S.Hf[0]), smem_u32(S.Wf[0][0]), smem_u32(S.Wf[0][1]), kIdF16); })) {
        aborted = true;
        break;
      }
      wait();
      hidden(1);
      if (!issue([&] { gemm64(tm + 128u, smem_u32(S.Hf[1]), smem_u32(S.Wf[1][0]), smem_u32(S.Wf[1][1]), kIdF16); })) {
        aborted = true;
        break;
      }
      wait();
      hidden(2);
      delta(2);
      // backward: e2 = d3 W3', e1 = d2 W2'
      if (!issue([&] { gemm64(tm + 192u, smem_u32(S.Ds[2]), smem_u32(S.Wt[1][0]), smem_u32(S.Wt[1][1]), kId); })) {
        aborted = true;
        break;
      }
      wait();
      delta(1);
      if (!issue([&] { gemm64(tm + 192u, smem_u32(S.Ds[1]), smem_u32(S.Wt[0][0]), smem_u32(S.Wt[0][1]), kId); })) {
        aborted = true;
        break;
      }
      wait();
      delta(0);
      __syncthreads();  // every tile row written before the weight-gradient MMAs read them
      grad_mma(S, gp0, acc0);
      if (has1) grad_mma(S, gp1, acc1);
      tc_fence_before();
      __syncthreads();  // operands and TMEM free for the next tile
      tc_fence_after();
    }
    aborted = __syncthreads_or(aborted || !ok) != 0;
  }
  float* part = partials + (size_t)blockIdx.x * kFoldedFloats;
  grad_store(gp0, acc0, part, accumulate != 0);
  if (has1) grad_store(gp1, acc1, part, accumulate != 0);
  tc_fence_before();
  __syncthreads();
  if (aborted && tid == 0) (void)mbar_wait(&S.mbar, phase ^ 1u);  // bounded: the last commit before TMEM is freed
  __syncthreads();
  if (warp == 0) tmem_dealloc(S.tmem_base, 256);
}

// Weight gradients: the sum over the CTAs' partials in a fixed order. CTA
// x owns 32 consecutive elements; warp w sums the slots w, w + 8, ... in
// order, then the eight warp sums are added in warp order.
constexpr int kReduceCtas = (kFoldedFloats + 31) / 32;

__global__ void __launch_bounds__(256) k_grad_reduce(const float* __restrict__ partials, int nparts, GradArgs G) {
  __shared__ float wsum[8][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (e < kFoldedFloats) {
#pragma unroll 4
    for (int c = w; c < nparts; c += 8) s += partials[(size_t)c * kFoldedFloats + e];
  }
  wsum[w][lane] = s;
  __syncthreads();
  if (w != 0 || e >= kFoldedFloats) return;
  float t = 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q) t += wsum[q][lane];
  if (e < kOffB1) G.W1[e - kOffW1] = t;
  else if (e < kOffW2) G.b1[e - kOffB1] = t;
  else if (e < kOffB2) G.W2[e - kOffW2] = t;
  else if (e < kOffW3) G.b2[e - kOffB2] = t;
  else if (e < kOffB3) G.W3[e - kOffW3] = t;
  else if (e < kOffW4) G.b3[e - kOffB3] = t;
  else if (e < kOffB4) G.W4[e - kOffW4] = t;
  else G.b4[e - kOffB4] = t;
}

}  // namespace pb
