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
//                  backward through it and the weight gradients on tcgen05,
//                  the latter accumulated in TMEM over all the CTA's tiles
//                  (and summed into the CTA's partial slot over chunks)
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

// Asynchronous 16-byte copies, committed as one group with whatever the
// caller issued before; the caller waits (cp_async_wait_all and a barrier).
template <int PM>
__device__ void stage_bwd(const Particles<PM>& S, const JetArgs& J, const BwdArgs& X, int n, int h0, int hr,
                          unsigned char* buf) {
  const int m = S.m, m16 = round16(m), hb = bwd_head_bytes(m), tb = bwd_tensor_bytes(m);
  const int total = hr * m16 * 8, nthr = blockDim.x;
  for (int idx = threadIdx.x; idx < total; idx += nthr) {
    const int part = idx & 7, j = (idx >> 3) % m16, hh = (idx >> 3) / m16;
    const bool valid = j < m;
    const uint16_t* src = part < 2 ? X.q : (part < 4 ? X.k : (part < 6 ? X.v : X.dout));
    cp_async16(buf + hh * hb + (part >> 1) * tb + j * kKStride * 2 + (part & 1) * 16,
               src + (valid ? qkv_off<PM>(S, J, n, h0 + hh, j) : 0) + (part & 1) * 8, valid ? 16u : 0u);
  }
  cp_async_commit();
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

// The CTA's kHG heads of a jet's bias triangle, copied from the records into
// shared memory (kHG halves per pair): one asynchronous 8-byte copy per pair
// (the record's heads h0 .. h0 + 3), left uncommitted for the next commit.
template <int kHG>
__device__ void stage_bias_heads(const uint4* __restrict__ rec, int npairs, int h0, __half* U) {
  static_assert(kHG == 4, "8-byte pieces of 4 heads");
  const uint32_t u0 = smem_u32(U);
  const char* src0 = reinterpret_cast<const char*>(rec) + h0 * 2;
  for (int p = threadIdx.x; p < npairs; p += blockDim.x)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(u0 + 8u * (uint32_t)p), "l"(src0 + 16 * (size_t)p)
                 : "memory");
}

struct SmemUBias4 {  // the CTA's 4 heads from h0, staged by stage_bias_heads
  const __half* U;
  int h0;
  __device__ __forceinline__ TriBlockS<4> head(int h) const { return TriBlockS<4>{U + (h - h0)}; }
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
      const int tiles = (m + 15) >> 4, npairs = m * (m + 1) / 2;
      // the bias from shared memory when all the CTA's heads and their
      // triangle fit the stage at once, else from the records in L2
      const bool u_smem = HR == kHG && kHG * hb + npairs * kHG * 2 <= kBwdStageBytes;
      __half* Us = reinterpret_cast<__half*>(S.stage + kHG * hb);
      auto pass = [&](const auto& ub) {
        for (int h0 = hg * kHG; h0 < (hg + 1) * kHG; h0 += HR) {
          const int hr = min(HR, (hg + 1) * kHG - h0);
          if (u_smem) stage_bias_heads<kHG>(X.urec + rowbase, npairs, hg * kHG, Us);
          stage_bwd<PM>(S.part, J, X, n, h0, hr, S.stage);
          cp_async_wait_all();
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
      };
      if (in_bounds(hb <= kBwdStageBytes)) {
        if (u_smem) pass(SmemUBias4{Us, hg * kHG});
        else pass(RecordUBias{reinterpret_cast<const __half*>(X.urec + rowbase)});
      }
    }
    // masked rows of every head: dq and dk by the jet's first CTA, dv by its second
    if (hg == 0) {
      zero_masked_rows<PM>(S.part, J, X.dq, n);
      zero_masked_rows<PM>(S.part, J, X.dk, n);
    }
    if (hg == kBwdHeadGroups - 1) zero_masked_rows<PM>(S.part, J, X.dv, n);
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
// 16c + 15 of each 64-wide accumulator), all products on tcgen05:
//   z1 = W1' f + b1', h1 = GELU(z1), z2 = W2' h1 + b2', ... h3
//   e3 = g W4 (issued with z1), d3 = e3 * GELU'(z3), e2 = d3 W3', d2, e1 = d2 W2', d1
//   [dW2' | db2'; dW1' | db1'] += [d2 | d1]^T [f | h1 | 1]
//   [dW3' | db3'; dW4 | db4]   += [d3 | g]^T  [h2 | h3 | 1]
// The recompute multiplies f16 h (two per TMEM column, the A operand read
// from TMEM) by the f16 weights, as the forward kernels do, and adds the
// layer's bias through one more MMA (a TMEM block of ones times [hi b | lo b]);
// the backward products take bf16 d and bf16 hi + lo weights; f, g and the
// folded layer-1 weights and bias enter as bf16 hi + lo terms. The weight
// gradients are two MMAs per tile over the tile's rows (K = 128) with both
// operands read transposed (MN-major) from the same row-major tiles,
// accumulated in fp32 TMEM over all the CTA's tiles; issued behind e1 and
// after the last delta step, they run while the next tile's z1 is staged
// and computed. GELU is the tanh form the forward kernels use; GELU'(z) is
// computed with h and parked in TMEM (f16, in the first half of the
// quarter's z columns, h in the second half) until the backward step needs
// it.

constexpr int kBwdMaxCtas = 256;     // partial-gradient slots in the workspace
constexpr int kFoldedFloats = 9160;  // W1 b1 W2 b2 W3 b3 W4 b4, as pb_fold_affine lays them out
constexpr int kOffW1 = 0, kOffB1 = 256, kOffW2 = 320, kOffB2 = 4416, kOffW3 = 4480, kOffB3 = 8576,
              kOffW4 = 8640, kOffB4 = 9152;

struct GradArgs {
  float *W1, *b1, *W2, *b2, *W3, *b3, *W4, *b4;
};

// Operand tiles of one 128-row tile (bf16, columns as listed; each in the
// canonical no-swizzle layout of cofs with its own width):
//   Z1A [hi f | lo f | hi f | 1 1 0 0]           16 wide: A of z1 (the ones carry b1)
//   G4  [hi g | lo g]                            16 wide: A of e3
//   F1  [hi f | lo f | hi f | 0 | h1 | 1 | 0]    96 wide: B of the first gradient MMA
//   H23 [h2 | h3 | 1 | 0]                       144 wide: B of the second gradient MMA
//   D12 [d1 | d2]                               128 wide: A^T of the first gradient MMA
//   D3G [d3 | hi g | lo g | 0]                  128 wide: A^T of the second gradient MMA
// Z1A and G4 are written at a tile's start; the f and g columns of F1 and D3G
// only once the tile's z1 is done, which in MMA order is after the previous
// tile's gradient MMAs: the next tile never waits for those.
constexpr int kF1W = 96, kH23W = 144, kDW = 128;
constexpr int kF1Ones = 80, kH23Ones = 128, kD3G = 64;
constexpr uint32_t kOnesBf16x2 = 0x3F803F80u;  // bf16 1.0 in both halves

template <int PM>
struct MlpBwdSmem {
  __nv_bfloat16 F1[kTileM * kF1W];
  __nv_bfloat16 H23[kTileM * kH23W];
  __nv_bfloat16 D12[kTileM * kDW];
  __nv_bfloat16 D3G[kTileM * kDW];
  __nv_bfloat16 Z1A[kTileM * 16];
  __nv_bfloat16 G4[kTileM * 16];
  __nv_bfloat16 W1f[64 * 16];        // [hi(W1') | hi(W1') | lo(W1') | hi b1' lo b1' 0 0] per output row
  __half Wf[2][64 * 64];             // W2', W3' as [out][in], f16
  __half Bz[2][64 * 16];             // [hi b | lo b | 0] per output row, f16: b2', b3'
  __nv_bfloat16 Wt[2][2][64 * 64];   // W2'^T, W3'^T as [in][out]: hi, lo
  __nv_bfloat16 W4t[2][64 * 16];     // [W4^T | W4^T] as [in][out]: hi, lo
  uint64_t mbar;                     // the tile's chain of MMAs
  uint64_t mbar_g;                   // the tile's gradient MMAs
  uint32_t tmem_base;
  int stop;  // set by the epilogue warps at a hand-off: the issuer stops
  int n0;    // the CTA's first jet
  Particles<PM> part;
};
// The kernel takes all 512 TMEM columns: one CTA per SM.
static_assert(sizeof(MlpBwdSmem<128>) > 116 * 1024, "k_mlp_bwd must not fit twice on an SM");

// TMEM columns: z1 [0, 64), z2 [64, 128), z3 [128, 192), e3 / e2 / e1
// [192, 256), the gradient accumulators [256, 352) and [352, 496), a block
// of ones [496, 504) (f16: K elements 0 and 1 of every row are 1).
constexpr uint32_t kTmG12 = 256, kTmG3G = 352, kTmOnes = 496, kBwdTmemCols = 512;

// Weights in the canonical K-major layouts of their MMA roles, and the
// constant columns of the operand tiles (ones, zeros). load() issues every
// global load of the thread at once (one round trip); store() converts and
// writes whole 8- or 16-byte pieces of core-matrix rows: Wf rows from float4
// of 4 consecutive inputs, Wt rows (8 consecutive outputs of one input) from
// 8 loads coalesced across the warp's consecutive inputs, W1f and W4t rows
// (16 columns) from one row of W1 or one column of W4. Needs >= 512 threads.
struct BwdWeightLoad {
  static constexpr int kWfJobs = 2 * 1024, kWtJobs = 2 * 512;  // (layer, float4), (layer, input, 8-output block)
  static constexpr int kPer = (kWfJobs + kWtJobs + 511) / 512;
  float v[kPer][8];
  float4 w1;   // threads 0..63: row tid of W1
  float b;      // threads 0..63: b1[tid]; 128..255: b2, b3
  float w4[8];  // threads 64..127: column tid - 64 of W4
  __device__ void load(const MlpArgs& W, int tid, int nthr) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int q = tid + j * nthr;
      if (q < kWfJobs) {
        const float4 x = reinterpret_cast<const float4*>(q < 1024 ? W.W2 : W.W3)[q & 1023];
        v[j][0] = x.x; v[j][1] = x.y; v[j][2] = x.z; v[j][3] = x.w;
      } else if (q < kWfJobs + kWtJobs) {
        const int t = q - kWfJobs, i = t & 63, ob = (t >> 6) & 7;
        const float* Wl = t < 512 ? W.W2 : W.W3;
#pragma unroll
        for (int u = 0; u < 8; ++u) v[j][u] = Wl[(ob * 8 + u) * 64 + i];
      }
    }
    if (tid < 64) {
      w1 = reinterpret_cast<const float4*>(W.W1)[tid];
      b = W.b1[tid];
    }
    if (tid >= 64 && tid < 128) {
#pragma unroll
      for (int u = 0; u < 8; ++u) w4[u] = W.W4[u * 64 + tid - 64];
    }
    if (tid >= 128 && tid < 256) b = (tid < 192 ? W.b2 : W.b3)[tid & 63];
  }
  template <class Smem>
  __device__ void store(Smem& S, int tid, int nthr) const {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int q = tid + j * nthr;
      if (q < kWfJobs) {
        const int L = q >> 10, e = (q & 1023) * 4, o = e >> 6, i = e & 63;
        *reinterpret_cast<uint2*>(&S.Wf[L][cofs(o, i, 64)]) =
            make_uint2(cvt_f16x2(v[j][0], v[j][1]), cvt_f16x2(v[j][2], v[j][3]));
      } else if (q < kWfJobs + kWtJobs) {
        const int t = q - kWfJobs, L = t >> 9, i = t & 63, ob = (t >> 6) & 7;
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          hw[u] = cvt_bf16x2(v[j][2 * u], v[j][2 * u + 1]);
          lw[u] = cvt_bf16x2(v[j][2 * u] - bf16lo(hw[u]), v[j][2 * u + 1] - bf16hi(hw[u]));
        }
        *reinterpret_cast<uint4*>(&S.Wt[L][0][cofs(i, ob * 8, 64)]) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(&S.Wt[L][1][cofs(i, ob * 8, 64)]) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    }
    if (tid < 64) {  // W1f row tid: [hi W1 | hi W1 | lo W1 | hi b1 lo b1 0 0]
      const uint32_t h01 = cvt_bf16x2(w1.x, w1.y), h23 = cvt_bf16x2(w1.z, w1.w);
      const uint32_t l01 = cvt_bf16x2(w1.x - bf16lo(h01), w1.y - bf16hi(h01));
      const uint32_t l23 = cvt_bf16x2(w1.z - bf16lo(h23), w1.w - bf16hi(h23));
      const float bh = bf16lo(cvt_bf16x2(b, 0.f));
      *reinterpret_cast<uint4*>(&S.W1f[cofs(tid, 0, 16)]) = make_uint4(h01, h23, h01, h23);
      *reinterpret_cast<uint4*>(&S.W1f[cofs(tid, 8, 16)]) = make_uint4(l01, l23, cvt_bf16x2(bh, b - bh), 0u);
    }
    if (tid >= 64 && tid < 128) {  // W4t rows (input tid - 64): [W4^T | W4^T], hi and lo
      const int i = tid - 64;
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        hw[u] = cvt_bf16x2(w4[2 * u], w4[2 * u + 1]);
        lw[u] = cvt_bf16x2(w4[2 * u] - bf16lo(hw[u]), w4[2 * u + 1] - bf16hi(hw[u]));
      }
      const uint4 h = make_uint4(hw[0], hw[1], hw[2], hw[3]), l = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      *reinterpret_cast<uint4*>(&S.W4t[0][cofs(i, 0, 16)]) = h;
      *reinterpret_cast<uint4*>(&S.W4t[0][cofs(i, 8, 16)]) = h;
      *reinterpret_cast<uint4*>(&S.W4t[1][cofs(i, 0, 16)]) = l;
      *reinterpret_cast<uint4*>(&S.W4t[1][cofs(i, 8, 16)]) = l;
    }
    if (tid >= 128 && tid < 256) {  // Bz row: [hi b | lo b | 0], f16
      const float bh = __half2float(__float2half_rn(b));
      __half* row = &S.Bz[(tid - 128) >> 6][cofs(tid & 63, 0, 16)];
      *reinterpret_cast<uint4*>(row) = make_uint4(cvt_f16x2(bh, b - bh), 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(&S.Bz[(tid - 128) >> 6][cofs(tid & 63, 8, 16)]) = make_uint4(0u, 0u, 0u, 0u);
    }
    // constant columns, 8 at a time: F1 [80, 96) = 1 1 1 1 1 1 1 1 | 0 ..., H23 [128, 144) alike, D3G [80, 128) = 0
    const uint4 ones = make_uint4(kOnesBf16x2, kOnesBf16x2, kOnesBf16x2, kOnesBf16x2);
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int e = tid; e < kTileM * 10; e += nthr) {
      const int r = e & 127, g = e >> 7;  // g: 0, 1 of F1; 2, 3 of H23; 4..9 of D3G
      if (g < 2) *reinterpret_cast<uint4*>(&S.F1[cofs(r, kF1Ones + 8 * g, kF1W)]) = g == 0 ? ones : zero;
      else if (g < 4) *reinterpret_cast<uint4*>(&S.H23[cofs(r, kH23Ones + 8 * (g - 2), kH23W)]) = g == 2 ? ones : zero;
      else *reinterpret_cast<uint4*>(&S.D3G[cofs(r, kD3G + 16 + 8 * (g - 4), kDW)]) = zero;
    }
  }
};

// GELU(z) = z s and GELU'(z) = s + 2 s (1 - s) z u'(z), with s = sigma(2u) =
// (1 + tanh u) / 2, u = sqrt(2/pi) (z + 0.044715 z^3). s comes from
// exp(-2u) and one reciprocal, so 1 - s and the sech^2 u = 4 s (1 - s) term
// keep their accuracy where tanh saturates (1 - tanh^2 of an approximate
// tanh would not, and its error there is the same for every pair with large
// |u|). For very negative z, exp(-2u) overflows to +inf and s, h and GELU'
// all come out 0, their limits.
__device__ __forceinline__ void gelu_tanh_and_grad(float z, float& h, float& dh) {
  constexpr float kC0 = 0.7978845608028654f, kC1 = 0.044715f;
  constexpr float kA0 = -2.f * kLog2e * kC0, kA1 = kA0 * kC1;  // -2 log2(e) u = z (kA0 + kA1 z^2)
  constexpr float kQ0 = 2.f * kC0, kQ1 = 6.f * kC0 * kC1;      // 2 u'(z) = kQ0 + kQ1 z^2
  const float z2 = z * z;
  const float w = ex2(z * fmaf(kA1, z2, kA0));
  float s;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(s) : "f"(1.f + w));
  h = z * s;
  const float ss = fmaf(-s, s, s);
  dh = fmaf(z * fmaf(kQ1, z2, kQ0), ss, s);
}

// The k-th 16-column quarter of a row's packed f16 pair words, as floats.
__device__ __forceinline__ void unpack_f16x8(const uint32_t* w, float* v) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ void tmem_ld8u_wait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
}

// Instruction descriptor of the weight-gradient MMAs: bf16, M = 128, both
// operands MN-major (the tiles' row index is the contraction index).
__host__ __device__ constexpr uint32_t idesc_bf16_m128_mn(int n) {
  return idesc_bf16_m128(n) | (1u << 15) | (1u << 16);
}

// One 16-column chunk of a gradient accumulator row into the CTA's partial
// (folded layout), staged in shared memory. `lane` is the accumulator row
// (= A^T row), `col` the chunk's first column; the caller's warp holds all 32
// lanes of its quadrant. Every folded element is written exactly once.
struct GradOut {
  float* stage;
  __device__ __forceinline__ void put(int idx, float v) const { stage[idx] = v; }
  // first accumulator: rows 0..63 d1 (W1, b1), rows 64..127 d2 (W2, b2)
  __device__ void g12(int lane, int col, const float* v) const {
    if (lane < 64) {
      if (col == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) put(kOffW1 + lane * 4 + i, v[i] + v[4 + i]);  // hi f + lo f
      } else if (col == kF1Ones) {
        put(kOffB1 + lane, v[0]);
      }
    } else if (col >= 16 && col < 80) {
#pragma unroll
      for (int i = 0; i < 16; ++i) put(kOffW2 + (lane - 64) * 64 + col - 16 + i, v[i]);
    } else if (col == kF1Ones) {
      put(kOffB2 + lane - 64, v[0]);
    }
  }
  // second accumulator: rows 0..63 d3 (W3, b3), rows 64..71 hi g and
  // 72..79 lo g (W4, b4: their sum), rows 80..127 zero
  __device__ void g3g(int lane, int col, float* v) const {
    if (lane >= 64 && lane < 96) {  // one warp: add the lo-g rows to the hi-g rows
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] += __shfl_down_sync(0xffffffffu, v[i], 8);
    }
    if (lane < 64) {
      if (col < 64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) put(kOffW3 + lane * 64 + col + i, v[i]);
      } else if (col == kH23Ones) {
        put(kOffB3 + lane, v[0]);
      }
    } else if (lane < 72) {
      if (col >= 64 && col < 128) {
#pragma unroll
        for (int i = 0; i < 16; ++i) put(kOffW4 + (lane - 64) * 64 + col - 64 + i, v[i]);
      } else if (col == kH23Ones) {
        put(kOffB4 + lane - 64, v[0]);
      }
    }
  }
};

// The T[N] tiles are split evenly over the CTAs (a CTA's range may start and
// end inside a jet); the CTA's weight-gradient partial goes to slot
// blockIdx.x, added to it when `accumulate` (later chunks of a batch).
// Warps 0..15 stage the operands and run the epilogues; warp 16 issues the
// MMAs. Each hand-off is an OR-barrier of the 16 warps (any failed wait
// stops the tile) followed by warp 0's arrive on a barrier the issuer waits
// on; the epilogue warps then wait for the step's commit, so the issuer has
// always taken one hand-off before the next one is offered.
constexpr int kBwdThreads = 544, kBwdIssuer = 16;
constexpr uint32_t kBarHandoff = 1, kBarEpi = 2;
enum BwdStep : int { kStepZ1, kStepZ2, kStepZ3, kStepE2, kStepE1, kStepG12, kBwdSteps };

__device__ __forceinline__ void named_bar_arrive(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int PM>
__global__ void __launch_bounds__(kBwdThreads, 1) k_mlp_bwd(JetArgs J, MlpArgs W, BwdArgs X,
                                                            float* __restrict__ partials, int accumulate) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  MlpBwdSmem<PM>& S = *reinterpret_cast<MlpBwdSmem<PM>*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool issuer = warp == kBwdIssuer;
  const int r = tid & 127, c = (tid >> 7) & 3;  // tile row (TMEM lane) and column quarter (epilogue warps)
  // this CTA's tiles [lo, hi) of the T[N] and the first jet n0 whose tiles
  // reach past lo: T is nondecreasing, so n0 is the least n with
  // T[n + 1] > lo, found by all threads at once (one round trip of loads)
  BwdWeightLoad wl;
  wl.load(W, tid, blockDim.x);  // in flight during the search
  const long long Ttot = X.T[J.N];
  const long long lo = Ttot * blockIdx.x / gridDim.x, hi = Ttot * (blockIdx.x + 1) / gridDim.x;
  if (tid == 0) S.n0 = J.N;
  __syncthreads();
  {
    int first = J.N;
#pragma unroll 4
    for (int i = tid; i < J.N; i += blockDim.x) {  // independent loads, no early exit
      const bool past = X.T[i + 1] > lo;
      first = (past && i < first) ? i : first;
    }
    if (first < J.N) atomicMin(&S.n0, first);
  }
  __syncthreads();
  const int n0 = S.n0;
  if (tid == 32 && lo < hi) prefetch_jet(J, n0);  // into L2 while the weights are converted
  wl.store(S, tid, blockDim.x);
  if (tid == 0) {
    mbar_init(&S.mbar, 1);
    mbar_init(&S.mbar_g, 1);
    fence_mbar_init();
    S.stop = 0;
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, kBwdTmemCols);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = S.tmem_base, lane_off = (uint32_t)((warp & 3) * 32) << 16;
  if (warp < 4) {  // the ones block, every lane: f16 1.0 as K elements 0 and 1
    const uint32_t ones[8] = {0x3C003C00u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    tmem_st8_wait(tm + lane_off + kTmOnes, ones);
  }
  uint32_t phase = 0u, phase_g = 0u;
  bool ok = true, aborted = false, pending = false, any_tile = false;
  bool g_open = false;  // a gradient commit not yet seen complete (its parity: phase_g)

  // ---- issuer (warp 16, lane 0 issues): one hand-off per step
  constexpr uint32_t kId = idesc_bf16_m128(64), kIdF16 = idesc_f16_m128(64);
  constexpr uint32_t kIdG12 = idesc_bf16_m128_mn(kF1W), kIdG3G = idesc_bf16_m128_mn(kH23W);
  constexpr uint32_t kF1Sbo = kF1W / 8 * 128, kH23Sbo = kH23W / 8 * 128, kDSbo = kDW / 8 * 128;
  // z = b + A W, K = 64, A (f16 h) from TMEM (K step j at column 16j + 8 of
  // the layer's 64-column block), the bias through the ones block
  auto gemm_z = [&](uint32_t d, uint32_t a_tm, uint32_t w, uint32_t bz) {
    mma_f16_ta(d, tm + kTmOnes, smem_desc(bz, 128, 256), kIdF16, 0u);
#pragma unroll
    for (int k = 0; k < 4; ++k) mma_f16_ta(d, a_tm + 16u * k + 8u, smem_desc(w + 256u * k, 128, 1024), kIdF16, 1u);
  };
  // D = A (W_hi + W_lo), K = 64, A (bf16 d) from TMEM: the weights' rounding
  // error is the same for every pair row and would not average out of the
  // gradient sums, so they enter as two terms
  auto gemm64_ta = [&](uint32_t d, uint32_t a_tm, uint32_t b_hi, uint32_t b_lo, uint32_t id) {
#pragma unroll
    for (int part = 0; part < 2; ++part)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_f16_ta(d, a_tm + 16u * k + 8u, smem_desc((part ? b_lo : b_hi) + 256u * k, 128, 1024), id,
                   (part | k) != 0 ? 1u : 0u);
  };
  // D += A^T B over the tile's 128 rows (K steps of 16 rows = two 8-row
  // groups); MN-major descriptors: lbo = 8-row group stride, sbo = 8-column
  // group stride. The first tile's first step overwrites.
  auto gemm_grad = [&](uint32_t d, uint32_t a, uint32_t a_rows, uint32_t b, uint32_t b_rows, uint32_t id) {
#pragma unroll
    for (int k = 0; k < kTileM / 16; ++k)
      mma_f16(d, smem_desc(a + 2u * a_rows * k, a_rows, 128), smem_desc(b + 2u * b_rows * k, b_rows, 128), id,
              (any_tile || k != 0) ? 1u : 0u);
  };
  auto issue_step = [&](int step) {
    const uint32_t f1 = smem_u32(S.F1), h23 = smem_u32(S.H23), d12 = smem_u32(S.D12), d3g = smem_u32(S.D3G);
    switch (step) {
      case kStepZ1: {  // z1 = [hi f | lo f | hi f | 1 1] [hi W1 | hi W1 | lo W1 | hi b1 lo b1];
                       // behind it e3 = [hi g | lo g] [W4 | W4]
        mma_f16(tm, smem_desc(smem_u32(S.Z1A), 128, 256), smem_desc(smem_u32(S.W1f), 128, 256), kId, 0u);
        mma_commit(&S.mbar);
        const uint64_t ga = smem_desc(smem_u32(S.G4), 128, 256);
        mma_f16(tm + 192u, ga, smem_desc(smem_u32(S.W4t[0]), 128, 256), kId, 0u);
        mma_f16(tm + 192u, ga, smem_desc(smem_u32(S.W4t[1]), 128, 256), kId, 1u);
        break;
      }
      case kStepZ2:  // its commit also covers e3
        gemm_z(tm + 64u, tm, smem_u32(S.Wf[0]), smem_u32(S.Bz[0]));
        mma_commit(&S.mbar);
        break;
      case kStepZ3:
        gemm_z(tm + 128u, tm + 64u, smem_u32(S.Wf[1]), smem_u32(S.Bz[1]));
        mma_commit(&S.mbar);
        break;
      case kStepE2:  // e2 = d3 W3' (d3 bf16 in TMEM over z3)
        gemm64_ta(tm + 192u, tm + 128u, smem_u32(S.Wt[1][0]), smem_u32(S.Wt[1][1]), kId);
        mma_commit(&S.mbar);
        break;
      case kStepE1:  // e1 = d2 W2', then (not delaying e1) [d3 | g]^T [h2 | h3 | 1]
        gemm64_ta(tm + 192u, tm + 64u, smem_u32(S.Wt[0][0]), smem_u32(S.Wt[0][1]), kId);
        mma_commit(&S.mbar);
        gemm_grad(tm + kTmG3G, d3g, kDSbo, h23, kH23Sbo, kIdG3G);
        break;
      default:  // [d1 | d2]^T [f | h1 | 1]; its commit (on the gradient barrier) also covers the one above
        gemm_grad(tm + kTmG12, d12, kDSbo, f1, kF1Sbo, kIdG12);
        mma_commit(&S.mbar_g);
        break;
    }
  };
  // one tile's steps; false when the epilogue warps stopped
  auto issue_tile = [&]() -> bool {
    for (int step = 0; step < kBwdSteps; ++step) {
      named_bar(kBarHandoff, 64);
      tc_fence_after();
      if (*reinterpret_cast<volatile int*>(&S.stop)) return false;
      if (lane == 0) issue_step(step);
      __syncwarp();
    }
    any_tile = true;
    return true;
  };

  // ---- epilogue warps
  // operand writes published and offered to the issuer; false (for all 16
  // warps) once any of their waits has failed
  auto handoff = [&]() -> bool {
    fence_proxy_async_smem();
    tc_fence_before();
    const bool stop = named_bar_or(kBarEpi, 512, !ok);
    if (warp == 0) {
      if (lane == 0) S.stop = stop ? 1 : 0;
      __syncwarp();
      named_bar_arrive(kBarHandoff, 64);
    }
    return !stop;
  };
  auto wait = [&]() {
    const bool done = mbar_wait(&S.mbar, phase);
    phase ^= 1u;
    ok = ok && done;
    tc_fence_after();
  };
  auto wait_g = [&]() {  // one commit per tile, waited before the next tile's is issued
    const bool done = mbar_wait(&S.mbar_g, phase_g);
    if (done) {
      phase_g ^= 1u;
      g_open = false;
    }
    ok = ok && done;
    tc_fence_after();
  };
  auto store16 = [&](__nv_bfloat16* T, int width, int col, const float* v) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = cvt_bf16x2(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(T + cofs(r, col, width)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(T + cofs(r, col + 8, width)) = make_uint4(w[4], w[5], w[6], w[7]);
  };
  // d (bf16) into the second half of the quarter's TMEM columns of block k:
  // the A operand of the next backward product
  auto d_to_tmem = [&](int k, const float* v) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = cvt_bf16x2(v[2 * i], v[2 * i + 1]);
    tmem_st8_wait(tm + lane_off + 64u * k + 16u * c + 8u, w);
  };
  // z_k (bias included) -> h (bf16 to `T` at column `col`; for k < 2 f16
  // into TMEM as the next layer's A operand) and GELU' (f16 into TMEM, k < 2)
  // or, for k = 2, d3 = e3 GELU'(z3) to D3G and TMEM
  auto hidden = [&](int k, __nv_bfloat16* T, int width, int col) {
    float z[16], h[16];
    const uint32_t ta = tm + lane_off + 64u * k + 16u * c;
    tmem_ld16_wait(ta, z);
#pragma unroll
    for (int i = 0; i < 16; ++i) gelu_tanh_and_grad(z[i], h[i], z[i]);
    store16(T, width, col, h);
    if (k < 2) {
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        w[i] = cvt_f16x2(z[2 * i], z[2 * i + 1]);
        w[8 + i] = cvt_f16x2(h[2 * i], h[2 * i + 1]);
      }
      tmem_st16_wait_u(ta, w);
    } else {
      float e[16];
      tmem_ld16_wait(tm + lane_off + 192u + 16u * c, e);
#pragma unroll
      for (int i = 0; i < 16; ++i) e[i] *= z[i];
      store16(S.D3G, kDW, 16 * c, e);
      d_to_tmem(2, e);
    }
  };
  // d_k = e_k GELU'(z_k) (k = 1, 0) into D12 (and d2 into TMEM)
  auto delta = [&](int k) {
    uint32_t gw[8];
    float gp[16], e[16];
    tmem_ld8u_wait(tm + lane_off + 64u * k + 16u * c, gw);
    tmem_ld16_wait(tm + lane_off + 192u + 16u * c, e);
    unpack_f16x8(gw, gp);
#pragma unroll
    for (int i = 0; i < 16; ++i) e[i] *= gp[i];
    store16(S.D12, kDW, 64 * k + 16 * c, e);
    if (k == 1) d_to_tmem(1, e);
  };
  // tile t's row r as operand words: features (c = 0: [hi f | lo f], [hi f | 0 0])
  // or the gradient record (c = 1: hi g, lo g); zero past the jet's pairs
  auto prep = [&](int t, int m, const float* gjet, uint4& w0, uint4& w1) {
    const int p = t * kTileM + r;
    bool valid = p < m * (m + 1) / 2;
    w0 = make_uint4(0u, 0u, 0u, 0u);
    w1 = w0;
    if (c == 0) {
      int a = 0, b = 0;
      if (valid) {
        TriPairs{}.map(p, a, b);
        valid = in_bounds(a >= 0 && a <= b && b < m);
      }
      float f[4] = {0.f, 0.f, 0.f, 0.f};
      if (valid) pair_feat<PM, true>(S.part, a, b, f);  // the forward MLP's features
      const uint32_t h01 = cvt_bf16x2(f[0], f[1]), h23w = cvt_bf16x2(f[2], f[3]);
      const uint32_t l01 = cvt_bf16x2(f[0] - bf16lo(h01), f[1] - bf16hi(h01));
      const uint32_t l23 = cvt_bf16x2(f[2] - bf16lo(h23w), f[3] - bf16hi(h23w));
      w0 = make_uint4(h01, h23w, l01, l23);
      w1 = make_uint4(h01, h23w, 0u, 0u);
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
      w0 = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      w1 = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  };
  // one tile; false when stopped
  auto epilogue_tile = [&](int t, int t_last, int m, const float* gjet, uint4& w0, uint4& w1, bool& have) -> bool {
    if (!have) prep(t, m, gjet, w0, w1);
    have = false;
    // z1's and e3's operands (the previous tile's z1 and e3 are long done)
    if (c == 0) {
      *reinterpret_cast<uint4*>(S.Z1A + cofs(r, 0, 16)) = w0;
      *reinterpret_cast<uint4*>(S.Z1A + cofs(r, 8, 16)) = make_uint4(w1.x, w1.y, kOnesBf16x2, 0u);
    } else if (c == 1) {
      *reinterpret_cast<uint4*>(S.G4 + cofs(r, 0, 16)) = w0;
      *reinterpret_cast<uint4*>(S.G4 + cofs(r, 8, 16)) = w1;
    }
    if (!handoff()) return false;  // z1, e3
    wait();
    if (pending) {  // the previous tile's gradient MMAs read F1, H23, D12 and D3G (done before z1 was)
      wait_g();
      pending = false;
    }
    if (c == 0) {  // f and g for this tile's gradient MMAs
      *reinterpret_cast<uint4*>(S.F1 + cofs(r, 0, kF1W)) = w0;
      *reinterpret_cast<uint4*>(S.F1 + cofs(r, 8, kF1W)) = w1;
    } else if (c == 1) {
      *reinterpret_cast<uint4*>(S.D3G + cofs(r, kD3G, kDW)) = w0;
      *reinterpret_cast<uint4*>(S.D3G + cofs(r, kD3G + 8, kDW)) = w1;
    }
    hidden(0, S.F1, kF1W, 16 + 16 * c);
    if (!handoff()) return false;  // z2
    wait();
    hidden(1, S.H23, kH23W, 16 * c);
    if (!handoff()) return false;  // z3
    wait();
    hidden(2, S.H23, kH23W, 64 + 16 * c);
    if (!handoff()) return false;  // e2
    if (t + 1 < t_last) {          // the next tile's operand words while e2 runs
      prep(t + 1, m, gjet, w0, w1);
      have = true;
    }
    wait();
    delta(1);
    if (!handoff()) return false;  // e1, then the [d3 | g] gradient
    wait();
    delta(0);
    if (!handoff()) return false;  // the [d1 | d2] gradient
    pending = true;
    g_open = true;
    any_tile = true;
    return true;
  };

  int n = n0;
  uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
  for (; n < J.N && X.T[n] < hi && !aborted; ++n) {
    const long long tj0 = X.T[n], tj1 = X.T[n + 1];
    if (tj1 <= tj0) continue;  // no pairs
    stage_jet<PM>(S.part, J, n);
    if (tid == 32 && X.T[n + 1] < hi) prefetch_jet(J, n + 1);  // this CTA's next jet, if it has one
    const int m = S.part.m;
    const float* gjet = X.grec + (size_t)tj0 * kTileM * 8;
    const int t_first = (int)(max(lo, tj0) - tj0), t_last = (int)(min(hi, tj1) - tj0);
    bool have = false;
    for (int t = t_first; t < t_last && !aborted; ++t)
      aborted = issuer ? !issue_tile() : !epilogue_tile(t, t_last, m, gjet, w0, w1, have);
    aborted = __syncthreads_or(aborted || !ok) != 0;
  }
  if (pending && !aborted) wait_g();
  aborted = __syncthreads_or(aborted || !ok) != 0;
  tc_fence_after();
  any_tile = __syncthreads_or(any_tile) != 0;
  // the accumulators (all-zero when the CTA had no tile) into the partial,
  // through shared memory (the gradient operand tiles, free now) so that the
  // global writes are whole float4 rows
  float* stage = reinterpret_cast<float*>(S.D12);
  static_assert(sizeof(S.D12) + sizeof(S.D3G) >= kFoldedFloats * sizeof(float) &&
                    offsetof(MlpBwdSmem<PM>, D3G) == offsetof(MlpBwdSmem<PM>, D12) + sizeof(S.D12),
                "the staged partial spans D12 and D3G");
  if (!aborted && !issuer) {
    const GradOut go{stage};
    // quarter c reads the 16-column chunks c, c + 4, ... of the 15 (6 + 9)
    for (int q = c; q < (kF1W + kH23W) / 16; q += 4) {
      float v[16];
      const bool g12 = q < kF1W / 16;
      const int col = g12 ? 16 * q : 16 * q - kF1W;
      if (any_tile) {
        tmem_ld16_wait(tm + lane_off + (g12 ? kTmG12 : kTmG3G) + (uint32_t)col, v);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
      if (g12) go.g12(r, col, v); else go.g3g(r, col, v);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (!aborted) {
    float4* part = reinterpret_cast<float4*>(partials + (size_t)blockIdx.x * kFoldedFloats);
    const float4* st4 = reinterpret_cast<const float4*>(stage);
    for (int q = tid; q < kFoldedFloats / 4; q += blockDim.x) {
      float4 v = st4[q];
      if (accumulate) {
        const float4 o = part[q];
        v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
      }
      part[q] = v;
    }
  }
  if (aborted && tid == 0) {  // bounded: the last commits before TMEM is freed
    (void)mbar_wait(&S.mbar, phase ^ 1u);
    if (g_open) (void)mbar_wait(&S.mbar_g, phase_g);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(S.tmem_base, kBwdTmemCols);
}

// Weight gradients: the sum over the CTAs' partials in a fixed order. CTA
// x owns 32 consecutive float4 columns (128 elements); warp w of 16 sums the
// slots w, w + 16, ... in order (all its loads in flight at once), then the
// sixteen warp sums are added in warp order. The folded arrays start at
// multiples of 4 elements, so a column never straddles two of them.
constexpr int kReduceCols = kFoldedFloats / 4;
constexpr int kReduceCtas = (kReduceCols + 31) / 32;
constexpr int kReduceWarps = 16;
static_assert(kBwdMaxCtas <= 16 * kReduceWarps, "one fully unrolled pass over the slots");
static_assert(kFoldedFloats % 4 == 0 && kOffB1 % 4 == 0 && kOffW2 % 4 == 0 && kOffB2 % 4 == 0 &&
                  kOffW3 % 4 == 0 && kOffB3 % 4 == 0 && kOffW4 % 4 == 0 && kOffB4 % 4 == 0,
              "float4 columns of the folded layout");

__global__ void __launch_bounds__(32 * kReduceWarps) k_grad_reduce(const float* __restrict__ partials, int nparts,
                                                                   GradArgs G) {
  __shared__ float4 wsum[kReduceWarps][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int j = blockIdx.x * 32 + lane;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (j < kReduceCols) {
    const float4* P = reinterpret_cast<const float4*>(partials) + j;
    float4 v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = w + i * kReduceWarps;
      v[i] = c < nparts ? P[(size_t)c * kReduceCols] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      s.x += v[i].x; s.y += v[i].y; s.z += v[i].z; s.w += v[i].w;
    }
  }
  wsum[w][lane] = s;
  __syncthreads();
  if (w != 0 || j >= kReduceCols) return;
  float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int q = 0; q < kReduceWarps; ++q) {
    const float4 v = wsum[q][lane];
    t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
  }
  const int e = 4 * j;
  float* dst;
  if (e < kOffB1) dst = G.W1 + (e - kOffW1);
  else if (e < kOffW2) dst = G.b1 + (e - kOffB1);
  else if (e < kOffB2) dst = G.W2 + (e - kOffW2);
  else if (e < kOffW3) dst = G.b2 + (e - kOffB2);
  else if (e < kOffB3) dst = G.W3 + (e - kOffW3);
  else if (e < kOffW4) dst = G.b3 + (e - kOffB3);
  else if (e < kOffB4) dst = G.W4 + (e - kOffW4);
  else dst = G.b4 + (e - kOffB4);
  dst[0] = t.x;
  dst[1] = t.y;
  dst[2] = t.z;
  dst[3] = t.w;
}

}  // namespace pb
