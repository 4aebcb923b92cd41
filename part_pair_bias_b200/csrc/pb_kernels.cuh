// pb_kernels.cuh -- the pair-bias hot path for sm_100a.
//
// Kernels (one launch per C-ABI call):
//   k_pairfeat      features only                      -> feat [N,P,P,4] fp32
//   k_mlp_bias      features + folded MLP (tcgen05)    -> U [N,8,P,P] bf16/fp32
//   k_attn_bias     attention reading a bf16 U from HBM
//   k_fused         features + MLP + attention, the bias kept in shared memory
//
// Sources: "Event Classification with Masked Transformer Autoencoders",
// sections "Fusion 2 -- Pairwise Features + Conv1d MLP -> FusedPairMLP" and
// "Fusion 3 -- Self-Attention + Additive Bias -> Fused Triton Attention".
#pragma once

#include <cuda_bf16.h>
#include <math.h>

#include "pb_device.cuh"

namespace pb {

constexpr float kLnEps = -18.420680743952367f;  // ln(1e-8)
constexpr float kLog2e = 1.4426950408889634f;
constexpr double kPi = 3.14159265358979323846;

struct JetArgs {
  const float *E, *px, *py, *pz;
  const uint8_t* mask;
  const int32_t* ptr;
  int N, P;
  long long tokens;
};

struct MlpArgs {
  const float *W1, *b1, *W2, *b2, *W3, *b3, *W4, *b4;
};

struct QkvArgs {
  const uint16_t *q, *k, *v;
  uint16_t* out;
};

// ============================================================ particle staging

// Valid particles of one jet, compacted in slot order, with the per-particle
// quantities every pair needs. The cancellation-prone ones are fp64:
// rapidity y and azimuth phi (their differences feed dR), and the light-cone
// components E - pz, E + pz and px, py (their sums feed m^2).
template <int PM>
struct Particles {
  double y[PM], phi[PM], wm[PM], wp[PM], px[PM], py[PM];
  float lnpt[PM], pt[PM];
  int16_t slot[PM];  // compact index -> slot (padded) / local token (packed)
  int16_t comp[PM];  // slot -> compact index, -1 if masked or absent
  int warp_cnt[32];
  int m;
  long long base;    // element index of slot 0 of this jet in the momentum arrays
};

// Block-wide; blockDim.x must be a multiple of 32 and >= J.P.
template <int PM>
__device__ void stage_jet(Particles<PM>& S, const JetArgs& J, int n) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  long long base;
  int cnt;
  if (J.ptr) {
    const long long lo = J.ptr[n], hi = J.ptr[n + 1];
    if (lo < 0 || hi < lo || hi > J.tokens || hi - lo > J.P) {
      if (tid == 0) raise_status(kStBadPtr);
      base = 0;
      cnt = 0;
    } else {
      base = lo;
      cnt = (int)(hi - lo);
    }
  } else {
    base = (long long)n * J.P;
    cnt = J.P;
  }
  bool valid = false;
  if (tid < J.P) valid = J.ptr ? (tid < cnt) : (J.mask[base + tid] != 0);
  const unsigned ballot = __ballot_sync(0xffffffffu, valid);
  if (lane == 0) S.warp_cnt[warp] = __popc(ballot);
  __syncthreads();
  int off = 0, total = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    const int c = S.warp_cnt[w];
    off += (w < warp) ? c : 0;
    total += c;
  }
  const int c = off + __popc(ballot & ((1u << lane) - 1u));
  if (tid < J.P) S.comp[tid] = valid ? (int16_t)c : (int16_t)-1;
  if (valid) {
    const long long e = base + tid;
    const double E = J.E[e], px = J.px[e], py = J.py[e], pz = J.pz[e];
    const double wm = E - pz, wp = E + pz;  // exact: differences of fp32 values
    const double pt = sqrt(px * px + py * py);
    S.y[c] = 0.5 * log(wp / wm);
    S.phi[c] = atan2(py, px);
    S.wm[c] = wm;
    S.wp[c] = wp;
    S.px[c] = px;
    S.py[c] = py;
    S.pt[c] = (float)pt;
    S.lnpt[c] = (float)log(pt);
    S.slot[c] = (int16_t)tid;
  }
  if (tid == 0) {
    S.m = total;
    S.base = base;
  }
  __syncthreads();
}

// ============================================================== pair features

// (ln kT, ln z, ln dR, ln m^2) of compact particles a, b. Symmetric by
// construction when called with (min, max). m^2 uses the light-cone form
// (E_s - pz_s)(E_s + pz_s) - px_s^2 - py_s^2 of the pair sum s, in fp64, which
// equals the definition (E_a+E_b)^2 - |p_a+p_b|^2 without its cancellation.
// kFastLog selects the hardware log2 approximation (absolute error ~1e-7 in
// ln); the feature output path uses the accurate logf.
template <bool kFastLog>
__device__ __forceinline__ float flog(float x) {
  return kFastLog ? __logf(x) : logf(x);
}

template <int PM, bool kFastLog = false>
__device__ __forceinline__ void pair_feat(const Particles<PM>& S, int a, int b, float f[4]) {
  const double dy = S.y[a] - S.y[b];
  double dphi = S.phi[a] - S.phi[b];
  if (dphi > kPi) dphi -= 2.0 * kPi;
  else if (dphi <= -kPi) dphi += 2.0 * kPi;
  const float fy = (float)dy, fp = (float)dphi;
  const float dr2 = fmaf(fy, fy, fp * fp);
  const float lndr = 0.5f * flog<kFastLog>(dr2);  // -inf for dR = 0, clamped below
  const float lnptmin = fminf(S.lnpt[a], S.lnpt[b]);
  f[0] = fmaxf(lnptmin + lndr, kLnEps);
  f[1] = fmaxf(lnptmin - flog<kFastLog>(S.pt[a] + S.pt[b]), kLnEps);
  f[2] = fmaxf(lndr, kLnEps);
  const double sx = S.px[a] + S.px[b], sy = S.py[a] + S.py[b];
  const double m2 = fma(S.wm[a] + S.wm[b], S.wp[a] + S.wp[b], -(sx * sx + sy * sy));
  f[3] = m2 > 1e-8 ? flog<kFastLog>((float)m2) : kLnEps;
}

// ----------------------------------------------------- k_pairfeat (features)

template <int PM>
__global__ void __launch_bounds__(256) k_pairfeat(JetArgs J, float* __restrict__ feat) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Particles<PM>& S = *reinterpret_cast<Particles<PM>*>(smem_raw);
  const int P = J.P;
  for (int n = blockIdx.x; n < J.N; n += gridDim.x) {
    stage_jet<PM>(S, J, n);
    float4* out = reinterpret_cast<float4*>(feat) + (size_t)n * P * P;
    for (int idx = threadIdx.x; idx < P * P; idx += blockDim.x) {
      const int ca = S.comp[idx / P], cb = S.comp[idx % P];
      float f[4] = {0.f, 0.f, 0.f, 0.f};
      if (ca >= 0 && cb >= 0) pair_feat<PM>(S, min(ca, cb), max(ca, cb), f);
      out[idx] = make_float4(f[0], f[1], f[2], f[3]);
    }
    __syncthreads();
  }
}

// ================================================================ MLP engine
//
// Numerics of the tensor-core MLP (all exact rescalings are powers of two):
//   layer 1: y1 = W1 f + b1 with f and W1 split into f16 hi + lo parts, the
//            bias through a column of ones, so y1 carries ~22 bits;
//   hidden:  the stored activation is h = y (1 + tanh(a y + b y^3)) = 2 GELU(y)
//            in packed f16x2 (a, b fitted minimax to the erf GELU: max
//            deviation 2.7e-4); the next layer's weights carry the factor 1/2;
//   layers 2..4: f16 operands, fp32 accumulation in TMEM, each bias entering
//            through two constant A columns (1, 1) against (hi(b), lo(b)).

constexpr int kAK = 80;    // A-tile / weight K width: 64 activations + 16 bias columns
constexpr int kSBO = kAK / 8 * 128;  // byte stride between 8-row groups (1280)

// Element index of (row r, column k) of an f16 tile with K columns in the
// tensor-core canonical K-major layout without swizzle: 8x8 core matrices of
// 128 contiguous bytes, K-adjacent core matrices 128 B apart, 8-row groups
// K/8 core matrices apart.
__device__ __forceinline__ int cofs(int r, int k, int K) {
  return (((r >> 3) * (K >> 3) + (k >> 3)) << 6) + ((r & 7) << 3) + (k & 7);
}

template <int NG>
struct MlpSmem {
  __half A[NG][kTileM * kAK];  // per-group activation tile; columns 64, 65 hold 1.0 during a pass
  __half W1[64 * 16];          // [hi(W1) | lo(W1) | hi(W1) | hi(b1) lo(b1) 0 0], K = 16 layout
  __half W2[64 * kAK];         // [W2/2 | hi(b2) lo(b2) 0 ...]
  __half W3[64 * kAK];
  __half W4[16 * kAK];         // rows 8..15 zero (N = 16 MMA)
  uint64_t mbar[NG];
  uint32_t tmem_base;
};

// f16 hi/lo split: x = hi + lo to about 22 bits.
__device__ __forceinline__ void split_half(float x, __half& hi, __half& lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

template <int NG>
__device__ void load_weights(MlpSmem<NG>& S, const MlpArgs& W) {
  for (int i = threadIdx.x; i < 64 * 16; i += blockDim.x) {
    const int n = i >> 4, k = i & 15;
    __half v = __float2half_rn(0.f), hi, lo;
    if (k < 12) {
      split_half(W.W1[n * 4 + (k & 3)], hi, lo);
      v = (k >= 4 && k < 8) ? lo : hi;
    } else if (k < 14) {
      split_half(W.b1[n], hi, lo);
      v = (k == 12) ? hi : lo;
    }
    S.W1[cofs(n, k, 16)] = v;
  }
  // hidden layers: the stored activation is 2 GELU, so the weights carry 1/2
  for (int i = threadIdx.x; i < 64 * kAK; i += blockDim.x) {
    const int n = i / kAK, k = i % kAK;
    __half v2 = __float2half_rn(0.f), v3 = v2, hi, lo;
    if (k < 64) {
      v2 = __float2half_rn(0.5f * W.W2[n * 64 + k]);
      v3 = __float2half_rn(0.5f * W.W3[n * 64 + k]);
    } else if (k < 66) {
      split_half(W.b2[n], hi, lo);
      v2 = (k == 64) ? hi : lo;
      split_half(W.b3[n], hi, lo);
      v3 = (k == 64) ? hi : lo;
    }
    S.W2[cofs(n, k, kAK)] = v2;
    S.W3[cofs(n, k, kAK)] = v3;
  }
  for (int i = threadIdx.x; i < 16 * kAK; i += blockDim.x) {
    const int n = i / kAK, k = i % kAK;
    __half v = __float2half_rn(0.f), hi, lo;
    if (n < 8) {
      if (k < 64) {
        v = __float2half_rn(0.5f * W.W4[n * 64 + k]);
      } else if (k < 66) {
        split_half(W.b4[n], hi, lo);
        v = (k == 64) ? hi : lo;
      }
    }
    S.W4[cofs(n, k, kAK)] = v;
  }
}

// Once per CTA: weights, mbarriers, TMEM (warp 0 allocates NG*64 columns).
template <int NG>
__device__ void mlp_setup(MlpSmem<NG>& S, const MlpArgs& W) {
  load_weights<NG>(S, W);
  if (threadIdx.x == 0) {
    for (int g = 0; g < NG; ++g) mbar_init(&S.mbar[g], 1);
    fence_mbar_init();
  }
  if ((threadIdx.x >> 5) == 0) tmem_alloc(&S.tmem_base, NG * 64);
  fence_proxy_async_smem();  // weight tiles are read by the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

template <int NG>
__device__ void mlp_teardown(MlpSmem<NG>& S, bool aborted, const uint32_t* phase) {
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (aborted && (threadIdx.x & 127) == 0) {
    // A wait that ran out may leave the group's last commit in flight: give it
    // one more bounded wait before the TMEM it writes is released.
    const int g = threadIdx.x >> 7;
    if (g < NG) mbar_wait(&S.mbar[g], phase[0] ^ 1u);
  }
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) tmem_dealloc(S.tmem_base, NG * 64);
}

// 2 GELU(y) for two packed f16 values: y (1 + tanh(y (a + b y^2))).
__device__ __forceinline__ uint32_t gelu2_f16x2(uint32_t y) {
  const uint32_t kA = 0x3A67u * 0x10001u;  // f16 0.80029297 in both halves
  const uint32_t kB = 0x2871u * 0x10001u;  // f16 0.03469849 in both halves
  const uint32_t y2 = hmul2(y, y);
  const uint32_t u = hmul2(y, hfma2(y2, kB, kA));
  return hfma2(y, htanh2(u), y);
}

// Pair enumerations of one MLP pass: row p -> compact particles (a, b).
struct TriPairs {  // unordered pairs a <= b, p = b(b+1)/2 + a
  __device__ __forceinline__ void map(int p, int& a, int& b) const {
    int r = (int)((sqrtf(8.0f * (float)p + 1.0f) - 1.0f) * 0.5f);
    while (r * (r + 1) / 2 > p) --r;
    while ((r + 1) * (r + 2) / 2 <= p) ++r;
    b = r;
    a = p - r * (r + 1) / 2;
  }
};
struct RectPairs {  // ordered pairs (i0 + p / m, p % m): a query block against all keys
  int i0, m;
  __device__ __forceinline__ void map(int p, int& a, int& b) const {
    a = i0 + p / m;
    b = p - (a - i0) * m;
  }
};

// Runs the 4-layer MLP over `npairs` rows in 128-row tiles. Group g (threads
// 128g .. 128g+127) takes tiles g, g+NG, ...; thread row r of a group owns
// TMEM lane r (its warp's lane quadrant). For each valid row the sink gets
// (p, a, b, u[8]). Returns false if the group aborted on a timed-out wait.
template <int PM, int NG, bool kFastLog, class Pairs, class Sink>
__device__ bool mlp_pass(MlpSmem<NG>& S, const Particles<PM>& P, int npairs, const Pairs& pairs,
                         Sink& sink, uint32_t& phase) {
  const int g = threadIdx.x >> 7;
  const int row = threadIdx.x & 127;
  const uint32_t bar_id = 1 + g;
  const bool leader = row == 0;
  const uint32_t t_d = S.tmem_base + (uint32_t)(g * 64);
  const uint32_t t_ld = S.tmem_base + ((uint32_t)(row & 96) << 16) + (uint32_t)(g * 64);
  __half* A = S.A[g];
  const uint32_t a_addr = smem_u32(A);
  const uint32_t w_addr[4] = {smem_u32(S.W1), smem_u32(S.W2), smem_u32(S.W3), smem_u32(S.W4)};
  constexpr uint32_t kId64 = idesc_f16_m128(64), kId16 = idesc_f16_m128(16);
  const int ntiles = (npairs + kTileM - 1) / kTileM;
  bool ok = true;
  // The bias columns of this thread's activation row: (1, 1, 0, ..., 0). They
  // are rewritten on every pass because the tiles double as scratch between
  // passes (the fused kernel stages K and V there).
  *reinterpret_cast<uint4*>(A + cofs(row, 64, kAK)) = make_uint4(0x3C003C00u, 0u, 0u, 0u);
  *reinterpret_cast<uint4*>(A + cofs(row, 72, kAK)) = make_uint4(0u, 0u, 0u, 0u);

  // Publish this thread's operand writes and TMEM reads, meet the group, issue
  // one layer's MMAs from the leader, wait for them to complete.
  auto layer = [&](int L) -> bool {
    fence_proxy_async_smem();
    tc_fence_before();
    if (named_bar_or(bar_id, 128, !ok)) return false;
    if (leader) {
      tc_fence_after();
      if (L == 0) {
        mma_f16(t_d, smem_desc(a_addr, 128, kSBO), smem_desc(w_addr[0], 128, 256), kId64, 0);
      } else {
#pragma unroll
        for (int s = 0; s < kAK / 16; ++s)
          mma_f16(t_d, smem_desc(a_addr + 256u * s, 128, kSBO), smem_desc(w_addr[L] + 256u * s, 128, kSBO),
                  L == 3 ? kId16 : kId64, s > 0 ? 1u : 0u);
      }
      mma_commit(&S.mbar[g]);
    }
    ok = mbar_wait(&S.mbar[g], phase);
    phase ^= 1u;
    tc_fence_after();
    return true;
  };

  // TMEM accumulator row (bias included) -> 2 GELU in f16x2 -> next A tile.
  auto hidden = [&]() {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float v[32];
      tmem_ld32_wait(t_ld + 32u * half, v);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = gelu2_f16x2(cvt_f16x2(v[8 * c + 2 * j], v[8 * c + 2 * j + 1]));
        *reinterpret_cast<uint4*>(A + cofs(row, 32 * half + 8 * c, kAK)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  };

  for (int t = g; t < ntiles; t += NG) {
    const int p = t * kTileM + row;
    const bool valid = p < npairs;
    int a = 0, b = 0;
    float f[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) {
      pairs.map(p, a, b);
      pair_feat<PM, kFastLog>(P, min(a, b), max(a, b), f);
    }
    // layer-1 operand row: [hi(f) | hi(f) | lo(f) | 1 1 0 0] against
    // [hi(W1) | lo(W1) | hi(W1) | hi(b1) lo(b1) 0 0] gives W1 f + b1 to ~22 bits
    {
      __half hi[4], lo[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) split_half(f[i], hi[i], lo[i]);
      const __half one = __float2half_rn(valid ? 1.f : 0.f), zero = __float2half_rn(0.f);
      __half r0[8] = {hi[0], hi[1], hi[2], hi[3], hi[0], hi[1], hi[2], hi[3]};
      __half r1[8] = {lo[0], lo[1], lo[2], lo[3], one, one, zero, zero};
      *reinterpret_cast<uint4*>(A + cofs(row, 0, kAK)) = *reinterpret_cast<uint4*>(r0);
      *reinterpret_cast<uint4*>(A + cofs(row, 8, kAK)) = *reinterpret_cast<uint4*>(r1);
    }
    if (!layer(0)) return false;
    hidden();
    if (!layer(1)) return false;
    hidden();
    if (!layer(2)) return false;
    hidden();
    if (!layer(3)) return false;
    float u[8];
    tmem_ld8_wait(t_ld, u);
    if (valid) sink(p, a, b, u);
  }
  // the TMEM reads of the last tile must finish before anyone reuses it
  tc_fence_before();
  return ok;
}

// ----------------------------------------------- k_mlp_bias (materialised U)

template <int PM, bool F32OUT>
struct GlobalUSink {
  const Particles<PM>* S;
  void* U;
  int n, P;
  __device__ __forceinline__ void operator()(int, int a, int b, const float* u) const {
    const size_t plane = (size_t)P * P;
    const size_t base = (size_t)n * kH * plane;
    const int sa = S->slot[a], sb = S->slot[b];
#pragma unroll
    for (int h = 0; h < kH; ++h) {
      const size_t i0 = base + h * plane + (size_t)sa * P + sb;
      const size_t i1 = base + h * plane + (size_t)sb * P + sa;
      if (F32OUT) {
        static_cast<float*>(U)[i0] = u[h];
        static_cast<float*>(U)[i1] = u[h];
      } else {
        const uint16_t bits = f32_to_bf16(u[h]);
        static_cast<uint16_t*>(U)[i0] = bits;
        static_cast<uint16_t*>(U)[i1] = bits;
      }
    }
  }
};

// Zero every U entry of jet n that has a masked (or absent) end.
template <int PM, bool F32OUT>
__device__ void zero_masked_pairs(const Particles<PM>& S, void* U, int n, int P) {
  const size_t plane = (size_t)P * P;
  for (int idx = threadIdx.x; idx < kH * P * P; idx += blockDim.x) {
    const int b = idx % P, a = (idx / P) % P;
    if (S.comp[a] < 0 || S.comp[b] < 0) {
      const size_t i = (size_t)n * kH * plane + idx;
      if (F32OUT) static_cast<float*>(U)[i] = 0.f;
      else static_cast<uint16_t*>(U)[i] = 0;
    }
  }
}

template <int PM, int NG>
struct MlpBiasSmem {
  MlpSmem<NG> mlp;
  Particles<PM> part;
};

template <int PM, int NG, bool F32OUT>
__global__ void __launch_bounds__(NG * 128) k_mlp_bias(JetArgs J, MlpArgs W, void* __restrict__ U) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  MlpBiasSmem<PM, NG>& S = *reinterpret_cast<MlpBiasSmem<PM, NG>*>(smem_raw);
  mlp_setup<NG>(S.mlp, W);
  uint32_t phase = 0;
  bool aborted = false;
  for (int n = blockIdx.x; n < J.N; n += gridDim.x) {
    stage_jet<PM>(S.part, J, n);
    zero_masked_pairs<PM, F32OUT>(S.part, U, n, J.P);
    const int m = S.part.m;
    GlobalUSink<PM, F32OUT> sink{&S.part, U, n, J.P};
    const bool ok = mlp_pass<PM, NG, true>(S.mlp, S.part, m * (m + 1) / 2, TriPairs{}, sink, phase);
    aborted = __syncthreads_or(!ok) != 0;
    if (aborted) break;
  }
  mlp_teardown<NG>(S.mlp, aborted, &phase);
}

// ========================================================== attention engine

// Element offset of (jet, head h, compact particle c) in Q/K/V/out.
template <int PM>
__device__ __forceinline__ size_t qkv_off(const Particles<PM>& S, const JetArgs& J, int n, int h, int c) {
  if (J.ptr) return ((size_t)(S.base + c) * kH + h) * kD;
  return (((size_t)n * kH + h) * J.P + S.slot[c]) * kD;
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 r, float* f) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 f32x8_to_bf16(const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = (uint32_t)f32_to_bf16(f[2 * i]) | ((uint32_t)f32_to_bf16(f[2 * i + 1]) << 16);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Masked multi-head attention for queries [i_lo, i_hi) of the staged jet,
// all valid keys, on CUDA cores: one thread per (query, head), keys streamed
// from shared memory in chunks of 8 with an online (running-max) softmax in
// the log2 domain. ubias(i, j, h) returns U[h, i, j]. `stage` holds K and V
// of up to `stage_floats / (32 m)` heads at a time as fp32.
template <int PM, class UBias>
__device__ void attention_block(const Particles<PM>& S, const JetArgs& J, const QkvArgs& X, int n, int i_lo,
                                int i_hi, float* stage, int stage_floats, const UBias& ubias) {
  const int m = S.m;
  const int nq = i_hi - i_lo;
  const int tid = threadIdx.x, nthr = blockDim.x;
  if (m <= 0 || nq <= 0) return;
  const int HR = min(kH, stage_floats / (32 * m));
  const float qscale = 0.25f * kLog2e;  // 1/sqrt(D) with D = 16, in log2 units
  for (int h0 = 0; h0 < kH; h0 += HR) {
    const int hr = min(HR, kH - h0);
    for (int idx = tid; idx < hr * m * 4; idx += nthr) {
      const int part = idx & 3, j = (idx >> 2) % m, hh = (idx >> 2) / m;
      const uint16_t* src = (part < 2 ? X.k : X.v) + qkv_off<PM>(S, J, n, h0 + hh, j) + (part & 1) * 8;
      float f[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(src), f);
      float4* dst = reinterpret_cast<float4*>(stage + (hh * m + j) * 32 + (part >> 1) * 16 + (part & 1) * 8);
      dst[0] = make_float4(f[0], f[1], f[2], f[3]);
      dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    __syncthreads();
    for (int item = tid; item < hr * nq; item += nthr) {
      const int hh = item / nq, i = i_lo + item % nq, h = h0 + hh;
      float q[16];
      const uint16_t* qp = X.q + qkv_off<PM>(S, J, n, h, i);
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(qp), q);
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(qp + 8), q + 8);
#pragma unroll
      for (int d = 0; d < 16; ++d) q[d] *= qscale;
      float o[16];
#pragma unroll
      for (int d = 0; d < 16; ++d) o[d] = 0.f;
      float l = 0.f, mx = -INFINITY;
      const float* kv = stage + hh * m * 32;
      for (int j0 = 0; j0 < m; j0 += 8) {
        float s[8];
        float cmax = mx;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = j0 + jj;
          s[jj] = -INFINITY;
          if (j < m) {
            const float4* kr = reinterpret_cast<const float4*>(kv + j * 32);
            float acc = 0.f;
#pragma unroll
            for (int d4 = 0; d4 < 4; ++d4) {
              const float4 k4 = kr[d4];
              acc = fmaf(q[4 * d4], k4.x, acc);
              acc = fmaf(q[4 * d4 + 1], k4.y, acc);
              acc = fmaf(q[4 * d4 + 2], k4.z, acc);
              acc = fmaf(q[4 * d4 + 3], k4.w, acc);
            }
            s[jj] = fmaf(ubias(i, j, h), kLog2e, acc);
            cmax = fmaxf(cmax, s[jj]);
          }
        }
        const float corr = ex2(mx - cmax);
        l *= corr;
#pragma unroll
        for (int d = 0; d < 16; ++d) o[d] *= corr;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = j0 + jj;
          if (j < m) {
            const float pj = ex2(s[jj] - cmax);
            l += pj;
            const float4* vr = reinterpret_cast<const float4*>(kv + j * 32 + 16);
#pragma unroll
            for (int d4 = 0; d4 < 4; ++d4) {
              const float4 v4 = vr[d4];
              o[4 * d4] = fmaf(pj, v4.x, o[4 * d4]);
              o[4 * d4 + 1] = fmaf(pj, v4.y, o[4 * d4 + 1]);
              o[4 * d4 + 2] = fmaf(pj, v4.z, o[4 * d4 + 2]);
              o[4 * d4 + 3] = fmaf(pj, v4.w, o[4 * d4 + 3]);
            }
          }
        }
        mx = cmax;
      }
      const float inv = 1.0f / l;
#pragma unroll
      for (int d = 0; d < 16; ++d) o[d] *= inv;
      uint16_t* op = X.out + qkv_off<PM>(S, J, n, h, i);
      *reinterpret_cast<uint4*>(op) = f32x8_to_bf16(o);
      *reinterpret_cast<uint4*>(op + 8) = f32x8_to_bf16(o + 8);
    }
    __syncthreads();
  }
}

// Masked query rows of a padded jet are 0 (all of them when the jet is empty).
template <int PM>
__device__ void zero_masked_rows(const Particles<PM>& S, const JetArgs& J, uint16_t* out, int n) {
  if (J.ptr) return;
  const int P = J.P;
  for (int idx = threadIdx.x; idx < kH * P * 2; idx += blockDim.x) {
    const int half = idx & 1, s = (idx >> 1) % P, h = (idx >> 1) / P;
    if (S.comp[s] < 0)
      *reinterpret_cast<uint4*>(out + (((size_t)n * kH + h) * P + s) * kD + half * 8) = make_uint4(0, 0, 0, 0);
  }
}

// ------------------------------------------- k_attn_bias (bias read from HBM)

template <int PM>
struct GlobalUBias {
  const Particles<PM>* S;
  const uint16_t* U;
  int n, P;
  __device__ __forceinline__ float operator()(int i, int j, int h) const {
    return bf16_to_f32(U[(((size_t)n * kH + h) * P + S->slot[i]) * P + S->slot[j]]);
  }
};

constexpr int kAttnStageFloats = 16384;  // 64 KB of K/V staging

template <int PM>
struct AttnSmem {
  float stage[kAttnStageFloats];
  Particles<PM> part;
};

template <int PM>
__global__ void __launch_bounds__(256) k_attn_bias(JetArgs J, QkvArgs X, const uint16_t* __restrict__ U) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  AttnSmem<PM>& S = *reinterpret_cast<AttnSmem<PM>*>(smem_raw);
  for (int n = blockIdx.x; n < J.N; n += gridDim.x) {
    stage_jet<PM>(S.part, J, n);
    GlobalUBias<PM> ub{&S.part, U, n, J.P};
    attention_block<PM>(S.part, J, X, n, 0, S.part.m, S.stage, kAttnStageFloats, ub);
    zero_masked_rows<PM>(S.part, J, X.out, n);
    __syncthreads();
  }
}

// ======================================================= k_fused (one pass)

// The bias of the jet's pairs lives in shared memory as 8 f16 (one per head)
// per pair: the whole upper triangle when it fits (UCap pairs), otherwise one
// query block against all keys at a time. UCap is what is left of the
// per-CTA shared memory after the MLP tiles and the particles.
constexpr int kSmemLimit = 232448;  // 227 KB per CTA on sm_100

template <int PM, int NG>
struct FusedLayout {
  static constexpr int kFixed = (int)(sizeof(MlpSmem<NG>) + sizeof(Particles<PM>)) + 1024;
  static constexpr int kUCap = (kSmemLimit - kFixed) / 16;
};

struct SmemUSink {
  uint4* U8;
  __device__ __forceinline__ void operator()(int p, int, int, const float* u) const {
    U8[p] = make_uint4(pack_half2(u[0], u[1]), pack_half2(u[2], u[3]), pack_half2(u[4], u[5]),
                       pack_half2(u[6], u[7]));
  }
};

struct TriUBias {  // U of pair (i, j) at index max(i,j)(max(i,j)+1)/2 + min(i,j)
  const __half* U;
  __device__ __forceinline__ float operator()(int i, int j, int h) const {
    const int hi = max(i, j), lo = min(i, j);
    return __half2float(U[(hi * (hi + 1) / 2 + lo) * 8 + h]);
  }
};

struct RectUBias {  // U of (query i, key j) at index (i - i0) * m + j
  const __half* U;
  int i0, m;
  __device__ __forceinline__ float operator()(int i, int j, int h) const {
    return __half2float(U[((i - i0) * m + j) * 8 + h]);
  }
};

template <int PM, int NG>
struct FusedSmem {
  MlpSmem<NG> mlp;
  Particles<PM> part;
  uint4 U8[FusedLayout<PM, NG>::kUCap];
};

template <int PM, int NG>
__global__ void __launch_bounds__(NG * 128) k_fused(JetArgs J, MlpArgs W, QkvArgs X) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  FusedSmem<PM, NG>& S = *reinterpret_cast<FusedSmem<PM, NG>*>(smem_raw);
  mlp_setup<NG>(S.mlp, W);
  // during attention the activation tiles hold K and V
  float* stage = reinterpret_cast<float*>(&S.mlp.A[0][0]);
  constexpr int kStageFloats = NG * kTileM * kAK / 2;
  constexpr int kUCap = FusedLayout<PM, NG>::kUCap;
  uint32_t phase = 0;
  bool aborted = false;
  for (int n = blockIdx.x; n < J.N && !aborted; n += gridDim.x) {
    stage_jet<PM>(S.part, J, n);
    const int m = S.part.m;
    SmemUSink sink{S.U8};
    if (m * (m + 1) / 2 <= kUCap) {
      const bool ok = mlp_pass<PM, NG, true>(S.mlp, S.part, m * (m + 1) / 2, TriPairs{}, sink, phase);
      aborted = __syncthreads_or(!ok) != 0;
      if (aborted) break;
      TriUBias ub{reinterpret_cast<const __half*>(S.U8)};
      attention_block<PM>(S.part, J, X, n, 0, m, stage, kStageFloats, ub);
    } else {
      const int qb = kUCap / m;
      for (int i0 = 0; i0 < m; i0 += qb) {
        const int i1 = min(m, i0 + qb);
        const bool ok = mlp_pass<PM, NG, true>(S.mlp, S.part, (i1 - i0) * m, RectPairs{i0, m}, sink, phase);
        aborted = __syncthreads_or(!ok) != 0;
        if (aborted) break;
        RectUBias ub{reinterpret_cast<const __half*>(S.U8), i0, m};
        attention_block<PM>(S.part, J, X, n, i0, i1, stage, kStageFloats, ub);
      }
      if (aborted) break;
    }
    zero_masked_rows<PM>(S.part, J, X.out, n);
    __syncthreads();
  }
  mlp_teardown<NG>(S.mlp, aborted, &phase);
}

}  // namespace pb
