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

#include <type_traits>

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

// The MLP with int8 inputs to layers 2..4: layer 1 as MlpArgs (fp32,
// folded); layers 2..4 as int8 weight codes T (row-major [out][in]), one
// fp32 scale alpha per output row (W' = alpha T) and the folded fp32 bias.
struct MlpI8Args {
  const float *W1, *b1;
  const int8_t *T2, *T3, *T4;
  const float *a2, *a3, *a4;
  const float *b2, *b3, *b4;
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

// Stage jets into shared memory: the valid particles get compact indices in
// slot order and, with kKin, their fp64 kinematics (the attention needs only
// m, base and the slot map). Groups of ceil(P/32) warps take one jet each, as
// many jets at a time as the block holds groups; jet_of(k) is the jet of ring
// entry k. Block-wide; blockDim.x must be a multiple of 32 and >= J.P.
template <int PM, bool kKin, class JetOf>
__device__ void stage_jets(Particles<PM>* ring, const JetArgs& J, int K, const JetOf& jet_of) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wpj = (J.P + 31) >> 5;                   // warps per jet
  const int per = (int)(blockDim.x >> 5) / wpj;      // jets staged at once
  const int g = warp / wpj, lw = warp - g * wpj, t = lw * 32 + lane;
  for (int k0 = 0; k0 < K; k0 += per) {
    const int k = k0 + g;
    const bool act = g < per && k < K;
    Particles<PM>& S = ring[act ? k : 0];
    long long base = 0;
    int cnt = 0;
    bool valid = false;
    float fE = 0.f, fx = 0.f, fy = 0.f, fz = 0.f;  // loaded with the mask: one round trip
    if (act) {
      const int n = jet_of(k);
      if (J.ptr) {
        const long long lo = J.ptr[n], hi = J.ptr[n + 1];
        if (lo < 0 || hi < lo || hi > J.tokens || hi - lo > J.P) {
          if (t == 0) raise_status(kStBadPtr);
        } else {
          base = lo;
          cnt = (int)(hi - lo);
        }
      } else {
        base = (long long)n * J.P;
        cnt = J.P;
      }
      if (t < J.P) {
        valid = J.ptr ? (t < cnt) : (J.mask[base + t] != 0);
        if (kKin && t < cnt) {
          const long long e = base + t;
          fE = J.E[e];
          fx = J.px[e];
          fy = J.py[e];
          fz = J.pz[e];
        }
      }
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, valid);
    if (act && lane == 0) S.warp_cnt[lw] = __popc(ballot);
    __syncthreads();
    if (act) {
      int off = 0, total = 0;
      for (int w = 0; w < wpj; ++w) {
        const int c = S.warp_cnt[w];
        off += (w < lw) ? c : 0;
        total += c;
      }
      const int c = off + __popc(ballot & ((1u << lane) - 1u));
      if (t < J.P) S.comp[t] = valid ? (int16_t)c : (int16_t)-1;
      if (valid) {
        S.slot[c] = (int16_t)t;
        if (kKin) {
          const double E = fE, px = fx, py = fy, pz = fz;
          const double wm = E - pz, wp = E + pz;  // exact: differences of fp32 values
          const double pt = sqrt(px * px + py * py);
          S.y[c] = 0.5 * log(wp / wm);
          S.phi[c] = atan2(py, px);
          S.wm[c] = wm;
          S.wp[c] = wp;
          S.px[c] = px;
          S.py[c] = py;
          S.pt[c] = (float)pt;
          S.lnpt[c] = logf((float)pt);
        }
      }
      if (t == 0) {
        S.m = total;
        S.base = base;
      }
    }
    __syncthreads();
  }
}

// Prefetch jet n's momenta (and mask) rows into L2 ahead of stage_jet. One
// thread; only rows that are 16-byte aligned and whole (16-byte aligned
// arrays, padded rows of P % 4 == 0 floats, masks of P % 16 == 0 bytes;
// packed jets need their ptr entries, so they are left alone).
__device__ __forceinline__ void prefetch_jet(const JetArgs& J, int n) {
  if (J.ptr || n >= J.N || (J.P & 3) != 0) return;
  if (((reinterpret_cast<uintptr_t>(J.E) | reinterpret_cast<uintptr_t>(J.px) | reinterpret_cast<uintptr_t>(J.py) |
        reinterpret_cast<uintptr_t>(J.pz)) & 15) != 0)
    return;
  const size_t e = (size_t)n * J.P;
  const uint32_t bytes = (uint32_t)J.P * 4;
  prefetch_l2(J.E + e, bytes);
  prefetch_l2(J.px + e, bytes);
  prefetch_l2(J.py + e, bytes);
  prefetch_l2(J.pz + e, bytes);
  if ((J.P & 15) == 0 && (reinterpret_cast<uintptr_t>(J.mask) & 15) == 0) prefetch_l2(J.mask + e, (uint32_t)J.P);
}

// One jet with the whole block (thread = slot); same result as stage_jets.
template <int PM, bool kKin = true>
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
  float fE = 0.f, fx = 0.f, fy = 0.f, fz = 0.f;  // loaded with the mask: one round trip
  if (tid < J.P) {
    valid = J.ptr ? (tid < cnt) : (J.mask[base + tid] != 0);
    if (kKin && tid < cnt) {
      const long long e = base + tid;
      fE = J.E[e];
      fx = J.px[e];
      fy = J.py[e];
      fz = J.pz[e];
    }
  }
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
    S.slot[c] = (int16_t)tid;
    if (kKin) {
      const double E = fE, px = fx, py = fy, pz = fz;
      const double wm = E - pz, wp = E + pz;  // exact: differences of fp32 values
      const double pt = sqrt(px * px + py * py);
      S.y[c] = 0.5 * log(wp / wm);
      S.phi[c] = atan2(py, px);
      S.wm[c] = wm;
      S.wp[c] = wp;
      S.px[c] = px;
      S.py[c] = py;
      S.pt[c] = (float)pt;
      S.lnpt[c] = logf((float)pt);
    }
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
//   hidden:  layers 1..3 accumulate in f16 in TMEM (the row is read back as
//            packed f16x2, so no conversion is needed) and are activated on
//            two pipes: 5 of every 8 columns with the tanh
//            form h = y (1 + tanh(a y + b y^3)) = 2 GELU(y) (one MUFU op per
//            two values; a, b fitted minimax to the erf GELU, max deviation
//            2.7e-4), the other 3 with h = relu(y) + s q(s), s = min(|y|, 3.5),
//            q a degree-6 polynomial fitted to GELU - relu (f16 evaluation,
//            max deviation 4.8e-3), on the FMA pipe only. The next layer's
//            weights carry 1/2 on the tanh columns;
//   layers 2..4: f16 operands; layer 4 accumulates in fp32; each bias enters
//            through an extra K step: a constant column block of ones times
//            the weights' (hi(b), lo(b)) columns.
// Data flow: every operand A of the four layers lives in tensor memory. A
// tile group's 128-column TMEM slot holds its accumulator D (64 columns) and
// its A operand (40 columns: 64 f16 activations two per column, then the
// ones block); the epilogue reads D with tcgen05.ld and writes the activated
// row back with tcgen05.st, and the MMAs read A from TMEM and only the
// weights (B) from shared memory. An N = 64 MMA whose A and B both came from
// shared memory would move 6 KB through it, 48 clk at 128 B/clk, against
// 32 clk of tensor math; with A in TMEM it moves 2 KB.

constexpr int kAK = 64;              // activation tile width
constexpr int kWK = 80;              // weight K width: 64 activations + 16 bias columns
constexpr int kASBO = kAK / 8 * 128;   // 8-row group stride of an activation tile (1024 B)
constexpr int kWSBO = kWK / 8 * 128;   // 8-row group stride of a weight tile (1280 B)
constexpr int kTanhChunks = 5;       // of the 8 eight-column chunks of a hidden layer

// Element index of (row r, column k) of an f16 tile with K columns in the
// tensor-core canonical K-major layout without swizzle: 8x8 core matrices of
// 128 contiguous bytes, K-adjacent core matrices 128 B apart, 8-row groups
// K/8 core matrices apart.
__device__ __forceinline__ int cofs(int r, int k, int K) {
  return (((r >> 3) * (K >> 3) + (k >> 3)) << 6) + ((r & 7) << 3) + (k & 7);
}

// NG tile groups of 128 threads; each group keeps SL tiles in flight (slots
// SL*g .. SL*g+SL-1), so one tile's epilogue overlaps another's MMAs.
template <int NG, int SL>
struct MlpSmem {
  __half A[NG * SL][kTileM * kAK];  // per-slot activation tile (layer 1 uses its first 16 columns)
  __half Ones[kTileM * 16];         // [1 1 0 ... 0] per row: the bias K step
  __half W1[64 * 16];               // [hi(W1) | lo(W1) | hi(W1) | hi(b1) lo(b1) 0 0], K = 16 layout
  __half W2[64 * kWK];              // [W2 scaled per column | hi(b2) lo(b2) 0 ...]
  __half W3[64 * kWK];
  __half W4[16 * kWK];              // rows 8..15 zero (N = 16 MMA)
  uint64_t mbar[NG * SL];
  uint32_t tmem_base;
};

// TMEM of the MLP: one 128-column slot per tile group (D at +0, A at +64,
// the ones block of the bias K step at +96); the SL activation tiles of
// MlpSmem are not used by the MLP and serve the kernels as staging space.
constexpr int kSlotCols = 128;
constexpr int kSlotA = 64;
constexpr int kSlotOnes = kSlotA + 32;
__host__ __device__ constexpr int kTmemCols(int ng, int) { return ng * kSlotCols; }

// f16 hi/lo split: x = hi + lo to about 22 bits.
__device__ __forceinline__ void split_half(float x, __half& hi, __half& lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

__device__ __forceinline__ uint32_t h2bits(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// Scale of input column k of layers 2..4: the tanh columns hold 2 GELU.
__device__ __forceinline__ float act_scale(int k) { return (k >> 3) < kTanhChunks ? 0.5f : 1.0f; }

// The folded weights of one thread's share, held in registers between the
// global loads and the shared-memory stores, so that other latency (the
// first jet's staging, the jet table) can overlap the loads.
struct WeightRegs {
  static constexpr int kPer = (2 * 1024 + 255) / 256;  // float4 loads of W2 and W3 per thread (>= 256 threads)
  float4 w[kPer], w4, w1;
  float bias1, bias2, bias3, bias4;
  // Threads tid = 0 .. nthr - 1 of the loading set (by default the block).
  __device__ void load(const MlpArgs& W) { load(W, threadIdx.x, blockDim.x); }
  __device__ void load(const MlpArgs& W, int tid, int nthr) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int q = tid + j * nthr;
      w[j] = q < 2048 ? reinterpret_cast<const float4*>(q < 1024 ? W.W2 : W.W3)[q & 1023] : make_float4(0, 0, 0, 0);
    }
    w4 = tid < 128 ? reinterpret_cast<const float4*>(W.W4)[tid] : make_float4(0, 0, 0, 0);
    w1 = tid < 64 ? reinterpret_cast<const float4*>(W.W1)[tid] : make_float4(0, 0, 0, 0);
    bias1 = tid < 64 ? W.b1[tid] : 0.f;
    bias2 = tid < 64 ? W.b2[tid] : 0.f;
    bias3 = tid < 64 ? W.b3[tid] : 0.f;
    bias4 = tid < 8 ? W.b4[tid] : 0.f;
  }
};

// Weight tiles in the canonical layout, from the registers of WeightRegs
// (loaded by the same set of threads tid = 0 .. nthr - 1).
template <int NG, int SL>
__device__ void store_weights(MlpSmem<NG, SL>& S, const WeightRegs& R, int tid, int nthr) {
#pragma unroll
  for (int j = 0; j < WeightRegs::kPer; ++j) {
    const int q = tid + j * nthr;
    if (q < 2048) {
      const int e = (q & 1023) * 4, n = e >> 6, k = e & 63;  // 4 consecutive k of one chunk
      const float sc = act_scale(k);
      __half* dst = (q < 1024 ? S.W2 : S.W3) + cofs(n, k, kWK);
      reinterpret_cast<uint2*>(dst)[0] =
          make_uint2(h2bits(__float2half_rn(sc * R.w[j].x), __float2half_rn(sc * R.w[j].y)),
                     h2bits(__float2half_rn(sc * R.w[j].z), __float2half_rn(sc * R.w[j].w)));
    }
  }
  if (tid < 128) {  // W4 rows 0..7, zero rows 8..15
    const int e = tid * 4, n = e >> 6, k = e & 63;
    const float sc = act_scale(k);
    reinterpret_cast<uint2*>(S.W4 + cofs(n, k, kWK))[0] =
        make_uint2(h2bits(__float2half_rn(sc * R.w4.x), __float2half_rn(sc * R.w4.y)),
                   h2bits(__float2half_rn(sc * R.w4.z), __float2half_rn(sc * R.w4.w)));
    reinterpret_cast<uint2*>(S.W4 + cofs(8 + n, k, kWK))[0] = make_uint2(0u, 0u);
  }
  if (tid < 64) {  // layer-1 row n = tid, and the bias columns of W2, W3, W4
    const int n = tid;
    __half h[4], l[4], bh, bl;
    split_half(R.w1.x, h[0], l[0]);
    split_half(R.w1.y, h[1], l[1]);
    split_half(R.w1.z, h[2], l[2]);
    split_half(R.w1.w, h[3], l[3]);
    split_half(R.bias1, bh, bl);
    const __half z = __float2half_rn(0.f);
    *reinterpret_cast<uint4*>(S.W1 + cofs(n, 0, 16)) =
        make_uint4(h2bits(h[0], h[1]), h2bits(h[2], h[3]), h2bits(l[0], l[1]), h2bits(l[2], l[3]));
    *reinterpret_cast<uint4*>(S.W1 + cofs(n, 8, 16)) =
        make_uint4(h2bits(h[0], h[1]), h2bits(h[2], h[3]), h2bits(bh, bl), h2bits(z, z));
    split_half(R.bias2, bh, bl);
    *reinterpret_cast<uint4*>(S.W2 + cofs(n, 64, kWK)) = make_uint4(h2bits(bh, bl), 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(S.W2 + cofs(n, 72, kWK)) = make_uint4(0u, 0u, 0u, 0u);
    split_half(R.bias3, bh, bl);
    *reinterpret_cast<uint4*>(S.W3 + cofs(n, 64, kWK)) = make_uint4(h2bits(bh, bl), 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(S.W3 + cofs(n, 72, kWK)) = make_uint4(0u, 0u, 0u, 0u);
    if (n < 16) {  // thread n < 8 holds b4[n]; rows 8..15 get zeros
      split_half(n < 8 ? R.bias4 : 0.f, bh, bl);
      *reinterpret_cast<uint4*>(S.W4 + cofs(n, 64, kWK)) = make_uint4(h2bits(bh, bl), 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(S.W4 + cofs(n, 72, kWK)) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  for (int r = tid; r < kTileM; r += nthr) {
    *reinterpret_cast<uint4*>(S.Ones + cofs(r, 0, 16)) = make_uint4(0x3C003C00u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(S.Ones + cofs(r, 8, 16)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Once per CTA: weights (loaded into R beforehand), mbarriers, TMEM (warp 0
// allocates NG*SL*64 columns).
template <int NG, int SL>
__device__ void mlp_setup(MlpSmem<NG, SL>& S, const WeightRegs& R) {
  store_weights<NG, SL>(S, R, threadIdx.x, blockDim.x);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NG * SL; ++i) mbar_init(&S.mbar[i], 1);
    fence_mbar_init();
  }
  if ((threadIdx.x >> 5) == 0) tmem_alloc(&S.tmem_base, kTmemCols(NG, SL));
  fence_proxy_async_smem();  // weight tiles are read by the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// The part of mlp_setup that threads tid = 0 .. nthr - 1 of warps 1 and up
// do while warp 0 is busy elsewhere (the set's first thread initialises the
// mbarriers). Warp 0 then allocates the TMEM (it also frees it in
// mlp_teardown) and the caller completes the set-up with tc_fence_before, a
// block barrier and tc_fence_after.
template <int NG, int SL>
__device__ void mlp_setup_part(MlpSmem<NG, SL>& S, const WeightRegs& R, int tid, int nthr) {
  store_weights<NG, SL>(S, R, tid, nthr);
  if (tid == 0) {
    for (int i = 0; i < NG * SL; ++i) mbar_init(&S.mbar[i], 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();  // weight tiles are read by the tensor cores
}

template <int NG, int SL>
__device__ void mlp_setup(MlpSmem<NG, SL>& S, const MlpArgs& W) {
  WeightRegs R;
  R.load(W);
  mlp_setup<NG, SL>(S, R);
}

template <int NG, int SL>
__device__ void mlp_teardown(MlpSmem<NG, SL>& S, bool aborted, const uint32_t* phase) {
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (aborted && (threadIdx.x & 127) == 0) {
    // A wait that ran out may leave the group's last commit in flight: give
    // it one more bounded wait before the TMEM it writes is released.
    const int g = threadIdx.x >> 7;
    if (g < NG) mbar_wait(&S.mbar[g], (*phase & 1u) ^ 1u);
  }
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) tmem_dealloc(S.tmem_base, kTmemCols(NG, SL));
}

// 2 GELU(y) for two packed f16 values: y (1 + tanh(y (a + b y^2))).
__device__ __forceinline__ uint32_t gelu2_f16x2(uint32_t y) {
  const uint32_t kA = 0x3A67u * 0x10001u;  // f16 0.80029297 in both halves
  const uint32_t kB = 0x2871u * 0x10001u;  // f16 0.03469849 in both halves
  const uint32_t y2 = hmul2(y, y);
  const uint32_t u = hmul2(y, hfma2(y2, kB, kA));
  return hfma2(y, htanh2(u), y);
}

// GELU(y) for two packed f16 values on the FMA pipe only:
// relu(y) + s q(s), s = min(|y|, 3.5), q(s) = c1 + c2 s + ... + c6 s^5.
__device__ __forceinline__ uint32_t gelu_poly_f16x2(uint32_t y) {
  uint32_t s, r;
  asm("and.b32 %0, %1, 0x7FFF7FFF;" : "=r"(s) : "r"(y));
  asm("min.f16x2 %0, %1, %2;" : "=r"(s) : "r"(s), "r"(0x43004300u));
  asm("max.f16x2 %0, %1, %2;" : "=r"(r) : "r"(y), "r"(0u));
  uint32_t q = hfma2(0x98779877u, s, 0x25652565u);  // c6 s + c5
  q = hfma2(q, s, 0xAB11AB11u);                     // + c4
  q = hfma2(q, s, 0xAB4AAB4Au);                     // + c3
  q = hfma2(q, s, 0x371E371Eu);                     // + c2
  q = hfma2(q, s, 0xB814B814u);                     // + c1
  return hfma2(q, s, r);
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

// Runs the 4-layer MLP over the source's rows in 128-row tiles. Group g
// (threads 128g .. 128g+127) takes tiles g, g+NG, ... one at a time through
// its TMEM slot; thread row r of a group owns TMEM lane r. The groups run
// independently, so one group's epilogue overlaps the others' MMAs. For each
// valid row the sink gets (p, a, b, u[8]). Bit 0 of *phase tracks the
// group's mbarrier parity. Returns false if the group aborted on a timed-out
// wait.
// A source of MLP rows for one pass: ntiles() tiles; row(t, r, ...) gives
// the features of row r of tile t and the (p, a, b) its sink receives, or
// false for a padding row.
template <int PM, class Pairs, bool kFastLog>
struct JetTiles {  // the pairs of one staged jet
  const Particles<PM>* P;
  int npairs;
  Pairs pairs;
  __device__ __forceinline__ int ntiles() const { return (npairs + kTileM - 1) / kTileM; }
  __device__ __forceinline__ bool row(int t, int r, int& p, int& a, int& b, float f[4]) const {
    p = t * kTileM + r;
    if (p >= npairs) return false;
    pairs.map(p, a, b);
    if (!in_bounds(a >= 0 && b >= 0 && a < P->m && b < P->m)) return false;
    pair_feat<PM, kFastLog>(*P, min(a, b), max(a, b), f);
    return true;
  }
};

template <int NG, int SL, class Source, class Sink>
__device__ bool mlp_pass(MlpSmem<NG, SL>& S, const Source& src, Sink& sink, uint32_t* phase) {
  const int g = threadIdx.x >> 7;
  if (g >= NG) return true;  // threads past the MLP's groups take no tiles
  const int row = threadIdx.x & 127;
  const uint32_t bar_id = 1 + g;
  const bool leader = row == 0;
  const uint32_t w_addr[4] = {smem_u32(S.W1), smem_u32(S.W2), smem_u32(S.W3), smem_u32(S.W4)};
  // layers 1..3 accumulate in f16 (read back packed, no conversion), layer 4 in fp32
  constexpr uint32_t kId64 = idesc_f16_m128(64, false), kId16 = idesc_f16_m128(16, true);
  const int ntiles = src.ntiles();
  uint64_t* const mbar = &S.mbar[g];
  const uint32_t lane_off = (uint32_t)(row & 96) << 16;
  const uint32_t t_d = S.tmem_base + (uint32_t)(g * kSlotCols);  // accumulator, 64 columns
  const uint32_t t_a = t_d + kSlotA;                             // A operand, 40 columns
  bool ok = true;

  // Publish this thread's TMEM stores and reads, meet the group and have the
  // leader issue layer L; its completion arrives on the group's mbarrier.
  auto issue = [&](int L) -> bool {
    tc_fence_before();
    if (named_bar_or(bar_id, 128, !ok)) return false;
    if (leader) {
      tc_fence_after();
      if (L == 0) {
        mma_f16_ta(t_d, t_a, smem_desc(w_addr[0], 128, 256), kId64, 0u);
      } else {
        const uint32_t w = L == 1 ? w_addr[1] : (L == 2 ? w_addr[2] : w_addr[3]);
        const uint32_t id = L == 3 ? kId16 : kId64;
        // bias step first (initialises the accumulator), then the 64 activations
        mma_f16_ta(t_d, t_d + kSlotOnes, smem_desc(w + 1024u, 128, kWSBO), id, 0u);
#pragma unroll
        for (int k = 0; k < kAK / 16; ++k)
          mma_f16_ta(t_d, t_a + 8u * k, smem_desc(w + 256u * k, 128, kWSBO), id, 1u);
      }
      mma_commit(mbar);
    }
    return true;
  };
  auto wait = [&]() {
    const bool done = mbar_wait(mbar, *phase & 1u);
    ok = ok && done;
    *phase ^= 1u;
    tc_fence_after();
  };

  // The ones block of the bias K step, [1 1 0 ... 0] per row (K columns
  // 64..79 of A); written on every pass, since other users of the TMEM
  // (the projections) may have overwritten it.
  {
    const uint32_t ones[8] = {0x3C003C00u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    tmem_st8_wait(t_d + kSlotOnes + lane_off, ones);
  }

  // TMEM accumulator row (bias included, f16) -> activation in f16x2 -> the
  // group's A operand.
  auto hidden = [&]() {
    uint32_t y[32];
    tmem_ld64_f16_wait(t_d + lane_off, y);
#pragma unroll
    for (int chunk = 0; chunk < 8; ++chunk)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        y[4 * chunk + j] = chunk < kTanhChunks ? gelu2_f16x2(y[4 * chunk + j]) : gelu_poly_f16x2(y[4 * chunk + j]);
    tmem_st32_wait(t_a + lane_off, y);
  };

  // Features of tile t as the layer-1 operand row: [hi(f) | hi(f) | lo(f) |
  // 1 1 0 0] against [hi(W1) | lo(W1) | hi(W1) | hi(b1) lo(b1) 0 0] gives
  // W1 f + b1 to ~22 bits. Returns the row's sink key (-1 for a padding row)
  // and its particles.
  auto features = [&](int t, uint32_t* a1, int& p_out, int& a_out, int& b_out) {
    int p = -1, a = 0, b = 0;
    float f[4] = {0.f, 0.f, 0.f, 0.f};
    const bool valid = src.row(t, row, p, a, b, f);
    if (!valid) {
      f[0] = f[1] = f[2] = f[3] = 0.f;
      a = b = 0;
    }
    p_out = valid ? p : -1;
    a_out = a;
    b_out = b;
    __half hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split_half(f[i], hi[i], lo[i]);
    const __half one = __float2half_rn(valid ? 1.f : 0.f), zero = __float2half_rn(0.f);
    a1[0] = h2bits(hi[0], hi[1]);
    a1[1] = h2bits(hi[2], hi[3]);
    a1[2] = a1[0];
    a1[3] = a1[1];
    a1[4] = h2bits(lo[0], lo[1]);
    a1[5] = h2bits(lo[2], lo[3]);
    a1[6] = h2bits(one, one);
    a1[7] = h2bits(zero, zero);
  };

  // Per tile: layer 1 is issued from features computed during the previous
  // tile's last MMA, and the previous tile's row goes to the sink while this
  // tile's first MMA runs, so neither sits between two MMAs of the group.
  uint32_t a1[8];
  int pk = -1, pa = 0, pb = 0;       // the current tile's row
  int qk = -1, qa = 0, qb = 0;       // the previous tile's row, waiting for the sink
  float u[8];
  int t = g;
  if (t < ntiles) features(t, a1, pk, pa, pb);
#pragma unroll 1
  while (t < ntiles) {
    tmem_st8_wait(t_a + lane_off, a1);
    if (!issue(0)) return false;
    if (qk >= 0) sink(qk, qa, qb, u);
#pragma unroll 1
    for (int L = 1; L <= 3; ++L) {
      wait();
      hidden();
      if (!issue(L)) return false;
    }
    const int ck = pk, ca = pa, cb = pb;
    t += NG;
    if (t < ntiles) features(t, a1, pk, pa, pb);
    wait();
    tmem_ld8_wait(t_d + lane_off, u);
    qk = ck;
    qa = ca;
    qb = cb;
  }
  if (qk >= 0) sink(qk, qa, qb, u);
  // the TMEM reads of the last tile must finish before anyone reuses them
  tc_fence_before();
  return ok;
}

// ============================================== int8 engine (kind::i8)
//
// The variant of the MLP whose hidden layers take int8 inputs with zero
// points and int8 weights ("Economical Jet Taggers", section
// "Kwantiseringsstrategieen": inputs of linear layers int8 with zero-point
// quantisation, weights binary or ternary). Per pair row:
//   layer 1  y1 = W1 f + b1 as in the f16 engine (f16 hi + lo operands), but
//            accumulated in fp32;
//   hidden   h = GELU(y) in fp32 with erff (an approximation of GELU would
//            move codes across rounding boundaries); the row's 64 values are
//            quantised on their own: lo = min(0, min h), hi = max(0, max h),
//            s = (hi - lo) / 255 (1 if hi == lo), z = -128 - rint(lo / s),
//            q = clamp(rint(h / s) + z, -128, 127) (round half to even);
//            the 64 codes go to TMEM as the next layer's A operand;
//   layers 2..4  tcgen05.mma kind::i8 (s8 x s8 -> s32, K = 32 per MMA, A
//            from TMEM, four codes per column; B, the weight codes, from
//            shared memory); then y_o = alpha_o s (acc_o - z sum_i T_oi) +
//            b_o in fp32, the zero-point term being an exact integer.
// Shared memory: the f16 engine's W2 / W3 / W4 tiles hold instead the code
// tiles (K-major, 16-byte core-matrix rows of 16 codes) and each layer's
// alpha, bias and code row sums.

constexpr int kI8TileBytes = 64 * 64;     // one 64 x 64 code tile
constexpr int kI8Alpha = kI8TileBytes;    // byte offsets inside a layer's region
constexpr int kI8Bias = kI8Alpha + 256;
constexpr int kI8Tsum = kI8Bias + 256;
constexpr int kI8W4Alpha = 16 * 64;       // layer 4: 16 code rows (8 used), then 8 + 8 + 8 values
constexpr int kI8W4Bias = kI8W4Alpha + 32;
constexpr int kI8W4Tsum = kI8W4Bias + 32;

// Byte offset of code (row r, column k) of a K-major code tile with 64
// columns: 8 x 16-byte core matrices, 4 along K per 8-row group.
__device__ __forceinline__ int i8ofs(int r, int k) { return (((r >> 3) * 4 + (k >> 4)) << 7) + ((r & 7) << 4) + (k & 15); }

// kind::i8 instruction descriptor: s8 A and B, both K-major, s32 D, M = 128.
__host__ __device__ constexpr uint32_t idesc_i8_m128(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_i8_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st16_wait_u(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Once per CTA: layer 1 as in the f16 engine, the code tiles and per-row
// constants of layers 2..4, mbarriers, TMEM.
template <int NG, int SL>
__device__ void mlp_setup_i8(MlpSmem<NG, SL>& S, const MlpI8Args& W) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  unsigned char* R2 = reinterpret_cast<unsigned char*>(S.W2);
  unsigned char* R3 = reinterpret_cast<unsigned char*>(S.W3);
  unsigned char* R4 = reinterpret_cast<unsigned char*>(S.W4);
  for (int e = tid; e < 64 * 64 / 4; e += nthr) {  // 4 codes of one row at a time
    const int r = e >> 4, k = (e & 15) * 4;
    *reinterpret_cast<uint32_t*>(R2 + i8ofs(r, k)) = reinterpret_cast<const uint32_t*>(W.T2)[e];
    *reinterpret_cast<uint32_t*>(R3 + i8ofs(r, k)) = reinterpret_cast<const uint32_t*>(W.T3)[e];
    if (r < 16) *reinterpret_cast<uint32_t*>(R4 + i8ofs(r, k)) = r < 8 ? reinterpret_cast<const uint32_t*>(W.T4)[e] : 0u;
  }
  if (tid < 64) {
    const int r = tid;
    int s2 = 0, s3 = 0, s4 = 0;
    for (int k = 0; k < 64; ++k) {
      s2 += W.T2[r * 64 + k];
      s3 += W.T3[r * 64 + k];
      if (r < 8) s4 += W.T4[r * 64 + k];
    }
    reinterpret_cast<float*>(R2 + kI8Alpha)[r] = W.a2[r];
    reinterpret_cast<float*>(R2 + kI8Bias)[r] = W.b2[r];
    reinterpret_cast<int*>(R2 + kI8Tsum)[r] = s2;
    reinterpret_cast<float*>(R3 + kI8Alpha)[r] = W.a3[r];
    reinterpret_cast<float*>(R3 + kI8Bias)[r] = W.b3[r];
    reinterpret_cast<int*>(R3 + kI8Tsum)[r] = s3;
    if (r < 8) {
      reinterpret_cast<float*>(R4 + kI8W4Alpha)[r] = W.a4[r];
      reinterpret_cast<float*>(R4 + kI8W4Bias)[r] = W.b4[r];
      reinterpret_cast<int*>(R4 + kI8W4Tsum)[r] = s4;
    }
    // layer-1 row r: [hi(W1) | lo(W1) | hi(W1) | hi(b1) lo(b1) 0 0] (K = 16)
    __half h[4], l[4], bh, bl;
    const float w1[4] = {W.W1[4 * r], W.W1[4 * r + 1], W.W1[4 * r + 2], W.W1[4 * r + 3]};
    for (int i = 0; i < 4; ++i) split_half(w1[i], h[i], l[i]);
    split_half(W.b1[r], bh, bl);
    const __half z = __float2half_rn(0.f);
    *reinterpret_cast<uint4*>(S.W1 + cofs(r, 0, 16)) =
        make_uint4(h2bits(h[0], h[1]), h2bits(h[2], h[3]), h2bits(l[0], l[1]), h2bits(l[2], l[3]));
    *reinterpret_cast<uint4*>(S.W1 + cofs(r, 8, 16)) =
        make_uint4(h2bits(h[0], h[1]), h2bits(h[2], h[3]), h2bits(bh, bl), h2bits(z, z));
  }
  if (tid == 0) {
    for (int i = 0; i < NG * SL; ++i) mbar_init(&S.mbar[i], 1);
    fence_mbar_init();
  }
  if ((tid >> 5) == 0) tmem_alloc(&S.tmem_base, kTmemCols(NG, SL));
  fence_proxy_async_smem();  // code and weight tiles are read by the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

__device__ __forceinline__ float gelu_erf(float y) { return 0.5f * y * (1.f + erff(y * 0.70710678118654752f)); }

// The int8 variant of mlp_pass (same scheduling, sources and sinks).
template <int NG, int SL, class Source, class Sink>
__device__ bool mlp_pass_i8(MlpSmem<NG, SL>& S, const Source& src, Sink& sink, uint32_t* phase) {
  const int g = threadIdx.x >> 7;
  if (g >= NG) return true;
  const int row = threadIdx.x & 127;
  const uint32_t bar_id = 1 + g;
  const bool leader = row == 0;
  const unsigned char* const R2 = reinterpret_cast<const unsigned char*>(S.W2);
  const unsigned char* const R3 = reinterpret_cast<const unsigned char*>(S.W3);
  const unsigned char* const R4 = reinterpret_cast<const unsigned char*>(S.W4);
  auto region = [&](int L) { return L == 1 ? R2 : (L == 2 ? R3 : R4); };  // layer L + 1's constants
  const uint32_t w1_addr = smem_u32(S.W1);
  constexpr uint32_t kIdL1 = idesc_f16_m128(64, true), kId64 = idesc_i8_m128(64), kId16 = idesc_i8_m128(16);
  const int ntiles = src.ntiles();
  uint64_t* const mbar = &S.mbar[g];
  const uint32_t lane_off = (uint32_t)(row & 96) << 16;
  const uint32_t t_d = S.tmem_base + (uint32_t)(g * kSlotCols);
  const uint32_t t_a = t_d + kSlotA;
  bool ok = true;

  auto issue = [&](int L) -> bool {
    tc_fence_before();
    if (named_bar_or(bar_id, 128, !ok)) return false;
    if (leader) {
      tc_fence_after();
      if (L == 0) {
        mma_f16_ta(t_d, t_a, smem_desc(w1_addr, 128, 256), kIdL1, 0u);
      } else {
        const uint32_t w = smem_u32(region(L));
        const uint32_t id = L == 3 ? kId16 : kId64;
#pragma unroll
        for (int k = 0; k < 2; ++k) mma_i8_ta(t_d, t_a + 8u * k, smem_desc(w + 256u * k, 128, 512), id, k);
      }
      mma_commit(mbar);
    }
    return true;
  };
  auto wait = [&]() {
    const bool done = mbar_wait(mbar, *phase & 1u);
    ok = ok && done;
    *phase ^= 1u;
    tc_fence_after();
  };
  // y of one output column o of layer L (1..3: hidden; the accumulator word
  // is fp32 for layer 1, s32 for the others) from the row's scale and zero point
  auto dequant = [&](int L, int o, uint32_t accw, float s, int z) -> float {
    if (L == 0) return __uint_as_float(accw);
    const unsigned char* Rl = region(L);
    const bool last = L == 3;
    const float al = reinterpret_cast<const float*>(Rl + (last ? kI8W4Alpha : kI8Alpha))[o];
    const float bi = reinterpret_cast<const float*>(Rl + (last ? kI8W4Bias : kI8Bias))[o];
    const int ts = reinterpret_cast<const int*>(Rl + (last ? kI8W4Tsum : kI8Tsum))[o];
    const int d = (int)accw - z * ts;
    return fmaf((float)d, al * s, bi);
  };
  // Layer L's accumulators -> GELU -> int8 codes of the next layer's input;
  // the row's new scale and zero point replace (s, z).
  auto hidden = [&](int L, float& s, int& z) {
    float h[64];
    {
      uint32_t w[64];
      tmem_ld64_wait(t_d + lane_off, reinterpret_cast<float*>(w));
#pragma unroll
      for (int o = 0; o < 64; ++o) h[o] = gelu_erf(dequant(L, o, w[o], s, z));
    }
    float lo = 0.f, hi = 0.f;
#pragma unroll
    for (int o = 0; o < 64; ++o) {
      lo = fminf(lo, h[o]);
      hi = fmaxf(hi, h[o]);
    }
    const float sn = hi > lo ? (hi - lo) / 255.f : 1.f;
    const float inv = 1.f / sn;
    const int zn = -128 - __float2int_rn(lo / sn);
    uint32_t codes[16];
#pragma unroll
    for (int w4 = 0; w4 < 16; ++w4) {
      int c[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) c[j] = max(-128, min(127, __float2int_rn(h[4 * w4 + j] * inv) + zn));
      codes[w4] = (uint32_t)(c[0] & 255) | ((uint32_t)(c[1] & 255) << 8) | ((uint32_t)(c[2] & 255) << 16) |
                  ((uint32_t)(c[3] & 255) << 24);
    }
    tmem_st16_wait_u(t_a + lane_off, codes);
    s = sn;
    z = zn;
  };
  auto features = [&](int t, uint32_t* a1, int& p_out, int& a_out, int& b_out) {
    int p = -1, a = 0, b = 0;
    float f[4] = {0.f, 0.f, 0.f, 0.f};
    const bool valid = src.row(t, row, p, a, b, f);
    if (!valid) {
      f[0] = f[1] = f[2] = f[3] = 0.f;
      a = b = 0;
    }
    p_out = valid ? p : -1;
    a_out = a;
    b_out = b;
    __half hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split_half(f[i], hi[i], lo[i]);
    const __half one = __float2half_rn(valid ? 1.f : 0.f), zero = __float2half_rn(0.f);
    a1[0] = h2bits(hi[0], hi[1]);
    a1[1] = h2bits(hi[2], hi[3]);
    a1[2] = a1[0];
    a1[3] = a1[1];
    a1[4] = h2bits(lo[0], lo[1]);
    a1[5] = h2bits(lo[2], lo[3]);
    a1[6] = h2bits(one, one);
    a1[7] = h2bits(zero, zero);
  };

  uint32_t a1[8];
  int pk = -1, pa = 0, pb = 0, qk = -1, qa = 0, qb = 0;
  float u[8];
  int t = g;
  if (t < ntiles) features(t, a1, pk, pa, pb);
#pragma unroll 1
  while (t < ntiles) {
    tmem_st8_wait(t_a + lane_off, a1);
    if (!issue(0)) return false;
    if (qk >= 0) sink(qk, qa, qb, u);
    float s = 1.f;
    int z = 0;
#pragma unroll 1
    for (int L = 0; L < 3; ++L) {
      wait();
      hidden(L, s, z);
      if (!issue(L + 1)) return false;
    }
    const int ck = pk, ca = pa, cb = pb;
    t += NG;
    if (t < ntiles) features(t, a1, pk, pa, pb);
    wait();
    {
      float w[8];
      tmem_ld8_wait(t_d + lane_off, w);
#pragma unroll
      for (int o = 0; o < 8; ++o) u[o] = dequant(3, o, __float_as_uint(w[o]), s, z);
    }
    qk = ck;
    qa = ca;
    qb = cb;
  }
  if (qk >= 0) sink(qk, qa, qb, u);
  tc_fence_before();
  return ok;
}

// The engine of a weight-argument type: f16 (MlpArgs) or int8 (MlpI8Args).
template <int NG, int SL>
__device__ void mlp_setup_any(MlpSmem<NG, SL>& S, const MlpArgs& W) { mlp_setup<NG, SL>(S, W); }
template <int NG, int SL>
__device__ void mlp_setup_any(MlpSmem<NG, SL>& S, const MlpI8Args& W) { mlp_setup_i8<NG, SL>(S, W); }

template <class WA, int NG, int SL, class Source, class Sink>
__device__ bool mlp_run(MlpSmem<NG, SL>& S, const Source& src, Sink& sink, uint32_t* phase) {
  if constexpr (std::is_same<WA, MlpI8Args>::value) return mlp_pass_i8<NG, SL>(S, src, sink, phase);
  else return mlp_pass<NG, SL>(S, src, sink, phase);
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
    if (!in_bounds(sa >= 0 && sb >= 0 && sa < P && sb < P)) return;
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
  MlpSmem<NG, 2> mlp;
  Particles<PM> part;
};

template <int PM, int NG, bool F32OUT, class WA = MlpArgs>
__global__ void __launch_bounds__(NG * 128, 1) k_mlp_bias(JetArgs J, WA W, void* __restrict__ U) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  MlpBiasSmem<PM, NG>& S = *reinterpret_cast<MlpBiasSmem<PM, NG>*>(smem_raw);
  mlp_setup_any<NG, 2>(S.mlp, W);
  uint32_t phase = 0u;
  bool aborted = false;
  for (int n = blockIdx.x; n < J.N; n += gridDim.x) {
    stage_jet<PM>(S.part, J, n);
    zero_masked_pairs<PM, F32OUT>(S.part, U, n, J.P);
    const int m = S.part.m;
    GlobalUSink<PM, F32OUT> sink{&S.part, U, n, J.P};
    const bool ok = mlp_run<WA, NG, 2>(S.mlp, JetTiles<PM, TriPairs, true>{&S.part, m * (m + 1) / 2, TriPairs{}}, sink, &phase);
    aborted = __syncthreads_or(!ok) != 0;
    if (aborted) break;
  }
  mlp_teardown<NG, 2>(S.mlp, aborted, &phase);
}

// ========================================================== attention engine

// Element offset of (jet, head h, compact particle c) in Q/K/V/out.
template <int PM>
__device__ __forceinline__ size_t qkv_off(const Particles<PM>& S, const JetArgs& J, int n, int h, int c) {
  if (!in_bounds(c >= 0 && c < S.m && h >= 0 && h < kH && n >= 0 && n < J.N)) return 0;
  if (J.ptr) return ((size_t)(S.base + c) * kH + h) * kD;
  return (((size_t)n * kH + h) * J.P + S.slot[c]) * kD;
}

// Prefetch the Q, K and V rows of the staged jet n into L2: per tensor and
// head the slots [slot[0], slot[m-1]] (padded) or the jet's tokens (packed).
// Threads 0..23 issue one bulk prefetch each; no barrier.
template <int PM>
__device__ __forceinline__ void prefetch_qkv(const Particles<PM>& S, const JetArgs& J, const QkvArgs& X, int n) {
  const int t = threadIdx.x;
  if (t >= 3 * kH || S.m <= 0) return;
  const uint16_t* base = t < kH ? X.q : (t < 2 * kH ? X.k : X.v);
  const int h = t % kH;
  if (J.ptr) {
    if (h == 0) prefetch_l2(base + (size_t)S.base * kH * kD, (uint32_t)S.m * kH * kD * 2);
  } else {
    const int s0 = S.slot[0], s1 = S.slot[S.m - 1];
    prefetch_l2(base + (((size_t)n * kH + h) * J.P + s0) * kD, (uint32_t)(s1 - s0 + 1) * kD * 2);
  }
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

// ---------------------------------------------------- attention on tensor cores
//
// Per (jet, head): S = Q K^T on m16n8k16 tensor-core tiles (bf16 operands,
// fp32 accumulation) held in registers, the bias and the key mask added to S
// there, an online softmax over blocks of 16 keys in the log2 domain, then
// O += P V with P rounded to bf16 (P in [0, 1]: relative rounding 2^-9).
// One warp owns 16 queries of one head. K and V of a head are staged in
// shared memory as bf16, zero beyond m: K row-major [m16][kKStride] and V
// transposed [16][m16 + 8]; both strides make the fragment loads of a warp
// hit 32 distinct banks.

constexpr int kKStride = 24;  // halves per staged K or V row (48 bytes)

__host__ __device__ constexpr int round16(int m) { return (m + 15) & ~15; }

// The forward attention stages K and V rows unpadded (32 bytes, two 16-byte
// chunks) with chunk c of row r at chunk c ^ ((r >> 2) & 1): the 8 rows of an
// ldmatrix phase then cover all 32 banks once.
__host__ __device__ constexpr int kv16_bytes(int m) { return 2 * round16(m) * 32; }
__device__ __forceinline__ uint32_t kv_off(int r, int c) { return (uint32_t)(r * 32 + ((c ^ ((r >> 2) & 1)) << 4)); }

// ldmatrix: four (or two) 8x8 b16 matrices from shared memory into the
// fragment layout of mma.sync; .trans delivers each matrix transposed.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Byte offsets, inside a staged [rows][kKStride] tensor, of this lane's
// ldmatrix row for the three fragment shapes used (add the tile's first row
// times the row pitch):
//   A  (16 rows x 16 cols, x4):            rows 0-7 | 8-15, cols 0-7 | 8-15
//   Bn (two n8 blocks of rows, d = K, x4):  b0,b1 of rows 0-7, then of rows 8-15
//   Bt (rows = K, d = N, x4.trans):         b0,b1 of d 0-7, then of d 8-15
__device__ __forceinline__ uint32_t frag_a_off(int lane) {
  return (uint32_t)(((lane & 7) + ((lane >> 3) & 1) * 8) * kKStride * 2 + (lane >> 4) * 16);
}
__device__ __forceinline__ uint32_t frag_bn_off(int lane) {
  return (uint32_t)(((lane & 7) + ((lane >> 4) & 1) * 8) * kKStride * 2 + ((lane >> 3) & 1) * 16);
}
__device__ __forceinline__ uint32_t frag_bt_off(int lane) {
  return (uint32_t)(((lane & 7) + ((lane >> 3) & 1) * 8) * kKStride * 2 + ((lane >> 4) & 1) * 16);
}

// 16-byte global -> shared copy that bypasses the registers; with
// src_bytes = 0 nothing is read and the destination is zero-filled.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// K and V of heads [h0, h0 + hr) of the staged jet n into buf, one head
// after another (kv16_bytes(m) each): K rows then V rows, bf16 [m16][16] in
// the swizzled chunk order of kv_off, zero rows past m. Asynchronous 16-byte copies, committed as one group: the
// caller waits with cp_async_wait_all() and a barrier. Block-wide.
template <int PM>
__device__ void stage_kv16(const Particles<PM>& S, const JetArgs& J, const QkvArgs& X, int n, int h0, int hr,
                           uint16_t* buf) {
  const int m = S.m, m16 = round16(m), hb = kv16_bytes(m) / 2;
  const int total = hr * m16 * 4, nthr = blockDim.x;
  for (int idx = threadIdx.x; idx < total; idx += nthr) {
    const int part = idx & 3, j = (idx >> 2) % m16, hh = (idx >> 2) / m16;
    const uint16_t* base = part < 2 ? X.k : X.v;
    const bool valid = j < m;
    const uint16_t* src = base + (valid ? qkv_off<PM>(S, J, n, h0 + hh, j) : 0) + (part & 1) * 8;
    cp_async16(buf + hh * hb + (part >> 1) * m16 * 16 + kv_off(j, part & 1) / 2, src, valid ? 16u : 0u);
  }
  cp_async_commit();
}

// D += A B on one m16n8k16 tile: A 16x16 bf16 (row), B 16x8 bf16 (col), D fp32.
__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Bias blocks: the 8 values of U[h, ., .] a lane needs for one key block
// (see attend_tile16), from the storage layouts the kernels use.

// Triangle of records of RS halves (one per head: 8 for all heads, 2 where
// a CTA holds two heads), pair (a, b) with a >= b at record a(a+1)/2 + b;
// U points at head h of record 0. Query tiles and key blocks are aligned to
// 16, so a full key block lies wholly below the tile's rows (records
// i(i+1)/2 + j, contiguous in j), wholly above them (records j(j+1)/2 + i),
// or on the diagonal, which takes the general formula.
template <int RS>
struct TriBlockS {
  const __half* U;
  __device__ __forceinline__ void operator()(int n0, int i0, int ia, int ib, int t, int m, float* u) const {
    const int jb = n0 + 2 * t;
    if (n0 + 16 <= m && n0 + 16 <= i0) {
      const __half* ra = U + (ia * (ia + 1) / 2 + jb) * RS;
      const __half* rb = U + (ib * (ib + 1) / 2 + jb) * RS;
      u[0] = __half2float(ra[0]);
      u[1] = __half2float(ra[RS]);
      u[4] = __half2float(ra[8 * RS]);
      u[5] = __half2float(ra[9 * RS]);
      u[2] = __half2float(rb[0]);
      u[3] = __half2float(rb[RS]);
      u[6] = __half2float(rb[8 * RS]);
      u[7] = __half2float(rb[9 * RS]);
    } else if (n0 + 16 <= m && n0 >= i0 + 16) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = jb + (c & 1) + (c & 2) * 4, e = (c & 2) * 2 + (c & 1);
        const __half* cj = U + (j * (j + 1) / 2) * RS;
        u[e] = __half2float(cj[ia * RS]);
        u[e + 2] = __half2float(cj[ib * RS]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = e & 2 ? ib : ia, j = min(m - 1, jb + (e & 4 ? 8 : 0) + (e & 1));
        const int hi = max(i, j), lo = min(i, j);
        u[e] = __half2float(U[(hi * (hi + 1) / 2 + lo) * RS]);
      }
    }
  }
};
using TriBlock = TriBlockS<8>;

// Rectangle of 8-half records, (query i, key j) at record (i - r0) * m + j;
// U points at head h of record 0.
struct RectBlock {
  const __half* U;
  int r0, m;
  __device__ __forceinline__ void operator()(int n0, int, int ia, int ib, int t, int, float* u) const {
    const int jb = n0 + 2 * t;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = e & 2 ? ib : ia, j = min(m - 1, jb + (e & 4 ? 8 : 0) + (e & 1));
      u[e] = __half2float(U[((i - r0) * m + j) * 8]);
    }
  }
};

// A fragment of the 16 queries [i0, i0 + nrows) (zero rows past nrows);
// qrow(i) gives the bf16 row of query i. Warp-wide.
template <class QRow>
__device__ __forceinline__ void q_frag(int i0, int nrows, const QRow& qrow, uint32_t* a) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  a[0] = a[1] = a[2] = a[3] = 0u;
  if (g < nrows) {
    const uint16_t* q = qrow(i0 + g);
    a[0] = *reinterpret_cast<const uint32_t*>(q + 2 * t);
    a[2] = *reinterpret_cast<const uint32_t*>(q + 2 * t + 8);
  }
  if (g + 8 < nrows) {
    const uint16_t* q = qrow(i0 + g + 8);
    a[1] = *reinterpret_cast<const uint32_t*>(q + 2 * t);
    a[3] = *reinterpret_cast<const uint32_t*>(q + 2 * t + 8);
  }
}

// Queries [i0, i0 + nrows) (nrows <= 16, A fragment a from q_frag) of one
// head against its m staged keys: kh = staged K, vh = staged V of that head
// (rows in kv_off order; the Q K^T operand comes through ldmatrix, the P V
// operand through ldmatrix.trans). orow(i) gives the bf16 output row of query i; ub(n0, i0, ia, ib, t,
// m, u) fills the bias of the 8 score elements a lane holds for the key
// block n0 (element e: row e & 2 ? ib : ia, key n0 + 8 (e >> 2) + 2 t +
// (e & 1), keys past m clamped to m - 1). Warp-wide.
// Normalise and store the two output rows of a lane (o as accumulated, la /
// lb the lane's partial row sums of p).
template <class ORow>
__device__ __forceinline__ void store_out16(const float* o, float la, float lb, bool va, bool vb, int ia, int ib,
                                            int t, const ORow& orow) {
  la += __shfl_xor_sync(0xffffffffu, la, 1);
  la += __shfl_xor_sync(0xffffffffu, la, 2);
  lb += __shfl_xor_sync(0xffffffffu, lb, 1);
  lb += __shfl_xor_sync(0xffffffffu, lb, 2);
  if (va) {
    const float r = 1.0f / la;
    uint16_t* op = orow(ia);
    *reinterpret_cast<uint32_t*>(op + 2 * t) = cvt_bf16x2(o[0] * r, o[1] * r);
    *reinterpret_cast<uint32_t*>(op + 8 + 2 * t) = cvt_bf16x2(o[4] * r, o[5] * r);
  }
  if (vb) {
    const float r = 1.0f / lb;
    uint16_t* op = orow(ib);
    *reinterpret_cast<uint32_t*>(op + 2 * t) = cvt_bf16x2(o[2] * r, o[3] * r);
    *reinterpret_cast<uint32_t*>(op + 8 + 2 * t) = cvt_bf16x2(o[6] * r, o[7] * r);
  }
}

// Jets of at most 16 NKB keys: every block's scores stay in registers, so the
// softmax takes two passes (one row maximum, then the exponentials and P V)
// and the blocks' products and exponentials are independent of each other,
// with no rescaling chain between blocks.
template <int NKB, class ORow, class UBlock>
__device__ __forceinline__ void attend_tile16_short(uint32_t k_base, uint32_t v_base, int m, int i0, int ia, int ib,
                                                    bool va, bool vb, const uint32_t* a, const ORow& orow,
                                                    const UBlock& ub) {
  const int t = threadIdx.x & 3;
  const float qs = 0.25f * kLog2e;  // 1/sqrt(D) with D = 16, in log2 units
  float s[NKB][8];
#pragma unroll
  for (int kb = 0; kb < NKB; ++kb) {
#pragma unroll
    for (int e = 0; e < 8; ++e) s[kb][e] = 0.f;
    uint32_t bk[4];
    ldsm_x4(k_base + (uint32_t)kb * 512u, bk);
    mma_16816(s[kb], a, bk[0], bk[1]);
    mma_16816(s[kb] + 4, a, bk[2], bk[3]);
  }
  float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
  for (int kb = 0; kb < NKB; ++kb) {
    float u[8];
    ub(16 * kb, i0, ia, ib, t, m, u);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = 16 * kb + (e & 4 ? 8 : 0) + 2 * t + (e & 1);
      s[kb][e] = j < m ? fmaf(s[kb][e], qs, u[e] * kLog2e) : -INFINITY;
    }
    mxa = fmaxf(mxa, fmaxf(fmaxf(s[kb][0], s[kb][1]), fmaxf(s[kb][4], s[kb][5])));
    mxb = fmaxf(mxb, fmaxf(fmaxf(s[kb][2], s[kb][3]), fmaxf(s[kb][6], s[kb][7])));
  }
  // key 0 < m is valid for every row, so the maxima are finite
  mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
  mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
  mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
  mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
  float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float la = 0.f, lb = 0.f;
#pragma unroll
  for (int kb = 0; kb < NKB; ++kb) {
    float p[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) p[e] = ex2(s[kb][e] - (e & 2 ? mxb : mxa));
    la += (p[0] + p[1]) + (p[4] + p[5]);
    lb += (p[2] + p[3]) + (p[6] + p[7]);
    const uint32_t pa[4] = {cvt_bf16x2(p[0], p[1]), cvt_bf16x2(p[2], p[3]), cvt_bf16x2(p[4], p[5]),
                            cvt_bf16x2(p[6], p[7])};
    uint32_t bv[4];
    ldsm_x4_t(v_base + (uint32_t)kb * 512u, bv);
    mma_16816(o, pa, bv[0], bv[1]);
    mma_16816(o + 4, pa, bv[2], bv[3]);
  }
  store_out16(o, la, lb, va, vb, ia, ib, t, orow);
}

template <class ORow, class UBlock>
__device__ __forceinline__ void attend_tile16(const uint16_t* kh, const uint16_t* vh, int m, int i0, int nrows,
                                              const uint32_t* a, const ORow& orow, const UBlock& ub) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  // lane rows of the two fragment shapes (see frag_bn_off / frag_bt_off); a
  // 16-row step keeps the swizzle phase
  const uint32_t k_base = smem_u32(kh) + kv_off((lane & 7) + ((lane >> 4) & 1) * 8, (lane >> 3) & 1);
  const uint32_t v_base = smem_u32(vh) + kv_off((lane & 7) + ((lane >> 3) & 1) * 8, (lane >> 4) & 1);
  const bool va = g < nrows, vb = g + 8 < nrows;
  const int ia = i0 + (va ? g : 0), ib = i0 + (vb ? g + 8 : 0);  // rows past the block alias row i0
  switch ((m + 15) >> 4) {
    case 1: attend_tile16_short<1>(k_base, v_base, m, i0, ia, ib, va, vb, a, orow, ub); return;
    case 2: attend_tile16_short<2>(k_base, v_base, m, i0, ia, ib, va, vb, a, orow, ub); return;
    case 3: attend_tile16_short<3>(k_base, v_base, m, i0, ia, ib, va, vb, a, orow, ub); return;
    case 4: attend_tile16_short<4>(k_base, v_base, m, i0, ia, ib, va, vb, a, orow, ub); return;
    default: break;
  }
  const float qs = 0.25f * kLog2e;  // 1/sqrt(D) with D = 16, in log2 units
  float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float mxa = -INFINITY, mxb = -INFINITY, la = 0.f, lb = 0.f;
  for (int n0 = 0; n0 < m; n0 += 16) {
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    uint32_t bk[4];
    ldsm_x4(k_base + (uint32_t)n0 * 32u, bk);
    mma_16816(s, a, bk[0], bk[1]);
    mma_16816(s + 4, a, bk[2], bk[3]);
    float u[8];
    ub(n0, i0, ia, ib, t, m, u);
    if (n0 + 16 <= m) {
#pragma unroll
      for (int e = 0; e < 8; ++e) s[e] = fmaf(s[e], qs, u[e] * kLog2e);
    } else {  // the last, partial block: keys past m are masked
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j = n0 + (e & 4 ? 8 : 0) + 2 * t + (e & 1);
        s[e] = j < m ? fmaf(s[e], qs, u[e] * kLog2e) : -INFINITY;
      }
    }
    float bma = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[4], s[5]));
    float bmb = fmaxf(fmaxf(s[2], s[3]), fmaxf(s[6], s[7]));
    bma = fmaxf(bma, __shfl_xor_sync(0xffffffffu, bma, 1));
    bma = fmaxf(bma, __shfl_xor_sync(0xffffffffu, bma, 2));
    bmb = fmaxf(bmb, __shfl_xor_sync(0xffffffffu, bmb, 1));
    bmb = fmaxf(bmb, __shfl_xor_sync(0xffffffffu, bmb, 2));
    // key n0 < m is valid for every row, so the new maxima are finite
    const float nma = fmaxf(mxa, bma), nmb = fmaxf(mxb, bmb);
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
    const uint32_t pa[4] = {cvt_bf16x2(p[0], p[1]), cvt_bf16x2(p[2], p[3]), cvt_bf16x2(p[4], p[5]),
                            cvt_bf16x2(p[6], p[7])};
    uint32_t bv[4];
    ldsm_x4_t(v_base + (uint32_t)n0 * 32u, bv);
    mma_16816(o, pa, bv[0], bv[1]);
    mma_16816(o + 4, pa, bv[2], bv[3]);
  }
  store_out16(o, la, lb, va, vb, ia, ib, t, orow);
}

// Masked multi-head attention for queries [i_lo, i_hi) of the staged jet
// against all its valid keys, heads [h_lo, h_hi), on tensor cores: K and V of
// as many heads as `stage` holds are staged at a time, then the warps take
// (head, 16-query tile) items. ubias.head(h) gives the bias blocks of head h.
// With `prestaged`, the K and V of all heads [h_lo, h_hi) were already
// issued there by this block (stage_kv16, one group per thread): the copies
// are awaited and `stage` is not used.
template <int PM, class UBias>
__device__ void attention_block(const Particles<PM>& S, const JetArgs& J, const QkvArgs& X, int n, int i_lo,
                                int i_hi, float* stage, int stage_floats, const UBias& ubias, int h_lo = 0,
                                int h_hi = kH, uint16_t* prestaged = nullptr) {
  const int m = S.m;
  const int nq = i_hi - i_lo;
  if (m <= 0 || nq <= 0) {
    if (prestaged) cp_async_wait_all();
    return;
  }
  const int hb = kv16_bytes(m);
  const int HR = prestaged ? h_hi - h_lo : max(1, min(kH, stage_floats * 4 / hb));
  const int tiles = (nq + 15) >> 4;
  const int warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  uint16_t* buf = prestaged ? prestaged : reinterpret_cast<uint16_t*>(stage);
  if (!prestaged && !in_bounds(hb <= stage_floats * 4)) return;  // one head's K and V must fit
  for (int h0 = h_lo; h0 < h_hi; h0 += HR) {
    const int hr = min(HR, h_hi - h0);
    // the Q fragment of a warp's next item is loaded ahead: the first one
    // before the staging barrier, the others while the previous item runs
    uint32_t a[4] = {0u, 0u, 0u, 0u};
    auto qload = [&](int it, uint32_t* f) {
      const int h = h0 + it / tiles, i0 = i_lo + (it % tiles) * 16;
      q_frag(i0, min(16, i_hi - i0), [&](int i) { return X.q + qkv_off<PM>(S, J, n, h, i); }, f);
    };
    if (warp < hr * tiles) qload(warp, a);
    if (!prestaged) stage_kv16<PM>(S, J, X, n, h0, hr, buf);
    cp_async_wait_all();
    __syncthreads();
    for (int it = warp; it < hr * tiles; it += nwarp) {
      uint32_t an[4] = {0u, 0u, 0u, 0u};
      if (it + nwarp < hr * tiles) qload(it + nwarp, an);
      const int hh = it / tiles, i0 = i_lo + (it % tiles) * 16, h = h0 + hh;
      const uint16_t* kh = buf + hh * (hb / 2);
      attend_tile16(
          kh, kh + round16(m) * 16, m, i0, min(16, i_hi - i0), a,
          [&](int i) { return X.out + qkv_off<PM>(S, J, n, h, i); }, ubias.head(h));
#pragma unroll
      for (int e = 0; e < 4; ++e) a[e] = an[e];
    }
    __syncthreads();
  }
}

// Masked query rows of a padded jet are 0 (all of them when the jet is
// empty). Block-wide (blockDim.x a multiple of 16): 16 threads per slot,
// thread (head, half) of it, no division.
template <int PM>
__device__ void zero_masked_rows(const Particles<PM>& S, const JetArgs& J, uint16_t* out, int n) {
  if (J.ptr) return;
  const int P = J.P, h = (threadIdx.x >> 1) & 7, half = threadIdx.x & 1;
  for (int s = threadIdx.x >> 4; s < P; s += blockDim.x >> 4)
    if (S.comp[s] < 0)
      *reinterpret_cast<uint4*>(out + (((size_t)n * kH + h) * P + s) * kD + half * 8) = make_uint4(0, 0, 0, 0);
}
static_assert(kH == 8, "zero_masked_rows maps 16 threads to (head, half) of a slot");

// ------------------------------------------- k_attn_bias (bias read from HBM)

template <int PM>
struct GlobalUBias {  // U[n, h, slot i, slot j] of a bf16 [N, 8, P, P] tensor
  const Particles<PM>* S;
  const uint16_t* U;
  int n, P;
  struct Block {
    const int16_t* slot;
    const uint16_t* Uh;  // U[n, h]
    int P;
    __device__ __forceinline__ void operator()(int n0, int, int ia, int ib, int t, int m, float* u) const {
      const size_t ra = (size_t)slot[ia] * P, rb = (size_t)slot[ib] * P;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j = min(m - 1, n0 + 2 * t + (e & 4 ? 8 : 0) + (e & 1));
        u[e] = bf16_to_f32(Uh[(e & 2 ? rb : ra) + slot[j]]);
      }
    }
  };
  __device__ __forceinline__ Block head(int h) const { return Block{S->slot, U + ((size_t)n * kH + h) * P * P, P}; }
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
    stage_jet<PM, false>(S.part, J, n);
    GlobalUBias<PM> ub{&S.part, U, n, J.P};
    attention_block<PM>(S.part, J, X, n, 0, S.part.m, S.stage, kAttnStageFloats, ub);
    zero_masked_rows<PM>(S.part, J, X.out, n);
    __syncthreads();
  }
}

// ============================================ k_proj (projections either side)
//
// The in-projection of a ParT attention block (x -> Q, K, V) and its output
// projection (O -> y) as one tensor-core GEMM kernel over particle rows:
// out[r, :] = W in[r, :] + b for every row r of the padded slots (N * P) or
// the packed tokens, with E = 128 input features. The whole weight matrix
// (kNout x 128 bf16) stays in shared memory in the K-major layout of the MMA
// operands; each CTA streams 128-row tiles of the input through a double
// buffer, one thread issues 8 K steps x kNout/128 tcgen05 MMAs (bf16
// operands, fp32 accumulation in TMEM), and 8 warps read the accumulator
// back (TMEM lane = row), add the bias and store bf16.

constexpr int kEmbed = kH * kD;  // 128

enum ProjIn { kInRows = 0, kInHeads = 1 };     // [rows, 128] | attention layout [N, H, P, D]
enum ProjOut { kOutQKV = 0, kOutRows = 1 };    // Q, K, V in attention layout | [rows, 128]

struct ProjArgs {
  const uint16_t* in;   // kInRows: x [rows, 128]; kInHeads: O in the layout of Q
  const uint16_t* W;    // [kNout, 128] bf16, row-major (out x in)
  const float* bias;    // [kNout]
  uint16_t* out0;       // kOutQKV: Q; kOutRows: y [rows, 128]
  uint16_t* out1;       // kOutQKV: K
  uint16_t* out2;       // kOutQKV: V
};

template <int kNout>
struct ProjSmem {
  __nv_bfloat16 W[kNout * kEmbed];      // B operand, K-major, 8-row groups of 2,048 B
  __nv_bfloat16 A[2][kTileM * kEmbed];  // A operand double buffer
  float bias[kNout];
  uint64_t mbar;
  uint32_t tmem_base;
};

__host__ __device__ constexpr uint32_t proj_tmem_cols(int nout) { return nout <= 128 ? 128u : (nout <= 256 ? 256u : 512u); }

// Rows of the GEMM: N * P padded slots or the packed tokens.
__device__ __forceinline__ long long proj_rows(const JetArgs& J) { return J.ptr ? J.tokens : (long long)J.N * J.P; }

// Row r of the output written? (the in-projection skips masked slots, whose
// Q/K/V are never read; the out-projection writes 0 there)
__device__ __forceinline__ bool proj_row_valid(const JetArgs& J, long long r) { return J.ptr || J.mask[r] != 0; }

// Input tile t (rows t*128 ..): 128 rows x 16 chunks of 8 bf16, loaded into
// eight registers per thread (rows past the end are zero), then stored to
// A in the operand layout. Block-wide (256 threads); no barrier.
constexpr int kTileChunksPerThread = kTileM * (kEmbed / 8) / 256;  // 8

// Chunk idx of a [rows][16 chunks] operand -> (row, chunk). A warp takes 8
// rows x 4 chunks: the 16-byte bank group of a chunk in the operand layout
// is its row mod 8, so each quarter-warp stores to 8 distinct bank groups,
// and the warp still reads whole 32-byte sectors of every row.
__device__ __forceinline__ void chunk_rc(int idx, int& r, int& kc) {
  const int w = idx >> 5, l = idx & 31;
  r = (w >> 2) * 8 + (l & 7);
  kc = (w & 3) * 4 + (l >> 3);
}

template <int kIn>
__device__ __forceinline__ void proj_fetch_tile(uint4* v, const JetArgs& J, const ProjArgs& X, long long t,
                                                long long R) {
#pragma unroll
  for (int u = 0; u < kTileChunksPerThread; ++u) {
    int rr, kc;
    chunk_rc(threadIdx.x + u * 256, rr, kc);
    const long long r = t * kTileM + rr;
    v[u] = make_uint4(0, 0, 0, 0);
    if (r < R) {
      const uint16_t* src;
      if (kIn == kInRows || J.ptr) {
        src = X.in + r * kEmbed + kc * 8;
      } else {  // O[n, h, slot, d] with column kc * 8 = h * 16 + (kc & 1) * 8
        const long long n = r / J.P, slot = r % J.P;
        src = X.in + ((n * kH + (kc >> 1)) * J.P + slot) * kD + (kc & 1) * 8;
      }
      v[u] = *reinterpret_cast<const uint4*>(src);
    }
  }
}

__device__ __forceinline__ void proj_store_tile(__nv_bfloat16* A, const uint4* v) {
#pragma unroll
  for (int u = 0; u < kTileChunksPerThread; ++u) {
    int rr, kc;
    chunk_rc(threadIdx.x + u * 256, rr, kc);
    *reinterpret_cast<uint4*>(A + cofs(rr, kc * 8, kEmbed)) = v[u];
  }
}

template <int kIn>
__device__ __forceinline__ void proj_load_tile(__nv_bfloat16* A, const JetArgs& J, const ProjArgs& X, long long t,
                                               long long R) {
  uint4 v[kTileChunksPerThread];
  proj_fetch_tile<kIn>(v, J, X, t, R);
  proj_store_tile(A, v);
}

template <int kNout, int kIn, int kOut>
__global__ void __launch_bounds__(256, 1) k_proj(JetArgs J, ProjArgs X) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ProjSmem<kNout>& S = *reinterpret_cast<ProjSmem<kNout>*>(smem_raw);
  constexpr uint32_t kCols = proj_tmem_cols(kNout);
  constexpr uint32_t kIdesc = idesc_bf16_m128(128);
  constexpr uint32_t kSBO = kEmbed / 8 * 128;  // 2,048 B between 8-row groups
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long R = proj_rows(J);
  const long long ntiles = (R + kTileM - 1) / kTileM;

  // the first input tile and the weights (K-major), once per CTA, with
  // sixteen 16-byte loads per thread in flight before their stores
  long long t = blockIdx.x;
  {
    uint4 a[kTileChunksPerThread];
    if (t < ntiles) proj_fetch_tile<kIn>(a, J, X, t, R);
    constexpr int kW = kNout * (kEmbed / 8) / 256;  // weight chunks per thread: 24 or 8
    static_assert(kNout * (kEmbed / 8) % 256 == 0, "whole weight chunks per thread");
#pragma unroll
    for (int b0 = 0; b0 < kW; b0 += 16) {
      uint4 w[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        int n, kc;
        chunk_rc(tid + (b0 + u) * 256, n, kc);
        if (b0 + u < kW) w[u] = *reinterpret_cast<const uint4*>(X.W + (size_t)n * kEmbed + kc * 8);
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        int n, kc;
        chunk_rc(tid + (b0 + u) * 256, n, kc);
        if (b0 + u < kW) *reinterpret_cast<uint4*>(S.W + cofs(n, kc * 8, kEmbed)) = w[u];
      }
    }
    if (t < ntiles) proj_store_tile(S.A[0], a);
  }
  for (int i = tid; i < kNout; i += blockDim.x) S.bias[i] = X.bias[i];
  if (tid == 0) {
    mbar_init(&S.mbar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, kCols);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  uint32_t phase = 0;
  bool ok = true;
  int buf = 0;
  for (; t < ntiles; t += gridDim.x, buf ^= 1) {
    if (tid == 0) {
      const uint32_t a0 = smem_u32(S.A[buf]), w0 = smem_u32(S.W);
#pragma unroll 1
      for (int c = 0; c < kNout / 128; ++c)
#pragma unroll
        for (int s = 0; s < kEmbed / 16; ++s)
          mma_f16(tmem + 128u * c, smem_desc(a0 + 256u * s, 128, kSBO),
                  smem_desc(w0 + (uint32_t)c * 128u * kSBO / 8u + 256u * s, 128, kSBO), kIdesc, s > 0 ? 1u : 0u);
      mma_commit(&S.mbar);
    }
    // the next tile loads while the MMAs run
    if (t + gridDim.x < ntiles) proj_load_tile<kIn>(S.A[buf ^ 1], J, X, t + gridDim.x, R);
    const bool done = mbar_wait(&S.mbar, phase);
    if (done) phase ^= 1u;  // on a timeout the teardown waits on the same phase once more
    ok = __syncthreads_and(done && ok) != 0;
    tc_fence_after();
    if (!ok) break;
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. and half w / 4 of the columns
    {
      const int rr = (warp & 3) * 32 + lane;
      const long long r = t * kTileM + rr;
      const bool in_range = r < R;
      const bool valid = in_range && proj_row_valid(J, r);
      const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
      constexpr int kHalf = kNout / 2;
#pragma unroll 1
      for (int c64 = (warp >> 2) * kHalf; c64 < (warp >> 2) * kHalf + kHalf; c64 += 64) {
        float v64[64];
        tmem_ld64_wait(lane_base + (uint32_t)c64, v64);  // warp-wide: every lane, in range or not
#pragma unroll
       for (int half = 0; half < 2; ++half) {
        const int c0 = c64 + 32 * half;
        const float* v = v64 + 32 * half;
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = valid ? cvt_bf16x2(v[2 * i] + S.bias[c0 + 2 * i], v[2 * i + 1] + S.bias[c0 + 2 * i + 1]) : 0u;
        if (kOut == kOutRows && in_range) {
          uint4* dst = reinterpret_cast<uint4*>(X.out0 + r * kEmbed + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        } else if (kOut == kOutQKV && valid) {
          // columns c0 .. c0 + 31: two heads of one of Q, K, V
          const int tensor = c0 / kEmbed, cc = c0 % kEmbed;
          uint16_t* base = tensor == 0 ? X.out0 : (tensor == 1 ? X.out1 : X.out2);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int h = cc / kD + hh;
            size_t off;
            if (J.ptr) off = ((size_t)r * kH + h) * kD;
            else off = (((size_t)(r / J.P) * kH + h) * J.P + (size_t)(r % J.P)) * kD;
            uint4* dst = reinterpret_cast<uint4*>(base + off);
            dst[0] = make_uint4(w[8 * hh], w[8 * hh + 1], w[8 * hh + 2], w[8 * hh + 3]);
            dst[1] = make_uint4(w[8 * hh + 4], w[8 * hh + 5], w[8 * hh + 6], w[8 * hh + 7]);
          }
        }
       }
      }
    }
    // TMEM is read and the next A tile written before the next MMAs
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (!ok && tid == 0) raise_status(kStTimeout);
  tc_fence_before();
  __syncthreads();
  if (!ok) {
    // an MMA may still be in flight: wait once more (bounded) before freeing TMEM
    if (tid == 0) (void)mbar_wait(&S.mbar, phase);
    __syncthreads();
  }
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kCols);
}


// ------------------------------------- per-jet projections inside k_fused
//
// With the projections fused, k_fused maps each jet's particle embeddings x
// to Q, K, V before its MLP and its attention output O to y after it, on
// the tensor cores, in the free activation tiles: a 128-row tile of input
// rows and one 128-row chunk of the weights at a time (64 KB), 8 K steps of
// M = 128, N = 128 into TMEM columns 0..127, then all 16 warps store the
// chunk's 128 columns (bias added, bf16) for the valid rows. Q, K, V and O
// live in the caller's workspace, in L2 for batches up to ~100 MB of them.

// 128 rows of `in` from row r0 (rows >= r_end zero) into A, K-major operand
// layout; 4 loads in flight per thread. Block-wide, no barrier.
template <int kIn>
__device__ void proj_stage_rows(__nv_bfloat16* A, const JetArgs& J, const uint16_t* in, long long r0,
                                long long r_end) {
  const int nthr = blockDim.x;
  for (int base = threadIdx.x; base < kTileM * (kEmbed / 8); base += 4 * nthr) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * nthr;
      v[u] = make_uint4(0, 0, 0, 0);
      if (idx < kTileM * (kEmbed / 8)) {
        int rr, kc;
        chunk_rc(idx, rr, kc);
        const long long r = r0 + rr;
        if (r < r_end) {
          const uint16_t* src;
          if (kIn == kInRows || J.ptr) {
            src = in + r * kEmbed + kc * 8;
          } else {
            const long long n = r / J.P, slot = r % J.P;
            src = in + ((n * kH + (kc >> 1)) * J.P + slot) * kD + (kc & 1) * 8;
          }
          v[u] = *reinterpret_cast<const uint4*>(src);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * nthr;
      if (idx < kTileM * (kEmbed / 8)) {
        int rr, kc;
        chunk_rc(idx, rr, kc);
        *reinterpret_cast<uint4*>(A + cofs(rr, kc * 8, kEmbed)) = v[u];
      }
    }
  }
}

// Rows c*128 .. c*128+127 of a row-major [.][128] bf16 weight into Wsm.
__device__ void proj_stage_w(__nv_bfloat16* Wsm, const uint16_t* W, int c) {
  const int nthr = blockDim.x;
  for (int base = threadIdx.x; base < kTileM * (kEmbed / 8); base += 4 * nthr) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * nthr;
      int n, kc;
      chunk_rc(idx, n, kc);
      if (idx < kTileM * (kEmbed / 8))
        v[u] = *reinterpret_cast<const uint4*>(W + ((size_t)c * kTileM + n) * kEmbed + kc * 8);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * nthr;
      int n, kc;
      chunk_rc(idx, n, kc);
      if (idx < kTileM * (kEmbed / 8)) *reinterpret_cast<uint4*>(Wsm + cofs(n, kc * 8, kEmbed)) = v[u];
    }
  }
}

// One row tile (rows r0 .., rows >= r_end zero) into A and weight chunks
// 0 .. NW-1 (rows 128 c ..) into Wsm + c * 128 * 128, with every load of a
// thread in flight before its stores (512 threads: 4 chunks per operand).
// Block-wide, no barrier.
template <int kIn, int NW>
__device__ void proj_stage_tile_and_weights(__nv_bfloat16* A, __nv_bfloat16* Wsm, const JetArgs& J,
                                            const uint16_t* in, long long r0, long long r_end, const uint16_t* W) {
  constexpr int kChunks = kTileM * (kEmbed / 8);  // 2048 per operand
  constexpr int kPer = kChunks / 512;             // 4
  uint4 v[(1 + NW) * kPer];
#pragma unroll
  for (int o = 0; o <= NW; ++o)
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      int rr, kc;
      chunk_rc(threadIdx.x + u * 512, rr, kc);
      uint4 x = make_uint4(0, 0, 0, 0);
      if (o == 0) {
        const long long r = r0 + rr;
        if (r < r_end) {
          const uint16_t* src;
          if (kIn == kInRows || J.ptr) {
            src = in + r * kEmbed + kc * 8;
          } else {
            const long long n = r / J.P, slot = r % J.P;
            src = in + ((n * kH + (kc >> 1)) * J.P + slot) * kD + (kc & 1) * 8;
          }
          x = *reinterpret_cast<const uint4*>(src);
        }
      } else {
        x = *reinterpret_cast<const uint4*>(W + ((size_t)(o - 1) * kTileM + rr) * kEmbed + kc * 8);
      }
      v[o * kPer + u] = x;
    }
#pragma unroll
  for (int o = 0; o <= NW; ++o)
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      int rr, kc;
      chunk_rc(threadIdx.x + u * 512, rr, kc);
      __nv_bfloat16* dst = o == 0 ? A : Wsm + (size_t)(o - 1) * kTileM * kEmbed;
      *reinterpret_cast<uint4*>(dst + cofs(rr, kc * 8, kEmbed)) = v[o * kPer + u];
    }
}

// NW products of A with weight chunks Wsm + c * 128 * 128 into TMEM columns
// tmem + 128 c, one commit and one wait. Block-wide; false if the wait ran out.
template <int NW>
__device__ bool proj_mma_n(__nv_bfloat16* A, __nv_bfloat16* Wsm, uint32_t tmem, uint64_t* mbar, uint32_t* phase) {
  constexpr uint32_t kSBO = kEmbed / 8 * 128;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    const uint32_t a0 = smem_u32(A), w0 = smem_u32(Wsm);
#pragma unroll
    for (int c = 0; c < NW; ++c)
#pragma unroll
      for (int s = 0; s < kEmbed / 16; ++s)
        mma_f16(tmem + 128u * c, smem_desc(a0 + 256u * s, 128, kSBO),
                smem_desc(w0 + (uint32_t)c * kTileM * kEmbed * 2u + 256u * s, 128, kSBO), idesc_bf16_m128(128),
                s > 0 ? 1u : 0u);
    mma_commit(mbar);
  }
  const bool done = mbar_wait(mbar, *phase & 1u);
  if (done) *phase ^= 1u;
  tc_fence_after();
  return __syncthreads_and(done) != 0;
}

// One 128 x 128 x 128 product into TMEM columns tmem .. tmem+127 and its
// wait: the operands were written by the block (generic proxy) before the
// call. Block-wide; returns false if the wait ran out.
__device__ bool proj_mma(__nv_bfloat16* A, __nv_bfloat16* Wsm, uint32_t tmem, uint64_t* mbar, uint32_t* phase) {
  constexpr uint32_t kSBO = kEmbed / 8 * 128;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    const uint32_t a0 = smem_u32(A), w0 = smem_u32(Wsm);
#pragma unroll
    for (int s = 0; s < kEmbed / 16; ++s)
      mma_f16(tmem, smem_desc(a0 + 256u * s, 128, kSBO), smem_desc(w0 + 256u * s, 128, kSBO),
              idesc_bf16_m128(128), s > 0 ? 1u : 0u);
    mma_commit(mbar);
  }
  const bool done = mbar_wait(mbar, *phase & 1u);
  if (done) *phase ^= 1u;
  tc_fence_after();
  return __syncthreads_and(done) != 0;
}

// The 128 accumulator columns of rows r0 .. r0+127 (rows >= r_end skipped):
// + bias, bf16, stored for valid rows either as tensor `tensor` (0 Q, 1 K,
// 2 V) of the attention layout (kOutQKV, masked slots skipped) or as y rows
// (kOutRows, masked slots written 0). 16 warps: warp w reads TMEM lanes
// 32 (w % 4) and columns 32 (w / 4) ..
template <int kOut>
__device__ void proj_store(uint32_t tmem, const float* bias, const JetArgs& J, long long r0, long long r_end,
                           uint16_t* out, int tensor) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = (warp & 3) * 32 + lane, c0 = (warp >> 2) * 32;
  const long long r = r0 + rr;
  float v[32];
  tmem_ld32_wait(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)c0, v);  // every lane of the warp
  if (r >= r_end) return;
  const bool valid = J.ptr || J.mask[r] != 0;
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    w[i] = valid ? cvt_bf16x2(v[2 * i] + __ldg(bias + tensor * kEmbed + c0 + 2 * i),
                              v[2 * i + 1] + __ldg(bias + tensor * kEmbed + c0 + 2 * i + 1))
                 : 0u;
  if (kOut == kOutRows) {
    uint4* dst = reinterpret_cast<uint4*>(out + r * kEmbed + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  } else if (valid) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int h = c0 / kD + hh;
      size_t off;
      if (J.ptr) off = ((size_t)r * kH + h) * kD;
      else off = (((size_t)(r / J.P) * kH + h) * J.P + (size_t)(r % J.P)) * kD;
      uint4* dst = reinterpret_cast<uint4*>(out + off);
      dst[0] = make_uint4(w[8 * hh], w[8 * hh + 1], w[8 * hh + 2], w[8 * hh + 3]);
      dst[1] = make_uint4(w[8 * hh + 4], w[8 * hh + 5], w[8 * hh + 6], w[8 * hh + 7]);
    }
  }
}

// ======================================================= k_fused (one pass)

// The bias of the jet's pairs lives in shared memory as 8 f16 (one per head)
// per pair: the whole upper triangle when it fits (UCap pairs), otherwise one
// query block against all keys at a time. UCap is what is left of the
// per-CTA shared memory after the MLP tiles and the particles.
constexpr int kSmemLimit = 232448;  // 227 KB per CTA on sm_100

// MLP tiles of the fused kernel: kNG tile groups of 128 threads, kSL tiles
// in flight per group. Eight tiles in flight for P <= 128 (the bias triangle
// of such jets is small), four for P = 256 (room for wider jets'
// triangles). Every warp of the CTA works on the MLP's epilogues, which bound
// it: two groups with four tiles each measured 26 % slower than four groups
// with two.
template <int PM, int NG>
struct FusedLayout {
  static constexpr int kNG = NG;
  static constexpr int kSL = (PM <= 128 ? 8 : 4) / kNG;
  static constexpr int kFixed = (int)(sizeof(MlpSmem<kNG, kSL>) + sizeof(Particles<PM>)) + 1024;
  static constexpr int kUCap = (kSmemLimit - kFixed) / 16;
};

struct SmemUSink {
  uint4* U8;
  int cap;  // records the region holds
  __device__ __forceinline__ void operator()(int p, int, int, const float* u) const {
    if (!in_bounds(p >= 0 && p < cap)) return;
    U8[p] = make_uint4(pack_half2(u[0], u[1]), pack_half2(u[2], u[3]), pack_half2(u[4], u[5]),
                       pack_half2(u[6], u[7]));
  }
};

struct TriUBias {  // U of pair (i, j) at record max(i,j)(max(i,j)+1)/2 + min(i,j), 8 halves per record
  const __half* U;
  __device__ __forceinline__ TriBlock head(int h) const { return TriBlock{U + h}; }
};

struct RectUBias {  // U of (query i, key j) at record (i - i0) * m + j
  const __half* U;
  int i0, m;
  __device__ __forceinline__ RectBlock head(int h) const { return RectBlock{U + h, i0, m}; }
};

template <int PM, int NG>
struct FusedSmem {
  MlpSmem<FusedLayout<PM, NG>::kNG, FusedLayout<PM, NG>::kSL> mlp;
  Particles<PM> part;
  uint4 U8[FusedLayout<PM, NG>::kUCap];
  uint64_t proj_mbar;  // completion of the projections' MMAs (kProj)
};

// kProj: the jet's Q, K, V (X.q/k/v) are first computed from its embeddings
// (Pin: x, Wqkv, bqkv) and its output O (X.out) is finally projected to y
// (Pout: O, Wo, bo); see "per-jet projections inside k_fused" above.
template <int PM, int NG, bool kProj, class WA = MlpArgs>
__global__ void __launch_bounds__(NG * 128, 1) k_fused(JetArgs J, WA W, QkvArgs X, ProjArgs Pin,
                                                       ProjArgs Pout) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  FusedSmem<PM, NG>& S = *reinterpret_cast<FusedSmem<PM, NG>*>(smem_raw);
  constexpr int SL = FusedLayout<PM, NG>::kSL, MG = FusedLayout<PM, NG>::kNG;
  if (threadIdx.x == 0) {
    prefetch_jet(J, blockIdx.x);  // overlaps the weight loads
    if (kProj) {
      mbar_init(&S.proj_mbar, 1);
      fence_mbar_init();  // made visible by the barrier at the end of mlp_setup
    }
  }
  if constexpr (std::is_same<WA, MlpArgs>::value) {
    // the weights' loads are in flight while the first jet is staged
    WeightRegs wr;
    wr.load(W);
    if (blockIdx.x < J.N) stage_jet<PM>(S.part, J, blockIdx.x);
    mlp_setup<MG, SL>(S.mlp, wr);
  } else {
    if (blockIdx.x < J.N) stage_jet<PM>(S.part, J, blockIdx.x);
    mlp_setup_i8<MG, SL>(S.mlp, W);
  }
  // during attention the activation tiles hold K and V
  float* stage = reinterpret_cast<float*>(&S.mlp.A[0][0]);
  constexpr int kStageFloats = MG * SL * kTileM * kAK / 2;
  constexpr int kUCap = FusedLayout<PM, NG>::kUCap;
  uint32_t phase = 0u, pphase = 0u;
  bool aborted = false, proj_stuck = false;
  __nv_bfloat16* const PA = reinterpret_cast<__nv_bfloat16*>(stage);  // projection operands: rows,
  __nv_bfloat16* const PW = PA + kTileM * kEmbed;                     // then one weight chunk
  for (int n = blockIdx.x; n < J.N && !aborted; n += gridDim.x) {
    if (n != (int)blockIdx.x) stage_jet<PM>(S.part, J, n);
    if (threadIdx.x == 32) prefetch_jet(J, n + gridDim.x);  // this CTA's next jet
    // the jet's rows: padded slots n*P .. n*P+P-1, or its packed tokens
    const long long r_lo = J.ptr ? S.part.base : (long long)n * J.P;
    const long long r_hi = J.ptr ? r_lo + S.part.m : r_lo + J.P;
    if (kProj) {
      // Q, K, V of the jet's valid rows, one 128-row tile and one of the three weight chunks at a time
      for (long long r0 = r_lo; r0 < r_hi && !aborted; r0 += kTileM) {
        if (kStageFloats * 4 >= 4 * kTileM * kEmbed * 2) {
          // the stage holds the row tile and all three weight chunks: one round of loads, one wait
          proj_stage_tile_and_weights<kInRows, 3>(PA, PW, J, Pin.in, r0, r_hi, Pin.W);
          if (!proj_mma_n<3>(PA, PW, S.mlp.tmem_base, &S.proj_mbar, &pphase)) {
            aborted = proj_stuck = true;
            break;
          }
#pragma unroll 1
          for (int c = 0; c < 3; ++c)
            proj_store<kOutQKV>(S.mlp.tmem_base + 128u * c, Pin.bias, J, r0, r_hi,
                                c == 0 ? Pin.out0 : (c == 1 ? Pin.out1 : Pin.out2), c);
          tc_fence_before();
          __syncthreads();
          tc_fence_after();
          continue;
        }
        proj_stage_rows<kInRows>(PA, J, Pin.in, r0, r_hi);
        for (int c = 0; c < 3; ++c) {
          proj_stage_w(PW, Pin.W, c);
          if (!proj_mma(PA, PW, S.mlp.tmem_base, &S.proj_mbar, &pphase)) {
            aborted = proj_stuck = true;
            break;
          }
          proj_store<kOutQKV>(S.mlp.tmem_base, Pin.bias, J, r0, r_hi, c == 0 ? Pin.out0 : (c == 1 ? Pin.out1 : Pin.out2), c);
          tc_fence_before();  // TMEM read and the weight chunk consumed before the next one
          __syncthreads();
          tc_fence_after();
        }
      }
      if (aborted) break;
    } else {
      prefetch_qkv<PM>(S.part, J, X, n);  // read by the attention after the MLP
    }
    const int m = S.part.m;
    SmemUSink sink{S.U8, kUCap};
    const int np = m * (m + 1) / 2;
    if (np <= kUCap) {
      // the K and V of all heads are copied in while the MLP runs: into the
      // stage (the MLP keeps its operands in TMEM), or behind the bias
      // triangle when the stage is too small (P = 256 jets above 128)
      uint16_t* early = nullptr;
      if (m > 0 && kH * kv16_bytes(m) <= kStageFloats * 4) {
        early = reinterpret_cast<uint16_t*>(stage);
        stage_kv16<PM>(S.part, J, X, n, 0, kH, early);
      } else if (m > 0 && np + kH * kv16_bytes(m) / 16 <= kUCap) {
        early = reinterpret_cast<uint16_t*>(S.U8 + np);
        stage_kv16<PM>(S.part, J, X, n, 0, kH, early);
      }
      const bool ok = mlp_run<WA, MG, SL>(S.mlp, JetTiles<PM, TriPairs, true>{&S.part, np, TriPairs{}}, sink, &phase);
      aborted = __syncthreads_or(!ok) != 0;
      if (aborted) {
        if (early) cp_async_wait_all();
        break;
      }
      TriUBias ub{reinterpret_cast<const __half*>(S.U8)};
      attention_block<PM>(S.part, J, X, n, 0, m, stage, kStageFloats, ub, 0, kH, early);
    } else {
      const int qb = kUCap / m;
      for (int i0 = 0; i0 < m; i0 += qb) {
        const int i1 = min(m, i0 + qb);
        const bool ok = mlp_run<WA, MG, SL>(S.mlp, JetTiles<PM, RectPairs, true>{&S.part, (i1 - i0) * m, RectPairs{i0, m}}, sink, &phase);
        aborted = __syncthreads_or(!ok) != 0;
        if (aborted) break;
        RectUBias ub{reinterpret_cast<const __half*>(S.U8), i0, m};
        attention_block<PM>(S.part, J, X, n, i0, i1, stage, kStageFloats, ub);
      }
      if (aborted) break;
    }
    zero_masked_rows<PM>(S.part, J, X.out, n);
    __syncthreads();
    if (kProj) {
      // y = O Wo^T + bo for the jet's rows (masked slots 0)
      for (long long r0 = r_lo; r0 < r_hi && !aborted; r0 += kTileM) {
        proj_stage_tile_and_weights<kInHeads, 1>(PA, PW, J, X.out, r0, r_hi, Pout.W);
        if (!proj_mma_n<1>(PA, PW, S.mlp.tmem_base, &S.proj_mbar, &pphase)) {
          aborted = proj_stuck = true;
          break;
        }
        proj_store<kOutRows>(S.mlp.tmem_base, Pout.bias, J, r0, r_hi, Pout.out0, 0);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
      }
    }
  }
  if (kProj && proj_stuck && threadIdx.x == 0) (void)mbar_wait(&S.proj_mbar, pphase & 1u);  // bounded, before TMEM is freed
  mlp_teardown<MG, SL>(S.mlp, aborted, &phase);
}

// ================================================= k_fused_grid (balanced)
//
// The fused path spread over the whole GPU. One CTA per SM, all resident
// (cooperative launch); a caller-provided workspace holds two barrier
// counters and the bias records of every pair (8 f16 per pair, 16 bytes,
// 2 MB for 128 jets of ~40 particles: it stays in the 126 MB L2).
//   phase 0  every CTA derives the same jet table: the number of 128-row MLP
//            tiles of each jet and their exclusive prefix T (shared memory);
//   phase A  the T[N] tiles are split evenly over the CTAs; a CTA stages up
//            to kBatch jets of its range at a time and streams their tiles
//            through the MLP pipeline without draining between jets; each
//            row's 8 biases go to record T[n] * 128 + p of the workspace;
//   barrier  (bounded; counters reset by the last CTA to leave)
//   phase B  the 8 N (jet, head) attention items, weighted by the jet's tiles,
//            are split evenly over the CTAs and run with the bias read back
//            from the records.
// Phases A and B run in rounds of consecutive jets whose records fit
// kRoundTiles tiles (24 MB), a grid barrier between rounds, so that the
// records of a round stay in L2 however large the batch.
// Jets of any multiplicity up to P use the unordered triangle.

constexpr int kGridMaxJets = 8192;    // jet-table capacity (shared memory)
constexpr long long kRoundTiles = 12288;  // MLP tiles per round: 24 MB of bias records, kept in L2
constexpr size_t kWsHeader = 256;     // barrier counters, then the records

template <int PM>
struct GridCfg {
  static constexpr int kBatch = PM <= 128 ? 4 : 2;  // jets staged at once in phase A
};

template <int PM>
struct BatchInfo {  // the jets of one phase-A batch
  int K;                                  // jets in the batch
  int tbeg[GridCfg<PM>::kBatch + 1];      // prefix of their tiles within the batch
  int t_lo[GridCfg<PM>::kBatch];          // first tile of each jet taken by this CTA
  int npairs[GridCfg<PM>::kBatch];
  int jet[GridCfg<PM>::kBatch];
  long long rowbase[GridCfg<PM>::kBatch]; // record index of the jet's pair 0
};

template <int PM>
struct AttnBatch {  // the jets of one phase-B round, attended together
  int K;                                  // jets gathered (and staged)
  int Kf;                                 // leading jets whose data fit in the stage together
  int next;                               // first jet of the next round
  int jet[GridCfg<PM>::kBatch];
  int hl[GridCfg<PM>::kBatch], hh[GridCfg<PM>::kBatch];   // head range of each jet
  int uoff[GridCfg<PM>::kBatch], kvoff[GridCfg<PM>::kBatch];  // stage offsets (floats)
  int ib[GridCfg<PM>::kBatch + 1];        // prefix of (head, query) items
};

template <int PM>
struct FusedGridSmem {
  MlpSmem<4, 2> mlp;                       // activation tiles double as scratch in phases 0 and B
  Particles<PM> ring[GridCfg<PM>::kBatch];
  int T[kGridMaxJets + 1];                 // exclusive prefix of tiles per jet
  BatchInfo<PM> batch;
  AttnBatch<PM> ab;
  int warp_sums[32];
  int flag;
};

// Tiles of a staged batch, in order; row keys are record indices.
template <int PM>
struct BatchTiles {
  const Particles<PM>* ring;
  const BatchInfo<PM>* B;
  __device__ __forceinline__ int ntiles() const { return B->tbeg[B->K]; }
  __device__ __forceinline__ bool row(int bt, int r, int& p, int& a, int& b, float f[4]) const {
    int k = 0;
#pragma unroll
    for (int q = 1; q < GridCfg<PM>::kBatch; ++q) k += (q < B->K && B->tbeg[q] <= bt) ? 1 : 0;
    const int pl = (B->t_lo[k] + bt - B->tbeg[k]) * kTileM + r;
    if (pl >= B->npairs[k]) return false;
    TriPairs{}.map(pl, a, b);
    if (!in_bounds(a >= 0 && a <= b && b < ring[k].m)) return false;
    pair_feat<PM, true>(ring[k], min(a, b), max(a, b), f);
    p = (int)(B->rowbase[k] + pl);  // record index (fits: < 2^31 for N <= 8192, P <= 256)
    return true;
  }
};

struct RecordSink {  // the 8 biases of a pair as 8 f16 in one 16-byte record
  uint4* rec;
  long long cap;  // records of this launch: 128 per MLP tile
  __device__ __forceinline__ void operator()(int p, int, int, const float* u) const {
    if (!in_bounds(p >= 0 && p < cap)) return;
    rec[p] = make_uint4(pack_half2(u[0], u[1]), pack_half2(u[2], u[3]), pack_half2(u[4], u[5]),
                        pack_half2(u[6], u[7]));
  }
};

struct RecordUBias {  // U[h, i, j] from the jet's records in global memory (unordered-pair index)
  const __half* rec;   // record 0 of the jet, as halves
  __device__ __forceinline__ TriBlock head(int h) const { return TriBlock{rec + h}; }
};

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier over `nblk` resident CTAs on a counter that only grows
// within a launch. Bounded: returns false (status raised) if it runs out.
__device__ bool grid_barrier(unsigned long long* ctr, unsigned nblk, int* smem_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned long long old = atomicAdd(ctr, 1ull);
    const unsigned long long target = (old / nblk + 1) * nblk;
    bool ok = true;
    unsigned long long t0 = 0;
    for (uint32_t it = 0; ld_acquire_u64(ctr) < target; ++it) {
      if ((it & 63u) == 63u) {
        const unsigned long long now = global_ns();
        if (t0 == 0) {
          t0 = now;
        } else if (now - t0 > kWaitNs) {
          raise_status(kStTimeout);
          ok = false;
          break;
        }
      }
    }
    __threadfence();
    *smem_flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *smem_flag != 0;
}

// Nonzero bytes of a 32-bit word.
__device__ __forceinline__ int nonzero_bytes(uint32_t w) { return __popc(__vcmpne4(w, 0u)) >> 3; }

// Phase 0: the valid particles of every jet into T[1..N], all threads in
// parallel (bounds of a packed jet as stage_jets checks them; a padded mask
// read 16 bytes at a time when its rows allow it).
__device__ void jet_counts(const JetArgs& J, int* T) {
  const int tid = threadIdx.x, nthr = blockDim.x, N = J.N;
  if (J.ptr) {
#pragma unroll 4
    for (int n = tid; n < N; n += nthr) {
      const long long lo = J.ptr[n], hi = J.ptr[n + 1];
      T[n + 1] = (lo < 0 || hi < lo || hi > J.tokens || hi - lo > J.P) ? 0 : (int)(hi - lo);
    }
    return;
  }
  for (int n = tid; n < N; n += nthr) T[n + 1] = 0;
  __syncthreads();
  if ((J.P & 15) == 0 && (reinterpret_cast<uintptr_t>(J.mask) & 15) == 0) {
    const int cpj = J.P >> 4;  // 16-byte chunks per jet
    const uint4* mk = reinterpret_cast<const uint4*>(J.mask);
    const int nc = N * cpj;
#pragma unroll 4
    for (int c = tid; c < nc; c += nthr) {
      const uint4 w = mk[c];
      const int k = nonzero_bytes(w.x) + nonzero_bytes(w.y) + nonzero_bytes(w.z) + nonzero_bytes(w.w);
      if (k) atomicAdd(&T[c / cpj + 1], k);
    }
  } else {
    const int ne = N * J.P;
#pragma unroll 4
    for (int e = tid; e < ne; e += nthr)
      if (J.mask[e]) atomicAdd(&T[e / J.P + 1], 1);
  }
}

// This CTA's share (part of parts) of [base, base + bytes) into L2, in whole
// 16-byte units; nothing for an array that is not 16-byte aligned. One thread.
__device__ __forceinline__ void prefetch_slice(const void* base, size_t bytes, int part, int parts) {
  if (reinterpret_cast<uintptr_t>(base) & 15) return;
  const size_t chunk = ((bytes + parts - 1) / parts + 15) & ~(size_t)15;
  const size_t lo = chunk * (size_t)part;
  if (lo >= bytes) return;
  const size_t n = (bytes - lo < chunk ? bytes - lo : chunk) & ~(size_t)15;
  if (n) prefetch_l2(static_cast<const char*>(base) + lo, (uint32_t)n);
}

// kBiasOnly: phase 0 and phase A only (no barrier, no attention, counters
// untouched); CTA 0 also writes the tile prefix T[0..N] to Tout. The bias
// records then serve the backward pass.
template <int PM, bool kBiasOnly = false>
__global__ void __launch_bounds__(512, 1) k_fused_grid(JetArgs J, MlpArgs W, QkvArgs X, unsigned char* ws,
                                                       int* Tout) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  FusedGridSmem<PM>& S = *reinterpret_cast<FusedGridSmem<PM>*>(smem_raw);
  constexpr int NG = 4, SL = 2, JB = GridCfg<PM>::kBatch;
  unsigned long long* bar_ctr = reinterpret_cast<unsigned long long*>(ws);
  unsigned long long* exit_ctr = bar_ctr + 1;
  uint4* rec = reinterpret_cast<uint4*>(ws + kWsHeader);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, b = blockIdx.x;
  const int N = J.N;

  // the weights' loads are in flight during phase 0
  WeightRegs wr;
  wr.load(W);

  // ---------------------------------------------------------------- phase 0
  // multiplicities into T[n + 1], tiles per jet, then an exclusive scan
  jet_counts(J, S.T);
  if (tid == 0) S.T[0] = 0;
  __syncthreads();
  for (int n = tid; n < N; n += blockDim.x) {
    const int m = S.T[n + 1];
    S.T[n + 1] = (m * (m + 1) / 2 + kTileM - 1) / kTileM;
  }
  __syncthreads();
  {
    // each thread scans a contiguous chunk, warps then the block combine
    const int per = (N + blockDim.x - 1) / blockDim.x;
    const int c0 = 1 + tid * per, c1 = min(N + 1, c0 + per);
    int sum = 0;
    for (int i = c0; i < c1; ++i) sum += S.T[i];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) S.warp_sums[warp] = incl;
    __syncthreads();
    int woff = 0;
    for (int w = 0; w < warp; ++w) woff += S.warp_sums[w];
    int run = woff + incl - sum;
    __syncthreads();
    for (int i = c0; i < c1; ++i) {
      run += S.T[i];
      S.T[i] = run;
    }
  }
  __syncthreads();

  mlp_setup<NG, SL>(S.mlp, wr);
  uint32_t phase = 0u;
  bool aborted = false;

  // Rounds: consecutive jets whose records fit kRoundTiles tiles (at least
  // one jet), so that a round's records stay in L2 between its MLP and its
  // attention; a round's records are indexed from its first tile. The
  // bias-only launch keeps every record: one round. Every CTA takes the same
  // barriers in every round, a CTA that aborted included.
  for (int r0 = 0; r0 < N;) {
    const long long T0 = S.T[r0];
    int r1 = N;
    if (!kBiasOnly) {  // the largest r1 > r0 with T[r1] - T0 <= kRoundTiles
      int l = r0 + 1, r = N;
      while (l < r) {
        const int mid = (l + r + 1) >> 1;
        if (S.T[mid] - T0 <= kRoundTiles) l = mid; else r = mid - 1;
      }
      r1 = l;
    }
    const long long Tr = S.T[r1] - T0;
    const int Nr = r1 - r0;
    // ---------------------------------------------------------------- phase A
    {
      const long long lo = T0 + Tr * b / G, hi = T0 + Tr * (b + 1) / G;
      // first jet whose tiles reach past lo
      int n = r0;
      {
        int l = r0, r = r1;  // smallest n with T[n + 1] > lo
        while (l < r) {
          const int mid = (l + r) >> 1;
          if (S.T[mid + 1] > lo) r = mid; else l = mid + 1;
        }
        n = l;
      }
      while (!aborted && n < r1 && S.T[n] < hi) {
        // gather up to JB jets with tiles in [lo, hi)
        if (tid == 0) {
          int K = 0, acc = 0;
          int nn = n;
          while (K < JB && nn < r1 && S.T[nn] < hi) {
            const long long a0 = max((long long)S.T[nn], lo), a1 = min((long long)S.T[nn + 1], hi);
            if (a1 > a0) {
              S.batch.tbeg[K] = acc;
              S.batch.t_lo[K] = (int)(a0 - S.T[nn]);
              S.batch.rowbase[K] = (long long)(S.T[nn] - T0) * kTileM;
              S.batch.jet[K] = nn;
              acc += (int)(a1 - a0);
              ++K;
            }
            ++nn;
          }
          S.batch.tbeg[K] = acc;
          S.batch.K = K;
          S.flag = nn;  // next jet to look at
        }
        __syncthreads();
        const int K = S.batch.K;
        const int n_next = S.flag;
        stage_jets<PM, true>(S.ring, J, K, [&S](int k) { return S.batch.jet[k]; });
        if (tid == 0)
          for (int k = 0; k < K; ++k) S.batch.npairs[k] = S.ring[k].m * (S.ring[k].m + 1) / 2;
        __syncthreads();
        RecordSink sink{rec, Tr * kTileM};
        const bool ok = mlp_pass<NG, SL>(S.mlp, BatchTiles<PM>{S.ring, &S.batch}, sink, &phase);
        aborted = __syncthreads_or(!ok) != 0;
        n = n_next;
      }
    }

    if (kBiasOnly) break;

    // --------------------------------------------------------------- barrier
    const bool passed = grid_barrier(bar_ctr, (unsigned)G, &S.flag);
    aborted = aborted || !passed;

    // phase B's share of this CTA: item (n, h) of the round costs tiles_n + 1
    // and starts at 8 (T[n] - T0 + n - r0) + h (tiles_n + 1)
    const long long CB = 8ll * (Tr + Nr);
    const long long loB = CB * b / G, hiB = CB * (b + 1) / G;
    int nB = r0;
    {
      int l = r0, r = r1;  // smallest n whose items end past loB
      while (l < r) {
        const int mid = (l + r) >> 1;
        if (8ll * ((long long)(S.T[mid + 1] - T0) + mid + 1 - r0) > loB) r = mid; else l = mid + 1;
      }
      nB = l;
    }

    // ---------------------------------------------------------------- phase B
    if (!aborted) {
      const long long lo = loB, hi = hiB;
      int n = nB;
      float* stage = reinterpret_cast<float*>(&S.mlp.A[0][0]);
      constexpr int kStageFloats = NG * SL * kTileM * kAK / 2;
      AttnBatch<PM>& A = S.ab;
      while (n < r1 && 8ll * ((long long)(S.T[n] - T0) + n - r0) < hi) {
        // up to JB jets with heads in [lo, hi), staged (slots only) together
        if (tid == 0) {
          int K = 0, nn = n;
          while (K < JB && nn < r1 && 8ll * ((long long)(S.T[nn] - T0) + nn - r0) < hi) {
            const long long base = 8ll * ((long long)(S.T[nn] - T0) + nn - r0);
            const long long c = (long long)(S.T[nn + 1] - S.T[nn]) + 1;
            int h_lo = 0, h_hi = 0;
            for (int h = 0; h < kH; ++h) {
              const long long st = base + h * c;
              if (st < lo) h_lo = h + 1;
              if (st < hi) h_hi = h + 1;
            }
            if (h_lo < h_hi) {
              A.jet[K] = nn;
              A.hl[K] = h_lo;
              A.hh[K] = h_hi;
              ++K;
            }
            ++nn;
          }
          A.K = K;
          A.next = nn;
        }
        __syncthreads();
        const int K = A.K;
        stage_jets<PM, false>(S.ring, J, K, [&A](int k) { return A.jet[k]; });
        // the leading jets whose records and K/V fit in the stage together
        if (tid == 0) {
          int used = 0, items = 0, Kf = 0;
          for (; Kf < K; ++Kf) {
            const int m = S.ring[Kf].m, hr = A.hh[Kf] - A.hl[Kf];
            const int need = m * (m + 1) / 2 * 4 + hr * (kv16_bytes(m) / 4);
            if (used + need > kStageFloats) break;
            A.uoff[Kf] = used;
            A.kvoff[Kf] = used + m * (m + 1) / 2 * 4;
            A.ib[Kf] = items;
            used += need;
            items += hr * ((m + 15) >> 4);
          }
          A.ib[Kf] = items;
          A.Kf = Kf;
          // jets that did not fit are staged again in the next round
          if (Kf > 0 && Kf < K) A.next = A.jet[Kf];
          else if (Kf == 0 && K > 1) A.next = A.jet[1];
        }
        __syncthreads();
        const int Kf = A.Kf, n_next = A.next;
        if (K == 0) {
          // [lo, hi) lies inside one jet's head: nothing to do in this round
        } else if (Kf == 0) {
          // one jet too wide for the stage: its bias is read from the records
          const int nj = A.jet[0];
          RecordUBias ub{reinterpret_cast<const __half*>(rec + (size_t)(S.T[nj] - T0) * kTileM)};
          attention_block<PM>(S.ring[0], J, X, nj, 0, S.ring[0].m, stage, kStageFloats, ub, A.hl[0], A.hh[0]);
          if (A.hl[0] == 0) zero_masked_rows<PM>(S.ring[0], J, X.out, nj);
        } else {
          // warp items: (jet, head, 16-query tile); Q fragments are loaded ahead
          const int items = A.ib[Kf], nwarp = (int)(blockDim.x >> 5);
          auto qload = [&](int it, uint32_t* f) {
            int k = 0;
  #pragma unroll
            for (int q = 1; q < JB; ++q) k += (q < Kf && A.ib[q] <= it) ? 1 : 0;
            const Particles<PM>& P = S.ring[k];
            const int m = P.m, tiles = (m + 15) >> 4, loc = it - A.ib[k];
            const int h = A.hl[k] + loc / tiles, i0 = (loc % tiles) * 16, nj = A.jet[k];
            q_frag(i0, min(16, m - i0), [&](int i) { return X.q + qkv_off<PM>(P, J, nj, h, i); }, f);
          };
          uint32_t a[4] = {0u, 0u, 0u, 0u};
          if (warp < items) qload(warp, a);
          for (int k = 0; k < Kf; ++k) {
            const int nj = A.jet[k], m = S.ring[k].m, np = m * (m + 1) / 2;
            const uint4* jrec = rec + (size_t)(S.T[nj] - T0) * kTileM;
            uint4* U8 = reinterpret_cast<uint4*>(stage + A.uoff[k]);
            for (int r0 = tid; r0 < np; r0 += 4 * (int)blockDim.x) {
              uint4 v[4];
  #pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int r = r0 + u * (int)blockDim.x;
                v[u] = r < np ? __ldcg(jrec + r) : make_uint4(0, 0, 0, 0);
              }
  #pragma unroll
              for (int u = 0; u < 4; ++u)
                if (r0 + u * (int)blockDim.x < np) U8[r0 + u * (int)blockDim.x] = v[u];
            }
            stage_kv16<PM>(S.ring[k], J, X, nj, A.hl[k], A.hh[k] - A.hl[k], reinterpret_cast<uint16_t*>(stage + A.kvoff[k]));
          }
          cp_async_wait_all();
          __syncthreads();
          for (int it = warp; it < items; it += nwarp) {
            uint32_t an[4] = {0u, 0u, 0u, 0u};
            if (it + nwarp < items) qload(it + nwarp, an);
            int k = 0;
  #pragma unroll
            for (int q = 1; q < JB; ++q) k += (q < Kf && A.ib[q] <= it) ? 1 : 0;
            const Particles<PM>& P = S.ring[k];
            const int m = P.m, tiles = (m + 15) >> 4, loc = it - A.ib[k];
            const int hh = loc / tiles, i0 = (loc % tiles) * 16, h = A.hl[k] + hh, nj = A.jet[k];
            const uint16_t* kh = reinterpret_cast<const uint16_t*>(stage + A.kvoff[k]) + hh * (kv16_bytes(m) / 2);
            const TriBlock ub{reinterpret_cast<const __half*>(stage + A.uoff[k]) + h};
            attend_tile16(
                kh, kh + round16(m) * 16, m, i0, min(16, m - i0), a,
                [&](int i) { return X.out + qkv_off<PM>(P, J, nj, h, i); }, ub);
  #pragma unroll
            for (int e = 0; e < 4; ++e) a[e] = an[e];
          }
          for (int k = 0; k < Kf; ++k)
            if (A.hl[k] == 0) zero_masked_rows<PM>(S.ring[k], J, X.out, A.jet[k]);
        }
        __syncthreads();
        n = n_next;
      }
    }

    r0 = r1;
    if (r0 < N) {  // the next round overwrites the records this one read
      const bool again = grid_barrier(bar_ctr, (unsigned)G, &S.flag);
      aborted = aborted || !again;
    }
  }

  if (kBiasOnly) {
    if (b == 0)
      for (int n = tid; n <= N; n += blockDim.x) Tout[n] = S.T[n];
    mlp_teardown<NG, SL>(S.mlp, aborted, &phase);
    return;
  }

  mlp_teardown<NG, SL>(S.mlp, aborted, &phase);
  // the last CTA to leave resets both counters for the next launch
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(exit_ctr, 1ull) == (unsigned long long)(G - 1)) {
      atomicExch(bar_ctr, 0ull);
      atomicExch(exit_ctr, 0ull);
      __threadfence();
    }
  }
}

// Workspace bytes of the balanced path: header + one 16-byte record per row
// of every jet's tiles (bounded from N, P and, packed, the token count).
__host__ __device__ inline size_t grid_workspace_bytes(int N, int P, long long tokens, bool packed) {
  const long long per_jet_tiles = ((long long)P * (P + 1) / 2 + kTileM - 1) / kTileM;
  long long rows = (long long)N * per_jet_tiles * kTileM;
  if (packed) {
    // sum over jets of ceil(m(m+1)/2 / 128) * 128 <= tokens (P + 1) / 2 + 127 N
    const long long alt = tokens * (P + 1) / 2 + (long long)(kTileM - 1) * N + kTileM;
    rows = alt < rows ? alt : rows;
  }
  return kWsHeader + (size_t)rows * 16;
}


// ============================================== k_fused_cluster (4-CTA jets)
//
// The fused path for batches of few jets, where one CTA per jet would wait
// for the widest one: a thread-block cluster of 4 CTAs takes up to 4 jets
// (the host deals the jets over as many clusters as run at once).
//   - every CTA stages the cluster's jets; their unordered pairs, one jet
//     after another, are packed into 128-row MLP tiles (no padding between
//     jets), split evenly over the 4 CTAs (contiguous tile ranges);
//   - a tile row's 8 biases go straight to the CTA that owns their heads:
//     CTA q keeps heads 2q, 2q + 1 of every pair of the 4 jets, 4 bytes per
//     pair, written through distributed shared memory (st.shared::cluster);
//   - a cluster barrier publishes them; CTA q then attends heads 2q, 2q + 1
//     of each jet from its own shared memory.
// When the 4 jets' pairs do not fit the triangles together, consecutive
// groups of them that fit run one after another (one P <= 128 jet always
// fits). Cluster barriers are hardware barriers that every CTA reaches the
// same number of times on every path (a CTA whose wait ran out still takes
// them); the first one makes sure all 4 CTAs run before any remote store:
// each CTA arrives on it at its start and waits on it right before its MLP.

constexpr int kCJ = 4;                // jets and CTAs per cluster
constexpr int kClusterMaxJets = 256;  // batch size the jet table holds
constexpr int kMaxJetTiles = (128 * 129 / 2 + kTileM - 1) / kTileM;  // MLP tiles of a full P = 128 jet

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}
// The two halves of a cluster barrier that publishes nothing (it only tells
// that every CTA of the cluster runs): arrive early, wait where it matters.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

template <int PM>
struct ClusterHead {
  MlpSmem<4, 2> mlp;  // activation tiles double as the attention stage
  Particles<PM> ring[kCJ];
  int tri_off[kCJ + 1];  // prefix of the jets' pairs
  int lo, hi;            // this CTA's tiles of the current group's list
  int G;                 // jets in the current group
  int kvoff[kCJ + 1];    // staged K/V of each jet of the group (halves) in the attention
  int ib[kCJ + 1];       // prefix of each group jet's (head, query tile) items
  int jets[kCJ];         // this cluster's jets
  int cnt[kClusterMaxJets + 1];  // multiplicity of every jet of the batch (cnt[n + 1])
  int bin[kMaxJetTiles + 2];     // jets per tile count, then the next free rank of each
  int order[kClusterMaxJets];    // jets by decreasing MLP tiles
};

template <int PM>
struct ClusterSmem {
  static constexpr int kHead = ((int)sizeof(ClusterHead<PM>) + 15) & ~15;
  static constexpr int kUCap = (kSmemLimit - kHead - 1024) / 16 * 4;
  ClusterHead<PM> h;
  alignas(16) uint32_t U[kUCap];  // heads 2q, 2q + 1 of every pair (f16x2), jet after jet; or 16-byte 8-head records
};

// The rows of this CTA's tiles of the group's jets: the jets' unordered
// pairs one jet after another, packed into 128-row tiles without padding
// between jets; the row's index there is also the sink key (the pair's index
// in the group's triangles).
template <int PM>
struct ClusterTiles {
  const ClusterHead<PM>* H;
  int g0;  // the group's first jet
  __device__ __forceinline__ int ntiles() const { return H->hi - H->lo; }
  __device__ __forceinline__ bool row(int t, int r, int& p, int& a, int& b, float f[4]) const {
    const int pg = (H->lo + t) * kTileM + r;
    if (pg >= H->tri_off[kCJ]) return false;
    int k = 0;
#pragma unroll
    for (int q = 1; q < kCJ; ++q) k += H->tri_off[q] <= pg ? 1 : 0;
    const int pl = pg - H->tri_off[k];
    const Particles<PM>& P = H->ring[g0 + k];
    const int m = P.m;
    if (!in_bounds(pl < m * (m + 1) / 2)) return false;
    TriPairs{}.map(pl, a, b);
    if (!in_bounds(a >= 0 && a <= b && b < m)) return false;
    pair_feat<PM, true>(P, a, b, f);
    p = pg;
    return true;
  }
};

struct ClusterUSink {  // pair p's heads 2q, 2q + 1 to CTA q's entry p
  uint32_t base[kCJ];  // shared::cluster address of U in each CTA
  int cap;
  __device__ __forceinline__ void operator()(int p, int, int, const float* u) const {
    if (!in_bounds(p >= 0 && p < cap)) return;
#pragma unroll
    for (int q = 0; q < kCJ; ++q) st_cluster_u32(base[q] + 4u * (uint32_t)p, pack_half2(u[2 * q], u[2 * q + 1]));
  }
};

struct ClusterUBias {  // heads h0, h0 + 1 of one jet's triangle, 2 halves per pair
  const __half* U;
  int h0;
  __device__ __forceinline__ TriBlockS<2> head(int h) const { return TriBlockS<2>{U + (h - h0)}; }
};

template <int PM>
__global__ void __launch_bounds__(512, 1) k_fused_cluster(JetArgs J, MlpArgs W, QkvArgs X) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ClusterSmem<PM>& S = *reinterpret_cast<ClusterSmem<PM>*>(smem_raw);
  ClusterHead<PM>& H = S.h;
  constexpr int NG = 4, SL = 2;
  constexpr int kUCap = ClusterSmem<PM>::kUCap;
  const int q = (int)cluster_ctarank();
  const int c = blockIdx.x / kCJ, ncl = gridDim.x / kCJ;
  cluster_arrive_relaxed();  // this CTA runs; waited for before the first remote store
  if (threadIdx.x == 0) {  // this CTA's slice of the momenta into L2, for the staging below
    const size_t bytes = (J.ptr ? (size_t)J.tokens : (size_t)J.N * J.P) * 4;
    prefetch_slice(J.E, bytes, blockIdx.x, gridDim.x);
    prefetch_slice(J.px, bytes, blockIdx.x, gridDim.x);
    prefetch_slice(J.py, bytes, blockIdx.x, gridDim.x);
    prefetch_slice(J.pz, bytes, blockIdx.x, gridDim.x);
  }
  // warps 1.. load the weights (in flight while the jets are counted) and
  // set up the MLP while warp 0 sorts the jets
  const int wt = (int)threadIdx.x - 32, wn = (int)blockDim.x - 32;
  WeightRegs wr;
  if (wt >= 0) wr.load(W, wt, wn);
  // Every CTA counts every jet and sorts them by MLP tiles, largest first,
  // ties in jet order (a stable counting sort: every CTA must come to the
  // same order); cluster c takes the jets at ranks c, 2 ncl - 1 - c,
  // 2 ncl + c, ... (a snake over the clusters), so the clusters' tile sums
  // come out close.
  for (int t = threadIdx.x; t < kMaxJetTiles + 2; t += blockDim.x) H.bin[t] = 0;
  jet_counts(J, H.cnt);
  __syncthreads();
  auto jet_tiles = [&H](int n) {
    const int m = H.cnt[n + 1];
    return min(kMaxJetTiles, (m * (m + 1) / 2 + kTileM - 1) / kTileM);
  };
  for (int n = threadIdx.x; n < J.N; n += blockDim.x) atomicAdd(&H.bin[jet_tiles(n)], 1);
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    {  // first rank of each tile count, largest counts first: an exclusive
       // scan over the bins from kMaxJetTiles down, kPer bins per lane
      constexpr int kPer = (kMaxJetTiles + 1 + 31) / 32;
      int v[kPer], sum = 0;
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int t = kMaxJetTiles - (lane * kPer + e);
        v[e] = t >= 0 ? H.bin[t] : 0;
        sum += v[e];
      }
      int incl = sum;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += o;
      }
      int run = incl - sum;
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int t = kMaxJetTiles - (lane * kPer + e);
        if (t >= 0) H.bin[t] = run;
        run += v[e];
      }
    }
    __syncwarp();
    // 32 jets at a time in jet order: equal counts within a chunk take
    // consecutive ranks by lane, and the last of them advances the count's
    // next free rank for the following chunks
    for (int n0 = 0; n0 < J.N; n0 += 32) {
      const int n = n0 + lane;
      const int t = n < J.N ? jet_tiles(n) : kMaxJetTiles + 1;
      const unsigned same = __match_any_sync(0xffffffffu, t);
      const int before = __popc(same & ((1u << lane) - 1u));
      const int pos = H.bin[t] + before;
      __syncwarp();
      if (n < J.N) {
        H.order[pos] = n;
        if ((same >> lane) == 1u) H.bin[t] = pos + 1;  // highest lane of the group
      }
      __syncwarp();
    }
    tmem_alloc(&H.mlp.tmem_base, kTmemCols(NG, SL));
  } else {
    mlp_setup_part<NG, SL>(H.mlp, wr, wt, wn);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  int K = 0;
#pragma unroll
  for (int r = 0; r < kCJ; ++r) {
    const int p = r * ncl + ((r & 1) ? ncl - 1 - c : c);
    if (p < J.N) {
      if (threadIdx.x == 0) H.jets[K] = H.order[p];
      ++K;
    }
  }
  __syncthreads();
  stage_jets<PM, true>(H.ring, J, K, [&H](int k) { return H.jets[k]; });
  // groups of consecutive jets whose triangles fit together (identical in
  // every CTA of the cluster: the same jets, the same order); thread 0 lays
  // out the group starting at jet g0
  auto plan = [&](int g0) {
    if (threadIdx.x == 0) {
      int G = 0, pairs = 0;
      while (g0 + G < K) {
        const int m = H.ring[g0 + G].m, np = m * (m + 1) / 2;
        if (G > 0 && pairs + np > kUCap) break;
        H.tri_off[G] = pairs;
        pairs += np;
        ++G;
      }
      for (int k = G; k <= kCJ; ++k) H.tri_off[k] = pairs;
      const int tiles = (pairs + kTileM - 1) / kTileM;  // the group's pairs, packed
      H.kvoff[0] = 0;
      H.ib[0] = 0;
      for (int k = 0; k < kCJ; ++k) {
        const int m = k < G ? H.ring[g0 + k].m : 0;
        H.kvoff[k + 1] = H.kvoff[k] + (m > 0 ? kv16_bytes(m) : 0);  // two heads of kv16_bytes / 2 halves
        H.ib[k + 1] = H.ib[k] + (m > 0 ? 2 * ((m + 15) >> 4) : 0);
      }
      H.lo = tiles * q / kCJ;
      H.hi = tiles * (q + 1) / kCJ;
      H.G = G;
    }
  };
  plan(0);
  __syncthreads();
  cluster_wait();  // all 4 CTAs run: their shared memory may be written
  float* stage = reinterpret_cast<float*>(&H.mlp.A[0][0]);
  uint32_t phase = 0u;
  bool aborted = false;
  ClusterUSink sink;
  {
    const uint32_t local = smem_u32(S.U);
#pragma unroll
    for (int cc = 0; cc < kCJ; ++cc) sink.base[cc] = map_shared_rank(local, (uint32_t)cc);
    sink.cap = kUCap;
  }
  for (int g0 = 0; g0 < K;) {
    __syncthreads();
    const int G = H.G;
    // heads 2q, 2q + 1 of the group's jets at once: K and V of every (jet,
    // head) are copied into the stage while the MLP runs (its operands live
    // in TMEM), then the warps take (jet, head, 16-query tile) items, the
    // next item's Q fragment loaded ahead; the first Q fragment is loaded
    // before the barrier that waits for the other CTAs' MLP.
    uint16_t* kv = reinterpret_cast<uint16_t*>(stage);
    if (!aborted)
      for (int k = 0; k < G; ++k)
        if (H.ring[g0 + k].m > 0) stage_kv16<PM>(H.ring[g0 + k], J, X, H.jets[g0 + k], 2 * q, 2, kv + H.kvoff[k]);
    if (!aborted) {
      const bool ok = mlp_pass<NG, SL>(H.mlp, ClusterTiles<PM>{&H, g0}, sink, &phase);
      aborted = !ok;
    }
    aborted = __syncthreads_or(aborted) != 0;
    const int* kvoff = H.kvoff;
    const int* ib = H.ib;
    const int items = ib[kCJ], warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    auto locate = [&](int it, int& k, int& h, int& i0) {
      k = 0;
#pragma unroll
      for (int cc = 1; cc < kCJ; ++cc) k += ib[cc] <= it ? 1 : 0;
      const int tiles = (H.ring[g0 + k].m + 15) >> 4, loc = it - ib[k];
      h = 2 * q + loc / tiles;
      i0 = (loc % tiles) * 16;
    };
    auto qload = [&](int it, uint32_t* f) {
      int k, h, i0;
      locate(it, k, h, i0);
      const Particles<PM>& P = H.ring[g0 + k];
      q_frag(i0, min(16, P.m - i0), [&](int i) { return X.q + qkv_off<PM>(P, J, H.jets[g0 + k], h, i); }, f);
    };
    uint32_t a[4] = {0u, 0u, 0u, 0u};
    if (!aborted && warp < items) qload(warp, a);
    cluster_sync_all();  // every CTA's stores into this one are visible
    if (aborted) cp_async_wait_all();  // no copy may still land after the kernel
    if (!aborted) {
      cp_async_wait_all();
      __syncthreads();
      for (int it = warp; it < items; it += nwarp) {
        uint32_t an[4] = {0u, 0u, 0u, 0u};
        if (it + nwarp < items) qload(it + nwarp, an);
        int k, h, i0;
        locate(it, k, h, i0);
        const Particles<PM>& P = H.ring[g0 + k];
        const int m = P.m;
        const uint16_t* kh = kv + kvoff[k] + (h - 2 * q) * (kv16_bytes(m) / 2);
        const ClusterUBias ub{reinterpret_cast<const __half*>(S.U + H.tri_off[k]), 2 * q};
        attend_tile16(
            kh, kh + round16(m) * 16, m, i0, min(16, m - i0), a,
            [&](int i) { return X.out + qkv_off<PM>(P, J, H.jets[g0 + k], h, i); }, ub.head(h));
#pragma unroll
        for (int e = 0; e < 4; ++e) a[e] = an[e];
      }
    }
    g0 += G;
    if (g0 < K) {
      __syncthreads();  // the stage and this group's tables are free again
      plan(g0);
      __syncthreads();
      cluster_sync_all();  // no CTA still reads the triangles the next group overwrites
    }
  }
  if (!aborted && q < K) zero_masked_rows<PM>(H.ring[q], J, X.out, H.jets[q]);
  mlp_teardown<NG, SL>(H.mlp, aborted, &phase);
}

// ================================================= k_wait_selftest (diagnostic)
//
// Exercises the failure path of the library's bounded waits: an mbarrier
// wait that nothing completes and a grid barrier whose target nothing
// reaches, both with the library's own wait code and limit (2 s each). Each
// runs out, raises kStTimeout and returns; the kernel then ends normally and
// the context stays usable. One CTA of 32 threads.
__device__ unsigned long long g_selftest_ctr[2];

__global__ void k_wait_selftest() {
  __shared__ uint64_t bar;
  __shared__ int flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  (void)mbar_wait(&bar, 0);  // no arrival: runs out after the library's limit
  __syncthreads();
  // a grid barrier for two CTAs, launched as one: the target is never reached
  (void)grid_barrier(&g_selftest_ctr[0], 2u, &flag);
  if (threadIdx.x == 0) g_selftest_ctr[0] = 0;  // leave the counter as found
}

}  // namespace pb
