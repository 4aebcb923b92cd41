// pairbias.cu -- C-ABI entry points of the pair-bias library (include/pairbias.h).
//
// Host side only validates arguments, picks the template instance for P
// (<= 128 or <= 256), sizes a persistent grid from the SM count and the
// occupancy of that instance, and launches the entry point's kernels (one;
// three for pair_block_forward, four for pair_attention_backward) on the
// caller's stream. Nothing is allocated and nothing is synchronised here.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "pairbias.h"
#include "pb_backward.cuh"
#include "pb_kernels.cuh"

namespace {

thread_local char g_err[512] = "";

pb_status fail(pb_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Per-device launch facts, filled once per device and kernel instance.
constexpr int kMaxDev = 64;
struct DevInfo {
  int sms = 0;
  int clusters = -1;  // co-resident 4-CTA clusters of the cluster kernel (-1: not asked yet)
};
DevInfo g_dev[kMaxDev];
std::mutex g_mu;

pb_status device_sms(int* dev_out, int* sms_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(PB_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDev) return fail(PB_ECUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev[dev].sms == 0) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(PB_ECUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    g_dev[dev].sms = sms;
  }
  *dev_out = dev;
  *sms_out = g_dev[dev].sms;
  return PB_OK;
}

// Resident CTAs per SM of a kernel instance on a device, found once (the
// shared-memory attribute is raised at the same time) and cached, so that a
// launch costs no runtime queries after the first.
constexpr int kMaxKernels = 64;
struct KernelFacts {
  const void* fn = nullptr;
  int per_sm[kMaxDev] = {};
};
KernelFacts g_kernels[kMaxKernels];

pb_status resident_per_sm(const void* fn, int dev, size_t smem, int threads, int* per_sm_out) {
  std::lock_guard<std::mutex> lk(g_mu);
  int slot = -1;
  for (int i = 0; i < kMaxKernels; ++i) {
    if (g_kernels[i].fn == fn || g_kernels[i].fn == nullptr) {
      slot = i;
      break;
    }
  }
  if (slot < 0) return fail(PB_ECUDA, "kernel cache full");
  KernelFacts& f = g_kernels[slot];
  if (f.fn == nullptr) f.fn = fn;
  if (f.per_sm[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(PB_ECUDA, "cudaFuncSetAttribute(%zu B smem): %s", smem, cudaGetErrorString(e));
    // every kernel of the library asks for the same (maximal) shared-memory
    // carveout, so that consecutive launches need no L1/shared repartition
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return fail(PB_ECUDA, "cudaFuncSetAttribute(carveout): %s", cudaGetErrorString(e));
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem);
    if (e != cudaSuccess) return fail(PB_ECUDA, "occupancy query: %s", cudaGetErrorString(e));
    if (per_sm < 1) return fail(PB_ECUDA, "kernel does not fit on an SM (%zu B smem)", smem);
    f.per_sm[dev] = per_sm;
  }
  *per_sm_out = f.per_sm[dev];
  return PB_OK;
}

// The persistent grid size of `kernel`: SMs x resident CTAs, at most `work`.
template <class K>
pb_status prepare(K kernel, size_t smem, int threads, int work, int* grid) {
  int dev = 0, sms = 0, per_sm = 0;
  pb_status st = device_sms(&dev, &sms);
  if (st != PB_OK) return st;
  if ((st = resident_per_sm((const void*)kernel, dev, smem, threads, &per_sm)) != PB_OK) return st;
  long long g = (long long)sms * per_sm;
  if (g > work) g = work;
  *grid = (int)(g < 1 ? 1 : g);
  return PB_OK;
}

pb_status launched(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PB_ECUDA, "%s launch: %s", what, cudaGetErrorString(e));
  return PB_OK;
}

pb_status check_jets(const pb_jets* j, pb::JetArgs* out) {
  if (!j) return fail(PB_EINVAL, "jets is NULL");
  if (j->N < 0) return fail(PB_EINVAL, "N = %d < 0", j->N);
  if (j->P < 1 || j->P > 256) return fail(PB_EUNSUPPORTED, "P = %d outside [1, 256]", j->P);
  *out = pb::JetArgs{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, j->P, 0};
  if (j->N == 0) return PB_OK;  // nothing to read or write: pointers may be NULL
  if (!j->E || !j->px || !j->py || !j->pz) return fail(PB_EINVAL, "a momentum pointer is NULL");
  if (!aligned(j->E, 4) || !aligned(j->px, 4) || !aligned(j->py, 4) || !aligned(j->pz, 4))
    return fail(PB_EINVAL, "momentum arrays must be 4-byte aligned");
  if (j->ptr) {
    if (!aligned(j->ptr, 4)) return fail(PB_EINVAL, "ptr must be 4-byte aligned");
    if (j->tokens < 0) return fail(PB_EINVAL, "tokens = %lld < 0", (long long)j->tokens);
  } else if (!j->mask) {
    return fail(PB_EINVAL, "padded layout needs a mask (or pass ptr for the packed layout)");
  }
  *out = pb::JetArgs{j->E, j->px, j->py, j->pz, j->ptr ? nullptr : j->mask, j->ptr, j->N, j->P,
                     (long long)j->tokens};
  return PB_OK;
}

pb_status check_mlp(const pb_mlp* w, pb::MlpArgs* out) {
  if (!w) return fail(PB_EINVAL, "mlp is NULL");
  if (!w->W1 || !w->b1 || !w->W2 || !w->b2 || !w->W3 || !w->b3 || !w->W4 || !w->b4)
    return fail(PB_EINVAL, "an MLP parameter pointer is NULL");
  if (!aligned(w->W1, 16) || !aligned(w->W2, 16) || !aligned(w->W3, 16) || !aligned(w->W4, 16))
    return fail(PB_EINVAL, "the MLP weight matrices W1..W4 must be 16-byte aligned");
  *out = pb::MlpArgs{w->W1, w->b1, w->W2, w->b2, w->W3, w->b3, w->W4, w->b4};
  return PB_OK;
}

pb_status check_mlp_i8(const pb_mlp_i8* w, pb::MlpI8Args* out) {
  if (!w) return fail(PB_EINVAL, "mlp is NULL");
  if (!w->W1 || !w->b1 || !w->T2 || !w->T3 || !w->T4 || !w->a2 || !w->a3 || !w->a4 || !w->b2 || !w->b3 || !w->b4)
    return fail(PB_EINVAL, "an int8 MLP parameter pointer is NULL");
  if (!aligned(w->T2, 16) || !aligned(w->T3, 16) || !aligned(w->T4, 16))
    return fail(PB_EINVAL, "the weight code arrays must be 16-byte aligned");
  *out = pb::MlpI8Args{w->W1, w->b1, w->T2, w->T3, w->T4, w->a2, w->a3, w->a4, w->b2, w->b3, w->b4};
  return PB_OK;
}

constexpr int kGroups = 4;  // tensor-core tile groups per CTA (128 threads each)

template <int PM>
pb_status run_pairfeat(const pb::JetArgs& J, float* feat, cudaStream_t s) {
  auto k = pb::k_pairfeat<PM>;
  const size_t smem = sizeof(pb::Particles<PM>);
  int grid = 0;
  pb_status st = prepare(k, smem, 256, J.N, &grid);
  if (st != PB_OK) return st;
  k<<<grid, 256, smem, s>>>(J, feat);
  return launched("k_pairfeat");
}

template <int PM, bool F32, class WA = pb::MlpArgs>
pb_status run_mlp_bias(const pb::JetArgs& J, const WA& W, void* U, cudaStream_t s) {
  auto k = pb::k_mlp_bias<PM, kGroups, F32, WA>;
  const size_t smem = sizeof(pb::MlpBiasSmem<PM, kGroups>);
  int grid = 0;
  pb_status st = prepare(k, smem, kGroups * 128, J.N, &grid);
  if (st != PB_OK) return st;
  k<<<grid, kGroups * 128, smem, s>>>(J, W, U);
  return launched("k_mlp_bias");
}

template <int PM>
pb_status run_attn_bias(const pb::JetArgs& J, const pb::QkvArgs& X, const uint16_t* U, cudaStream_t s) {
  auto k = pb::k_attn_bias<PM>;
  const size_t smem = sizeof(pb::AttnSmem<PM>);
  int grid = 0;
  pb_status st = prepare(k, smem, 256, J.N, &grid);
  if (st != PB_OK) return st;
  k<<<grid, 256, smem, s>>>(J, X, U);
  return launched("k_attn_bias");
}

template <int PM, bool kProj = false, class WA = pb::MlpArgs>
pb_status run_fused(const pb::JetArgs& J, const WA& W, const pb::QkvArgs& X, cudaStream_t s,
                    const pb::ProjArgs& Pin = pb::ProjArgs{}, const pb::ProjArgs& Pout = pb::ProjArgs{}) {
  auto k = pb::k_fused<PM, kGroups, kProj, WA>;
  const size_t smem = sizeof(pb::FusedSmem<PM, kGroups>);
  int grid = 0;
  pb_status st = prepare(k, smem, kGroups * 128, J.N, &grid);
  if (st != PB_OK) return st;
  k<<<grid, kGroups * 128, smem, s>>>(J, W, X, Pin, Pout);
  return launched(kProj ? "k_fused (with projections)" : "k_fused");
}

// The 4-CTA cluster kernel takes batches of at most this many jets per SM
// (one jet per CTA); larger batches already balance over the persistent CTAs.
// Small batches take it too: dealt one jet per cluster, each jet's MLP is
// split over 4 CTAs.
constexpr int kClusterJetsPerSm = 1;
constexpr int kClusterMinJets = 1;

// The jets are dealt over as many clusters as run at once (cluster sizes
// need not divide a GPC's SMs, so that number comes from the occupancy query,
// once per device), at most one cluster per jet and never fewer than
// ceil(N / 4): N = 128 runs on 37 clusters of 3 or 4 jets rather than 32 of 4.
template <int PM>
pb_status run_fused_cluster(const pb::JetArgs& J, const pb::MlpArgs& W, const pb::QkvArgs& X, cudaStream_t s) {
  auto k = pb::k_fused_cluster<PM>;
  const size_t smem = sizeof(pb::ClusterSmem<PM>);
  int dev = 0, sms = 0, per_sm = 0;
  pb_status st = device_sms(&dev, &sms);
  if (st != PB_OK) return st;
  if ((st = resident_per_sm((const void*)k, dev, smem, 512, &per_sm)) != PB_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(512);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = pb::kCJ;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int cap = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_dev[dev].clusters < 0) {
      cfg.gridDim = dim3((unsigned)(sms / pb::kCJ * pb::kCJ));
      int n = 0;
      const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, k, &cfg);
      if (e != cudaSuccess) return fail(PB_ECUDA, "cluster occupancy query: %s", cudaGetErrorString(e));
      g_dev[dev].clusters = n;
    }
    cap = g_dev[dev].clusters;
  }
  const int need = (J.N + pb::kCJ - 1) / pb::kCJ;
  const int ncl = std::max(need, std::min(J.N, cap));
  cfg.gridDim = dim3((unsigned)(ncl * pb::kCJ));
  cudaError_t e = cudaLaunchKernelEx(&cfg, k, J, W, X);
  if (e != cudaSuccess) return fail(PB_ECUDA, "k_fused_cluster launch: %s", cudaGetErrorString(e));
  return PB_OK;
}

bool cluster_applies(const pb::JetArgs& J) {
  int dev = 0, sms = 0;
  if (device_sms(&dev, &sms) != PB_OK) return false;
  return J.P <= 128 && J.N >= kClusterMinJets && J.N <= kClusterJetsPerSm * sms && J.N <= pb::kClusterMaxJets;
}

constexpr long long kGridMaxMaskBytes = 1ll << 21;  // padded N*P scanned by every CTA in phase 0

bool grid_applies(const pb::JetArgs& J) {
  if (J.N < 1 || J.N > pb::kGridMaxJets) return false;
  if (!J.ptr && (long long)J.N * J.P > kGridMaxMaskBytes) return false;
  return true;
}

template <int PM>
pb_status run_fused_grid(const pb::JetArgs& J, const pb::MlpArgs& W, const pb::QkvArgs& X, void* ws,
                         cudaStream_t s) {
  auto k = pb::k_fused_grid<PM>;
  const size_t smem = sizeof(pb::FusedGridSmem<PM>);
  int dev = 0, sms = 0, per_sm = 0;
  pb_status st = device_sms(&dev, &sms);
  if (st != PB_OK) return st;
  if ((st = resident_per_sm((const void*)k, dev, smem, 512, &per_sm)) != PB_OK) return st;
  long long g = sms;  // one CTA per SM, all resident
  if (g > 8ll * J.N) g = 8ll * J.N;
  unsigned char* wsb = static_cast<unsigned char*>(ws);
  int* no_table = nullptr;
  void* args[] = {(void*)&J, (void*)&W, (void*)&X, (void*)&wsb, (void*)&no_table};
  cudaError_t e = cudaLaunchCooperativeKernel((const void*)k, dim3((unsigned)g), dim3(512), args, smem, s);
  if (e != cudaSuccess) return fail(PB_ECUDA, "k_fused_grid cooperative launch: %s", cudaGetErrorString(e));
  return PB_OK;
}

// Scratch of pair_attention_forward_noalloc: the balanced kernel's workspace
// (barrier counters, then the bias records) as a file-scope device array, so
// that this entry point allocates nothing. Each device holds its own copy,
// zero at module load; all calls on a device share it.
static __device__ __align__(256) unsigned char g_static_scratch[PB_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch on the current device, looked up once
// per device (the host-side name is only a stand-in for the symbol).
void* g_static_scratch_ptr[kMaxDev] = {};

pb_status static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(PB_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDev) return fail(PB_ECUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_static_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return fail(PB_ECUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
    g_static_scratch_ptr[dev] = p;
  }
  *out = g_static_scratch_ptr[dev];
  return PB_OK;
}

template <int kNout, int kIn, int kOut>
pb_status run_proj(const pb::JetArgs& J, const pb::ProjArgs& X, cudaStream_t s, const char* what) {
  auto k = pb::k_proj<kNout, kIn, kOut>;
  const size_t smem = sizeof(pb::ProjSmem<kNout>);
  const long long rows = J.ptr ? J.tokens : (long long)J.N * J.P;
  const long long tiles = (rows + pb::kTileM - 1) / pb::kTileM;
  int grid = 0;
  pb_status st = prepare(k, smem, 256, (int)(tiles < 1 ? 1 : (tiles > (1ll << 30) ? (1ll << 30) : tiles)), &grid);
  if (st != PB_OK) return st;
  k<<<grid, 256, smem, s>>>(J, X);
  return launched(what);
}

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// Backward: jets are processed in chunks that the balanced bias kernel
// accepts (at most kGridMaxJets jets and, padded, N*P <= kGridMaxMaskBytes).
// Workspace: the 256-byte header of the bias kernel, the bias records (16
// bytes per row), the gradient records (32 bytes per row), the tile prefix of
// a chunk, then kBwdMaxCtas weight-gradient partials. Record rows are bounded
// for a chunk as for the balanced forward path.
int bwd_chunk_jets(const pb::JetArgs& J) {
  long long c = pb::kGridMaxJets;
  if (!J.ptr && (long long)c * J.P > kGridMaxMaskBytes) c = kGridMaxMaskBytes / J.P;
  return (int)(J.N < c ? J.N : c);
}

struct BwdLayout {
  size_t urec, grec, table, partials, total;
};

BwdLayout bwd_layout(const pb::JetArgs& J) {
  const int nc = bwd_chunk_jets(J);
  const size_t rows = (pb::grid_workspace_bytes(nc, J.P, J.tokens, J.ptr != nullptr) - pb::kWsHeader) / 16;
  BwdLayout L;
  L.urec = pb::kWsHeader;
  L.grec = round256(L.urec + rows * 16);
  L.table = round256(L.grec + rows * 32);
  L.partials = round256(L.table + (size_t)(nc + 1) * sizeof(int));
  L.total = round256(L.partials + (size_t)pb::kBwdMaxCtas * pb::kFoldedFloats * sizeof(float));
  return L;
}

// One chunk of jets: bias records, attention backward, MLP backward.
template <int PM>
pb_status run_backward_chunk(const pb::JetArgs& J, const pb::MlpArgs& W, const pb::BwdArgs& X, unsigned char* ws,
                             int* table, float* partials, int mlp_grid, bool accumulate, cudaStream_t s) {
  int dev = 0, sms = 0, per_sm = 0;
  pb_status st = device_sms(&dev, &sms);
  if (st != PB_OK) return st;
  {
    auto k = pb::k_fused_grid<PM, true>;
    const size_t smem = sizeof(pb::FusedGridSmem<PM>);
    if ((st = resident_per_sm((const void*)k, dev, smem, 512, &per_sm)) != PB_OK) return st;
    long long g = sms;
    if (g > 8ll * J.N) g = 8ll * J.N;
    k<<<(unsigned)g, 512, smem, s>>>(J, W, pb::QkvArgs{nullptr, nullptr, nullptr, nullptr}, ws, table);
    if ((st = launched("k_fused_grid (bias records)")) != PB_OK) return st;
  }
  {
    auto k = pb::k_attn_bwd<PM>;
    const size_t smem = sizeof(pb::AttnBwdSmem<PM>);
    int grid = 0;
    if ((st = prepare(k, smem, 256, J.N * pb::kBwdHeadGroups, &grid)) != PB_OK) return st;
    k<<<grid, 256, smem, s>>>(J, X);
    if ((st = launched("k_attn_bwd")) != PB_OK) return st;
  }
  auto k = pb::k_mlp_bwd<PM>;
  k<<<mlp_grid, pb::kBwdThreads, sizeof(pb::MlpBwdSmem<PM>), s>>>(J, W, X, partials, accumulate ? 1 : 0);
  return launched("k_mlp_bwd");
}

template <int PM>
pb_status run_backward(const pb::JetArgs& J, const pb::MlpArgs& W, pb::BwdArgs X, const pb::GradArgs& G,
                       unsigned char* ws, cudaStream_t s) {
  const BwdLayout L = bwd_layout(J);
  int* table = reinterpret_cast<int*>(ws + L.table);
  float* partials = reinterpret_cast<float*>(ws + L.partials);
  X.urec = reinterpret_cast<const uint4*>(ws + L.urec);
  X.grec = reinterpret_cast<float*>(ws + L.grec);
  X.T = table;
  // the MLP backward's grid is fixed (one partial slot per CTA for all chunks)
  int dev = 0, sms = 0, per_sm = 0;
  pb_status st = device_sms(&dev, &sms);
  if (st != PB_OK) return st;
  auto kb = pb::k_mlp_bwd<PM>;
  if ((st = resident_per_sm((const void*)kb, dev, sizeof(pb::MlpBwdSmem<PM>), pb::kBwdThreads, &per_sm)) != PB_OK) return st;
  const int mlp_grid = sms * per_sm < pb::kBwdMaxCtas ? sms * per_sm : pb::kBwdMaxCtas;
  const int nc = bwd_chunk_jets(J);
  for (int c0 = 0; c0 < J.N; c0 += nc) {
    const int cn = J.N - c0 < nc ? J.N - c0 : nc;
    pb::JetArgs Jc = J;
    pb::BwdArgs Xc = X;
    Jc.N = cn;
    if (J.ptr) {
      Jc.ptr = J.ptr + c0;  // token indices stay global: momenta and q/k/v rows are shared
    } else {
      const size_t e = (size_t)c0 * J.P, r = e * pb::kH * pb::kD;
      Jc.E += e; Jc.px += e; Jc.py += e; Jc.pz += e; Jc.mask += e;
      Xc.q += r; Xc.k += r; Xc.v += r; Xc.dout += r; Xc.dq += r; Xc.dk += r; Xc.dv += r;
    }
    if ((st = run_backward_chunk<PM>(Jc, W, Xc, ws, table, partials, mlp_grid, c0 > 0, s)) != PB_OK) return st;
  }
  pb::k_grad_reduce<<<pb::kReduceCtas, 32 * pb::kReduceWarps, 0, s>>>(partials, mlp_grid, G);
  return launched("k_grad_reduce");
}

}  // namespace

extern "C" {

const char* pb_last_error(void) { return g_err; }

const char* pb_version(void) { return "pairbias-b200 0.1 (sm_100a)"; }

pb_status pairfeat_compute(const pb_jets* jets, float* feat, void* stream) {
  pb::JetArgs J;
  pb_status st = check_jets(jets, &J);
  if (st != PB_OK || J.N == 0) return st;
  if (!feat || !aligned(feat, 16)) return fail(PB_EINVAL, "feat must be a non-NULL 16-byte aligned pointer");
  if (J.N == 0) return PB_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return J.P <= 128 ? run_pairfeat<128>(J, feat, s) : run_pairfeat<256>(J, feat, s);
}

pb_status pairbias_mlp_forward(const pb_jets* jets, const pb_mlp* mlp, void* U, pb_dtype dtype, void* stream) {
  pb::JetArgs J;
  pb::MlpArgs W;
  pb_status st = check_jets(jets, &J);
  if (st != PB_OK || J.N == 0) return st;
  if ((st = check_mlp(mlp, &W)) != PB_OK) return st;
  if (!U || !aligned(U, 16)) return fail(PB_EINVAL, "U must be a non-NULL 16-byte aligned pointer");
  if (dtype != PB_BF16 && dtype != PB_F32) return fail(PB_EINVAL, "dtype %d is not PB_BF16 or PB_F32", (int)dtype);
  if (J.N == 0) return PB_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == PB_F32)
    return J.P <= 128 ? run_mlp_bias<128, true>(J, W, U, s) : run_mlp_bias<256, true>(J, W, U, s);
  return J.P <= 128 ? run_mlp_bias<128, false>(J, W, U, s) : run_mlp_bias<256, false>(J, W, U, s);
}

pb_status pairbias_mlp_forward_i8(const pb_jets* jets, const pb_mlp_i8* mlp, void* U, pb_dtype dtype,
                                  void* stream) {
  pb::JetArgs J;
  pb::MlpI8Args W;
  pb_status st = check_jets(jets, &J);
  if (st != PB_OK || J.N == 0) return st;
  if ((st = check_mlp_i8(mlp, &W)) != PB_OK) return st;
  if (!U || !aligned(U, 16)) return fail(PB_EINVAL, "U must be a non-NULL 16-byte aligned pointer");
  if (dtype != PB_BF16 && dtype != PB_F32) return fail(PB_EINVAL, "dtype %d is not PB_BF16 or PB_F32", (int)dtype);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == PB_F32)
    return J.P <= 128 ? run_mlp_bias<128, true>(J, W, U, s) : run_mlp_bias<256, true>(J, W, U, s);
  return J.P <= 128 ? run_mlp_bias<128, false>(J, W, U, s) : run_mlp_bias<256, false>(J, W, U, s);
}

pb_status pair_attention_forward_i8(const pb_jets* jets, const pb_mlp_i8* mlp, int H, int D, const uint16_t* q,
                                    const uint16_t* k, const uint16_t* v, uint16_t* out, void* stream) {
  pb::JetArgs J;
  pb::MlpI8Args W;
  pb_status st = check_jets(jets, &J);
  if (st != PB_OK) return st;
  if (H != pb::kH || D != pb::kD) return fail(PB_EUNSUPPORTED, "H = %d, D = %d; only H = 8, D = 16", H, D);
  if ((st = check_mlp_i8(mlp, &W)) != PB_OK) return st;
  if (J.N == 0) return PB_OK;
  if (!q || !k || !v || !out) return fail(PB_EINVAL, "q, k, v and out must be non-NULL");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return fail(PB_EINVAL, "q, k, v and out must be 16-byte aligned");
  const pb::QkvArgs X{q, k, v, out};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return J.P <= 128 ? run_fused<128, false>(J, W, X, s) : run_fused<256, false>(J, W, X, s);
}

pb_status pb_quantize_mlp_i8(const float* folded, int8_t* codes, float* alpha) {
  if (!folded || !codes || !alpha) return fail(PB_EINVAL, "NULL argument");
  struct Layer {
    int off, rows, code_off, alpha_off;
  } const L[3] = {{PB_OFF_W2, 64, PB_I8_T2, PB_I8_A2}, {PB_OFF_W3, 64, PB_I8_T3, PB_I8_A3},
                  {PB_OFF_W4, 8, PB_I8_T4, PB_I8_A4}};
  for (const Layer& l : L)
    for (int r = 0; r < l.rows; ++r) {
      const float* w = folded + l.off + r * 64;
      double mx = 0.0;
      for (int c = 0; c < 64; ++c) mx = fmax(mx, fabs((double)w[c]));
      const double a = mx > 0.0 ? mx / 127.0 : 1.0;
      for (int c = 0; c < 64; ++c) codes[l.code_off + r * 64 + c] = (int8_t)nearbyint((double)w[c] / a);
      alpha[l.alpha_off + r] = (float)a;
    }
  return PB_OK;
}

size_t pb_workspace_bytes(const pb_jets* jets) {
  pb::JetArgs J;
  if (check_jets(jets, &J) != PB_OK || !grid_applies(J)) return 0;
  return pb::grid_workspace_bytes(J.N, J.P, J.tokens, J.ptr != nullptr);
}

pb_status pair_attention_forward(const pb_jets* jets, const pb_mlp* mlp, const uint16_t* U, int H, int D,
                                 const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  pb::JetArgs J;
  pb_status st = check_jets(jets, &J);
  if (st != PB_OK) return st;
  if (H != pb::kH || D != pb::kD) return fail(PB_EUNSUPPORTED, "H = %d, D = %d; only H = 8, D = 16", H, D);
  if ((mlp == nullptr) == (U == nullptr)) return fail(PB_EINVAL, "pass exactly one of mlp and U");
  if (J.N == 0) return PB_OK;
  if (!q || !k || !v || !out) return fail(PB_EINVAL, "q, k, v and out must be non-NULL");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || (U && !aligned(U, 16)))
    return fail(PB_EINVAL, "q, k, v, out and U must be 16-byte aligned");
  pb::QkvArgs X{q, k, v, out};
  if (J.N == 0) return PB_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (mlp) {
    pb::MlpArgs W;
    if ((st = check_mlp(mlp, &W)) != PB_OK) return st;
    if (workspace) {
      if (!aligned(workspace, 256)) return fail(PB_EINVAL, "workspace must be 256-byte aligned");
      if (grid_applies(J) &&
          workspace_bytes >= pb::grid_workspace_bytes(J.N, J.P, J.tokens, J.ptr != nullptr))
        return J.P <= 128 ? run_fused_grid<128>(J, W, X, workspace, s) : run_fused_grid<256>(J, W, X, workspace, s);
    }
    if (cluster_applies(J)) return run_fused_cluster<128>(J, W, X, s);
    return J.P <= 128 ? run_fused<128>(J, W, X, s) : run_fused<256>(J, W, X, s);
  }
  return J.P <= 128 ? run_attn_bias<128>(J, X, U, s) : run_attn_bias<256>(J, X, U, s);
}

pb_status pair_attention_forward_noalloc(const pb_jets* jets, const pb_mlp* mlp, int H, int D, const uint16_t* q,
                                         const uint16_t* k, const uint16_t* v, uint16_t* out, void* stream) {
  pb::JetArgs J;
  pb::MlpArgs W;
  pb_status st = check_jets(jets, &J);
  if (st != PB_OK) return st;
  if (H != pb::kH || D != pb::kD) return fail(PB_EUNSUPPORTED, "H = %d, D = %d; only H = 8, D = 16", H, D);
  if ((st = check_mlp(mlp, &W)) != PB_OK) return st;
  if (J.N == 0) return PB_OK;
  if (!q || !k || !v || !out) return fail(PB_EINVAL, "q, k, v and out must be non-NULL");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return fail(PB_EINVAL, "q, k, v and out must be 16-byte aligned");
  if (!grid_applies(J))
    return fail(PB_EUNSUPPORTED, "static-scratch path needs 1 <= N <= %d and, padded, N*P <= %lld (N = %d, P = %d)",
                pb::kGridMaxJets, kGridMaxMaskBytes, J.N, J.P);
  const size_t need = pb::grid_workspace_bytes(J.N, J.P, J.tokens, J.ptr != nullptr);
  if (need > (size_t)PB_STATIC_SCRATCH_BYTES)
    return fail(PB_EUNSUPPORTED, "batch needs %zu bytes of scratch, the static scratch holds %zu (N = %d, P = %d)",
                need, (size_t)PB_STATIC_SCRATCH_BYTES, J.N, J.P);
  void* ws = nullptr;
  if ((st = static_scratch(&ws)) != PB_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the barrier counters must start at zero (a timed-out call may leave them set)
  cudaError_t e = cudaMemsetAsync(ws, 0, pb::kWsHeader, s);
  if (e != cudaSuccess) return fail(PB_ECUDA, "clearing the static scratch header: %s", cudaGetErrorString(e));
  const pb::QkvArgs X{q, k, v, out};
  return J.P <= 128 ? run_fused_grid<128>(J, W, X, ws, s) : run_fused_grid<256>(J, W, X, ws, s);
}

size_t pb_block_workspace_bytes(const pb_jets* jets) {
  pb::JetArgs J;
  if (check_jets(jets, &J) != PB_OK) return 0;
  const long long rows = J.ptr ? J.tokens : (long long)J.N * J.P;
  return 4 * round256((size_t)rows * pb::kEmbed * 2);
}

pb_status pair_block_forward(const pb_jets* jets, const pb_mlp* mlp, const pb_proj* proj, int H, int D, int E,
                             const uint16_t* x, uint16_t* y, void* workspace, size_t workspace_bytes,
                             void* stream) {
  pb::JetArgs J;
  pb::MlpArgs W;
  pb_status st = check_jets(jets, &J);
  if (st != PB_OK) return st;
  if (H != pb::kH || D != pb::kD || E != pb::kEmbed)
    return fail(PB_EUNSUPPORTED, "H = %d, D = %d, E = %d; only H = 8, D = 16, E = 128", H, D, E);
  if ((st = check_mlp(mlp, &W)) != PB_OK) return st;
  if (!proj) return fail(PB_EINVAL, "proj is NULL");
  if (!proj->Wqkv || !proj->bqkv || !proj->Wo || !proj->bo) return fail(PB_EINVAL, "a projection pointer is NULL");
  if (!aligned(proj->Wqkv, 16) || !aligned(proj->Wo, 16) || !aligned(proj->bqkv, 4) || !aligned(proj->bo, 4))
    return fail(PB_EINVAL, "Wqkv and Wo must be 16-byte aligned, the biases 4-byte aligned");
  if (J.N == 0) return PB_OK;
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16)) return fail(PB_EINVAL, "x and y must be non-NULL and 16-byte aligned");
  const long long rows = J.ptr ? J.tokens : (long long)J.N * J.P;
  const size_t tb = round256((size_t)rows * pb::kEmbed * 2);
  if (!workspace || !aligned(workspace, 256)) return fail(PB_EINVAL, "workspace must be non-NULL and 256-byte aligned");
  if (workspace_bytes < 4 * tb)
    return fail(PB_EINVAL, "workspace of %zu bytes, %zu needed (pb_block_workspace_bytes)", workspace_bytes, 4 * tb);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  uint16_t* q = reinterpret_cast<uint16_t*>(ws);
  uint16_t* k = reinterpret_cast<uint16_t*>(ws + tb);
  uint16_t* v = reinterpret_cast<uint16_t*>(ws + 2 * tb);
  uint16_t* o = reinterpret_cast<uint16_t*>(ws + 3 * tb);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (rows == 0) return PB_OK;  // packed jets that are all empty: nothing to read or write
  const pb::ProjArgs in{x, proj->Wqkv, proj->bqkv, q, k, v};
  const pb::QkvArgs X{q, k, v, o};
  const pb::ProjArgs out{o, proj->Wo, proj->bo, y, nullptr, nullptr};
  int dev = 0, sms = 0;
  if ((st = device_sms(&dev, &sms)) != PB_OK) return st;
  if (J.N <= sms) {
    // at most one jet per CTA: the projections run inside the fused kernel,
    // jet by jet, with Q, K, V and O kept in the (L2-resident) workspace
    return J.P <= 128 ? run_fused<128, true>(J, W, X, s, in, out) : run_fused<256, true>(J, W, X, s, in, out);
  }
  // many jets per CTA: per-jet projection latency would add up, so the two
  // projections run as GEMM kernels over all rows around the fused attention
  if ((st = run_proj<384, pb::kInRows, pb::kOutQKV>(J, in, s, "k_proj (in)")) != PB_OK) return st;
  st = J.P <= 128 ? run_fused<128>(J, W, X, s) : run_fused<256>(J, W, X, s);
  if (st != PB_OK) return st;
  return run_proj<128, pb::kInHeads, pb::kOutRows>(J, out, s, "k_proj (out)");
}

size_t pb_backward_workspace_bytes(const pb_jets* jets) {
  pb::JetArgs J;
  if (check_jets(jets, &J) != PB_OK || J.N == 0) return 0;
  return bwd_layout(J).total;
}

pb_status pair_attention_backward(const pb_jets* jets, const pb_mlp* mlp, int H, int D, const uint16_t* q,
                                  const uint16_t* k, const uint16_t* v, const uint16_t* dout, uint16_t* dq,
                                  uint16_t* dk, uint16_t* dv, const pb_mlp_grad* dmlp, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  pb::JetArgs J;
  pb::MlpArgs W;
  pb_status st = check_jets(jets, &J);
  if (st != PB_OK) return st;
  if (H != pb::kH || D != pb::kD) return fail(PB_EUNSUPPORTED, "H = %d, D = %d; only H = 8, D = 16", H, D);
  if ((st = check_mlp(mlp, &W)) != PB_OK) return st;
  if (!dmlp) return fail(PB_EINVAL, "dmlp is NULL");
  float* gp[8] = {dmlp->W1, dmlp->b1, dmlp->W2, dmlp->b2, dmlp->W3, dmlp->b3, dmlp->W4, dmlp->b4};
  for (float* p : gp)
    if (!p || !aligned(p, 4)) return fail(PB_EINVAL, "the gradient buffers of dmlp must be non-NULL and 4-byte aligned");
  const pb::GradArgs G{gp[0], gp[1], gp[2], gp[3], gp[4], gp[5], gp[6], gp[7]};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (J.N == 0) {  // no pairs: the weight gradients are zero
    pb::k_grad_reduce<<<pb::kReduceCtas, 32 * pb::kReduceWarps, 0, s>>>(nullptr, 0, G);
    return launched("k_grad_reduce");
  }
  if (!q || !k || !v || !dout || !dq || !dk || !dv) return fail(PB_EINVAL, "q, k, v, dout, dq, dk and dv must be non-NULL");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dout, 16) || !aligned(dq, 16) ||
      !aligned(dk, 16) || !aligned(dv, 16))
    return fail(PB_EINVAL, "q, k, v, dout, dq, dk and dv must be 16-byte aligned");
  const size_t need = bwd_layout(J).total;
  if (!workspace || !aligned(workspace, 256)) return fail(PB_EINVAL, "workspace must be non-NULL and 256-byte aligned");
  if (workspace_bytes < need)
    return fail(PB_EINVAL, "workspace of %zu bytes, %zu needed (pb_backward_workspace_bytes)", workspace_bytes, need);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const pb::BwdArgs X{q, k, v, dout, dq, dk, dv, nullptr, nullptr, nullptr};
  return J.P <= 128 ? run_backward<128>(J, W, X, G, ws, s) : run_backward<256>(J, W, X, G, ws, s);
}

pb_status pb_unfold_grad(const pb_mlp_unfolded* in, const float* folded_grad, float* out) {
  if (!in || !folded_grad || !out) return fail(PB_EINVAL, "NULL argument");
  const float* need[] = {in->a0, in->c0, in->W1, in->b1, in->a1, in->c1, in->W2, in->b2,
                         in->a2, in->c2, in->W3, in->b3, in->a3, in->c3, in->W4, in->b4};
  for (const float* p : need)
    if (!p) return fail(PB_EINVAL, "an unfolded parameter pointer is NULL");
  const float* g = folded_grad;
  // layer 1: W1' = a1 W1 a0 (per row and column), b1' = a1 (W1 c0 + b1) + c1
  for (int j = 0; j < 4; ++j) {
    double da0 = 0.0, dc0 = 0.0;
    for (int o = 0; o < 64; ++o) {
      const double aw = (double)in->a1[o] * (double)in->W1[o * 4 + j];
      da0 += aw * (double)g[PB_OFF_W1 + o * 4 + j];
      dc0 += aw * (double)g[PB_OFF_B1 + o];
    }
    out[PB_UOFF_A0 + j] = (float)da0;
    out[PB_UOFF_C0 + j] = (float)dc0;
  }
  for (int o = 0; o < 64; ++o) {
    const double a1 = in->a1[o], gb = g[PB_OFF_B1 + o];
    double t = in->b1[o], da1 = 0.0;
    for (int j = 0; j < 4; ++j) {
      const double w = in->W1[o * 4 + j], gw = g[PB_OFF_W1 + o * 4 + j];
      out[PB_UOFF_W1 + o * 4 + j] = (float)(a1 * ((double)in->a0[j] * gw + (double)in->c0[j] * gb));
      da1 += w * (double)in->a0[j] * gw;
      t += w * (double)in->c0[j];
    }
    out[PB_UOFF_B1 + o] = (float)(a1 * gb);
    out[PB_UOFF_A1 + o] = (float)(da1 + t * gb);
    out[PB_UOFF_C1 + o] = (float)gb;
  }
  // layers 2, 3: W' = a W, b' = a b + c
  const float* Ws[2] = {in->W2, in->W3};
  const float* bs[2] = {in->b2, in->b3};
  const float* as[2] = {in->a2, in->a3};
  const int gW[2] = {PB_OFF_W2, PB_OFF_W3}, gB[2] = {PB_OFF_B2, PB_OFF_B3};
  const int uW[2] = {PB_UOFF_W2, PB_UOFF_W3}, uB[2] = {PB_UOFF_B2, PB_UOFF_B3};
  const int uA[2] = {PB_UOFF_A2, PB_UOFF_A3}, uC[2] = {PB_UOFF_C2, PB_UOFF_C3};
  for (int L = 0; L < 2; ++L)
    for (int o = 0; o < 64; ++o) {
      const double a = as[L][o], gb = g[gB[L] + o];
      double da = (double)bs[L][o] * gb;
      for (int i = 0; i < 64; ++i) {
        const double gw = g[gW[L] + o * 64 + i];
        out[uW[L] + o * 64 + i] = (float)(a * gw);
        da += (double)Ws[L][o * 64 + i] * gw;
      }
      out[uB[L] + o] = (float)(a * gb);
      out[uA[L] + o] = (float)da;
      out[uC[L] + o] = (float)gb;
    }
  memcpy(out + PB_UOFF_W4, g + PB_OFF_W4, sizeof(float) * 8 * 64);
  memcpy(out + PB_UOFF_B4, g + PB_OFF_B4, sizeof(float) * 8);
  return PB_OK;
}

pb_status pb_selftest_wait_timeouts(void* stream) {
  pb::k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return launched("k_wait_selftest");
}

pb_status pb_get_device_status(void* stream, uint32_t* bits) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PB_ECUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  unsigned int word = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, pb::g_status, sizeof word);
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(pb::g_status, &zero, sizeof zero);
  if (e != cudaSuccess) return fail(PB_ECUDA, "status word copy: %s", cudaGetErrorString(e));
  if (bits) *bits = word;
  if (word) return fail(PB_EDEVICE, "device status bits 0x%x", word);
  return PB_OK;
}

pb_status pb_fold_affine(const pb_mlp_unfolded* in, float* out) {
  if (!in || !out) return fail(PB_EINVAL, "NULL argument");
  const float* need[] = {in->a0, in->c0, in->W1, in->b1, in->a1, in->c1, in->W2, in->b2,
                         in->a2, in->c2, in->W3, in->b3, in->a3, in->c3, in->W4, in->b4};
  for (const float* p : need)
    if (!p) return fail(PB_EINVAL, "an unfolded parameter pointer is NULL");
  // layer 1: a1*(W1 (a0 f + c0) + b1) + c1 = (a1 W1 a0) f + a1 (W1 c0 + b1) + c1
  for (int o = 0; o < 64; ++o) {
    double bias = in->b1[o];
    for (int i = 0; i < 4; ++i) {
      const double w = in->W1[o * 4 + i];
      out[PB_OFF_W1 + o * 4 + i] = (float)((double)in->a1[o] * w * (double)in->a0[i]);
      bias += w * (double)in->c0[i];
    }
    out[PB_OFF_B1 + o] = (float)((double)in->a1[o] * bias + (double)in->c1[o]);
  }
  // layers 2, 3: a*(W h + b) + c = (a W) h + (a b + c)
  const float* Ws[2] = {in->W2, in->W3};
  const float* bs[2] = {in->b2, in->b3};
  const float* as[2] = {in->a2, in->a3};
  const float* cs[2] = {in->c2, in->c3};
  const int offW[2] = {PB_OFF_W2, PB_OFF_W3}, offB[2] = {PB_OFF_B2, PB_OFF_B3};
  for (int L = 0; L < 2; ++L)
    for (int o = 0; o < 64; ++o) {
      for (int i = 0; i < 64; ++i)
        out[offW[L] + o * 64 + i] = (float)((double)as[L][o] * (double)Ws[L][o * 64 + i]);
      out[offB[L] + o] = (float)((double)as[L][o] * (double)bs[L][o] + (double)cs[L][o]);
    }
  memcpy(out + PB_OFF_W4, in->W4, sizeof(float) * 8 * 64);
  memcpy(out + PB_OFF_B4, in->b4, sizeof(float) * 8);
  return PB_OK;
}

}  // extern "C"
