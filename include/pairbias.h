/*
 * pairbias.h -- C ABI of the B200 (sm_100a) Particle-Transformer pair-bias library.
 *
 * The operations are those of "Event Classification with Masked Transformer
 * Autoencoders" (ml4sci_cms_e2e26 README):
 *   - section "Fusion 2 -- Pairwise Features + Conv1d MLP -> FusedPairMLP":
 *     four Lorentz-invariant features per particle pair (ln kT, ln z, ln dR,
 *     ln m^2) and the pair-embedding MLP 4 -> 64 -> 64 -> 64 -> 8 with its
 *     batch-norm affines folded into the weights and GELU after each hidden
 *     layer, producing one attention bias per head, U[h, i, j];
 *   - section "Fusion 3 -- Self-Attention + Additive Bias -> Fused Triton
 *     Attention": softmax(Q K^T / sqrt(D) + U) V with masked keys excluded.
 * Feature definitions: dy = y_a - y_b (rapidity), dphi wrapped to (-pi, pi],
 * dR = sqrt(dy^2 + dphi^2), kT = min(pT) dR, z = min(pT) / (pT_a + pT_b),
 * m^2 = (E_a + E_b)^2 - |p_a + p_b|^2, each feature ln(max(x, 1e-8)).
 * Diagonal pairs (i == j) are included. Masked query rows of the attention
 * output are 0.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers owned by the caller, except in
 *     pb_fold_affine and pb_unfold_grad (host). Nothing is allocated inside
 *     the library.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and does not synchronise. It launches
 *     exactly one kernel (the balanced fused path as a cooperative launch),
 *     except: pair_block_forward launches one (projections fused in) for at
 *     most one jet per SM and three otherwise; pair_attention_forward_noalloc
 *     clears its scratch header with one cudaMemsetAsync first;
 *     pair_attention_backward launches three per chunk of up to 8192 jets
 *     and one more, in order.
 *     Host-side argument errors return before any launch; device-side
 *     problems (an invalid ptr array, a bounded wait that ran out) set bits
 *     of a per-device status word, read with pb_get_device_status.
 *   - H must be 8 and D must be 16 (the MLP output width fixes H);
 *     1 <= P <= 256. Other values return PB_EUNSUPPORTED.
 *   - Q, K, V, out and U pointers must be 16-byte aligned; momentum, mask and
 *     ptr arrays 4-byte aligned (mask: 1-byte). Violations return PB_EINVAL.
 *   - bf16 values travel as raw uint16_t bit patterns.
 *   - Every element of every output is written: entries of masked pairs of
 *     feat and U are 0, masked query rows of out are 0.
 *   - On error, pb_last_error() returns a message (thread-local).
 */
#ifndef PAIRBIAS_H
#define PAIRBIAS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PB_OK = 0,
  PB_EINVAL = 1,        /* null / misaligned pointer, negative size, bad dtype  */
  PB_EUNSUPPORTED = 2,  /* H != 8, D != 16, P outside [1, 256]                   */
  PB_ECUDA = 3,         /* a CUDA runtime call failed (launch, attribute, copy)  */
  PB_EDEVICE = 4        /* the device status word reported an error              */
} pb_status;

typedef enum { PB_BF16 = 0, PB_F32 = 1 } pb_dtype;

/* Device status bits (pb_get_device_status). */
#define PB_DEV_TIMEOUT 1u   /* a bounded wait inside a kernel ran out; outputs invalid */
#define PB_DEV_BADPTR 2u    /* a packed jet had ptr[n] > ptr[n+1], more than P tokens,
                               or reached past `tokens`; that jet was skipped          */
#define PB_DEV_BOUNDS 4u    /* only in a library built with PB_DEBUG_BOUNDS: a computed
                               index (pair unpacking, bias slot or record, Q/K/V/out
                               offset, attention staging) left its range; that access
                               was skipped                                             */

/* One batch of jets. Exactly one layout is used.
 * Padded (ptr == NULL): E, px, py, pz and mask are [N*P] (jet n, slot s at
 *   n*P + s); mask != 0 marks a valid particle, any pattern is allowed.
 *   Q/K/V/out are [N, H, P, D].
 * Packed (ptr != NULL, mask ignored): jet n owns tokens ptr[n] .. ptr[n+1]-1
 *   of the [tokens] momentum arrays ("ptr" jet boundaries as in
 *   lloca.backbone.transformer_v2.Transformer.forward); every token is valid;
 *   P is the largest multiplicity allowed; Q/K/V/out are [tokens, H, D].
 * Momenta are energy-first (E, px, py, pz), fp32, GeV. */
typedef struct pb_jets {
  const float *E, *px, *py, *pz;
  const uint8_t *mask;
  const int32_t *ptr;
  int32_t N;
  int32_t P;
  int64_t tokens;        /* packed only: length of the momentum arrays */
} pb_jets;

/* Folded pair-embedding MLP, fp32, device pointers, row-major [out][in]; the
 * matrices W1..W4 16-byte aligned (the kernels read them as float4; a
 * misaligned one returns PB_EINVAL). The flat buffer of pb_fold_affine,
 * 16-byte aligned, meets this at every offset below. */
typedef struct pb_mlp {
  const float *W1, *b1;  /* [64][4], [64]  (input affine and layer-1 affine folded in) */
  const float *W2, *b2;  /* [64][64], [64] (layer-2 affine folded in)                  */
  const float *W3, *b3;  /* [64][64], [64] (layer-3 affine folded in)                  */
  const float *W4, *b4;  /* [8][64], [8]   (plain output Linear)                       */
} pb_mlp;

/* Unfolded MLP as a model holds it, host pointers, fp32:
 *   x = a0*f + c0;  h_k = GELU(a_k*(W_k h_{k-1} + b_k) + c_k), k = 1..3;
 *   U = W4 h_3 + b4.  (a_k, c_k are the eval-mode batch-norm scale and shift.) */
typedef struct pb_mlp_unfolded {
  const float *a0, *c0;              /* [4]                      */
  const float *W1, *b1, *a1, *c1;    /* [64][4], [64], [64], [64] */
  const float *W2, *b2, *a2, *c2;    /* [64][64], [64] x 3        */
  const float *W3, *b3, *a3, *c3;    /* [64][64], [64] x 3        */
  const float *W4, *b4;              /* [8][64], [8]              */
} pb_mlp_unfolded;

/* Projections of the attention inside a ParT block (embedding E = H*D = 128):
 * q, k, v = x Wq^T + bq, x Wk^T + bk, x Wv^T + bv and y = o Wo^T + bo, where
 * o is the concatenation of the 8 heads' attention outputs. Device pointers,
 * row-major (out x in); the bf16 matrices 16-byte aligned. */
typedef struct {
  const uint16_t *Wqkv;   /* bf16 [3*128][128]: rows 0..127 Wq, 128..255 Wk, 256..383 Wv */
  const float *bqkv;      /* [3*128]                                                     */
  const uint16_t *Wo;     /* bf16 [128][128]                                             */
  const float *bo;        /* [128]                                                       */
} pb_proj;

/* Offsets (in floats) of the folded parameters inside the flat buffer that
 * pb_fold_affine writes; PB_FOLDED_FLOATS is its length. */
enum {
  PB_OFF_W1 = 0, PB_OFF_B1 = 256, PB_OFF_W2 = 320, PB_OFF_B2 = 4416,
  PB_OFF_W3 = 4480, PB_OFF_B3 = 8576, PB_OFF_W4 = 8640, PB_OFF_B4 = 9152,
  PB_FOLDED_FLOATS = 9160
};

/* Offsets (in floats) of the unfolded parameters' gradients inside the flat
 * buffer that pb_unfold_grad writes (the order of pb_mlp_unfolded);
 * PB_UNFOLDED_FLOATS is its length. */
enum {
  PB_UOFF_A0 = 0, PB_UOFF_C0 = 4, PB_UOFF_W1 = 8, PB_UOFF_B1 = 264, PB_UOFF_A1 = 328,
  PB_UOFF_C1 = 392, PB_UOFF_W2 = 456, PB_UOFF_B2 = 4552, PB_UOFF_A2 = 4616, PB_UOFF_C2 = 4680,
  PB_UOFF_W3 = 4744, PB_UOFF_B3 = 8840, PB_UOFF_A3 = 8904, PB_UOFF_C3 = 8968, PB_UOFF_W4 = 9032,
  PB_UOFF_B4 = 9544, PB_UNFOLDED_FLOATS = 9552
};

/* Gradients with respect to the folded MLP parameters (the pb_mlp that the
 * forward consumed): fp32 device buffers with pb_mlp's shapes, row-major
 * [out][in]; every element is overwritten. */
typedef struct {
  float *W1, *b1;  /* [64][4], [64]   */
  float *W2, *b2;  /* [64][64], [64]  */
  float *W3, *b3;  /* [64][64], [64]  */
  float *W4, *b4;  /* [8][64], [8]    */
} pb_mlp_grad;

/* The MLP with int8 inputs to its hidden layers ("Economical Jet Taggers",
 * section "Kwantiseringsstrategieen": the inputs of linear layers are int8
 * with zero-point quantisation, the weights binary or ternary). Device
 * pointers. Layer 1 keeps its fp32 weights (W1, b1 as in pb_mlp, folded);
 * layers 2, 3 and 4 hold int8 weight codes T (row-major [out][in], 16-byte
 * aligned: 64x64, 64x64, 8x64) and one fp32 scale per output row, so that
 * the folded weight is alpha_o * T_oi; b2, b3, b4 are the folded fp32
 * biases. pb_quantize_mlp_i8 makes T and alpha from pb_fold_affine's output
 * (exactly, for weights that are a per-row scale times {-1, 0, +1}). */
typedef struct pb_mlp_i8 {
  const float *W1, *b1;             /* [64][4], [64]                   */
  const int8_t *T2, *T3, *T4;       /* [64][64], [64][64], [8][64]      */
  const float *a2, *a3, *a4;        /* [64], [64], [8] row scales       */
  const float *b2, *b3, *b4;        /* [64], [64], [8] folded biases    */
} pb_mlp_i8;

/* Offsets inside the buffers that pb_quantize_mlp_i8 writes: codes
 * (PB_I8_CODES int8 values) and alpha (PB_I8_ALPHAS floats). */
enum {
  PB_I8_T2 = 0, PB_I8_T3 = 4096, PB_I8_T4 = 8192, PB_I8_CODES = 8704,
  PB_I8_A2 = 0, PB_I8_A3 = 64, PB_I8_A4 = 128, PB_I8_ALPHAS = 136
};

/* pairfeat_compute -- the four pair features of every slot pair.
 * feat: fp32 [N, P, P, 4], channel order (ln kT, ln z, ln dR, ln m^2);
 * feat[n, i, j] == feat[n, j, i] bit for bit; pairs with a masked (or, packed,
 * absent) end are 0. Source: "Fusion 2" (features half). */
pb_status pairfeat_compute(const pb_jets *jets, float *feat, void *stream);

/* pairbias_mlp_forward -- features and folded MLP, materialising the bias.
 * U: [N, 8, P, P] in `dtype` (PB_BF16 raw bits or PB_F32); U[n,h,i,j] ==
 * U[n,h,j,i]; entries with a masked end are 0. The MLP runs on tcgen05 tensor
 * cores with f16 operands (hidden layers accumulate in f16, the output layer
 * in fp32); hidden activations never leave the chip. Source: "Fusion 2". */
pb_status pairbias_mlp_forward(const pb_jets *jets, const pb_mlp *mlp, void *U, pb_dtype dtype,
                               void *stream);

/* pair_attention_forward -- masked multi-head attention with the pair bias.
 * Exactly one of `mlp` and `U` is non-NULL:
 *   mlp != NULL: the fused path -- features, MLP and attention in one kernel;
 *                the bias is produced and consumed on chip (shared memory,
 *                or with a workspace the L2-resident records), never read
 *                back from HBM;
 *   U   != NULL: the bias is read from a bf16 [N, 8, P, P] array (as written
 *                by pairbias_mlp_forward with PB_BF16).
 * q, k, v, out: bf16 in the layout of `jets` (padded [N,H,P,D], packed
 * [tokens,H,D]). out = softmax(q k^T / sqrt(D) + U) v over valid keys, with
 * fp32 scores, softmax and accumulation; masked query rows are 0.
 * workspace / workspace_bytes: optional, fused path only (see
 * pb_workspace_bytes); NULL / 0 otherwise.
 * Source: "Fusion 3" (with the bias of "Fusion 2"). */
pb_status pair_attention_forward(const pb_jets *jets, const pb_mlp *mlp, const uint16_t *U,
                                 int H, int D, const uint16_t *q, const uint16_t *k,
                                 const uint16_t *v, uint16_t *out, void *workspace,
                                 size_t workspace_bytes, void *stream);

/* pairbias_mlp_forward_i8 -- pairbias_mlp_forward with the int8 MLP
 * (pb_mlp_i8). Per pair row: y1 = W1 f + b1 (f16 hi + lo operands, fp32
 * accumulation); for each of layers 2, 3 and 4 the 64 inputs h of the row
 * (h = GELU(y) of the layer before, erf form, fp32) are quantised on their
 * own: lo = min(0, min h), hi = max(0, max h), s = (hi - lo) / 255 (1 if
 * hi == lo), z = -128 - rint(lo / s), q = clamp(rint(h / s) + z, -128, 127)
 * (rint rounds half to even); the layer runs on int8 tensor cores (s32
 * accumulation) and y_o = alpha_o s (sum_i T_oi q_i - z sum_i T_oi) + b_o in
 * fp32. U as in pairbias_mlp_forward. Codes near a rounding boundary may
 * land on the other side than in exact arithmetic (one quantisation step).
 * Source: "Fusion 2" with the quantisation of "Economical Jet Taggers". */
pb_status pairbias_mlp_forward_i8(const pb_jets *jets, const pb_mlp_i8 *mlp, void *U, pb_dtype dtype,
                                  void *stream);

/* pair_attention_forward_i8 -- the fused path of pair_attention_forward
 * with the int8 MLP (arithmetic of pairbias_mlp_forward_i8), one CTA per jet
 * at a time, the bias kept in shared memory. Arguments and errors as
 * pair_attention_forward with mlp given and no workspace. */
pb_status pair_attention_forward_i8(const pb_jets *jets, const pb_mlp_i8 *mlp, int H, int D,
                                    const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                    uint16_t *out, void *stream);

/* pb_quantize_mlp_i8 -- host helper, not on the GPU path: per output row of
 * the folded W2, W3 and W4 (pb_fold_affine's buffer, PB_OFF_* layout),
 * alpha = max |w| / 127 (1 for a zero row) and codes round(w / alpha), in
 * double. codes: host buffer of PB_I8_CODES int8 (PB_I8_T* offsets);
 * alpha: host buffer of PB_I8_ALPHAS floats (PB_I8_A* offsets). Returns
 * PB_EINVAL for a NULL pointer. */
pb_status pb_quantize_mlp_i8(const float *folded, int8_t *codes, float *alpha);

/* pb_workspace_bytes -- size of the optional workspace of the fused path.
 * With a workspace of at least this size (device memory, 256-byte aligned,
 * zero-filled before its first use; every call leaves its first 256 bytes
 * zero again), pair_attention_forward(mlp != NULL) spreads the MLP tiles of
 * all jets evenly over all SMs and keeps each pair's 8 biases in the
 * workspace (16 bytes per pair, read back from L2) between the MLP and the
 * attention; this needs N <= 8192 and, padded, N*P <= 2^21. Without one (NULL
 * or too small) each CTA runs whole jets and keeps their bias in shared
 * memory. Returns 0 when the balanced path does not apply to `jets`. A call
 * that reports PB_DEV_TIMEOUT may leave the workspace header non-zero: zero it
 * again before reuse. Calls sharing one workspace must not overlap on the
 * device. */
size_t pb_workspace_bytes(const pb_jets *jets);

/* pair_block_forward -- the attention of a ParT block with its projections:
 * from particle embeddings x to y = MHA(x; U) with the pair bias U of
 * pairbias_mlp_forward (the projections either side of "Fusion 3", with the
 * bias of "Fusion 2"; the ParT blocks of the same page use embedding 128 and
 * 8 heads).
 *   x, y: bf16 [N*P][128] (padded, slot order) or [tokens][128] (packed),
 *         16-byte aligned; rows of masked slots of y are written as 0 and
 *         those of x are never used for y.
 *   proj: the projection weights (see pb_proj); H = 8, D = 16, E = 128.
 *   workspace: device memory of at least pb_block_workspace_bytes(jets)
 *         bytes, 256-byte aligned, for Q, K, V and O (bf16, the layout of
 *         pair_attention_forward's q); its contents need no initialisation.
 * Launches on `stream`: for at most one jet per SM, one kernel that runs
 * both projections inside the fused pair-bias attention, jet by jet (Q, K,
 * V and O go through the workspace); otherwise, in order, the in-projection
 * GEMM (tensor cores), the fused pair-bias attention (pair_attention_forward
 * with mlp) and the output-projection GEMM. Calls that share a workspace
 * must not overlap on the device. Errors as for pair_attention_forward. */
pb_status pair_block_forward(const pb_jets *jets, const pb_mlp *mlp, const pb_proj *proj, int H, int D, int E,
                             const uint16_t *x, uint16_t *y, void *workspace, size_t workspace_bytes,
                             void *stream);

/* pb_block_workspace_bytes -- workspace size of pair_block_forward: four
 * bf16 tensors of rows x 128 (rows = N*P padded, tokens packed), each
 * rounded up to 256 bytes. 0 if `jets` is invalid. */
size_t pb_block_workspace_bytes(const pb_jets *jets);

/* PB_STATIC_SCRATCH_BYTES -- size of the library's static per-device scratch
 * array used by pair_attention_forward_noalloc (32 MiB). The array belongs
 * to the library's one device module, so every process that loads the
 * library onto a device holds these 32 MiB there until it exits, whichever
 * entry points it calls. */
#define PB_STATIC_SCRATCH_BYTES (32u << 20)

/* pair_attention_forward_noalloc -- the fused path of pair_attention_forward
 * (mlp given) with the balanced kernel, for callers that cannot allocate
 * device memory: instead of a caller workspace it uses a static device array
 * inside the library, PB_STATIC_SCRATCH_BYTES per device. The paper has no
 * counterpart; it is an interface variant, the arithmetic is that of
 * pair_attention_forward.
 *   Arguments as in pair_attention_forward (bf16 q/k/v/out, H = 8, D = 16).
 *   Rejects (PB_EUNSUPPORTED, message with both sizes) a batch whose
 *   pb_workspace_bytes bound is 0 or exceeds PB_STATIC_SCRATCH_BYTES; this is
 *   decided on the host from N, P and tokens before any device call.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture. The address is kept for the life of the
 *   process: after a cudaDeviceReset (or any reset of the device's primary
 *   context) restart the process before calling this entry point again. Every call then clears the array's 256-byte
 *   header (barrier counters) on `stream` with cudaMemsetAsync and launches
 *   one cooperative kernel. It calls no cudaMalloc, cudaFree or other
 *   allocating routine.
 *   All calls on a device share the one array: calls that overlap on the
 *   device (unordered streams, concurrent host threads) race and produce
 *   wrong results; order them on one stream. */
pb_status pair_attention_forward_noalloc(const pb_jets *jets, const pb_mlp *mlp, int H, int D,
                                         const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                         uint16_t *out, void *stream);

/* pair_attention_backward -- gradients of the fused path of
 * pair_attention_forward (mlp given): for an upstream gradient dout of out,
 * dq, dk, dv and the gradients of the folded MLP parameters. The section
 * "Fusion 3" ships its biased attention with a backward kernel; the MLP
 * gradients are the chain rule of the "Fusion 2" MLP, each unordered pair's
 * bias row receiving dL/dU[h,i,j] + dL/dU[h,j,i]. The pair features are not
 * differentiated (the momenta are data).
 *   q, k, v, dout: bf16 inputs, dq, dk, dv: bf16 outputs, all in the layout
 *     of `jets` (as pair_attention_forward's q), 16-byte aligned; masked rows
 *     of dq, dk, dv are written as 0.
 *   dmlp: device gradient buffers (see pb_mlp_grad), overwritten, also when
 *     N = 0 (zeros).
 *   workspace: device memory of at least pb_backward_workspace_bytes(jets)
 *     bytes, 256-byte aligned, no initialisation needed; calls sharing one
 *     workspace must not overlap on the device.
 * Arithmetic: the bias of every unordered valid pair is recomputed by the
 * fused path's balanced MLP kernel (the forward's own values: f16 operands,
 * hidden layers accumulated in f16, the same GELU approximations) and kept
 * in the workspace as one 16-byte record of 8 f16 values per pair. The
 * attention gradients use bf16 m16n8k16 tensor-core operands with fp32
 * accumulation and fp32 softmax statistics; dL/dU[h,i,j] + dL/dU[h,j,i] is
 * kept as one 32-byte record of 8 fp32 values per unordered pair. The MLP
 * backward recomputes layers 1-3 on tcgen05 with fp32 accumulation in TMEM
 * (features, layer-1 weights and bias as bf16 hi + lo terms; h1, h2, W2 and
 * W3 as f16, the forward's own operands; b2, b3 as f16 hi + lo terms) and
 * the tanh approximation of GELU,
 * GELU(z) = z/2 (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))), with its exact
 * derivative; the products of the backward pass use bf16 operands (weights
 * as hi + lo terms) with fp32 accumulation. The weight gradients are tcgen05
 * products (bf16 d and h, fp32 accumulation in TMEM over each CTA's tiles)
 * and are summed over CTAs in a fixed order, so the result does not depend
 * on timing.
 * Launches, in order on `stream`: the balanced kernel's MLP phase (the bias
 * records), the attention backward, the MLP backward and a gradient-sum
 * kernel (per chunk of up to 8192 jets the first three; with
 * N = 0 only the last, writing zeros). Errors as for
 * pair_attention_forward; PB_EINVAL also for a missing or small workspace
 * or a NULL gradient buffer. */
pb_status pair_attention_backward(const pb_jets *jets, const pb_mlp *mlp, int H, int D,
                                  const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                  const uint16_t *dout, uint16_t *dq, uint16_t *dk, uint16_t *dv,
                                  const pb_mlp_grad *dmlp, void *workspace, size_t workspace_bytes,
                                  void *stream);

/* pb_backward_workspace_bytes -- workspace size of pair_attention_backward.
 * With c = the jets of one chunk (min(N, 8192), and padded also at most
 * 2^21 / P) and R = the bias-record rows of such a chunk (padded:
 * c * ceil(P (P + 1) / 2 / 128) * 128; packed: the smaller of that and
 * tokens * (P + 1) / 2 + 127 c + 128), it is the sum of, each part rounded
 * up to 256 bytes: a 256-byte header, R * 16 bytes of bias records (8 f16
 * per pair), R * 32 bytes of gradient records (8 fp32 per pair), (c + 1)
 * int32 tile offsets and 256 partial gradients of PB_FOLDED_FLOATS fp32
 * values. 0 if `jets` is invalid. */
size_t pb_backward_workspace_bytes(const pb_jets *jets);

/* pb_unfold_grad -- host helper, not on the GPU path: gradients of the
 * unfolded parameters (a0, c0, W1, b1, a1, c1, ... as in pb_mlp_unfolded)
 * from those of the folded ones, by the chain rule of pb_fold_affine's
 * folding (computed in double, rounded once to fp32).
 * folded_grad: host buffer of PB_FOLDED_FLOATS floats (PB_OFF_* layout);
 * out: host buffer of PB_UNFOLDED_FLOATS floats (PB_UOFF_* layout).
 * Returns PB_EINVAL for a NULL pointer. */
pb_status pb_unfold_grad(const pb_mlp_unfolded *in, const float *folded_grad, float *out);

/* pb_get_device_status -- synchronise `stream`, then read and clear the
 * status word of the current device. *bits (may be NULL) receives the
 * PB_DEV_* bits. Returns PB_OK when no bit was set, PB_EDEVICE otherwise,
 * PB_ECUDA if the synchronisation itself failed. */
pb_status pb_get_device_status(void *stream, uint32_t *bits);

/* pb_selftest_wait_timeouts -- diagnostic of the failure path; no
 * counterpart in the paper. Launches one small kernel whose two waits, an
 * mbarrier that nothing completes and a grid barrier whose target nothing
 * reaches, use the same bounded-wait code and limit (2 s) as the library's
 * kernels. Both run out, PB_DEV_TIMEOUT is set, and the kernel ends
 * normally, so the context stays usable. About 4 s of device time. */
pb_status pb_selftest_wait_timeouts(void *stream);

/* pb_fold_affine -- host helper, not on the GPU path: fold the batch-norm
 * affines of an unfolded MLP into Linear weights and biases (the eval-time
 * folding of "Fusion 2"), computing in double and rounding once to fp32.
 * out: host buffer of PB_FOLDED_FLOATS floats, laid out by the PB_OFF_*
 * offsets. Returns PB_EINVAL for a NULL pointer. */
pb_status pb_fold_affine(const pb_mlp_unfolded *in, float *out);

/* pb_last_error -- message for the last non-OK status of this thread. */
const char *pb_last_error(void);

/* pb_version -- library version string. */
const char *pb_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PAIRBIAS_H */
