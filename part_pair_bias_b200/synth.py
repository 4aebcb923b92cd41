"""Seeded synthetic jets, MLP parameters and Q/K/V for the pair-bias path.

This module builds inputs only. It holds none of the method's arithmetic:
no pair features, no MLP evaluation, no attention. The CUDA path and the
oracle both consume what it returns, so random choices never affect parity.

The recipe follows the workload text of the Particle Transformer
interaction-block benchmark (see ``configs.py``):

* multiplicity per jet: uniform integer in [lo, hi] or Poisson(lam) clipped
  to [lo, hi];
* jet pT ~ U(pt_lo, pt_hi), split over the constituents by Dirichlet(alpha=1)
  fractions;
* one-prong jets: constituent eta ~ N(eta_J, 0.2), phi ~ N(phi_J, 0.2) about
  a jet axis eta_J ~ U(-2, 2), phi_J ~ U(-pi, pi);
* three-prong jets: three sub-axes offset N(0, 0.3) in eta and phi from the
  jet axis; each constituent picks a prong uniformly and scatters N(0, 0.1)
  about it;
* massless constituents stored as fp32 (E, px, py, pz) = pT (cosh eta,
  cos phi, sin phi, sinh eta), energy first;
* MLP: weights N(0, 1/fan_in) (variance), biases and affine shifts
  N(0, 0.1) (standard deviation), affine scales U(0.5, 1.5);
* Q, K, V ~ N(0, 1) rounded to bf16 (round to nearest even), kept as raw
  uint16 bit patterns.

Padded layout: [N, P] slots per momentum component plus a uint8 mask
(1 = valid) and Q/K/V of shape [N, H, P, D]. Packed layout: [tokens]
momentum arrays, int32 ``ptr`` of length N+1 with jet n at tokens
ptr[n] .. ptr[n+1]-1, and Q/K/V of shape [tokens, H, D].
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional

import numpy as np

H_HEADS = 8
D_HEAD = 16
HIDDEN = 64
N_FEAT = 4

# Parameter names of the unfolded pair-embedding MLP, in network order.
PARAM_NAMES = (
    "a0", "c0",
    "W1", "b1", "a1", "c1",
    "W2", "b2", "a2", "c2",
    "W3", "b3", "a3", "c3",
    "W4", "b4",
)


@dataclass
class JetBatch:
    """One batch of synthetic jets in either the padded or the packed layout."""

    layout: str                      # "padded" or "packed"
    N: int                           # number of jets
    P: int                           # slots per jet (padded) / max multiplicity (packed)
    mult: np.ndarray                 # int32 [N] valid particles per jet
    E: np.ndarray                    # float32 [N*P] or [tokens]
    px: np.ndarray
    py: np.ndarray
    pz: np.ndarray
    mask: Optional[np.ndarray]       # uint8 [N*P] (padded) else None
    ptr: Optional[np.ndarray]        # int32 [N+1] (packed) else None
    q: np.ndarray                    # uint16 bf16 bits, [N,H,P,D] or [tokens,H,D]
    k: np.ndarray
    v: np.ndarray
    params: Dict[str, np.ndarray] = field(default_factory=dict)  # unfolded, float32

    @property
    def tokens(self) -> int:
        return int(self.E.shape[0])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return raw bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((b >> 16) & 1) + np.uint32(0x7FFF)
    return ((b + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bit patterns exactly to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _multiplicities(rng, n, dist, lo, hi, lam, mults=None):
    if mults is not None:
        return np.asarray(mults, dtype=np.int32).reshape(n)
    if dist == "uniform":
        return rng.integers(lo, hi + 1, size=n).astype(np.int32)
    if dist == "poisson":
        return np.clip(rng.poisson(lam, size=n), lo, hi).astype(np.int32)
    if dist == "full":
        return np.full(n, hi, dtype=np.int32)
    raise ValueError(f"unknown multiplicity distribution {dist!r}")


def _constituents(rng, m, pt_lo, pt_hi, prongs):
    """Massless constituents of one jet, as float64 (E, px, py, pz) columns."""
    if m == 0:
        z = np.zeros(0)
        return z, z, z, z
    jet_pt = rng.uniform(pt_lo, pt_hi)
    frac = rng.dirichlet(np.ones(m))
    pt = jet_pt * frac
    eta_j = rng.uniform(-2.0, 2.0)
    phi_j = rng.uniform(-np.pi, np.pi)
    if prongs == 1:
        eta = eta_j + rng.normal(0.0, 0.2, size=m)
        phi = phi_j + rng.normal(0.0, 0.2, size=m)
    else:
        sub_eta = eta_j + rng.normal(0.0, 0.3, size=prongs)
        sub_phi = phi_j + rng.normal(0.0, 0.3, size=prongs)
        pick = rng.integers(0, prongs, size=m)
        eta = sub_eta[pick] + rng.normal(0.0, 0.1, size=m)
        phi = sub_phi[pick] + rng.normal(0.0, 0.1, size=m)
    return pt * np.cosh(eta), pt * np.cos(phi), pt * np.sin(phi), pt * np.sinh(eta)


def _ternary(rng, rows, fan):
    """Rows tau * t with t in {-1, 0, +1} (P(0) = 1/3) and one tau per row,
    tau = sqrt(1.5 / fan): the variance 1/fan of the Gaussian weights."""
    t = rng.integers(-1, 2, size=(rows, fan)).astype(np.float64)
    return np.sqrt(1.5 / fan) * rng.uniform(0.8, 1.2, size=(rows, 1)) * t


def make_params(rng, weights: str = "gaussian") -> Dict[str, np.ndarray]:
    """Unfolded pair-embedding MLP parameters (4 -> 64 -> 64 -> 64 -> 8), float32.

    ``weights="ternary"`` draws the Linear weights of layers 2..4 (the layers
    whose inputs are hidden activations) as one scale per output row times
    {-1, 0, +1}, the weights of a ternary-quantised network; layer 1 and every
    other parameter keep their Gaussian / uniform draws."""
    if weights not in ("gaussian", "ternary"):
        raise ValueError(f"unknown weight kind {weights!r}")
    p = {}
    p["a0"] = rng.uniform(0.5, 1.5, N_FEAT)
    p["c0"] = rng.normal(0.0, 0.1, N_FEAT)
    fan = N_FEAT
    for k in (1, 2, 3):
        if weights == "ternary" and k > 1:
            p[f"W{k}"] = _ternary(rng, HIDDEN, fan)
        else:
            p[f"W{k}"] = rng.normal(0.0, 1.0 / np.sqrt(fan), (HIDDEN, fan))
        p[f"b{k}"] = rng.normal(0.0, 0.1, HIDDEN)
        p[f"a{k}"] = rng.uniform(0.5, 1.5, HIDDEN)
        p[f"c{k}"] = rng.normal(0.0, 0.1, HIDDEN)
        fan = HIDDEN
    if weights == "ternary":
        p["W4"] = _ternary(rng, H_HEADS, HIDDEN)
    else:
        p["W4"] = rng.normal(0.0, 1.0 / np.sqrt(HIDDEN), (H_HEADS, HIDDEN))
    p["b4"] = rng.normal(0.0, 0.1, H_HEADS)
    return {k: np.ascontiguousarray(v, dtype=np.float32) for k, v in p.items()}


def make_jets(*, N: int, P: int, layout: str = "padded", dist: str = "poisson",
              mult_lo: int = 2, mult_hi: Optional[int] = None, lam: float = 40.0,
              pt_lo: float = 500.0, pt_hi: float = 550.0, prongs: int = 1,
              mask_mode: str = "prefix", seed: int = 0, mults=None, weights: str = "gaussian") -> JetBatch:
    """Draw one batch of jets, MLP parameters and Q/K/V from PCG64(seed).

    ``mask_mode="prefix"`` puts the m valid particles in slots 0..m-1;
    ``"scrambled"`` places them in m random slots of the P (padded only).
    ``mults`` fixes the multiplicity of every jet instead of drawing it;
    ``weights`` selects Gaussian or ternary hidden-layer weights (make_params).
    Draw order: parameters, multiplicities, per-jet kinematics, slot
    permutations, Q, K, V.
    """
    if mult_hi is None:
        mult_hi = P
    rng = np.random.Generator(np.random.PCG64(seed))
    params = make_params(rng, weights)
    mult = _multiplicities(rng, N, dist, mult_lo, mult_hi, lam, mults)
    kin = [_constituents(rng, int(m), pt_lo, pt_hi, prongs) for m in mult]

    if layout == "padded":
        E = np.zeros((N, P)); px = np.zeros((N, P)); py = np.zeros((N, P)); pz = np.zeros((N, P))
        mask = np.zeros((N, P), dtype=np.uint8)
        for n, m in enumerate(mult):
            slots = np.arange(m) if mask_mode == "prefix" else np.sort(rng.permutation(P)[:m])
            E[n, slots], px[n, slots], py[n, slots], pz[n, slots] = kin[n]
            mask[n, slots] = 1
        shape = (N, H_HEADS, P, D_HEAD)
        ptr = None
        mask = mask.reshape(-1)
        flat = lambda a: a.reshape(-1)
    elif layout == "packed":
        ptr = np.zeros(N + 1, dtype=np.int32)
        ptr[1:] = np.cumsum(mult)
        E = np.concatenate([k[0] for k in kin]) if N else np.zeros(0)
        px = np.concatenate([k[1] for k in kin]) if N else np.zeros(0)
        py = np.concatenate([k[2] for k in kin]) if N else np.zeros(0)
        pz = np.concatenate([k[3] for k in kin]) if N else np.zeros(0)
        shape = (int(ptr[-1]), H_HEADS, D_HEAD)
        mask = None
        flat = lambda a: a
    else:
        raise ValueError(f"unknown layout {layout!r}")

    q = f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))
    k = f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))
    v = f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))
    f32 = lambda a: np.ascontiguousarray(flat(a), dtype=np.float32)
    return JetBatch(layout=layout, N=N, P=P, mult=mult, E=f32(E), px=f32(px), py=f32(py),
                    pz=f32(pz), mask=mask, ptr=ptr, q=q, k=k, v=v, params=params)


def slice_jets(b: JetBatch, lo: int, hi: int) -> JetBatch:
    """Jets lo..hi-1 of a batch as a batch of their own (same layout)."""
    if b.layout == "padded":
        s = slice(lo * b.P, hi * b.P)
        return JetBatch("padded", hi - lo, b.P, b.mult[lo:hi].copy(), b.E[s].copy(), b.px[s].copy(),
                        b.py[s].copy(), b.pz[s].copy(), b.mask[s].copy(), None,
                        b.q[lo:hi].copy(), b.k[lo:hi].copy(), b.v[lo:hi].copy(), b.params)
    t0, t1 = int(b.ptr[lo]), int(b.ptr[hi])
    s = slice(t0, t1)
    ptr = (b.ptr[lo:hi + 1] - t0).astype(np.int32)
    return JetBatch("packed", hi - lo, b.P, b.mult[lo:hi].copy(), b.E[s].copy(), b.px[s].copy(),
                    b.py[s].copy(), b.pz[s].copy(), None, ptr,
                    b.q[s].copy(), b.k[s].copy(), b.v[s].copy(), b.params)


# ------------------------------------------------ projections around the attention

EMBED = H_HEADS * D_HEAD  # 128: the particle embedding width of a ParT block


@dataclass
class BlockInputs:
    """Particle embeddings and the attention's in/out projections.

    x: bf16 bits [rows, EMBED] with rows = N * P (padded, slot order) or
    tokens (packed); Wqkv: bf16 bits [3 * EMBED, EMBED], rows 0..127 the
    query, 128..255 the key and 256..383 the value projection (out x in);
    bqkv: float32 [3 * EMBED]; Wo: bf16 bits [EMBED, EMBED]; bo: float32
    [EMBED].
    """

    x: np.ndarray
    Wqkv: np.ndarray
    bqkv: np.ndarray
    Wo: np.ndarray
    bo: np.ndarray


def make_block_inputs(b: JetBatch, seed: int) -> BlockInputs:
    """Embeddings x ~ N(0, 1) for every slot or token, projection weights
    N(0, 1/EMBED) (variance) and biases N(0, 0.1) (standard deviation), all
    rounded like the model's bf16 tensors (biases stay fp32). Drawn from a
    stream of their own, so a batch's other inputs do not change."""
    rng = np.random.default_rng([int(seed), 0xB10C])
    rows = b.N * b.P if b.layout == "padded" else int(b.ptr[-1])
    x = f32_to_bf16_bits(rng.standard_normal((rows, EMBED)).astype(np.float32))
    s = 1.0 / np.sqrt(EMBED)
    Wqkv = f32_to_bf16_bits((rng.standard_normal((3 * EMBED, EMBED)) * s).astype(np.float32))
    bqkv = (rng.standard_normal(3 * EMBED) * 0.1).astype(np.float32)
    Wo = f32_to_bf16_bits((rng.standard_normal((EMBED, EMBED)) * s).astype(np.float32))
    bo = (rng.standard_normal(EMBED) * 0.1).astype(np.float32)
    return BlockInputs(x, Wqkv, bqkv, Wo, bo)


def slice_block_inputs(b: JetBatch, bi: BlockInputs, lo: int, hi: int) -> BlockInputs:
    """The embeddings of jets lo..hi-1 (same weights)."""
    if b.layout == "padded":
        x = bi.x[lo * b.P:hi * b.P].copy()
    else:
        x = bi.x[int(b.ptr[lo]):int(b.ptr[hi])].copy()
    return BlockInputs(x, bi.Wqkv, bi.bqkv, bi.Wo, bi.bo)


def make_upstream(b: JetBatch, seed: int) -> np.ndarray:
    """An upstream gradient dL/dout for the backward pass: N(0, 1) values
    rounded to bf16 (raw bits), in the layout of b.q, from a stream of its
    own. Masked rows hold values too; the forward output there is constant 0,
    so they carry no gradient."""
    rng = np.random.default_rng([int(seed), 0xD0])
    return f32_to_bf16_bits(rng.standard_normal(b.q.shape).astype(np.float32))


def slice_rows(b: JetBatch, x: np.ndarray, lo: int, hi: int) -> np.ndarray:
    """The rows of jets lo..hi-1 of an array in the layout of b.q."""
    if b.layout == "padded":
        return x[lo:hi].copy()
    return x[int(b.ptr[lo]):int(b.ptr[hi])].copy()
