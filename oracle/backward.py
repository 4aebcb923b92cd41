"""Gradients of the pair-bias attention block in fp64 (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
may import this module; the product path never does.

What is differentiated is the forward pass of "Event Classification with
Masked Transformer Autoencoders", sections "Fusion 2 -- Pairwise Features +
Conv1d MLP -> FusedPairMLP" (features -> 4 -> 64 -> 64 -> 64 -> 8 MLP with the
batch-norm affines and erf-GELU, giving one bias per head and ordered pair)
and "Fusion 3 -- Self-Attention + Additive Bias -> Fused Triton Attention"
(softmax(Q K^T / sqrt(D) + U) V over each jet's valid particles, which that
section ships with a backward kernel). For an upstream gradient dO of the
output, the gradients are the plain chain rule of those definitions:

  attention, per jet and head, over valid queries i and keys j:
    P = softmax_j(S), S_ij = q_i . k_j / sqrt(D) + U_ij, O = P V
    dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(P * dP)),
    dQ = dS K / sqrt(D),  dK = dS^T Q / sqrt(D),  dU = dS
  MLP: every ordered valid pair (i, j) is one row with features f(i, j) and
  upstream gradient dU[:, i, j]; parameter gradients are sums over all rows.

The features are not differentiated (they are functions of the input
momenta, which are data). Everything here is numpy in float64; the features
come from the C oracle. The folded parameters are the ones the product
consumes:
  W1' = diag(a1) W1 diag(a0), b1' = a1 (W1 c0 + b1) + c1,
  Wk' = diag(ak) Wk, bk' = ak bk + ck (k = 2, 3), W4' = W4, b4' = b4,
so that z_k = Wk' h_{k-1} + bk' is the pre-activation of hidden layer k and
h_0 = f the raw features.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

from . import D, H, _bf16_bits_to_f64, features

SQRT2 = np.sqrt(2.0)
INV_SQRT_2PI = 1.0 / np.sqrt(2.0 * np.pi)

PARAM_NAMES = ("a0", "c0", "W1", "b1", "a1", "c1", "W2", "b2", "a2", "c2",
               "W3", "b3", "a3", "c3", "W4", "b4")
FOLDED_NAMES = ("W1", "b1", "W2", "b2", "W3", "b3", "W4", "b4")


def gelu(z):
    """GELU with the Gaussian CDF written through erf."""
    return 0.5 * z * (1.0 + erf(z / SQRT2))


def gelu_grad(z):
    """d GELU / dz = Phi(z) + z phi(z)."""
    return 0.5 * (1.0 + erf(z / SQRT2)) + z * INV_SQRT_2PI * np.exp(-0.5 * z * z)


def as_f64(params):
    return {k: np.asarray(v, np.float64) for k, v in params.items()}


def fold(params):
    """Folded parameters (the definition above) in fp64."""
    p = as_f64(params)
    W1 = p["a1"][:, None] * p["W1"] * p["a0"][None, :]
    b1 = p["a1"] * (p["W1"] @ p["c0"] + p["b1"]) + p["c1"]
    out = {"W1": W1, "b1": b1, "W4": p["W4"].copy(), "b4": p["b4"].copy()}
    for k in (2, 3):
        out[f"W{k}"] = p[f"a{k}"][:, None] * p[f"W{k}"]
        out[f"b{k}"] = p[f"a{k}"] * p[f"b{k}"] + p[f"c{k}"]
    return out


# ----------------------------------------------------------------- MLP

def mlp_forward(f, params):
    """Unfolded MLP over rows f [R, 4] -> (U [R, 8], cache)."""
    p = as_f64(params)
    x0 = p["a0"] * f + p["c0"]
    c = {"f": f, "x0": x0}
    h = x0
    for k in (1, 2, 3):
        t = h @ p[f"W{k}"].T + p[f"b{k}"]
        z = p[f"a{k}"] * t + p[f"c{k}"]
        c[f"t{k}"], c[f"z{k}"] = t, z
        h = gelu(z)
        c[f"h{k}"] = h
    U = h @ p["W4"].T + p["b4"]
    return U, c


def mlp_forward_folded(f, folded):
    """The same MLP in the folded form: z_k = Wk' h_{k-1} + bk'."""
    h = np.asarray(f, np.float64)
    for k in (1, 2, 3):
        h = gelu(h @ folded[f"W{k}"].T + folded[f"b{k}"])
    return h @ folded["W4"].T + folded["b4"]


def mlp_backward(g, cache, params):
    """Parameter gradients for upstream dU rows g [R, 8].

    Returns (unfolded, folded): dicts of gradients with the parameters'
    shapes, the second one with respect to the folded parameters."""
    p = as_f64(params)
    un, fo = {}, {}
    un["W4"] = fo["W4"] = g.T @ cache["h3"]
    un["b4"] = fo["b4"] = g.sum(axis=0)
    e = g @ p["W4"]                                   # dL/dh3
    for k in (3, 2, 1):
        dz = e * gelu_grad(cache[f"z{k}"])            # dL/dz_k
        h_prev_folded = cache["h2"] if k == 3 else (cache["h1"] if k == 2 else cache["f"])
        fo[f"W{k}"] = dz.T @ h_prev_folded
        fo[f"b{k}"] = dz.sum(axis=0)
        un[f"c{k}"] = dz.sum(axis=0)
        un[f"a{k}"] = (dz * cache[f"t{k}"]).sum(axis=0)
        dt = dz * p[f"a{k}"]                          # dL/dt_k
        h_prev = cache["h2"] if k == 3 else (cache["h1"] if k == 2 else cache["x0"])
        un[f"W{k}"] = dt.T @ h_prev
        un[f"b{k}"] = dt.sum(axis=0)
        e = dt @ p[f"W{k}"]                           # dL/dh_{k-1} (k = 1: dL/dx0)
    un["a0"] = (e * cache["f"]).sum(axis=0)
    un["c0"] = e.sum(axis=0)
    return un, fo


# ----------------------------------------------------------- attention

def attention_forward(q, k, v, U):
    """One jet: q, k, v [H, m, D], U [H, m, m] -> (O, P)."""
    S = np.einsum("hid,hjd->hij", q, k) / np.sqrt(D) + U
    S = S - S.max(axis=2, keepdims=True)
    E = np.exp(S)
    P = E / E.sum(axis=2, keepdims=True)
    return np.einsum("hij,hjd->hid", P, v), P


def attention_backward(q, k, v, P, dO):
    """One jet: gradients (dq, dk, dv, dU) for upstream dO [H, m, D]."""
    dv = np.einsum("hij,hid->hjd", P, dO)
    dP = np.einsum("hid,hjd->hij", dO, v)
    dS = P * (dP - (P * dP).sum(axis=2, keepdims=True))
    dq = np.einsum("hij,hjd->hid", dS, k) / np.sqrt(D)
    dk = np.einsum("hij,hid->hjd", dS, q) / np.sqrt(D)
    return dq, dk, dv, dS


# ---------------------------------------------------------------- batch

def jet_index(b, n):
    """(local slots, rows of the [rows, H, D] view of q) of jet n's valid particles."""
    if b.layout == "padded":
        slots = np.flatnonzero(b.mask[n * b.P:(n + 1) * b.P])
        return slots, slots
    cnt = int(b.ptr[n + 1] - b.ptr[n])
    return np.arange(cnt), int(b.ptr[n]) + np.arange(cnt)


def heads_view(b, x):
    """[N*P or tokens, ...] arrays in the layout of q as a function (n, rows) -> [H, m, D]."""
    if b.layout == "padded":
        x4 = x.reshape(b.N, H, b.P, D)
        return lambda n, rows: x4[n][:, rows, :]
    x3 = x.reshape(-1, H, D)
    return lambda n, rows: x3[rows].transpose(1, 0, 2)


def backward(b, dout, params=None, q=None, k=None, v=None, feat=None):
    """Gradients of the whole block for upstream gradient `dout`.

    b: a ``synth.JetBatch``; dout, q, k, v: raw bf16 bits (uint16) or float64
    arrays in the layout of b.q (q, k, v default to b's). Returns a dict with
    "out" (the forward output), "dq", "dk", "dv" (float64, layout of q, 0 on
    masked rows), "unfolded" and "folded" (parameter gradients)."""
    params = b.params if params is None else params
    q = _to_f64(b.q if q is None else q)
    k = _to_f64(b.k if k is None else k)
    v = _to_f64(b.v if v is None else v)
    dO = _to_f64(dout)
    feat = features(b) if feat is None else feat
    res = {name: np.zeros_like(q) for name in ("out", "dq", "dk", "dv")}
    un = {name: np.zeros(np.shape(params[name])) for name in PARAM_NAMES}
    fo = {name: np.zeros(np.shape(params[name])) for name in FOLDED_NAMES}
    views = {name: heads_view(b, arr) for name, arr in
             (("q", q), ("k", k), ("v", v), ("dO", dO))}
    for n in range(b.N):
        slots, rows = jet_index(b, n)
        m = len(slots)
        if m == 0:
            continue
        f = feat[n][np.ix_(slots, slots)].reshape(m * m, 4)
        Urows, cache = mlp_forward(f, params)
        U = Urows.reshape(m, m, H).transpose(2, 0, 1)
        qh, kh, vh, dOh = (views[s](n, rows) for s in ("q", "k", "v", "dO"))
        O, P = attention_forward(qh, kh, vh, U)
        dq, dk, dv, dS = attention_backward(qh, kh, vh, P, dOh)
        g = dS.transpose(1, 2, 0).reshape(m * m, H)
        ju, jf = mlp_backward(g, cache, params)
        for name in PARAM_NAMES:
            un[name] += ju[name]
        for name in FOLDED_NAMES:
            fo[name] += jf[name]
        for name, val in (("out", O), ("dq", dq), ("dk", dk), ("dv", dv)):
            _scatter(b, res[name], n, rows, val)
    res["unfolded"], res["folded"] = un, fo
    return res


def loss(b, dout, params=None, q=None, k=None, v=None, feat=None, folded=None):
    """sum(O * dO) over all outputs: the scalar whose gradients `backward`
    returns (used by the finite-difference checks). With `folded`, the MLP
    runs in the folded form with those parameters instead of `params`."""
    params = b.params if params is None else params
    q = _to_f64(b.q if q is None else q)
    k = _to_f64(b.k if k is None else k)
    v = _to_f64(b.v if v is None else v)
    dO = _to_f64(dout)
    feat = features(b) if feat is None else feat
    views = {name: heads_view(b, arr) for name, arr in (("q", q), ("k", k), ("v", v), ("dO", dO))}
    total = 0.0
    for n in range(b.N):
        slots, rows = jet_index(b, n)
        m = len(slots)
        if m == 0:
            continue
        f = feat[n][np.ix_(slots, slots)].reshape(m * m, 4)
        Urows = mlp_forward_folded(f, folded) if folded is not None else mlp_forward(f, params)[0]
        U = Urows.reshape(m, m, H).transpose(2, 0, 1)
        O, _ = attention_forward(*(views[s](n, rows) for s in ("q", "k", "v")), U)
        total += float((O * views["dO"](n, rows)).sum())
    return total


def _to_f64(x):
    x = np.asarray(x)
    return _bf16_bits_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)


def _scatter(b, dst, n, rows, val):
    """val [H, m, D] into dst (layout of q) at jet n's rows."""
    if b.layout == "padded":
        dst.reshape(b.N, H, b.P, D)[n][:, rows, :] = val
    else:
        dst.reshape(-1, H, D)[rows] = val.transpose(1, 0, 2)
