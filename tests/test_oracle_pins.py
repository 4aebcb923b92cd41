"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Features: hand-derived closed forms (tests/golden), the massless and the
transverse-mass identities for m^2, invariance under azimuthal rotations and
longitudinal boosts (ParT pair features are invariant under SO(2) x SO+(1,1),
"De deugden en ondeugden van equivariante transformers", section
"Methodologie"), and bitwise i<->j symmetry.
MLP: the erf GELU against the normal CDF of scipy, its odd-part identity,
all-zero weights, and the purely linear regime, where the network must reduce
to the composed affine maps (this catches a transposed weight, a misplaced
affine or a dropped bias).
Attention: the bias-free and the biased cases against torch's
scaled_dot_product_attention in fp64, one-particle jets, constant keys, mask
exclusion, padded == packed, and permutation equivariance.
Block (attention with its in and out projections): against torch's
multi_head_attention_forward in fp64 jet by jet, reduction to the pinned
attention under identity projections, masked rows 0, and the output-bias
shift.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from part_pair_bias_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pair_features_worked.json")
LN_EPS = math.log(1e-8)


def _eval(expr):
    ns = {"pi": math.pi, "log": math.log, "cos": math.cos, "sin": math.sin,
          "cosh": math.cosh, "sinh": math.sinh, "__builtins__": {}}
    return float(eval(expr, ns))


# ------------------------------------------------------------------ features

def test_worked_examples(oracle_lib):
    fx = json.load(open(GOLDEN))
    assert fx["cases"]
    for case in fx["cases"]:
        a = [_eval(e) for e in case["a"]]
        b = [_eval(e) for e in case["b"]]
        want = np.array([_eval(e) for e in case["features"]])
        got = oracle_lib.pair_features(a, b)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12, err_msg=case["name"])
        # the same pair in the other order
        np.testing.assert_allclose(oracle_lib.pair_features(b, a), want, rtol=0, atol=1e-12)


def _massless(pt, y, phi):
    return np.array([pt * np.cosh(y), pt * np.cos(phi), pt * np.sin(phi), pt * np.sinh(y)])


def _massive(pt, y, phi, m):
    mt = np.sqrt(pt * pt + m * m)
    return np.array([mt * np.cosh(y), pt * np.cos(phi), pt * np.sin(phi), mt * np.sinh(y)])


def _wrap(d):
    d = math.fmod(d, 2 * math.pi)
    if d > math.pi:
        d -= 2 * math.pi
    elif d <= -math.pi:
        d += 2 * math.pi
    return d


def test_massless_mass_identity(oracle_lib):
    """m^2 = 2 pT_a pT_b (cosh dy - cos dphi) for massless pairs."""
    rng = np.random.default_rng(11)
    for _ in range(300):
        pa, pb = rng.uniform(0.5, 200, 2)
        ya, yb = rng.uniform(-3, 3, 2)
        fa, fb = rng.uniform(-math.pi, math.pi, 2)
        f = oracle_lib.pair_features(_massless(pa, ya, fa), _massless(pb, yb, fb))
        m2 = 2 * pa * pb * (math.cosh(ya - yb) - math.cos(fa - fb))
        assert m2 > 1e-6
        assert abs(f[3] - math.log(m2)) < 1e-9
        dr = math.hypot(ya - yb, _wrap(fa - fb))
        assert abs(f[2] - math.log(dr)) < 1e-10
        assert abs(f[0] - math.log(min(pa, pb) * dr)) < 1e-10
        assert abs(f[1] - math.log(min(pa, pb) / (pa + pb))) < 1e-12


def test_massive_transverse_mass_identity(oracle_lib):
    """m^2 = m_a^2 + m_b^2 + 2 (mT_a mT_b cosh dy - pT_a pT_b cos dphi)."""
    rng = np.random.default_rng(12)
    for _ in range(300):
        pa, pb = rng.uniform(0.5, 200, 2)
        ma, mb = rng.uniform(0.0, 20, 2)
        ya, yb = rng.uniform(-3, 3, 2)
        fa, fb = rng.uniform(-math.pi, math.pi, 2)
        mta, mtb = math.hypot(pa, ma), math.hypot(pb, mb)
        m2 = ma * ma + mb * mb + 2 * (mta * mtb * math.cosh(ya - yb) - pa * pb * math.cos(fa - fb))
        f = oracle_lib.pair_features(_massive(pa, ya, fa, ma), _massive(pb, yb, fb, mb))
        assert abs(f[3] - math.log(m2)) < 1e-8


def _boost_rotate(p, dy, dphi):
    E, px, py, pz = p
    c, s = math.cos(dphi), math.sin(dphi)
    px2, py2 = c * px - s * py, s * px + c * py
    ch, sh = math.cosh(dy), math.sinh(dy)
    return np.array([ch * E + sh * pz, px2, py2, sh * E + ch * pz])


def test_invariance_rotation_and_longitudinal_boost(oracle_lib):
    rng = np.random.default_rng(13)
    for _ in range(200):
        a = _massive(*rng.uniform(1, 100, 1), *rng.uniform(-2, 2, 1), *rng.uniform(-3, 3, 1),
                     *rng.uniform(0, 5, 1))
        b = _massive(*rng.uniform(1, 100, 1), *rng.uniform(-2, 2, 1), *rng.uniform(-3, 3, 1),
                     *rng.uniform(0, 5, 1))
        f0 = oracle_lib.pair_features(a, b)
        dy, dphi = rng.uniform(-1.5, 1.5), rng.uniform(-math.pi, math.pi)
        f1 = oracle_lib.pair_features(_boost_rotate(a, dy, dphi), _boost_rotate(b, dy, dphi))
        np.testing.assert_allclose(f1, f0, rtol=0, atol=1e-9)


def test_feature_symmetry_bitwise_and_masked_zero(oracle_lib):
    b = synth.make_jets(N=6, P=32, dist="uniform", mult_lo=2, mult_hi=32, seed=3,
                        mask_mode="scrambled")
    f = oracle_lib.features(b)
    assert np.array_equal(f, f.transpose(0, 2, 1, 3))
    m = b.mask.reshape(b.N, b.P).astype(bool)
    pair = m[:, :, None] & m[:, None, :]
    assert np.all(f[~pair] == 0.0)
    assert np.all(np.isfinite(f[pair]))
    # the diagonal: dR = 0 -> ln kT = ln dR = ln 1e-8, z = 1/2
    n, s = np.nonzero(m)
    assert np.allclose(f[n, s, s, 0], LN_EPS) and np.allclose(f[n, s, s, 2], LN_EPS)
    assert np.allclose(f[n, s, s, 1], math.log(0.5), atol=1e-15)


# ----------------------------------------------------------------------- MLP

def test_gelu_against_normal_cdf(oracle_lib):
    from scipy.special import ndtr
    for x in np.linspace(-9, 9, 181):
        assert abs(oracle_lib.gelu(x) - x * ndtr(x)) < 1e-14 * max(1.0, abs(x))
    assert oracle_lib.gelu(0.0) == 0.0
    assert abs(oracle_lib.gelu(1.0) - 0.8413447460685429) < 1e-15   # Phi(1)
    for x in np.linspace(-6, 6, 49):
        assert abs(oracle_lib.gelu(x) - oracle_lib.gelu(-x) - x) < 1e-14


def _params_like(p, **over):
    q = {k: v.copy() for k, v in p.items()}
    q.update({k: np.asarray(v, np.float32) for k, v in over.items()})
    return q


def test_mlp_zero_weights_gives_output_bias(oracle_lib):
    p = synth.make_params(np.random.default_rng(1))
    z = _params_like(p, W4=np.zeros((8, 64)))
    f = np.array([1.0, -2.0, 0.5, 3.0])
    np.testing.assert_array_equal(oracle_lib.mlp_row(f, z), p["b4"].astype(np.float64))


def test_mlp_linear_regime_is_composed_affine(oracle_lib):
    """With every GELU input above 40, GELU(x) = x to far below fp64 rounding
    and the MLP is the composition of its affine maps. Large shifts c_k and
    small (not zero) W2, W3 keep every pre-activation in that regime."""
    rng = np.random.default_rng(2)
    p = synth.make_params(rng)
    p = _params_like(p, c1=np.full(64, 200.0), c2=np.full(64, 50.0), c3=np.full(64, 50.0),
                     W2=p["W2"] * 1e-3, W3=p["W3"] * 1e-3)
    g = {k: v.astype(np.float64) for k, v in p.items()}
    for _ in range(20):
        f = rng.uniform(-18, 10, 4)
        x = g["a0"] * f + g["c0"]
        h1 = g["a1"] * (g["W1"] @ x + g["b1"]) + g["c1"]
        h2 = g["a2"] * (g["W2"] @ h1 + g["b2"]) + g["c2"]
        h3 = g["a3"] * (g["W3"] @ h2 + g["b3"]) + g["c3"]
        assert min(h1.min(), h2.min(), h3.min()) > 40.0
        want = g["W4"] @ h3 + g["b4"]
        np.testing.assert_allclose(oracle_lib.mlp_row(f, p), want, rtol=1e-13, atol=1e-11)
    # far below zero every GELU returns (minus) zero and only b4 survives
    n = _params_like(p, c1=np.full(64, -400.0), c2=np.full(64, -400.0), c3=np.full(64, -400.0))
    np.testing.assert_allclose(oracle_lib.mlp_row(np.array([1.0, 2, 3, 4]), n), p["b4"], atol=1e-12)


def test_bias_symmetry_bitwise(oracle_lib):
    b = synth.make_jets(N=4, P=32, dist="uniform", mult_lo=2, mult_hi=32, seed=4)
    U = oracle_lib.pair_bias(b)
    assert np.array_equal(U, U.transpose(0, 1, 3, 2))


# ----------------------------------------------------------------- attention

def _dense(b, U, q=None, k=None, v=None):
    """q/k/v [N,H,P,D] float64, boolean key mask [N,P], bias [N,H,P,P]."""
    f = lambda a: synth.bf16_bits_to_f64(a)
    return (f(b.q if q is None else q), f(b.k if k is None else k), f(b.v if v is None else v),
            b.mask.reshape(b.N, b.P).astype(bool), U)


@pytest.mark.parametrize("with_bias", [False, True])
def test_attention_matches_torch_sdpa(oracle_lib, with_bias):
    b = synth.make_jets(N=5, P=24, dist="uniform", mult_lo=1, mult_hi=24, seed=5,
                        mask_mode="scrambled")
    rng = np.random.default_rng(6)
    U = rng.normal(0, 2.0, (b.N, 8, b.P, b.P)) if with_bias else np.zeros((b.N, 8, b.P, b.P))
    out = oracle_lib.attention(b, U)
    q, k, v, m, U = _dense(b, U)
    add = torch.tensor(U).clone()
    add.masked_fill_(~torch.tensor(m)[:, None, None, :], float("-inf"))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v), attn_mask=add).numpy()
    ref = ref * m[:, None, :, None]             # masked query rows are 0
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    assert np.all(out[~np.broadcast_to(m[:, None, :, None], out.shape)] == 0.0)


def test_attention_single_particle_and_constant_keys(oracle_lib):
    b = synth.make_jets(N=3, P=8, dist="uniform", mult_lo=1, mult_hi=1, seed=7)
    out = oracle_lib.attention(b, np.random.default_rng(0).normal(size=(3, 8, 8, 8)))
    v = synth.bf16_bits_to_f64(b.v)
    np.testing.assert_array_equal(out[:, :, 0, :], v[:, :, 0, :])   # softmax over one key is 1
    # all keys zero and no bias: every valid query averages the valid values
    b = synth.make_jets(N=3, P=16, dist="uniform", mult_lo=3, mult_hi=16, seed=8)
    out = oracle_lib.attention(b, np.zeros((3, 8, 16, 16)), k=np.zeros_like(b.k))
    v = synth.bf16_bits_to_f64(b.v)
    for n, mlt in enumerate(b.mult):
        mean = v[n, :, :mlt, :].mean(axis=1)
        np.testing.assert_allclose(out[n, :, :mlt, :], np.broadcast_to(mean[:, None, :], (8, mlt, 16)),
                                   atol=1e-14)


def test_mask_exclusion_bitwise(oracle_lib):
    b = synth.make_jets(N=4, P=32, dist="uniform", mult_lo=2, mult_hi=30, seed=9, mask_mode="scrambled")
    out0 = oracle_lib.forward(b)
    rng = np.random.default_rng(10)
    hole = b.mask == 0
    for name in ("E", "px", "py", "pz"):
        arr = getattr(b, name)
        arr[hole] = rng.normal(0, 50, hole.sum()).astype(np.float32)
    hole4 = hole.reshape(b.N, 1, b.P, 1)
    for name in ("q", "k", "v"):
        arr = getattr(b, name)
        noise = synth.f32_to_bf16_bits(rng.normal(0, 3, arr.shape).astype(np.float32))
        setattr(b, name, np.where(hole4, noise, arr))
    out1 = oracle_lib.forward(b)
    assert np.array_equal(out0, out1)


def _permute_slots(b, perms):
    """The same jets with jet n's slots reordered: new slot s holds old slot perms[n][s]."""
    c = lambda a: a.reshape(b.N, b.P)[np.arange(b.N)[:, None], perms].reshape(-1).copy()
    h = lambda a: a[np.arange(b.N)[:, None, None], np.arange(a.shape[1])[None, :, None], perms[:, None, :]].copy()
    return synth.JetBatch("padded", b.N, b.P, b.mult.copy(), c(b.E), c(b.px), c(b.py), c(b.pz), c(b.mask),
                          None, h(b.q), h(b.k), h(b.v), b.params)


def test_permutation_equivariance(oracle_lib):
    """Reordering a jet's slots reorders its features, bias and output rows
    the same way and changes nothing else (the block acts on a set of
    particles). Features and bias are per-pair values, so they move bit for
    bit; the output's sums run in another order, so it moves to within fp64
    rounding. A slot used where a compact index belongs, or the reverse,
    breaks this."""
    b = synth.make_jets(N=3, P=24, dist="uniform", mult_lo=3, mult_hi=24, seed=21, mask_mode="scrambled")
    rng = np.random.default_rng(21)
    perms = np.stack([rng.permutation(b.P) for _ in range(b.N)])
    bp = _permute_slots(b, perms)
    n3 = np.arange(b.N)[:, None, None]
    f0, f1 = oracle_lib.features(b), oracle_lib.features(bp)
    assert np.array_equal(f1, f0[n3, perms[:, :, None], perms[:, None, :]])
    u0, u1 = oracle_lib.pair_bias(b), oracle_lib.pair_bias(bp)
    assert np.array_equal(u1, u0[n3[..., None], np.arange(8)[None, :, None, None], perms[:, None, :, None],
                                 perms[:, None, None, :]])
    o0, o1 = oracle_lib.forward(b), oracle_lib.forward(bp)
    moved = o0[np.arange(b.N)[:, None, None], np.arange(8)[None, :, None], perms[:, None, :]]
    np.testing.assert_allclose(o1, moved, rtol=0, atol=1e-12 * max(1.0, np.abs(o0).max()))
    assert not np.allclose(o1, o0)  # the permutation did move rows


def _to_packed(b):
    """The same jets as a packed batch (prefix masks only)."""
    m = b.mult
    ptr = np.zeros(b.N + 1, np.int32)
    ptr[1:] = np.cumsum(m)
    take = lambda a: np.concatenate([a.reshape(b.N, b.P)[n, :m[n]] for n in range(b.N)])
    tok = lambda a: np.concatenate([a[n, :, :m[n], :].transpose(1, 0, 2) for n in range(b.N)])
    return synth.JetBatch("packed", b.N, b.P, m.copy(), take(b.E), take(b.px), take(b.py), take(b.pz),
                          None, ptr, tok(b.q), tok(b.k), tok(b.v), b.params)


def test_forward_equals_bias_then_attention_and_packed_equals_padded(oracle_lib):
    b = synth.make_jets(N=5, P=20, dist="uniform", mult_lo=2, mult_hi=20, seed=14)
    o_fwd = oracle_lib.forward(b)
    assert np.array_equal(o_fwd, oracle_lib.attention(b, oracle_lib.pair_bias(b)))
    pk = _to_packed(b)
    o_pk = oracle_lib.forward(pk)
    f_pd, f_pk = oracle_lib.features(b), oracle_lib.features(pk)
    for n, m in enumerate(b.mult):
        t0 = pk.ptr[n]
        assert np.array_equal(f_pd[n, :m, :m], f_pk[n, :m, :m])
        assert np.array_equal(o_fwd[n, :, :m, :].transpose(1, 0, 2), o_pk[t0:t0 + m])


# ---------------------------------------------------------------- block


def _block_batch(layout="padded", seed=11):
    b = synth.make_jets(N=6, P=24, layout=layout, dist="uniform", mult_lo=1, mult_hi=24,
                        mask_mode="scrambled" if layout == "padded" else "prefix", seed=seed)
    return b, synth.make_block_inputs(b, seed)


def _jet_rows(b, n):
    if b.layout == "padded":
        slots = np.flatnonzero(b.mask[n * b.P:(n + 1) * b.P])
        return n * b.P + slots, slots
    rows = np.arange(int(b.ptr[n]), int(b.ptr[n + 1]))
    return rows, np.arange(len(rows))


@pytest.mark.parametrize("layout", ["padded", "packed"])
def test_block_matches_torch_multi_head_attention(oracle_lib, layout):
    """torch's own MHA (its in-projection, head split, scaling and out
    projection) in fp64, with the pair bias as a per-head additive mask."""
    b, bi = _block_batch(layout)
    y = oracle_lib.block_forward(b, bi)
    U = oracle_lib.pair_bias(b)
    x = synth.bf16_bits_to_f64(bi.x)
    for n in range(b.N):
        rows, local = _jet_rows(b, n)
        if len(rows) == 0:
            continue
        X = torch.from_numpy(x[rows]).unsqueeze(1)                       # (L, batch 1, E)
        mask = torch.from_numpy(U[n][:, local][:, :, local].copy())       # (heads, L, L)
        ref, _ = torch.nn.functional.multi_head_attention_forward(
            X, X, X, 128, 8,
            torch.from_numpy(synth.bf16_bits_to_f64(bi.Wqkv)), torch.from_numpy(bi.bqkv.astype(np.float64)),
            None, None, False, 0.0,
            torch.from_numpy(synth.bf16_bits_to_f64(bi.Wo)), torch.from_numpy(bi.bo.astype(np.float64)),
            training=False, need_weights=False, attn_mask=mask)
        np.testing.assert_allclose(y[rows], ref[:, 0].numpy(), rtol=1e-10, atol=1e-12)


def test_block_with_identity_projections_is_the_pinned_attention(oracle_lib):
    """q = k = v = x and y = o when every projection is the identity: the
    block's attention must then equal the C attention pinned above."""
    b, bi = _block_batch("padded", seed=12)
    one = synth.f32_to_bf16_bits(np.eye(128, dtype=np.float32))
    ident = synth.BlockInputs(bi.x, np.concatenate([one, one, one]), np.zeros(384, np.float32), one,
                              np.zeros(128, np.float32))
    y = oracle_lib.block_forward(b, ident)
    qkv = bi.x.reshape(b.N, b.P, 8, 16).transpose(0, 2, 1, 3).copy()     # [N, H, P, D]
    ref = oracle_lib.attention(b, oracle_lib.pair_bias(b), qkv, qkv, qkv)
    np.testing.assert_allclose(y.reshape(b.N, b.P, 8, 16).transpose(0, 2, 1, 3), ref, rtol=1e-12, atol=1e-13)


def test_block_masked_rows_zero_and_output_bias_shift(oracle_lib):
    b, bi = _block_batch("padded", seed=13)
    y = oracle_lib.block_forward(b, bi)
    valid = b.mask.astype(bool)
    assert np.all(y[~valid] == 0.0)
    shifted = synth.BlockInputs(bi.x, bi.Wqkv, bi.bqkv, bi.Wo, bi.bo + np.float32(0.5))
    y2 = oracle_lib.block_forward(b, shifted)
    np.testing.assert_allclose(y2[valid] - y[valid], 0.5, atol=1e-12)
    assert np.all(y2[~valid] == 0.0)
