"""Pins of the fp64 backward oracle (oracle/backward.py), checked against
things other than itself: central finite differences of the scalar
sum(O * dO), the C oracle's forward, closed forms of the softmax gradient,
the U = 0 special case against torch's own attention backward in fp64, the
m = 1 jet, and permutation equivariance. A dropped term, a wrong sign or a transposed operand in any of
the gradient formulas fails at least one of these."""
import numpy as np
import pytest
import torch

from part_pair_bias_b200 import synth


@pytest.fixture(scope="module")
def bw(oracle_lib):
    from oracle import backward
    return backward


def tiny(seed=0, layout="padded", mults=(3, 5), P=6):
    kw = dict(N=len(mults), P=P, mults=list(mults), seed=seed, layout=layout)
    if layout == "padded":
        kw["mask_mode"] = "scrambled"
    return synth.make_jets(**kw)


def upstream(b, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(b.q.shape)


def test_forward_matches_c_oracle(bw, oracle_lib):
    for layout in ("padded", "packed"):
        b = tiny(1, layout)
        r = bw.backward(b, upstream(b, 1))
        ref = oracle_lib.forward(b)
        assert np.max(np.abs(r["out"] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_folded_form_equals_unfolded(bw):
    b = tiny(2)
    f = np.random.default_rng(2).standard_normal((50, 4)) * 5.0
    u1 = bw.mlp_forward(f, b.params)[0]
    u2 = bw.mlp_forward_folded(f, bw.fold(b.params))
    assert np.max(np.abs(u1 - u2)) <= 1e-11 * max(1.0, np.max(np.abs(u1)))


def test_gelu_grad_finite_difference(bw):
    z = np.linspace(-6, 6, 97)
    eps = 1e-6
    fd = (bw.gelu(z + eps) - bw.gelu(z - eps)) / (2 * eps)
    assert np.max(np.abs(fd - bw.gelu_grad(z))) <= 1e-8


def _fd_check(fn, x, idx, analytic, eps_rel=1e-6, tol=2e-6):
    # central differences: truncation ~h^2, rounding ~1e-16 |L| / h
    floor = 1e-8 * max(1.0, abs(fn()))
    for i in idx:
        h = eps_rel * max(1.0, abs(x.flat[i]))
        old = x.flat[i]
        x.flat[i] = old + h
        lp = fn()
        x.flat[i] = old - h
        lm = fn()
        x.flat[i] = old
        fd = (lp - lm) / (2 * h)
        an = analytic.flat[i]
        assert abs(fd - an) <= tol * abs(an) + floor, f"index {i}: fd {fd:.9e} analytic {an:.9e}"


@pytest.mark.parametrize("layout", ["padded", "packed"])
def test_qkv_gradients_finite_difference(bw, oracle_lib, layout):
    b = tiny(3, layout)
    dO = upstream(b, 3)
    feat = oracle_lib.features(b)
    r = bw.backward(b, dO, feat=feat)
    rng = np.random.default_rng(3)
    for name in ("q", "k", "v"):
        x = bw._to_f64(getattr(b, name)).copy()
        valid = np.flatnonzero(np.abs(r["d" + name]).reshape(-1) > 0)
        idx = rng.choice(valid, size=24, replace=False)

        def fn():
            return bw.loss(b, dO, feat=feat, **{name: x})
        _fd_check(fn, x, idx, r["d" + name])


def test_unfolded_parameter_gradients_finite_difference(bw, oracle_lib):
    b = tiny(4, mults=(4, 6))
    dO = upstream(b, 4)
    feat = oracle_lib.features(b)
    r = bw.backward(b, dO, feat=feat)
    params = bw.as_f64(b.params)
    rng = np.random.default_rng(4)
    for name in bw.PARAM_NAMES:
        x = params[name]
        idx = rng.choice(x.size, size=min(6, x.size), replace=False)
        _fd_check(lambda: bw.loss(b, dO, params=params, feat=feat), x, idx, r["unfolded"][name])


def test_folded_parameter_gradients_finite_difference(bw, oracle_lib):
    b = tiny(5, mults=(5, 2))
    dO = upstream(b, 5)
    feat = oracle_lib.features(b)
    r = bw.backward(b, dO, feat=feat)
    folded = bw.fold(b.params)
    rng = np.random.default_rng(5)
    for name in bw.FOLDED_NAMES:
        x = folded[name]
        idx = rng.choice(x.size, size=min(6, x.size), replace=False)
        _fd_check(lambda: bw.loss(b, dO, feat=feat, folded=folded), x, idx, r["folded"][name])


def test_softmax_gradient_closed_forms(bw):
    """Rows of dS sum to zero, so the last bias gets no gradient (db4 = 0),
    and the columns of P sum the upstream gradient into dV: sum_j dV_j =
    sum_i dO_i per jet and head."""
    b = tiny(6, mults=(7, 1, 4), P=8)
    dO = upstream(b, 6)
    r = bw.backward(b, dO)
    scale = np.abs(r["folded"]["W4"]).max()
    assert np.max(np.abs(r["folded"]["b4"])) <= 1e-12 * max(1.0, scale)
    dO64 = dO.reshape(b.N, 8, b.P, 16)
    dv = r["dv"].reshape(b.N, 8, b.P, 16)
    for n in range(b.N):
        slots = np.flatnonzero(b.mask[n * b.P:(n + 1) * b.P])
        np.testing.assert_allclose(dv[n][:, slots].sum(axis=1), dO64[n][:, slots].sum(axis=1), rtol=0, atol=1e-12)


def test_zero_bias_reduces_to_torch_attention_backward(bw):
    """W4 = 0, b4 = 0 gives U = 0: dq, dk, dv are those of plain masked
    attention (torch autograd of scaled_dot_product_attention, fp64), and no
    gradient reaches the hidden layers."""
    b = tiny(7, mults=(5, 3, 6), P=6)
    params = dict(b.params)
    params["W4"] = np.zeros_like(params["W4"])
    params["b4"] = np.zeros_like(params["b4"])
    dO = upstream(b, 7)
    r = bw.backward(b, dO, params=params)
    shape = (b.N, 8, b.P, 16)
    q, k, v = (torch.tensor(bw._to_f64(x).reshape(shape), requires_grad=True) for x in (b.q, b.k, b.v))
    mask = torch.tensor(b.mask.reshape(b.N, b.P).astype(bool))
    attn_mask = mask[:, None, None, :].expand(b.N, 8, b.P, b.P)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=attn_mask)
    rows = mask[:, None, :, None].to(torch.float64)
    (o * rows * torch.tensor(dO.reshape(shape))).sum().backward()
    for name, t in (("dq", q), ("dk", k), ("dv", v)):
        np.testing.assert_allclose(r[name].reshape(shape), (t.grad * rows).numpy(), rtol=0, atol=1e-12)
    for name in ("W1", "b1", "W2", "b2", "W3", "b3"):
        assert np.all(r["folded"][name] == 0.0)
    for name in ("a0", "c0", "a1", "c1", "a2", "c2", "a3", "c3"):
        assert np.all(r["unfolded"][name] == 0.0)


def test_single_particle_jet(bw):
    """m = 1: o = v exactly, dv = dO, and dq = dk = dU = 0."""
    b = tiny(8, mults=(1,), P=4)
    dO = upstream(b, 8)
    r = bw.backward(b, dO)
    s = int(np.flatnonzero(b.mask)[0])
    v = bw._to_f64(b.v).reshape(1, 8, 4, 16)
    np.testing.assert_array_equal(r["out"].reshape(1, 8, 4, 16)[0][:, s], v[0][:, s])
    np.testing.assert_array_equal(r["dv"].reshape(1, 8, 4, 16)[0][:, s], dO.reshape(1, 8, 4, 16)[0][:, s])
    assert np.all(r["dq"] == 0) and np.all(r["dk"] == 0)
    for name in bw.FOLDED_NAMES:
        assert np.all(r["folded"][name] == 0.0)


def test_permutation_equivariance(bw):
    """Reordering a jet's slots (momenta, mask, q, k, v and the upstream
    gradient alike) moves dq, dk, dv with them and leaves the parameter
    gradients, sums over all pairs, unchanged up to fp64 rounding."""
    b = tiny(9, mults=(5, 7, 3), P=8)
    dO = upstream(b, 9)
    rng = np.random.default_rng(9)
    perms = np.stack([rng.permutation(b.P) for _ in range(b.N)])
    c = lambda a: a.reshape(b.N, b.P)[np.arange(b.N)[:, None], perms].reshape(-1).copy()
    h = lambda a: a.reshape(b.N, 8, b.P, 16)[np.arange(b.N)[:, None, None], np.arange(8)[None, :, None],
                                             perms[:, None, :]].copy()
    bp = synth.JetBatch("padded", b.N, b.P, b.mult.copy(), c(b.E), c(b.px), c(b.py), c(b.pz), c(b.mask), None,
                        h(b.q), h(b.k), h(b.v), b.params)
    r0, r1 = bw.backward(b, dO), bw.backward(bp, h(dO))
    for name in ("out", "dq", "dk", "dv"):
        np.testing.assert_allclose(r1[name].reshape(b.N, 8, b.P, 16), h(r0[name]), rtol=0,
                                   atol=1e-12 * max(1.0, np.abs(r0[name]).max()))
    for name in bw.FOLDED_NAMES:
        np.testing.assert_allclose(r1["folded"][name], r0["folded"][name], rtol=1e-10,
                                   atol=1e-12 * max(1.0, np.abs(r0["folded"][name]).max()))
