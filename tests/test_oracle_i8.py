"""Pins of the oracle's int8 variant (CPU).

The variant follows "Economical Jet Taggers -- Equivariant, Slim and
Quantised", section "Kwantiseringsstrategieen": inputs of the hidden linear
layers are int8 with zero-point quantisation, weights ternary. Each pin
checks a property the definition fixes, not a retyped formula:
  quantiser   codes in [-128, 127]; the row's lower end (min(0, min x))
              maps to -128 and its upper end to 127; 0 is represented
              exactly (code z); every value within half a step s;
  weights     ternary rows are represented exactly (alpha * T == W, codes
              +-127 and 0); other rows within alpha / 2, largest |code| 127;
  layer       on inputs that lie on the quantisation grid, with ternary
              weights, the int8 layer equals the float layer W x + b; off the
              grid, the first-order error bound of the two roundings holds;
  MLP row     the int8 row equals the composition, in the order the reading
              states, of the pinned pieces (layer 1 float, then for layers
              2..4: quantise the row, int8 layer, GELU for 2 and 3), and
              differs from the float MLP by a small, non-zero amount.
"""
import numpy as np
import pytest

from part_pair_bias_b200 import configs, synth


@pytest.fixture(scope="module")
def orc(oracle_lib):
    return oracle_lib


def _rows():
    rng = np.random.default_rng(5)
    yield rng.normal(0.0, 1.0, 64)                    # mixed signs
    yield np.abs(rng.normal(0.0, 3.0, 64))             # non-negative (GELU-like)
    yield -np.abs(rng.normal(0.0, 0.2, 64))            # non-positive
    yield np.concatenate([[-0.17], rng.uniform(-0.17, 30.0, 63)])   # a hidden row with a diagonal-pair tail
    yield np.zeros(64)                                 # all zero
    yield np.full(64, 2.5)                             # constant positive
    yield np.array([1e-30, -1e-30] * 32)               # tiny


@pytest.mark.parametrize("i", range(7))
def test_quantizer_round_trip(orc, i):
    x = list(_rows())[i]
    q, s, z = orc.quantize_act(x)
    q = q.astype(np.int64)
    assert q.min() >= -128 and q.max() <= 127
    lo, hi = min(0.0, x.min()), max(0.0, x.max())
    assert s > 0
    assert -128 <= z <= 127
    # 0 is represented exactly
    assert np.all(q[x == 0.0] == z)
    # every value within half a step
    assert np.all(np.abs(s * (q - z) - x) <= 0.5 * s * (1 + 1e-12))
    if hi > lo:
        # the ends of the row's range map to the ends of the code range
        if x.min() < 0:
            assert q[np.argmin(x)] == -128
        if x.max() > 0:
            assert q[np.argmax(x)] == 127
        assert np.isclose(s * 255.0, hi - lo, rtol=1e-14)
    else:
        assert s == 1.0 and z == -128 and np.all(q == -128)


def test_weight_codes(orc):
    rng = np.random.default_rng(6)
    t = rng.integers(-1, 2, size=(64, 64)).astype(np.float64)
    tau = rng.uniform(0.1, 0.3, size=(64, 1))
    W = tau * t
    T, alpha = orc.quantize_weights(W)
    assert set(np.unique(T)) <= {-127, 0, 127}
    np.testing.assert_allclose(alpha[:, None] * T, W, rtol=1e-15, atol=0)
    G = rng.normal(0.0, 0.125, size=(8, 64))
    G[3] = 0.0
    T, alpha = orc.quantize_weights(G)
    assert np.all(np.abs(alpha[:, None] * T - G) <= 0.5 * alpha[:, None] * (1 + 1e-12))
    assert np.all(np.abs(T[[0, 1, 2, 4, 5, 6, 7]]).max(axis=1) == 127)
    assert alpha[3] == 1.0 and np.all(T[3] == 0)


def test_int8_layer_exact_on_the_grid(orc):
    rng = np.random.default_rng(7)
    s0, z0 = 0.037, -57
    n = rng.integers(-128, 128, 64)
    n[:3] = (-128, 127, z0)                           # both ends and the zero point
    x = s0 * (n - z0)
    W = rng.uniform(0.05, 0.2, (64, 1)) * rng.integers(-1, 2, (64, 64))
    b = rng.normal(0.0, 0.1, 64)
    y = orc.int8_linear(x, W, b)
    np.testing.assert_allclose(y, W @ x + b, rtol=1e-12, atol=1e-12)


def test_int8_layer_error_bound(orc):
    rng = np.random.default_rng(8)
    for _ in range(20):
        x = rng.normal(0.0, 1.0, 64) * rng.uniform(0.1, 10.0)
        W = rng.normal(0.0, 0.125, (64, 64))
        b = rng.normal(0.0, 0.1, 64)
        y = orc.int8_linear(x, W, b)
        _, s, _ = orc.quantize_act(x)
        _, alpha = orc.quantize_weights(W)
        bound = np.abs(W).sum(1) * s / 2 + np.abs(x).sum() * alpha / 2 + 64 * alpha * s / 4
        assert np.all(np.abs(y - (W @ x + b)) <= bound * (1 + 1e-9))


def _folded(p, k):
    W = p[f"W{k}"].astype(np.float64)
    b = p[f"b{k}"].astype(np.float64)
    if k == 4:
        return W, b
    a, c = p[f"a{k}"].astype(np.float64), p[f"c{k}"].astype(np.float64)
    return a[:, None] * W, a * b + c


@pytest.mark.parametrize("weights", ["ternary", "gaussian"])
def test_mlp_row_is_the_composition(orc, weights):
    b = synth.make_jets(**configs.workload("pr1_n8_p32", seed=2), weights=weights)
    p = b.params
    rng = np.random.default_rng(9)
    gelu = np.vectorize(orc.gelu)
    for _ in range(40):
        f = rng.normal(0.0, 3.0, 4)
        x = p["a0"].astype(np.float64) * f + p["c0"].astype(np.float64)
        W1, b1 = _folded(p, 1)
        h = gelu(W1 @ x + b1)
        for k in (2, 3, 4):
            Wk, bk = _folded(p, k)
            y = orc.int8_linear(h, Wk, bk)
            h = gelu(y) if k < 4 else y
        np.testing.assert_allclose(orc.mlp_row_i8(f, p), h, rtol=1e-12, atol=1e-12)


def test_int8_bias_close_to_float_and_symmetric(orc):
    b = synth.make_jets(**configs.workload("pr1_n8_p32", seed=0), weights="ternary")
    U8, U = orc.pair_bias_i8(b), orc.pair_bias(b)
    m = b.mask.reshape(b.N, b.P).astype(bool)
    vp = np.broadcast_to((m[:, :, None] & m[:, None, :])[:, None], U.shape)
    d = U8[vp] - U[vp]
    rel = np.linalg.norm(d) / np.linalg.norm(U[vp])
    assert 1e-4 < rel < 5e-2                           # quantised, but close
    assert np.array_equal(U8, U8.transpose(0, 1, 3, 2))
    assert np.all(U8[~vp] == 0.0)
    out = orc.forward_i8(b)
    assert np.all(out[~np.broadcast_to(m[:, None, :, None], out.shape)] == 0.0)
