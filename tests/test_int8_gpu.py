"""GPU parity of the int8 variant (int8 zero-point inputs to the hidden
layers on kind::i8 tensor cores) against the int8 variant of the fp64
oracle, through the C ABI.

Bars (tests/parity.py): U relative L2 <= 1e-2, >= 99 % of pair rows within
1e-3, every row within 0.25 (codes one rounding step apart, see
check_bias_i8); the bf16 U is the fp32 U rounded; the fused attention meets
the attention bars per (jet, head). Workloads: ternary hidden-layer weights
(the weights of a ternary-quantised network) and Gaussian ones (general
int8 codes), small cases in full and large ones on sampled jets.
"""
import numpy as np
import pytest
import torch

from part_pair_bias_b200 import configs, ops, synth
from tests import parity as pt

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    torch.cuda.set_device(0)
    ops.lib()
    yield
    assert ops.get_device_status() == 0


def sample_ranges(b):
    if b.N <= 128:
        return [(0, b.N)]
    w = 16 if b.N <= 512 else 32
    return [(0, w), (b.N // 2, b.N // 2 + w), (b.N - w, b.N)]


def per_jet(b, full, lo, hi):
    if b.layout == "padded":
        return full[lo:hi]
    return full[b.ptr[lo]:b.ptr[hi]]


@pytest.mark.parametrize("name,weights", [("pr1_n8_p32", "ternary"), ("n128_p128", "ternary"),
                                          ("n128_p128", "gaussian"), ("packed_8192", "ternary"),
                                          ("n256_p256_3prong", "ternary")])
def test_int8_bias_and_attention(oracle_lib, name, weights):
    b = synth.make_jets(**configs.workload(name, seed=0), weights=weights)
    d = pt.Device(b)
    U = pt.to_np(d.bias_i8())
    Ub = d.bias_i8(torch.bfloat16)
    out = pt.to_np(d.fused_i8())
    assert ops.get_device_status() == 0
    # the bf16 U is the fp32 U rounded (the same kernel, a different store)
    assert torch.equal(Ub, torch.from_numpy(U.astype(np.float32)).to(torch.bfloat16).cuda())
    stats = []
    for lo, hi in sample_ranges(b):
        s = synth.slice_jets(b, lo, hi)
        stats.append(pt.check_bias_i8(U[lo:hi], oracle_lib.pair_bias_i8(s), s))
        pt.check_attention(per_jet(b, out, lo, hi), oracle_lib.forward_i8(s), s)
    frac = min(x[0] for x in stats)
    print(f"\nint8 {name} {weights}: rows agreeing {frac * 100:.2f} %, worst row {max(x[1] for x in stats):.3e}, "
          f"rel L2 {max(x[2] for x in stats):.3e}")


def test_int8_edge_cases(oracle_lib):
    """Odd P, scrambled masks, empty / one-particle / full jets; packed with
    empty jets; P = 2..8."""
    cases = [dict(N=8, P=37, mults=[0, 1, 2, 37, 17, 36, 5, 33], mask_mode="scrambled", seed=3),
             dict(N=6, P=64, layout="packed", mults=[3, 0, 64, 1, 0, 20], seed=6),
             dict(N=5, P=256, mults=[256, 200, 129, 3, 0], pt_lo=800, pt_hi=1000, prongs=3, seed=5)]
    cases += [dict(N=8, P=P, mults=[0, 1, P, max(1, P - 1), 2, P, 0, P // 2 + 1], mask_mode="scrambled",
                   seed=30 + P) for P in (2, 3, 5, 8)]
    for kw in cases:
        b = synth.make_jets(**kw, weights="ternary")
        d = pt.Device(b)
        pt.check_bias_i8(pt.to_np(d.bias_i8()), oracle_lib.pair_bias_i8(b), b)
        pt.check_attention(pt.to_np(d.fused_i8()), oracle_lib.forward_i8(b), b)
        assert ops.get_device_status() == 0


def test_int8_deterministic_and_empty():
    b = synth.make_jets(**configs.workload("n128_p128", seed=1), weights="ternary")
    d = pt.Device(b)
    assert torch.equal(d.fused_i8(), d.fused_i8())
    assert torch.equal(d.bias_i8(), d.bias_i8())
    e = synth.make_jets(N=0, P=16, mults=np.zeros(0, int), seed=1)
    de = pt.Device(e)
    ops.pair_attention_forward_i8(de.jets, de.mlp_i8, de.q, de.k, de.v, torch.empty_like(de.q))
    assert ops.get_device_status() == 0
