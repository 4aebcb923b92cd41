"""The allocation-free fused entry point (static per-device scratch) against
the allocating one, through the C ABI, on two calls in a row: bit for bit
against pair_attention_forward given a caller workspace (the same balanced
kernel, deterministic), and against the fp64 oracle at the attention bar.

Collected last on purpose: it must hold both in a fresh process, where the
first call performs the per-device set-up, and after every other test has
run on the same device.
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


@pytest.mark.parametrize("name", ["pr1_n8_p32", "n128_p128"])
def test_noalloc_matches_fused_entry_point(oracle_lib, name):
    b = synth.make_jets(**configs.workload(name, seed=0))
    d = pt.Device(b)
    ref = d.fused(balanced=True)                  # the same kernel with a caller workspace
    assert ops.get_device_status() == 0
    oref = oracle_lib.forward(b)
    for _call in range(2):
        out = torch.full_like(d.q, float("nan"))
        ops.pair_attention_forward_noalloc(d.jets, d.mlp, d.q, d.k, d.v, out)
        assert ops.get_device_status() == 0
        assert torch.equal(out, ref), "noalloc output differs from the workspace call"
        pt.check_attention(pt.to_np(out), oref, b)


def test_noalloc_rejects_batches_beyond_the_static_scratch():
    b = synth.make_jets(N=256, P=256, mults=np.full(256, 4), seed=2)
    d = pt.Device(b)
    out = torch.empty_like(d.q)
    with pytest.raises(ops.PairBiasError) as ei:
        ops.pair_attention_forward_noalloc(d.jets, d.mlp, d.q, d.k, d.v, out)
    assert ei.value.status == ops.PB_EUNSUPPORTED
    assert "static scratch" in str(ei.value)
