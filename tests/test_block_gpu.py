"""GPU parity of the attention block with its projections (pair_block_forward)
against the fp64 oracle, through the C ABI.

y is checked like the attention output: relative L2 over the valid rows of
the batch and of every jet on its own (y mixes the heads), every element
within 0.1 * max(1, rms of the jet's rows), masked rows exactly 0. The in-projection alone is checked element by element on
the Q, K, V it leaves in the workspace: fp32 accumulation of exact bf16
products, then one bf16 rounding, so every element lies within half a bf16
ulp (plus a small accumulation allowance) of x W^T + b computed in fp64.
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


class Block:
    def __init__(self, b, seed=0):
        self.b = b
        self.bi = synth.make_block_inputs(b, seed)
        self.d = pt.Device(b)
        self.proj = ops.proj_to_device(self.bi)
        self.x = ops.bf16_to_device(self.bi.x)
        self.ws = torch.zeros(ops.block_workspace_bytes(self.d.jets), dtype=torch.uint8, device="cuda")

    def run(self):
        y = torch.full_like(self.x, float("nan"))
        ops.pair_block_forward(self.d.jets, self.d.mlp, self.proj, self.x, y, self.ws)
        return y


def valid_row_mask(b):
    if b.layout == "padded":
        return b.mask.astype(bool)
    return np.ones(int(b.ptr[-1]), bool)


def check_block(got, ref, b):
    vr = valid_row_mask(b)
    g, o = got[vr], ref[vr]
    rel = np.linalg.norm(g - o) / np.linalg.norm(o)
    assert rel <= pt.ATT_RELL2, f"block rel L2 {rel:.3e}"
    assert np.all(got[~vr] == 0.0), "masked rows of y must be 0"
    # per jet: y of the jet's valid rows as one [m, 1, 128] block
    if b.layout == "padded":
        gj = got.reshape(b.N, 1, b.P, -1)
        oj = ref.reshape(b.N, 1, b.P, -1)
    else:
        gj, oj = got[:, None, :], ref[:, None, :]
    pt.check_jet_heads(gj, oj, b, pt.ATT_RELL2, pt.ATT_OUTLIER)
    return float(rel)


def sample_ranges(b):
    if b.N <= 128:
        return [(0, b.N)]
    w = 16 if b.N <= 512 else 32
    return [(0, w), (b.N // 2, b.N // 2 + w), (b.N - w, b.N)]


@pytest.mark.parametrize("name", ["pr1_n8_p32", "n128_p128", "n512_p128", "packed_8192", "n256_p256_3prong"])
def test_block_against_oracle(oracle_lib, name):
    b = synth.make_jets(**configs.workload(name, seed=0))
    blk = Block(b)
    y = pt.to_np(blk.run())
    assert ops.get_device_status() == 0
    for lo, hi in sample_ranges(b):
        s = synth.slice_jets(b, lo, hi)
        si = synth.slice_block_inputs(b, blk.bi, lo, hi)
        rows = slice(lo * b.P, hi * b.P) if b.layout == "padded" else slice(int(b.ptr[lo]), int(b.ptr[hi]))
        check_block(y[rows], oracle_lib.block_forward(s, si), s)


def test_in_projection_within_bf16_rounding():
    b = synth.make_jets(N=6, P=37, mults=[0, 1, 37, 20, 5, 36], mask_mode="scrambled", seed=21)
    blk = Block(b, seed=3)
    blk.run()
    torch.cuda.synchronize()
    rows = b.N * b.P
    tb = (rows * 128 * 2 + 255) // 256 * 256
    x = synth.bf16_bits_to_f64(blk.bi.x)
    ref = x @ synth.bf16_bits_to_f64(blk.bi.Wqkv).T + blk.bi.bqkv.astype(np.float64)   # [rows, 384]
    valid = b.mask.astype(bool)
    for t in range(3):
        buf = blk.ws[t * tb:t * tb + rows * 256].view(torch.bfloat16).float().cpu().numpy().astype(np.float64)
        got = buf.reshape(b.N, 8, b.P, 16).transpose(0, 2, 1, 3).reshape(rows, 128)     # [N, H, P, D] -> rows
        r = ref[:, t * 128:(t + 1) * 128]
        err = np.abs(got[valid] - r[valid])
        tol = pt.bf16_half_ulp(r[valid]) * 1.001 + 1e-5 * np.abs(r[valid]) + 1e-6
        assert np.all(err <= tol), f"tensor {t}: max excess {(err - tol).max():.3e}"


def test_block_odd_p_scrambled_and_wide_jets(oracle_lib):
    for b in (synth.make_jets(N=8, P=37, mults=[0, 1, 2, 37, 17, 36, 5, 33], mask_mode="scrambled", seed=22),
              synth.make_jets(N=4, P=256, mults=[256, 200, 129, 3], pt_lo=800, pt_hi=1000, prongs=3, seed=23),
              synth.make_jets(N=6, P=64, layout="packed", mults=[3, 0, 64, 1, 0, 20], seed=24)):
        blk = Block(b, seed=5)
        check_block(pt.to_np(blk.run()), oracle_lib.block_forward(b, blk.bi), b)
    assert ops.get_device_status() == 0


def test_block_deterministic():
    b = synth.make_jets(**configs.workload("n128_p128", seed=1))
    blk = Block(b, seed=1)
    assert torch.equal(blk.run(), blk.run())
