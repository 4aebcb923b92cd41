"""The C-ABI library without a GPU: it builds, loads, exports every declared
symbol, rejects bad arguments on the host, and its batch-norm folding agrees
with the oracle's unfolded MLP."""
import ctypes as C
import os
import re

import numpy as np
import pytest
from scipy.special import erf

from part_pair_bias_b200 import ops, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pairbias.h")


@pytest.fixture(scope="module")
def L():
    from part_pair_bias_b200 import build
    build.build()
    return ops.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(\w+)\s*\(", text, flags=re.M)


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert {"pairfeat_compute", "pairbias_mlp_forward", "pair_attention_forward",
            "pb_get_device_status", "pb_fold_affine", "pb_last_error", "pb_version",
            "pb_workspace_bytes", "pair_attention_forward_noalloc", "pair_attention_backward",
            "pb_backward_workspace_bytes", "pb_unfold_grad"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in pairbias.h but not exported"
    assert ops.version().startswith("pairbias-b200")


def test_build_watches_every_source():
    """A change to any file under csrc/ (or the header) makes the library stale."""
    from part_pair_bias_b200 import build
    csrc = os.path.join(ROOT, "part_pair_bias_b200", "csrc")
    sources = {os.path.join(csrc, f) for f in os.listdir(csrc)} | {HEADER}
    assert sources <= set(build.DEPS)


def _jets(N=2, P=8, ptr=False, aligned=True):
    buf = np.zeros(64, np.float32)
    base = buf.ctypes.data + (0 if aligned else 1)
    m = np.ones(N * P, np.uint8)
    p = np.zeros(N + 1, np.int32)
    js = ops._Jets(base, base, base, base, m.ctypes.data, p.ctypes.data if ptr else None, N, P, 0)
    return js, (buf, m, p)


def test_host_validation(L):
    js, keep = _jets()
    dummy = np.zeros(64, np.float32)
    d = dummy.ctypes.data
    assert L.pairfeat_compute(None, d, None) == ops.PB_EINVAL
    assert "NULL" in ops.lib().pb_last_error().decode()
    js.P = 0
    assert L.pairfeat_compute(C.byref(js), d, None) == ops.PB_EUNSUPPORTED
    js.P = 257
    assert L.pairfeat_compute(C.byref(js), d, None) == ops.PB_EUNSUPPORTED
    js.P = 8
    js.N = -1
    assert L.pairfeat_compute(C.byref(js), d, None) == ops.PB_EINVAL
    js.N = 2
    assert L.pairfeat_compute(C.byref(js), d + 4, None) == ops.PB_EINVAL   # feat not 16-byte aligned
    js.mask = None
    assert L.pairfeat_compute(C.byref(js), d, None) == ops.PB_EINVAL       # padded without mask
    js2, keep2 = _jets(aligned=False)
    assert L.pairfeat_compute(C.byref(js2), d, None) == ops.PB_EINVAL      # misaligned momenta
    js3, keep3 = _jets()
    mlp = ops._Mlp(*([d] * 8))
    assert L.pair_attention_forward(C.byref(js3), C.byref(mlp), None, 4, 16, d, d, d, d, None, 0, None) == ops.PB_EUNSUPPORTED
    assert L.pair_attention_forward(C.byref(js3), C.byref(mlp), None, 8, 32, d, d, d, d, None, 0, None) == ops.PB_EUNSUPPORTED
    assert L.pair_attention_forward(C.byref(js3), C.byref(mlp), d, 8, 16, d, d, d, d, None, 0, None) == ops.PB_EINVAL
    assert L.pair_attention_forward(C.byref(js3), None, None, 8, 16, d, d, d, d, None, 0, None) == ops.PB_EINVAL
    assert L.pair_attention_forward(C.byref(js3), C.byref(mlp), None, 8, 16, d + 2, d, d, d, None, 0, None) == ops.PB_EINVAL
    assert L.pairbias_mlp_forward(C.byref(js3), C.byref(mlp), d, 7, None) == ops.PB_EINVAL
    bad = ops._Mlp(*([d] * 7 + [0]))
    assert L.pairbias_mlp_forward(C.byref(js3), C.byref(bad), d, 0, None) == ops.PB_EINVAL
    # misaligned workspace on the fused path (16 bytes past a 256-byte boundary)
    wbuf = np.zeros(1024, np.uint8)
    ws = (wbuf.ctypes.data + 255) // 256 * 256 + 16
    assert L.pair_attention_forward(C.byref(js3), C.byref(mlp), None, 8, 16, d, d, d, d, ws, 1 << 20,
                                    None) == ops.PB_EINVAL
    # N = 0 is a no-op that needs no device
    js3.N = 0
    assert L.pairfeat_compute(C.byref(js3), d, None) == ops.PB_OK


def test_fold_affine_matches_unfolded_oracle(L, oracle_lib):
    """The folded network (product host helper) equals the oracle's unfolded
    MLP up to the fp32 rounding of the folded parameters."""
    rng = np.random.default_rng(21)
    for seed in range(3):
        p = synth.make_params(np.random.default_rng(seed))
        flat = ops.fold_affine(p).astype(np.float64)
        get = lambda name: flat[ops.FOLDED_OFFSETS[name][0]:][:int(np.prod(ops.FOLDED_OFFSETS[name][1]))].reshape(
            ops.FOLDED_OFFSETS[name][1])
        gelu = lambda x: 0.5 * x * (1 + erf(x / np.sqrt(2)))
        for _ in range(50):
            f = rng.uniform(-18.4, 12, 4)
            h = gelu(get("W1") @ f + get("b1"))
            h = gelu(get("W2") @ h + get("b2"))
            h = gelu(get("W3") @ h + get("b3"))
            u = get("W4") @ h + get("b4")
            ref = oracle_lib.mlp_row(f, p)
            assert np.max(np.abs(u - ref)) < 2e-5 * max(1.0, np.max(np.abs(ref)))
    assert L.pb_fold_affine(None, None) == ops.PB_EINVAL


def test_workspace_size_rules(L):
    """The balanced fused path's workspace: header + 16 bytes per row of every
    jet's 128-row tiles; 0 where the path does not apply."""
    js, keep = _jets(N=128, P=128)
    tiles = (128 * 129 // 2 + 127) // 128
    assert L.pb_workspace_bytes(C.byref(js)) == 256 + 128 * tiles * 128 * 16
    js.N = 9000                       # more jets than the jet table holds
    assert L.pb_workspace_bytes(C.byref(js)) == 0
    js.N = 0
    assert L.pb_workspace_bytes(C.byref(js)) == 0
    js4, keep4 = _jets(N=8192, P=128, ptr=True)
    js4.tokens = 327680               # packed: bounded by the token count
    assert L.pb_workspace_bytes(C.byref(js4)) == 256 + (327680 * 129 // 2 + 127 * 8192 + 128) * 16


def test_noalloc_host_rejections(L):
    """The static-scratch entry point decides on the host, before any device
    call, that a batch does not fit its scratch or its kernel."""
    js, keep = _jets(N=256, P=256)
    d = np.zeros(64, np.float32).ctypes.data
    mlp = ops._Mlp(*([d] * 8))
    need = 256 + 256 * ((256 * 257 // 2 + 127) // 128) * 128 * 16
    assert need > ops.PB_STATIC_SCRATCH_BYTES
    assert L.pair_attention_forward_noalloc(C.byref(js), C.byref(mlp), 8, 16, d, d, d, d, None) == ops.PB_EUNSUPPORTED
    assert "static scratch" in L.pb_last_error().decode()
    js.N = 9000                       # beyond the balanced kernel's jet table
    assert L.pair_attention_forward_noalloc(C.byref(js), C.byref(mlp), 8, 16, d, d, d, d, None) == ops.PB_EUNSUPPORTED
    js.N = 2
    assert L.pair_attention_forward_noalloc(C.byref(js), None, 8, 16, d, d, d, d, None) == ops.PB_EINVAL
    assert L.pair_attention_forward_noalloc(C.byref(js), C.byref(mlp), 8, 16, d + 2, d, d, d, None) == ops.PB_EINVAL
    js.N = 0                          # nothing to do: no device needed
    assert L.pair_attention_forward_noalloc(C.byref(js), C.byref(mlp), 8, 16, d, d, d, d, None) == ops.PB_OK


def test_block_host_validation_and_workspace(L):
    js, keep = _jets(N=2, P=8)
    d = np.zeros(64, np.float32).ctypes.data
    mlp = ops._Mlp(*([d] * 8))
    proj = ops._Proj(d, d, d, d)
    need = 4 * ((2 * 8 * 128 * 2 + 255) // 256 * 256)
    assert L.pb_block_workspace_bytes(C.byref(js)) == need
    wbuf = np.zeros(need + 512, np.uint8)
    ws = (wbuf.ctypes.data + 255) // 256 * 256
    call = lambda **kw: L.pair_block_forward(C.byref(js), C.byref(mlp), kw.get("proj", C.byref(proj)), 8, 16,
                                             kw.get("E", 128), kw.get("x", d), d, kw.get("ws", ws),
                                             kw.get("wsb", need), None)
    assert call(E=64) == ops.PB_EUNSUPPORTED
    assert call(proj=None) == ops.PB_EINVAL
    assert call(x=d + 8) == ops.PB_EINVAL                   # x not 16-byte aligned
    assert call(wsb=need - 1) == ops.PB_EINVAL              # workspace too small
    assert call(ws=ws + 16) == ops.PB_EINVAL                # workspace not 256-byte aligned
    bad = ops._Proj(d, d, None, d)
    assert call(proj=C.byref(bad)) == ops.PB_EINVAL
    js.N = 0                                                # nothing to do, no device needed
    assert call() == ops.PB_OK


def _r256(b):
    return (b + 255) // 256 * 256


def test_backward_workspace_size(L):
    """Header, 16-byte bias and 32-byte gradient records for the rows of a
    chunk's tiles (at most 8192 jets, padded N*P <= 2^21), the chunk's tile
    prefix and 256 fp32 partials of the folded weight gradients."""
    def want(N, P, tokens=None):
        nc = min(N, 8192 if tokens is not None else min(8192, (1 << 21) // P))
        rows = nc * ((P * (P + 1) // 2 + 127) // 128) * 128
        if tokens is not None:
            rows = min(rows, tokens * (P + 1) // 2 + 127 * nc + 128)
        grec = _r256(256 + rows * 16)
        table = _r256(grec + rows * 32)
        part = _r256(table + (nc + 1) * 4)
        return _r256(part + 256 * ops.FOLDED_FLOATS * 4)
    for N, P in ((2, 8), (128, 128), (300, 37), (20000, 256)):
        js, keep = _jets(N=N, P=P)
        assert L.pb_backward_workspace_bytes(C.byref(js)) == want(N, P)
    js, keep = _jets(N=8192, P=128, ptr=True)
    js.tokens = 327680
    assert L.pb_backward_workspace_bytes(C.byref(js)) == want(8192, 128, 327680)
    js.P = 300
    assert L.pb_backward_workspace_bytes(C.byref(js)) == 0


def test_backward_host_rejections(L):
    """Argument errors of pair_attention_backward return before any launch."""
    js, keep = _jets(N=2, P=8)
    buf = np.zeros(1 << 16, np.uint8)
    d = (buf.ctypes.data + 255) // 256 * 256
    mlp = ops._Mlp(*([d] * 8))
    grad = ops._Mlp(*([d] * 8))
    need = L.pb_backward_workspace_bytes(C.byref(js))
    call = lambda H=8, D=16, m=mlp, q=d, dout=d, g=grad, ws=d, wsb=need: L.pair_attention_backward(
        C.byref(js), None if m is None else C.byref(m), H, D, q, d, d, dout, d, d, d,
        None if g is None else C.byref(g), ws, wsb, None)
    assert call(H=4) == ops.PB_EUNSUPPORTED
    assert call(D=32) == ops.PB_EUNSUPPORTED
    assert call(m=None) == ops.PB_EINVAL
    assert call(g=None) == ops.PB_EINVAL
    assert call(g=ops._Mlp(*([d] * 7 + [0]))) == ops.PB_EINVAL
    assert call(g=ops._Mlp(*([d] * 7 + [d + 2]))) == ops.PB_EINVAL       # misaligned gradient buffer
    assert call(q=None) == ops.PB_EINVAL
    assert call(dout=d + 2) == ops.PB_EINVAL                            # misaligned upstream gradient
    assert call(ws=None) == ops.PB_EINVAL
    assert call(ws=d + 16) == ops.PB_EINVAL                             # workspace not 256-byte aligned
    assert call(wsb=need - 1) == ops.PB_EINVAL
    assert "pb_backward_workspace_bytes" in L.pb_last_error().decode()


def test_unfold_grad_matches_oracle(L, oracle_lib):
    """The host helper's chain rule through the folding reproduces the
    oracle's directly computed gradients of the unfolded parameters."""
    from oracle import backward as bw
    for seed in range(3):
        b = synth.make_jets(N=3, P=8, mults=[5, 8, 3], mask_mode="scrambled", seed=40 + seed)
        dO = np.random.default_rng(seed).standard_normal(b.q.shape)
        r = bw.backward(b, dO)
        flat = np.zeros(ops.FOLDED_FLOATS)
        for name, (off, shape) in ops.FOLDED_OFFSETS.items():
            flat[off:off + int(np.prod(shape))] = r["folded"][name].reshape(-1)
        got = ops.unfold_grad(b.params, flat)
        for name, ref in r["unfolded"].items():
            scale = max(np.max(np.abs(ref)), 1e-30)
            assert np.max(np.abs(got[name] - ref)) <= 1e-5 * scale, name
    assert L.pb_unfold_grad(None, None, None) == ops.PB_EINVAL
