"""Property test of the C ABI's host-side argument checks.

Every generated call carries at least one argument that the header declares
invalid: a NULL or misaligned pointer, a size out of range, an unsupported
H, D or E, both or neither of mlp and U, a workspace that is too small. Each
such call must be refused on the host with PB_EINVAL or PB_EUNSUPPORTED and a
message, before any CUDA call: without a GPU, a check that let the call
through would surface as PB_ECUDA instead. Only refusable calls are made, so
no kernel ever launches with these host addresses, on any machine."""
import ctypes as C

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from part_pair_bias_b200 import ops

# one 256-byte aligned host arena supplies every pointer; a misaligned
# pointer is an aligned one plus 2 bytes (breaks 4-, 16- and 256-byte rules)
_ARENA = np.zeros(1 << 16, np.uint8)
_BASE = (_ARENA.ctypes.data + 255) // 256 * 256


def _ptr(i):
    return _BASE + 256 * i


@pytest.fixture(scope="module")
def L():
    from part_pair_bias_b200 import build
    build.build()
    return ops.lib()


JET_VIOLATIONS = ["jets_null", "n_negative", "p_zero", "p_too_big", "momentum_null", "momentum_misaligned",
                  "layout_missing", "ptr_misaligned", "tokens_negative"]
ENTRY_VIOLATIONS = {
    "pairfeat": ["feat_null", "feat_misaligned"],
    "mlp_forward": ["mlp_null", "mlp_field_null", "mlp_misaligned", "u_null", "u_misaligned", "dtype_bad"],
    "attention": ["hd_bad", "mlp_and_u", "neither", "qkvo_null", "qkvo_misaligned", "u_misaligned",
                  "mlp_field_null", "mlp_misaligned", "ws_misaligned"],
    "noalloc": ["hd_bad", "mlp_null", "mlp_field_null", "mlp_misaligned", "qkvo_null", "qkvo_misaligned"],
    "block": ["hde_bad", "mlp_null", "mlp_misaligned", "proj_null", "proj_field_null", "proj_misaligned", "xy_null",
              "xy_misaligned", "ws_null", "ws_misaligned", "ws_small"],
    "backward": ["hd_bad", "mlp_null", "mlp_misaligned", "dmlp_null", "dmlp_field_null", "dmlp_misaligned", "qkv_grad_null",
                 "qkv_grad_misaligned", "ws_null", "ws_misaligned", "ws_small"],
    "mlp_forward_i8": ["mlp_null", "i8_field_null", "i8_codes_misaligned", "u_null", "u_misaligned", "dtype_bad"],
    "attention_i8": ["hd_bad", "mlp_null", "i8_field_null", "i8_codes_misaligned", "qkvo_null", "qkvo_misaligned"],
}


def _make_jets(N, P, packed, v):
    js = ops._Jets(_ptr(0), _ptr(1), _ptr(2), _ptr(3), None if packed else _ptr(4), _ptr(5) if packed else None,
                   N, P, N if packed else 0)
    if "n_negative" in v:
        js.N = -1 - N
    if "p_zero" in v:
        js.P = 0
    if "p_too_big" in v:
        js.P = 257 + P
    if "momentum_null" in v:
        js.py = None
    if "momentum_misaligned" in v:
        js.px = _ptr(1) + 2
    if "layout_missing" in v:
        js.mask, js.ptr = None, None
    if "ptr_misaligned" in v and packed:
        js.ptr = _ptr(5) + 2
    if "tokens_negative" in v and packed:
        js.tokens = -1
    return None if "jets_null" in v else C.byref(js), js


def _applicable(entry, packed):
    jet = [x for x in JET_VIOLATIONS if packed or x not in ("ptr_misaligned", "tokens_negative")]
    return jet + ENTRY_VIOLATIONS[entry]


def _call(L, entry, jets, v):
    d = _ptr(8)
    mis = lambda p, bad: p + 2 if bad else p  # noqa: E731
    mlp = None if "mlp_null" in v else ops._Mlp(*([_ptr(10)] * 7 + [0 if "mlp_field_null" in v else _ptr(11)]))
    if mlp is not None and "mlp_misaligned" in v:
        mlp.W3 = _ptr(10) + 4  # 4-byte aligned floats, but the matrices need 16
    mlp_ref = None if mlp is None else C.byref(mlp)
    q, k, vv, out = (None if "qkvo_null" in v and i == 3 else mis(_ptr(12 + i), "qkvo_misaligned" in v and i == 1)
                     for i in range(4))
    m8 = ops._MlpI8(*([_ptr(90 + i) for i in range(11)]))
    if "i8_field_null" in v:
        m8.a3 = None
    if "i8_codes_misaligned" in v:
        m8.T4 = _ptr(94) + 4
    m8_ref = None if "mlp_null" in v else C.byref(m8)
    if entry == "mlp_forward_i8":
        U = None if "u_null" in v else mis(_ptr(20), "u_misaligned" in v)
        return L.pairbias_mlp_forward_i8(jets, m8_ref, U, 5 if "dtype_bad" in v else 0, None)
    if entry == "attention_i8":
        H, D = (8, 8) if "hd_bad" in v else (8, 16)
        return L.pair_attention_forward_i8(jets, m8_ref, H, D, q, k, vv, out, None)
    if entry == "pairfeat":
        return L.pairfeat_compute(jets, None if "feat_null" in v else mis(d, "feat_misaligned" in v), None)
    if entry == "mlp_forward":
        U = None if "u_null" in v else mis(_ptr(20), "u_misaligned" in v)
        return L.pairbias_mlp_forward(jets, mlp_ref, U, 5 if "dtype_bad" in v else 0, None)
    if entry == "attention":
        H, D = (4, 16) if "hd_bad" in v else (8, 16)
        U = mis(_ptr(20), "u_misaligned" in v)
        if "mlp_and_u" in v:
            m, u = mlp_ref, U
        elif "neither" in v:
            m, u = None, None
        elif "u_misaligned" in v:
            m, u = None, U
        else:
            m, u = mlp_ref, None
        ws = mis(_ptr(24), True) if "ws_misaligned" in v else None
        return L.pair_attention_forward(jets, m, u, H, D, q, k, vv, out, ws, 1 << 20 if ws else 0, None)
    if entry == "noalloc":
        H, D = (8, 32) if "hd_bad" in v else (8, 16)
        return L.pair_attention_forward_noalloc(jets, mlp_ref, H, D, q, k, vv, out, None)
    if entry == "block":
        H, D, E = (8, 16, 64) if "hde_bad" in v else (8, 16, 128)
        pr = ops._Proj(_ptr(30), _ptr(31), None if "proj_field_null" in v else _ptr(32), _ptr(33))
        if "proj_misaligned" in v:
            pr.Wqkv = _ptr(30) + 2
        proj = None if "proj_null" in v else C.byref(pr)
        x = None if "xy_null" in v else _ptr(34)
        y = mis(_ptr(35), "xy_misaligned" in v)
        ws = None if "ws_null" in v else mis(_ptr(40), "ws_misaligned" in v)
        return L.pair_block_forward(jets, mlp_ref, proj, H, D, E, x, y, ws, 0 if "ws_small" in v else 1 << 40, None)
    if entry == "backward":
        H, D = (16, 16) if "hd_bad" in v else (8, 16)
        g = ops._Mlp(*([_ptr(50)] * 7 + [None if "dmlp_field_null" in v else _ptr(51)]))
        if "dmlp_misaligned" in v:
            g.W2 = _ptr(50) + 2
        dmlp = None if "dmlp_null" in v else C.byref(g)
        t = [_ptr(60 + i) for i in range(7)]
        if "qkv_grad_null" in v:
            t[5] = None
        if "qkv_grad_misaligned" in v:
            t[2] += 2
        ws = None if "ws_null" in v else mis(_ptr(80), "ws_misaligned" in v)
        return L.pair_attention_backward(jets, mlp_ref, H, D, *t, dmlp, ws, 0 if "ws_small" in v else 1 << 40,
                                         None)
    raise AssertionError(entry)


@settings(max_examples=400, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(entry=st.sampled_from(sorted(ENTRY_VIOLATIONS)), N=st.integers(1, 300), P=st.integers(1, 256),
       packed=st.booleans(), data=st.data())
def test_invalid_calls_are_refused_on_the_host(L, entry, N, P, packed, data):
    choices = _applicable(entry, packed)
    v = set(data.draw(st.lists(st.sampled_from(choices), min_size=1, max_size=3, unique=True)))
    jets, keep = _make_jets(N, P, packed, v)
    st_ = _call(L, entry, jets, v)
    assert st_ in (ops.PB_EINVAL, ops.PB_EUNSUPPORTED), (entry, sorted(v), st_, L.pb_last_error())
    assert L.pb_last_error(), "a refusal carries a message"
