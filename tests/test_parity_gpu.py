"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small workloads are compared element by element in full; the large ones run
at full size on the GPU (the launch the benchmark times) and are compared on
sampled jets that the oracle computes one range at a time. Edge cases: odd P,
scrambled masks, empty / one-particle / full jets, P = 256 jets whose bias
does not fit on chip (query-block path), packed jets, an invalid ptr array.
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


_BATCHES = {}


def batch(name, **over):
    key = (name, tuple(sorted(over.items())))
    if key not in _BATCHES:
        _BATCHES[key] = synth.make_jets(**configs.workload(name, seed=0, **over))
    return _BATCHES[key]


def sample_ranges(b):
    """Jet ranges the oracle recomputes for a large batch."""
    N = b.N
    if N <= 128:
        return [(0, N)]
    w = 16 if N <= 512 else 32
    rs = [(0, w), (N // 2, N // 2 + w), (N - w, N)]
    big = int(np.argmax(b.mult))  # the widest jet (query-block path when m > 128)
    if not any(lo <= big < hi for lo, hi in rs):
        rs.append((big, big + 1))
    return rs


def per_jet(b, full, lo, hi):
    if b.layout == "padded" or full.shape[0] == b.N:
        return full[lo:hi]
    return full[b.ptr[lo]:b.ptr[hi]]


ALL = ["pr1_n8_p32", "n128_p128", "n512_p128", "packed_8192", "n256_p256_3prong"]


@pytest.mark.parametrize("name", ALL)
def test_features(oracle_lib, name):
    b = batch(name)
    d = pt.Device(b)
    got = pt.to_np(d.features())
    assert ops.get_device_status() == 0
    for lo, hi in sample_ranges(b):
        s = synth.slice_jets(b, lo, hi)
        pt.check_features(got[lo:hi], oracle_lib.features(s), s)


@pytest.mark.parametrize("name", ALL)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bias(oracle_lib, name, dtype):
    b = batch(name)
    d = pt.Device(b)
    got = pt.to_np(d.bias(dtype))
    assert ops.get_device_status() == 0
    worst = (0.0, 0.0)
    for lo, hi in sample_ranges(b):
        s = synth.slice_jets(b, lo, hi)
        e = pt.check_bias(got[lo:hi], oracle_lib.pair_bias(s), s, bf16=dtype == torch.bfloat16)
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    print(f"\nU error {name} {dtype}: max-abs {worst[0]:.3e}, rel L2 {worst[1]:.3e}")


@pytest.mark.parametrize("name", ALL)
@pytest.mark.parametrize("balanced", [False, True])
def test_fused_attention(oracle_lib, name, balanced):
    b = batch(name)
    d = pt.Device(b)
    got = pt.to_np(d.fused(balanced))
    assert ops.get_device_status() == 0
    for lo, hi in sample_ranges(b):
        s = synth.slice_jets(b, lo, hi)
        pt.check_attention(per_jet(b, got, lo, hi), oracle_lib.forward(s), s)


@pytest.mark.parametrize("name", ["pr1_n8_p32", "n128_p128", "n512_p128", "n256_p256_3prong"])
def test_materialised_bias_then_attention(oracle_lib, name):
    """The standalone path: bf16 U written to HBM, then attention reading it."""
    b = batch(name)
    d = pt.Device(b)
    U = d.bias(torch.bfloat16)
    got = pt.to_np(d.with_bias(U))
    assert ops.get_device_status() == 0
    for lo, hi in sample_ranges(b):
        s = synth.slice_jets(b, lo, hi)
        pt.check_attention(per_jet(b, got, lo, hi), oracle_lib.forward(s), s)


@pytest.mark.parametrize("name", ["pr1_n8_p32", "n128_p128"])
def test_attention_kernel_alone(oracle_lib, name):
    """Attention with the oracle's own bias (rounded to bf16) isolates the
    attention kernel: the oracle sees exactly the bias the kernel reads."""
    b = batch(name)
    d = pt.Device(b)
    U = pt.bf16_round(oracle_lib.pair_bias(b))
    Ud = torch.from_numpy(U.astype(np.float32)).to(torch.bfloat16).cuda()
    got = pt.to_np(d.with_bias(Ud))
    rel = pt.check_attention(got, oracle_lib.attention(b, U), b)
    assert rel < 5e-3


def test_odd_p_scrambled_masks_and_degenerate_jets(oracle_lib):
    b = synth.make_jets(N=8, P=37, mults=[0, 1, 2, 37, 17, 36, 5, 33], mask_mode="scrambled", seed=3)
    d = pt.Device(b)
    pt.check_features(pt.to_np(d.features()), oracle_lib.features(b), b)
    pt.check_bias(pt.to_np(d.bias()), oracle_lib.pair_bias(b), b)
    ref = oracle_lib.forward(b)
    for balanced in (False, True):
        got = pt.to_np(d.fused(balanced))
        pt.check_attention(got, ref, b)
        assert np.all(got[0] == 0.0)                 # empty jet: every row masked
    assert ops.get_device_status() == 0


def test_wide_jets_query_block_path(oracle_lib):
    """P = 256 with jets above 128 particles: the bias of a whole jet no longer
    fits on chip and the fused kernel tiles queries."""
    b = synth.make_jets(N=5, P=256, mults=[256, 200, 129, 128, 3], pt_lo=800, pt_hi=1000, prongs=3, seed=5)
    d = pt.Device(b)
    pt.check_bias(pt.to_np(d.bias()), oracle_lib.pair_bias(b), b)
    ref = oracle_lib.forward(b)
    pt.check_attention(pt.to_np(d.fused()), ref, b)
    pt.check_attention(pt.to_np(d.fused(balanced=True)), ref, b)   # whole triangles in the records
    assert ops.get_device_status() == 0


@pytest.mark.parametrize("P,mults", [(128, [61, 62, 88, 89, 1]), (256, [94, 95, 122, 123, 2])])
def test_staging_path_boundaries(oracle_lib, P, mults):
    """Jets on either side of the per-CTA kernel's layout limits: K and V
    copied in behind the bias triangle during the MLP (up to m = 61 at
    P = 128, 94 at P = 256), staged after it (triangle up to m = 88 / 122),
    and the query-block path beyond."""
    b = synth.make_jets(N=len(mults), P=P, mults=mults, mask_mode="scrambled", seed=31)
    d = pt.Device(b)
    ref = oracle_lib.forward(b)
    pt.check_attention(pt.to_np(d.fused()), ref, b)
    pt.check_attention(pt.to_np(d.fused(balanced=True)), ref, b)
    assert ops.get_device_status() == 0


CLUSTER_MULTS = [120, 89, 88, 86, 85, 65, 64, 63, 40, 33, 17, 7, 3, 2, 1, 0, 0]


@pytest.mark.parametrize("layout", ["padded", "packed"])
@pytest.mark.parametrize("reps", [1, 5])
def test_cluster_kernel_mixed_jets(oracle_lib, layout, reps):
    """Batches of 16 to one-per-SM jets take the 4-CTA cluster kernel, the
    jets dealt over the clusters that run at once by size: 17 jets (one per
    cluster) and 85 (two or three per cluster), with empty, one-particle and
    120-particle jets, biases exchanged between the CTAs."""
    kw = dict(mask_mode="scrambled") if layout == "padded" else {}
    mults = CLUSTER_MULTS * reps
    b = synth.make_jets(N=len(mults), P=128, layout=layout, mults=mults, seed=33, **kw)
    d = pt.Device(b)
    ref = oracle_lib.forward(b)
    got = pt.to_np(d.fused())
    pt.check_attention(got, ref, b)
    assert ops.get_device_status() == 0
    assert torch.equal(d.fused(), d.fused())


_GROUP_MIX = [128, 127, 100, 99, 90, 80, 75, 70, 68, 50, 40, 30, 20, 10, 5, 1]
GROUP_MULTS = {  # 148 jets: 37 clusters of 4 (one per SM) whatever the device's cluster capacity
    "groups_of_1": [128] * 148,                  # one triangle at a time, 4 groups per cluster
    "groups_of_2": [90] * 148,                   # 2 + 2
    "groups_of_3_1": [75] * 148,                 # 3 + 1
    "mixed": (_GROUP_MIX * 10)[:148],
}


@pytest.mark.parametrize("name", list(GROUP_MULTS))
def test_cluster_kernel_jet_groups(oracle_lib, name):
    """Clusters whose four bias triangles do not fit together run their jets
    in consecutive groups that do (all four CTAs on each group, the same
    cluster barriers in every CTA)."""
    b = synth.make_jets(N=148, P=128, mults=GROUP_MULTS[name], mask_mode="scrambled", seed=34)
    d = pt.Device(b)
    got = d.fused()
    pt.check_attention(pt.to_np(got), oracle_lib.forward(b), b)
    assert ops.get_device_status() == 0
    assert torch.equal(got, d.fused())


def test_packed_wide_jets(oracle_lib):
    """Packed jets of up to 200 particles (the P = 256 kernels): triangle,
    query-block and balanced paths against the oracle."""
    b = synth.make_jets(N=4, P=200, layout="packed", mults=[200, 150, 0, 7], pt_lo=800, pt_hi=1000, prongs=3,
                        seed=10)
    d = pt.Device(b)
    ref = oracle_lib.forward(b)
    pt.check_attention(pt.to_np(d.fused()), ref, b)
    pt.check_attention(pt.to_np(d.fused(balanced=True)), ref, b)
    pt.check_features(pt.to_np(d.features()), oracle_lib.features(b), b)
    assert ops.get_device_status() == 0


def test_packed_with_empty_jets(oracle_lib):
    b = synth.make_jets(N=6, P=64, layout="packed", mults=[3, 0, 64, 1, 0, 20], seed=6)
    d = pt.Device(b)
    pt.check_features(pt.to_np(d.features()), oracle_lib.features(b), b)
    ref = oracle_lib.forward(b)
    pt.check_attention(pt.to_np(d.fused()), ref, b)
    pt.check_attention(pt.to_np(d.fused(balanced=True)), ref, b)
    assert ops.get_device_status() == 0


def test_invalid_ptr_sets_status_and_skips_jet():
    b = synth.make_jets(N=3, P=32, layout="packed", mults=[10, 10, 10], seed=7)
    d = pt.Device(b)
    d.jets.ptr = torch.tensor([0, 20, 10, 30], dtype=torch.int32, device="cuda")  # jet 1 runs backwards
    f = d.features()
    bits = ops.get_device_status()
    assert bits & ops.PB_DEV_BADPTR
    assert torch.all(f[1] == 0)
    assert ops.get_device_status() == 0              # reading clears the word


def test_deterministic_and_empty_batch():
    b = batch("n128_p128")
    d = pt.Device(b)
    o1, o2 = d.fused(), d.fused()
    assert torch.equal(o1, o2)
    w1, w2 = d.fused(True), d.fused(True)          # balanced path: same bits on a reused workspace
    assert torch.equal(w1, w2)
    e = synth.make_jets(N=0, P=16, mults=np.zeros(0, int), seed=1)
    de = pt.Device(e)
    ops.pair_attention_forward(de.jets, de.mlp, None, de.q, de.k, de.v, torch.empty_like(de.q))
    assert ops.get_device_status() == 0


def test_many_jets_per_cta(oracle_lib):
    """More jets than resident CTAs: every CTA runs several jets in a row, so
    any state left over from one jet (shared-memory scratch, barrier phases,
    TMEM) would corrupt the next."""
    b = synth.make_jets(N=700, P=24, dist="uniform", mult_lo=1, mult_hi=24, mask_mode="scrambled", seed=8)
    d = pt.Device(b)
    pt.check_bias(pt.to_np(d.bias()), oracle_lib.pair_bias(b), b)
    ref = oracle_lib.forward(b)
    pt.check_attention(pt.to_np(d.fused()), ref, b)
    pt.check_attention(pt.to_np(d.fused(balanced=True)), ref, b)
    assert ops.get_device_status() == 0


@pytest.mark.parametrize("P", [2, 3, 5, 8])
def test_tiny_jets_elementwise(oracle_lib, P):
    """P = 2..8 with scrambled masks, empty and full jets: every entry point
    against the oracle element by element."""
    mults = [0, 1, P, max(1, P - 1), 2, P, 0, P // 2 + 1]
    b = synth.make_jets(N=len(mults), P=P, mults=mults, mask_mode="scrambled", seed=30 + P)
    d = pt.Device(b)
    pt.check_features(pt.to_np(d.features()), oracle_lib.features(b), b)
    pt.check_bias(pt.to_np(d.bias()), oracle_lib.pair_bias(b), b)
    pt.check_bias(pt.to_np(d.bias(torch.bfloat16)), oracle_lib.pair_bias(b), b, bf16=True)
    ref = oracle_lib.forward(b)
    pt.check_attention(pt.to_np(d.fused()), ref, b)
    pt.check_attention(pt.to_np(d.fused(balanced=True)), ref, b)
    pt.check_attention(pt.to_np(d.with_bias(d.bias(torch.bfloat16))), ref, b)
    assert ops.get_device_status() == 0


def test_hybrid_lorentzpart_interaction_embed(oracle_lib):
    """The hybrid Lorentz-equivariant ParT's pair-bias path (InteractionEmbed
    [64, 64, 64], one output per head of 8): the same MLP shape on the same
    four pair features with the hybrid model's own parameters, through the
    bias, fused, balanced and int8 entry points."""
    from part_pair_bias_b200 import configs as cf
    e = cf.HYBRID_INTERACTION_EMBED
    assert e["hidden"] == (64, 64, 64) and e["heads"] == ops.H and e["features"] == 4
    b = synth.make_jets(**cf.workload("hybrid_n128_p128", seed=0))
    assert b.params["W1"].shape == (64, 4) and b.params["W4"].shape == (8, 64)
    d = pt.Device(b)
    pt.check_bias(pt.to_np(d.bias()), oracle_lib.pair_bias(b), b)
    ref = oracle_lib.forward(b)
    pt.check_attention(pt.to_np(d.fused()), ref, b)
    pt.check_attention(pt.to_np(d.fused(balanced=True)), ref, b)
    pt.check_attention(pt.to_np(d.fused_i8()), oracle_lib.forward_i8(b), b)
    assert ops.get_device_status() == 0


@pytest.mark.parametrize("N", [20, 300])
def test_balanced_full_jets(oracle_lib, N):
    """Full P = 128 jets on the balanced path: a jet's records and K/V do not
    fit the stage together, so its attention reads the bias from the
    records, the heads of one jet split over CTAs (N = 20) or whole jets per
    CTA (N = 300)."""
    b = synth.make_jets(N=N, P=128, dist="full", seed=41)
    d = pt.Device(b)
    got = pt.to_np(d.fused(balanced=True))
    assert ops.get_device_status() == 0
    lo, hi = (0, N) if N <= 20 else (N - 12, N)
    s = synth.slice_jets(b, lo, hi)
    pt.check_attention(got[lo:hi], oracle_lib.forward(s), s)
