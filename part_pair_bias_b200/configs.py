"""The five synthetic workloads of the pair-bias benchmark.

Each entry gives the generator arguments of ``synth.make_jets``. Sizes follow
the Particle Transformer kernel table (N=128 jets, P=128 slots, H=8, D=16)
and the training batch of the fused PairEmbed description (N=512); the
packed and three-prong entries exercise ragged jets and P=256.
"""
from __future__ import annotations

WORKLOADS = {
    # small correctness case: multiplicity uniform in [8, 32]
    "pr1_n8_p32": dict(N=8, P=32, layout="padded", dist="uniform", mult_lo=8, mult_hi=32,
                       pt_lo=500.0, pt_hi=550.0, prongs=1),
    # the headline kernel shape
    "n128_p128": dict(N=128, P=128, layout="padded", dist="poisson", lam=40.0, mult_lo=2,
                      mult_hi=128, pt_lo=500.0, pt_hi=550.0, prongs=1),
    # training batch size; also run through the bias-materialising path
    "n512_p128": dict(N=512, P=128, layout="padded", dist="poisson", lam=40.0, mult_lo=2,
                      mult_hi=128, pt_lo=500.0, pt_hi=550.0, prongs=1),
    # packed ragged jets, no padding
    "packed_8192": dict(N=8192, P=128, layout="packed", dist="poisson", lam=40.0, mult_lo=2,
                        mult_hi=128, pt_lo=500.0, pt_hi=550.0, prongs=1),
    # wide jets, three prongs, P=256
    "n256_p256_3prong": dict(N=256, P=256, layout="padded", dist="poisson", lam=100.0,
                             mult_lo=2, mult_hi=256, pt_lo=800.0, pt_hi=1000.0, prongs=3),
    # the pair-bias path of the hybrid Lorentz-equivariant ParT of the same
    # page's architecture table: its InteractionEmbed has hidden widths
    # [64, 64, 64] and one output per head of its 8-head ParticleAttention
    # blocks, i.e. the same 4 -> 64 -> 64 -> 64 -> 8 MLP on the same four
    # pair features; its own parameters (seed offset) on the kernel shape
    "hybrid_n128_p128": dict(N=128, P=128, layout="padded", dist="poisson", lam=40.0, mult_lo=2,
                             mult_hi=128, pt_lo=500.0, pt_hi=550.0, prongs=1, seed_offset=1000),
}

ORDER = ["pr1_n8_p32", "n128_p128", "n512_p128", "packed_8192", "n256_p256_3prong"]
# the hybrid model's pair MLP: hidden widths and output width (heads)
HYBRID_INTERACTION_EMBED = dict(hidden=(64, 64, 64), heads=8, features=4)


def workload(name: str, seed: int = 0, **overrides):
    """Generator keyword arguments for a named workload (with overrides)."""
    kw = dict(WORKLOADS[name])
    kw.update(overrides)
    kw["seed"] = seed + kw.pop("seed_offset", 0)
    return kw
