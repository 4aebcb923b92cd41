"""The multi-rank path on CPU: two gloo ranks, the sharding and reduction
helpers that bench.py uses with NCCL on GPUs.

Jets are independent, so a batch split over ranks by cost and run rank by
rank must reproduce the unsplit run exactly; under weak scaling every rank
draws its own batch; the timed region is reduced by a max over ranks; a rank
that leaves early surfaces as an error on the others, not as a hang.
"""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

from part_pair_bias_b200 import configs, shard, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s=60):
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _sharded_forward(rank, world, port, out_dir):
    import oracle
    _init(rank, world, port)
    b = synth.make_jets(**configs.workload("pr1_n8_p32", seed=0))
    lo, hi = shard.balanced_ranges(b.mult, world)[rank]
    mine = oracle.forward(synth.slice_jets(b, lo, hi)) if hi > lo else np.zeros((0, 8, b.P, 16))
    # ranks exchange their outputs only to check them here; the path itself has no collective
    got = [None] * world
    dist.all_gather_object(got, mine)
    # weak scaling: each rank's own batch
    wb = synth.make_jets(**configs.workload("pr1_n8_p32", seed=shard.rank_seed(0, rank)))
    sums = [None] * world
    dist.all_gather_object(sums, float(wb.E.sum()))
    mx = shard.reduce_max([rank + 1.0, 10.0 - rank, float(rank == 1) * 4.0])
    if rank == 0:
        np.save(os.path.join(out_dir, "sharded.npy"), np.concatenate(got))
        np.save(os.path.join(out_dir, "meta.npy"), np.array([sums[0], sums[1]] + mx))
    dist.barrier()
    dist.destroy_process_group()


def _leaver(rank, world, port, out_dir):
    _init(rank, world, port, timeout_s=10)
    if rank == 1:
        os._exit(0)                      # leaves between steps, no collective in flight
    err = ""
    try:
        dist.barrier()
    except Exception as e:               # the peer's exit ends the barrier with an error
        err = type(e).__name__ or "error"
    with open(os.path.join(out_dir, "rank0.txt"), "w") as f:
        f.write(err)


def test_balanced_ranges_partition_and_balance():
    rng = np.random.default_rng(3)
    for world in (1, 2, 3, 8):
        m = rng.integers(0, 129, size=257)
        rs = shard.balanced_ranges(m, world)
        assert rs[0][0] == 0 and rs[-1][1] == len(m)
        assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
        cost = [int((m[lo:hi].astype(np.int64) ** 2).sum()) for lo, hi in rs]
        share = (m.astype(np.int64) ** 2).sum() / world
        assert max(cost) <= share + (m.astype(np.int64) ** 2).max()
    assert shard.balanced_ranges([5, 5], 4)[-1][1] == 2          # more ranks than jets
    assert shard.job_rate(128, 4, 0.5) == 1024.0


def test_two_gloo_ranks_reproduce_the_unsplit_batch(oracle_lib, tmp_path):
    port = _free_port()
    mp.start_processes(_sharded_forward, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    b = synth.make_jets(**configs.workload("pr1_n8_p32", seed=0))
    ref = oracle_lib.forward(b)
    got = np.load(tmp_path / "sharded.npy")
    assert np.array_equal(got, ref)                                 # jets are independent: bitwise
    meta = np.load(tmp_path / "meta.npy")
    assert meta[0] != meta[1]                                       # distinct weak-scaling batches
    assert list(meta[2:]) == [2.0, 10.0, 4.0]                       # element-wise max over ranks


def test_a_rank_that_leaves_is_an_error_not_a_hang(tmp_path):
    port = _free_port()
    ctx = mp.start_processes(_leaver, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=False)
    for p in ctx.processes:
        p.join(timeout=120)
    alive = [p for p in ctx.processes if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank hung"
    assert (tmp_path / "rank0.txt").read_text() != ""
