"""Multi-rank host logic of the benchmark on CPU: two gloo ranks, as torchrun would start
them on two GPUs.

Heads are independent and W is shared, so a data-parallel job gives every rank its own
heads (weak scaling) and the only exchange is the sum of dW over ranks.  Here each rank
computes the float64 oracle gradient of W for the heads ``bench.rank_heads`` assigns it,
the ranks add them with ``bench.allreduce_dw`` (gloo all-reduce), and the result must equal
the gradient of W over all heads computed in one process.  ``bench.max_over_ranks`` must
return the slowest rank's time on every rank.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2
HEADS_PER_RANK = 2


def _workload():
    from linear_lsh_sketch_race_b200 import inputs as I
    return I.Workload("multirank", H=WORLD * HEADS_PER_RANK, N=160, d=64, L=2, P=4, tau=0.5,
                      causal=True, dtype="fp32", backward=True, seed=13)


def _dw_of_heads(heads):
    import oracle
    from linear_lsh_sketch_race_b200 import inputs as I
    wl = _workload()
    x = I.make_inputs(wl, "cpu", heads=heads)
    f = {k: v.double().numpy() for k, v in x.items()}
    _, _, _, dW = oracle.backward_heads(f["q"], f["k"], f["v"], f["W"], wl.tau, True,
                                        f["dout"])
    return dW


def _rank_main(rank, port, out_path):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        heads = bench.rank_heads(rank, HEADS_PER_RANK)
        dW = torch.from_numpy(_dw_of_heads(heads))
        bench.allreduce_dw(dW, WORLD)
        slowest = bench.max_over_ranks(10.0 + rank, WORLD, "cpu")
        if rank == 0:
            np.save(out_path, dW.numpy())
        assert slowest == 10.0 + (WORLD - 1)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_rank_heads_partition_the_global_heads():
    sys.path.insert(0, ROOT)
    import bench
    owned = [h for r in range(WORLD) for h in bench.rank_heads(r, HEADS_PER_RANK)]
    assert sorted(owned) == list(range(WORLD * HEADS_PER_RANK))


def test_two_gloo_ranks_sum_dw_like_one_process(tmp_path):
    out = str(tmp_path / "dw.npy")
    mp.start_processes(_rank_main, args=(_free_port(), out), nprocs=WORLD, join=True,
                       start_method="spawn")
    got = np.load(out)
    ref = _dw_of_heads(list(range(WORLD * HEADS_PER_RANK)))
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()
