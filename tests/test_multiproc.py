"""The N > 1 host path on CPU with two gloo ranks: sequences of a varlen batch
are split over ranks with no exchange on the data path, each rank computes
its own shard (here with the oracle, as the CUDA path needs a GPU), and the
gathered shards equal the unsharded result; the max-over-ranks timing
reduction used by bench.py is exercised too."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sliding_window_attention_sink_b200 import workloads as wl


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, result_path):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = wl.prefill_case([40, 0, 65, 7, 90, 1], 4, 2, 16, 16, sink="normal", seed=9)
        lo, hi = wl.shard_units(len(c["seqlens"]), world, rank)
        sub = wl.slice_sequences(c, lo, hi)
        if sub["total"] > 0:
            o, lse, _ = oracle.prefill(sub["q"], sub["k"], sub["v"], sub["cu_seqlens"], 4, 2,
                                       16, 16, sink=c["sink"], nthreads=1)
        else:
            o = np.zeros((0, 4, 16))
            lse = np.zeros((4, 0))
        gathered = [None] * world
        dist.all_gather_object(gathered, (sub["token_range"], o, lse))
        # bench.py's timing: the max over ranks of each rank's elapsed time
        t = torch.tensor([float(rank + 1)])
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            torch.save({"gathered": gathered, "tmax": float(t.item())}, result_path)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_sharding_matches_unsharded(tmp_path):
    import oracle
    world = 2
    path = str(tmp_path / "res.pt")
    mp.start_processes(_worker, args=(world, _free_port(), path), nprocs=world,
                       start_method="spawn")
    res = torch.load(path, weights_only=False)
    assert res["tmax"] == float(world)
    c = wl.prefill_case([40, 0, 65, 7, 90, 1], 4, 2, 16, 16, sink="normal", seed=9)
    o, lse, _ = oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], 4, 2, 16, 16,
                               sink=c["sink"], nthreads=1)
    covered = 0
    for (a, b), so, sl in res["gathered"]:
        assert np.array_equal(o[a:b], so)
        assert np.array_equal(lse[:, a:b], sl)
        covered += b - a
    assert covered == c["total"]


@pytest.mark.parametrize("n,world", [(16, 2), (7, 4), (3, 8), (0, 2), (256, 8)])
def test_shard_units_partition(n, world):
    spans = [wl.shard_units(n, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for (a, b), (c, d) in zip(spans, spans[1:]):
        assert b == c
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1
