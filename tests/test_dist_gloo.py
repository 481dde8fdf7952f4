"""Multi-rank host logic on CPU: two gloo ranks, as bench.py runs replicas under torchrun.

Each rank takes its share of independent sequences, computes them (here with the oracle, on
the CPU), and the ranks agree on the max of their timings; the union of the shards equals the
single-process result, which is what makes the replicas' work add up to the whole job."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    from gated_causal_fir_b200 import dist as D
    import oracle
    r, lr, w = D.init("gloo", timeout_s=60)
    assert (r, lr, w) == (rank, rank, world)
    # replicas: rank r owns sequences [start, stop) of a 5-sequence job
    B, L, Dm, d_g, l_h = 5, 40, 8, 4, 6
    rng = np.random.default_rng(123)
    q, k, v = (rng.standard_normal((B, L, Dm)) for _ in range(3))
    h = rng.standard_normal((Dm // d_g, l_h))
    start, stop = D.shard(B, r, w)
    y = oracle.gated_fir(q[start:stop], k[start:stop], v[start:stop], h, d_g)
    np.save(os.path.join(out, "y%d.npy" % r), y)
    # timing reduction: every rank sees the slowest rank's time
    assert D.max_over_ranks(1.5 + r) == 1.5 + (w - 1)
    assert D.sum_over_ranks(stop - start) == B
    seeds = torch.tensor([D.rank_seed(100, r)], dtype=torch.int64)
    gathered = [torch.zeros_like(seeds) for _ in range(w)]
    torch.distributed.all_gather(gathered, seeds)
    assert len({int(s) for s in gathered}) == w, "replica seeds collide"
    D.barrier()
    D.finalize()


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    import oracle
    B, L, Dm, d_g, l_h = 5, 40, 8, 4, 6
    rng = np.random.default_rng(123)
    q, k, v = (rng.standard_normal((B, L, Dm)) for _ in range(3))
    h = rng.standard_normal((Dm // d_g, l_h))
    full = oracle.gated_fir(q, k, v, h, d_g)
    parts = np.concatenate([np.load(tmp_path / ("y%d.npy" % r)) for r in range(world)])
    assert np.array_equal(parts, full)


@pytest.mark.parametrize("n,world", [(5, 2), (8, 4), (1, 3), (0, 2), (4096, 7)])
def test_shard_covers_units(n, world):
    from gated_causal_fir_b200 import dist as D
    spans = [D.shard(n, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for (a, b), (c, d) in zip(spans, spans[1:]):
        assert b == c
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1
