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


def _halo_worker(rank, world, port, out, n_rows, lengths):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    from gated_causal_fir_b200 import dist as D
    import oracle
    r, _, w = D.init("gloo", timeout_s=60)
    B, Dm, d_g = 2, 8, 4
    L = sum(lengths)
    gen = torch.Generator().manual_seed(77)
    q, k, v = (torch.randn(B, L, Dm, generator=gen) for _ in range(3))
    h = torch.randn(Dm // d_g, n_rows + 1, generator=gen)
    start = sum(lengths[:r])
    stop = start + lengths[r]
    kl, vl = k[:, start:stop].contiguous(), v[:, start:stop].contiguous()
    try:
        kh, vh = D.halo_exchange(kl, vl, n_rows)
    except ValueError:
        np.save(os.path.join(out, "err%d.npy" % r), np.ones(1))
        D.finalize()
        return
    # the history is exactly the previous piece's last rows (none on rank 0)
    lo = max(0, start - n_rows) if r > 0 else start
    assert torch.equal(kh, k[:, lo:start]) and torch.equal(vh, v[:, lo:start]), r
    # this rank's rows through the oracle with that history (test-side composition of the
    # kernel's semantics: zero before the history, rows after it exact)
    Lh = kh.shape[1]
    qq = torch.cat([torch.zeros(B, Lh, Dm), q[:, start:stop]], 1)
    yy = oracle.gated_fir(qq, torch.cat([kh, kl], 1), torch.cat([vh, vl], 1), h, d_g)
    np.save(os.path.join(out, "y%d.npy" % r), yy[:, Lh:])
    D.barrier()
    D.finalize()


@pytest.mark.parametrize("world,n_rows,lengths", [
    (2, 5, (20, 17)),
    (3, 9, (12, 30, 9)),
    (4, 0, (3, 3, 3, 3)),       # l_h = 1: nothing to exchange
])
def test_sequence_sharding_halo(tmp_path, world, n_rows, lengths):
    """Sequence cut across gloo ranks: the point-to-point halo gives every rank exactly the
    previous piece's last l_h - 1 rows of k and v, and the pieces' outputs (oracle with that
    history) put together equal the whole sequence's, bit for bit."""
    port = _free_port()
    mp.start_processes(_halo_worker, args=(world, port, str(tmp_path), n_rows, lengths),
                       nprocs=world, join=True, start_method="spawn")
    import torch
    import oracle
    B, Dm, d_g = 2, 8, 4
    L = sum(lengths)
    gen = torch.Generator().manual_seed(77)
    q, k, v = (torch.randn(B, L, Dm, generator=gen) for _ in range(3))
    h = torch.randn(Dm // d_g, n_rows + 1, generator=gen)
    full = oracle.gated_fir(q, k, v, h, d_g)
    parts = np.concatenate([np.load(tmp_path / ("y%d.npy" % r)) for r in range(world)], axis=1)
    assert np.array_equal(parts, full)


def test_sequence_sharding_short_piece_raises_everywhere(tmp_path):
    """A piece shorter than the history the next rank needs is refused on every rank before
    any data moves (no rank is left waiting in the exchange)."""
    world, port = 3, _free_port()
    mp.start_processes(_halo_worker, args=(world, port, str(tmp_path), 6, (10, 4, 10)),
                       nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        assert (tmp_path / ("err%d.npy" % r)).exists(), r
