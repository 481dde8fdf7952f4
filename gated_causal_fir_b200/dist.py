"""Multi-rank plumbing of the forward pass (one process per GPU).

Two ways to spread the work:

* Replicas: sequences (and channel groups) are independent, so N ranks each run the full
  kernel on their own batch with no exchange.  The helpers set up the process group, derive
  each rank's seed and batch slice, and reduce the ranks' timings (max over ranks).
* Sequence sharding (context parallelism, named on the StripedHyena 2 overview page, Sec. 5,
  "a2a, p2p"): every sequence is cut along time into consecutive pieces, rank r holding the
  r-th.  Output chunk n of the block-Toeplitz form needs input chunk n - 1 (page 04, Sec. 3),
  so the only exchange is a point-to-point halo: rank r sends the last l_h - 1 rows of its k
  and v to rank r + 1 (``halo_exchange``), which passes them to ``hyena_conv_fwd_hist`` as the
  history of its rows.  No other collective touches the data.
"""
import datetime
import os

import torch
import torch.distributed as dist


def env_world():
    """(rank, local_rank, world_size) from the torchrun environment (defaults: one process)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0):
    """Join the process group if WORLD_SIZE > 1; returns (rank, local_rank, world_size)."""
    rank, local_rank, world = env_world()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        kwargs = dict(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
        if backend == "nccl":
            kwargs["device_id"] = torch.device("cuda", local_rank)
        dist.init_process_group(**kwargs)
    return rank, local_rank, world


def barrier():
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The largest of every rank's value (identity with one process)."""
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Distinct, reproducible input seed of each replica."""
    return base + 7919 * rank


def shard(n: int, rank: int, world: int):
    """[start, stop) of rank's share of n independent units (sizes differ by at most one)."""
    per, rem = divmod(n, world)
    start = rank * per + min(rank, rem)
    return start, start + per + (1 if rank < rem else 0)


def _group_rank_world(group):
    if not dist.is_initialized():
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def halo_exchange(k, v, n_rows: int, group=None):
    """The history of this rank's piece of every sequence: the last ``n_rows`` rows of the
    previous rank's k and v.

    k, v: [B, L_local, D] on this rank's device (CUDA under NCCL, CPU under gloo), rank r
    holding rows that directly follow rank r - 1's.  Rank r sends k[:, -n_rows:], v[:, -n_rows:]
    to rank r + 1 and receives rank r - 1's (point-to-point; no other data moves).  Returns
    (k_hist, v_hist), contiguous [B, n_rows, D]; rank 0 gets [B, 0, D] (zero history).
    Every rank's L_local must be at least n_rows (one all-reduce of the lengths checks it on
    all ranks before anything is sent, so a short piece raises ValueError everywhere).
    """
    rank, world = _group_rank_world(group)
    B, L, Dm = k.shape
    if v.shape != k.shape or v.dtype != k.dtype:
        raise ValueError("k and v must have the same shape and dtype")
    if world > 1:
        t = torch.tensor([L], dtype=torch.int64, device=k.device)
        dist.all_reduce(t, op=dist.ReduceOp.MIN, group=group)
        shortest = int(t.item())
    else:
        shortest = L
    if shortest < n_rows:
        raise ValueError("a rank holds %d rows, fewer than the %d history rows the next rank "
                         "needs" % (shortest, n_rows))
    empty = k.new_empty((B, 0, Dm)), v.new_empty((B, 0, Dm))
    if world == 1 or n_rows == 0:
        return empty
    peer = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
    ops, out = [], None
    if rank > 0:
        out = (k.new_empty((B, n_rows, Dm)), v.new_empty((B, n_rows, Dm)))
        ops += [dist.P2POp(dist.irecv, x, peer(rank - 1), group) for x in out]
    if rank < world - 1:
        send = (k[:, L - n_rows:].contiguous(), v[:, L - n_rows:].contiguous())
        ops += [dist.P2POp(dist.isend, x, peer(rank + 1), group) for x in send]
    for req in dist.batch_isend_irecv(ops):
        req.wait()
    return out if out is not None else empty


def sequence_sharded_forward(q, k, v, h, d_g: int, l_b: int, group=None, stream=None):
    """Forward of sequences cut along time across the ranks of ``group`` (rank r holds the r-th
    consecutive piece of every sequence: q, k, v [B, L_r, D] on its GPU).  Exchanges the l_h - 1
    history rows point-to-point, then runs ``hyena_conv_fwd_hist``; returns this rank's y
    [B, L_r, D], equal to the same rows of the forward over the whole sequences."""
    import gated_causal_fir_b200 as g
    kh, vh = halo_exchange(k, v, h.shape[1] - 1, group)
    return g.hyena_conv_fwd_hist(q, k, v, h, d_g, l_b, kh, vh, stream=stream)


def finalize():
    if dist.is_initialized():
        dist.destroy_process_group()
