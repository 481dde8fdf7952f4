"""Helpers of the GPU parity tests: tolerance checks against the fp64 oracle and sampled
windows for sizes the oracle cannot take whole.

Tolerances (written here, used by every GPU test):
  * bf16 q/k/v/y: |y - y_ref| <= 1e-2 + 1e-2 * |y_ref| elementwise.
  * fp32 q/k/v/y: max|y - y_ref| / max|y_ref| <= 1e-5 (normwise; elementwise relative error
    is ill-posed where y_ref ~ 0).
"""
import numpy as np
import torch

import oracle

BF16_ATOL = 1e-2
BF16_RTOL = 1e-2
F32_NORMWISE = 1e-5


def bf16_ratio(y, ref) -> float:
    """max over elements of |y - ref| / (atol + rtol |ref|); <= 1 passes."""
    y = y.detach().to("cpu").double().numpy() if isinstance(y, torch.Tensor) else y
    if ref.size == 0:
        return 0.0
    err = np.abs(y - ref)
    return float((err / (BF16_ATOL + BF16_RTOL * np.abs(ref))).max())


def f32_normwise(y, ref) -> float:
    y = y.detach().to("cpu").double().numpy() if isinstance(y, torch.Tensor) else y
    if ref.size == 0:
        return 0.0
    scale = max(float(np.abs(ref).max()), 1e-300)
    return float(np.abs(y - ref).max() / scale)


def assert_parity(y, ref, dtype):
    assert np.all(np.isfinite(y.detach().to("cpu").float().numpy())), "non-finite output"
    if dtype == torch.float32:
        r = f32_normwise(y, ref)
        assert r <= F32_NORMWISE, "fp32 normwise error %.3e > %.1e" % (r, F32_NORMWISE)
        return r
    r = bf16_ratio(y, ref)
    assert r <= 1.0, "bf16 error/bound ratio %.3f > 1" % r
    return r


def oracle_full(q, k, v, h, d_g):
    return oracle.gated_fir(q, k, v, h, d_g)


def oracle_window(q, k, v, h, d_g, b, t0, t1, l_h):
    """Oracle outputs for rows [t0, t1) of sequence b, from the l_h - 1 rows of history before
    t0 (zero history before the start of the sequence)."""
    s = max(0, t0 - (l_h - 1))
    sl = slice(s, t1)
    ref = oracle.gated_fir(q[b, sl], k[b, sl], v[b, sl], h, d_g)
    return ref[t0 - s:]


def sample_chunks(L, l_b, n_random, seed, extra_rows=()):
    """Chunk start rows: n_random random chunks, the first three, the tail chunk and the chunks
    holding each row in extra_rows (with the two chunks after it)."""
    nchunks = (L + l_b - 1) // l_b
    rng = np.random.default_rng(seed)
    picks = set(int(x) for x in rng.integers(0, nchunks, n_random))
    picks |= {0, 1, 2, nchunks - 1}
    for r in extra_rows:
        c = r // l_b
        picks |= {c, c + 1, c + 2}
    return sorted(c * l_b for c in picks if 0 <= c < nchunks)


def tc_cta_seam_rows(B, L, D, d_g, sm_count, tile_rows=128):
    """Time rows where a CTA of the tensor-core kernel starts its range inside a sequence
    (the kernel splits tiles ordered (group, batch, time) evenly over one CTA per SM)."""
    nT = (L + tile_rows - 1) // tile_rows
    W = (D // d_g) * B * nT
    grid = min(W, sm_count)
    per, rem = divmod(W, grid)
    rows = []
    for c in range(grid):
        w = c * per + min(c, rem)
        i = w % nT
        seq = w // nT
        if i > 0:
            rows.append((seq // B, seq % B, i * tile_rows))  # (group, b, row)
    return rows


# (log2 N, channel pairs per CTA) of the block FFT kernel's transform lengths, by I/O type
FFTBLK_CONFIGS = {"bf16": ((10, 8), (11, 4), (12, 2), (13, 1)),
                  "f32": ((10, 4), (11, 2), (12, 1))}


def fftblk_plan(L, D, d_g, l_h, dtype="bf16"):
    """The block FFT's choice for a shape (tensors 16-byte aligned): (N, P, M) with the least
    N log N per block times blocks per sequence, weighted per transform length as the library
    weights it (1 up to N = 2048, 2.2 at 4096, 2.6 at 8192), or None where no length applies."""
    best = None
    for lgn, P in FFTBLK_CONFIGS[dtype]:
        N = 1 << lgn
        if N < l_h or d_g % (2 * P) or D % (2 * P):
            continue
        M = N - l_h + 1
        ntb = -(-L // M)
        if M < N // 8 and ntb > 1:
            continue
        cost = ntb * N * lgn * (1.0 if lgn <= 11 else (2.2 if lgn == 12 else 2.6))
        if best is None or cost < best[0]:
            best = (cost, N, P, M)
    return None if best is None else best[1:]
