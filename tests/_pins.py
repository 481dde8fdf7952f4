"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Every function takes an ``oracle.OracleLib`` and raises ``AssertionError`` when the oracle
disagrees.  ``test_oracle_pins.py`` runs them on the real oracle; ``test_oracle_mutants.py``
runs them on deliberately broken copies of the oracle, each of which must fail at least one.

Sources: StripedHyena 2 page "04. Hardware-aware convolution kernels": Sec. 1 (causal FIR sum
and its lower-triangular Toeplitz form), Sec. 2 (block convolution), Sec. 3 (two-stage form,
worked example with l = 6, l_h = 4, l_b = 3), Sec. 5 (F.conv1d as the naive baseline),
Sec. 7 (Toeplitz tile materialised from the row/column index difference).
"""
import os

import numpy as np
import scipy.linalg
import scipy.signal
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_worked_example():
    """Parse tests/golden/worked_example_two_stage.txt -> (l, l_h, l_b, {name: index table})."""
    meta, mats, cur = {}, {}, None
    with open(os.path.join(GOLDEN, "worked_example_two_stage.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if len(parts) == 2 and parts[0] in ("l", "l_h", "l_b"):
                meta[parts[0]] = int(parts[1])
            elif len(parts) == 1:
                cur = parts[0]
                mats[cur] = []
            else:
                mats[cur].append([None if p == "-" else int(p) for p in parts])
    return meta["l"], meta["l_h"], meta["l_b"], mats


def symbolic_to_numeric(table, h):
    return np.array([[0.0 if e is None else h[e] for e in row] for row in table])


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _close(a, b, rtol=1e-12, atol=1e-12):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.abs(a - b).max() if a.size else 0.0
    assert np.allclose(a, b, rtol=rtol, atol=atol), "max abs diff %.3e" % err


# ---------------------------------------------------------------- worked example (Sec. 3)

def pin_worked_example_symbolic(o):
    """The oracle's H0, H1 for (l_h=4, l_b=3) hold exactly the printed taps."""
    _, l_h, l_b, mats = load_worked_example()
    h = np.array([2.0, 3.0, 5.0, 7.0])  # distinct primes: every tap is identifiable
    assert h.size == l_h
    H = o.toeplitz_blocks(h, l_b, 2)
    assert np.array_equal(H[0], symbolic_to_numeric(mats["H0"], h))
    assert np.array_equal(H[1], symbolic_to_numeric(mats["H1"], h))


def pin_worked_example_two_stage(o):
    """Integer-exact: printed-matrix two-stage product == block_conv == direct sum."""
    l, l_h, l_b, mats = load_worked_example()
    h = np.array([1.0, -2.0, 3.0, 4.0])
    x = np.array([3.0, 1.0, -4.0, 1.0, 5.0, -9.0])
    assert x.size == l and h.size == l_h
    H0 = symbolic_to_numeric(mats["H0"], h)
    H1 = symbolic_to_numeric(mats["H1"], h)
    X = x.reshape(-1, l_b)
    printed = np.concatenate([H0 @ X[0], H0 @ X[1] + H1 @ X[0]])
    ones = np.ones((l, 1))
    direct = o.gated_fir(ones, ones, x[:, None], h[None, :], 1)[:, 0]
    blocks = o.block_conv(h, x, l_b, 2)
    assert np.array_equal(printed, direct), (printed, direct)
    assert np.array_equal(blocks, direct), (blocks, direct)


# ---------------------------------------------------------------- Sec. 1: definition forms

def pin_dense_toeplitz(o):
    """y = q * (T (k v)) with T the dense lower-triangular Toeplitz matrix (scipy builds T)."""
    rng = np.random.default_rng(11)
    B, L, D, d_g, l_h = 2, 37, 6, 3, 5
    q, k, v = _rand(rng, B, L, D), _rand(rng, B, L, D), _rand(rng, B, L, D)
    h = _rand(rng, D // d_g, l_h)
    y = o.gated_fir(q, k, v, h, d_g)
    ref = np.empty_like(q)
    for g in range(D // d_g):
        col = np.zeros(L)
        col[:l_h] = h[g]
        T = scipy.linalg.toeplitz(col, np.zeros(L))
        for c in range(g * d_g, (g + 1) * d_g):
            for b in range(B):
                ref[b, :, c] = q[b, :, c] * (T @ (k[b, :, c] * v[b, :, c]))
    _close(y, ref)


def pin_numpy_convolve(o):
    rng = np.random.default_rng(12)
    B, L, D, d_g, l_h = 1, 50, 8, 4, 9
    q, k, v = _rand(rng, B, L, D), _rand(rng, B, L, D), _rand(rng, B, L, D)
    h = _rand(rng, D // d_g, l_h)
    y = o.gated_fir(q, k, v, h, d_g)
    for c in range(D):
        ref = q[0, :, c] * np.convolve(k[0, :, c] * v[0, :, c], h[c // d_g])[:L]
        _close(y[0, :, c], ref)


def pin_lfilter(o):
    """An FIR filter is lfilter(b=h, a=[1]) with zero initial state."""
    rng = np.random.default_rng(13)
    B, L, D, d_g, l_h = 2, 64, 4, 2, 17
    q, k, v = _rand(rng, B, L, D), _rand(rng, B, L, D), _rand(rng, B, L, D)
    h = _rand(rng, D // d_g, l_h)
    y = o.gated_fir(q, k, v, h, d_g)
    for b in range(B):
        for c in range(D):
            ref = q[b, :, c] * scipy.signal.lfilter(h[c // d_g], [1.0], k[b, :, c] * v[b, :, c])
            _close(y[b, :, c], ref)


def pin_torch_conv1d(o):
    """The pages' naive baseline: depthwise conv1d, flipped weight, left padding l_h - 1."""
    rng = np.random.default_rng(14)
    B, L, D, d_g, l_h = 2, 40, 8, 4, 6
    q, k, v = _rand(rng, B, L, D), _rand(rng, B, L, D), _rand(rng, B, L, D)
    h = _rand(rng, D // d_g, l_h)
    y = o.gated_fir(q, k, v, h, d_g)
    x = torch.from_numpy(k * v).permute(0, 2, 1)                       # [B, D, L]
    w = torch.from_numpy(np.repeat(h, d_g, axis=0)[:, ::-1].copy())[:, None, :]  # [D,1,l_h]
    conv = torch.nn.functional.conv1d(torch.nn.functional.pad(x, (l_h - 1, 0)), w, groups=D)
    ref = q * conv.permute(0, 2, 1).numpy()
    _close(y, ref)


# ---------------------------------------------------------------- invariants

def pin_rows_match_the_full_sum(o):
    """Selected rows of the direct sum equal the same rows of the full direct sum (incl. the
    first row, a row inside the filter's reach of t = 0 and the last), and numpy.convolve for
    one channel."""
    rng = np.random.default_rng(41)
    B, L, D, d_g, l_h = 2, 57, 6, 3, 20
    q, k, v = (rng.standard_normal((B, L, D)) for _ in range(3))
    h = rng.standard_normal((D // d_g, l_h))
    full = o.gated_fir(q, k, v, h, d_g)
    rows = [(0, 0), (0, 5), (1, 19), (1, 20), (0, 56), (1, 56)]
    got = o.gated_fir_rows(q, k, v, h, d_g, rows)
    for i, (b, t) in enumerate(rows):
        assert np.array_equal(got[i], full[b, t]), (b, t)
    x = k[1, :, 4] * v[1, :, 4]
    ref = np.convolve(x, h[4 // d_g])[:L]
    assert np.allclose(got[3, 4], q[1, 20, 4] * ref[20], rtol=1e-12, atol=1e-12)


def pin_impulse(o):
    """x = delta_0, q = 1: the output is the filter itself, then zeros."""
    L, l_h = 20, 7
    h = np.array([[0.5, -1.25, 2.0, 3.5, -0.75, 1.5, 4.0]])
    x = np.zeros((L, 1))
    x[0] = 1.0
    ones = np.ones((L, 1))
    y = o.gated_fir(ones, ones, x, h, 1)[:, 0]
    ref = np.zeros(L)
    ref[:l_h] = h[0]
    assert np.array_equal(y, ref), y


def pin_shift(o):
    """h = e_m delays the gated input by m samples."""
    rng = np.random.default_rng(15)
    L, l_h = 30, 8
    for m in range(l_h):
        h = np.zeros((1, l_h))
        h[0, m] = 1.0
        q, k, v = _rand(rng, L, 1), _rand(rng, L, 1), _rand(rng, L, 1)
        y = o.gated_fir(q, k, v, h, 1)[:, 0]
        x = k[:, 0] * v[:, 0]
        ref = q[:, 0] * np.concatenate([np.zeros(m), x[:L - m]])
        assert np.array_equal(y, ref), m


def pin_linearity(o):
    rng = np.random.default_rng(16)
    B, L, D, d_g, l_h = 1, 33, 4, 2, 5
    q, k = _rand(rng, B, L, D), _rand(rng, B, L, D)
    v1, v2 = _rand(rng, B, L, D), _rand(rng, B, L, D)
    h = _rand(rng, D // d_g, l_h)
    lhs = o.gated_fir(q, k, v1 + 2.0 * v2, h, d_g)
    rhs = o.gated_fir(q, k, v1, h, d_g) + 2.0 * o.gated_fir(q, k, v2, h, d_g)
    _close(lhs, rhs, rtol=1e-10, atol=1e-10)


def pin_causality(o):
    """Changing the input at t0 changes the output only for t0 <= t < t0 + l_h."""
    rng = np.random.default_rng(17)
    L, l_h, t0 = 40, 6, 13
    q, k, v = _rand(rng, L, 1), _rand(rng, L, 1), _rand(rng, L, 1)
    h = _rand(rng, 1, l_h) + 3.0  # no zero taps
    y0 = o.gated_fir(q, k, v, h, 1)[:, 0]
    v2 = v.copy()
    v2[t0] += 1.0
    y1 = o.gated_fir(q, k, v2, h, 1)[:, 0]
    changed = np.nonzero(y0 != y1)[0]
    assert changed.size > 0
    assert changed.min() == t0 and changed.max() == t0 + l_h - 1, changed


def pin_single_tap(o):
    """l_h = 1: y = q * h0 * k * v, elementwise."""
    rng = np.random.default_rng(18)
    B, L, D, d_g = 2, 9, 6, 3
    q, k, v = _rand(rng, B, L, D), _rand(rng, B, L, D), _rand(rng, B, L, D)
    h = _rand(rng, D // d_g, 1)
    y = o.gated_fir(q, k, v, h, d_g)
    ref = q * np.repeat(h[:, 0], d_g)[None, None, :] * (k * v)
    _close(y, ref, rtol=1e-15, atol=0)


def pin_geometric(o):
    """h_j = r^j on a constant input: y_t = (1 - r^(min(t, l_h-1)+1)) / (1 - r)."""
    r, l_h, L = 0.5, 10, 25
    h = r ** np.arange(l_h)[None, :]
    ones = np.ones((L, 1))
    y = o.gated_fir(ones, ones, ones, h, 1)[:, 0]
    n = np.minimum(np.arange(L), l_h - 1) + 1
    _close(y, (1 - r ** n) / (1 - r), rtol=1e-15, atol=1e-15)


def pin_grouping(o):
    """Channel c uses filter c // d_g: group g's filter is a delay by g + 1."""
    rng = np.random.default_rng(19)
    L, G, d_g, l_h = 16, 3, 4, 5
    D = G * d_g
    h = np.zeros((G, l_h))
    for g in range(G):
        h[g, g + 1] = 1.0
    q, k, v = np.ones((L, D)), np.ones((L, D)), _rand(rng, L, D)
    y = o.gated_fir(q, k, v, h, d_g)
    for c in range(D):
        m = c // d_g + 1
        assert np.array_equal(y[:, c], np.concatenate([np.zeros(m), v[:L - m, c]])), c


def pin_batch_independence(o):
    """Every sequence starts from zero history: y[b] == oracle on sequence b alone."""
    rng = np.random.default_rng(20)
    B, L, D, d_g, l_h = 3, 21, 4, 2, 6
    q, k, v = _rand(rng, B, L, D), _rand(rng, B, L, D), _rand(rng, B, L, D)
    h = _rand(rng, D // d_g, l_h)
    y = o.gated_fir(q, k, v, h, d_g)
    for b in range(B):
        assert np.array_equal(y[b], o.gated_fir(q[b], k[b], v[b], h, d_g)), b


# ---------------------------------------------------------------- Sec. 2/3 block forms

def pin_stages_needed(o):
    """stages_needed(l_h, l_b) == number of sub-block diagonals with a non-zero entry."""
    import oracle
    for l_b in (1, 2, 3, 5, 16):
        for l_h in range(1, 3 * l_b + 4):
            H = o.toeplitz_blocks(np.ones(l_h), l_b, l_h + 2)
            nz = [m for m in range(H.shape[0]) if np.any(H[m])]
            assert nz == list(range(len(nz))), (l_h, l_b, nz)
            assert len(nz) == oracle.stages_needed(l_h, l_b), (l_h, l_b)


def pin_block_forms(o):
    """S-stage block form == direct for every (l_h, l_b); two-stage only when l_h <= l_b + 1."""
    import oracle
    rng = np.random.default_rng(21)
    for l_b in (2, 3, 5, 8):
        for l_h in range(1, 2 * l_b + 3):
            L = 4 * l_b + 3  # ragged tail chunk
            h = rng.integers(-5, 6, l_h).astype(np.float64)
            h[-1] = 7.0  # the last tap is non-zero
            x = rng.integers(-5, 6, L).astype(np.float64)
            ones = np.ones((L, 1))
            direct = o.gated_fir(ones, ones, x[:, None], h[None, :], 1)[:, 0]
            S = oracle.stages_needed(l_h, l_b)
            assert np.array_equal(o.block_conv(h, x, l_b, S), direct), (l_h, l_b)
            two = o.block_conv(h, x, l_b, 2)
            if l_h <= l_b + 1:
                assert np.array_equal(two, direct), (l_h, l_b)
            else:
                assert not np.array_equal(two, direct), (l_h, l_b)


def pin_two_stage_counterexample(o):
    """l_b = 2, l_h = 4 (inside the pages' stated l_h <= 2 l_b): impulse at t = 1 reaches t = 4
    through h_3, which only the third sub-block diagonal H_2 holds."""
    h = np.array([1.0, 2.0, 3.0, 4.0])
    x = np.zeros(6)
    x[1] = 1.0
    ones = np.ones((6, 1))
    direct = o.gated_fir(ones, ones, x[:, None], h[None, :], 1)[:, 0]
    assert direct[4] == h[3]
    assert o.block_conv(h, x, 2, 2)[4] == 0.0
    assert o.block_conv(h, x, 2, 3)[4] == h[3]


def pin_index_difference_tile(o):
    """Sec. 7 builds a Toeplitz tile from the index difference (row r from l_h - 1, column c),
    masked to [0, l_h), reading the filter from memory; that tile is H0 when the memory holds
    the filter reversed (the cross-correlation storage that conv1d weights use)."""
    for l_h, chunk in ((4, 3), (7, 16), (16, 16), (5, 8)):
        h = np.arange(1.0, l_h + 1.0)
        stored = h[::-1].copy()
        r = np.arange(l_h - 1, chunk + l_h - 1)[None, :]
        c = np.arange(chunk)[:, None]
        idx = r - c
        mask = (idx >= 0) & (idx < l_h)
        tile = np.where(mask, stored[np.clip(idx, 0, l_h - 1)], 0.0)
        assert np.array_equal(tile, o.toeplitz_blocks(h, chunk, 1)[0]), (l_h, chunk)


# ---------------------------------------------------------------- backward (Sec. 7)

def _bwd_case(seed, B=2, L=23, D=6, d_g=3, l_h=5):
    rng = np.random.default_rng(seed)
    q, k, v, dy = (_rand(rng, B, L, D) for _ in range(4))
    return q, k, v, _rand(rng, D // d_g, l_h), dy, d_g


def pin_bwd_directional_derivatives(o):
    """y is linear in each of q, k, v and h separately, so for sum(dy * y) the central
    difference with step 1 along any direction is the directional derivative, exactly: it
    must equal <gradient, direction> for every one of the four gradients."""
    q, k, v, h, dy, d_g = _bwd_case(31)
    dq, dk, dv, dh = o.gated_fir_bwd(q, k, v, h, dy, d_g)
    rng = np.random.default_rng(32)
    f = lambda q_, k_, v_, h_: float(np.sum(dy * o.gated_fir(q_, k_, v_, h_, d_g)))
    for name, grad in (("q", dq), ("k", dk), ("v", dv), ("h", dh)):
        args = {"q": q, "k": k, "v": v, "h": h}
        d = rng.standard_normal(args[name].shape)
        up, dn = dict(args), dict(args)
        up[name] = args[name] + d
        dn[name] = args[name] - d
        num = (f(**{a + "_": up[a] for a in up}) - f(**{a + "_": dn[a] for a in dn})) / 2
        assert abs(num - float(np.sum(grad * d))) <= 1e-9 * (1 + abs(num)), name


def pin_bwd_adjoint_toeplitz(o):
    """dk = v * T^T (q * dy) with T the dense lower-triangular Toeplitz matrix (scipy)."""
    q, k, v, h, dy, d_g = _bwd_case(33, B=1, L=19, D=4, d_g=2, l_h=6)
    dq, dk, dv, dh = o.gated_fir_bwd(q, k, v, h, dy, d_g)
    L = q.shape[1]
    for c in range(q.shape[2]):
        col = np.zeros(L)
        col[:h.shape[1]] = h[c // d_g]
        T = scipy.linalg.toeplitz(col, np.zeros(L))
        dx = T.T @ (q[0, :, c] * dy[0, :, c])
        _close(dk[0, :, c], dx * v[0, :, c])
        _close(dv[0, :, c], dx * k[0, :, c])
        z = T @ (k[0, :, c] * v[0, :, c])
        _close(dq[0, :, c], dy[0, :, c] * z)


def pin_bwd_filter_gradient_correlation(o):
    """dh[g, j] = sum over sequences and the group's channels of the cross-correlation of
    dz = q dy with x = k v at lag j (scipy.signal.correlate)."""
    q, k, v, h, dy, d_g = _bwd_case(34, B=2, L=30, D=6, d_g=3, l_h=7)
    _, _, _, dh = o.gated_fir_bwd(q, k, v, h, dy, d_g)
    B, L, D = q.shape
    ref = np.zeros_like(h)
    for b in range(B):
        for c in range(D):
            cc = scipy.signal.correlate(q[b, :, c] * dy[b, :, c], k[b, :, c] * v[b, :, c], "full")
            ref[c // d_g] += cc[L - 1:L - 1 + h.shape[1]]
    _close(dh, ref, rtol=1e-11, atol=1e-11)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
