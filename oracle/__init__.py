"""fp64 CPU oracle for the gated, grouped, depthwise causal FIR (Hyena-SE / Hyena-MR).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.  It
shares no code with the CUDA path and does not import it.

The arithmetic lives in ``fir_oracle.c`` (plain C, fp64, OpenMP over rows); this module only
marshals numpy arrays.  What each function computes, with its source on the StripedHyena 2
page "04. Hardware-aware convolution kernels":

* :func:`gated_fir` -- the direct sum of Sec. 1, gated: y = q * sum_j h_g[j] (k v)[t-j].
* :func:`gated_fir_rows` -- the same direct sum for selected output rows only.
* :func:`toeplitz_blocks` -- the l_b x l_b sub-blocks H_m[i][j] = h[m l_b + i - j] of the
  lower-triangular Toeplitz matrix (Sec. 2; index rule fixed by the Sec. 3 worked example).
* :func:`block_conv` -- the S-stage block form Yhat_n = sum_{m<S} H_m Xhat_{n-m} (Sec. 2/3;
  S = 2 is the two-stage algorithm).
* :func:`stages_needed` -- the number S of non-zero sub-block diagonals, 1 + ceil((l_h-1)/l_b).
"""
import ctypes

import numpy as np

from . import build as _build

_dp = ctypes.POINTER(ctypes.c_double)


def _f64(a):
    """Exact upcast to a C-contiguous float64 array (bf16/fp16/fp32 -> fp64 is exact)."""
    if hasattr(a, "detach"):  # torch tensor: upcast on its own side, then hand over
        a = a.detach().to("cpu").double().contiguous().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return a.ctypes.data_as(_dp)


class OracleLib:
    """The oracle's C entry points loaded from one shared library (``path``)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        i64 = ctypes.c_int64
        lib.oracle_gated_fir_f64.argtypes = [_dp, _dp, _dp, _dp, _dp, i64, i64, i64, i64, i64,
                                             ctypes.c_int]
        lib.oracle_gated_fir_f64.restype = ctypes.c_int
        lib.oracle_gated_fir_rows_f64.argtypes = [_dp, _dp, _dp, _dp,
                                                  ctypes.POINTER(ctypes.c_int64), i64, _dp, i64,
                                                  i64, i64, i64, i64, ctypes.c_int]
        lib.oracle_gated_fir_rows_f64.restype = ctypes.c_int
        lib.oracle_toeplitz_blocks_f64.argtypes = [_dp, i64, i64, i64, _dp]
        lib.oracle_toeplitz_blocks_f64.restype = ctypes.c_int
        lib.oracle_block_conv_f64.argtypes = [_dp, i64, i64, i64, _dp, i64, _dp]
        lib.oracle_block_conv_f64.restype = ctypes.c_int
        lib.oracle_gated_fir_bwd_f64.argtypes = [_dp] * 9 + [i64, i64, i64, i64, i64, ctypes.c_int]
        lib.oracle_gated_fir_bwd_f64.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def max_threads(self) -> int:
        """Threads the oracle's OpenMP loops use on this host."""
        return int(self.lib.oracle_max_threads())

    def gated_fir(self, q, k, v, h, d_g: int, nthreads: int = 0) -> np.ndarray:
        """Direct fp64 gated grouped causal FIR.

        q, k, v: [B, L, D] or [L, D] (numpy or torch, any float dtype; upcast exactly).
        h: [D // d_g, l_h], natural tap order (h[g, 0] multiplies the current token).
        Returns y (float64, same shape as q): y[b,t,c] = q[b,t,c] * sum_{j<=min(l_h-1,t)}
        h[c//d_g, j] * k[b,t-j,c] * v[b,t-j,c], zero history before t = 0 in every sequence.
        """
        q, k, v, h = _f64(q), _f64(k), _f64(v), _f64(h)
        squeeze = q.ndim == 2
        if squeeze:
            q, k, v = q[None], k[None], v[None]
        B, L, D = q.shape
        assert k.shape == q.shape and v.shape == q.shape, "q, k, v shapes differ"
        assert h.ndim == 2 and h.shape[0] * d_g == D, "h must be [D // d_g, l_h]"
        l_h = h.shape[1]
        y = np.empty_like(q)
        rc = self.lib.oracle_gated_fir_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(h), _ptr(y),
                                           B, L, D, d_g, l_h, nthreads)
        if rc != 0:
            raise ValueError("oracle_gated_fir_f64 rejected its arguments (rc=%d)" % rc)
        return y[0] if squeeze else y

    def gated_fir_rows(self, q, k, v, h, d_g: int, rows, nthreads: int = 0) -> np.ndarray:
        """y[b, t, :] of :meth:`gated_fir` for each (b, t) in ``rows`` only: [len(rows), D]."""
        q, k, v, h = _f64(q), _f64(k), _f64(v), _f64(h)
        if q.ndim == 2:
            q, k, v = q[None], k[None], v[None]
        B, L, D = q.shape
        assert k.shape == q.shape and v.shape == q.shape, "q, k, v shapes differ"
        assert h.ndim == 2 and h.shape[0] * d_g == D, "h must be [D // d_g, l_h]"
        flat = np.ascontiguousarray([b * L + t for b, t in rows], dtype=np.int64)
        out = np.empty((len(flat), D), dtype=np.float64)
        rc = self.lib.oracle_gated_fir_rows_f64(
            _ptr(q), _ptr(k), _ptr(v), _ptr(h),
            flat.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), len(flat), _ptr(out), B, L, D,
            d_g, h.shape[1], nthreads)
        if rc != 0:
            raise ValueError("oracle_gated_fir_rows_f64 rejected its arguments (rc=%d)" % rc)
        return out

    def gated_fir_bwd(self, q, k, v, h, dy, d_g: int, nthreads: int = 0):
        """Gradients (dq, dk, dv, dh) of sum(dy * y) for y = gated_fir(q, k, v, h, d_g)."""
        q, k, v, h, dy = _f64(q), _f64(k), _f64(v), _f64(h), _f64(dy)
        squeeze = q.ndim == 2
        if squeeze:
            q, k, v, dy = q[None], k[None], v[None], dy[None]
        B, L, D = q.shape
        assert k.shape == q.shape and v.shape == q.shape and dy.shape == q.shape
        assert h.ndim == 2 and h.shape[0] * d_g == D, "h must be [D // d_g, l_h]"
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        dh = np.empty_like(h)
        rc = self.lib.oracle_gated_fir_bwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(h), _ptr(dy),
                                               _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dh), B, L, D,
                                               d_g, h.shape[1], nthreads)
        if rc != 0:
            raise ValueError("oracle_gated_fir_bwd_f64 rejected its arguments (rc=%d)" % rc)
        if squeeze:
            dq, dk, dv = dq[0], dk[0], dv[0]
        return dq, dk, dv, dh

    def toeplitz_blocks(self, h, l_b: int, S: int) -> np.ndarray:
        """[S, l_b, l_b]: H[m][i][j] = h[m*l_b + i - j] inside [0, l_h), else 0."""
        h = _f64(h).reshape(-1)
        H = np.empty((S, l_b, l_b), dtype=np.float64)
        rc = self.lib.oracle_toeplitz_blocks_f64(_ptr(h), h.size, l_b, S, _ptr(H))
        if rc != 0:
            raise ValueError("oracle_toeplitz_blocks_f64 rejected its arguments (rc=%d)" % rc)
        return H

    def block_conv(self, h, x, l_b: int, S: int) -> np.ndarray:
        """One channel through the S-stage block form Yhat_n = sum_{m<S} H_m Xhat_{n-m}."""
        h = _f64(h).reshape(-1)
        x = _f64(x).reshape(-1)
        y = np.empty_like(x)
        rc = self.lib.oracle_block_conv_f64(_ptr(h), h.size, l_b, S, _ptr(x), x.size, _ptr(y))
        if rc != 0:
            raise ValueError("oracle_block_conv_f64 rejected its arguments (rc=%d)" % rc)
        return y


_DEFAULT = None


def default() -> OracleLib:
    """The oracle built from ``fir_oracle.c`` (compiled on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = OracleLib(_build.build())
    return _DEFAULT


def max_threads() -> int:
    return default().max_threads()


def gated_fir(q, k, v, h, d_g: int, nthreads: int = 0) -> np.ndarray:
    return default().gated_fir(q, k, v, h, d_g, nthreads)


def gated_fir_rows(q, k, v, h, d_g: int, rows, nthreads: int = 0) -> np.ndarray:
    return default().gated_fir_rows(q, k, v, h, d_g, rows, nthreads)


def toeplitz_blocks(h, l_b: int, S: int) -> np.ndarray:
    return default().toeplitz_blocks(h, l_b, S)


def gated_fir_bwd(q, k, v, h, dy, d_g: int, nthreads: int = 0):
    return default().gated_fir_bwd(q, k, v, h, dy, d_g, nthreads)


def block_conv(h, x, l_b: int, S: int) -> np.ndarray:
    return default().block_conv(h, x, l_b, S)


def stages_needed(l_h: int, l_b: int) -> int:
    """Non-zero sub-block diagonals of the Toeplitz matrix: 1 + ceil((l_h - 1) / l_b)."""
    return 1 + (l_h - 1 + l_b - 1) // l_b
