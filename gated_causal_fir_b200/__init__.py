"""B200-native gated, grouped, depthwise causal FIR: the Hyena-SE / Hyena-MR forward.

    y[b,t,c] = q[b,t,c] * sum_{j<l_h, j<=t} h[c // d_g, j] * k[b,t-j,c] * v[b,t-j,c]

computed by the sm_100a kernels of ``libhyena_conv.so`` through its C ABI
(``include/hyena_conv.h``).  The functions here carry the C names and only marshal torch CUDA
tensors into pointers, sizes and the current stream; PyTorch provides device memory and
streams, nothing else.  There is no CPU path: without a CUDA device or the built library every
call raises.

Importing the package does not load the library; the first call does.
"""
import ctypes

from . import _native
from ._native import (HYENA_ALGO_AUTO, HYENA_ALGO_DIRECT, HYENA_ALGO_FFT, HYENA_ALGO_TENSOR,
                      HYENA_ALGO_WINDOW, HYENA_DEVICE_F16_RANGE, HYENA_DEVICE_TIMEOUT,
                      HYENA_DTYPE_BF16, HYENA_DTYPE_F32, ALGO_NAMES, HyenaError)

__all__ = [
    "hyena_conv_fwd", "hyena_conv_fwd_f32", "hyena_conv_fwd_ex", "hyena_select_algo",
    "hyena_build_toeplitz", "hyena_conv_bwd", "hyena_conv_bwd_ex", "hyena_select_bwd_algo",
    "hyena_conv_bwd_workspace_bytes",
    "hyena_device_status", "hyena_status_string", "hyena_abi_version",
    "HyenaError", "HYENA_ALGO_AUTO", "HYENA_ALGO_TENSOR", "HYENA_ALGO_WINDOW",
    "HYENA_ALGO_DIRECT", "HYENA_ALGO_FFT", "HYENA_DTYPE_BF16", "HYENA_DTYPE_F32",
    "HYENA_DEVICE_TIMEOUT",
    "HYENA_DEVICE_F16_RANGE", "ALGO_NAMES", "hyena_conv_fwd_from_host",
    "hyena_toeplitz_stages", "hyena_build_toeplitz_blocks", "hyena_conv_fwd_hist",
    "hyena_conv_fwd_fft", "hyena_conv_fwd_fft_workspace_bytes",
    "hyena_conv_fwd_from_host_workspace_bytes",
]


def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return HYENA_DTYPE_BF16
    if t.dtype == torch.float32:
        return HYENA_DTYPE_F32
    raise TypeError("q, k, v must be bfloat16 or float32, got %s" % t.dtype)


def _check(q, k, v, h, d_g, y):
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v), ("h", h)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError("%s must be a CUDA tensor" % name)
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous" % name)
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, L, D] shape")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    if h.dtype != torch.float32 or h.dim() != 2:
        raise TypeError("h must be float32 [D // d_g, l_h]")
    B, L, D = q.shape
    if d_g < 1 or D % d_g != 0 or h.shape[0] * d_g != D:
        raise ValueError("h has %d rows; D=%d with d_g=%d needs D // d_g" % (h.shape[0], D, d_g))
    if y is None:
        y = torch.empty_like(q)
    elif (not isinstance(y, torch.Tensor) or y.shape != q.shape or y.dtype != q.dtype
          or not y.is_cuda or not y.is_contiguous()):
        raise ValueError("y must be a contiguous CUDA tensor like q")
    return y


def hyena_conv_fwd_ex(q, k, v, h, d_g, l_b, algo=HYENA_ALGO_AUTO, y=None, stream=None):
    """Forward with the algorithm chosen by the caller (HYENA_ALGO_*); returns y.

    q, k, v: CUDA [B, L, D], all bf16 or all fp32.  h: CUDA fp32 [D // d_g, l_h].
    l_b: block size of the decomposition (any l_h >= 1 is accepted; the result does not depend
    on l_b).  y: optional preallocated output.  Runs asynchronously on ``stream`` (default: the
    current torch stream).
    """
    y = _check(q, k, v, h, d_g, y)
    B, L, D = q.shape
    rc = _native.lib().hyena_conv_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), h.data_ptr(),
                                         y.data_ptr(), B, L, D, d_g, h.shape[1], l_b,
                                         _dtype_code(q), algo, _stream(stream))
    _native.check("hyena_conv_fwd_ex", rc)
    return y


def hyena_conv_fwd_hist(q, k, v, h, d_g, l_b, k_hist, v_hist, algo=HYENA_ALGO_AUTO, y=None,
                        stream=None):
    """Forward of one shard of longer sequences: k_hist, v_hist [B, L_hist, D] are the rows that
    precede row 0 of every sequence (their last l_h - 1 rows are read); returns y [B, L, D].
    L_hist = 0 (or k_hist None) is zero history."""
    torch = _torch()
    y = _check(q, k, v, h, d_g, y)
    B, L, D = q.shape
    if k_hist is None or k_hist.shape[1] == 0:
        kp = vp = None
        L_hist = 0
    else:
        for t in (k_hist, v_hist):
            if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != q.dtype \
                    or t.dim() != 3 or not t.is_contiguous() or t.device != q.device:
                raise TypeError("k_hist, v_hist must be contiguous CUDA [B, L_hist, D] tensors of "
                                "q's dtype on q's device")
        if k_hist.shape != v_hist.shape or k_hist.shape[0] != B or k_hist.shape[2] != D:
            raise ValueError("k_hist, v_hist must both be [B, L_hist, D] with q's B and D")
        kp, vp = k_hist.data_ptr(), v_hist.data_ptr()
        L_hist = k_hist.shape[1]
    rc = _native.lib().hyena_conv_fwd_hist(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           h.data_ptr(), y.data_ptr(), kp, vp, L_hist, B, L, D,
                                           d_g, h.shape[1], l_b, _dtype_code(q), algo,
                                           _stream(stream))
    _native.check("hyena_conv_fwd_hist", rc)
    return y


def hyena_conv_fwd_fft_workspace_bytes(B, L, D, d_g, l_h):
    """Bytes of workspace hyena_conv_fwd_fft needs (raises where the FFT path does not apply)."""
    n = int(_native.lib().hyena_conv_fwd_fft_workspace_bytes(B, L, D, d_g, l_h))
    if n < 0:
        _native.check("hyena_conv_fwd_fft_workspace_bytes", -n)
    return n


def hyena_conv_fwd_fft(q, k, v, h, d_g, l_b, workspace=None, y=None, stream=None):
    """Forward by FFT convolution (long filters): same operation and arguments as
    hyena_conv_fwd_ex; ``workspace`` is a CUDA uint8 tensor of at least
    hyena_conv_fwd_fft_workspace_bytes() bytes (allocated here when None)."""
    torch = _torch()
    y = _check(q, k, v, h, d_g, y)
    B, L, D = q.shape
    need = hyena_conv_fwd_fft_workspace_bytes(B, L, D, d_g, h.shape[1])
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    rc = _native.lib().hyena_conv_fwd_fft(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          h.data_ptr(), y.data_ptr(), B, L, D, d_g, h.shape[1],
                                          l_b, _dtype_code(q), workspace.data_ptr(),
                                          workspace.numel() * workspace.element_size(),
                                          _stream(stream))
    _native.check("hyena_conv_fwd_fft", rc)
    return y


def hyena_conv_fwd(q, k, v, h, d_g, l_b, y=None, stream=None):
    """bf16 forward, fastest supported algorithm (C: hyena_conv_fwd); returns y."""
    y = _check(q, k, v, h, d_g, y)
    if _dtype_code(q) != HYENA_DTYPE_BF16:
        raise TypeError("hyena_conv_fwd takes bf16 q, k, v; use hyena_conv_fwd_f32 for fp32")
    B, L, D = q.shape
    rc = _native.lib().hyena_conv_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), h.data_ptr(),
                                      y.data_ptr(), B, L, D, d_g, h.shape[1], l_b,
                                      _stream(stream))
    _native.check("hyena_conv_fwd", rc)
    return y


def hyena_conv_fwd_f32(q, k, v, h, d_g, l_b, y=None, stream=None):
    """fp32 forward (C: hyena_conv_fwd_f32); returns y."""
    y = _check(q, k, v, h, d_g, y)
    if _dtype_code(q) != HYENA_DTYPE_F32:
        raise TypeError("hyena_conv_fwd_f32 takes fp32 q, k, v")
    B, L, D = q.shape
    rc = _native.lib().hyena_conv_fwd_f32(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          h.data_ptr(), y.data_ptr(), B, L, D, d_g, h.shape[1],
                                          l_b, _stream(stream))
    _native.check("hyena_conv_fwd_f32", rc)
    return y


def hyena_select_algo(B, L, D, d_g, l_h, l_b, dtype=HYENA_DTYPE_BF16, ptrs=(16, 16, 16, 16, 16)):
    """Host-only: the algorithm AUTO would run (HYENA_ALGO_*), or raises HyenaError.

    ``ptrs`` are the (q, k, v, h, y) addresses whose alignment counts (plain integers); the
    defaults stand for distinct 16-byte aligned buffers.
    """
    n = B * L * D * (4 if dtype == HYENA_DTYPE_F32 else 2)
    q, k, v, h, y = ptrs
    if ptrs == (16, 16, 16, 16, 16):  # distinct, non-overlapping, aligned stand-ins
        q, k, v, h, y = (16 + i * (n + 64) for i in range(5))
    rc = _native.lib().hyena_select_algo(q, k, v, h, y, B, L, D, d_g, l_h, l_b, dtype)
    if rc < 0:
        raise HyenaError("hyena_select_algo", -rc)
    return rc


def hyena_conv_bwd_workspace_bytes(B, L, D, d_g, l_h):
    """Host-only: device workspace bytes hyena_conv_bwd needs for this shape."""
    n = _native.lib().hyena_conv_bwd_workspace_bytes(B, L, D, d_g, l_h)
    if n < 0:
        raise HyenaError("hyena_conv_bwd_workspace_bytes", -n)
    return n


def hyena_conv_bwd(q, k, v, h, dy, d_g, l_b, workspace=None, grads=None, stream=None):
    """Backward, fastest supported algorithm (C: hyena_conv_bwd); see hyena_conv_bwd_ex."""
    return hyena_conv_bwd_ex(q, k, v, h, dy, d_g, l_b, HYENA_ALGO_AUTO, workspace, grads,
                             stream)


def hyena_select_bwd_algo(B, L, D, d_g, l_h, l_b, dtype=HYENA_DTYPE_BF16):
    """Host-only: the backward algorithm AUTO would run for distinct 16-byte aligned buffers."""
    n = B * L * D * (4 if dtype == HYENA_DTYPE_F32 else 2)
    p = [16 + i * (n + 64) for i in range(8)]
    rc = _native.lib().hyena_select_bwd_algo(*p, B, L, D, d_g, l_h, l_b, dtype)
    if rc < 0:
        raise HyenaError("hyena_select_bwd_algo", -rc)
    return rc


def hyena_conv_bwd_ex(q, k, v, h, dy, d_g, l_b, algo=HYENA_ALGO_AUTO, workspace=None,
                      grads=None, stream=None):
    """Backward of the gated FIR with the algorithm chosen by the caller; returns
    (dq, dk, dv, dh).

    q, k, v, dy: CUDA [B, L, D], one dtype (bf16 or fp32).  h: CUDA fp32 [D // d_g, l_h].
    dq, dk, dv come back in the dtype of q, dh in fp32 [D // d_g, l_h] (overwritten, not
    accumulated).  ``workspace``: optional CUDA uint8 tensor of at least
    hyena_conv_bwd_workspace_bytes() bytes (allocated here from torch when omitted).
    ``grads``: optional preallocated (dq, dk, dv, dh).
    """
    torch = _torch()
    _check(q, k, v, h, d_g, None)
    if (not isinstance(dy, torch.Tensor) or not dy.is_cuda or dy.shape != q.shape
            or dy.dtype != q.dtype or not dy.is_contiguous()):
        raise ValueError("dy must be a contiguous CUDA tensor like q")
    B, L, D = q.shape
    l_h = h.shape[1]
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(q), torch.empty_like(q),
                 torch.empty_like(h))
    dq, dk, dv, dh = grads
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        if (t.shape != q.shape or t.dtype != q.dtype or not t.is_cuda
                or not t.is_contiguous()):
            raise ValueError("%s must be a contiguous CUDA tensor like q" % name)
    if dh.shape != h.shape or dh.dtype != torch.float32 or not dh.is_cuda \
            or not dh.is_contiguous():
        raise ValueError("dh must be a contiguous CUDA float32 tensor like h")
    need = hyena_conv_bwd_workspace_bytes(B, L, D, d_g, l_h)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = _native.lib().hyena_conv_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         h.data_ptr(), dy.data_ptr(), dq.data_ptr(),
                                         dk.data_ptr(), dv.data_ptr(), dh.data_ptr(), B, L, D,
                                         d_g, l_h, l_b, _dtype_code(q), algo,
                                         workspace.data_ptr(), ws_bytes, _stream(stream))
    _native.check("hyena_conv_bwd_ex", rc)
    return dq, dk, dv, dh


def hyena_build_toeplitz(h, l_b, stream=None):
    """H0, H1, H2 (fp32 [G, l_b, l_b] CUDA tensors): H_m[g][i][j] = h[g][m l_b + i - j]."""
    torch = _torch()
    if not isinstance(h, torch.Tensor) or not h.is_cuda or h.dtype != torch.float32 \
            or h.dim() != 2 or not h.is_contiguous():
        raise TypeError("h must be a contiguous CUDA float32 [G, l_h] tensor")
    G, l_h = h.shape
    H = torch.empty((3, G, l_b, l_b), dtype=torch.float32, device=h.device)
    rc = _native.lib().hyena_build_toeplitz(h.data_ptr(), H[0].data_ptr(), H[1].data_ptr(),
                                            H[2].data_ptr(), G, l_h, l_b, _stream(stream))
    _native.check("hyena_build_toeplitz", rc)
    return H[0], H[1], H[2]


def hyena_toeplitz_stages(l_h, l_b):
    """Sub-block diagonals S = 1 + ceil((l_h - 1) / l_b) of the block-Toeplitz decomposition."""
    rc = int(_native.lib().hyena_toeplitz_stages(l_h, l_b))
    if rc < 0:
        _native.check("hyena_toeplitz_stages", -rc)
    return rc


def hyena_build_toeplitz_blocks(h, l_b, S=None, stream=None):
    """fp32 CUDA tensor [S, G, l_b, l_b] with Hm[m][g][i][j] = h[g][m l_b + i - j] (zero outside
    [0, l_h)); S defaults to the number of non-zero sub-block diagonals."""
    torch = _torch()
    if not isinstance(h, torch.Tensor) or not h.is_cuda or h.dtype != torch.float32 \
            or h.dim() != 2 or not h.is_contiguous():
        raise TypeError("h must be a contiguous CUDA float32 [G, l_h] tensor")
    G, l_h = h.shape
    if S is None:
        S = hyena_toeplitz_stages(l_h, l_b)
    H = torch.empty((S, G, l_b, l_b), dtype=torch.float32, device=h.device)
    rc = _native.lib().hyena_build_toeplitz_blocks(h.data_ptr(), H.data_ptr(), S, G, l_h, l_b,
                                                   _stream(stream))
    _native.check("hyena_build_toeplitz_blocks", rc)
    return H


def hyena_device_status(clear=True):
    """The current device's status word (HYENA_DEVICE_* bits); synchronises the device."""
    out = ctypes.c_uint(0)
    _native.check("hyena_device_status",
                  _native.lib().hyena_device_status(ctypes.byref(out), 1 if clear else 0))
    return out.value


def hyena_status_string(status):
    return _native.status_string(status)


def hyena_abi_version():
    return int(_native.lib().hyena_abi_version())


_HOST_WS = {}


def hyena_conv_fwd_from_host_workspace_bytes(B, L, D, d_g, l_h, dtype="bf16", chunk=2048):
    code = HYENA_DTYPE_F32 if dtype in ("f32", "float32") else HYENA_DTYPE_BF16
    n = int(_native.lib().hyena_conv_fwd_from_host_workspace_bytes(B, L, D, d_g, l_h, code,
                                                                   chunk))
    if n < 0:
        raise _native.HyenaError("hyena_conv_fwd_from_host_workspace_bytes", -n)
    return n


def hyena_conv_fwd_from_host(q, k, v, h, d_g, l_b, out=None, device="cuda", stream=None,
                             chunk=2048, workspace=None):
    """End-to-end forward for HOST tensors through the C entry point of the same name: q, k, v
    (bf16 or fp32 [B, L, D], contiguous; pinned for overlapped copies) and h (fp32
    [D / d_g, l_h]) go to ``device`` chunk by chunk, the forward runs there and y comes back
    into ``out`` (a host tensor, pinned when created here).  The library queues every copy and
    kernel; this wrapper only supplies the device workspace (cached per shape when not given)
    and the stream.  Synchronise ``stream`` (default: the current stream) before reading
    ``out``."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v), ("h", h)):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise TypeError("%s must be a contiguous host tensor" % name)
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share shape and dtype")
    if h.dtype != torch.float32:
        raise TypeError("h must be float32")
    B, L, D = q.shape
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    elif out.device.type != "cpu" or not out.is_contiguous() or out.shape != q.shape or \
            out.dtype != q.dtype:
        raise TypeError("out must be a contiguous host tensor like q")
    dev = torch.device(device)
    if workspace is None:
        need = int(_native.lib().hyena_conv_fwd_from_host_workspace_bytes(
            B, L, D, d_g, h.shape[1], dt, chunk))
        if need < 0:
            raise _native.HyenaError("hyena_conv_fwd_from_host", -need)
        key = (str(dev), need)
        workspace = _HOST_WS.get(key)
        if workspace is None:
            _HOST_WS.clear()
            workspace = _HOST_WS[key] = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream(dev) if stream is None else stream
    # the library's streams finish before `st` goes on: the allocator must not hand the
    # workspace out again before `st` has passed this call
    workspace.record_stream(st)
    with torch.cuda.device(dev):
        _native.check("hyena_conv_fwd_from_host", _native.lib().hyena_conv_fwd_from_host(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), h.data_ptr(), out.data_ptr(), B, L, D,
            d_g, h.shape[1], l_b, dt, chunk, workspace.data_ptr(), workspace.numel(),
            st.cuda_stream))
    return out
