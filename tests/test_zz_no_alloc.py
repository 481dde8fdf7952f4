"""hyena_conv_bwd_static_scratch (partials in the library's fixed device array) against
hyena_conv_bwd (partials in a caller workspace), both called through the C ABI, and both
against the fp64 oracle.

The entry point serves callers that cannot hand the library device memory: a C host program
with no device allocator of its own, or a runtime that reserves all device memory up front and
allows no allocation afterwards.  Collected last on purpose: it must hold both alone and after
every other test has run kernels on the device.  Tolerances are those of the backward parity
tests (tests/test_bwd_gpu.py): the forward's bf16 bound for dq, dk, dv; for dh normwise 1e-4
between the two entry points, and against the oracle 2e-3 on the tensor-core path (fp16
operands), 1e-4 on the CUDA-core paths (fp32).
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_causal_fir_b200 as g
from gated_causal_fir_b200 import _native
from gated_causal_fir_b200.workloads import custom, make_grad, make_inputs
from tests import _gpu_util as U
import oracle

pytestmark = pytest.mark.gpu

DH_NORMWISE = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_causal_fir_b200 import build
    build.build()
    g.hyena_device_status(clear=True)
    yield
    assert g.hyena_device_status(clear=True) == 0, "a kernel raised its device status word"


def _ptrs(*ts):
    return [t.data_ptr() for t in ts]


def _call_static(q, k, v, h, dy, wl, dtype_code):
    dq, dk, dv, dh = (torch.empty_like(q), torch.empty_like(q), torch.empty_like(q),
                      torch.full_like(h, float("nan")))
    B, L, D = q.shape
    rc = _native.lib().hyena_conv_bwd_static_scratch(
        *_ptrs(q, k, v, h, dy, dq, dk, dv, dh), B, L, D, wl.d_g, wl.l_h, wl.l_b, dtype_code,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, _native.status_string(rc)
    return dq, dk, dv, dh


def _call_workspace(q, k, v, h, dy, wl, dtype_code):
    dq, dk, dv, dh = (torch.empty_like(q), torch.empty_like(q), torch.empty_like(q),
                      torch.empty_like(h))
    B, L, D = q.shape
    need = _native.lib().hyena_conv_bwd_workspace_bytes(B, L, D, wl.d_g, wl.l_h)
    assert need >= 0
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    rc = _native.lib().hyena_conv_bwd(
        *_ptrs(q, k, v, h, dy, dq, dk, dv, dh), B, L, D, wl.d_g, wl.l_h, wl.l_b, dtype_code,
        ws.data_ptr(), ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, _native.status_string(rc)
    return dq, dk, dv, dh


def _close(got, want, dtype):
    for a, b in zip(got[:3], want[:3]):
        U.assert_parity(a, b.detach().cpu().double().numpy(), dtype)
    r = U.f32_normwise(got[3].cpu().double().numpy(), want[3].cpu().double().numpy())
    assert r <= DH_NORMWISE, "dh normwise difference %.3e" % r


def _close_to_oracle(got, ref, dtype, dh_tol):
    for a, b in zip(got[:3], ref[:3]):
        U.assert_parity(a, b, dtype)
    r = U.f32_normwise(got[3].cpu().double().numpy(), ref[3])
    assert r <= dh_tol, "dh normwise error against the oracle %.3e > %.0e" % (r, dh_tol)


CASES = [
    # name, B, L, D, d_g, l_h, l_b, dtype, dtype code, backward algorithm, dh tolerance
    # the full D = 4096, d_g = 64, l_h = 128 shape at 8192 tokens (4 MiB of partials): tcgen05
    ("mr", 1, 8192, 4096, 64, 128, 64, "bf16", g.HYENA_DTYPE_BF16, g.HYENA_ALGO_TENSOR, 2e-3),
    # the SE shape class (d_g = 16, l_h = 7): the register-window backward
    ("se", 1, 4096, 1024, 16, 7, 16, "bf16", g.HYENA_DTYPE_BF16, g.HYENA_ALGO_WINDOW, 1e-4),
    # 2^27 elements at l_h = 16: one partial per 16-byte channel vector and 128-row run would
    # need 10 MiB, more than the 8 MiB scratch, so the window backward lengthens its runs to
    # 160 rows to fit (the caller-workspace call gets room for the 128-row runs).  d_g = 32
    # keeps the least workspace any algorithm needs (the CUDA-core partials, 5 MiB) inside the
    # scratch, which the entry point requires.
    ("window_runs_fit_scratch", 1, 327680, 512, 32, 16, 16, "bf16", g.HYENA_DTYPE_BF16,
     g.HYENA_ALGO_WINDOW, 1e-4),
    # the CUDA-core kernels (d_g = 6 fits neither fast path)
    ("ragged_f32", 2, 301, 12, 6, 5, 4, "f32", g.HYENA_DTYPE_F32, g.HYENA_ALGO_DIRECT, 1e-4),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_static_scratch_matches_workspace_entry(case):
    name, B, L, D, d_g, l_h, l_b, dt, code, algo, dh_tol = case
    wl = custom(name, B, L, D, d_g, l_h, l_b, dt, filt="mr" if l_h > 16 else "se", seed=21)
    assert g.hyena_select_bwd_algo(B, L, D, d_g, l_h, l_b, code) == algo
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    want = _call_workspace(q, k, v, h, dy, wl, code)
    first = _call_static(q, k, v, h, dy, wl, code)
    second = _call_static(q, k, v, h, dy, wl, code)  # the scratch is reused as left
    torch.cuda.synchronize()
    _close(first, want, q.dtype)
    _close(second, want, q.dtype)
    assert np.isfinite(second[3].cpu().numpy()).all()
    ref = oracle.gated_fir_bwd(q, k, v, h, dy, d_g)
    _close_to_oracle(first, ref, q.dtype, dh_tol)
    _close_to_oracle(second, ref, q.dtype, dh_tol)
