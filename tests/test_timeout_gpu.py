"""Failure detection of the tensor-core forward, made to fire without faulting the GPU (needs a
B200).

Every wait between the kernel's warp roles is bounded.  The test entry point
hyena_testing_fwd_fault shortens that bound to 20 ms and has the MMA issuer withhold the arrive
that tells the epilogue the first tile's accumulator is ready, so the epilogue's wait runs out.
The kernel must then record HYENA_DEVICE_TIMEOUT, let every role leave, drain its copies and
MMAs, free tensor memory and return well within a second; the next ordinary call on the same
device must run normally and match the oracle.
"""
import time

import pytest
import torch

import gated_causal_fir_b200 as g
from gated_causal_fir_b200 import _native
from gated_causal_fir_b200.workloads import custom, make_inputs
from tests import _gpu_util as U

pytestmark = pytest.mark.gpu

WAIT_NS = 20 * 1000 * 1000  # 20 ms


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_causal_fir_b200 import build
    build.build()
    g.hyena_device_status(clear=True)
    yield
    assert g.hyena_device_status(clear=True) == 0, "a kernel raised its device status word"


def _call(q, k, v, h, y, wl, fault):
    B, L, D = q.shape
    return _native.lib().hyena_testing_fwd_fault(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), h.data_ptr(), y.data_ptr(), B, L, D, wl.d_g,
        wl.l_h, fault, WAIT_NS, torch.cuda.current_stream().cuda_stream)


def test_short_limit_without_fault_runs_normally():
    wl = custom("timeout_ok", 1, 700, 128, 64, 128, 64, "bf16", "mr", seed=81)
    q, k, v, h = make_inputs(wl, device="cuda")
    y = torch.empty_like(q)
    assert g.hyena_device_status(clear=True) == 0
    assert _call(q, k, v, h, y, wl, 0) == _native.HYENA_OK
    torch.cuda.synchronize()
    assert g.hyena_device_status(clear=True) == 0
    U.assert_parity(y, U.oracle_full(q, k, v, h, wl.d_g), q.dtype)


def test_withheld_arrive_times_out_and_the_device_recovers():
    wl = custom("timeout", 1, 700, 128, 64, 128, 64, "bf16", "mr", seed=82)
    q, k, v, h = make_inputs(wl, device="cuda")
    y = torch.empty_like(q)
    torch.cuda.synchronize()
    assert g.hyena_device_status(clear=True) == 0
    t0 = time.perf_counter()
    assert _call(q, k, v, h, y, wl, 1) == _native.HYENA_OK
    torch.cuda.synchronize()  # the kernel returns: no hang, no fault
    dt = time.perf_counter() - t0
    status = g.hyena_device_status(clear=True)
    assert status & g.HYENA_DEVICE_TIMEOUT, "status word %#x lacks HYENA_DEVICE_TIMEOUT" % status
    assert dt < 1.0, "the timed-out kernel took %.3f s" % dt
    # the context is usable: an ordinary call on the same device matches the oracle
    y2 = g.hyena_conv_fwd(q, k, v, h, wl.d_g, wl.l_b)
    torch.cuda.synchronize()
    assert g.hyena_device_status(clear=True) == 0
    U.assert_parity(y2, U.oracle_full(q, k, v, h, wl.d_g), q.dtype)
