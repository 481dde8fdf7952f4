"""Backward of the gated FIR on the GPU vs the fp64 oracle's gradients, through the C ABI.

Tolerances:
  * dq, dk, dv: those of the forward (bf16: 1e-2 + 1e-2 |ref| elementwise; fp32 normwise 1e-5);
    each is one fp32 sum of at most l_h exact products, rounded once to the output type.
  * dh (fp32 output): normwise max|dh - ref| <= 1e-4 max|ref|.  Each dh[g][j] is a sum of
    N = B * L * d_g terms of rms ~1 for these inputs, so |ref| ~ sqrt(N).  The kernels add
    them as fp32 partials of 64 rows x (up to) 64 channels, then a fixed-order sum of the
    partials; rounding errors of random sign give about u * 64 * sqrt(4096) * sqrt(N / 4096)
    ~ 2e-6 sqrt(N), i.e. ~2e-6 normwise, so 1e-4 keeps a 50x margin while a single dropped
    or doubled term (~1 / sqrt(N) normwise, 1.4e-3 at the MR size) still fails.
  * Integer-valued inputs (test_integer_exact): every product and partial sum is an exact
    integer, so all four gradients must equal the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

import gated_causal_fir_b200 as g
from gated_causal_fir_b200.workloads import (WORKLOADS, custom, make_grad, make_inputs,
                                             make_integer_inputs)
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


def _bwd(q, k, v, h, dy, wl):
    out = g.hyena_conv_bwd(q, k, v, h, dy, wl.d_g, wl.l_b)
    torch.cuda.synchronize()
    return out


def _check_all(out, ref, dtype):
    dq, dk, dv, dh = out
    rq, rk, rv, rh = ref
    U.assert_parity(dq, rq, dtype)
    U.assert_parity(dk, rk, dtype)
    U.assert_parity(dv, rv, dtype)
    got = dh.detach().cpu().double().numpy()
    assert np.all(np.isfinite(got)), "non-finite dh"
    r = U.f32_normwise(got, rh)
    assert r <= DH_NORMWISE, "dh normwise error %.3e > %.1e" % (r, DH_NORMWISE)


@pytest.mark.parametrize("name", ["tiny", "se", "mr"])
def test_bwd_workload(name):
    wl = WORKLOADS[name]
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    out = _bwd(q, k, v, h, dy, wl)
    ref = oracle.gated_fir_bwd(q, k, v, h, dy, wl.d_g)
    _check_all(out, ref, q.dtype)


SHAPES = [
    # name, B, L, D, d_g, l_h, l_b, dtype
    ("mr_ragged", 2, 1000, 256, 64, 128, 64, "bf16"),
    ("dg32_odd_D", 3, 777, 96, 32, 33, 32, "bf16"),
    ("dg48", 1, 530, 96, 48, 20, 16, "bf16"),
    ("short_seq", 1, 77, 128, 64, 128, 64, "bf16"),
    ("single_token", 1, 1, 64, 64, 7, 16, "bf16"),
    ("single_tap", 2, 513, 256, 64, 1, 1, "bf16"),
    ("max_halo", 1, 700, 128, 64, 129, 65, "bf16"),
    ("long_filter", 1, 600, 64, 64, 200, 100, "bf16"),
    ("f32_dg6", 2, 301, 12, 6, 5, 4, "f32"),
    ("f32_mr", 1, 900, 128, 64, 128, 64, "f32"),
]


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_bwd_shapes(shape):
    name, B, L, D, d_g, l_h, l_b, dt = shape
    wl = custom(name, B, L, D, d_g, l_h, l_b, dt, filt="mr" if l_h > 16 else "se", seed=11)
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    out = _bwd(q, k, v, h, dy, wl)
    ref = oracle.gated_fir_bwd(q, k, v, h, dy, wl.d_g)
    _check_all(out, ref, q.dtype)


INT_SHAPES = [
    ("mr", 2, 1500, 256, 64, 128, 64, "bf16"),
    ("se", 1, 2000, 512, 16, 7, 16, "bf16"),
    ("dg32", 1, 1000, 128, 32, 65, 64, "bf16"),
    ("f32", 2, 700, 64, 8, 12, 8, "f32"),
]


@pytest.mark.parametrize("shape", INT_SHAPES, ids=[s[0] for s in INT_SHAPES])
def test_integer_exact(shape):
    name, B, L, D, d_g, l_h, l_b, dt = shape
    assert B * L * d_g * 16 < 2 ** 24
    wl = custom("int_" + name, B, L, D, d_g, l_h, l_b, dt, seed=5)
    q, k, v, dy, h = make_integer_inputs(wl, device="cuda")
    dq, dk, dv, dh = _bwd(q, k, v, h, dy, wl)
    rq, rk, rv, rh = oracle.gated_fir_bwd(q, k, v, h, dy, wl.d_g)
    tdt = q.dtype
    for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        want = torch.from_numpy(ref).to(tdt)  # the exact value rounded once, as the kernels do
        assert torch.equal(got.cpu(), want), "%s differs from the exact gradient" % nm
    assert np.array_equal(dh.cpu().double().numpy(), rh), "dh differs from the exact sum"


def test_bwd_deterministic():
    wl = custom("det", 2, 1000, 256, 64, 128, 64, "bf16", filt="mr", seed=3)
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    a = [t.clone() for t in _bwd(q, k, v, h, dy, wl)]
    b = _bwd(q, k, v, h, dy, wl)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bwd_empty_zeroes_dh():
    wl = custom("empty", 1, 0, 64, 64, 7, 16, "bf16")
    q, k, v, h = make_inputs(custom("e1", 1, 1, 64, 64, 7, 16, "bf16"), device="cuda")
    z = torch.empty((1, 0, 64), dtype=torch.bfloat16, device="cuda")
    dh = torch.full_like(h, 5.0)
    g.hyena_conv_bwd(z, z, z, h, z, wl.d_g, wl.l_b,
                     grads=(torch.empty_like(z), torch.empty_like(z), torch.empty_like(z), dh))
    torch.cuda.synchronize()
    assert torch.count_nonzero(dh).item() == 0


def test_bwd_rejects_bad_workspace_and_overlap():
    wl = custom("bad", 1, 300, 128, 64, 16, 16, "bf16")
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    need = g.hyena_conv_bwd_workspace_bytes(1, 300, 128, 64, 16)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(g.HyenaError) as e:
        g.hyena_conv_bwd(q, k, v, h, dy, 64, 16, workspace=small)
    assert e.value.status == 1
    dq = torch.empty_like(q)
    with pytest.raises(g.HyenaError) as e:
        g.hyena_conv_bwd(q, k, v, h, dy, 64, 16, grads=(dq, dq, torch.empty_like(q),
                                                        torch.empty_like(h)))
    assert e.value.status == 1
