"""Backward of the gated FIR on the GPU vs the fp64 oracle's gradients, through the C ABI.

Tolerances:
  * dq, dk, dv: those of the forward (bf16: 1e-2 + 1e-2 |ref| elementwise; fp32 normwise 1e-5);
    each is one fp32 sum of at most l_h exact products, rounded once to the output type.
  * dh (fp32 output), CUDA-core path: normwise max|dh - ref| <= 1e-4 max|ref|.  Each
    dh[g][j] is a sum of N = B * L * d_g terms of rms ~1 for these inputs, so |ref| ~ sqrt(N).
    The kernels add them as fp32 partials of 64 rows x (up to) 64 channels, then a fixed-order
    sum of the partials; rounding errors of random sign give about
    u * 64 * sqrt(4096) * sqrt(N / 4096) ~ 2e-6 sqrt(N), i.e. ~2e-6 normwise, so 1e-4 keeps a
    50x margin while a single dropped or doubled term (~1 / sqrt(N) normwise, 1.4e-3 at the MR
    size) still fails.
  * dh, window path (l_h <= 16): normwise 1e-4, as the CUDA-core path: each thread sums
    dz[t + j] x[t] over its run (at most 128 rows) and its 4 or 8 channels, a fixed-order sum
    of those partials follows; the same error estimate holds.
  * dh, tensor path: normwise 2e-3.  Its products take x = k v and dz = q dy rounded to fp16
    (relative error <= 2^-11 each, ~4e-4 rms per product); the sum of N such errors of random
    sign is ~4e-4 sqrt(N), i.e. ~4e-4 / 3.5 ~ 1.2e-4 of max|ref| on average and ~5e-4 at the
    worst of the G * l_h outputs.  2e-3 keeps a 4x margin; a wrong lag, tile or group moves
    dh by O(max|ref|).  The integer cases pin this path exactly.
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

DH_NORMWISE = {g.HYENA_ALGO_DIRECT: 1e-4, g.HYENA_ALGO_TENSOR: 2e-3,
               g.HYENA_ALGO_WINDOW: 1e-4}
ALGOS = {"direct": g.HYENA_ALGO_DIRECT, "tensor": g.HYENA_ALGO_TENSOR,
         "window": g.HYENA_ALGO_WINDOW}


def _tensor_fits(B, L, D, d_g, l_h, dt):
    return dt == "bf16" and d_g == 64 and D % 64 == 0 and l_h <= 129


def _window_fits(B, L, D, d_g, l_h, dt):
    return l_h <= 16 and d_g % (4 if dt == "f32" else 8) == 0


def _fits(algo, shape):
    if algo == "direct":
        return True
    fits = _tensor_fits if algo == "tensor" else _window_fits
    return fits(*shape[1:6], shape[7])


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_causal_fir_b200 import build
    build.build()
    g.hyena_device_status(clear=True)
    yield
    assert g.hyena_device_status(clear=True) == 0, "a kernel raised its device status word"


def _bwd(q, k, v, h, dy, wl, algo=g.HYENA_ALGO_AUTO):
    out = g.hyena_conv_bwd_ex(q, k, v, h, dy, wl.d_g, wl.l_b, algo=algo)
    torch.cuda.synchronize()
    return out


def _check_all(out, ref, dtype, algo):
    dq, dk, dv, dh = out
    rq, rk, rv, rh = ref
    U.assert_parity(dq, rq, dtype)
    U.assert_parity(dk, rk, dtype)
    U.assert_parity(dv, rv, dtype)
    got = dh.detach().cpu().double().numpy()
    assert np.all(np.isfinite(got)), "non-finite dh"
    r = U.f32_normwise(got, rh)
    tol = DH_NORMWISE[algo]
    assert r <= tol, "dh normwise error %.3e > %.1e" % (r, tol)


@pytest.mark.parametrize("name", ["tiny", "se", "mr"])
def test_bwd_workload(name):
    """The default entry point on the workloads; MR runs the fused tensor kernel."""
    wl = WORKLOADS[name]
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    algo = g.hyena_select_bwd_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b,
                                   g.HYENA_DTYPE_F32 if wl.dtype == "f32" else g.HYENA_DTYPE_BF16)
    assert algo == (g.HYENA_ALGO_TENSOR if name == "mr" else g.HYENA_ALGO_WINDOW)
    out = g.hyena_conv_bwd(q, k, v, h, dy, wl.d_g, wl.l_b)
    torch.cuda.synchronize()
    ref = oracle.gated_fir_bwd(q, k, v, h, dy, wl.d_g)
    _check_all(out, ref, q.dtype, algo)


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
    ("runs_across_seqs", 3, 3000, 512, 64, 100, 64, "bf16"),
    ("long_seq_one_group", 1, 40000, 64, 64, 128, 64, "bf16"),
    ("batched_halo16", 4, 2048, 128, 64, 17, 16, "bf16"),
    ("three_blocks", 2, 900, 192, 64, 64, 64, "bf16"),  # odd block count: unpaired walk
    ("se_window", 2, 1500, 256, 16, 7, 16, "bf16"),
    ("window_16_taps", 1, 700, 128, 8, 16, 16, "bf16"),
    ("window_f32_ragged", 3, 333, 32, 4, 3, 4, "f32"),
    ("window_runs_short", 2, 20, 64, 16, 7, 16, "bf16"),   # one run shorter than the halo
]
CASES = [(s, a) for s in SHAPES for a in ALGOS if _fits(a, s)]


@pytest.mark.parametrize("shape,algo", CASES, ids=["%s-%s" % (s[0], a) for s, a in CASES])
def test_bwd_shapes(shape, algo):
    name, B, L, D, d_g, l_h, l_b, dt = shape
    wl = custom(name, B, L, D, d_g, l_h, l_b, dt, filt="mr" if l_h > 16 else "se", seed=11)
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    out = _bwd(q, k, v, h, dy, wl, ALGOS[algo])
    ref = oracle.gated_fir_bwd(q, k, v, h, dy, wl.d_g)
    _check_all(out, ref, q.dtype, ALGOS[algo])


def test_bwd_window_unsupported_is_rejected():
    wl = custom("w17", 1, 300, 128, 16, 17, 16, "bf16")  # 17 taps: past the register window
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    with pytest.raises(g.HyenaError) as e:
        _bwd(q, k, v, h, dy, wl, g.HYENA_ALGO_WINDOW)
    assert e.value.status == 2


def test_bwd_tensor_unsupported_is_rejected():
    wl = custom("dg32", 1, 300, 128, 32, 16, 16, "bf16")
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    with pytest.raises(g.HyenaError) as e:
        _bwd(q, k, v, h, dy, wl, g.HYENA_ALGO_TENSOR)
    assert e.value.status == 2


INT_SHAPES = [
    ("mr", 2, 1500, 256, 64, 128, 64, "bf16"),
    ("mr_halo_129", 1, 3000, 128, 64, 129, 65, "bf16"),
    ("se", 1, 2000, 512, 16, 7, 16, "bf16"),
    ("dg32", 1, 1000, 128, 32, 65, 64, "bf16"),
    ("f32", 2, 700, 64, 8, 12, 8, "f32"),
]
INT_CASES = [(s, a) for s in INT_SHAPES for a in ALGOS if _fits(a, s)]


@pytest.mark.parametrize("shape,algo", INT_CASES,
                         ids=["%s-%s" % (s[0], a) for s, a in INT_CASES])
def test_integer_exact(shape, algo):
    name, B, L, D, d_g, l_h, l_b, dt = shape
    assert B * L * d_g * 16 < 2 ** 24
    wl = custom("int_" + name, B, L, D, d_g, l_h, l_b, dt, seed=5)
    q, k, v, dy, h = make_integer_inputs(wl, device="cuda")
    dq, dk, dv, dh = _bwd(q, k, v, h, dy, wl, ALGOS[algo])
    rq, rk, rv, rh = oracle.gated_fir_bwd(q, k, v, h, dy, wl.d_g)
    tdt = q.dtype
    for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        want = torch.from_numpy(ref).to(tdt)  # the exact value rounded once, as the kernels do
        assert torch.equal(got.cpu(), want), "%s differs from the exact gradient" % nm
    assert np.array_equal(dh.cpu().double().numpy(), rh), "dh differs from the exact sum"


@pytest.mark.parametrize("algo", list(ALGOS))
def test_bwd_deterministic(algo):
    if algo == "window":
        wl = custom("det_w", 2, 1000, 256, 16, 7, 16, "bf16", seed=3)
    else:
        wl = custom("det", 2, 1000, 256, 64, 128, 64, "bf16", filt="mr", seed=3)
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    a = [t.clone() for t in _bwd(q, k, v, h, dy, wl, ALGOS[algo])]
    b = _bwd(q, k, v, h, dy, wl, ALGOS[algo])
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
    small = torch.empty(256, dtype=torch.uint8, device="cuda")  # under any algorithm's need
    with pytest.raises(g.HyenaError) as e:
        g.hyena_conv_bwd(q, k, v, h, dy, 64, 16, workspace=small)
    assert e.value.status == 1
    dq = torch.empty_like(q)
    with pytest.raises(g.HyenaError) as e:
        g.hyena_conv_bwd(q, k, v, h, dy, 64, 16, grads=(dq, dq, torch.empty_like(q),
                                                        torch.empty_like(h)))
    assert e.value.status == 1
