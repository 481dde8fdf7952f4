"""Operands outside fp16's range on the tensor-core backward, against the fp64 oracle's
gradients (needs a B200).

The backward's tensor kernel rounds x = k v, dz = q dy and the filter taps to fp16, unscaled, for
its MMAs.  Where any of them holds a value above 65504 (it would round to inf), or a group's taps
all lie below 2^-10, the kernel writes the call's token into a flag in the workspace and raises
HYENA_DEVICE_F16_RANGE; the fp32 CUDA-core kernels queued behind it then rewrite dk, dv and dh.
dq always comes from the forward kernels, which handle the range themselves.  Every case must
match the oracle: dq, dk, dv normwise, max |d - d_ref| / max |d_ref| <= 2^-8 (bf16 rounding
alone costs up to 2^-9), and, where the inputs keep the O(1) scale the bound's absolute term
assumes, also under the bf16 bound |d - d_ref| <= 1e-2 + 1e-2 |d_ref| elementwise; dh normwise
<= 2e-3 (the tensor path's bound; the fp32 path is far inside it).  (With operands scaled by 2^s
the gradients scale too, and the elementwise bound's absolute term would have to scale with
them.)  An operand saturated at inf misses these bounds outright."""
import pytest
import torch

import gated_causal_fir_b200 as g
from gated_causal_fir_b200.workloads import custom, make_grad, make_inputs
from tests import _gpu_util as U
import oracle

pytestmark = pytest.mark.gpu

NORMWISE = 2.0 ** -8
DH_NORMWISE = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_causal_fir_b200 import build
    build.build()
    g.hyena_device_status(clear=True)
    yield
    g.hyena_device_status(clear=True)


# two sequences of 64 tiles over 4 groups: 512 tiles on at most 148 CTAs, so every CTA walks
# several tiles and sequence runs
SHAPE = dict(B=2, L=8192, D=256, d_g=64, l_h=128, l_b=64)


def _inputs(seed):
    wl = custom("bwd_range", SHAPE["B"], SHAPE["L"], SHAPE["D"], SHAPE["d_g"], SHAPE["l_h"],
                SHAPE["l_b"], "bf16", "mr", seed=seed)
    assert g.hyena_select_bwd_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b) == \
        g.HYENA_ALGO_TENSOR
    q, k, v, h = make_inputs(wl, device="cuda")
    dy = make_grad(wl, device="cuda")
    return wl, q, k, v, h, dy


def _check(wl, q, k, v, h, dy, elementwise=True):
    """Gradients through the tensor path against the oracle; returns the status word."""
    g.hyena_device_status(clear=True)
    out = g.hyena_conv_bwd_ex(q, k, v, h, dy, wl.d_g, wl.l_b, algo=g.HYENA_ALGO_TENSOR)
    torch.cuda.synchronize()
    status = g.hyena_device_status(clear=True)
    ref = oracle.gated_fir_bwd(q, k, v, h, dy, wl.d_g)
    for name, got, want in zip(("dq", "dk", "dv"), out[:3], ref[:3]):
        assert torch.isfinite(got).all(), "%s: non-finite gradient" % name
        if elementwise:
            U.assert_parity(got, want, torch.bfloat16)
        r = U.f32_normwise(got, want)
        assert r <= NORMWISE, "%s normwise error %.2e > %.2e" % (name, r, NORMWISE)
    r = U.f32_normwise(out[3].cpu().double().numpy(), ref[3])
    assert r <= DH_NORMWISE, "dh normwise error %.2e > %.0e" % (r, DH_NORMWISE)
    return status


def _bf16(x):
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("where", ["kv", "dz"])
def test_outlier_takes_the_fp32_path(where):
    """|k v| or |q dy| = 160000 > 65504 at one element: the kernel raises the flag and the fp32
    kernels redo dk, dv, dh; every gradient stays finite and matches."""
    wl, q, k, v, h, dy = _inputs(31)
    a, b = (k, v) if where == "kv" else (q, dy)
    a[1, 4000, 70] = 400.0
    b[1, 4000, 70] = 400.0
    status = _check(wl, q, k, v, h, dy)
    assert status & g.HYENA_DEVICE_F16_RANGE


@pytest.mark.parametrize("case", [
    # name, k scale, v scale, q scale, dy scale, h scale, the fp32 path runs
    ("kv_huge", 2.0 ** 8, 2.0 ** 8, 1.0, 1.0, 1.0, True),       # |x| up to ~2^20
    ("q_huge", 1.0, 1.0, 2.0 ** 9, 2.0 ** 9, 1.0, True),        # |dz| up to ~2^22
    ("q_tiny_dy_huge", 1.0, 1.0, 2.0 ** -20, 2.0 ** 20, 1.0, False),  # dz ~ 1
    ("taps_tiny", 1.0, 1.0, 1.0, 1.0, 2.0 ** -20, True),        # taps deep in the subnormals
    ("taps_large", 1.0, 1.0, 1.0, 1.0, 2.0 ** 14, False),       # taps up to ~2^14.3: in range
], ids=lambda c: c[0])
def test_scaled_operands(case):
    """Uniformly scaled operands: in range the tensor path runs alone (status 0); beyond it the
    fp32 path takes over; the gradients match either way."""
    name, sk, sv, sq, sdy, sh, fallback = case
    wl, q, k, v, h, dy = _inputs(37)
    q, k, v, dy = _bf16(q.float() * sq), _bf16(k.float() * sk), _bf16(v.float() * sv), \
        _bf16(dy.float() * sdy)
    h = h * sh
    status = _check(wl, q, k, v, h, dy, elementwise=False)
    if fallback:
        assert status & g.HYENA_DEVICE_F16_RANGE, name
    else:
        assert status == 0, "%s: a range fallback ran (status %d)" % (name, status)


def test_fallback_leaves_the_next_call_on_the_tensor_path():
    """The flag word in the workspace carries the call's token and is never reset: after a call
    that fell back, an ordinary call on the same workspace runs on the tensor path alone and
    matches."""
    wl, q, k, v, h, dy = _inputs(43)
    ws = torch.empty(g.hyena_conv_bwd_workspace_bytes(wl.B, wl.L, wl.D, wl.d_g, wl.l_h),
                     dtype=torch.uint8, device="cuda")
    k2 = k.clone()
    k2[0, 100, 3] = 400.0
    v2 = v.clone()
    v2[0, 100, 3] = 400.0
    for kk, vv, want_fallback in ((k2, v2, True), (k, v, False)):
        g.hyena_device_status(clear=True)
        out = g.hyena_conv_bwd_ex(q, kk, vv, h, dy, wl.d_g, wl.l_b, algo=g.HYENA_ALGO_TENSOR,
                                  workspace=ws)
        torch.cuda.synchronize()
        status = g.hyena_device_status(clear=True)
        assert bool(status & g.HYENA_DEVICE_F16_RANGE) == want_fallback
        ref = oracle.gated_fir_bwd(q, kk, vv, h, dy, wl.d_g)
        for got, want in zip(out[:3], ref[:3]):
            U.assert_parity(got, want, torch.bfloat16)
        assert U.f32_normwise(out[3].cpu().double().numpy(), ref[3]) <= DH_NORMWISE
