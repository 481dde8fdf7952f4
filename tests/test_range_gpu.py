"""Operands outside fp16's range on the tensor-core forward, against the fp64 oracle (needs a
B200).

The tensor path rounds x = k v and the filter taps to fp16 for the MMA.  It scales the taps of
each group, and x of each sequence run, by powers of two (exact), and recomputes in fp32 on the
CUDA cores any tile whose scaled operands still leave fp16's range; that raises
HYENA_DEVICE_F16_RANGE, which these tests read to see which mechanism ran.  Every case must
match the oracle under the bf16 bound |y - y_ref| <= 1e-2 + 1e-2 |y_ref| elementwise, and the
cases whose values would otherwise sit in fp16's subnormals or beyond its largest value also
normwise: max |y - y_ref| / max |y_ref| <= 2^-8.  Rounding y to bf16 alone costs up to 2^-9
of the largest element, and fp16 operands with fp32 accumulation add well under that again;
taps or products held as fp16 subnormals (relative spacing up to 1) or saturated at 65504
would miss this bound by far.
"""
import numpy as np
import pytest
import torch

import gated_causal_fir_b200 as g
from gated_causal_fir_b200.workloads import custom, make_inputs
from tests import _gpu_util as U
import oracle

pytestmark = pytest.mark.gpu

NORMWISE = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_causal_fir_b200 import build
    build.build()
    g.hyena_device_status(clear=True)
    yield
    assert g.hyena_device_status(clear=True) == 0, "a kernel raised its device status word"


def _bf16(x):
    return x.to(torch.bfloat16)


def _tensor_fwd(q, k, v, h, wl):
    y = g.hyena_conv_fwd_ex(q, k, v, h, wl.d_g, wl.l_b, algo=g.HYENA_ALGO_TENSOR)
    torch.cuda.synchronize()
    return y


def _check(y, ref, normwise=True):
    U.assert_parity(y, ref, torch.bfloat16)
    if normwise:
        r = U.f32_normwise(y, ref)
        assert r <= NORMWISE, "normwise error %.2e > %.2e" % (r, NORMWISE)


def _auto_matches(q, k, v, h, wl, ref):
    """The default entry point takes the same path (AUTO picks the tensor kernel here)."""
    assert g.hyena_select_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b) == g.HYENA_ALGO_TENSOR
    y = g.hyena_conv_fwd(q, k, v, h, wl.d_g, wl.l_b)
    torch.cuda.synchronize()
    U.assert_parity(y, ref, torch.bfloat16)


def test_kv_outlier_in_a_runs_first_tile():
    """|k v| = 160000 > 65504 in the first tile: the run's scale takes it in, no recomputation."""
    wl = custom("outlier_first", 1, 256, 64, 64, 8, 8, "bf16", "se", seed=11)
    q, k, v, h = make_inputs(wl, device="cuda")
    k[0, 100, 5] = 400.0
    v[0, 100, 5] = 400.0
    assert g.hyena_device_status(clear=True) == 0
    y = _tensor_fwd(q, k, v, h, wl)
    assert g.hyena_device_status(clear=True) == 0, "first-tile outlier should need no fallback"
    ref = U.oracle_full(q, k, v, h, wl.d_g)
    _check(y, ref)
    _auto_matches(q, k, v, h, wl, ref)
    assert g.hyena_device_status(clear=True) == 0
    # the CUDA-core kernels agree as well (fp32 throughout)
    y2 = g.hyena_conv_fwd_ex(q, k, v, h, wl.d_g, wl.l_b, algo=g.HYENA_ALGO_WINDOW)
    torch.cuda.synchronize()
    U.assert_parity(y2, ref, torch.bfloat16)


@pytest.mark.parametrize("shape", [
    # name, B, L, D, d_g, l_h, outlier rows
    ("mr", 2, 2048, 128, 64, 128, [(0, 1000, 5), (1, 1500, 70)]),
    ("lh300", 1, 1500, 64, 64, 300, [(0, 700, 9)]),
    ("dg16", 1, 1200, 128, 16, 40, [(0, 600, 17)]),
    ("dg32_tail", 1, 1000, 128, 32, 100, [(0, 999, 100)]),
], ids=lambda s: s[0])
def test_kv_outlier_later_in_a_run(shape):
    """|k v| = 160000 in a later tile of a run: the tiles that read it are recomputed in fp32
    (HYENA_DEVICE_F16_RANGE), the rest stay on tensor cores, and every output matches."""
    name, B, L, D, d_g, l_h, rows = shape
    wl = custom(name, B, L, D, d_g, l_h, 64, "bf16", "mr", seed=21)
    q, k, v, h = make_inputs(wl, device="cuda")
    for b, t, c in rows:
        k[b, t, c] = 400.0
        v[b, t, c] = -400.0
    assert g.hyena_device_status(clear=True) == 0
    y = _tensor_fwd(q, k, v, h, wl)
    assert g.hyena_device_status(clear=True) & g.HYENA_DEVICE_F16_RANGE
    ref = U.oracle_full(q, k, v, h, wl.d_g)
    _check(y, ref)
    _auto_matches(q, k, v, h, wl, ref)
    g.hyena_device_status(clear=True)


@pytest.mark.parametrize("scale_k,scale_v,scale_q", [
    (2.0 ** 8, 2.0 ** 8, 2.0 ** -16),      # |k v| ~ 2^16, beyond fp16's 65504 everywhere
    (2.0 ** -12, 2.0 ** -12, 2.0 ** 24),   # |k v| ~ 2^-24: fp16's smallest subnormal
    (2.0 ** -30, 2.0 ** -20, 2.0 ** 50),   # far below fp16 altogether (run scale 2^55)
], ids=["huge", "subnormal", "far_below"])
def test_kv_scaled_globally(scale_k, scale_v, scale_q):
    """k and v scaled by powers of two (q scaled back, so y keeps its size): the run scales
    absorb it on tensor cores (no fp32 recomputation), and the result agrees with the unscaled
    problem's to well within the bound (only values in fp16's subnormal range may round
    differently)."""
    wl = custom("kv_scaled", 2, 1100, 128, 64, 128, 64, "bf16", "mr", seed=31)
    q, k, v, h = make_inputs(wl, device="cuda")
    qs, ks, vs = _bf16(q.float() * scale_q), _bf16(k.float() * scale_k), _bf16(v.float() * scale_v)
    assert g.hyena_device_status(clear=True) == 0
    y = _tensor_fwd(qs, ks, vs, h, wl)
    assert g.hyena_device_status(clear=True) == 0
    ref = U.oracle_full(qs, ks, vs, h, wl.d_g)
    _check(y, ref)
    y0 = _tensor_fwd(q, k, v, h, wl)
    assert U.f32_normwise(y, y0.double().cpu().numpy()) <= NORMWISE


@pytest.mark.parametrize("scale_h", [2.0 ** -20, 2.0 ** 17, 2.0 ** -40],
                         ids=["tiny", "huge", "far_below"])
def test_taps_scaled_globally(scale_h):
    """Filter taps scaled by powers of two (2^-20: the decayed MR taps fall below fp16's normal
    range; 2^17: beyond 65504): the per-group tap scale absorbs it, normwise 2^-8 against the
    oracle, and elementwise with q scaled back."""
    wl = custom("h_scaled", 1, 1500, 128, 64, 128, 64, "bf16", "mr", seed=41)
    q, k, v, h = make_inputs(wl, device="cuda")
    hs = h * scale_h
    qs = _bf16(q.float() / scale_h) if 2.0 ** -126 < 1.0 / scale_h < 2.0 ** 127 else q
    assert g.hyena_device_status(clear=True) == 0
    y = _tensor_fwd(qs, k, v, hs, wl)
    assert g.hyena_device_status(clear=True) == 0, "a tap scale should need no fallback"
    ref = U.oracle_full(qs, k, v, hs, wl.d_g)
    _check(y, ref)


def test_kv_beyond_the_run_scale_range():
    """|k v| ~ 2^-100: beyond what a run's scale reaches (2^60), so every tile is recomputed in
    fp32 on the CUDA cores; still every output matches."""
    wl = custom("kv_far", 1, 700, 128, 64, 128, 64, "bf16", "mr", seed=32)
    q, k, v, h = make_inputs(wl, device="cuda")
    qs = _bf16(q.float() * 2.0 ** 100)
    ks, vs = _bf16(k.float() * 2.0 ** -60), _bf16(v.float() * 2.0 ** -40)
    assert g.hyena_device_status(clear=True) == 0
    y = _tensor_fwd(qs, ks, vs, h, wl)
    assert g.hyena_device_status(clear=True) & g.HYENA_DEVICE_F16_RANGE
    _check(y, U.oracle_full(qs, ks, vs, h, wl.d_g))


def test_taps_with_wide_dynamic_range():
    """A steeply decayed filter (taps from ~1 down to ~1e-11 within each group): the small taps
    stay normal fp16 after the group's scale down to 2^-14 of the largest; normwise 2^-8."""
    wl = custom("decay", 1, 1000, 128, 64, 128, 64, "bf16", "mr", seed=51)
    q, k, v, h = make_inputs(wl, device="cuda")
    t = torch.arange(wl.l_h, device="cuda", dtype=torch.float32)
    hs = (h * torch.exp(-0.2 * t)).contiguous()
    y = _tensor_fwd(q, k, v, hs, wl)
    _check(y, U.oracle_full(q, k, v, hs, wl.d_g))
    assert g.hyena_device_status(clear=True) == 0


def test_tiny_rows_after_a_normal_first_tile():
    """After a normal first tile, rows 2^-30 smaller (q 2^30 larger): those warps' values would
    be fp16 subnormals, so their tiles are recomputed in fp32; every output matches."""
    wl = custom("tiny_rows", 1, 1024, 64, 64, 64, 64, "bf16", "mr", seed=61)
    q, k, v, h = make_inputs(wl, device="cuda")
    k[:, 300:700] = _bf16(k[:, 300:700].float() * 2.0 ** -15)
    v[:, 300:700] = _bf16(v[:, 300:700].float() * 2.0 ** -15)
    q[:, 300:700] = _bf16(q[:, 300:700].float() * 2.0 ** 30)
    assert g.hyena_device_status(clear=True) == 0
    y = _tensor_fwd(q, k, v, h, wl)
    assert g.hyena_device_status(clear=True) & g.HYENA_DEVICE_F16_RANGE
    U.assert_parity(y, U.oracle_full(q, k, v, h, wl.d_g), torch.bfloat16)
    g.hyena_device_status(clear=True)


def test_outlier_with_history_rows():
    """The fp32 recomputation of a tile reads the rows before the shard from the history
    tensors (hyena_conv_fwd_hist): an outlier in the shard's first tile, after a normal history
    tile, sends that tile to it."""
    wl = custom("hist_outlier", 2, 512, 128, 64, 128, 64, "bf16", "mr", seed=71)
    q, k, v, h = make_inputs(wl, device="cuda")
    hw = custom("hist_rows", 2, 200, 128, 64, 128, 64, "bf16", "mr", seed=72)
    _, kh, vh, _ = make_inputs(hw, device="cuda")
    k[:, 5, 3] = 400.0
    v[:, 5, 3] = 400.0
    assert g.hyena_device_status(clear=True) == 0
    y = g.hyena_conv_fwd_hist(q, k, v, h, wl.d_g, wl.l_b, kh, vh, algo=g.HYENA_ALGO_TENSOR)
    torch.cuda.synchronize()
    assert g.hyena_device_status(clear=True) & g.HYENA_DEVICE_F16_RANGE
    pad = torch.zeros_like(kh)
    ref = oracle.gated_fir(torch.cat([pad, q], 1), torch.cat([kh, k], 1), torch.cat([vh, v], 1),
                           h, wl.d_g)[:, kh.shape[1]:]
    U.assert_parity(y, np.ascontiguousarray(ref), torch.bfloat16)
    g.hyena_device_status(clear=True)
