"""Single-pass block FFT forward (HYENA_ALGO_FFT: overlap-save blocks, no workspace) against
the fp64 oracle through the C ABI (needs a B200).

The oracle is the direct causal sum: the block FFT reaches it exactly up to rounding, because
the length-N cyclic convolution of a block's N input rows with the zero-padded filter equals the
causal sum at the block's last N - l_h + 1 rows.  The shapes cover every transform length
(N = 1024 .. 8192, so 8, 4, 2 and 1 channel pairs per CTA), blocks that end past L, filters as
long as the transform allows, several groups and sequences per CTA range, fp32 I/O, history rows
and the shapes AUTO now sends to this kernel."""
import pytest
import torch

import gated_causal_fir_b200 as g
from gated_causal_fir_b200.workloads import custom, make_inputs
from tests import _gpu_util as U
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_causal_fir_b200 import build
    build.build()
    g.hyena_device_status(clear=True)
    yield
    assert g.hyena_device_status(clear=True) == 0, "a kernel raised its device status word"


SHAPES = [
    # name, B, L, D, d_g, l_h, dtype; the transform length the plan picks in the comment
    ("n1024_lh17", 2, 3000, 128, 64, 17, "bf16"),        # 1024, 3 blocks, 8 pairs per CTA
    ("n1024_lh300", 1, 2500, 256, 16, 300, "bf16"),      # 1024
    ("n2048_lh514", 1, 3000, 256, 64, 514, "bf16"),      # forced: the tensor path takes it too
    ("n2048_lh1000_ragged", 3, 1777, 64, 8, 1000, "bf16"),   # 2048 (4 pairs: d_g = 8)
    ("n4096_lh1500", 1, 5000, 32, 4, 1500, "bf16"),      # 4096 (2 pairs: d_g = 4)
    ("n4096_lh2049", 2, 4000, 64, 32, 2049, "bf16"),
    ("n8192_lh4000", 1, 9000, 16, 2, 4000, "bf16"),      # 8192, one pair per CTA
    ("n8192_lh7000", 1, 1100, 16, 16, 7000, "bf16"),     # 8192, one block covers L
    ("lh_equals_L", 2, 1024, 64, 16, 1024, "bf16"),
    ("single_row", 1, 1, 64, 64, 600, "bf16"),
    ("short_seq", 3, 50, 128, 32, 40, "bf16"),
    ("single_tap", 1, 2000, 64, 16, 1, "bf16"),          # forced: N = 1024, M = 1024
    ("many_groups", 2, 2100, 512, 16, 200, "bf16"),      # ranges that cross groups and sequences
    ("f32_lh700", 1, 2500, 64, 8, 700, "f32"),
    ("f32_lh128_dg64", 2, 1500, 128, 64, 128, "f32"),
    ("f32_dg2", 1, 1300, 10, 2, 40, "f32"),              # 8192 with 10 channels (5 pairs)
]


def _run(q, k, v, h, d_g, algo=g.HYENA_ALGO_FFT):
    y = g.hyena_conv_fwd_ex(q, k, v, h, d_g, 64, algo=algo)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_fftblk_parity(shape):
    name, B, L, D, d_g, l_h, dtype = shape
    assert U.fftblk_plan(L, D, d_g, l_h, dtype) is not None, name
    wl = custom(name, B, L, D, d_g, l_h, 64, dtype, "mr", seed=L + l_h + D)
    q, k, v, h = make_inputs(wl, device="cuda")
    y = _run(q, k, v, h, d_g)
    U.assert_parity(y, U.oracle_full(q, k, v, h, d_g), q.dtype)


def test_fftblk_unsupported_shapes():
    """Odd group sizes and filters whose blocks would keep too few rows are refused, with
    nothing queued: AUTO then runs the direct sum."""
    wl = custom("odd_groups", 1, 300, 30, 3, 40, 64, "bf16", "mr", seed=3)
    q, k, v, h = make_inputs(wl, device="cuda")
    with pytest.raises(g.HyenaError):
        g.hyena_conv_fwd_ex(q, k, v, h, 3, 64, algo=g.HYENA_ALGO_FFT)
    assert U.fftblk_plan(20000, 64, 64, 8000) is None  # 8192-point blocks of 193 rows
    assert g.hyena_select_algo(1, 20000, 64, 64, 8000, 64) == g.HYENA_ALGO_DIRECT


def test_fftblk_bwd_is_refused():
    """HYENA_ALGO_FFT is forward only."""
    wl = custom("bwd", 1, 300, 64, 64, 40, 64, "bf16", "mr", seed=4)
    q, k, v, h = make_inputs(wl, device="cuda")
    with pytest.raises(g.HyenaError):
        g.hyena_conv_bwd_ex(q, k, v, h, torch.ones_like(q), 64, 64, algo=g.HYENA_ALGO_FFT)


def test_fftblk_history():
    """Rows before row 0 from the history tensors (sequence sharding), against the oracle run
    on history and shard together."""
    B, L, Lh, D, d_g, l_h = 2, 1500, 900, 64, 16, 700
    wl = custom("hist", B, L + Lh, D, d_g, l_h, 64, "bf16", "mr", seed=17)
    q, k, v, h = make_inputs(wl, device="cuda")
    qs, ks, vs = (t[:, Lh:].contiguous() for t in (q, k, v))
    kh, vh = k[:, :Lh].contiguous(), v[:, :Lh].contiguous()
    y = g.hyena_conv_fwd_hist(qs, ks, vs, h, d_g, 64, kh, vh, algo=g.HYENA_ALGO_FFT)
    torch.cuda.synchronize()
    ref = U.oracle_full(q, k, v, h, d_g)[:, Lh:]
    U.assert_parity(y, ref, q.dtype)


def test_fftblk_deterministic_and_auto():
    """The MR shape with l_h = 700 (past the tensor band): AUTO picks the block FFT, runs it
    bit for bit like the forced call, and repeats bit for bit; sampled rows against the
    oracle."""
    wl = custom("mr700", 1, 8192, 4096, 64, 700, 64, "bf16", "mr", seed=19)
    assert g.hyena_select_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b) == g.HYENA_ALGO_FFT
    q, k, v, h = make_inputs(wl, device="cuda")
    a = _run(q, k, v, h, 64, g.HYENA_ALGO_AUTO)
    b = _run(q, k, v, h, 64)
    assert torch.equal(a, b)
    assert torch.equal(a, _run(q, k, v, h, 64))
    # 4096-point blocks of 3397 rows
    rows = [(0, t) for t in (0, 1, 698, 699, 3396, 3397, 3398, 6793, 6794, 8191)]
    ref = oracle.gated_fir_rows(q, k, v, h, 64, rows)
    U.assert_parity(torch.stack([a[bb, t] for bb, t in rows]), ref, q.dtype)
