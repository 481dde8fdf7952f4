"""FFT path of the forward (``hyena_conv_fwd_fft``, long filters: the Hyena-LI class) vs the
fp64 oracle through the C ABI (needs a B200).

The oracle is the same direct causal sum as for the other kernels: the FFT path reaches it
exactly up to rounding (the cyclic convolution of length >= L + l_h - 1 equals the causal one
for t < L).  Small shapes are checked whole; long ones on sampled rows, each from its own
history window."""
import numpy as np
import pytest
import torch

import gated_causal_fir_b200 as g
from gated_causal_fir_b200.workloads import WORKLOADS, custom, make_inputs
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
    # name, B, L, D, d_g, l_h, dtype
    ("li_small", 2, 1000, 64, 16, 1000, "bf16"),      # l_h = L; N = 2048 (64 x 32)
    ("mr_filter", 1, 777, 128, 64, 128, "bf16"),
    ("filter_past_L", 1, 500, 32, 2, 600, "f32"),
    ("ragged_signals", 3, 2048, 40, 4, 2048, "bf16"),  # 20 channel pairs: a partial block
    ("tiny", 1, 8, 4, 2, 3, "bf16"),                   # the smallest transform, N = 256
    ("single_tap", 2, 300, 64, 8, 1, "f32"),
    ("f32_long", 2, 1500, 64, 32, 1500, "f32"),
    ("n512", 1, 300, 64, 16, 200, "bf16"),            # N = 512: 32 x 16 (R = 4 x 8 / 4 x 4)
    ("n2048", 2, 1500, 32, 8, 500, "bf16"),           # N = 2048: 64 x 32
    ("n32768_odd", 1, 20000, 32, 32, 10000, "f32"),   # N = 32768: 256 x 128
]


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_fft_parity(shape):
    name, B, L, D, d_g, l_h, dtype = shape
    wl = custom(name, B, L, D, d_g, l_h, 64, dtype, "mr", seed=L + l_h)
    q, k, v, h = make_inputs(wl, device="cuda")
    y = g.hyena_conv_fwd_fft(q, k, v, h, d_g, 64)
    torch.cuda.synchronize()
    U.assert_parity(y, oracle.gated_fir(q, k, v, h, d_g), q.dtype)


def test_fft_matches_the_tensor_path_on_mr():
    """Same operation, two methods: the FFT and the block-Toeplitz tensor path agree within the
    tolerance of each other and of the oracle."""
    wl = custom("mr_both", 2, 1500, 256, 64, 128, 64, "bf16", "mr", seed=4)
    q, k, v, h = make_inputs(wl, device="cuda")
    yf = g.hyena_conv_fwd_fft(q, k, v, h, 64, 64)
    yt = g.hyena_conv_fwd_ex(q, k, v, h, 64, 64, algo=g.HYENA_ALGO_TENSOR)
    torch.cuda.synchronize()
    ref = oracle.gated_fir(q, k, v, h, 64)
    U.assert_parity(yf, ref, q.dtype)
    U.assert_parity(yt, ref, q.dtype)


def _sampled_rows(y, q, k, v, h, d_g, rows):
    ref = oracle.gated_fir_rows(q, k, v, h, d_g, rows)
    got = torch.stack([y[b, t] for b, t in rows])
    U.assert_parity(got, ref, q.dtype)


def test_fft_largest_transform_sampled():
    """N = 65536 (256 x 256): L = l_h = 32768, checked on sampled rows incl. the first and
    last."""
    wl = custom("n64k", 1, 32768, 64, 64, 32768, 64, "bf16", "mr", seed=11)
    q, k, v, h = make_inputs(wl, device="cuda")
    y = g.hyena_conv_fwd_fft(q, k, v, h, 64, 64)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = [(0, 0), (0, 1), (0, 255), (0, 256), (0, 32767)] + \
        [(0, int(t)) for t in rng.integers(0, 32768, 12)]
    _sampled_rows(y.cpu(), q.cpu(), k.cpu(), v.cpu(), h.cpu(), 64, rows)


def test_fft_ragged_signal_block_and_split_group_at_the_largest_transform():
    """B = 4 at N = 65536 (256 x 256): D = 80 is 40 channel pairs, two full 16-pair blocks and a
    ragged one of 8, and d_g = 10 puts the group of pairs 15..19 across the first block
    boundary (the pass-2 filter lookup per signal)."""
    wl = custom("ragged", 4, 32768, 80, 10, 32768, 64, "bf16", "mr", seed=12)
    q, k, v, h = make_inputs(wl, device="cuda")
    y = g.hyena_conv_fwd_fft(q, k, v, h, 10, 64)
    torch.cuda.synchronize()
    rows = [(0, 0), (1, 32767), (2, 4097), (3, 20000), (3, 32766)]
    _sampled_rows(y.cpu(), q.cpu(), k.cpu(), v.cpu(), h.cpu(), 10, rows)


def test_fft_li_workload_sampled():
    """The Hyena-LI-shaped workload (B=1, L=8192, D=4096, d_g=64, l_h=8192) on sampled rows."""
    wl = WORKLOADS["li"]
    q, k, v, h = make_inputs(wl, device="cuda")
    y = g.hyena_conv_fwd_fft(q, k, v, h, wl.d_g, wl.l_b)
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    rows = [(0, 0), (0, 127), (0, 8191)] + [(0, int(t)) for t in rng.integers(0, 8192, 8)]
    _sampled_rows(y.cpu(), q.cpu(), k.cpu(), v.cpu(), h.cpu(), wl.d_g, rows)


def test_fft_deterministic_and_workspace_reuse():
    wl = custom("det", 2, 900, 128, 16, 900, 64, "bf16", "mr", seed=9)
    q, k, v, h = make_inputs(wl, device="cuda")
    ws = torch.empty(g.hyena_conv_fwd_fft_workspace_bytes(2, 900, 128, 16, 900),
                     dtype=torch.uint8, device="cuda")
    a = g.hyena_conv_fwd_fft(q, k, v, h, 16, 64, workspace=ws)
    b = g.hyena_conv_fwd_fft(q, k, v, h, 16, 64, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
