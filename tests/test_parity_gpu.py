"""CUDA path vs the fp64 oracle, element by element, through the C ABI (needs a B200).

Sizes are chosen so the oracle finishes in seconds while the kernels see several tiles, ragged
tails, CTA ranges that start inside a sequence, several sequences, and the degenerate cases
(single token, single tap, L shorter than the filter, maximum halo).
"""
import numpy as np
import pytest
import torch

import gated_causal_fir_b200 as g
from gated_causal_fir_b200.workloads import WORKLOADS, custom, make_inputs
from tests import _gpu_util as U
import oracle

pytestmark = pytest.mark.gpu

ALGOS = {"tensor": g.HYENA_ALGO_TENSOR, "window": g.HYENA_ALGO_WINDOW, "direct": g.HYENA_ALGO_DIRECT,
         "fft": g.HYENA_ALGO_FFT}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_causal_fir_b200 import build
    build.build()
    g.hyena_device_status(clear=True)
    yield
    assert g.hyena_device_status(clear=True) == 0, "a kernel raised its device status word"


def _run(q, k, v, h, wl, algo=g.HYENA_ALGO_AUTO):
    y = g.hyena_conv_fwd_ex(q, k, v, h, wl.d_g, wl.l_b, algo=algo)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("name", ["tiny", "se", "mr"])
def test_workload_full(name):
    """The three workloads the oracle takes whole, through the default entry points."""
    wl = WORKLOADS[name]
    q, k, v, h = make_inputs(wl, device="cuda")
    if wl.dtype == "f32":
        y = g.hyena_conv_fwd_f32(q, k, v, h, wl.d_g, wl.l_b)
    else:
        y = g.hyena_conv_fwd(q, k, v, h, wl.d_g, wl.l_b)
    torch.cuda.synchronize()
    ref = U.oracle_full(q, k, v, h, wl.d_g)
    U.assert_parity(y, ref, q.dtype)


SHAPES = [
    # name, B, L, D, d_g, l_h, l_b, dtype
    ("mr_ragged", 2, 1000, 256, 64, 128, 64, "bf16"),
    ("mr_multiseg", 3, 3000, 512, 64, 100, 64, "bf16"),
    ("short_seq", 1, 77, 128, 64, 128, 64, "bf16"),
    ("single_token", 1, 1, 64, 64, 7, 16, "bf16"),
    ("single_tap", 2, 513, 256, 64, 1, 1, "bf16"),
    ("max_halo", 1, 4100, 128, 64, 129, 65, "bf16"),
    ("halo_16", 2, 700, 192, 64, 17, 16, "bf16"),
    ("se_like", 2, 777, 512, 16, 7, 16, "bf16"),
    ("dg32", 1, 300, 96, 32, 16, 8, "bf16"),
    ("dg32_tc", 2, 1100, 256, 32, 40, 32, "bf16"),
    ("dg16_lh65", 1, 900, 128, 16, 65, 64, "bf16"),
    ("dg16_multiseg", 3, 2000, 512, 16, 7, 16, "bf16"),
    ("dg4", 1, 200, 60, 4, 5, 3, "bf16"),
    ("dg3_odd", 1, 300, 30, 3, 4, 2, "bf16"),
    ("long_filter", 1, 600, 128, 64, 200, 100, "bf16"),
    # filters past 2 l_b (the general block form; 2 to 4 earlier tiles feed each output tile)
    ("lh256_lb64", 2, 1500, 256, 64, 256, 64, "bf16"),
    ("lh385_ragged", 1, 2000, 128, 64, 385, 64, "bf16"),
    ("lh513_ragged", 2, 1700, 128, 64, 513, 32, "bf16"),
    ("lh300_multiseg", 3, 1100, 512, 64, 300, 64, "bf16"),
    ("lh513_short_runs", 1, 19200, 128, 64, 513, 64, "bf16"),
    ("lh514_ragged", 2, 1700, 128, 64, 514, 64, "bf16"),     # five history tiles
    ("lh641_runs", 1, 19200, 128, 64, 641, 64, "bf16"),
    ("lh400_L77", 1, 77, 128, 64, 400, 64, "bf16"),
    ("dg32_lh257", 1, 900, 128, 32, 257, 64, "bf16"),
    ("dg32_lh200_multiseg", 2, 3000, 256, 32, 200, 16, "bf16"),
    ("lh600_direct", 1, 400, 64, 64, 600, 64, "bf16"),
    ("f32_long", 1, 500, 64, 16, 300, 8, "f32"),
    ("f32_tiny_like", 2, 1000, 64, 16, 7, 16, "f32"),
    ("f32_mr_like", 1, 500, 128, 64, 128, 64, "f32"),
    ("f32_dg2", 1, 300, 10, 2, 3, 2, "f32"),
]


def _tensor_fits(D, d_g, l_h):
    """The tensor kernel's plan: 64-channel tiles of 64 / d_g groups, one Toeplitz band of
    (128 + halo) / 2 TMEM columns per group, next to 128 accumulator columns (512 in all);
    at most 4 earlier 128-row tiles of history (halo <= 512)."""
    if d_g not in (16, 32, 64) or D % 64 or l_h > 641:
        return False
    halo = (l_h - 1 + 15) // 16 * 16
    return (64 // d_g) * (128 + halo) // 2 <= 384


def _supported(algo, B, L, D, d_g, l_h, l_b, dtype):
    if algo == "direct":
        return True
    if algo == "fft":
        return U.fftblk_plan(L, D, d_g, l_h, dtype) is not None
    if algo == "tensor":
        return dtype == "bf16" and _tensor_fits(D, d_g, l_h)
    return l_h <= 16 and d_g % (4 if dtype == "f32" else 8) == 0


@pytest.mark.parametrize("algo", sorted(ALGOS))
@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_algorithm_parity(shape, algo):
    name, B, L, D, d_g, l_h, l_b, dtype = shape
    if not _supported(algo, B, L, D, d_g, l_h, l_b, dtype):
        pytest.skip("%s does not run %s" % (algo, name))
    wl = custom(name, B, L, D, d_g, l_h, l_b, dtype, "mr" if l_h > 16 else "se", seed=L + D)
    q, k, v, h = make_inputs(wl, device="cuda")
    y = _run(q, k, v, h, wl, ALGOS[algo])
    ref = U.oracle_full(q, k, v, h, d_g)
    U.assert_parity(y, ref, q.dtype)


def test_auto_matches_forced():
    """AUTO runs the same kernel as the algorithm hyena_select_algo names: identical bits."""
    wl = custom("auto", 2, 1000, 256, 64, 128, 64, "bf16", "mr", seed=5)
    q, k, v, h = make_inputs(wl, device="cuda")
    algo = g.hyena_select_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b)
    assert algo == g.HYENA_ALGO_TENSOR
    assert torch.equal(_run(q, k, v, h, wl), _run(q, k, v, h, wl, algo))


def test_deterministic():
    wl = custom("det", 2, 2000, 512, 64, 128, 64, "bf16", "mr", seed=6)
    q, k, v, h = make_inputs(wl, device="cuda")
    for algo in (g.HYENA_ALGO_TENSOR, g.HYENA_ALGO_DIRECT):
        a = _run(q, k, v, h, wl, algo)
        b = _run(q, k, v, h, wl, algo)
        assert torch.equal(a, b)


def test_batch_zero_history():
    """Every sequence starts from zero history: sequence b alone gives the same rows."""
    wl = custom("zh", 3, 640, 128, 64, 128, 64, "bf16", "mr", seed=8)
    q, k, v, h = make_inputs(wl, device="cuda")
    y = _run(q, k, v, h, wl)
    for b in range(3):
        yb = g.hyena_conv_fwd(q[b:b + 1].contiguous(), k[b:b + 1].contiguous(),
                              v[b:b + 1].contiguous(), h, wl.d_g, wl.l_b)
        torch.cuda.synchronize()
        assert torch.equal(y[b:b + 1], yb)


def test_misaligned_views_use_a_general_kernel():
    """Tensors offset by one element (2-byte aligned only) still give oracle results."""
    wl = custom("mis", 1, 300, 128, 64, 64, 64, "bf16", "mr", seed=9)
    q, k, v, h = make_inputs(wl, device="cuda")
    n = q.numel()
    bufs = [torch.empty(n + 1, dtype=q.dtype, device="cuda") for _ in range(4)]
    views = [b[1:].view(q.shape) for b in bufs]
    for src, dst in zip((q, k, v), views[:3]):
        dst.copy_(src)
    y = g.hyena_conv_fwd(views[0], views[1], views[2], h, wl.d_g, wl.l_b, y=views[3])
    torch.cuda.synchronize()
    U.assert_parity(y, U.oracle_full(q, k, v, h, wl.d_g), q.dtype)


def test_side_stream():
    wl = custom("stream", 1, 1500, 256, 64, 128, 64, "bf16", "mr", seed=10)
    q, k, v, h = make_inputs(wl, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        y = g.hyena_conv_fwd(q, k, v, h, wl.d_g, wl.l_b)
    s.synchronize()
    U.assert_parity(y, U.oracle_full(q, k, v, h, wl.d_g), q.dtype)


@pytest.mark.parametrize("l_h,l_b", [(4, 3), (7, 16), (65, 64), (128, 64), (1, 1), (16, 8)])
def test_toeplitz_builder(l_h, l_b):
    G = 3
    h = torch.randn(G, l_h, generator=torch.Generator().manual_seed(l_h)).cuda()
    H0, H1, H2 = g.hyena_build_toeplitz(h, l_b)
    torch.cuda.synchronize()
    for gi in range(G):
        ref = oracle.toeplitz_blocks(h[gi].cpu(), l_b, 3)
        for m, Hm in enumerate((H0, H1, H2)):
            assert np.array_equal(Hm[gi].cpu().double().numpy(), ref[m]), (gi, m)


@pytest.mark.parametrize("l_h,l_b,S", [(4, 3, None), (128, 64, None), (300, 64, None),
                                       (513, 32, None), (9, 4, 5), (200, 100, 1)])
def test_toeplitz_blocks_builder(l_h, l_b, S):
    """All sub-block diagonals of any filter length, against the oracle's decomposition."""
    G = 3
    h = torch.randn(G, l_h, generator=torch.Generator().manual_seed(l_h + 1)).cuda()
    Hm = g.hyena_build_toeplitz_blocks(h, l_b, S)
    torch.cuda.synchronize()
    S = oracle.stages_needed(l_h, l_b) if S is None else S
    assert Hm.shape == (S, G, l_b, l_b)
    for gi in range(G):
        ref = oracle.toeplitz_blocks(h[gi].cpu(), l_b, S)
        assert np.array_equal(Hm[:, gi].cpu().double().numpy(), ref), gi


@pytest.mark.parametrize("shape", [
    # name, B, L, D, d_g, l_h
    ("int_lh200", 2, 1300, 256, 64, 200),
    ("int_lh385", 1, 2100, 128, 64, 385),
    ("int_lh513", 3, 900, 128, 64, 513),
    ("int_lh513_runs", 1, 19200, 128, 64, 513),
    ("int_lh641", 2, 1500, 128, 64, 641),            # five history tiles, two k/v stages
    ("int_lh600_runs", 1, 19200, 128, 64, 600),
    ("int_dg32_lh250", 2, 1000, 128, 32, 250),
], ids=lambda s: s[0])
def test_long_filter_integer_exact(shape):
    """Integer inputs make every fp16 operand, product and fp32 partial sum exact, so the tensor
    path must give the oracle's result rounded once to bf16, bit for bit: any tap applied to
    the wrong row (a history tile or slot off by one) changes an output."""
    from gated_causal_fir_b200.workloads import make_integer_inputs
    name, B, L, D, d_g, l_h = shape
    wl = custom(name, B, L, D, d_g, l_h, 64, "bf16", "mr", seed=l_h)
    q, k, v, _, h = make_integer_inputs(wl, device="cuda")
    y = _run(q, k, v, h, wl, g.HYENA_ALGO_TENSOR)
    ref = torch.from_numpy(U.oracle_full(q, k, v, h, d_g)).to(torch.bfloat16)
    assert torch.equal(y.cpu(), ref)


def test_std_reading_of_filter_variance():
    """The filter recipe read with the second N() argument as a standard deviation (smaller
    |y|) also passes; the variance reading is the default everywhere else."""
    wl = WORKLOADS["mr"]
    q, k, v, h = make_inputs(wl, device="cuda")
    h = h * (wl.l_h ** -0.25) / (wl.l_h ** -0.5) ** 0.5  # std l_h^-1/2 instead of l_h^-1/4
    y = g.hyena_conv_fwd(q, k, v, h.contiguous(), wl.d_g, wl.l_b)
    torch.cuda.synchronize()
    U.assert_parity(y, U.oracle_full(q, k, v, h, wl.d_g), q.dtype)


def _sampled(wl, n_random, l_slice=0):
    q, k, v, h = make_inputs(wl, device="cuda", l_slice=l_slice)
    y = g.hyena_conv_fwd(q, k, v, h, wl.d_g, wl.l_b)
    torch.cuda.synchronize()
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    seams = U.tc_cta_seam_rows(wl.B, wl.L, wl.D, wl.d_g, sm)
    rng = np.random.default_rng(wl.seed)
    seam_rows = [s[2] for s in seams[:: max(1, len(seams) // 6)]]
    worst = 0.0
    hh = h.cpu()
    for b in sorted(set([0, wl.B - 1] + list(rng.integers(0, wl.B, 2)))):
        for t0 in U.sample_chunks(wl.L, wl.l_b, n_random // max(1, wl.B // 2), wl.seed + b,
                                  seam_rows):
            t1 = min(wl.L, t0 + wl.l_b)
            s = max(0, t0 - (wl.l_h - 1))
            win = [x[b:b + 1, s:t1].cpu() for x in (q, k, v)]
            ref = oracle.gated_fir(win[0][0], win[1][0], win[2][0], hh, wl.d_g)[t0 - s:]
            worst = max(worst, U.bf16_ratio(y[b, t0:t1], ref))
    assert worst <= 1.0, "bf16 error/bound ratio %.3f" % worst
    del q, k, v, y
    torch.cuda.empty_cache()


def test_mr_batched_sampled():
    _sampled(WORKLOADS["mr_batched"], 64)


def test_mr_1m_sampled():
    """L = 2^20, D = 4096: 2^32 elements per tensor (64-bit offsets), 64 random chunks plus the
    first chunks, the tail and CTA-range seams."""
    free, _ = torch.cuda.mem_get_info()
    if free < 40 * (1 << 30):
        pytest.skip("needs ~40 GiB free device memory")
    _sampled(WORKLOADS["mr_1m"], 64, l_slice=1 << 16)


HOST_CASES = [
    # name, B, L, D, d_g, l_h, l_b, dtype, chunk, pinned
    ("mr_chunks", 2, 1000, 128, 64, 128, 64, "bf16", 300, True),
    ("mr_one_chunk", 2, 1000, 128, 64, 128, 64, "bf16", 2048, True),
    ("f32_ragged", 3, 777, 96, 32, 33, 32, "f32", 250, True),
    ("se_window", 1, 5000, 256, 16, 7, 16, "bf16", 1024, True),
    ("chunk_shorter_than_halo", 1, 400, 64, 64, 100, 64, "bf16", 40, True),
    ("pageable", 2, 600, 128, 64, 64, 64, "bf16", 256, False),
]


@pytest.mark.parametrize("case", HOST_CASES, ids=[c[0] for c in HOST_CASES])
def test_from_host_pipeline(case):
    """Host tensors in, host tensor out through the C entry point: sequence chunks with l_h - 1
    history rows each, copies overlapped with compute over three rotating device slots; the
    result matches the oracle like the device path, and a second call (slots and events
    reused) gives the same bits."""
    name, B, L, D, d_g, l_h, l_b, dt, chunk, pinned = case
    wl = custom(name, B, L, D, d_g, l_h, l_b, dt, "mr" if l_h > 16 else "se", seed=12)
    q, k, v, h = (x.cpu() for x in make_inputs(wl, device="cuda"))
    qh, kh, vh = (x.pin_memory() for x in (q, k, v)) if pinned else (q, k, v)
    out = None if pinned else torch.empty_like(q)
    y = g.hyena_conv_fwd_from_host(qh, kh, vh, h, wl.d_g, wl.l_b, chunk=chunk, out=out)
    torch.cuda.synchronize()
    U.assert_parity(y, U.oracle_full(q, k, v, h, wl.d_g), q.dtype)
    y2 = g.hyena_conv_fwd_from_host(qh, kh, vh, h, wl.d_g, wl.l_b, chunk=chunk)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    assert g.hyena_device_status(clear=True) == 0
