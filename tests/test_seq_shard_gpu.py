"""Forward with given history rows (``hyena_conv_fwd_hist``): one shard of longer sequences,
the compute side of sequence sharding.  CUDA path vs the fp64 oracle through the C ABI (needs a
B200).

The oracle side composes the definition with history the plain way: the oracle over the history
rows followed by the shard's rows (zero before them), keeping the shard's rows.  The shards of
one GPU run one after the other, each taking its history from the previous shard's inputs, as
the ranks of a sequence-sharded job do after their halo exchange."""
import numpy as np
import pytest
import torch

import gated_causal_fir_b200 as g
from gated_causal_fir_b200.workloads import custom, make_inputs, make_integer_inputs
from tests import _gpu_util as U
import oracle

pytestmark = pytest.mark.gpu

ALGOS = {"tensor": g.HYENA_ALGO_TENSOR, "window": g.HYENA_ALGO_WINDOW,
         "direct": g.HYENA_ALGO_DIRECT, "fft": g.HYENA_ALGO_FFT}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_causal_fir_b200 import build
    build.build()
    g.hyena_device_status(clear=True)
    yield
    assert g.hyena_device_status(clear=True) == 0, "a kernel raised its device status word"


def _oracle_with_history(q, k, v, h, d_g, kh, vh):
    Lh = kh.shape[1]
    pad = torch.zeros_like(kh)
    ref = oracle.gated_fir(torch.cat([pad, q], 1), torch.cat([kh, k], 1), torch.cat([vh, v], 1),
                           h, d_g)
    return ref[:, Lh:]


CASES = [
    # name, B, L, L_hist, D, d_g, l_h, dtype
    ("mr_full_hist", 2, 700, 127, 256, 64, 128, "bf16"),
    ("mr_long_hist", 1, 400, 300, 128, 64, 128, "bf16"),     # only the last 127 rows count
    ("mr_short_hist", 2, 520, 40, 128, 64, 128, "bf16"),     # zero before the 40 rows
    ("lh300_hist", 1, 900, 299, 128, 64, 300, "bf16"),       # 3 history tiles
    ("lh513_hist", 2, 300, 700, 128, 64, 513, "bf16"),       # 4 history tiles, L < l_h
    ("lh600_hist", 1, 900, 650, 128, 64, 600, "bf16"),       # 5 history tiles
    ("se_hist", 2, 777, 6, 512, 16, 7, "bf16"),
    ("se_hist_1row", 1, 300, 1, 128, 16, 7, "bf16"),
    ("dg32_hist", 1, 640, 60, 128, 32, 40, "bf16"),
    ("f32_tiny_hist", 2, 500, 6, 64, 16, 7, "f32"),
    ("f32_mr_hist", 1, 300, 127, 128, 64, 128, "f32"),
    ("odd_dg3", 1, 200, 5, 30, 3, 4, "bf16"),
]


def _supported(algo, D, d_g, l_h, dtype, L):
    if algo == "direct":
        return True
    if algo == "fft":
        return U.fftblk_plan(L, D, d_g, l_h, dtype) is not None
    if algo == "tensor":
        if dtype != "bf16" or d_g not in (16, 32, 64) or D % 64 or l_h > 641:
            return False
        halo = (l_h - 1 + 15) // 16 * 16
        return (64 // d_g) * (128 + halo) // 2 <= 384
    return l_h <= 16 and d_g % (4 if dtype == "f32" else 8) == 0


@pytest.mark.parametrize("algo", sorted(ALGOS))
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_history_parity(case, algo):
    name, B, L, Lh, D, d_g, l_h, dtype = case
    if not _supported(algo, D, d_g, l_h, dtype, L):
        pytest.skip("%s does not run %s" % (algo, name))
    wl = custom(name, B, L + Lh, D, d_g, l_h, 64, dtype, "mr" if l_h > 16 else "se",
                seed=L + Lh)
    q, k, v, h = make_inputs(wl, device="cuda")
    qs, ks, vs = (t[:, Lh:].contiguous() for t in (q, k, v))
    kh, vh = k[:, :Lh].contiguous(), v[:, :Lh].contiguous()
    y = g.hyena_conv_fwd_hist(qs, ks, vs, h, d_g, 64, kh, vh, algo=ALGOS[algo])
    torch.cuda.synchronize()
    U.assert_parity(y, _oracle_with_history(qs, ks, vs, h, d_g, kh, vh), q.dtype)


@pytest.mark.parametrize("algo", sorted(ALGOS))
@pytest.mark.parametrize("bounds", [(0, 1024, 2048, 3072), (0, 640, 1000, 3072)],
                         ids=["aligned", "ragged"])
def test_shards_compose_to_the_whole_sequence(algo, bounds):
    """Pieces [b_r, b_{r+1}) of two sequences, each run with the previous piece's last l_h - 1
    rows as history, equal the whole-sequence forward: bit for bit where the pieces start on the
    tensor kernel's 128-row tiles (same products in the same order), within the tolerance
    otherwise.  The block FFT cuts its blocks where each piece starts, so its pieces agree with
    the whole within the tolerance only."""
    l_h = 128 if algo != "window" else 7
    d_g = 64 if algo != "window" else 16
    wl = custom("shards", 2, bounds[-1], 256, d_g, l_h, 64, "bf16", "mr", seed=3)
    q, k, v, h = make_inputs(wl, device="cuda")
    whole = g.hyena_conv_fwd_ex(q, k, v, h, d_g, 64, algo=ALGOS[algo])
    parts = []
    for s, e in zip(bounds, bounds[1:]):
        hs = max(0, s - (l_h - 1))
        parts.append(g.hyena_conv_fwd_hist(
            q[:, s:e].contiguous(), k[:, s:e].contiguous(), v[:, s:e].contiguous(), h, d_g, 64,
            k[:, hs:s].contiguous(), v[:, hs:s].contiguous(), algo=ALGOS[algo]))
    torch.cuda.synchronize()
    y = torch.cat(parts, 1)
    if algo in ("window", "direct") or (algo == "tensor" and all(s % 128 == 0 for s in bounds)):
        assert torch.equal(y, whole)
    U.assert_parity(y, oracle.gated_fir(q, k, v, h, d_g), q.dtype)


@pytest.mark.parametrize("l_h,Lh", [(128, 127), (200, 150), (513, 512), (385, 1000),
                                     (641, 700)])
def test_history_integer_exact(l_h, Lh):
    """Integer inputs: every fp16 operand and fp32 partial sum of the tensor path is exact, so
    the result equals the oracle's rounded once to bf16 -- any history row taken from the wrong
    place changes an output."""
    wl = custom("int_hist", 2, 600 + Lh, 128, 64, l_h, 64, "bf16", "mr", seed=l_h)
    q, k, v, _, h = make_integer_inputs(wl, device="cuda")
    qs, ks, vs = (t[:, Lh:].contiguous() for t in (q, k, v))
    kh, vh = k[:, :Lh].contiguous(), v[:, :Lh].contiguous()
    y = g.hyena_conv_fwd_hist(qs, ks, vs, h, 64, 64, kh, vh, algo=g.HYENA_ALGO_TENSOR)
    ref = torch.from_numpy(_oracle_with_history(qs, ks, vs, h, 64, kh, vh)).to(torch.bfloat16)
    assert torch.equal(y.cpu(), ref)


def test_empty_history_is_the_plain_forward():
    wl = custom("nohist", 2, 900, 256, 64, 128, 64, "bf16", "mr", seed=9)
    q, k, v, h = make_inputs(wl, device="cuda")
    y0 = g.hyena_conv_fwd(q, k, v, h, 64, 64)
    y1 = g.hyena_conv_fwd_hist(q, k, v, h, 64, 64, None, None)
    e = k[:, :0].contiguous()
    y2 = g.hyena_conv_fwd_hist(q, k, v, h, 64, 64, e, e)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1) and torch.equal(y0, y2)


def test_sharded_forward_single_rank():
    """dist.sequence_sharded_forward without a process group (one rank) is the plain forward."""
    from gated_causal_fir_b200 import dist as D
    wl = custom("one_rank", 1, 1000, 128, 64, 128, 64, "bf16", "mr", seed=4)
    q, k, v, h = make_inputs(wl, device="cuda")
    y = D.sequence_sharded_forward(q, k, v, h, 64, 64)
    torch.cuda.synchronize()
    assert torch.equal(y, g.hyena_conv_fwd(q, k, v, h, 64, 64))
