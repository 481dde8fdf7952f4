"""The C ABI on a host without a GPU: the library builds and loads, exports every function
include/hyena_conv.h declares, and rejects bad arguments on the host before touching a device.
No call here reaches a kernel launch."""
import ctypes
import shutil

import pytest

import gated_causal_fir_b200 as g
from gated_causal_fir_b200 import _native, build

pytestmark = pytest.mark.skipif(
    shutil.which("nvcc") is None and not __import__("os").path.exists(_native.LIB_PATH),
    reason="needs nvcc or a built library")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _native.lib()


def test_exports_every_header_function(lib):
    declared = _native.header_functions()
    assert len(declared) >= 8
    assert set(declared) == set(_native.SIGNATURES), "binding table out of step with the header"
    for name in declared:
        assert hasattr(lib, name), name
    testing = _native.header_functions(_native.TESTING_HEADER_PATH)
    assert set(testing) == set(_native.TESTING_SIGNATURES)
    for name in testing:
        assert hasattr(lib, name), name


def test_testing_entry_point_rejects_bad_arguments(lib):
    """The test hook checks its own arguments on the host (nothing is launched)."""
    fn = lib.hyena_testing_fwd_fault
    p = 256
    # fault out of range, wait limit out of [1 ms, 2 s], unsupported shape
    assert fn(p, p, p, p, 1 << 20, 1, 128, 64, 64, 7, 2, 10 ** 7, None) == _native.HYENA_ERR_INVALID_ARG
    assert fn(p, p, p, p, 1 << 20, 1, 128, 64, 64, 7, 1, 10 ** 5, None) == _native.HYENA_ERR_INVALID_ARG
    assert fn(p, p, p, p, 1 << 20, 1, 128, 64, 64, 7, 1, 3 * 10 ** 9, None) == \
        _native.HYENA_ERR_INVALID_ARG
    assert fn(p, p, p, p, 1 << 20, 1, 128, 96, 32, 40, 1, 10 ** 7, None) == \
        _native.HYENA_ERR_UNSUPPORTED
    assert fn(p, p, p, p, 1 << 20, 0, 128, 64, 64, 7, 1, 10 ** 7, None) == _native.HYENA_OK  # empty


def test_status_strings_and_version(lib):
    assert g.hyena_abi_version() == 1
    assert g.hyena_status_string(0) == "ok"
    for code in (1, 2, 3, 4):
        assert g.hyena_status_string(code) not in ("ok", "unknown status")
    assert g.hyena_status_string(99) == "unknown status"


def test_select_algo_for_the_workloads(lib):
    from gated_causal_fir_b200.workloads import WORKLOADS
    want = {"tiny": g.HYENA_ALGO_WINDOW, "se": g.HYENA_ALGO_WINDOW, "mr": g.HYENA_ALGO_TENSOR,
            "mr_batched": g.HYENA_ALGO_TENSOR, "mr_1m": g.HYENA_ALGO_TENSOR,
            "li": g.HYENA_ALGO_DIRECT}  # l_h = L = 8192: blocks of one row; FFT entry point
    for name, wl in WORKLOADS.items():
        dt = g.HYENA_DTYPE_F32 if wl.dtype == "f32" else g.HYENA_DTYPE_BF16
        assert g.hyena_select_algo(wl.B, wl.L, wl.D, wl.d_g, wl.l_h, wl.l_b, dt) == want[name]


def test_select_algo_fallbacks(lib):
    bf, f32 = g.HYENA_DTYPE_BF16, g.HYENA_DTYPE_F32
    assert g.hyena_select_algo(1, 100, 256, 64, 642, 65, bf) == g.HYENA_ALGO_FFT     # l_h > 641
    assert g.hyena_select_algo(1, 100, 256, 64, 641, 65, bf) == g.HYENA_ALGO_TENSOR  # 5 tiles back
    assert g.hyena_select_algo(1, 100, 256, 64, 130, 65, bf) == g.HYENA_ALGO_TENSOR  # 2 tiles back
    assert g.hyena_select_algo(1, 100, 256, 64, 129, 65, bf) == g.HYENA_ALGO_TENSOR
    assert g.hyena_select_algo(1, 100, 128, 32, 40, 32, bf) == g.HYENA_ALGO_TENSOR
    assert g.hyena_select_algo(1, 100, 96, 32, 40, 32, bf) == g.HYENA_ALGO_DIRECT   # D % 64 != 0
    assert g.hyena_select_algo(1, 4096, 96, 32, 40, 32, bf) == g.HYENA_ALGO_FFT     # long enough
    assert g.hyena_select_algo(1, 100, 96, 32, 16, 32, f32) == g.HYENA_ALGO_WINDOW
    assert g.hyena_select_algo(1, 100, 90, 30, 40, 32, bf) == g.HYENA_ALGO_DIRECT   # 8192-point
    # d_g = 30: only the 8192-point length applies (one channel pair per CTA, its slowest
    # configuration): at 40 taps the direct sum wins, at 400 the block FFT
    assert g.hyena_select_algo(1, 8192, 90, 30, 40, 32, bf) == g.HYENA_ALGO_DIRECT
    assert g.hyena_select_algo(1, 8192, 90, 30, 400, 32, bf) == g.HYENA_ALGO_FFT
    assert g.hyena_select_algo(1, 100, 93, 31, 40, 32, bf) == g.HYENA_ALGO_DIRECT   # odd groups
    assert g.hyena_select_algo(1, 100, 96, 32, 16, 32, bf) == g.HYENA_ALGO_WINDOW
    assert g.hyena_select_algo(1, 100, 128, 16, 65, 64, bf) == g.HYENA_ALGO_TENSOR  # 4 bands fit
    assert g.hyena_select_algo(1, 100, 128, 16, 7, 16, bf) == g.HYENA_ALGO_WINDOW   # 36 MMAs/tile
    assert g.hyena_select_algo(1, 100, 128, 32, 7, 16, bf) == g.HYENA_ALGO_TENSOR   # 18 MMAs/tile
    assert g.hyena_select_algo(1, 100, 128, 16, 66, 64, bf) == g.HYENA_ALGO_DIRECT  # they do not
    assert g.hyena_select_algo(1, 100, 128, 8, 7, 16, bf) == g.HYENA_ALGO_WINDOW    # d_g = 8
    assert g.hyena_select_algo(1, 100, 96, 4, 3, 2, bf) == g.HYENA_ALGO_DIRECT      # 4 ch < 16 B
    assert g.hyena_select_algo(1, 100, 96, 4, 3, 2, f32) == g.HYENA_ALGO_WINDOW
    assert g.hyena_select_algo(1, 64, 128, 64, 128, 64, f32) == g.HYENA_ALGO_DIRECT  # L = 64
    assert g.hyena_select_algo(1, 2048, 128, 64, 128, 64, f32) == g.HYENA_ALGO_FFT
    assert g.hyena_select_algo(1, 64, 128, 64, 16, 64, f32) == g.HYENA_ALGO_WINDOW
    n = 64 * 128 * 2
    odd = (16 + 2, 16 + n + 64, 16 + 2 * (n + 64), 16 + 3 * (n + 64), 16 + 4 * (n + 64))
    assert g.hyena_select_algo(1, 64, 128, 64, 128, 64, bf, ptrs=odd) == g.HYENA_ALGO_DIRECT


BASE = dict(B=1, L=64, D=128, d_g=64, l_h=16, l_b=16)


def _call(lib, q=0x10000, k=0x20000, v=0x30000, h=0x40000, y=0x50000, dtype=0, algo=0, **kw):
    a = dict(BASE, **kw)
    return lib.hyena_conv_fwd_ex(q, k, v, h, y, a["B"], a["L"], a["D"], a["d_g"], a["l_h"],
                                 a["l_b"], dtype, algo, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(v=None), 1), (dict(h=None), 1), (dict(y=None), 1),
    (dict(B=-1), 1), (dict(L=-5), 1), (dict(D=0), 1), (dict(d_g=0), 1), (dict(d_g=48), 1),
    (dict(l_h=0), 1), (dict(l_b=0), 1), (dict(dtype=7), 1),
    (dict(algo=9), 1), (dict(y=0x10000 + 64), 1), (dict(q=0x10001), 3), (dict(h=0x40002), 3),
    (dict(algo=1, dtype=1), 2), (dict(algo=1, d_g=8, l_h=8, l_b=8), 2),
    (dict(algo=2, l_h=17, l_b=16), 2),
    (dict(algo=1, q=0x10002), 2),
    (dict(algo=1, l_h=642, l_b=16), 2),                  # past the tensor path's 641 taps
    (dict(algo=1, d_g=32, l_h=258, l_b=16), 2),          # d_g 32: bands fit up to 257 taps
    (dict(algo=4, D=96, d_g=3, l_h=40), 2),              # block FFT: channel pairs need even d_g
])
def test_host_validation(lib, kw, code):
    assert _call(lib, **kw) == code


def test_empty_problem_is_ok_without_launch(lib):
    assert _call(lib, B=0) == 0
    assert _call(lib, L=0, q=None, k=None, v=None, y=None) == 0


def test_size_overflow_rejected(lib):
    assert _call(lib, B=1 << 40, L=1 << 20, D=1 << 12) == 1


def test_toeplitz_validation(lib):
    f = lib.hyena_build_toeplitz
    assert f(None, 0x2000, 0x3000, 0x4000, 4, 4, 3, None) == 1
    assert f(0x1000, 0x2000, 0x3000, None, 4, 5, 3, None) == 1  # l_h >= l_b + 2 needs H2
    assert f(0x1000, 0x2000, 0x3000, 0x4000, 4, 9, 4, None) == 1  # l_h > 2 l_b
    assert f(0x1000, 0x2000, 0x3000, 0x4000, 0, 4, 3, None) == 1
    assert f(0x1001, 0x2000, 0x3000, 0x4000, 4, 4, 3, None) == 3


def test_toeplitz_blocks_validation(lib):
    f = lib.hyena_build_toeplitz_blocks
    assert f(None, 0x2000, 3, 4, 9, 4, None) == 1
    assert f(0x1000, None, 3, 4, 9, 4, None) == 1
    assert f(0x1000, 0x2000, 0, 4, 9, 4, None) == 1
    assert f(0x1000, 0x2000, 3, 0, 9, 4, None) == 1
    assert f(0x1000, 0x2000, 3, 4, 0, 4, None) == 1
    assert f(0x1000, 0x2000, 3, 4, 9, 0, None) == 1
    assert f(0x1000, 0x2000, 1 << 30, 1 << 30, 9, 1 << 20, None) == 1  # too large to index
    assert f(0x1002, 0x2000, 3, 4, 9, 4, None) == 3
    assert f(0x1000, 0x2001, 3, 4, 9, 4, None) == 3


@pytest.mark.parametrize("l_h,l_b,S", [(1, 1, 1), (2, 1, 2), (4, 3, 2), (5, 3, 3), (7, 16, 2),
                                       (17, 16, 2), (18, 16, 3), (128, 64, 3), (129, 64, 3),
                                       (130, 64, 4), (300, 64, 6), (1000, 7, 144)])
def test_toeplitz_stages(lib, l_h, l_b, S):
    import oracle
    assert lib.hyena_toeplitz_stages(l_h, l_b) == S == oracle.stages_needed(l_h, l_b)


def test_toeplitz_stages_validation(lib):
    assert lib.hyena_toeplitz_stages(0, 4) == -1
    assert lib.hyena_toeplitz_stages(4, 0) == -1


def test_long_filters_select_an_algorithm():
    bf = g.HYENA_DTYPE_BF16
    assert g.hyena_select_algo(1, 8192, 4096, 64, 130, 64, bf) == g.HYENA_ALGO_TENSOR
    assert g.hyena_select_algo(1, 8192, 4096, 64, 513, 64, bf) == g.HYENA_ALGO_TENSOR
    assert g.hyena_select_algo(1, 8192, 4096, 64, 514, 64, bf) == g.HYENA_ALGO_TENSOR
    assert g.hyena_select_algo(1, 8192, 4096, 64, 641, 64, bf) == g.HYENA_ALGO_TENSOR
    assert g.hyena_select_algo(1, 8192, 4096, 64, 642, 64, bf) == g.HYENA_ALGO_FFT
    assert g.hyena_select_algo(1, 8192, 4096, 32, 257, 64, bf) == g.HYENA_ALGO_TENSOR
    assert g.hyena_select_algo(1, 8192, 4096, 32, 258, 64, bf) == g.HYENA_ALGO_FFT
    assert g.hyena_select_algo(1, 8192, 4096, 16, 66, 16, bf) == g.HYENA_ALGO_FFT
    assert g.hyena_select_algo(1, 8192, 4096, 64, 300, 64, g.HYENA_DTYPE_F32) == \
        g.HYENA_ALGO_FFT
    assert g.hyena_select_algo(1, 8192, 4096, 64, 6000, 64, bf) == g.HYENA_ALGO_FFT
    # 8192-point blocks would keep fewer than 1024 rows: the direct sum
    assert g.hyena_select_algo(1, 8192, 4096, 64, 7200, 64, bf) == g.HYENA_ALGO_DIRECT


def test_history_validation(lib):
    f = lib.hyena_conv_fwd_hist
    q, k, v, h, y = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000
    kh, vh = 0x60000, 0x70000
    a = (1, 64, 128, 64, 16, 16, 0, 0, None)  # B, L, D, d_g, l_h, l_b, dtype, algo, stream
    assert f(q, k, v, h, y, kh, vh, -1, *a) == 1                    # negative L_hist
    assert f(q, k, v, h, y, None, vh, 8, *a) == 1                   # missing history
    assert f(q, k, v, h, y, kh, None, 8, *a) == 1
    assert f(q, k, v, h, y, kh + 1, vh, 8, *a) == 3                 # misaligned history
    assert f(q, k, v, h, y, y + 64, vh, 8, *a) == 1                 # history overlaps y
    assert f(q, k, v, h, y, y - 1024, vh, 8, *a) == 1               # history runs into y
    assert f(q, k, v, h, y, kh, vh, 8, 0, 64, 128, 64, 16, 16, 0, 0, None) == 0  # empty: no launch


def test_fft_workspace_bytes(lib):
    f = lib.hyena_conv_fwd_fft_workspace_bytes
    # L = l_h = 8192, D = 4096, d_g = 64: N = 16384; 4 B N D of data spectra + 2 x 8 N G
    assert f(1, 8192, 4096, 64, 8192) == 4 * 16384 * 4096 + 2 * 8 * 16384 * 64
    assert f(2, 8, 4, 2, 3) == 2 * 256 * 2 * 8 + 2 * 256 * 2 * 8   # N = 256, the smallest
    assert f(1, 8192, 4096, 63, 8192) == -1                  # D % d_g
    assert f(1, 8192, 4095, 4095, 10) == -2                  # odd D: channel pairs
    assert f(1, 100, 96, 3, 10) == -2                        # odd d_g
    assert f(1, 40000, 64, 64, 30000) == -2                  # L + l_h - 1 > 65536
    assert f(0, 100, 64, 2, 10) == 0


def test_fft_validation(lib):
    f = lib.hyena_conv_fwd_fft
    q, k, v, h, y = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    a = (1, 64, 128, 64, 16, 16, 0)   # B, L, D, d_g, l_h, l_b, dtype
    need = lib.hyena_conv_fwd_fft_workspace_bytes(1, 64, 128, 64, 16)
    assert f(q, k, v, h, y, *a, None, need, None) == 1               # no workspace
    assert f(q, k, v, h, y, *a, 0x600000, need - 1, None) == 1       # too small
    assert f(q, k, v, h, y, *a, 0x600008, need, None) == 3           # misaligned
    assert f(q, k, v, h, y, 1, 64, 128, 3, 16, 16, 0, 0x600000, need, None) == 1  # D % d_g
    assert f(q, k, v, h, y, 1, 64, 126, 63, 16, 16, 0, 0x600000, need, None) == 2  # odd d_g
    assert f(q, k, v, h, y, 0, 64, 128, 64, 16, 16, 0, None, 0, None) == 0  # empty: no launch


def test_from_host_workspace_bytes(lib):
    f = lib.hyena_conv_fwd_from_host_workspace_bytes
    # MR, 2048-row chunks: 3 slots x 4 tensors x (2048 + 127) rows x 4096 x 2 B, plus h
    assert f(1, 8192, 4096, 64, 128, 0, 2048) == 3 * 4 * 2175 * 4096 * 2 + 64 * 128 * 4
    # chunk longer than L: a slot tensor holds L + l_h - 1 = 104 rows of 12 fp32 (4992 B,
    # rounded up to 5120); h (2 x 5 floats) rounds up to 256
    assert f(2, 100, 12, 6, 5, 1, 4096) == 3 * 4 * 5120 + 256
    assert f(1, 100, 64, 63, 5, 0, 64) == -1        # D % d_g
    assert f(1, 100, 64, 64, 5, 0, 0) == -1         # chunk < 1
    assert f(1, 100, 64, 64, 5, 7, 64) == -1        # dtype
    assert f(0, 100, 64, 64, 5, 0, 64) == 0


def test_from_host_validation(lib):
    f = lib.hyena_conv_fwd_from_host
    q, k, v, h, y = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    need = lib.hyena_conv_fwd_from_host_workspace_bytes(1, 64, 128, 64, 16, 0, 32)
    a = (1, 64, 128, 64, 16, 16, 0, 32)               # B, L, D, d_g, l_h, l_b, dtype, chunk
    assert f(q, k, v, h, y, *a, None, need, None) == 1              # no workspace
    assert f(q, k, v, h, y, *a, 0x600000, need - 1, None) == 1      # short workspace
    assert f(q, k, v, h, y, *a, 0x600010, need, None) == 3          # workspace not 256-aligned
    assert f(q, k, v, h, y, 1, 64, 128, 64, 16, 16, 0, 0, 0x600000, need, None) == 1  # chunk 0
    assert f(None, k, v, h, y, *a, 0x600000, need, None) == 1       # null input
    assert f(q, k, v, h, q, *a, 0x600000, need, None) == 1          # y aliases q
    assert f(q + 1, k, v, h, y, *a, 0x600000, need, None) == 3      # misaligned element
    assert f(q, k, v, h, y, 0, 64, 128, 64, 16, 16, 0, 32, None, 0, None) == 0  # empty


def test_device_status_needs_out(lib):
    assert lib.hyena_device_status(None, 0) == 1


def test_from_host_binding_checks_before_any_device_work():
    """hyena_conv_fwd_from_host takes contiguous host tensors (and fp32 filters) only; the checks
    run before anything touches a device."""
    import torch
    q = torch.zeros(1, 8, 64, dtype=torch.bfloat16)
    h = torch.zeros(1, 4)
    with pytest.raises(TypeError):
        g.hyena_conv_fwd_from_host(q.transpose(1, 2), q, q, h, d_g=64, l_b=4)  # not contiguous
    with pytest.raises(TypeError):
        g.hyena_conv_fwd_from_host(q, q, q, h.double(), d_g=64, l_b=4)         # fp64 filters
    with pytest.raises(TypeError):
        g.hyena_conv_fwd_from_host(q, q.float(), q, h, d_g=64, l_b=4)          # mixed dtypes
    with pytest.raises(TypeError):
        g.hyena_conv_fwd_from_host(q, q, q, h, d_g=64, l_b=4, out=torch.zeros(1, 8, 32))


def test_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 8, 64, dtype=torch.bfloat16)
    h = torch.zeros(1, 4)
    with pytest.raises(TypeError):
        g.hyena_conv_fwd(q, q, q, h, d_g=64, l_b=4)


def test_bwd_workspace_bytes(lib):
    # D = 4096, d_g = 64 (pieces of 64 channels), l_h = 128, 8192 tokens: 128 chunks x 64 x 128
    # partials, then 256 bytes for the tensor path's operand-range flag
    assert lib.hyena_conv_bwd_workspace_bytes(1, 8192, 4096, 64, 128) == 128 * 64 * 128 * 4 + 256
    assert lib.hyena_conv_bwd_workspace_bytes(1, 8192, 4096, 63, 128) == -1
    assert lib.hyena_conv_bwd_workspace_bytes(0, 8192, 4096, 64, 128) == 0
    assert lib.hyena_conv_bwd_workspace_bytes(1, 1, 6, 6, 5) == 512  # rounded up, + the flag
    # SE (l_h = 7, d_g = 16): the window kernel's partials at its shortest runs, one per
    # 32-row block and 4-channel vector (the fp32 width): 256 x 1024 x 7 floats
    assert lib.hyena_conv_bwd_workspace_bytes(1, 8192, 4096, 16, 7) == 256 * 1024 * 7 * 4


def test_bwd_static_scratch_rejects_oversize_on_host(lib):
    # 16448 tokens of the D = 4096, d_g = 64, l_h = 128 shape need 257 chunks of partials
    # (8.4 MB > 8 MiB): rejected before any device work.  Distinct aligned stand-in addresses.
    B, L, D = 1, 16448, 4096
    n = B * L * D * 2 + 4096
    p = [4096 + i * n for i in range(9)]
    assert lib.hyena_conv_bwd_workspace_bytes(B, L, D, 64, 128) > _native.HYENA_BWD_STATIC_SCRATCH_BYTES
    rc = lib.hyena_conv_bwd_static_scratch(*p, B, L, D, 64, 128, 64, 0, None)
    assert rc == _native.HYENA_ERR_UNSUPPORTED
    rc = lib.hyena_conv_bwd_static_scratch(*p, B, L, D, 63, 128, 64, 0, None)
    assert rc == _native.HYENA_ERR_INVALID_ARG


def test_select_bwd_algo(lib):
    T, Dd, W = g.HYENA_ALGO_TENSOR, g.HYENA_ALGO_DIRECT, g.HYENA_ALGO_WINDOW
    assert g.hyena_select_bwd_algo(1, 8192, 4096, 64, 128, 64) == T   # MR: fused tensor kernel
    assert g.hyena_select_bwd_algo(1, 8192, 4096, 16, 7, 16) == W     # SE: register window
    assert g.hyena_select_bwd_algo(1, 8192, 4096, 16, 17, 16) == Dd   # 17 taps: past the window
    assert g.hyena_select_bwd_algo(1, 8192, 4092, 6, 7, 16) == Dd     # 6-channel groups
    assert g.hyena_select_bwd_algo(1, 8192, 4096, 64, 128, 64, g.HYENA_DTYPE_F32) == Dd
    assert g.hyena_select_bwd_algo(1, 300, 4096, 64, 130, 65) == Dd   # l_h > 129
    assert g.hyena_select_bwd_algo(1, 300, 96, 32, 16, 16) == W
    assert g.hyena_select_bwd_algo(1, 300, 4096, 64, 300, 16) == Dd   # l_h > 2 l_b: block form


def test_fft_block_refuses_short_blocks_on_host(lib):
    """A filter whose 8192-point blocks would keep fewer than 1024 of their rows (and no shorter
    transform holds it): the forced block FFT returns HYENA_ERR_UNSUPPORTED before any device
    work.  Distinct stand-in addresses, 16 MiB apart."""
    B, L, D, d_g, l_h = 1, 20000, 128, 64, 8000
    p = [0x1000000 * (i + 1) for i in range(5)]
    rc = lib.hyena_conv_fwd_ex(*p, B, L, D, d_g, l_h, 64, 0, g.HYENA_ALGO_FFT, None)
    assert rc == _native.HYENA_ERR_UNSUPPORTED


def test_backward_refuses_the_forward_only_fft(lib):
    """HYENA_ALGO_FFT is a forward algorithm: the backward refuses it on the host."""
    B, L, D, d_g, l_h = 1, 256, 128, 64, 16
    p = [0x1000000 * (i + 1) for i in range(9)]
    need = lib.hyena_conv_bwd_workspace_bytes(B, L, D, d_g, l_h)
    ws = 0x1000000 * 12
    rc = lib.hyena_conv_bwd_ex(*p, B, L, D, d_g, l_h, 16, 0, g.HYENA_ALGO_FFT, ws, need, None)
    assert rc == _native.HYENA_ERR_UNSUPPORTED
