"""ctypes binding of the C ABI in include/hyena_conv.h.

Argument marshalling only: every step of the computation runs in the CUDA kernels of
``libhyena_conv.so``.  There is no fallback; if the library is missing the first call raises.
"""
import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhyena_conv.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "hyena_conv.h")
TESTING_HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "hyena_conv_testing.h")

HYENA_OK = 0
HYENA_ERR_INVALID_ARG = 1
HYENA_ERR_UNSUPPORTED = 2
HYENA_ERR_MISALIGNED = 3
HYENA_ERR_CUDA = 4

HYENA_DTYPE_BF16 = 0
HYENA_DTYPE_F32 = 1

HYENA_ALGO_AUTO = 0
HYENA_ALGO_TENSOR = 1
HYENA_ALGO_WINDOW = 2
HYENA_ALGO_DIRECT = 3
HYENA_ALGO_FFT = 4
ALGO_NAMES = {HYENA_ALGO_AUTO: "auto", HYENA_ALGO_TENSOR: "tensor", HYENA_ALGO_WINDOW: "window",
              HYENA_ALGO_DIRECT: "direct", HYENA_ALGO_FFT: "fft"}

HYENA_DEVICE_TIMEOUT = 1
HYENA_DEVICE_F16_RANGE = 2

HYENA_BWD_STATIC_SCRATCH_BYTES = 8 << 20

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int

# name -> (restype, argtypes); must match include/hyena_conv.h
SIGNATURES = {
    "hyena_conv_fwd": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _vp]),
    "hyena_conv_fwd_f32": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32,
                                  _vp]),
    "hyena_conv_fwd_ex": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32,
                                 _i32, _i32, _vp]),
    "hyena_conv_fwd_hist": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                   _i32, _i32, _i32, _i32, _i32, _vp]),
    "hyena_conv_fwd_fft_workspace_bytes": (_i64, [_i64, _i64, _i64, _i32, _i32]),
    "hyena_conv_fwd_fft": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32,
                                  _i32, _vp, ctypes.c_size_t, _vp]),
    "hyena_conv_fwd_from_host_workspace_bytes": (_i64, [_i64, _i64, _i64, _i32, _i32, _i32,
                                                         _i64]),
    "hyena_conv_fwd_from_host": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32,
                                        _i32, _i32, _i64, _vp, ctypes.c_size_t, _vp]),
    "hyena_select_algo": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32,
                                 _i32]),
    "hyena_conv_bwd_workspace_bytes": (_i64, [_i64, _i64, _i64, _i32, _i32]),
    "hyena_conv_bwd": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                              _i32, _i32, _i32, _i32, _vp, ctypes.c_size_t, _vp]),
    "hyena_conv_bwd_ex": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                 _i32, _i32, _i32, _i32, _i32, _vp, ctypes.c_size_t, _vp]),
    "hyena_select_bwd_algo": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                     _i32, _i32, _i32, _i32]),
    "hyena_conv_bwd_static_scratch": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64,
                                             _i64, _i64, _i32, _i32, _i32, _i32, _vp]),
    "hyena_build_toeplitz": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp]),
    "hyena_toeplitz_stages": (_i32, [_i32, _i32]),
    "hyena_build_toeplitz_blocks": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _vp]),
    "hyena_device_status": (_i32, [ctypes.POINTER(ctypes.c_uint), _i32]),
    "hyena_status_string": (ctypes.c_char_p, [_i32]),
    "hyena_abi_version": (_i32, []),
}

# include/hyena_conv_testing.h: test hooks, not part of the operation's interface
TESTING_SIGNATURES = {
    "hyena_testing_fwd_fault": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32,
                                       _i32, ctypes.c_uint64, _vp]),
}

_LIB = None


class HyenaError(RuntimeError):
    """A C-ABI call returned a status other than HYENA_OK."""

    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (fn, status_string(status), status))


def header_functions(path=HEADER_PATH):
    """Names of the functions a header (default include/hyena_conv.h) declares."""
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hyena_[a-z0-9_]+)\s*\(", src)))


def lib():
    """The loaded library (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libhyena_conv.so is not built (%s); run "
                              "`python -m gated_causal_fir_b200.build`" % LIB_PATH)
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in list(SIGNATURES.items()) + list(TESTING_SIGNATURES.items()):
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def status_string(status: int) -> str:
    return lib().hyena_status_string(int(status)).decode()


def check(fn: str, status: int):
    if status != HYENA_OK:
        raise HyenaError(fn, status)
