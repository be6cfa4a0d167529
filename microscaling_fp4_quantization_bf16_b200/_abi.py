"""ctypes declarations of the C ABI in include/fp4q.h (libfp4q.so).

Argument marshalling only: every step of quantization runs in the CUDA
kernels behind these entry points. Loading fails loudly when the library has
not been built; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp4q.so")

# Every symbol declared in include/fp4q.h, with (restype, argtypes).
_p = C.c_void_p
_i64 = C.c_int64
_i32 = C.c_int
_f32 = C.c_float
SIGNATURES = {
    "fp4q_quantize": (_i32, [_p, _i64, _i64, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p,
                             _i32, _p]),
    "fp4q_dequantize": (_i32, [_p, _p, _p, _i64, _i64, _i32, _i32, _p, _i32, _p]),
    "fp4q_dequantize_unrotate": (_i32, [_p, _p, _p, _i64, _i64, _i32, _i32, _i32, _p, _i32, _p]),
    "fp4q_block_mse": (_i32, [_p, _p, _p, _p, _i64, _i64, _i32, _i32, _i32, _p, _p]),
    "fp4q_focus_fwd": (_i32, [_p, _p, _i64, _i64, _i32, _i32, _i32, _p, _p, _p, _i32, _p, _p,
                              _p]),
    "fp4q_focus_bwd": (_i32, [_p, _p, _p, _i64, _i64, _i32, _p, _p]),
    "fp4q_focus_update": (_i32, [_p, _p, _p, _p, _p, _p, _i64, _i64, _i32, _i32, _f32, _f32,
                                 _f32, _f32, _i64, _p]),
    "fp4q_focus_step": (_i32, [_p, _i64, _i64, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p, _p,
                               _i32, _f32, _f32, _f32, _f32, _i64, _p]),
    "fp4q_gptq": (_i32, [_p, _i64, _i64, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p, _p]),
    "fp4q_global_amax": (_i32, [_p, _i64, _i64, _i32, _p, _p]),
    "fp4q_e2m1_encode": (_i32, [_p, _i64, _p, _p]),
    "fp4q_e4m3_encode": (_i32, [_p, _i64, _p, _p]),
    "fp4q_gemm_noalloc": (_i32, [_p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i32, _p, _i32, _p]),
    "fp4q_quantize_mma": (_i32, [_p, _i64, _i64, _i32, _i32, _i32, _p, _p, _p, _p, _p]),
    "fp4q_mma_scale_bytes": (C.c_size_t, [_i64, _i64, _i32]),
    "fp4q_scales_to_mma": (_i32, [_p, _i64, _i64, _i32, _p, _p]),
    "fp4q_gemm": (_i32, [_p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i32, _p, _p, _i32, _p]),
    "fp4q_status_string": (C.c_char_p, [_i32]),
    "fp4q_last_cuda_error": (_i32, []),
    "fp4q_debug_fail_launches": (None, [_i32]),
    "fp4q_device_errors": (_i32, []),
}

_lib = None
_lock = threading.Lock()


class Fp4qError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


def load(path: str = LIB_PATH):
    """Loads libfp4q.so; raises if it is missing (build it with build.py)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    f"CUDA library {path} is missing: run "
                    "`python -m microscaling_fp4_quantization_bf16_b200.build` (needs nvcc)")
            lib = C.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def call(name: str, *args) -> None:
    lib = load()
    st = getattr(lib, name)(*args)
    if st != 0:
        msg = lib.fp4q_status_string(st).decode()
        if st == 6:
            msg += f"; cudaError {lib.fp4q_last_cuda_error()}"
        raise Fp4qError(name, st, msg)


def status(name: str, *args) -> int:
    """Calls an entry point and returns its raw status (for error-path tests)."""
    return getattr(load(), name)(*args)
