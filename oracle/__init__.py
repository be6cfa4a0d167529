"""Python (ctypes + numpy) wrapper over the C oracle.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the product package
never does. Arrays are numpy: bf16 and fp16 tensors travel as their uint16 bit
patterns, codes and scales as uint8.

Every function here only marshals arguments; the arithmetic is in
``fp4q_ref.c``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

FMT_NVFP4, FMT_MXFP4, FMT_UE5M3 = 0, 1, 2
ABSMAX, PREVENT_ZERO, FOUR_OVER_SIX, BRUTE_FORCE = 0, 1, 2, 3
_FMT = {"nvfp4": FMT_NVFP4, "mxfp4": FMT_MXFP4, "ue5m3": FMT_UE5M3}
_STRAT = {"absmax": ABSMAX, "prevent_zero": PREVENT_ZERO, "four_over_six": FOUR_OVER_SIX,
          "brute_force": BRUTE_FORCE}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        p = C.c_void_p
        i64, i32 = C.c_int64, C.c_int
        L.ref_e2m1_magnitude.restype = C.c_double
        L.ref_e2m1_magnitude.argtypes = [i32]
        L.ref_e2m1_value.restype = C.c_double
        L.ref_e2m1_value.argtypes = [i32]
        L.ref_e4m3_value.restype = C.c_double
        L.ref_e4m3_value.argtypes = [i32]
        L.ref_e8m0_value.restype = C.c_double
        L.ref_e8m0_value.argtypes = [i32]
        L.ref_bf16_to_float.restype = C.c_float
        L.ref_bf16_to_float.argtypes = [C.c_uint16]
        L.ref_fp16_to_float.restype = C.c_float
        L.ref_fp16_to_float.argtypes = [C.c_uint16]
        L.ref_float_to_bf16.restype = C.c_uint16
        L.ref_float_to_bf16.argtypes = [C.c_float]
        L.ref_rne_e2m1.restype = i32
        L.ref_rne_e2m1.argtypes = [C.c_float]
        L.ref_rne_e4m3_sat.restype = i32
        L.ref_rne_e4m3_sat.argtypes = [C.c_float]
        L.ref_e8m0_exponent.restype = i32
        L.ref_e8m0_exponent.argtypes = [C.c_float]
        L.ref_tsum.restype = C.c_float
        L.ref_tsum.argtypes = [p, i32]
        L.ref_hadamard_k.restype = C.c_float
        L.ref_hadamard_k.argtypes = [i32]
        L.ref_fwht.restype = None
        L.ref_fwht.argtypes = [p, i32]
        L.ref_fwht_array.restype = None
        L.ref_fwht_array.argtypes = [p, i64, i32]
        L.ref_global_amax.restype = C.c_float
        L.ref_global_amax.argtypes = [p, i64, i64, i32]
        L.ref_global_scale.restype = C.c_float
        L.ref_global_scale.argtypes = [C.c_float]
        L.ref_quantize.restype = i32
        L.ref_quantize.argtypes = [p, i64, i64, i32, i32, i32, i32, p, p, p, p, p, p, p]
        L.ref_dequantize.restype = i32
        L.ref_dequantize.argtypes = [p, p, p, i64, i64, i32, i32, p, p]
        L.ref_block_mse.restype = i32
        L.ref_block_mse.argtypes = [p, p, p, p, i64, i64, i32, i32, i32, p]
        L.ref_focus_fwd.restype = i32
        L.ref_focus_fwd.argtypes = [p, p, i64, i64, i32, i32, i32, p, p, p, p, p, p]
        L.ref_focus_bwd.restype = i32
        L.ref_focus_bwd.argtypes = [p, p, p, i64, i64, i32, p]
        L.ref_ue5m3_value.restype = C.c_double
        L.ref_ue5m3_value.argtypes = [i32]
        L.ref_rne_ue5m3_sat.restype = i32
        L.ref_rne_ue5m3_sat.argtypes = [C.c_float]
        L.ref_rne_ue5m3_array.restype = None
        L.ref_rne_ue5m3_array.argtypes = [p, i64, p]
        L.ref_rne_ue5m3_bits_range.restype = None
        L.ref_rne_ue5m3_bits_range.argtypes = [C.c_uint32, i64, p]
        L.ref_gptq.restype = i32
        L.ref_gptq.argtypes = [p, i64, i64, i32, i32, i32, p, C.c_float, p, p, p]
        L.ref_float_to_fp16.restype = C.c_uint16
        L.ref_float_to_fp16.argtypes = [C.c_float]
        f32 = C.c_float
        L.ref_focus_update.restype = i32
        L.ref_focus_update.argtypes = [p, p, p, p, p, p, i64, i64, i32, i32, f32, f32, f32, f32,
                                       i64]
        L.ref_focus_step.restype = i32
        L.ref_focus_step.argtypes = [p, i64, i64, i32, i32, i32, p, p, p, p, p, p, p, i32, f32,
                                     f32, f32, f32, i64]
        L.ref_fp4_gemm.restype = i32
        L.ref_fp4_gemm.argtypes = [p, p, C.c_float, p, p, C.c_float, i64, i64, i64, i32, p]
        L.ref_dequantize_unrotate.restype = i32
        L.ref_dequantize_unrotate.argtypes = [p, p, p, i64, i64, i32, i32, i32, p, p]
        for name in ("ref_rne_e2m1_array", "ref_rne_e4m3_array"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [p, i64, p]
        for name in ("ref_rne_e2m1_bits_range", "ref_rne_e4m3_bits_range"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [C.c_uint32, i64, p]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        a = a.view(np.uint16)
    return a


def _fmt(fmt):
    return _FMT[fmt] if isinstance(fmt, str) else int(fmt)


def _strat(s):
    return _STRAT[s] if isinstance(s, str) else int(s)


# ---------------------------------------------------------------- scalars

def e2m1_value(code: int) -> float:
    return lib().ref_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    return lib().ref_e4m3_value(int(code))


def e8m0_value(b: int) -> float:
    return lib().ref_e8m0_value(int(b))


def ue5m3_value(code: int) -> float:
    return lib().ref_ue5m3_value(code)


def rne_ue5m3_sat(v: float) -> int:
    return lib().ref_rne_ue5m3_sat(v)


def rne_ue5m3_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32)
    out = np.zeros(v.shape, np.uint8)
    lib().ref_rne_ue5m3_array(_ptr(v), v.size, _ptr(out))
    return out


def rne_ue5m3_bits_range(first: int, n: int) -> np.ndarray:
    out = np.zeros(n, np.uint8)
    lib().ref_rne_ue5m3_bits_range(first, n, _ptr(out))
    return out


def rne_e2m1(u: float) -> int:
    return lib().ref_rne_e2m1(float(u))


def rne_e4m3_sat(v: float) -> int:
    return lib().ref_rne_e4m3_sat(float(v))


def e8m0_exponent(a: float) -> int:
    return lib().ref_e8m0_exponent(float(a))


def hadamard_k(n: int) -> float:
    return lib().ref_hadamard_k(int(n))


def global_scale(g: float) -> np.float32:
    return np.float32(lib().ref_global_scale(float(g)))


def bf16_to_float(h: int) -> np.float32:
    return np.float32(lib().ref_bf16_to_float(int(h)))


def fp16_to_float(h: int) -> np.float32:
    return np.float32(lib().ref_fp16_to_float(int(h)))


def float_to_bf16(v) -> int:
    return int(lib().ref_float_to_bf16(float(np.float32(v))))


# ---------------------------------------------------------------- arrays

def rne_e2m1_array(u: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(u, dtype=np.float32)
    out = np.empty(u.shape, np.uint8)
    lib().ref_rne_e2m1_array(_ptr(u), u.size, _ptr(out))
    return out


def rne_e4m3_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().ref_rne_e4m3_array(_ptr(v), v.size, _ptr(out))
    return out


def rne_e2m1_bits_range(first: int, n: int) -> np.ndarray:
    out = np.empty(n, np.uint8)
    lib().ref_rne_e2m1_bits_range(first, n, _ptr(out))
    return out


def rne_e4m3_bits_range(first: int, n: int) -> np.ndarray:
    out = np.empty(n, np.uint8)
    lib().ref_rne_e4m3_bits_range(first, n, _ptr(out))
    return out


def tsum(v: np.ndarray) -> np.float32:
    v = np.array(v, dtype=np.float32, copy=True)
    return np.float32(lib().ref_tsum(_ptr(v), v.size))


def fwht(t: np.ndarray, n: int | None = None) -> np.ndarray:
    """Normalised FWHT of every consecutive n-chunk of t (float32 copy)."""
    t = np.array(t, dtype=np.float32, copy=True)
    n = t.shape[-1] if n is None else n
    assert t.size % n == 0
    lib().ref_fwht_array(_ptr(t), t.size // n, n)
    return t


def global_amax(x_bf16: np.ndarray, rot: int = 0) -> np.float32:
    x = _u16(x_bf16)
    rows, cols = x.shape
    return np.float32(lib().ref_global_amax(_ptr(x), rows, cols, rot))


def quantize(x_bf16, fmt="nvfp4", block=16, strategy="absmax", rot=0, global_amax=None,
             want_mse=True, dq=None):
    """Returns dict(codes, scales, global_scale, mse, dq). dq: None | 'f32' | 'bf16'."""
    x = _u16(x_bf16)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // block), np.uint8)
    gs = np.zeros(1, np.float32)
    ga = None if global_amax is None else np.array([global_amax], np.float32)
    mse = np.zeros((rows, cols // block), np.float32) if want_mse else None
    dqf = np.zeros((rows, cols), np.float32) if dq == "f32" else None
    dqb = np.zeros((rows, cols), np.uint16) if dq == "bf16" else None
    rc = lib().ref_quantize(_ptr(x), rows, cols, _fmt(fmt), block, _strat(strategy), rot,
                            _ptr(ga), _ptr(gs), _ptr(codes), _ptr(scales), _ptr(mse),
                            _ptr(dqf), _ptr(dqb))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return {"codes": codes, "scales": scales, "global_scale": gs[0], "mse": mse,
            "dq": dqf if dq == "f32" else dqb}


def dequantize(codes, scales, global_scale, rows, cols, fmt="nvfp4", block=16, out="f32"):
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    gs = np.array([global_scale if global_scale is not None else 1.0], np.float32)
    of = np.zeros((rows, cols), np.float32) if out == "f32" else None
    ob = np.zeros((rows, cols), np.uint16) if out == "bf16" else None
    rc = lib().ref_dequantize(_ptr(codes), _ptr(scales), _ptr(gs), rows, cols, _fmt(fmt), block,
                              _ptr(of), _ptr(ob))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return of if out == "f32" else ob


def dequantize_unrotate(codes, scales, global_scale, rows, cols, fmt="nvfp4", block=16, rot=0,
                        out="f32"):
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    gs = np.array([1.0 if global_scale is None else global_scale], np.float32)
    of = np.zeros((rows, cols), np.float32) if out == "f32" else None
    ob = np.zeros((rows, cols), np.uint16) if out == "bf16" else None
    rc = lib().ref_dequantize_unrotate(_ptr(codes), _ptr(scales), _ptr(gs), rows, cols,
                                       _fmt(fmt), block, rot, _ptr(of), _ptr(ob))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return of if out == "f32" else ob


def fp4_gemm(a_codes, a_scales, a_sg, b_codes, b_scales, b_sg, fmt="nvfp4"):
    """D = s_a s_b A B^T from packed codes and row-major block scales (float32)."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_scales = np.ascontiguousarray(a_scales, np.uint8)
    b_scales = np.ascontiguousarray(b_scales, np.uint8)
    M, K = a_codes.shape[0], 2 * a_codes.shape[1]
    N = b_codes.shape[0]
    d = np.zeros((M, N), np.float32)
    rc = lib().ref_fp4_gemm(_ptr(a_codes), _ptr(a_scales), float(a_sg or 1.0), _ptr(b_codes),
                            _ptr(b_scales), float(b_sg or 1.0), M, N, K, _fmt(fmt), _ptr(d))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return d


def block_mse(x_bf16, codes, scales, global_scale, fmt="nvfp4", block=16, rot=0):
    x = _u16(x_bf16)
    rows, cols = x.shape
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    gs = np.array([global_scale if global_scale is not None else 1.0], np.float32)
    mse = np.zeros((rows, cols // block), np.float32)
    rc = lib().ref_block_mse(_ptr(x), _ptr(codes), _ptr(scales), _ptr(gs), rows, cols,
                             _fmt(fmt), block, rot, _ptr(mse))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return mse


def focus_fwd(w_bf16, c_fp16, fmt="nvfp4", block=16, sub=8, global_amax=None, out="bf16",
              want_codes=True):
    w = _u16(w_bf16)
    c = _u16(c_fp16)
    rows, cols = w.shape
    assert c.size == rows * cols // sub
    gs = np.zeros(1, np.float32)
    ga = None if global_amax is None else np.array([global_amax], np.float32)
    of = np.zeros((rows, cols), np.float32) if out == "f32" else None
    ob = np.zeros((rows, cols), np.uint16) if out == "bf16" else None
    codes = np.zeros((rows, cols // 2), np.uint8) if want_codes else None
    scales = np.zeros((rows, cols // block), np.uint8) if want_codes else None
    rc = lib().ref_focus_fwd(_ptr(w), _ptr(c), rows, cols, _fmt(fmt), block, sub, _ptr(ga),
                             _ptr(gs), _ptr(of), _ptr(ob), _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return {"w_hat": of if out == "f32" else ob, "codes": codes, "scales": scales,
            "global_scale": gs[0]}


def focus_bwd(w_bf16, g_bf16, c_fp16, sub=8):
    w = _u16(w_bf16)
    g = _u16(g_bf16)
    c = _u16(c_fp16)
    rows, cols = w.shape
    dc = np.zeros((rows, cols // sub), np.float32)
    rc = lib().ref_focus_bwd(_ptr(w), _ptr(g), _ptr(c), rows, cols, sub, _ptr(dc))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return dc


def gptq(w_bf16, scales, global_scale, U, perm=None, fmt="nvfp4", block=16, rot=0):
    """GPTQ error feedback with static groups (fixed block scales); U: fp32
    [K, K] upper Cholesky factor of the inverse Hessian in processing order;
    perm: int32 [K] processing position -> original column (None: identity);
    rot > 0: the rows are first rotated blockwise (MR-GPTQ), and scales, U and
    perm belong to the rotated basis. Returns packed codes [rows, K/2] in the
    original column order."""
    w = _u16(w_bf16)
    rows, K = w.shape
    scales = np.ascontiguousarray(scales, np.uint8)
    U = np.ascontiguousarray(U, np.float32)
    pm = None if perm is None else np.ascontiguousarray(perm, np.int32)
    codes = np.zeros((rows, K // 2), np.uint8)
    sg = 1.0 if global_scale is None else float(global_scale)
    rc = lib().ref_gptq(_ptr(w), rows, K, _fmt(fmt), block, rot, _ptr(scales), sg, _ptr(U), _ptr(pm),
                        _ptr(codes))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return codes


OPT_SGD, OPT_ADAM = 0, 1
_OPT = {"sgd": OPT_SGD, "adam": OPT_ADAM}


def float_to_fp16(v) -> int:
    return int(lib().ref_float_to_fp16(float(v)))


def _opt_state(c, m, v, opt):
    c = np.array(c, np.float32, copy=True)
    if opt == "adam":
        m = np.zeros_like(c) if m is None else np.array(m, np.float32, copy=True)
        v = np.zeros_like(c) if v is None else np.array(v, np.float32, copy=True)
    else:
        m = v = None
    return c, m, v


def focus_update(w_bf16, g_bf16, c, m=None, v=None, sub=8, opt="adam", lr=1e-3, beta1=0.9,
                 beta2=0.999, eps=1e-8, t=1):
    """One coefficient update from an external gradient g; returns new copies
    {"c", "c_half", "m", "v"} (inputs are not modified)."""
    w = _u16(w_bf16)
    g = _u16(g_bf16)
    rows, cols = w.shape
    c, m, v = _opt_state(c, m, v, opt)
    ch = np.zeros(c.shape, np.uint16)
    rc = lib().ref_focus_update(_ptr(w), _ptr(g), _ptr(c), _ptr(ch), _ptr(m), _ptr(v), rows,
                                cols, sub, _OPT[opt], lr, beta1, beta2, eps, t)
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return {"c": c, "c_half": ch, "m": m, "v": v}


def focus_step(w_bf16, c, m=None, v=None, fmt="nvfp4", block=16, sub=8, global_amax=None,
               opt="adam", lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, t=1):
    """One fused calibration step on the weight-reconstruction loss; returns new
    copies {"c", "c_half", "m", "v", "sse", "global_scale"}."""
    w = _u16(w_bf16)
    rows, cols = w.shape
    c, m, v = _opt_state(c, m, v, opt)
    ch = np.zeros(c.shape, np.uint16)
    sse = np.zeros(c.shape, np.float32)
    gs = np.zeros(1, np.float32)
    ga = None if global_amax is None else np.array([global_amax], np.float32)
    rc = lib().ref_focus_step(_ptr(w), rows, cols, _fmt(fmt), block, sub, _ptr(ga), _ptr(gs),
                              _ptr(c), _ptr(ch), _ptr(m), _ptr(v), _ptr(sse), _OPT[opt], lr,
                              beta1, beta2, eps, t)
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return {"c": c, "c_half": ch, "m": m, "v": v, "sse": sse, "global_scale": gs[0]}


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """Packed bytes [.., n/2] -> 4-bit codes [.., n] (low nibble first)."""
    codes = np.asarray(codes, np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 15
    out[..., 1::2] = codes >> 4
    return out
