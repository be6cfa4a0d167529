"""B200-native block-scaled FP4 quantization (MXFP4 / NVFP4) and FOCUS.

PyTorch is used for device memory and streams only: every function below
allocates its outputs with torch (unless given preallocated ones), then calls
the C ABI of libfp4q.so on ``torch.cuda.current_stream()``. All arithmetic
runs in the library's sm_100a kernels. Nothing here computes on the CPU.

Pages: "Finer is Better (with the Right Scaling)" (scale strategies, block
sizes), "Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization" (MXFP4 / NVFP4, blockwise Hadamard rotation), "FOCUS: FP4
Optimization via Coupled-Relaxation and Dual-Granularity Scaling" (decoupled
fake quantization and its straight-through gradient).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from ._abi import Fp4qError, load  # noqa: F401
from . import _abi

FORMATS = {"nvfp4": 0, "mxfp4": 1, "ue5m3": 2}
STRATEGIES = {"absmax": 0, "prevent_zero": 1, "four_over_six": 2, "brute_force": 3}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _check(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def _strat(s) -> int:
    return STRATEGIES[s] if isinstance(s, str) else int(s)


@dataclass
class Quantized:
    codes: torch.Tensor                   # uint8 [rows, cols/2]
    scales: torch.Tensor                  # uint8 [rows, cols/block]
    global_scale: Optional[torch.Tensor]  # float32 [1] (NVFP4) or None
    mse: Optional[torch.Tensor]           # float32 [rows, cols/block] or None
    dq: Optional[torch.Tensor]            # [rows, cols] float32/bfloat16 or None


def quantize(x: torch.Tensor, fmt="nvfp4", block: int = 16, strategy="absmax", rot: int = 0,
             global_amax: Optional[torch.Tensor] = None, want_mse: bool = False,
             dq_dtype: Optional[torch.dtype] = None, out: Optional[Quantized] = None) -> Quantized:
    """Quantize a bf16 [rows, cols] tensor. See fp4q_quantize in include/fp4q.h."""
    _check(x, torch.bfloat16, "x")
    rows, cols = x.shape
    f = _fmt(fmt)
    if out is None:
        dev = x.device
        out = Quantized(
            codes=torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(rows, cols // block, dtype=torch.uint8, device=dev),
            global_scale=torch.empty(1, dtype=torch.float32, device=dev) if f == 0 else None,
            mse=torch.empty(rows, cols // block, dtype=torch.float32, device=dev) if want_mse else None,
            dq=torch.empty(rows, cols, dtype=dq_dtype, device=dev) if dq_dtype is not None else None,
        )
    if global_amax is not None:
        _check(global_amax, torch.float32, "global_amax")
    _abi.call("fp4q_quantize", x.data_ptr(), rows, cols, f, block, _strat(strategy), rot,
              _ptr(global_amax), _ptr(out.global_scale), out.codes.data_ptr(),
              out.scales.data_ptr(), _ptr(out.mse), _ptr(out.dq),
              DTYPES[out.dq.dtype] if out.dq is not None else 0, _stream())
    return out


def dequantize(codes: torch.Tensor, scales: torch.Tensor, global_scale: Optional[torch.Tensor],
               fmt="nvfp4", block: int = 16, dtype: torch.dtype = torch.float32,
               out: Optional[torch.Tensor] = None, rot: int = 0) -> torch.Tensor:
    """value(code) * S; with rot > 0 the values are also taken back from the
    rotated domain (fp4q_dequantize_unrotate)."""
    rows, half = codes.shape
    cols = 2 * half
    if out is None:
        out = torch.empty(rows, cols, dtype=dtype, device=codes.device)
    if rot:
        _abi.call("fp4q_dequantize_unrotate", codes.data_ptr(), scales.data_ptr(),
                  _ptr(global_scale), rows, cols, _fmt(fmt), block, rot, out.data_ptr(),
                  DTYPES[out.dtype], _stream())
    else:
        _abi.call("fp4q_dequantize", codes.data_ptr(), scales.data_ptr(), _ptr(global_scale),
                  rows, cols, _fmt(fmt), block, out.data_ptr(), DTYPES[out.dtype], _stream())
    return out


def block_mse(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
              global_scale: Optional[torch.Tensor], fmt="nvfp4", block: int = 16, rot: int = 0,
              out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _check(x, torch.bfloat16, "x")
    rows, cols = x.shape
    if out is None:
        out = torch.empty(rows, cols // block, dtype=torch.float32, device=x.device)
    _abi.call("fp4q_block_mse", x.data_ptr(), codes.data_ptr(), scales.data_ptr(),
              _ptr(global_scale), rows, cols, _fmt(fmt), block, rot, out.data_ptr(), _stream())
    return out


@dataclass
class FocusOut:
    w_hat: torch.Tensor
    global_scale: Optional[torch.Tensor]
    codes: Optional[torch.Tensor]
    scales: Optional[torch.Tensor]


def focus_fwd(w: torch.Tensor, c: torch.Tensor, fmt="nvfp4", block: int = 16, sub: int = 8,
              global_amax: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.bfloat16,
              want_codes: bool = False, out: Optional[FocusOut] = None) -> FocusOut:
    """FOCUS fake quantization W_hat = S_dq * Q(W / (S_dq * c_k))."""
    _check(w, torch.bfloat16, "w")
    _check(c, torch.float16, "c")
    rows, cols = w.shape
    f = _fmt(fmt)
    if out is None:
        dev = w.device
        out = FocusOut(
            w_hat=torch.empty(rows, cols, dtype=out_dtype, device=dev),
            global_scale=torch.empty(1, dtype=torch.float32, device=dev) if f == 0 else None,
            codes=torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev) if want_codes else None,
            scales=torch.empty(rows, cols // block, dtype=torch.uint8, device=dev) if want_codes else None,
        )
    _abi.call("fp4q_focus_fwd", w.data_ptr(), c.data_ptr(), rows, cols, f, block, sub,
              _ptr(global_amax), _ptr(out.global_scale), out.w_hat.data_ptr(),
              DTYPES[out.w_hat.dtype], _ptr(out.codes), _ptr(out.scales), _stream())
    return out


def focus_bwd(w: torch.Tensor, g: torch.Tensor, c: torch.Tensor, sub: int = 8,
              out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Straight-through dL/dc_k = -(sum_k g * W) / c_k^2, fp32 [rows, cols/sub]."""
    _check(w, torch.bfloat16, "w")
    _check(g, torch.bfloat16, "g")
    _check(c, torch.float16, "c")
    rows, cols = w.shape
    if out is None:
        out = torch.empty(rows, cols // sub, dtype=torch.float32, device=w.device)
    _abi.call("fp4q_focus_bwd", w.data_ptr(), g.data_ptr(), c.data_ptr(), rows, cols, sub,
              out.data_ptr(), _stream())
    return out


OPTIMIZERS = {"sgd": 0, "adam": 1}


@dataclass
class FocusState:
    """FOCUS calibration state of one weight: fp32 master coefficients, their
    fp16 copy (what focus_fwd consumes), Adam's moments and step count."""
    c: torch.Tensor                # float32 [rows, cols/sub]
    c_half: torch.Tensor           # float16 [rows, cols/sub]
    m: Optional[torch.Tensor]      # float32 [rows, cols/sub] (Adam) or None
    v: Optional[torch.Tensor]
    opt: str = "adam"
    t: int = 0


def focus_state(rows: int, cols: int, sub: int = 8, opt: str = "adam",
                device=None) -> FocusState:
    """Coefficients initialised to 1 (FOCUS Metodologia §2), moments to 0."""
    n = (rows, cols // sub)
    adam = opt == "adam"
    return FocusState(
        c=torch.ones(n, dtype=torch.float32, device=device),
        c_half=torch.ones(n, dtype=torch.float16, device=device),
        m=torch.zeros(n, dtype=torch.float32, device=device) if adam else None,
        v=torch.zeros(n, dtype=torch.float32, device=device) if adam else None,
        opt=opt)


def _opt_args(state: FocusState, lr, beta1, beta2, eps):
    return (OPTIMIZERS[state.opt], float(lr), float(beta1), float(beta2), float(eps), state.t + 1)


def focus_update(w: torch.Tensor, g: torch.Tensor, state: FocusState, sub: int = 8,
                 lr: float = 1e-3, beta1: float = 0.9, beta2: float = 0.999,
                 eps: float = 1e-8) -> FocusState:
    """One optimizer step of the coefficients from g = dL/dW_hat (bf16), in place."""
    _check(w, torch.bfloat16, "w")
    _check(g, torch.bfloat16, "g")
    _check(state.c, torch.float32, "c")
    _check(state.c_half, torch.float16, "c_half")
    rows, cols = w.shape
    _abi.call("fp4q_focus_update", w.data_ptr(), g.data_ptr(), state.c.data_ptr(),
              state.c_half.data_ptr(), _ptr(state.m), _ptr(state.v), rows, cols, sub,
              *_opt_args(state, lr, beta1, beta2, eps), _stream())
    state.t += 1
    return state


def focus_step(w: torch.Tensor, state: FocusState, fmt="nvfp4", block: int = 16, sub: int = 8,
               global_amax: Optional[torch.Tensor] = None,
               global_scale: Optional[torch.Tensor] = None, want_sse: bool = False,
               lr: float = 1e-3, beta1: float = 0.9, beta2: float = 0.999,
               eps: float = 1e-8) -> Optional[torch.Tensor]:
    """One fused step on sum (W_hat - W)^2, in place; returns the per-sub-block
    SSE before the step (float32 [rows, cols/sub]) when want_sse."""
    _check(w, torch.bfloat16, "w")
    _check(state.c, torch.float32, "c")
    rows, cols = w.shape
    f = _fmt(fmt)
    if f == 0 and global_scale is None:
        global_scale = torch.empty(1, dtype=torch.float32, device=w.device)
    sse = torch.empty(rows, cols // sub, dtype=torch.float32, device=w.device) if want_sse else None
    _abi.call("fp4q_focus_step", w.data_ptr(), rows, cols, f, block, sub, _ptr(global_amax),
              _ptr(global_scale), state.c.data_ptr(), _ptr(state.c_half), _ptr(state.m),
              _ptr(state.v), _ptr(sse), *_opt_args(state, lr, beta1, beta2, eps), _stream())
    state.t += 1
    return sse


def gptq(w: torch.Tensor, scales: torch.Tensor, global_scale: Optional[torch.Tensor],
         U: torch.Tensor, perm: Optional[torch.Tensor] = None, fmt="nvfp4", block: int = 16,
         work: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
         rot: int = 0) -> torch.Tensor:
    """GPTQ error feedback with static groups (fixed block scales); returns the
    packed codes uint8 [rows, cols/2]. U: fp32 [cols, cols] upper Cholesky
    factor of the inverse Hessian in processing order; perm: int32 [cols];
    rot > 0: MR-GPTQ's blockwise rotation first (see fp4q_gptq)."""
    _check(w, torch.bfloat16, "w")
    _check(scales, torch.uint8, "scales")
    _check(U, torch.float32, "U")
    if perm is not None:
        _check(perm, torch.int32, "perm")
    rows, cols = w.shape
    if work is None:
        work = torch.empty(rows, cols, dtype=torch.float32, device=w.device)
    if out is None:
        out = torch.empty(rows, cols // 2, dtype=torch.uint8, device=w.device)
    _abi.call("fp4q_gptq", w.data_ptr(), rows, cols, _fmt(fmt), block, rot, scales.data_ptr(),
              _ptr(global_scale), U.data_ptr(), _ptr(perm), work.data_ptr(), out.data_ptr(),
              _stream())
    return out


def mma_scale_bytes(rows: int, K: int, fmt="nvfp4") -> int:
    n = _abi.load().fp4q_mma_scale_bytes(rows, K, _fmt(fmt))
    if n == 0:
        raise ValueError(f"no MMA scale layout for rows={rows}, K={K}, {fmt}")
    return n


def quantize_mma(x: torch.Tensor, fmt="nvfp4", strategy="absmax", rot: int = 0,
                 global_amax: Optional[torch.Tensor] = None,
                 out: Optional[Quantized] = None) -> Quantized:
    """quantize() with the scales written in the block-scaled MMA layout (block 16
    for NVFP4, 32 for MXFP4): the activation side of gemm() in one launch. The
    returned Quantized holds the flat MMA-layout scale bytes in .scales."""
    _check(x, torch.bfloat16, "x")
    rows, cols = x.shape
    f = _fmt(fmt)
    if out is None:
        dev = x.device
        out = Quantized(
            codes=torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev),
            scales=torch.zeros(mma_scale_bytes(rows, cols, fmt), dtype=torch.uint8, device=dev),
            global_scale=torch.empty(1, dtype=torch.float32, device=dev) if f == 0 else None,
            mse=None, dq=None)
    if global_amax is not None:
        _check(global_amax, torch.float32, "global_amax")
    _abi.call("fp4q_quantize_mma", x.data_ptr(), rows, cols, f, _strat(strategy), rot,
              _ptr(global_amax), _ptr(out.global_scale), out.codes.data_ptr(), out.scales.data_ptr(),
              _stream())
    return out


def scales_to_mma(scales: torch.Tensor, K: int, fmt="nvfp4",
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Row-major block scales [rows, K/block] -> the block-scaled MMA layout
    (flat uint8 of mma_scale_bytes(rows, K, fmt) bytes)."""
    _check(scales, torch.uint8, "scales")
    rows = scales.shape[0]
    if out is None:
        out = torch.empty(mma_scale_bytes(rows, K, fmt), dtype=torch.uint8, device=scales.device)
    _abi.call("fp4q_scales_to_mma", scales.data_ptr(), rows, K, _fmt(fmt), out.data_ptr(), _stream())
    return out


def gemm(a_codes: torch.Tensor, a_mma_scales: torch.Tensor, a_global_scale: Optional[torch.Tensor],
         b_codes: torch.Tensor, b_mma_scales: torch.Tensor, b_global_scale: Optional[torch.Tensor],
         fmt="nvfp4", out_dtype: torch.dtype = torch.bfloat16, out: Optional[torch.Tensor] = None,
         alpha_out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """W4A4 GEMM on the block-scaled tensor cores: [M, K] x [N, K]^T -> [M, N].
    Codes as written by quantize; scales converted by scales_to_mma."""
    for t, nm in ((a_codes, "a_codes"), (b_codes, "b_codes"), (a_mma_scales, "a_mma_scales"),
                  (b_mma_scales, "b_mma_scales")):
        _check(t, torch.uint8, nm)
    M, K = a_codes.shape[0], 2 * a_codes.shape[1]
    N = b_codes.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=a_codes.device)
    if alpha_out is None:
        alpha_out = torch.empty(1, dtype=torch.float32, device=a_codes.device)
    _abi.call("fp4q_gemm", a_codes.data_ptr(), a_mma_scales.data_ptr(), _ptr(a_global_scale),
              b_codes.data_ptr(), b_mma_scales.data_ptr(), _ptr(b_global_scale), M, N, K, _fmt(fmt),
              alpha_out.data_ptr(), out.data_ptr(), DTYPES[out.dtype], _stream())
    return out


def gemm_noalloc(a_codes: torch.Tensor, a_mma_scales: torch.Tensor,
                 a_global_scale: Optional[torch.Tensor], b_codes: torch.Tensor,
                 b_mma_scales: torch.Tensor, b_global_scale: Optional[torch.Tensor], fmt="nvfp4",
                 out: Optional[torch.Tensor] = None,
                 out_dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """gemm() using the library's own scratch float for alpha (no alpha_out);
    overlapping calls on one device race on it (see fp4q_gemm_noalloc)."""
    for t, nm in ((a_codes, "a_codes"), (b_codes, "b_codes"), (a_mma_scales, "a_mma_scales"),
                  (b_mma_scales, "b_mma_scales")):
        _check(t, torch.uint8, nm)
    M, K = a_codes.shape[0], 2 * a_codes.shape[1]
    N = b_codes.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=a_codes.device)
    _abi.call("fp4q_gemm_noalloc", a_codes.data_ptr(), a_mma_scales.data_ptr(), _ptr(a_global_scale),
              b_codes.data_ptr(), b_mma_scales.data_ptr(), _ptr(b_global_scale), M, N, K, _fmt(fmt),
              out.data_ptr(), DTYPES[out.dtype], _stream())
    return out


def global_amax(x: torch.Tensor, rot: int = 0, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _check(x, torch.bfloat16, "x")
    rows, cols = x.shape
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _abi.call("fp4q_global_amax", x.data_ptr(), rows, cols, rot, out.data_ptr(), _stream())
    return out


def e2m1_encode(u: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _check(u, torch.float32, "u")
    if out is None:
        out = torch.empty(u.shape, dtype=torch.uint8, device=u.device)
    _abi.call("fp4q_e2m1_encode", u.data_ptr(), u.numel(), out.data_ptr(), _stream())
    return out


def e4m3_encode(v: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _check(v, torch.float32, "v")
    if out is None:
        out = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _abi.call("fp4q_e4m3_encode", v.data_ptr(), v.numel(), out.data_ptr(), _stream())
    return out
