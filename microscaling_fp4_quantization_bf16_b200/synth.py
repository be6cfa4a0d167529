"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no quantization arithmetic: it only draws random numbers
(numpy ``default_rng`` / PCG64, float64), casts them to float32 and then to
bf16 (or fp16) with round-to-nearest-even. The same bytes are given to the
CUDA library and to the oracle.

Distributions follow the pages' descriptions of LLM tensors: Gaussian data for
the block-size study ("Finer is Better", 手法 1), Laplace weights/activations
before rotation ("Bridging the Gap ...", 技術概要 §2.1), heavy-tailed
Student-t tensors, rare large outliers and a few high-magnitude hidden
channels (the MXFP4 failure modes on the TORQ page, 問題定義 items 1-2).
"""
from __future__ import annotations

import numpy as np
import torch

# Full-size workloads: name -> (rows, cols)
SHAPES = {
    "c1_nvfp4_roundtrip": (1024, 1024),
    "c2_mxfp4_laplace_outliers": (4096, 4096),
    "c3_strategy_sweep_t3": (4096, 14336),
    "c4_focus": (4096, 4096),
    "c5_activation_channels": (16384, 8192),
}


def to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def to_fp16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.float16)


def gaussian(rows: int, cols: int, seed: int, std: float = 1.0) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    return to_bf16(rng.normal(0.0, std, size=(rows, cols)))


def laplace_outliers(rows: int, cols: int, seed: int, b: float = 0.02, frac: float = 0.001,
                     mult: float = 50.0) -> torch.Tensor:
    """Laplace(0, b) with round(frac * N) uniformly chosen entries times mult."""
    rng = np.random.default_rng(seed)
    a = rng.laplace(0.0, b, size=(rows, cols))
    n = rows * cols
    k = int(round(frac * n))
    if k:
        idx = rng.choice(n, k, replace=False)
        a.reshape(-1)[idx] *= mult
    return to_bf16(a)


def student_t(rows: int, cols: int, seed: int, nu: float = 3.0, scale: float = 0.02) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    return to_bf16(rng.standard_t(nu, size=(rows, cols)) * scale)


def laplace_channels(rows: int, cols: int, seed: int, b: float = 1.0, frac: float = 0.01,
                     mult: float = 20.0) -> torch.Tensor:
    """Laplace(0, b) activations with round(frac * cols) hidden channels times mult."""
    rng = np.random.default_rng(seed)
    a = rng.laplace(0.0, b, size=(rows, cols))
    k = int(round(frac * cols))
    if k:
        ch = rng.choice(cols, k, replace=False)
        a[:, ch] *= mult
    return to_bf16(a)


def focus_coeffs(rows: int, cols: int, sub: int, seed: int, lo: float = 0.9,
                 hi: float = 1.1) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    return to_fp16(rng.uniform(lo, hi, size=(rows, cols // sub)))


def gptq_problem(rows: int, cols: int, tokens: int, seed: int, damp: float = 0.01,
                 act_order: bool = True, rot: int = 0) -> dict:
    """Inputs of the GPTQ error-feedback step for one synthetic linear layer:
    W ~ N(0, 0.02^2) bf16 [rows, cols]; calibration inputs X [tokens, cols] with
    per-channel scales U[0.1, 2.1], 1% of the channels x20 and a random mixing
    (I + 0.3 N(0,1)/sqrt(cols)) so that channels correlate; the damped Hessian
    H = X^T X / tokens + damp * mean(diag) * I; the processing order (columns by
    decreasing diag(H) when act_order, else the identity); and the upper
    Cholesky factor U of H^-1 in that order, all computed in float64 and
    handed over as fp32 / int32 (the caller's preparation). rot > 0: the
    calibration inputs are taken in the rotated basis X R (R the block-diagonal
    normalised Sylvester Hadamard of width rot), so h, perm and u are those of
    R H R (h_orig keeps H); the weights stay as drawn (the rotation of W is the
    quantizer's own, applied by the GPTQ call)."""
    rng = np.random.default_rng(seed)
    w = gaussian(rows, cols, seed=seed + 1, std=0.02)
    x = rng.standard_normal((tokens, cols)) * rng.uniform(0.1, 2.1, cols)
    x[:, rng.choice(cols, max(1, cols // 100), replace=False)] *= 20
    x = x @ (np.eye(cols) + 0.3 * rng.standard_normal((cols, cols)) / np.sqrt(cols))
    h = x.T @ x / tokens
    h += damp * float(np.mean(np.diag(h))) * np.eye(cols)
    out = {"w": w}
    if rot:
        # the damping term commutes with R (R R = I, and the trace is invariant)
        import scipy.linalg
        r = np.kron(np.eye(cols // rot), scipy.linalg.hadamard(rot) / np.sqrt(rot))
        out["h_orig"] = h
        h = r @ h @ r
    perm = np.argsort(-np.diag(h), kind="stable") if act_order else np.arange(cols)
    hp = h[np.ix_(perm, perm)]
    u = np.linalg.cholesky(np.linalg.inv(hp)).T     # upper: H^-1 = U^T U
    out.update({"h": h, "perm": perm.astype(np.int32), "u": np.ascontiguousarray(u, np.float32)})
    return out


def workload(name: str, rows: int | None = None, cols: int | None = None) -> dict:
    """Tensors of one named workload; rows/cols override the full size (same
    distribution and seeds, smaller shape)."""
    R, Cc = SHAPES[name]
    R = R if rows is None else rows
    Cc = Cc if cols is None else cols
    if name == "c1_nvfp4_roundtrip":
        return {"x": gaussian(R, Cc, seed=0, std=1.0)}
    if name == "c2_mxfp4_laplace_outliers":
        return {"x": laplace_outliers(R, Cc, seed=1, b=0.02, frac=0.001, mult=50.0)}
    if name == "c3_strategy_sweep_t3":
        return {"x": student_t(R, Cc, seed=2, nu=3.0, scale=0.02)}
    if name == "c4_focus":
        return {"w": gaussian(R, Cc, seed=3, std=0.02),
                "c": focus_coeffs(R, Cc, 8, seed=4),
                "g": gaussian(R, Cc, seed=5, std=1.0)}
    if name == "c5_activation_channels":
        return {"x": laplace_channels(R, Cc, seed=6, b=1.0, frac=0.01, mult=20.0)}
    raise KeyError(name)


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16/fp16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
