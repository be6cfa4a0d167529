"""Brute-force scale search (every E4M3 code 0x01..0x7E, strictly lower SSE
wins, ties keep the lower code; "Finer is Better (with the Right Scaling)",
手法 2) on blocks built to stress a search that skips codes: ties at zero
error, blocks exactly on the E2M1 grid, constant and sparse blocks, heavy
tails, and some rows 8 to 40 octaves below the others so that their blocks
sit in the E4M3 subnormal range or collapse to the lowest code. GPU vs the oracle's exhaustive loop,
bit-exact (scale bytes, codes, MSE).
"""
import numpy as np
import pytest

from microscaling_fp4_quantization_bf16_b200 import synth

from test_gpu_parity import compare_quant, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])


def stress_rows(rows, cols, seed):
    rng = np.random.default_rng(seed)
    out = np.empty((rows, cols))
    for i in range(rows):
        k = i % 8
        if k == 0:
            v = rng.standard_normal(cols)
        elif k == 1:
            v = rng.uniform(-1, 1, cols)
        elif k == 2:  # constant blocks of random sign
            v = np.full(cols, rng.uniform(0.1, 10)) * rng.choice([-1, 1], cols)
        elif k == 3:  # three distinct magnitudes
            v = rng.choice(rng.uniform(0.01, 5, 3), cols) * rng.choice([-1, 1], cols)
        elif k == 4:  # one nonzero per 4 elements
            v = np.zeros(cols)
            v[::4] = rng.standard_normal(cols // 4)
        elif k == 5:  # magnitudes spread over 20 octaves
            v = 2.0 ** rng.uniform(-20, 0, cols) * rng.choice([-1, 1], cols)
        elif k == 6:  # exactly E2M1 grid values times one scale: zero-error ties
            v = rng.choice(GRID, cols) * rng.choice([-1, 1], cols) * 2.0 ** rng.integers(-6, 6)
        else:  # very heavy tails
            v = rng.standard_t(1.5, cols)
        # most rows within 8 octaves of the largest, every 16th far below it
        out[i] = v * 2.0 ** (rng.uniform(-40, -8) if i % 16 == 15 else rng.uniform(-8, 0))
    return synth.to_bf16(out)


@pytest.mark.parametrize("block", [4, 8, 16, 32])
@pytest.mark.parametrize("rot", [0, 16])
@pytest.mark.parametrize("gamax", [None, 1.0])
def test_brute_force_stress(gpu, block, rot, gamax):
    x = stress_rows(2048, 64, seed=100 + block + rot)
    g = gpu_quantize(gpu, x, "nvfp4", block, "brute_force", rot, gamax=gamax, mse=True)
    o = oracle_quantize(x, "nvfp4", block, "brute_force", rot, gamax=gamax, mse=True)
    compare_quant(g, o, "nvfp4", f"brute B{block} H{rot} gamax={gamax}")


@pytest.mark.parametrize("rot", [0, 32, 128])
def test_mxfp4_mse_grid_stress(gpu, rot):
    """The MXFP4 MSE-optimised E8M0 scale ("Bridging the Gap ...", 技術概要
    §2.2 item 1) on the same stress rows: GPU vs the oracle's scan of all
    255 bytes."""
    x = stress_rows(2048, 128, seed=300 + rot)
    g = gpu_quantize(gpu, x, "mxfp4", 32, "brute_force", rot, mse=True)
    o = oracle_quantize(x, "mxfp4", 32, "brute_force", rot, mse=True)
    compare_quant(g, o, "mxfp4", f"mxfp4 mse grid H{rot}")


def test_mxfp4_mse_grid_full_size_sampled(gpu):
    """C2 (4096x4096 Laplace + outliers) with the MSE-optimised E8M0 scale, rot
    0 and 32: every element of 64 sampled rows (MXFP4 needs no tensor-wide
    value, so a row's result depends on that row only)."""
    x = synth.workload("c2_mxfp4_laplace_outliers")["x"]
    rows = np.random.default_rng(3).choice(x.shape[0], 64, replace=False)
    for rot in (0, 32):
        g = gpu_quantize(gpu, x, "mxfp4", 32, "brute_force", rot, mse=True)
        o = oracle_quantize(x[rows], "mxfp4", 32, "brute_force", rot, mse=True)
        for k in ("codes", "scales", "mse"):
            g[k] = g[k][rows]
        compare_quant(g, o, "mxfp4", f"C2 mse grid H{rot}")
