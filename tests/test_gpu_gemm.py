"""W4A4 FP4 GEMM on the block-scaled tensor cores (fp4q_gemm) against the
oracle's double-precision product of the same codes and scales ("Bridging
the Gap Between Promise and Performance for Microscaling FP4 Quantization",
技術概要 §2.3), and the scale-layout conversion it reads, byte for byte.

The tensor cores accumulate in fp32 in an order the hardware fixes, so the
GEMM bar is the fp32 summation bound: |D - D_ref| <= K 2^-24 sum_k |a_k b_k|
|alpha| (+ the bf16 rounding of the output when bf16 is requested).
"""
import numpy as np
import pytest
import torch

import oracle
from microscaling_fp4_quantization_bf16_b200 import synth

pytestmark = pytest.mark.gpu


def mma_offsets(rows, nkb):
    """Byte offset of (row r, block j) in the MMA scale layout: 512-byte atoms of
    128 rows x 4 blocks, row r at 16 (r % 32) + 4 ((r / 32) % 4), block j at + j % 4,
    atoms along K first."""
    rows_pad = -(-rows // 128) * 128
    kb_pad = -(-nkb // 4) * 4
    r = np.arange(rows_pad)[:, None]
    j = np.arange(kb_pad)[None, :]
    off = ((r // 128) * (kb_pad // 4) + j // 4) * 512 + 16 * (r % 32) + 4 * ((r // 32) % 4) + j % 4
    return off, rows_pad, kb_pad


@pytest.mark.parametrize("fmt,block", [("nvfp4", 16), ("mxfp4", 32)])
@pytest.mark.parametrize("rows,K", [(128, 64), (300, 96), (5, 512)])
def test_scales_to_mma_layout(gpu, fmt, block, rows, K):
    rng = np.random.default_rng(rows + K)
    sc = rng.integers(1, 255, (rows, K // block), dtype=np.uint8)
    out = gpu.scales_to_mma(torch.from_numpy(sc).cuda(), K, fmt)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    off, rows_pad, kb_pad = mma_offsets(rows, K // block)
    assert got.size == rows_pad * kb_pad == gpu.mma_scale_bytes(rows, K, fmt)
    want = np.zeros(rows_pad * kb_pad, np.uint8)
    padded = np.zeros((rows_pad, kb_pad), np.uint8)
    padded[:rows, :K // block] = sc
    want[off.reshape(-1)] = padded.reshape(-1)
    assert np.array_equal(got, want)


def gemm_case(gpu, fmt, block, M, N, K, out_dtype, seed):
    a = synth.laplace_outliers(M, K, seed=seed)
    w = synth.gaussian(N, K, seed=seed + 1, std=0.02)
    qa = gpu.quantize(a.cuda(), fmt, block, "absmax", 0)
    qw = gpu.quantize(w.cuda(), fmt, block, "absmax", 0)
    sa = gpu.scales_to_mma(qa.scales, K, fmt)
    sw = gpu.scales_to_mma(qw.scales, K, fmt)
    d = gpu.gemm(qa.codes, sa, qa.global_scale, qw.codes, sw, qw.global_scale, fmt, out_dtype)
    torch.cuda.synchronize()
    ga = None if qa.global_scale is None else float(qa.global_scale.item())
    gw = None if qw.global_scale is None else float(qw.global_scale.item())
    ac, asc = qa.codes.cpu().numpy(), qa.scales.cpu().numpy()
    wc, wsc = qw.codes.cpu().numpy(), qw.scales.cpu().numpy()
    want = oracle.fp4_gemm(ac, asc, ga, wc, wsc, gw, fmt).astype(np.float64)
    da = oracle.dequantize(ac, asc, 1.0, M, K, fmt, block).astype(np.float64)
    dw = oracle.dequantize(wc, wsc, 1.0, N, K, fmt, block).astype(np.float64)
    alpha = (ga * gw) if fmt == "nvfp4" else 1.0
    mag = (np.abs(da) @ np.abs(dw).T) * abs(alpha)
    got = d.float().cpu().numpy().astype(np.float64)
    tol = K * 2.0 ** -24 * mag + 1e-30
    if out_dtype == torch.bfloat16:
        tol = tol + 2.0 ** -8 * np.abs(want)
    return got, want, tol


@pytest.mark.parametrize("fmt,block", [("nvfp4", 16), ("mxfp4", 32)])
@pytest.mark.parametrize("M,N,K", [(256, 384, 512), (200, 136, 352), (1, 8, 32), (640, 256, 2048)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_matches_oracle(gpu, fmt, block, M, N, K, out_dtype):
    if out_dtype == torch.float32 and N % 4 or out_dtype == torch.bfloat16 and N % 8:
        pytest.skip("output rows must be 16-byte multiples")
    got, want, tol = gemm_case(gpu, fmt, block, M, N, K, out_dtype, seed=M + N + K)
    bad = np.abs(got - want) > tol
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the fp32 summation bound"


@pytest.mark.parametrize("fmt,block,strat,rot", [("nvfp4", 16, "absmax", 0), ("nvfp4", 16, "four_over_six", 16),
                                                 ("mxfp4", 32, "absmax", 32), ("mxfp4", 32, "brute_force", 0)])
@pytest.mark.parametrize("rows,cols", [(300, 256), (128, 2048), (7, 64)])
def test_quantize_mma_equals_quantize_then_convert(gpu, fmt, block, strat, rot, rows, cols):
    """The fused quantizer writes the same codes as quantize() and the same scale
    bytes as scales_to_mma() of its row-major scales (padding zero)."""
    if cols % max(rot, 1):
        pytest.skip("cols must be a multiple of the rotation")
    x = synth.laplace_outliers(rows, cols, seed=rows + cols).cuda()
    q = gpu.quantize(x, fmt, block, strat, rot)
    conv = gpu.scales_to_mma(q.scales, cols, fmt)
    f = gpu.quantize_mma(x, fmt, strat, rot)
    torch.cuda.synchronize()
    assert np.array_equal(f.codes.cpu().numpy(), q.codes.cpu().numpy())
    assert np.array_equal(f.scales.cpu().numpy(), conv.cpu().numpy())
    if fmt == "nvfp4":
        assert f.global_scale.item() == q.global_scale.item()


@pytest.mark.parametrize("fmt,block", [("nvfp4", 16), ("mxfp4", 32)])
def test_gemm_benchmarked_shape_sampled_rows(gpu, fmt, block):
    """The benchmarked LLM layer, 8192 x 4096 x 14336 with bf16 output: 2048
    output tiles of 128 x 128 through the persistent tile scheduler (many
    waves on 148 SMs) and 56 K iterations of 256 each. Sampled rows of D,
    spread over the M tiles (first and last included), against the oracle's
    product of the same codes and scales, within the fp32 summation bound."""
    M, N, K = 8192, 4096, 14336
    a = synth.laplace_outliers(M, K, seed=21)
    w = synth.gaussian(N, K, seed=22, std=0.02)
    qa = gpu.quantize(a.cuda(), fmt, block, "absmax", 0)
    qw = gpu.quantize(w.cuda(), fmt, block, "absmax", 0)
    del a, w
    sa = gpu.scales_to_mma(qa.scales, K, fmt)
    sw = gpu.scales_to_mma(qw.scales, K, fmt)
    d = gpu.gemm(qa.codes, sa, qa.global_scale, qw.codes, sw, qw.global_scale, fmt, torch.bfloat16)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([np.linspace(0, M - 1, 16).astype(np.int64),
                                     rng.choice(M, 8, replace=False)]))
    ga = None if qa.global_scale is None else float(qa.global_scale.item())
    gw = None if qw.global_scale is None else float(qw.global_scale.item())
    ridx = torch.from_numpy(rows).cuda()
    ac = qa.codes[ridx].cpu().numpy()
    asc = qa.scales[ridx].cpu().numpy()
    wc, wsc = qw.codes.cpu().numpy(), qw.scales.cpu().numpy()
    want = oracle.fp4_gemm(ac, asc, ga, wc, wsc, gw, fmt).astype(np.float64)
    da = np.abs(oracle.dequantize(ac, asc, 1.0, len(rows), K, fmt, block)).astype(np.float64)
    mag = np.empty((len(rows), N))
    for n0 in range(0, N, 512):
        dw = oracle.dequantize(wc[n0:n0 + 512], wsc[n0:n0 + 512], 1.0, 512, K, fmt, block)
        mag[:, n0:n0 + 512] = da @ np.abs(dw).astype(np.float64).T
    alpha = (ga * gw) if fmt == "nvfp4" else 1.0
    got = d[ridx].float().cpu().numpy().astype(np.float64)
    tol = K * 2.0 ** -24 * mag * abs(alpha) + 2.0 ** -8 * np.abs(want) + 1e-30
    bad = np.abs(got - want) > tol
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the fp32 summation bound"
    assert np.abs(want).max() > 0
