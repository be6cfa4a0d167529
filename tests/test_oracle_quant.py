"""Pins of the oracle's quantizer, scale strategies, dequantizer, MSE and FOCUS.

Pages: "Finer is Better (with the Right Scaling)" (手法 1-2: E2M1 data, E4M3
scales, block sizes 4/8/16/32, abs-max / prevent-zero / 4-over-6 / brute force
/ hierarchical scaling; 主要な発見と結果: prevent-zero removes the underflow
spike, 4-over-6 lowers MSE, brute force improves strictly with finer blocks);
"Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization" (技術概要 §1: MXFP4 E8M0 scales; §2.1: rotation helps MXFP4
under RTN); "FOCUS: FP4 Optimization via Coupled-Relaxation and
Dual-Granularity Scaling" (Metodologia §1-§4).
"""
import math

import numpy as np
import pytest
import torch

from microscaling_fp4_quantization_bf16_b200 import synth

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def bf16_bits(a):
    return synth.bits16(synth.to_bf16(np.asarray(a, np.float64)))


def f32_of_bf16(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def e4m3_table(ref):
    return np.array([ref.e4m3_value(c) for c in range(0x7F)], np.float64)


# --------------------------------------------------------------- hand examples

def test_packing_and_scale_hand_example(ref):
    # s_g = 2688 / 2688 = 1; block max 6 -> raw = 6 / (6 * 1) = 1 -> E4M3 code 0x38,
    # S = 1, r = 1; element codes are then the E2M1 codes of the values themselves.
    y = [0.5, 1, 1.5, 2, 3, 4, 6, 0, -0.5, -1, -1.5, -2, -3, -4, -6, -0.0]
    x = bf16_bits([y])
    out = ref.quantize(x, "nvfp4", 16, "absmax", 0, global_amax=2688.0, dq="f32")
    assert out["global_scale"] == 1.0
    assert out["scales"].tolist() == [[0x38]]
    # element 2j -> low nibble, 2j+1 -> high nibble
    assert out["codes"].tolist() == [[0x21, 0x43, 0x65, 0x07, 0xA9, 0xCB, 0xED, 0x8F]]
    assert out["mse"].tolist() == [[0.0]]
    assert np.array_equal(out["dq"].view(np.uint32), np.array([y], np.float32).view(np.uint32))


def test_mxfp4_hand_example(ref):
    # block max 5.0 -> floor(log2 5) - 2 = 0 -> byte 127, S = 1; 5 -> tie 4/6 -> 4
    y = [5.0, -0.25, 0.75, 2.5] + [0.0] * 28
    out = ref.quantize(bf16_bits([y]), "mxfp4", 32, "absmax", 0, dq="f32")
    assert out["scales"].tolist() == [[127]]
    codes = ref.unpack_codes(out["codes"])[0]
    assert codes[:4].tolist() == [6, 8, 2, 4]  # 4, -0, 1, 2
    assert out["dq"][0, :4].tolist() == [4.0, -0.0, 1.0, 2.0]
    sse = (5 - 4) ** 2 + 0.25 ** 2 + 0.25 ** 2 + 0.5 ** 2
    assert out["mse"][0, 0] == np.float32(sse / 32)


# ------------------------------------------------------------------ round trips

@pytest.mark.parametrize("block", [4, 8, 16, 32])
@pytest.mark.parametrize("strategy", ["absmax", "prevent_zero", "four_over_six", "brute_force"])
def test_nvfp4_exact_round_trip(ref, block, strategy):
    rng = np.random.default_rng(block)
    rows, cols = 8, 64
    nb = cols // block
    c = rng.integers(1, 0x7F, size=(rows, nb))
    q = rng.integers(0, 16, size=(rows, cols))
    # force one element of every block to +-6 so the block abs-max is 6 * e4m3(c)
    q.reshape(rows, nb, block)[:, :, 0] = rng.choice([7, 15], size=(rows, nb))
    S = e4m3_table(ref)[c]
    y = E2M1[q] * np.repeat(S, block, axis=1)
    x = bf16_bits(y)
    assert np.array_equal(f32_of_bf16(x).astype(np.float64), y)  # exactly representable
    out = ref.quantize(x, "nvfp4", block, strategy, 0, global_amax=2688.0, dq="f32")
    assert np.array_equal(out["scales"], c.astype(np.uint8))
    assert np.array_equal(ref.unpack_codes(out["codes"]), q.astype(np.uint8))
    assert np.array_equal(out["dq"].astype(np.float64), y)
    assert np.all(out["mse"] == 0)


def test_mxfp4_exact_round_trip(ref):
    rng = np.random.default_rng(7)
    rows, cols = 16, 128
    e = rng.integers(-120, 120, size=(rows, cols // 32))
    q = rng.integers(0, 16, size=(rows, cols))
    q.reshape(rows, -1, 32)[:, :, 0] = rng.choice([6, 7, 14, 15], size=e.shape)  # max |val| in {4, 6}
    y = E2M1[q] * np.repeat(2.0 ** e, 32, axis=1)
    x = bf16_bits(y)
    out = ref.quantize(x, "mxfp4", 32, "absmax", 0, dq="f32")
    assert np.array_equal(out["scales"].astype(np.int64), e + 127)
    assert np.array_equal(ref.unpack_codes(out["codes"]), q.astype(np.uint8))
    assert np.array_equal(out["dq"].astype(np.float64), y)


# -------------------------------------------------------------- scales & zeros

def test_global_scale_closed_form(ref):
    x = synth.workload("c1_nvfp4_roundtrip", rows=64, cols=256)["x"]
    xb = synth.bits16(x)
    amax = np.abs(x.float().numpy()).max()  # library max over the widened tensor
    assert ref.global_amax(xb, 0) == amax
    out = ref.quantize(xb, "nvfp4", 16, "absmax", 0)
    assert out["global_scale"] == np.float32(amax) / np.float32(2688.0)
    assert ref.global_scale(0.0) == 1.0 and ref.global_scale(-1.0) == 1.0
    assert ref.global_scale(float("inf")) == 1.0 and ref.global_scale(float("nan")) == 1.0


def test_zero_tensor(ref):
    x = np.zeros((4, 64), np.uint16)
    nv = ref.quantize(x, "nvfp4", 16, "absmax", 0, dq="f32")
    assert nv["global_scale"] == 1.0
    assert np.all(nv["scales"] == 0) and np.all(nv["codes"] == 0) and np.all(nv["mse"] == 0)
    assert np.all(nv["dq"].view(np.uint32) == 0)
    pz = ref.quantize(x, "nvfp4", 16, "prevent_zero", 0)
    assert np.all(pz["scales"] == 1) and np.all(pz["codes"] == 0)
    mx = ref.quantize(x, "mxfp4", 32, "absmax", 0)
    assert np.all(mx["scales"] == 0) and np.all(mx["codes"] == 0)


def test_mxfp4_scale_bytes_from_frexp(ref):
    x = synth.workload("c2_mxfp4_laplace_outliers", rows=32, cols=512)["x"]
    xb = synth.bits16(x)
    for rot in (0, 32, 128):
        y = f32_of_bf16(xb)
        if rot:
            y = ref.fwht(y.reshape(-1, rot), rot).reshape(y.shape)
        amax = np.abs(y.reshape(32, -1, 32)).max(axis=2)
        want = np.array([[max(-127, min(127, math.frexp(float(a))[1] - 1 - 2)) + 127 if a > 0
                          else 0 for a in row] for row in amax])
        out = ref.quantize(xb, "mxfp4", 32, "absmax", rot)
        assert np.array_equal(out["scales"].astype(np.int64), want)


# ------------------------------------------------------------------ strategies

def _with_tiny_rows(x: torch.Tensor) -> torch.Tensor:
    a = x.float().numpy().copy()
    a[::4] *= 1e-6  # blocks far below the tensor abs-max: their E4M3 scale underflows
    return synth.to_bf16(a)


@pytest.mark.parametrize("block", [4, 8, 16, 32])
def test_strategy_relations_exact(ref, block):
    x = _with_tiny_rows(synth.workload("c3_strategy_sweep_t3", rows=32, cols=256)["x"])
    xb = synth.bits16(x)
    res = {s: ref.quantize(xb, "nvfp4", block, s, 0, dq="f32")
           for s in ("absmax", "prevent_zero", "four_over_six", "brute_force")}
    am, pz, fs, bf = (res[s] for s in ("absmax", "prevent_zero", "four_over_six", "brute_force"))
    sg = am["global_scale"]
    assert all(r["global_scale"] == sg for r in res.values())
    # prevent-zero never stores scale 0 and equals abs-max whenever abs-max's code >= 1
    assert np.all(pz["scales"] >= 1)
    same = am["scales"] >= 1
    assert np.any(~same), "the data must exercise the underflow regime"
    assert np.array_equal(pz["scales"][same], am["scales"][same])
    assert np.array_equal(pz["mse"][same], am["mse"][same])
    # ...and removes the underflow-to-zero error spike: never worse, element by element
    assert np.all(pz["mse"][~same] <= am["mse"][~same])
    assert np.mean(pz["mse"][~same]) < np.mean(am["mse"][~same])
    # 4-over-6: never worse than abs-max (its target-6 candidate IS abs-max)
    assert np.all(fs["mse"] <= am["mse"])
    moved = fs["scales"] != am["scales"]
    assert np.any(moved)
    assert np.all(fs["mse"][moved] < am["mse"][moved])  # target 4 only on a strict gain
    # brute force: the minimum over every positive code, so never worse than any
    # strategy that stores a positive code
    pos = fs["scales"] >= 1
    assert np.all(bf["mse"] <= pz["mse"]) and np.all(bf["mse"][pos] <= fs["mse"][pos])
    assert np.all(bf["scales"] >= 1)
    # dequantize / block_mse reproduce quantize's own outputs bit for bit
    for r in res.values():
        dq = ref.dequantize(r["codes"], r["scales"], sg, *xb.shape, "nvfp4", block, "f32")
        assert np.array_equal(dq.view(np.uint32), r["dq"].view(np.uint32))
        m = ref.block_mse(xb, r["codes"], r["scales"], sg, "nvfp4", block, 0)
        assert np.array_equal(m.view(np.uint32), r["mse"].view(np.uint32))
        # the MSE is the mean squared error, checked in float64
        err = (f32_of_bf16(xb).astype(np.float64) - r["dq"]) ** 2
        want = err.reshape(err.shape[0], -1, block).mean(axis=2)
        assert np.allclose(r["mse"], want, rtol=1e-5, atol=1e-45)


def _nearest_e2m1_double(u):
    mags = np.abs(E2M1[:8])
    a = np.minimum(np.abs(u), 6.0)
    idx = np.argmin(np.abs(a[..., None] - mags), axis=-1)
    return np.sign(u) * mags[idx]


def test_brute_force_is_minimum_in_double(ref):
    rng = np.random.default_rng(21)
    tab = e4m3_table(ref)
    for block in (4, 8):
        x = bf16_bits(rng.standard_t(3, size=(4, 8 * block)) * 0.02)
        out = ref.quantize(x, "nvfp4", block, "brute_force", 0)
        sg = float(out["global_scale"])
        y = f32_of_bf16(x).astype(np.float64).reshape(-1, block)
        S = tab[1:0x7F][:, None, None] * sg  # [126, 1, 1]
        sse = ((y[None] - _nearest_e2m1_double(y[None] / S) * S) ** 2).sum(axis=2)  # [126, nblk]
        best = sse.min(axis=0)
        chosen = sse[out["scales"].reshape(-1).astype(np.int64) - 1, np.arange(y.shape[0])]
        assert np.all(chosen <= best * (1 + 1e-5) + 1e-30)


def test_finer_is_better_exact_and_statistical(ref):
    x = synth.workload("c1_nvfp4_roundtrip", rows=64, cols=512)["x"]  # Gaussian data
    xb = synth.bits16(x)
    sse, means = {}, {}
    for B in (4, 8, 16, 32):
        o = ref.quantize(xb, "nvfp4", B, "brute_force", 0)
        sse[B] = o["mse"].astype(np.float32) * np.float32(B)  # exact: B is a power of two
        means[B] = float(np.mean(o["mse"]))
    for B in (4, 8, 16):
        l, r = sse[B][:, 0::2], sse[B][:, 1::2]
        assert np.all((l + r).astype(np.float32) <= sse[2 * B])
    assert means[4] < means[8] < means[16] < means[32]


def test_hadamard_helps_mxfp4_on_laplace_outliers(ref):
    x = synth.bits16(synth.workload("c2_mxfp4_laplace_outliers", rows=256, cols=1024)["x"])
    m0 = ref.quantize(x, "mxfp4", 32, "absmax", 0)["mse"].mean()
    m32 = ref.quantize(x, "mxfp4", 32, "absmax", 32)["mse"].mean()
    assert m32 < m0


# ----------------------------------------------------------------------- FOCUS

@pytest.mark.parametrize("fmt,block", [("nvfp4", 16), ("mxfp4", 32)])
def test_focus_unit_coefficients_equal_absmax_round_trip(ref, fmt, block):
    d = synth.workload("c4_focus", rows=32, cols=256)
    w = synth.bits16(d["w"])
    ones = synth.bits16(torch.ones(32, 256 // 8, dtype=torch.float16))
    f = ref.focus_fwd(w, ones, fmt, block, 8, out="f32")
    q = ref.quantize(w, fmt, block, "absmax", 0, dq="f32")
    assert np.array_equal(f["w_hat"].view(np.uint32), q["dq"].view(np.uint32))
    assert np.array_equal(f["codes"], q["codes"]) and np.array_equal(f["scales"], q["scales"])
    fb = ref.focus_fwd(w, ones, fmt, block, 8, out="bf16")
    qb = ref.quantize(w, fmt, block, "absmax", 0, dq="bf16")
    assert np.array_equal(fb["w_hat"], qb["dq"])


def test_focus_hand_example(ref):
    # s_g = 1 (amax 2688 supplied); block max 6 -> S_dq = 1. Sub-block 0 has c = 1,
    # sub-block 1 has c = 2: u = W * (1 / 2), so 6 -> 3 and 3 -> 1.5, dequantized
    # with S_dq = 1 (the coefficient is not stored).
    w = [6, 3, 0, 0, 0, 0, 0, 0, 6, 3, 1, 0, 0, 0, 0, 0]
    c = synth.bits16(torch.tensor([[1.0, 2.0]], dtype=torch.float16))
    f = ref.focus_fwd(bf16_bits([w]), c, "nvfp4", 16, 8, global_amax=2688.0, out="f32")
    assert f["scales"].tolist() == [[0x38]]
    assert f["w_hat"][0].tolist() == [6, 3, 0, 0, 0, 0, 0, 0, 3, 1.5, 0.5, 0, 0, 0, 0, 0]


def test_focus_coefficients_are_local_and_monotone(ref):
    d = synth.workload("c4_focus", rows=16, cols=128)
    w = synth.bits16(d["w"])
    c = d["c"].clone()
    base = ref.focus_fwd(w, synth.bits16(c), "nvfp4", 16, 8, out="f32")
    c2 = c.clone()
    c2[3, 5] = 1.5  # sub-block 5 of row 3: elements 40..47
    pert = ref.focus_fwd(w, synth.bits16(c2), "nvfp4", 16, 8, out="f32")
    diff = base["w_hat"] != pert["w_hat"]
    assert diff[3, 40:48].any() and diff.sum() == diff[3, 40:48].sum()
    assert np.array_equal(base["scales"], pert["scales"])  # S_dq does not depend on c
    # a larger c shrinks u = W / (S_dq c), so code magnitudes can only fall
    mag = lambda o: ref.unpack_codes(o["codes"]) & 7
    big = ref.focus_fwd(w, synth.bits16(c * 1.25), "nvfp4", 16, 8, out="f32")
    assert np.all(mag(big) <= mag(base)) and np.any(mag(big) < mag(base))


@pytest.mark.parametrize("sub", [4, 8, 16])
def test_focus_bwd_closed_form_and_ste(ref, sub):
    d = synth.workload("c4_focus", rows=16, cols=256)
    w, g = synth.bits16(d["w"]), synth.bits16(d["g"])
    c = synth.focus_coeffs(16, 256, sub, seed=9)
    dc = ref.focus_bwd(w, g, synth.bits16(c), sub)
    W = f32_of_bf16(w).astype(np.float64).reshape(16, -1, sub)
    G = f32_of_bf16(g).astype(np.float64).reshape(16, -1, sub)
    C = c.float().numpy().astype(np.float64)
    want = -(G * W).sum(axis=2) / C ** 2
    scale = np.maximum(np.abs(want), np.abs(G * W).sum(axis=2) / C ** 2)
    assert np.all(np.abs(dc - want) <= 1e-5 * scale)
    # straight-through surrogate: W_hat ~ W / c, L = sum g * W_hat; central differences
    h = 1e-6
    L = lambda cc: (G * W / cc[..., None]).sum(axis=2)
    fd = (L(C + h) - L(C - h)) / (2 * h)
    assert np.allclose(dc, fd, rtol=1e-4, atol=1e-6 * np.abs(fd).max())


# ----------------------------------------- MXFP4 MSE-optimised E8M0 scale

def test_mxfp4_mse_grid_hand_examples(ref):
    # [5, -0.25, 0.75, 2.5]: SSE 1.375 at S = 1 (byte 127, the abs-max byte) and
    # again at S = 2 (5/2 -> 2 -> 4, -0.125 -> 0, 0.375 -> 0.5 -> 1, 1.25 -> 1 -> 2);
    # S = 4 gives 1.875, S = 1/2 saturates: the tie keeps the lower byte.
    y = [5.0, -0.25, 0.75, 2.5] + [0.0] * 28
    out = ref.quantize(bf16_bits([y]), "mxfp4", 32, "brute_force", 0, dq="f32")
    assert out["scales"].tolist() == [[127]]
    assert out["mse"][0, 0] == np.float32(1.375 / 32)
    # 7.90625 alone: the abs-max byte 127 (S = 1) saturates it to 6; S = 2, 4, 8
    # and 16 all give 8 (error 0.09375^2); the lowest of them, byte 128, wins.
    z = [7.90625] + [0.0] * 31
    am = ref.quantize(bf16_bits([z]), "mxfp4", 32, "absmax", 0)
    bf = ref.quantize(bf16_bits([z]), "mxfp4", 32, "brute_force", 0, dq="f32")
    assert am["scales"].tolist() == [[127]] and am["mse"][0, 0] == np.float32(1.90625 ** 2 / 32)
    assert bf["scales"].tolist() == [[128]]
    assert bf["dq"][0, 0] == 8.0
    assert bf["mse"][0, 0] == np.float32(0.09375 ** 2 / 32)


def test_mxfp4_mse_grid_never_worse_than_absmax(ref):
    x = synth.bits16(synth.laplace_outliers(64, 256, seed=9))
    for rot in (0, 32, 128):
        am = ref.quantize(x, "mxfp4", 32, "absmax", rot, want_mse=True)
        bf = ref.quantize(x, "mxfp4", 32, "brute_force", rot, want_mse=True)
        assert np.all(bf["mse"] <= am["mse"])
        moved = bf["scales"] != am["scales"]
        assert np.all((bf["mse"] < am["mse"]) | (bf["scales"] < am["scales"]) | ~moved)
        assert moved.any()


def _sse64(y, S):
    """Block SSE in float64 with the E2M1 grid (nearest, ties to the even
    mantissa, saturating); S is a power of two, so y / S is exact."""
    u = y / S
    a = np.abs(u)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    idx = np.argmin(np.abs(a[:, None] - grid[None, :]), axis=1)
    # exact ties between two grid points go to the even index (even mantissa)
    d = np.abs(a[:, None] - grid[None, :])
    for i in range(a.size):
        cand = np.nonzero(d[i] == d[i].min())[0]
        idx[i] = cand[0] if len(cand) == 1 else [c for c in cand if c % 2 == 0][0]
    v = np.where(a >= 6, 6.0, grid[idx]) * np.sign(u)
    return float(np.sum((y - v * S) ** 2))


def test_mxfp4_mse_grid_minimum_in_double(ref):
    rng = np.random.default_rng(21)
    x = bf16_bits(rng.laplace(0, 1, (16, 32)) * np.where(rng.random((16, 32)) < 0.05, 30, 1))
    out = ref.quantize(x, "mxfp4", 32, "brute_force", 0, want_mse=True)
    y = f32_of_bf16(x).astype(np.float64)
    for i in range(16):
        all64 = [_sse64(y[i], 2.0 ** (b - 127)) for b in range(255)]
        chosen = _sse64(y[i], 2.0 ** (int(out["scales"][i, 0]) - 127))
        assert chosen <= min(all64) * (1 + 1e-5) + 1e-30


def test_mxfp4_mse_grid_exact_blocks(ref):
    # blocks exactly on the E2M1 grid times 2^e: some scale gives SSE 0; the
    # chosen byte is the lowest such byte (found here by exact rational checks)
    from fractions import Fraction
    rng = np.random.default_rng(5)
    grid = [Fraction(v) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    rows = []
    for _ in range(24):
        e = int(rng.integers(-20, 20))
        v = rng.choice([0, 0.5, 1, 1.5, 2, 3, 4, 6], 32) * rng.choice([-1, 1], 32)
        rows.append(v * 2.0 ** e)
    x = bf16_bits(rows)
    out = ref.quantize(x, "mxfp4", 32, "brute_force", 0, want_mse=True)
    y = f32_of_bf16(x).astype(np.float64)
    for i in range(24):
        want = next(b for b in range(255)
                    if all(abs(Fraction(float(t)) / Fraction(2) ** (b - 127)) in grid for t in y[i]))
        assert out["scales"][i, 0] == want
        assert out["mse"][i, 0] == 0.0


# ------------------------------------------- dequantization back to the original domain

def _h(n):
    from scipy.linalg import hadamard
    return hadamard(n).astype(np.float64) / math.sqrt(n)


@pytest.mark.parametrize("rot", [16, 32, 64, 128])
def test_dequantize_unrotate_matches_float64_rotation(ref, rot):
    # MXFP4 codes with E8M0 scales 2^-3 .. 2^3: the dequantized values are short
    # dyadic numbers, so for rot 16 and 64 (k_n = 1/4, 1/8) the fp32 transform is
    # exact and must equal the float64 product with the normalised Sylvester matrix
    rng = np.random.default_rng(rot)
    rows, cols = 6, 256
    codes = rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
    scales = rng.integers(124, 131, (rows, cols // 32), dtype=np.uint8)
    plain = ref.dequantize(codes, scales, None, rows, cols, "mxfp4", 32)
    got = ref.dequantize_unrotate(codes, scales, None, rows, cols, "mxfp4", 32, rot)
    want = (plain.astype(np.float64).reshape(rows, cols // rot, rot) @ _h(rot).T).reshape(rows, cols)
    if rot in (16, 64):
        assert np.array_equal(got.astype(np.float64), want)
    else:
        assert np.max(np.abs(got - want)) <= 1e-6 * np.max(np.abs(want))


def test_dequantize_unrotate_rot0_is_dequantize(ref):
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 256, (4, 32), dtype=np.uint8)
    scales = rng.integers(0, 127, (4, 4), dtype=np.uint8)
    a = ref.dequantize(codes, scales, 0.5, 4, 64, "nvfp4", 16)
    b = ref.dequantize_unrotate(codes, scales, 0.5, 4, 64, "nvfp4", 16, 0)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("fmt,block,rot", [("mxfp4", 32, 32), ("mxfp4", 32, 128), ("nvfp4", 16, 16)])
def test_rotated_round_trip_error_equals_block_sse(ref, fmt, block, rot):
    # the rotation is orthonormal (up to the rounding of k_n): the squared error of
    # quantize -> dequantize -> undo the rotation equals the sum of the block SSEs
    # measured in the rotated domain
    x = synth.bits16(synth.laplace_outliers(32, 512, seed=4))
    q = ref.quantize(x, fmt, block, "absmax", rot, want_mse=True)
    back = ref.dequantize_unrotate(q["codes"], q["scales"], q["global_scale"] if fmt == "nvfp4" else None,
                                   32, 512, fmt, block, rot)
    err = np.sum((f32_of_bf16(x).astype(np.float64) - back.astype(np.float64)) ** 2)
    sse = np.sum(q["mse"].astype(np.float64) * block)
    assert abs(err - sse) <= 1e-4 * sse


# ----------------------------------------------------- FP4 x FP4 matrix product

@pytest.mark.parametrize("fmt,block", [("nvfp4", 16), ("mxfp4", 32)])
def test_fp4_gemm_equals_product_of_dequantized(ref, fmt, block):
    # the product of the two dequantized operands (numpy's float64 matmul of the
    # oracle's own dequantized values) times the two global scales
    rng = np.random.default_rng(7)
    M, N, K = 5, 7, 4 * block
    ac = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    bc = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    hi = 0x50 if fmt == "nvfp4" else 140
    lo = 0x20 if fmt == "nvfp4" else 110
    asc = rng.integers(lo, hi, (M, K // block), dtype=np.uint8)
    bsc = rng.integers(lo, hi, (N, K // block), dtype=np.uint8)
    sa, sb = (0.75, 1.5) if fmt == "nvfp4" else (None, None)
    d = ref.fp4_gemm(ac, asc, sa, bc, bsc, sb, fmt)
    da = ref.dequantize(ac, asc, 1.0, M, K, fmt, block).astype(np.float64)
    db = ref.dequantize(bc, bsc, 1.0, N, K, fmt, block).astype(np.float64)
    want = (da @ db.T) * ((sa * sb) if fmt == "nvfp4" else 1.0)
    assert np.array_equal(d, want.astype(np.float32))


def test_fp4_gemm_one_hot_rows(ref):
    # B rows that select one column of A: code 0x2 (value 1) at k = j, scale 1
    M, K = 4, 32
    rng = np.random.default_rng(3)
    ac = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    asc = np.full((M, K // 16), 0x38, np.uint8)  # E4M3 1.0
    cols = [0, 5, 17, 31]
    bc = np.zeros((len(cols), K // 2), np.uint8)
    for n, j in enumerate(cols):
        bc[n, j // 2] = 0x2 << (4 * (j % 2))
    bsc = np.full((len(cols), K // 16), 0x38, np.uint8)
    d = ref.fp4_gemm(ac, asc, 2.0, bc, bsc, 0.5, "nvfp4")
    a = ref.dequantize(ac, asc, 1.0, M, K, "nvfp4", 16)
    assert np.array_equal(d, a[:, cols])


# ------------------------------------------------- UE5M3 block scales (R17)

def ue5m3_table(ref):
    return np.array([ref.ue5m3_value(c) for c in range(0xFF)], np.float64)


@pytest.mark.parametrize("block", [4, 8, 16, 32])
@pytest.mark.parametrize("strategy", ["absmax", "prevent_zero", "four_over_six", "brute_force"])
def test_ue5m3_exact_round_trip(ref, block, strategy):
    # y = value(q) * ue5m3(c) with one element per block at +-6: every strategy
    # must return c and q exactly (no global scale: the code is set by the block)
    rng = np.random.default_rng(100 + block)
    rows, cols = 8, 64
    nb = cols // block
    c = rng.integers(1, 0xFF, size=(rows, nb))
    c[0, 0], c[0, -1] = 1, 0xFE          # smallest subnormal and largest code
    q = rng.integers(0, 16, size=(rows, cols))
    q.reshape(rows, nb, block)[:, :, 0] = rng.choice([7, 15], size=(rows, nb))
    y = E2M1[q] * np.repeat(ue5m3_table(ref)[c], block, axis=1)
    x = bf16_bits(y)
    assert np.array_equal(f32_of_bf16(x).astype(np.float64), y)
    out = ref.quantize(x, "ue5m3", block, strategy, 0, dq="f32")
    assert np.array_equal(out["scales"], c.astype(np.uint8))
    assert np.array_equal(ref.unpack_codes(out["codes"]), q.astype(np.uint8))
    assert np.array_equal(out["dq"].astype(np.float64), y)
    assert np.all(out["mse"] == 0)


@pytest.mark.parametrize("block", [4, 16])
def test_ue5m3_strategy_relations_and_scale_shift(ref, block):
    x = _with_tiny_rows(synth.workload("c3_strategy_sweep_t3", rows=32, cols=256)["x"])
    xb = synth.bits16(x)
    res = {s: ref.quantize(xb, "ue5m3", block, s, 0, dq="f32")
           for s in ("absmax", "prevent_zero", "four_over_six", "brute_force")}
    am, pz, fs, bf = (res[s] for s in ("absmax", "prevent_zero", "four_over_six", "brute_force"))
    assert np.all(pz["scales"] >= 1) and np.all(bf["scales"] >= 1)
    assert np.all(fs["mse"] <= am["mse"])
    assert np.all(bf["mse"] <= pz["mse"])
    pos = fs["scales"] >= 1
    assert np.all(bf["mse"][pos] <= fs["mse"][pos])
    for r in res.values():
        dq = ref.dequantize(r["codes"], r["scales"], None, *xb.shape, "ue5m3", block, "f32")
        assert np.array_equal(dq.view(np.uint32), r["dq"].view(np.uint32))
        m = ref.block_mse(xb, r["codes"], r["scales"], None, "ue5m3", block, 0)
        assert np.array_equal(m.view(np.uint32), r["mse"].view(np.uint32))
    # no global scale: scaling the tensor by 2^k moves every normal-range code
    # by 8k (one exponent step is 8 codes) and keeps the element codes
    big = am["scales"] >= 8 + 8 * 3
    x8 = bf16_bits(f32_of_bf16(xb).astype(np.float64) / 8.0)
    a8 = ref.quantize(x8, "ue5m3", block, "absmax", 0)
    assert np.array_equal(a8["scales"][big].astype(np.int64), am["scales"][big].astype(np.int64) - 24)
    cb = ref.unpack_codes(am["codes"]).reshape(32, -1, block)
    c8 = ref.unpack_codes(a8["codes"]).reshape(32, -1, block)
    assert np.array_equal(cb[big], c8[big])
