"""Pins of the oracle's FOCUS calibration step: the fp16 rounding of the master
coefficients, the straight-through coefficient gradient inside the step, and
the SGD / Adam updates.

Pages: "FOCUS: FP4 Optimization via Coupled-Relaxation and Dual-Granularity
Scaling" (Metodologia §1: scales learned by gradient descent through the
straight-through estimator; §2: c is an FP16 learnable parameter initialised
to 1; §3: sub-block coefficients c_k with S_dq shared by the block). Adam is
Kingma & Ba's published algorithm; the pins below use properties of it that
hold in exact arithmetic, not a second copy of its formulas.
"""
from fractions import Fraction

import numpy as np
import pytest

from microscaling_fp4_quantization_bf16_b200 import synth

from focus_layer import layer_loss_and_grad, layer_problem


def bf16_bits(a):
    return synth.bits16(synth.to_bf16(np.asarray(a, np.float64)))


def f32_of_bf16(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------- fp32 -> fp16 rounding

def test_float_to_fp16_against_numpy(ref):
    # numpy's float32 -> float16 cast is IEEE round-to-nearest-even.
    halves = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    rng = np.random.default_rng(11)
    mids = ((halves[:-1].astype(np.float64) + halves[1:]) / 2).astype(np.float32)
    rand = rng.integers(0x33000000, 0x47900000, 20000, dtype=np.uint32).view(np.float32)
    extra = np.array([65504.0, 65519.99, 65520.0, 7e4, 1e-9, 2.0 ** -25, 2.0 ** -24 * 1.5],
                     np.float32)
    vals = np.concatenate([halves[::7], mids[::5], rand, extra])
    vals = np.concatenate([vals, -vals])
    got = np.array([ref.float_to_fp16(v) for v in vals], np.uint16)
    want = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_float_to_fp16_ties_to_even(ref):
    # 1 + 2^-11 is halfway between 1 and 1 + 2^-10: the even pattern (1.0) wins;
    # 1 + 3 * 2^-11 is halfway between 1 + 2^-10 (odd) and 1 + 2^-9 (even).
    assert ref.float_to_fp16(1 + 2.0 ** -11) == 0x3C00
    assert ref.float_to_fp16(1 + 3 * 2.0 ** -11) == 0x3C02
    assert ref.float_to_fp16(65520.0) == 0x7C00      # half-way to 2^16 overflows
    assert ref.float_to_fp16(-0.0) == 0x8000


# ------------------------------------------------------------------ SGD, exact

def test_sgd_update_exact_dyadic(ref):
    # dyadic values: every product and sum is exact, so the update must equal the
    # rational c - lr * (-(sum g w) / c^2) exactly, sub-block by sub-block.
    rng = np.random.default_rng(3)
    rows, cols, sub = 3, 32, 8
    w = rng.integers(-8, 9, (rows, cols)) / 8.0
    g = rng.integers(-8, 9, (rows, cols)) / 4.0
    c = np.full((rows, cols // sub), 2.0, np.float32)
    c[1, 2] = 0.5
    lr = 2.0 ** -6
    out = ref.focus_update(bf16_bits(w), bf16_bits(g), c, sub=sub, opt="sgd", lr=lr)
    for i in range(rows):
        for k in range(cols // sub):
            acc = sum(Fraction(g[i, k * sub + j]) * Fraction(w[i, k * sub + j])
                      for j in range(sub))
            ck = Fraction(float(c[i, k]))
            dc = -acc / (ck * ck)
            assert Fraction(float(out["c"][i, k])) == ck - Fraction(lr) * dc
    assert np.array_equal(out["c_half"], out["c"].astype(np.float16).view(np.uint16))


def test_update_uses_fp16_coefficient(ref):
    # the gradient is taken at fp16(c): a master value between two halves must
    # give the same dc as the half it rounds to (SGD step = -lr dc, c differs).
    w = bf16_bits(np.full((1, 8), 0.5))
    g = bf16_bits(np.full((1, 8), 1.0))
    c_a = np.array([[1.0]], np.float32)
    c_b = np.array([[1.0 + 2.0 ** -13]], np.float32)   # rounds to 1.0 in fp16
    lr = 2.0 ** -4
    a = ref.focus_update(w, g, c_a, sub=8, opt="sgd", lr=lr)
    b = ref.focus_update(w, g, c_b, sub=8, opt="sgd", lr=lr)
    # dc = -(8 * 0.5) / 1 = -4 -> c + 0.25
    assert a["c"][0, 0] == np.float32(1.25)
    assert b["c"][0, 0] == np.float32(1.0 + 2.0 ** -13 + 0.25)


# ---------------------------------------------------------- Adam, by properties

def _case(seed, rows=4, cols=64):
    rng = np.random.default_rng(seed)
    w = bf16_bits(rng.normal(0, 0.02, (rows, cols)))
    g = bf16_bits(rng.normal(0, 1.0, (rows, cols)))
    return w, g


def test_adam_first_step_is_sign_step(ref):
    # with m = v = 0 the first Adam step is lr * dc / (|dc| + eps): a step of
    # size lr against the sign of the gradient.
    w, g = _case(5)
    c = np.ones((4, 8), np.float32)
    lr = 1e-3
    dc = ref.focus_bwd(w, g, np.full((4, 8), 0x3C00, np.uint16), sub=8)
    out = ref.focus_update(w, g, c, sub=8, opt="adam", lr=lr, t=1)
    want = 1.0 - lr * np.sign(dc.astype(np.float64)) * np.abs(dc) / (np.abs(dc) + 1e-8)
    assert np.allclose(out["c"], want, rtol=0, atol=2e-7)
    assert np.array_equal(out["m"], np.float32(np.float32(1) - np.float32(0.9)) * dc)


def test_adam_constant_gradient_moves_t_lr(ref):
    # a constant gradient makes the bias-corrected moments equal dc and dc^2 at
    # every t, so T steps move c by T * lr against the gradient's sign; lr is
    # small enough that fp16(c) (and so dc) never changes.
    w, g = _case(6)
    c = np.ones((4, 8), np.float32)
    m = v = None
    lr, steps = 1e-5, 6
    dc = ref.focus_bwd(w, g, np.full((4, 8), 0x3C00, np.uint16), sub=8)
    for t in range(1, steps + 1):
        out = ref.focus_update(w, g, c, m, v, sub=8, opt="adam", lr=lr, t=t)
        c, m, v = out["c"], out["m"], out["v"]
        assert np.all(out["c_half"] == 0x3C00)
    moved = c.astype(np.float64) - 1.0
    assert np.allclose(moved, -steps * lr * np.sign(dc), rtol=2e-3, atol=0)


def test_adam_gradient_scale_invariance_exact(ref):
    # with eps = 0, scaling the gradient by 4 (exact in bf16) scales m by 4 and
    # v by 16 exactly and leaves the update bit-identical.
    w, g = _case(7)
    g4 = bf16_bits(f32_of_bf16(g).astype(np.float64) * 4)
    c = np.ones((4, 8), np.float32)
    s1 = ref.focus_update(w, g, c, sub=8, opt="adam", lr=1e-3, eps=0.0, t=1)
    s4 = ref.focus_update(w, g4, c, sub=8, opt="adam", lr=1e-3, eps=0.0, t=1)
    for t in (2, 3):
        s1 = ref.focus_update(w, g, s1["c"], s1["m"], s1["v"], sub=8, opt="adam", lr=1e-3,
                              eps=0.0, t=t)
        s4 = ref.focus_update(w, g4, s4["c"], s4["m"], s4["v"], sub=8, opt="adam", lr=1e-3,
                              eps=0.0, t=t)
    assert np.array_equal(s1["c"].view(np.uint32), s4["c"].view(np.uint32))
    assert np.array_equal(s4["m"], s1["m"] * 4)
    assert np.array_equal(s4["v"], s1["v"] * 16)


def test_adam_zero_gradient_keeps_c(ref):
    w = bf16_bits(np.zeros((2, 16)))
    g = bf16_bits(np.ones((2, 16)))
    c = np.full((2, 2), 1.5, np.float32)
    out = ref.focus_update(w, g, c, sub=8, opt="adam", lr=1e-2, t=1)
    assert np.array_equal(out["c"], c) and not np.any(out["m"]) and not np.any(out["v"])


def test_update_rejects_bad_arguments(ref):
    w, g = _case(8)
    with pytest.raises(ValueError):
        ref.focus_update(w, g, np.ones((4, 8), np.float32), sub=8, opt="adam", t=0)
    with pytest.raises(ValueError):
        ref.focus_update(w, g, np.ones((4, 21), np.float32), sub=3, opt="sgd")


# ------------------------------------------------------------- the fused step

def test_step_gradient_closed_form(ref):
    # Adam with beta1 = 0 stores m = dc exactly; compare dc with the closed form
    # -sum 2 (W_hat - W) W / c^2 recomputed in double from the FOCUS forward
    # (fp32 W_hat), within the fp32 rounding of the products and the tree.
    for fmt, block in (("nvfp4", 16), ("mxfp4", 32), ("nvfp4", 8)):
        w = synth.gaussian(6, 64, seed=21, std=0.02)
        wb = synth.bits16(w)
        rng = np.random.default_rng(4)
        c = rng.uniform(0.85, 1.15, (6, 8)).astype(np.float32)
        ch = c.astype(np.float16).view(np.uint16)
        fwd = ref.focus_fwd(wb, ch, fmt, block, 8, out="f32", want_codes=False)
        out = ref.focus_step(wb, c, fmt=fmt, block=block, sub=8, opt="adam", beta1=0.0,
                             beta2=0.0, lr=1e-3, t=1)
        assert out["global_scale"] == fwd["global_scale"]
        wf = f32_of_bf16(wb).astype(np.float64).reshape(6, 8, 8)
        wh = fwd["w_hat"].astype(np.float64).reshape(6, 8, 8)
        ck = ch.view(np.float16).astype(np.float64)
        dc = -(2 * (wh - wf) * wf).sum(-1) / ck ** 2
        bound = 8 * 2.0 ** -23 * (2 * np.abs(wh - wf) * np.abs(wf)).sum(-1) / ck ** 2
        assert np.all(np.abs(out["m"] - dc) <= bound + 1e-30)
        sse = ((wh - wf) ** 2).sum(-1)
        assert np.allclose(out["sse"], sse, rtol=1e-6, atol=0)


def test_step_direction_follows_rounding(ref):
    # MXFP4, block max 6 -> S_dq = 1. Elements 0.7 round down to 0.5 (toward
    # zero): the STE step lowers c so that W / (S_dq c) grows. Elements 0.8 round
    # up to 1.0: the step raises c.
    for val, sign in ((0.7, -1), (0.8, +1)):
        row = [6.0] + [val] * 31
        out = ref.focus_step(bf16_bits([row]), np.ones((1, 4), np.float32), fmt="mxfp4",
                             block=32, sub=8, opt="sgd", lr=2.0 ** -8)
        assert np.all(np.sign(out["c"].astype(np.float64) - 1.0) == sign)


def test_step_unit_coefficients_are_optimal(ref):
    # At c == 1 every element is rounded to its nearest point of the S_dq grid,
    # so no coefficient can lower the sub-block's reconstruction error.
    w = synth.student_t(8, 128, seed=9)
    wb = synth.bits16(w)
    base = ref.focus_step(wb, np.ones((8, 16), np.float32), fmt="nvfp4", block=16, sub=8,
                          opt="sgd", lr=0.0)["sse"]
    rng = np.random.default_rng(10)
    for _ in range(8):
        c = rng.uniform(0.7, 1.3, (8, 16)).astype(np.float32)
        sse = ref.focus_step(wb, c, fmt="nvfp4", block=16, sub=8, opt="sgd", lr=0.0)["sse"]
        assert np.all(sse.astype(np.float64) >= base * (1 - 1e-6))


def test_step_sgd_zero_lr_keeps_state(ref):
    w = synth.gaussian(2, 32, seed=1, std=0.02)
    c = np.full((2, 4), 1.0625, np.float32)
    out = ref.focus_step(synth.bits16(w), c, fmt="nvfp4", block=16, sub=8, opt="sgd", lr=0.0)
    assert np.array_equal(out["c"], c) and out["m"] is None


# ------------------------------------------- the loop on a layer-output loss

def test_adam_calibration_lowers_layer_loss(ref):
    # Unlike the weight-reconstruction loss, a layer-output loss couples the
    # elements of a row through H, and the straight-through Adam steps on c
    # lower it (the pages' claim for CRS + DGS, here on a synthetic layer).
    wb, h = layer_problem(128, 256, 1024, seed=0)
    c = np.ones((128, 32), np.float32)
    m = v = None
    first = None
    for t in range(1, 61):
        loss, g = layer_loss_and_grad(ref, wb, c, h)
        first = loss if first is None else first
        out = ref.focus_update(wb, g, c, m, v, sub=8, opt="adam", lr=2e-4, t=t)
        c, m, v = out["c"], out["m"], out["v"]
    last, _ = layer_loss_and_grad(ref, wb, c, h)
    assert last < 0.95 * first, (first, last)


# -------------------------------------------------------- the pages' facts

def test_calibration_state_follows_the_page():
    # the Python calibration state starts from the page's c = 1 in fp16, with
    # one coefficient per sub-block of the page's example size
    import os
    import torch
    import microscaling_fp4_quantization_bf16_b200 as fp4q
    kv = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "focus_facts.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                k, v = line.split()
                kv[k] = float(v)
    sub = int(kv["focus_sub_block_example"])
    st = fp4q.focus_state(4, 2 * int(kv["nvfp4_block"]), sub, "adam")   # CPU tensors
    assert st.c_half.dtype == torch.float16 and st.c_half.element_size() * 8 == kv["focus_coefficient_bits"]
    assert torch.all(st.c == kv["focus_coefficient_init"]) and torch.all(st.c_half == 1.0)
    assert st.c.shape == (4, 2 * int(kv["nvfp4_block"]) // sub)
    assert torch.all(st.m == 0) and torch.all(st.v == 0) and st.t == 0
    assert int(kv["mxfp4_block"]) % sub == 0 and int(kv["nvfp4_block"]) % sub == 0
