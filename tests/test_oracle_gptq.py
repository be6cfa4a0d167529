"""Pins of the oracle's GPTQ error feedback with static groups (MR-GPTQ).

Page: "Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization" (技術概要 §2.2: MR-GPTQ = GPTQ with the MSE-optimised grid,
static activation reordering and rotations). The error-feedback step is
GPTQ's (the error of each quantized column, divided by the diagonal of the
Cholesky factor U of the inverse Hessian, is spread over the later columns by
U's row). The pins: reduction to plain round-to-nearest when U has no
off-diagonal part, an exact dyadic case against an independent unblocked
float64 implementation, and the lower layer loss that error feedback buys.
"""
import numpy as np
import pytest

from microscaling_fp4_quantization_bf16_b200 import synth

E2M1_MAG = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def bf16_bits(a):
    return synth.bits16(synth.to_bf16(np.asarray(a, np.float64)))


def f32_of_bf16(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32)


def rne_e2m1_f64(u):
    """Nearest E2M1 value of u (float64), ties to the even magnitude index,
    saturating at 6; returns (codes, values). Written independently of the
    oracle's C rounding."""
    a = np.minimum(np.abs(u), 6.0)
    d = np.abs(a[..., None] - E2M1_MAG)
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    idx = np.where(cand, np.arange(8), 99)
    odd_tie = cand.sum(axis=-1) > 1
    m = np.where(odd_tie, np.where(cand & (np.arange(8) % 2 == 0), np.arange(8), 99).min(axis=-1),
                 idx.min(axis=-1))
    sign = np.signbit(u)
    return (m | (sign.astype(np.int64) << 3)), np.where(sign, -E2M1_MAG[m], E2M1_MAG[m])


def gptq_f64_unblocked(w, S, U, perm):
    """Plain GPTQ in float64, one column at a time, every later column updated
    at once: w[:, k] -= e_j U[j, k] for all k > j. S: per-element scale in the
    original column order. Returns 4-bit codes [rows, K] (original order)."""
    W = w[:, perm].astype(np.float64).copy()
    Sp = S[:, perm]
    rows, K = W.shape
    codes = np.zeros((rows, K), np.int64)
    for j in range(K):
        s = Sp[:, j]
        safe = np.where(s == 0, 1.0, s)
        q, v = rne_e2m1_f64(W[:, j] / safe)
        q = np.where(s == 0, 0, q)
        deq = np.where(s == 0, 0.0, v * s)
        e = (W[:, j] - deq) / U[j, j]
        W[:, j + 1:] -= e[:, None] * U[j, j + 1:][None, :]
        codes[:, perm[j]] = q
    return codes


def per_element_scales(ref, scales, fmt, block, sg=None):
    if fmt == "mxfp4":
        vals = np.array([ref.e8m0_value(int(b)) for b in range(256)])
    elif fmt == "ue5m3":
        vals = np.array([ref.ue5m3_value(int(b)) for b in range(256)])
    else:
        vals = np.array([ref.e4m3_value(int(b)) for b in range(256)]) * float(sg)
    return np.repeat(vals[scales], block, axis=1)


# -------------------------------------------------------------- reductions

@pytest.mark.parametrize("fmt,block,strat", [("nvfp4", 16, "absmax"), ("mxfp4", 32, "brute_force"),
                                             ("ue5m3", 8, "four_over_six")])
def test_no_feedback_is_round_to_nearest(ref, fmt, block, strat):
    # U with no off-diagonal part spreads no error: GPTQ with static groups is
    # then the quantizer's own round-to-nearest with the same scales, in any
    # processing order
    x = synth.workload("c3_strategy_sweep_t3", rows=12, cols=256)["x"]
    xb = synth.bits16(x)
    q = ref.quantize(xb, fmt, block, strat, 0)
    rng = np.random.default_rng(1)
    for U in (np.eye(256, dtype=np.float32), np.diag(rng.uniform(0.5, 2, 256)).astype(np.float32)):
        for perm in (None, rng.permutation(256).astype(np.int32)):
            codes = ref.gptq(xb, q["scales"], q["global_scale"], U, perm, fmt, block)
            assert np.array_equal(codes, q["codes"])


# ------------------------------------------------ exact dyadic vs float64

def test_dyadic_case_equals_unblocked_float64(ref):
    # Dyadic weights, MXFP4 scales of 1 and a unit-diagonal U whose sparse
    # off-diagonal entries are +-1/8 or +-1/4: every value stays a short dyadic
    # fraction, so fp32 and float64 compute the same numbers, and the blocked
    # fp32 oracle must equal plain unblocked GPTQ exactly -- every code,
    # including the ties on E2M1 midpoints.
    rng = np.random.default_rng(7)
    rows, K = 6, 256
    w = rng.integers(-40, 41, size=(rows, K)) / 16.0
    U = np.eye(K)
    mask = rng.random((K, K)) < 0.02
    U[np.triu(mask, 1)] = rng.choice([-0.25, -0.125, 0.125, 0.25], size=int(np.triu(mask, 1).sum()))
    perm = rng.permutation(K)
    scales = np.full((rows, K // 32), 127, np.uint8)           # E8M0 2^0
    got = ref.unpack_codes(ref.gptq(bf16_bits(w), scales, None, U.astype(np.float32),
                                    perm.astype(np.int32), "mxfp4", 32))
    want = gptq_f64_unblocked(w, np.ones((rows, K)), U, perm)
    assert np.array_equal(got.astype(np.int64), want)
    # the feedback changed codes (the case does exercise it)
    rtn = ref.unpack_codes(ref.quantize(bf16_bits(w), "mxfp4", 32, "absmax", 0)["codes"])
    assert not np.array_equal(got, rtn)


# -------------------------------------------------------- what GPTQ buys

@pytest.mark.parametrize("fmt,block,strat", [("nvfp4", 16, "absmax"), ("mxfp4", 32, "brute_force")])
def test_error_feedback_lowers_layer_loss(ref, fmt, block, strat):
    # on a layer with correlated input channels, GPTQ's codes give a lower
    # layer-output error tr(E H E^T) than round-to-nearest with the same
    # static scales, and the codes differ from the float64 unblocked
    # algorithm only at rare near-ties (the loss agrees to 1%)
    d = synth.gptq_problem(16, 256, 2048, seed=3)
    wb = synth.bits16(d["w"])
    q = ref.quantize(wb, fmt, block, strat, 0)
    sg = q["global_scale"] if fmt == "nvfp4" else None
    codes = ref.gptq(wb, q["scales"], sg, d["u"], d["perm"], fmt, block)
    S = per_element_scales(ref, q["scales"], fmt, block, sg)
    w = f32_of_bf16(wb).astype(np.float64)
    val = lambda c: np.where(ref.unpack_codes(c) >= 8, -1, 1) * E2M1_MAG[ref.unpack_codes(c) & 7] * S
    loss = lambda c: float(np.einsum("ij,jk,ik->", val(c) - w, d["h"], val(c) - w))
    l_gptq, l_rtn = loss(codes), loss(q["codes"])
    assert l_gptq < 0.8 * l_rtn, (l_gptq, l_rtn)
    c64 = gptq_f64_unblocked(w, S, d["u"].astype(np.float64), d["perm"])
    diff = np.mean(ref.unpack_codes(codes).astype(np.int64) != c64)
    v64 = np.where(c64 >= 8, -1, 1) * E2M1_MAG[c64 & 7] * S
    l64 = float(np.einsum("ij,jk,ik->", v64 - w, d["h"], v64 - w))
    assert diff < 0.02 and abs(l_gptq - l64) <= 0.01 * l64, (diff, l_gptq, l64)


def test_rejects_bad_arguments(ref):
    wb = bf16_bits(np.zeros((2, 256)))
    sc = np.zeros((2, 16), np.uint8)
    U = np.eye(256, dtype=np.float32)
    with pytest.raises(ValueError):
        ref.gptq(wb, sc, 1.0, U, np.zeros(256, np.int32), "nvfp4", 16)   # not a permutation
    with pytest.raises(ValueError):
        ref.gptq(bf16_bits(np.zeros((2, 192))), np.zeros((2, 12), np.uint8), 1.0,
                 np.eye(192, dtype=np.float32), None, "nvfp4", 16)        # K % 128


# ------------------------------------------- rotation in front (MR-GPTQ)

def hadamard_rows(w, n):
    """w times the block-diagonal normalised Sylvester Hadamard of width n, in
    float64 (scipy's matrix, rows taken chunk by chunk)."""
    import scipy.linalg
    rows, K = w.shape
    return (w.reshape(rows, K // n, n) @ scipy.linalg.hadamard(n)).reshape(rows, K) / np.sqrt(n)


@pytest.mark.parametrize("fmt,block,strat,rot", [("nvfp4", 16, "absmax", 16), ("mxfp4", 32, "absmax", 128),
                                                 ("ue5m3", 8, "four_over_six", 32)])
def test_rotated_no_feedback_is_rotated_round_to_nearest(ref, fmt, block, strat, rot):
    # with U diagonal, GPTQ behind the rotation is the quantizer's own
    # round-to-nearest of the rotated rows with the same scales: the rotation
    # is the quantizer's (same chunks, stages and factor), in any order
    x = synth.workload("c5_activation_channels", rows=12, cols=256)["x"]
    xb = synth.bits16(x)
    q = ref.quantize(xb, fmt, block, strat, rot)
    rng = np.random.default_rng(2)
    U = np.diag(rng.uniform(0.5, 2, 256)).astype(np.float32)
    for perm in (None, rng.permutation(256).astype(np.int32)):
        codes = ref.gptq(xb, q["scales"], q["global_scale"], U, perm, fmt, block, rot=rot)
        assert np.array_equal(codes, q["codes"])
    # and the rotation does change the codes (the case exercises it)
    assert not np.array_equal(ref.gptq(xb, q["scales"], q["global_scale"], U, None, fmt, block),
                              q["codes"])


def test_rotated_dyadic_case_equals_unblocked_float64(ref):
    # Dyadic weights rotated by the 16-wide Hadamard (factor 1/4: exact): the
    # rotated values are short dyadic fractions in fp32 and float64 alike, so
    # the oracle (rotation, then blocked fp32 GPTQ) must equal float64 GPTQ run
    # on scipy's rotation of the same rows, code for code.
    rng = np.random.default_rng(8)
    rows, K = 5, 256
    w = rng.integers(-24, 25, size=(rows, K)) / 16.0
    U = np.eye(K)
    mask = np.triu(rng.random((K, K)) < 0.02, 1)
    U[mask] = rng.choice([-0.25, -0.125, 0.125, 0.25], size=int(mask.sum()))
    perm = rng.permutation(K)
    scales = np.full((rows, K // 32), 127, np.uint8)           # E8M0 2^0
    got = ref.unpack_codes(ref.gptq(bf16_bits(w), scales, None, U.astype(np.float32),
                                    perm.astype(np.int32), "mxfp4", 32, rot=16))
    want = gptq_f64_unblocked(hadamard_rows(w, 16), np.ones((rows, K)), U, perm)
    assert np.array_equal(got.astype(np.int64), want)


@pytest.mark.parametrize("rot", [16, 128])
def test_rotated_error_feedback_and_loss_identity(ref, rot):
    # Behind the rotation, GPTQ's codes lower the layer loss below the rotated
    # round-to-nearest's, measured in the rotated basis with R H R; taken back
    # to the original basis (Ŵ R, R R = I) the same loss is measured with H:
    # the two must agree (float64), which pins the basis in which the scales,
    # U and the codes live.
    d = synth.gptq_problem(16, 256, 2048, seed=4, rot=rot)
    wb = synth.bits16(d["w"])
    q = ref.quantize(wb, "nvfp4", 16, "absmax", rot)
    sg = q["global_scale"]
    codes = ref.gptq(wb, q["scales"], sg, d["u"], d["perm"], "nvfp4", 16, rot=rot)
    S = per_element_scales(ref, q["scales"], "nvfp4", 16, sg)
    w = f32_of_bf16(wb).astype(np.float64)
    wr = hadamard_rows(w, rot)                                   # the rotated weights
    val = lambda c: np.where(ref.unpack_codes(c) >= 8, -1, 1) * E2M1_MAG[ref.unpack_codes(c) & 7] * S
    loss_rot = lambda c: float(np.einsum("ij,jk,ik->", val(c) - wr, d["h"], val(c) - wr))
    l_gptq, l_rtn = loss_rot(codes), loss_rot(q["codes"])
    assert l_gptq < 0.8 * l_rtn, (l_gptq, l_rtn)
    back = hadamard_rows(val(codes), rot)                        # Ŵ R: the original basis
    l_orig = float(np.einsum("ij,jk,ik->", back - w, d["h_orig"], back - w))
    assert abs(l_orig - l_gptq) <= 1e-6 * l_gptq, (l_orig, l_gptq)
