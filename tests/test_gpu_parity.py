"""CUDA path vs the oracle, element by element, through the C ABI.

Bar: codes, scale bytes, the global scale and dequantized values bit-exact
(fp32 and bf16, -0 included); per-block MSE within 1e-6 relative (the design
gives bit-exact, which is also reported); FOCUS gradients within 1e-5
relative. Small shapes span several segments and a ragged tail; full-size
workloads are compared on every element where the oracle is fast enough, and
on sampled rows (with the oracle's own full-tensor abs-max) where it is not.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from microscaling_fp4_quantization_bf16_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 256
POISON = 0xA5


# ----------------------------------------------------------------- helpers

def u16(t):
    return synth.bits16(t)


def bits_of(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def assert_exact(got, want, what):
    g, w = bits_of(got).reshape(-1), bits_of(want).reshape(-1)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    bad = np.nonzero(g != w)[0]
    assert bad.size == 0, (f"{what}: {bad.size}/{g.size} differ; first idx {bad[:4]} "
                           f"gpu {g[bad[:4]]} oracle {w[bad[:4]]}")


def assert_mse(got, want, what):
    """Within 1e-6 relative (equal values, infinities included, count as 0),
    then also bit-exact, which the pinned operation order gives."""
    got = np.asarray(got, np.float32)
    want = np.asarray(want, np.float32)
    g64, w64 = got.astype(np.float64), want.astype(np.float64)
    same = (got.view(np.uint32) == want.view(np.uint32))
    with np.errstate(invalid="ignore"):
        rel = np.where(same, 0.0, np.abs(g64 - w64) / np.maximum(np.abs(w64), 1e-38))
    assert float(rel.max(initial=0.0)) <= 1e-6, f"{what}: max rel err {rel.max()}"
    assert_exact(got, want, what + " (bit-exact)")


def guarded(shape, dtype):
    """A CUDA tensor followed by GUARD poisoned bytes; returns (view, backing)."""
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    back = torch.full((n + GUARD,), POISON, dtype=torch.uint8, device="cuda")
    return back[:n].view(dtype).view(shape), back


def guard_ok(back, n_bytes):
    tail = back[n_bytes:].cpu().numpy()
    return bool(np.all(tail == POISON))


def gpu_quantize(gpu, x, fmt, block, strat, rot, gamax=None, mse=True, dq=None):
    rows, cols = x.shape
    nv = fmt == "nvfp4"
    codes, cb = guarded((rows, cols // 2), torch.uint8)
    scales, sb = guarded((rows, cols // block), torch.uint8)
    m, mb = guarded((rows, cols // block), torch.float32) if mse else (None, None)
    d, db = guarded((rows, cols), dq) if dq is not None else (None, None)
    gs = torch.full((1,), -7.0, device="cuda") if nv else None
    out = gpu.Quantized(codes, scales, gs, m, d)
    ga = None if gamax is None else torch.tensor([gamax], dtype=torch.float32, device="cuda")
    gpu.quantize(x.cuda(), fmt, block, strat, rot, global_amax=ga, out=out)
    torch.cuda.synchronize()
    for t, b in ((codes, cb), (scales, sb), (m, mb), (d, db)):
        if t is not None:
            assert guard_ok(b, t.numel() * t.element_size()), "write past the end of an output"
    res = {"codes": codes.cpu().numpy(), "scales": scales.cpu().numpy(),
           "gs": None if gs is None else gs.cpu().numpy()[0],
           "mse": None if m is None else m.cpu().numpy(), "dq": None}
    if d is not None:
        res["dq"] = d.cpu().numpy() if dq == torch.float32 else u16(d)
    return res


def oracle_quantize(x, fmt, block, strat, rot, gamax=None, mse=True, dq=None):
    dqk = None if dq is None else ("f32" if dq == torch.float32 else "bf16")
    return oracle.quantize(u16(x), fmt, block, strat, rot, global_amax=gamax, want_mse=mse, dq=dqk)


def compare_quant(g, o, fmt, what):
    assert_exact(g["codes"], o["codes"], what + " codes")
    assert_exact(g["scales"], o["scales"], what + " scales")
    if fmt == "nvfp4":
        assert_exact(np.float32(g["gs"]), np.float32(o["global_scale"]), what + " global scale")
    if g["mse"] is not None:
        assert_mse(g["mse"], o["mse"], what + " mse")
    if g["dq"] is not None:
        assert_exact(g["dq"], o["dq"], what + " dq")


def mixed(rows, cols, seed):
    """Heavy-tailed data with underflowing rows, outliers, zeros and -0."""
    rng = np.random.default_rng(seed)
    a = rng.standard_t(3, size=(rows, cols)) * 0.02
    a[::3] *= 1e-6
    flat = a.reshape(-1)
    k = max(1, flat.size // 97)
    flat[rng.choice(flat.size, k, replace=False)] *= 50
    flat[rng.choice(flat.size, k, replace=False)] = 0.0
    flat[rng.choice(flat.size, k, replace=False)] = -0.0
    return synth.to_bf16(a)


# ------------------------------------------------------- all combinations

COMBOS = [(f, b, s, r) for f in ("nvfp4", "ue5m3") for b in (4, 8, 16, 32)
          for s in ("absmax", "prevent_zero", "four_over_six", "brute_force")
          for r in (0, 16, 32, 64, 128)] + [("mxfp4", 32, s, r) for s in ("absmax", "brute_force")
                                            for r in (0, 16, 32, 64, 128)]


def shapes_for(block, rot):
    unit = max(block, rot, 1)
    shapes = [(1, max(unit, 32)), (3, 2 * max(unit, 32)), (17, 4 * max(unit, 32) + (0 if rot else unit))]
    if rot <= 16:  # a flattened length that is not a multiple of 32: ragged last segment
        shapes.append((5, 3 * unit if unit >= 8 else 12))
    return shapes


@pytest.mark.parametrize("loads", ["direct", "tma"])
@pytest.mark.parametrize("fmt,block,strat,rot", COMBOS)
def test_quantize_small_shapes(gpu, monkeypatch, loads, fmt, block, strat, rot):
    """Every combination through the direct-load kernel (FP4Q_TMA=0) and
    (FP4Q_TMA=1, flattened length a multiple of 64) the TMA-fed kernel."""
    monkeypatch.setenv("FP4Q_TMA", "1" if loads == "tma" else "0")
    for k, (rows, cols) in enumerate(shapes_for(block, rot)):
        x = mixed(rows, cols, seed=1000 * block + rot + k)
        dq = (None, torch.float32, torch.bfloat16)[k % 3]
        g = gpu_quantize(gpu, x, fmt, block, strat, rot, dq=dq)
        o = oracle_quantize(x, fmt, block, strat, rot, dq=dq)
        compare_quant(g, o, fmt, f"{fmt} B{block} {strat} H{rot} {rows}x{cols}")
        if fmt == "nvfp4":  # single-pass form with a caller-supplied abs-max
            ga = float(oracle.global_amax(u16(x), rot))
            g1 = gpu_quantize(gpu, x, fmt, block, strat, rot, gamax=ga, mse=False)
            compare_quant(g1, oracle_quantize(x, fmt, block, strat, rot, gamax=ga, mse=False), fmt,
                          "supplied amax")


# ------------------------------------------------------- full-size workloads

def sample_rows(rows, k=24, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, rows - 1], rng.choice(rows, k, replace=False)]))


def test_c1_full_round_trip(gpu):
    x = synth.workload("c1_nvfp4_roundtrip")["x"]
    g = gpu_quantize(gpu, x, "nvfp4", 16, "absmax", 0, dq=torch.float32)
    o = oracle_quantize(x, "nvfp4", 16, "absmax", 0, dq=torch.float32)
    compare_quant(g, o, "nvfp4", "C1")


@pytest.mark.parametrize("rot", [0, 32])
def test_c2_full_mxfp4(gpu, rot):
    x = synth.workload("c2_mxfp4_laplace_outliers")["x"]
    g = gpu_quantize(gpu, x, "mxfp4", 32, "absmax", rot, mse=False)
    o = oracle_quantize(x, "mxfp4", 32, "absmax", rot, mse=False)
    compare_quant(g, o, "mxfp4", f"C2 H{rot}")


@pytest.mark.parametrize("block", [4, 8, 16, 32])
def test_c3_full_strategy_sweep_sampled(gpu, block):
    x = synth.workload("c3_strategy_sweep_t3")["x"]
    ga = float(oracle.global_amax(u16(x), 0))
    rows = sample_rows(x.shape[0], k=12, seed=block)
    xs = x[rows]
    for strat in ("absmax", "prevent_zero", "four_over_six", "brute_force"):
        g = gpu_quantize(gpu, x, "nvfp4", block, strat, 0)
        o = oracle_quantize(xs, "nvfp4", block, strat, 0, gamax=ga)
        assert_exact(np.float32(g["gs"]), np.float32(o["global_scale"]), "C3 global scale")
        g = {"codes": g["codes"][rows], "scales": g["scales"][rows], "gs": g["gs"],
             "mse": g["mse"][rows], "dq": None}
        compare_quant(g, o, "nvfp4", f"C3 B{block} {strat}")


@pytest.mark.parametrize("block", [4, 16])
def test_c3_full_ue5m3_sampled(gpu, block):
    # UE5M3 scales have no global scale: every row is independent
    x = synth.workload("c3_strategy_sweep_t3")["x"]
    rows = sample_rows(x.shape[0], k=12, seed=100 + block)
    xs = x[rows]
    for strat in ("absmax", "prevent_zero", "four_over_six", "brute_force"):
        g = gpu_quantize(gpu, x, "ue5m3", block, strat, 0)
        o = oracle_quantize(xs, "ue5m3", block, strat, 0)
        g = {"codes": g["codes"][rows], "scales": g["scales"][rows], "gs": None,
             "mse": g["mse"][rows], "dq": None}
        compare_quant(g, o, "ue5m3", f"C3 UE5M3 B{block} {strat}")


@pytest.mark.parametrize("fmt,block", [("nvfp4", 16), ("mxfp4", 32)])
def test_c4_full_focus(gpu, fmt, block):
    d = synth.workload("c4_focus")
    w, c, gr = d["w"], d["c"], d["g"]
    out = gpu.focus_fwd(w.cuda(), c.cuda(), fmt, block, 8, out_dtype=torch.bfloat16, want_codes=True)
    dc = gpu.focus_bwd(w.cuda(), gr.cuda(), c.cuda(), 8)
    torch.cuda.synchronize()
    o = oracle.focus_fwd(u16(w), u16(c), fmt, block, 8, out="bf16")
    assert_exact(u16(out.w_hat), o["w_hat"], "C4 w_hat")
    assert_exact(out.codes.cpu().numpy(), o["codes"], "C4 codes")
    assert_exact(out.scales.cpu().numpy(), o["scales"], "C4 scales")
    if fmt == "nvfp4":
        assert_exact(out.global_scale.cpu().numpy(), np.array([o["global_scale"]], np.float32), "C4 s_g")
    odc = oracle.focus_bwd(u16(w), u16(gr), u16(c), 8)
    gdc = dc.cpu().numpy()
    W = (u16(w).astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(4096, -1, 8)
    G = (u16(gr).astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(4096, -1, 8)
    C = c.float().numpy().astype(np.float64)
    scale = np.maximum(np.abs(odc), np.abs(G * W).sum(axis=2) / C ** 2)
    assert float((np.abs(gdc - odc) / np.maximum(scale, 1e-38)).max()) <= 1e-5
    assert_exact(gdc, odc, "C4 dc (bit-exact)")


@pytest.mark.parametrize("fmt,block,strat,rot", [("nvfp4", 16, "four_over_six", 16),
                                                 ("mxfp4", 32, "absmax", 128)])
def test_c5_full_activations_sampled(gpu, fmt, block, strat, rot):
    x = synth.workload("c5_activation_channels")["x"]
    rows = sample_rows(x.shape[0], k=10, seed=rot)
    xs = x[rows]
    ga = float(oracle.global_amax(u16(x), rot)) if fmt == "nvfp4" else None
    for supplied in ((False, True) if fmt == "nvfp4" else (False,)):
        g = gpu_quantize(gpu, x, fmt, block, strat, rot, gamax=ga if supplied else None, mse=False)
        o = oracle_quantize(xs, fmt, block, strat, rot, gamax=ga, mse=False)
        g = {"codes": g["codes"][rows], "scales": g["scales"][rows], "gs": g["gs"], "mse": None,
             "dq": None}
        compare_quant(g, o, fmt, f"C5 {fmt} H{rot} supplied={supplied}")


# ------------------------------------------------------------- edge cases

def test_empty_tensor(gpu):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    out = gpu.quantize(x, "nvfp4", 16, "absmax", 0)
    torch.cuda.synchronize()
    assert out.global_scale.item() == 1.0 == float(oracle.global_scale(0.0))
    out = gpu.quantize(x, "mxfp4", 32, "absmax", 0)
    assert out.codes.numel() == 0


@pytest.mark.parametrize("case", ["zeros", "tiny", "huge", "ties"])
def test_special_values(gpu, case):
    rng = np.random.default_rng(3)
    if case == "zeros":
        a = np.zeros((4, 128))
        a[1] = -0.0
    elif case == "tiny":  # bf16 subnormals and the smallest normals
        a = rng.choice([-1, 1], size=(4, 128)) * rng.integers(1, 200, size=(4, 128)) * 2.0 ** -133
    elif case == "huge":
        a = rng.standard_normal((4, 128)) * 1e37
    else:  # values on E2M1 midpoints once scaled by the block scale
        a = rng.choice([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -5.0, -0.25], size=(4, 128))
        a[:, ::16] = 6.0
    x = synth.to_bf16(a)
    for fmt, block, strat in [("nvfp4", 16, "absmax"), ("nvfp4", 16, "prevent_zero"),
                              ("nvfp4", 4, "four_over_six"), ("nvfp4", 8, "brute_force"),
                              ("mxfp4", 32, "absmax"), ("ue5m3", 16, "absmax"),
                              ("ue5m3", 4, "four_over_six"), ("ue5m3", 8, "brute_force"),
                              ("ue5m3", 32, "prevent_zero")]:
        rots = (0,) if case == "huge" else (0, 16, 128)
        for rot in rots:
            for ga in (None, 2688.0, 1e-30, 0.0, -1.0, float("inf")) if fmt == "nvfp4" else (None,):
                g = gpu_quantize(gpu, x, fmt, block, strat, rot, gamax=ga, dq=torch.float32)
                o = oracle_quantize(x, fmt, block, strat, rot, gamax=ga, dq=torch.float32)
                compare_quant(g, o, fmt, f"{case} {fmt} B{block} {strat} H{rot} ga={ga}")


# ------------------------------------------------------ dequant, block MSE

@pytest.mark.parametrize("fmt,block", [("nvfp4", 4), ("nvfp4", 8), ("nvfp4", 16), ("nvfp4", 32),
                                       ("mxfp4", 32), ("ue5m3", 4), ("ue5m3", 16), ("ue5m3", 32)])
def test_dequantize_and_block_mse_any_bytes(gpu, fmt, block):
    rng = np.random.default_rng(block)
    rows, cols = 7, 8 * block if block >= 8 else 36  # 7*36 = 252: ragged last segment
    codes = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    scales = rng.integers(0, 256, size=(rows, cols // block), dtype=np.uint8)
    sg = np.float32(3.1e-3)
    gs = torch.tensor([sg], device="cuda") if fmt == "nvfp4" else None
    for dt, name in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        out = gpu.dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), gs,
                             fmt, block, dt)
        torch.cuda.synchronize()
        got = out.cpu().numpy() if dt == torch.float32 else u16(out)
        want = oracle.dequantize(codes, scales, sg, rows, cols, fmt, block, name)
        gf = got.astype(np.float32) if name == "f32" else (got.astype(np.uint32) << 16).view(np.float32)
        wf = want if name == "f32" else (want.astype(np.uint32) << 16).view(np.float32)
        nan = np.isnan(wf)
        assert np.array_equal(np.isnan(gf), nan)
        assert_exact(got[~nan], want[~nan], f"dequant {fmt} B{block} {name}")
    # block MSE of real data against its own codes equals quantize's MSE
    for rot in (0, 16, 32):
        if cols % max(rot, 1):
            continue
        x = mixed(rows, cols, seed=block + rot)
        q = gpu_quantize(gpu, x, fmt, block, "absmax", rot)
        gs2 = torch.tensor([q["gs"]], device="cuda") if fmt == "nvfp4" else None
        m = gpu.block_mse(x.cuda(), torch.from_numpy(q["codes"]).cuda(),
                          torch.from_numpy(q["scales"]).cuda(), gs2, fmt, block, rot)
        torch.cuda.synchronize()
        want = oracle.block_mse(u16(x), q["codes"], q["scales"], q["gs"], fmt, block, rot)
        assert_mse(m.cpu().numpy(), want, f"block_mse {fmt} B{block} H{rot}")
        assert_exact(m.cpu().numpy(), q["mse"], "block_mse == quantize mse")


@pytest.mark.parametrize("fmt,block", [("nvfp4", 4), ("nvfp4", 8), ("nvfp4", 16), ("nvfp4", 32),
                                       ("mxfp4", 32), ("ue5m3", 8), ("ue5m3", 32)])
@pytest.mark.parametrize("rot", [16, 32, 64, 128])
def test_dequantize_unrotate(gpu, fmt, block, rot):
    """Dequantization back to the original domain (the normalised rotation
    applied again) on real codes of real data and on arbitrary code and scale
    bytes."""
    # a flattened length that is not a multiple of 32 where the shape allows it
    rows, cols = 9, 2 * max(rot, block, 32) + (16 if rot == 16 and block <= 16 else 0)
    x = mixed(rows, cols, seed=rot + block)
    q = gpu_quantize(gpu, x, fmt, block, "absmax", rot)
    rng = np.random.default_rng(rot * block)
    raw_codes = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    # scale bytes whose values stay finite through the butterflies (an infinity
    # would turn into NaN, whose bit pattern is not part of the contract)
    raw_scales = rng.integers(0, {"nvfp4": 127, "mxfp4": 201, "ue5m3": 255}[fmt],
                              size=(rows, cols // block), dtype=np.uint8)
    for codes, scales, sg, what in ((q["codes"], q["scales"], q["gs"], "quantized"),
                                    (raw_codes, raw_scales, np.float32(3.1e-3), "raw bytes")):
        gs = torch.tensor([sg], device="cuda") if fmt == "nvfp4" else None
        for dt, name in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
            out = gpu.dequantize(torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
                                 torch.from_numpy(np.ascontiguousarray(scales)).cuda(), gs, fmt,
                                 block, dt, rot=rot)
            torch.cuda.synchronize()
            got = out.cpu().numpy() if dt == torch.float32 else u16(out)
            want = oracle.dequantize_unrotate(codes, scales, sg if fmt == "nvfp4" else None, rows,
                                              cols, fmt, block, rot, name)
            assert_exact(got, want, f"dequant-unrotate {fmt} B{block} H{rot} {name} {what}")


def test_global_amax(gpu):
    x = mixed(9, 256, seed=5)
    for rot in (0, 16, 32, 64, 128):
        a = gpu.global_amax(x.cuda(), rot)
        torch.cuda.synchronize()
        assert_exact(a.cpu().numpy(), np.array([oracle.global_amax(u16(x), rot)], np.float32),
                     f"amax H{rot}")


# -------------------------------------------------------------------- FOCUS

@pytest.mark.parametrize("fmt,block", [("nvfp4", 4), ("nvfp4", 8), ("nvfp4", 16), ("nvfp4", 32),
                                       ("mxfp4", 32)])
@pytest.mark.parametrize("sub", [2, 4, 8, 16, 32])
def test_focus_small(gpu, fmt, block, sub):
    if sub > block:
        pytest.skip("sub-block larger than the block")
    rng = np.random.default_rng(block * 100 + sub)
    for rows, cols in ((3, 64), (5, 48 if block <= 16 else 96), (1, 32)):
        if cols % block:
            continue
        w = mixed(rows, cols, seed=sub + rows)
        cv = rng.uniform(0.5, 1.6, size=(rows, cols // sub))
        cv.reshape(-1)[:: 7] *= -1.0   # negative coefficients flip the codes' sign
        cv.reshape(-1)[3:: 11] = 1e-4  # tiny coefficients saturate the codes
        c = synth.to_fp16(cv)
        gr = mixed(rows, cols, seed=99 + rows)
        for dt, name in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
            out = gpu.focus_fwd(w.cuda(), c.cuda(), fmt, block, sub, out_dtype=dt, want_codes=True)
            torch.cuda.synchronize()
            o = oracle.focus_fwd(u16(w), u16(c), fmt, block, sub, out=name)
            got = out.w_hat.cpu().numpy() if name == "f32" else u16(out.w_hat)
            assert_exact(got, o["w_hat"], f"focus {fmt} B{block} sub{sub} {rows}x{cols} {name}")
            assert_exact(out.codes.cpu().numpy(), o["codes"], "focus codes")
            assert_exact(out.scales.cpu().numpy(), o["scales"], "focus scales")
        dc = gpu.focus_bwd(w.cuda(), gr.cuda(), c.cuda(), sub)
        torch.cuda.synchronize()
        assert_exact(dc.cpu().numpy(), oracle.focus_bwd(u16(w), u16(gr), u16(c), sub), "focus dc")


@pytest.mark.parametrize("loads", ["direct", "tma"])
def test_multi_tile_tma_tails(gpu, monkeypatch, loads):
    """Row counts around the 4096-element TMA tile and the persistent grid,
    including a last tile that is mostly past the end of the tensor."""
    monkeypatch.setenv("FP4Q_TMA", "1" if loads == "tma" else "0")
    for rows, cols in ((65, 64), (64 * 3 + 1, 128), (4096 * 2 + 64, 64), (1, 4096 * 4)):
        x = mixed(rows, cols, seed=rows)
        for fmt, block, strat, rot in (("nvfp4", 16, "four_over_six", 16), ("mxfp4", 32, "absmax", 64),
                                       ("nvfp4", 4, "absmax", 0)):
            g = gpu_quantize(gpu, x, fmt, block, strat, rot, dq=torch.bfloat16)
            o = oracle_quantize(x, fmt, block, strat, rot, dq=torch.bfloat16)
            compare_quant(g, o, fmt, f"tails {rows}x{cols} {fmt} B{block} {strat} H{rot}")
    assert gpu._abi.load().fp4q_device_errors() == 0


def test_side_stream(gpu):
    x = mixed(64, 256, seed=8).cuda()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = gpu.quantize(x, "nvfp4", 16, "four_over_six", 32, want_mse=True)
    s.synchronize()
    b = gpu.quantize(x, "nvfp4", 16, "four_over_six", 32, want_mse=True)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
    assert torch.equal(a.mse.view(torch.int32), b.mse.view(torch.int32))
    assert gpu._abi.load().fp4q_device_errors() == 0


# ---------------------------------------------- folded rotation factor

@pytest.mark.parametrize("rot", [16, 64])
def test_fold_boundaries_nvfp4(gpu, rot):
    """NVFP4 / UE5M3 behind a 16- or 64-wide rotation fold the factor 1/sqrt(n)
    (a power of two) into the reciprocal when s_g lies in [2^-105, 2^110]; just
    inside and outside both ends (s_g = amax / 2688, amax supplied), with data
    at the scale of the blocks, codes, scales, MSE and dq equal the oracle's."""
    rng = np.random.default_rng(rot)
    lo, hi = 2.0 ** -105 * 2688, 2.0 ** 110 * 2688
    for ga in (lo * 0.999, lo * 1.001, hi * 0.999, hi * 1.001, 3.0e38):
        # data at the blocks' scale, small enough that no butterfly sum overflows
        a = rng.standard_normal((6, 256)) * (ga / (2 * rot))
        a[0, :16] = ga / (2 * rot)    # a constant block (one large butterfly sum)
        a[1, 3] = ga * 1e-30          # an element far below its block's scale
        x = synth.to_bf16(np.clip(a, -3.3e38, 3.3e38))
        for fmt, block, strat in [("nvfp4", 16, "four_over_six"), ("nvfp4", 4, "absmax"),
                                  ("nvfp4", 8, "prevent_zero")]:
            for mse, dq in ((True, torch.float32), (False, None)):
                g = gpu_quantize(gpu, x, fmt, block, strat, rot, gamax=float(np.float32(ga)), mse=mse, dq=dq)
                o = oracle_quantize(x, fmt, block, strat, rot, gamax=float(np.float32(ga)), mse=mse, dq=dq)
                compare_quant(g, o, fmt, f"fold {fmt} B{block} {strat} H{rot} ga={ga:.3e} mse={mse}")


@pytest.mark.parametrize("rot", [16, 32, 64, 128])
def test_fold_mxfp4(gpu, rot):
    """MXFP4 folds 1/sqrt(n) into its power-of-two reciprocal when codes only are
    wanted and 2^-e stays normal after the fold (e <= 122, checked per
    segment). Ordinary, large and tiny blocks in one tensor, with and without
    the MSE output (which never folds). For 16- and 32-wide rotations, chunks
    of equal values put a rotated block maximum at 2^125 (e = 123: the unfolded
    branch) with every rotated value finite; for 64 and 128 that maximum would
    need a butterfly sum beyond the fp32 range (inputs whose rotation
    overflows are outside the contract)."""
    rng = np.random.default_rng(rot + 1)
    a = rng.standard_normal((8, 512))
    a[1] *= 2.0 ** 100             # large blocks, folded
    a[3] *= 2.0 ** -120            # tiny blocks (subnormal products)
    a[4, ::7] = 0.0
    if rot in (16, 32):
        # t = rot * c in the first butterfly output (finite), y = t k >= 2^125
        c = 2.0 ** 123 if rot == 16 else 1.5 * 2.0 ** 122
        a[2, :rot] = c             # one chunk: e = 123, unfolded
        a[2, 2 * rot:3 * rot] = c / 4  # e = 121: folded
    x = synth.to_bf16(a)
    for mse, dq in ((False, None), (True, torch.bfloat16), (False, torch.float32)):
        g = gpu_quantize(gpu, x, "mxfp4", 32, "absmax", rot, mse=mse, dq=dq)
        o = oracle_quantize(x, "mxfp4", 32, "absmax", rot, mse=mse, dq=dq)
        compare_quant(g, o, "mxfp4", f"mx fold H{rot} mse={mse} dq={dq}")
