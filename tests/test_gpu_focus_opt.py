"""FOCUS calibration kernels vs the oracle, bit for bit, through the C ABI:
fp4q_focus_update (coefficient step from an external gradient) and
fp4q_focus_step (fused forward + weight-reconstruction gradient + step), over
several consecutive steps so that the optimizer state is carried.

Bar: master coefficients, their fp16 copy, Adam's moments and the per-sub-block
SSE bit-identical (every operation is a single IEEE fp32 operation in both).
Outputs are surrounded by guard words that must stay untouched.
"""
import numpy as np
import pytest
import torch

import oracle
from microscaling_fp4_quantization_bf16_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 64


def u16(t):
    return synth.bits16(t)


def assert_exact(got, want, what):
    g = np.ascontiguousarray(got).reshape(-1)
    w = np.ascontiguousarray(want).reshape(-1)
    if g.dtype == np.float32:
        g, w = g.view(np.uint32), w.view(np.uint32)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    bad = np.nonzero(g != w)[0]
    assert bad.size == 0, f"{what}: {bad.size}/{g.size} differ; first {bad[:4]}: {g[bad[:4]]} vs {w[bad[:4]]}"


class Guarded:
    """A device buffer of n elements followed by GUARD poisoned elements."""

    def __init__(self, host: np.ndarray, dtype: torch.dtype, poison):
        self.n = host.size
        self.shape = host.shape
        full = torch.full((self.n + GUARD,), poison, dtype=dtype)
        full[: self.n] = torch.from_numpy(np.ascontiguousarray(host).reshape(-1).copy())
        self.buf = full.cuda()
        self.poison = poison

    @property
    def t(self):
        return self.buf[: self.n].view(self.shape)

    def host(self):
        full = self.buf.cpu()
        tail = full[self.n:]
        assert torch.all(tail == self.poison), "write past the end of an output"
        return full[: self.n].numpy().reshape(self.shape)


def coeffs(rows, nk, seed):
    rng = np.random.default_rng(seed)
    c = rng.uniform(0.8, 1.2, (rows, nk)).astype(np.float32)
    # values at and between fp16 ties around 1 (ulp 2^-10), one exact 1.0
    c.reshape(-1)[::13] = np.float32(1 + 2.0 ** -11)
    c.reshape(-1)[5::17] = np.float32(1 + 3 * 2.0 ** -11)
    c.reshape(-1)[7::19] = 1.0
    return c


def run_update(gpu, w, g, state, sub, opt, lr, t):
    L = gpu._abi.load()
    st = L.fp4q_focus_update(w.data_ptr(), g.data_ptr(), state["c"].t.data_ptr(),
                             state["ch"].t.data_ptr(),
                             state["m"].t.data_ptr() if opt == "adam" else None,
                             state["v"].t.data_ptr() if opt == "adam" else None,
                             w.shape[0], w.shape[1], sub, 1 if opt == "adam" else 0,
                             lr, 0.9, 0.999, 1e-8, t, None)
    assert st == 0, st


def run_step(gpu, w, state, fmt, block, sub, opt, lr, t, ga, gs, sse):
    L = gpu._abi.load()
    st = L.fp4q_focus_step(w.data_ptr(), w.shape[0], w.shape[1], 0 if fmt == "nvfp4" else 1,
                           block, sub, None if ga is None else ga.data_ptr(),
                           None if gs is None else gs.data_ptr(), state["c"].t.data_ptr(),
                           state["ch"].t.data_ptr(),
                           state["m"].t.data_ptr() if opt == "adam" else None,
                           state["v"].t.data_ptr() if opt == "adam" else None,
                           sse.t.data_ptr(), 1 if opt == "adam" else 0, lr, 0.9, 0.999, 1e-8, t,
                           None)
    assert st == 0, st


def new_state(c):
    z = np.zeros_like(c)
    return {"c": Guarded(c, torch.float32, -7.0), "ch": Guarded(np.zeros(c.shape, np.int16),
                                                               torch.int16, -21555),
            "m": Guarded(z, torch.float32, -7.0), "v": Guarded(z, torch.float32, -7.0)}


def check_state(state, o, opt, what):
    assert_exact(state["c"].host(), o["c"], what + " c")
    assert_exact(state["ch"].host().view(np.uint16), o["c_half"], what + " c_half")
    if opt == "adam":
        assert_exact(state["m"].host(), o["m"], what + " m")
        assert_exact(state["v"].host(), o["v"], what + " v")


@pytest.mark.parametrize("opt", ["sgd", "adam"])
@pytest.mark.parametrize("sub", [2, 4, 8, 16, 32])
def test_focus_update_parity(gpu, sub, opt):
    for rows, cols in ((37, 96), (3, 32), (129, 64)):
        if cols % sub:
            continue
        w = synth.gaussian(rows, cols, seed=rows + sub, std=0.02)
        c0 = coeffs(rows, cols // sub, seed=sub)
        state = new_state(c0)
        oc, om, ov = c0, None, None
        wd = w.cuda()
        for t in (1, 2, 3):
            g = synth.gaussian(rows, cols, seed=100 * t + sub)
            g.view(-1)[: sub] = 0          # one sub-block with a zero gradient
            run_update(gpu, wd, g.cuda(), state, sub, opt, 3e-3, t)
            o = oracle.focus_update(u16(w), u16(g), oc, om, ov, sub=sub, opt=opt, lr=3e-3, t=t)
            oc, om, ov = o["c"], o["m"], o["v"]
            check_state(state, o, opt, f"update {rows}x{cols} sub{sub} {opt} t{t}")
    assert gpu._abi.load().fp4q_device_errors() == 0


STEP_CASES = [("nvfp4", 4, 2), ("nvfp4", 4, 4), ("nvfp4", 8, 8), ("nvfp4", 16, 8),
              ("nvfp4", 16, 16), ("nvfp4", 32, 4), ("mxfp4", 32, 8), ("mxfp4", 32, 32),
              ("mxfp4", 32, 2)]


@pytest.mark.parametrize("opt", ["sgd", "adam"])
@pytest.mark.parametrize("fmt,block,sub", STEP_CASES)
def test_focus_step_parity(gpu, fmt, block, sub, opt):
    shapes = [(33, 160), (2, 32), (130, 64)] + ([(3, 48)] if block <= 16 else [])
    for rows, cols in shapes:
        w = synth.student_t(rows, cols, seed=rows * block + sub)
        w.view(-1)[32: 32 + block] = 0     # an all-zero block: S_dq = 0
        c0 = coeffs(rows, cols // sub, seed=block + sub)
        state = new_state(c0)
        sse = Guarded(np.zeros((rows, cols // sub), np.float32), torch.float32, -7.0)
        nv = fmt == "nvfp4"
        gs = torch.zeros(1, dtype=torch.float32, device="cuda") if nv else None
        oc, om, ov = c0, None, None
        wd = w.cuda()
        for t in (1, 2, 3):
            given = nv and t == 2            # step 2 is handed the abs-max, the others compute it
            amax = float(np.abs(w.float().numpy()).max())
            ga = torch.tensor([amax], dtype=torch.float32, device="cuda") if given else None
            run_step(gpu, wd, state, fmt, block, sub, opt, 2e-3, t, ga, gs, sse)
            o = oracle.focus_step(u16(w), oc, om, ov, fmt=fmt, block=block, sub=sub,
                                  global_amax=amax if given else None, opt=opt, lr=2e-3, t=t)
            oc, om, ov = o["c"], o["m"], o["v"]
            what = f"step {fmt} B{block} sub{sub} {opt} {rows}x{cols} t{t}"
            check_state(state, o, opt, what)
            assert_exact(sse.host(), o["sse"], what + " sse")
            if nv:
                assert_exact(gs.cpu().numpy(), np.array([o["global_scale"]], np.float32),
                             what + " s_g")
    assert gpu._abi.load().fp4q_device_errors() == 0


def test_focus_step_full_size_sampled_rows(gpu):
    """The 4096 x 4096 weight of the FOCUS workload (NVFP4 B16, sub-block 8, Adam,
    the launch the benchmark times): two steps on the whole tensor, compared on
    the first and last 48 rows with the oracle given the full tensor's abs-max."""
    rows = cols = 4096
    w = synth.gaussian(rows, cols, seed=3, std=0.02)
    amax = float(np.abs(w.float().numpy()).max())
    c0 = coeffs(rows, cols // 8, seed=4)
    wd = w.cuda()
    ga = torch.tensor([amax], dtype=torch.float32, device="cuda")
    gs = torch.zeros(1, dtype=torch.float32, device="cuda")
    c = torch.from_numpy(c0).cuda()
    ch = torch.empty(rows, cols // 8, dtype=torch.float16, device="cuda")
    m = torch.zeros_like(c)
    v = torch.zeros_like(c)
    sse = torch.empty_like(c)
    L = gpu._abi.load()
    for t in (1, 2):
        st = L.fp4q_focus_step(wd.data_ptr(), rows, cols, 0, 16, 8, ga.data_ptr(), gs.data_ptr(),
                               c.data_ptr(), ch.data_ptr(), m.data_ptr(), v.data_ptr(),
                               sse.data_ptr(), 1, 1e-3, 0.9, 0.999, 1e-8, t, None)
        assert st == 0
    torch.cuda.synchronize()
    wb = u16(w)
    for lo, hi in ((0, 48), (rows - 48, rows)):
        oc, om, ov = c0[lo:hi], None, None
        for t in (1, 2):
            o = oracle.focus_step(wb[lo:hi], oc, om, ov, fmt="nvfp4", block=16, sub=8,
                                  global_amax=amax, opt="adam", lr=1e-3, t=t)
            oc, om, ov = o["c"], o["m"], o["v"]
        assert_exact(c[lo:hi].cpu().numpy(), o["c"], f"full rows {lo}:{hi} c")
        assert_exact(u16(ch[lo:hi].cpu()), o["c_half"], f"full rows {lo}:{hi} c_half")
        assert_exact(m[lo:hi].cpu().numpy(), o["m"], f"full rows {lo}:{hi} m")
        assert_exact(v[lo:hi].cpu().numpy(), o["v"], f"full rows {lo}:{hi} v")
        assert_exact(sse[lo:hi].cpu().numpy(), o["sse"], f"full rows {lo}:{hi} sse")


def test_layer_objective_loop(gpu):
    """The calibration loop on a layer-output loss |X (W_hat - W)^T|^2: each step
    the GPU forward must equal the oracle's bit for bit; the gradient 2 E H is
    formed on the host from that (identical) W_hat, and the GPU update must
    equal the oracle's. The loss falls over the steps."""
    import focus_layer as prob
    rows, cols, sub = 128, 256, 8
    wb, h = prob.layer_problem(rows, cols, 1024, seed=0)
    wd = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).cuda()
    c0 = np.ones((rows, cols // sub), np.float32)
    state = gpu.focus_state(rows, cols, sub, "adam", device="cuda")
    oc, om, ov = c0, None, None
    losses = []
    for t in range(1, 31):
        out = gpu.focus_fwd(wd, state.c_half, "nvfp4", 16, sub, out_dtype=torch.float32)
        ch = np.asarray(oc, np.float32).astype(np.float16).view(np.uint16)
        ofwd = oracle.focus_fwd(wb, ch, "nvfp4", 16, sub, out="f32", want_codes=False)
        torch.cuda.synchronize()
        assert_exact(out.w_hat.cpu().numpy(), ofwd["w_hat"], f"layer loop fwd t{t}")
        loss, g = prob.layer_loss_and_grad(oracle, wb, oc, h)
        losses.append(loss)
        gpu.focus_update(wd, torch.from_numpy(g.view(np.int16)).view(torch.bfloat16).cuda(),
                         state, sub, lr=2e-4)
        o = oracle.focus_update(wb, g, oc, om, ov, sub=sub, opt="adam", lr=2e-4, t=t)
        oc, om, ov = o["c"], o["m"], o["v"]
        torch.cuda.synchronize()
        assert_exact(state.c.cpu().numpy(), oc, f"layer loop c t{t}")
        assert_exact(u16(state.c_half.cpu()), o["c_half"], f"layer loop c_half t{t}")
        assert_exact(state.m.cpu().numpy(), om, f"layer loop m t{t}")
    assert losses[-1] < losses[0]


def test_empty_inputs(gpu):
    """rows == 0: every new entry point returns without launching; NVFP4 still
    publishes s_g = 1 for the fused step, as the forward does."""
    L = gpu._abi.load()
    w = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.empty(0, 8, dtype=torch.float32, device="cuda")
    gs = torch.full((1,), -3.0, device="cuda")
    assert L.fp4q_focus_update(w.data_ptr(), w.data_ptr(), c.data_ptr(), None, c.data_ptr(),
                               c.data_ptr(), 0, 64, 8, 1, 1e-3, 0.9, 0.999, 1e-8, 1, None) == 0
    assert L.fp4q_focus_step(w.data_ptr(), 0, 64, 0, 16, 8, None, gs.data_ptr(), c.data_ptr(), None,
                             c.data_ptr(), c.data_ptr(), None, 1, 1e-3, 0.9, 0.999, 1e-8, 1,
                             None) == 0
    torch.cuda.synchronize()
    assert gs.item() == 1.0
    u = torch.eye(128, device="cuda")
    for rot in (0, 128):
        assert L.fp4q_gptq(w.data_ptr(), 0, 128, 1, 32, rot, c.data_ptr(), None, u.data_ptr(), None,
                           c.data_ptr(), c.data_ptr(), None) == 0
    q = gpu.quantize(w, "ue5m3", 16, "four_over_six")
    torch.cuda.synchronize()
    assert q.codes.numel() == 0 and q.global_scale is None
