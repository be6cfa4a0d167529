"""GPTQ error feedback with static groups on the GPU vs the oracle, bit for
bit, through the C ABI: every code of small layers in several formats, block
sizes, scale strategies and processing orders, and sampled rows of a
4096 x 4096 layer (rows are independent given the scales and U)."""
import numpy as np
import pytest
import torch

import oracle
from microscaling_fp4_quantization_bf16_b200 import synth

pytestmark = pytest.mark.gpu


def u16(t):
    return synth.bits16(t)


def run_gpu(gpu, wb, scales, sg, U, perm, fmt, block, rot=0):
    w = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).cuda()
    sc = torch.from_numpy(np.ascontiguousarray(scales)).cuda()
    gs = None if sg is None else torch.tensor([sg], dtype=torch.float32, device="cuda")
    Ud = torch.from_numpy(np.ascontiguousarray(U, np.float32)).cuda()
    pd = None if perm is None else torch.from_numpy(np.ascontiguousarray(perm, np.int32)).cuda()
    guard = torch.full((w.shape[0] * w.shape[1] // 2 + 64,), 0xA5, dtype=torch.uint8, device="cuda")
    codes = gpu.gptq(w, sc, gs, Ud, pd, fmt, block, out=guard[: w.shape[0] * w.shape[1] // 2]
                     .view(w.shape[0], -1), rot=rot)
    torch.cuda.synchronize()
    assert torch.all(guard[-64:] == 0xA5), "write past the end of the codes"
    return codes.cpu().numpy()


CASES = [("nvfp4", 16, "absmax"), ("nvfp4", 4, "prevent_zero"), ("mxfp4", 32, "brute_force"),
         ("ue5m3", 8, "four_over_six"), ("nvfp4", 32, "brute_force")]


@pytest.mark.parametrize("fmt,block,strat", CASES)
@pytest.mark.parametrize("act_order", [True, False])
def test_gptq_small_layers(gpu, fmt, block, strat, act_order):
    # (45, 1152): nine batches, the trailing updates beside the next batch
    # kernel, a partial CTA of rows
    for rows, K, seed in ((37, 256, 1), (9, 384, 2), (70, 128, 3), (45, 1152, 4)):
        d = synth.gptq_problem(rows, K, 1024, seed=seed, act_order=act_order)
        wb = u16(d["w"])
        q = oracle.quantize(wb, fmt, block, strat, 0, want_mse=False)
        sg = q["global_scale"] if fmt == "nvfp4" else None
        perm = d["perm"] if act_order else None
        want = oracle.gptq(wb, q["scales"], sg, d["u"], perm, fmt, block)
        got = run_gpu(gpu, wb, q["scales"], sg, d["u"], perm, fmt, block)
        bad = np.nonzero(got != want)
        assert bad[0].size == 0, f"{fmt} B{block} {strat} {rows}x{K}: {bad[0].size} bytes differ"
    assert gpu._abi.load().fp4q_device_errors() == 0


def test_gptq_full_layer_sampled_rows(gpu):
    """4096 x 4096 NVFP4 B16 with MSE-optimal (brute-force) static scales and the
    activation order; the GPU quantizes every row, the oracle 2 x 24 rows with
    the tensor's own s_g."""
    rows = K = 4096
    d = synth.gptq_problem(rows, K, 4096, seed=11)
    wb = u16(d["w"])
    w = d["w"].cuda()
    ga = float(oracle.global_amax(wb, 0))
    gq = gpu.quantize(w, "nvfp4", 16, "brute_force", 0,
                      global_amax=torch.tensor([ga], device="cuda"))
    Ud = torch.from_numpy(d["u"]).cuda()
    pd = torch.from_numpy(d["perm"]).cuda()
    codes = gpu.gptq(w, gq.scales, gq.global_scale, Ud, pd, "nvfp4", 16)
    torch.cuda.synchronize()
    sg = float(gq.global_scale.item())
    for lo in (0, rows - 24):
        sl = slice(lo, lo + 24)
        oq = oracle.quantize(wb[sl], "nvfp4", 16, "brute_force", 0, global_amax=ga, want_mse=False)
        assert np.float32(oq["global_scale"]) == np.float32(sg)
        assert np.array_equal(gq.scales[sl].cpu().numpy(), oq["scales"])
        want = oracle.gptq(wb[sl], oq["scales"], oq["global_scale"], d["u"], d["perm"], "nvfp4", 16)
        assert np.array_equal(codes[sl].cpu().numpy(), want), f"rows {lo}..{lo + 23}"
    assert gpu._abi.load().fp4q_device_errors() == 0


def test_gptq_out_of_range_order_is_counted(gpu):
    # an entry outside 0..K-1 is caught by the kernel's bounds check: counted,
    # column 0 read instead, no access outside the buffers
    d = synth.gptq_problem(8, 128, 256, seed=5)
    wb = u16(d["w"])
    q = oracle.quantize(wb, "mxfp4", 32, "absmax", 0, want_mse=False)
    perm = d["perm"].copy()
    perm[5] = 128
    run_gpu(gpu, wb, q["scales"], None, d["u"], perm, "mxfp4", 32)
    assert gpu._abi.load().fp4q_device_errors() > 0


@pytest.mark.parametrize("fmt,block,strat,rot", [("nvfp4", 16, "absmax", 16), ("mxfp4", 32, "brute_force", 128),
                                                 ("ue5m3", 8, "four_over_six", 32), ("nvfp4", 32, "brute_force", 64)])
def test_gptq_rotated_small_layers(gpu, fmt, block, strat, rot):
    """MR-GPTQ's blockwise rotation in front of the feedback (static scales from
    the rotated quantizer, U from the rotated-basis Hessian), every code."""
    for rows, K, seed in ((37, 256, 5), (9, 384, 6), (70, 128, 7), (3, 1152, 8)):
        d = synth.gptq_problem(rows, K, 1024, seed=seed, rot=rot)
        wb = u16(d["w"])
        q = oracle.quantize(wb, fmt, block, strat, rot, want_mse=False)
        sg = q["global_scale"] if fmt == "nvfp4" else None
        want = oracle.gptq(wb, q["scales"], sg, d["u"], d["perm"], fmt, block, rot=rot)
        got = run_gpu(gpu, wb, q["scales"], sg, d["u"], d["perm"], fmt, block, rot=rot)
        bad = np.nonzero(got != want)
        assert bad[0].size == 0, f"{fmt} B{block} {strat} H{rot} {rows}x{K}: {bad[0].size} bytes differ"
    assert gpu._abi.load().fp4q_device_errors() == 0
