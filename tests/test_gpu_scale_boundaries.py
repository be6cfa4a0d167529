"""E4M3 scale selection where the quotient a_b / (T s_g) sits on, or within a
few fp32 units of, an E4M3 rounding boundary (GPU vs oracle, bit-exact).

The kernels form the quotient as a * fl(1 / (T s_g)) and fall back to the IEEE
division only near an E4M3 midpoint; the oracle always divides ("Finer is
Better (with the Right Scaling)", 手法 2: the abs-max scale and the 4-over-6
candidates). The cases are found by a deterministic search over supplied
global abs-max values G near 2688 a / (T m) for E4M3 midpoints m: kept are the
G where fl(a * fl(1/den)) and fl(a / den) round to different E4M3 codes, or
where fl(a / den) is the midpoint itself (a round-half-to-even tie).
"""
import numpy as np
import pytest
import torch

import oracle
from microscaling_fp4_quantization_bf16_b200 import synth

from test_gpu_parity import assert_exact, compare_quant, gpu_quantize, oracle_quantize

F32 = np.float32


def boundary_cases(n_ties=24):
    mids = [(oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2 for c in range(0x7E)]
    picked = [mids[i] for i in (0, 1, 3, 7, 8, 9, 15, 30, 47, 63, 64, 80, 100, 110, 120, 124)]
    amaxes = [1.5, 0.375, 3.0, 1.25, 0.8125, 0.0234375, 7.0]  # bf16-exact
    differ, ties = [], []
    for T in (6, 4):
        for a in amaxes:
            a32 = F32(a)
            for m in picked:
                g = F32(2688.0 * a / (T * m))
                cands = [g]
                up = dn = g
                for _ in range(48):
                    up = np.nextafter(up, F32(np.inf))
                    dn = np.nextafter(dn, F32(0))
                    cands += [up, dn]
                for G in cands:
                    sg = F32(G) / F32(2688)
                    den = F32(T) * sg
                    qf = a32 * (F32(1) / den)
                    qe = a32 / den
                    if oracle.rne_e4m3_sat(float(qf)) != oracle.rne_e4m3_sat(float(qe)):
                        differ.append((T, a, float(G)))
                    elif float(qe) == m:
                        ties.append((T, a, float(G)))
    # every differing case, then some ties, in a deterministic order
    return differ + ties[::max(1, len(ties) // n_ties)][:n_ties], len(differ)


CASES, N_DIFFER = boundary_cases()


def block_row(a, block, pattern):
    """One row of 2 blocks whose abs-max is a (bf16-exact)."""
    row = np.zeros(2 * block, np.float64)
    if pattern == "single":
        row[0] = a
        row[block] = -a
    else:  # a spread of values below a
        for j in range(2 * block):
            row[j] = a * (1.0 - (j % block) / (block + 3.0)) * (-1.0) ** j
    return synth.to_bf16(row.reshape(1, -1))


def test_search_found_cases():
    """Host-only: the search yields genuine shortcut failures and ties."""
    assert N_DIFFER >= 8, N_DIFFER  # the search must produce real shortcut failures
    assert len(CASES) >= 16


@pytest.mark.gpu
@pytest.mark.parametrize("block", [4, 16])
@pytest.mark.parametrize("strat", ["absmax", "prevent_zero", "four_over_six"])
def test_quantize_scale_on_boundaries(gpu, block, strat):
    four_won = 0
    for T, a, G in CASES:
        if strat != "four_over_six" and T == 4:
            continue
        for pattern in ("single", "spread"):
            x = block_row(a, block, pattern)
            what = f"T={T} a={a} G={G!r} {pattern} B{block} {strat}"
            g = gpu_quantize(gpu, x, "nvfp4", block, strat, 0, gamax=G, mse=True, dq=torch.float32)
            o = oracle_quantize(x, "nvfp4", block, strat, 0, gamax=G, mse=True, dq=torch.float32)
            compare_quant(g, o, "nvfp4", what)
            if strat == "four_over_six":
                ab = oracle.quantize(synth.bits16(x), "nvfp4", block, "absmax", 0, global_amax=G)
                four_won += int(np.any(o["scales"] != ab["scales"]))
    if strat == "four_over_six":
        assert four_won > 0  # the 4 candidate's code was used somewhere


@pytest.mark.gpu
def test_focus_scale_on_boundaries(gpu):
    for T, a, G in CASES:
        if T != 6:
            continue
        x = block_row(a, 16, "spread")
        c = synth.to_fp16(np.ones((1, 32 // 8)))
        ga = torch.tensor([G], dtype=torch.float32, device="cuda")
        out = gpu.focus_fwd(x.cuda(), c.cuda(), "nvfp4", 16, 8, global_amax=ga,
                            out_dtype=torch.float32, want_codes=True)
        torch.cuda.synchronize()
        o = oracle.focus_fwd(synth.bits16(x), synth.bits16(c), "nvfp4", 16, 8, global_amax=G,
                             out="f32", want_codes=True)
        what = f"FOCUS a={a} G={G!r}"
        assert_exact(out.scales.cpu().numpy(), o["scales"], what + " scales")
        assert_exact(out.codes.cpu().numpy(), o["codes"], what + " codes")
        assert_exact(out.w_hat.cpu().numpy(), o["w_hat"], what + " w_hat")
