"""GPU rounding primitives against the oracle, over every fp32 bit pattern.

The oracle's E2M1 and E4M3 roundings are non-decreasing in |u| (pinned in
test_oracle_formats.py), so over the positive bit patterns (which order like
the floats) each is a step function. The interval boundaries are found by
bisection with oracle calls only; then all 2^32 GPU results are compared with
those oracle intervals on the device. A random and a dense subset are also
compared with direct oracle calls.
"""
import numpy as np
import pytest
import torch

import oracle
from microscaling_fp4_quantization_bf16_b200 import synth

pytestmark = pytest.mark.gpu

POS_INF = 0x7F800000


def _f(bits: int) -> float:
    return float(np.array([bits], np.uint32).view(np.float32)[0])


def oracle_steps(fn, lo: int, hi: int):
    """Intervals [start_k, start_{k+1}) of bit patterns in [lo, hi] on which
    the monotone oracle function fn(float) is constant: (starts, values)."""
    starts, vals = [lo], [fn(_f(lo))]
    b = lo
    while True:
        c = fn(_f(b))
        if fn(_f(hi)) == c:
            break
        a, z = b, hi  # fn(a) == c, fn(z) != c
        while z - a > 1:
            m = (a + z) // 2
            if fn(_f(m)) == c:
                a = m
            else:
                z = m
        starts.append(z)
        vals.append(fn(_f(z)))
        b = z
    return starts, vals


def _chunks(total: int, ch: int):
    for first in range(0, total, ch):
        yield first, min(ch, total - first)


def _patterns(first: int, n: int) -> torch.Tensor:
    base = first - (1 << 32) if first >= (1 << 31) else first
    return (torch.arange(n, dtype=torch.int64, device="cuda") + base).to(torch.int32)


def test_e2m1_all_patterns(gpu):
    starts, vals = oracle_steps(oracle.rne_e2m1, 0, POS_INF)
    assert vals == list(range(8))
    nstarts, nvals = oracle_steps(oracle.rne_e2m1, 0x80000000, 0x80000000 | POS_INF)
    assert nvals == list(range(8, 16))
    assert [s - 0x80000000 for s in nstarts] == starts  # sign-symmetric boundaries
    st = torch.tensor(starts, dtype=torch.int64, device="cuda")
    vt = torch.tensor(vals, dtype=torch.int64, device="cuda")
    checked = 0
    for first, n in _chunks(1 << 32, 1 << 28):
        bits = _patterns(first, n)
        codes = gpu.e2m1_encode(bits.view(torch.float32)).to(torch.int64)
        ub = bits.to(torch.int64) & 0xFFFFFFFF
        mag = ub & 0x7FFFFFFF
        keep = mag <= POS_INF  # NaN codes are unspecified
        want = vt[torch.searchsorted(st, mag, right=True) - 1] | ((ub >> 31) << 3)
        bad = (codes != want) & keep
        assert not bool(bad.any()), f"first mismatch at bits {int(ub[bad][0]):#x}"
        checked += int(keep.sum())
    assert checked == (1 << 32) - 2 * (0x7FFFFFFF - POS_INF)


def test_e4m3_all_nonnegative_patterns(gpu):
    starts, vals = oracle_steps(oracle.rne_e4m3_sat, 0, POS_INF)
    assert vals == list(range(0x7F))
    st = torch.tensor(starts, dtype=torch.int64, device="cuda")
    vt = torch.tensor(vals, dtype=torch.int64, device="cuda")
    for first, n in _chunks(POS_INF + 1, 1 << 28):
        bits = _patterns(first, n)
        codes = gpu.e4m3_encode(bits.view(torch.float32)).to(torch.int64)
        want = vt[torch.searchsorted(st, bits.to(torch.int64), right=True) - 1]
        bad = codes != want
        assert not bool(bad.any()), f"first mismatch at bits {int(bits[bad][0]):#x}"


def test_primitives_direct_oracle_sample(gpu):
    rng = np.random.default_rng(0)
    rnd = rng.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    pts = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 2 ** -10, 448.0, 432.0], np.float32)
    dense = (pts.view(np.uint32)[:, None].astype(np.int64) + np.arange(-2048, 2049)).ravel()
    bits = np.concatenate([rnd, dense.astype(np.uint32), dense.astype(np.uint32) | 0x80000000])
    u = bits.view(np.float32)
    finite = np.isfinite(u)
    got = gpu.e2m1_encode(torch.from_numpy(u.copy()).cuda()).cpu().numpy()
    assert np.array_equal(got[finite], oracle.rne_e2m1_array(u)[finite])
    v = np.abs(u[finite])
    got = gpu.e4m3_encode(torch.from_numpy(v.copy()).cuda()).cpu().numpy()
    assert np.array_equal(got, oracle.rne_e4m3_array(v))


def test_nibble_order_lane_layout(gpu):
    # element 2j -> low nibble: the packed codes of [0.5, 1] are 0x21
    x = synth.to_bf16(np.array([[0.5, 1.0] + [0.0] * 13 + [6.0]]))
    ga = torch.tensor([2688.0], device="cuda")
    out = gpu.quantize(x.cuda(), "nvfp4", 16, "absmax", 0, global_amax=ga)
    torch.cuda.synchronize()
    assert out.codes.cpu().numpy()[0, 0] == 0x21
    assert out.codes.cpu().numpy()[0, 7] == 0x70
