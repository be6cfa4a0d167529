"""The C-ABI library loads, exports every entry point declared in
include/fp4q.h, and rejects invalid arguments on the host before anything is
launched (so these run without a GPU).

Every call below has at least one invalid argument: the fake addresses are
never dereferenced because validation fails first.
"""
import ctypes as C
import os
import re

import pytest

from microscaling_fp4_quantization_bf16_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp4q.h")

OK, NULL, SHAPE, ALIGN, UNSUP, ALIAS, CUDA = range(7)
A = 0x100000     # a 16-byte-aligned fake device address
A2 = 0x200000
A3 = 0x300000
MIS = 0x100004   # 4-byte but not 16-byte aligned
NV, MX, UE = 0, 1, 2


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4q_[a-z0-9_]+)\s*\(", text)))


def test_header_and_library_agree(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in fp4q.h but not exported"
        assert n in _abi.SIGNATURES, f"{n} has no ctypes signature"
    assert sorted(_abi.SIGNATURES) == names


def test_status_strings(lib):
    for s in range(7):
        assert lib.fp4q_status_string(s)
    assert lib.fp4q_status_string(99) == b"unknown status"


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        _abi._lib_saved = _abi._lib
        try:
            _abi._lib = None
            _abi.load(str(tmp_path / "nope.so"))
        finally:
            _abi._lib = _abi._lib_saved


def q(lib, x=A, rows=4, cols=64, fmt=NV, block=16, strat=0, rot=0, gin=None, gout=A3 + 64,
      codes=A2, scales=A3, mse=None, dq=None, dqt=0):
    return lib.fp4q_quantize(x, rows, cols, fmt, block, strat, rot, gin, gout, codes, scales, mse,
                             dq, dqt, None)


def test_quantize_validation(lib):
    assert q(lib, x=None) == NULL
    assert q(lib, codes=None) == NULL
    assert q(lib, scales=None) == NULL
    assert q(lib, gout=None) == NULL                  # NVFP4 needs the global scale output
    assert q(lib, cols=24) == SHAPE                   # 24 % 16
    assert q(lib, rows=-1) == SHAPE
    assert q(lib, cols=-16) == SHAPE
    assert q(lib, rot=32, cols=48) == SHAPE           # 48 % 32
    assert q(lib, rows=1 << 30, cols=1 << 14) == SHAPE  # beyond 2^40 elements
    assert q(lib, x=MIS) == ALIGN
    assert q(lib, codes=MIS) == ALIGN
    assert q(lib, mse=MIS) == ALIGN
    assert q(lib, dq=MIS) == ALIGN
    assert q(lib, gout=A3 + 66) == ALIGN
    assert q(lib, fmt=MX, block=32, strat=2, gout=None) == UNSUP
    assert q(lib, fmt=MX, block=32, strat=1, gout=None) == UNSUP
    assert q(lib, fmt=MX, block=16, gout=None) == UNSUP
    assert q(lib, block=64) == UNSUP
    assert q(lib, block=2) == UNSUP
    assert q(lib, rot=8) == UNSUP
    assert q(lib, strat=4) == UNSUP
    assert q(lib, fmt=3) == UNSUP
    assert q(lib, fmt=UE, block=64, gout=None) == UNSUP   # UE5M3: blocks 4..32
    assert q(lib, fmt=UE, cols=24, gout=None) == SHAPE
    assert q(lib, fmt=UE, strat=4, gout=None) == UNSUP
    assert q(lib, fmt=UE, x=None, gout=None) == NULL       # no global scale needed, x is
    assert q(lib, dq=A, dqt=5) == UNSUP
    assert q(lib, gin=A3 + 64, gout=A3 + 64) == ALIAS


def test_other_entry_points_validation(lib):
    L = lib
    assert L.fp4q_dequantize(None, A, A, 4, 64, NV, 16, A, 0, None) == NULL
    assert L.fp4q_dequantize(A, A, None, 4, 64, NV, 16, A, 0, None) == NULL
    assert L.fp4q_dequantize(A, A, A, 4, 60, NV, 16, A, 0, None) == SHAPE
    assert L.fp4q_dequantize(A, MIS, A, 4, 64, NV, 16, A, 0, None) == ALIGN
    assert L.fp4q_dequantize(A, A, A, 4, 64, NV, 16, A, 3, None) == UNSUP
    du = lambda **k: L.fp4q_dequantize_unrotate(k.get("codes", A), A, k.get("gs", A), 4,
                                                k.get("cols", 128), NV, 16, k.get("rot", 32),
                                                k.get("out", A), k.get("ot", 0), None)
    assert du(rot=24) == UNSUP
    assert du(cols=96, rot=64) == SHAPE
    assert du(ot=4) == UNSUP
    assert du(codes=None) == NULL
    assert du(gs=None) == NULL
    assert du(out=MIS) == ALIGN
    assert L.fp4q_block_mse(A, A, A, A, 4, 64, NV, 16, 0, None, None) == NULL
    assert L.fp4q_block_mse(A, A, A, A, 4, 64, NV, 16, 128, A, None) == SHAPE
    assert L.fp4q_block_mse(A, A, A, MIS + 2, 4, 64, NV, 16, 0, A, None) == ALIGN
    # focus forward
    ff = lambda **k: L.fp4q_focus_fwd(k.get("w", A), k.get("c", A), 4, k.get("cols", 64),
                                      k.get("fmt", NV), k.get("block", 16), k.get("sub", 8),
                                      k.get("gin"), k.get("gout", A3), k.get("wh", A2),
                                      k.get("ot", 1), k.get("codes"), k.get("scales"), None)
    assert ff(sub=32) == UNSUP      # sub > block
    assert ff(sub=3) == UNSUP
    assert ff(sub=1) == UNSUP
    assert ff(ot=9) == UNSUP
    assert ff(codes=A) == NULL      # codes without scales
    assert ff(c=None) == NULL
    assert ff(w=MIS) == ALIGN
    assert ff(cols=40) == SHAPE
    assert ff(gin=A3, gout=A3) == ALIAS
    assert ff(fmt=UE) == UNSUP      # FOCUS is defined for NVFP4 and MXFP4
    # focus backward
    assert L.fp4q_focus_bwd(A, A, A, 4, 60, 8, A, None) == SHAPE
    assert L.fp4q_focus_bwd(A, A, A, 4, 64, 6, A, None) == UNSUP
    assert L.fp4q_focus_bwd(A, None, A, 4, 64, 8, A, None) == NULL
    assert L.fp4q_focus_bwd(A, A, A, 4, 64, 8, MIS, None) == ALIGN
    # focus calibration: coefficient update from a gradient, fused step
    fu = lambda **k: L.fp4q_focus_update(k.get("w", A), k.get("g", A), k.get("c", A),
                                         k.get("ch"), k.get("m", A2), k.get("v", A3), 4,
                                         k.get("cols", 64), k.get("sub", 8), k.get("opt", 1),
                                         1e-3, 0.9, 0.999, 1e-8, k.get("t", 1), None)
    assert fu(sub=6) == UNSUP
    assert fu(cols=60) == SHAPE
    assert fu(opt=2) == UNSUP
    assert fu(t=0) == UNSUP          # Adam counts steps from 1
    assert fu(m=None) == NULL        # Adam needs its moments
    assert fu(g=None) == NULL
    assert fu(ch=MIS) == ALIGN
    assert fu(v=MIS) == ALIGN
    fs = lambda **k: L.fp4q_focus_step(k.get("w", A), 4, k.get("cols", 64), k.get("fmt", NV),
                                       k.get("block", 16), k.get("sub", 8), k.get("gin"),
                                       k.get("gout", A3), k.get("c", A), None, k.get("m", A2),
                                       k.get("v", A2 + 4096), k.get("sse"), k.get("opt", 1),
                                       1e-3, 0.9, 0.999, 1e-8, k.get("t", 1), None)
    assert fs(sub=32) == UNSUP       # sub > block
    assert fs(fmt=MX, block=16) == UNSUP
    assert fs(cols=40) == SHAPE
    assert fs(opt=0, t=0, m=None, v=None, c=None) == NULL   # SGD ignores t, m, v; c required
    assert fs(t=-3) == UNSUP
    assert fs(v=None) == NULL
    assert fs(gout=None) == NULL     # NVFP4 writes s_g
    assert fs(sse=MIS) == ALIGN
    assert fs(gin=A3, gout=A3) == ALIAS
    assert fs(fmt=UE) == UNSUP
    # GPTQ error feedback
    gq = lambda **k: L.fp4q_gptq(k.get("w", A), 4, k.get("cols", 256), k.get("fmt", NV),
                                 k.get("block", 16), k.get("rot", 0), A, k.get("gs", A2), A3,
                                 k.get("perm"), k.get("work", A), k.get("codes", A2), None)
    assert gq(cols=192) == SHAPE      # cols % 128
    assert gq(cols=200) == SHAPE      # cols % block
    assert gq(block=64) == UNSUP
    assert gq(rot=24) == UNSUP
    assert gq(rot=128, cols=58368) == SHAPE   # rotated rows staged in 227 KB of shared memory
    assert gq(gs=None) == NULL        # NVFP4 needs s_g
    assert gq(work=None) == NULL
    assert gq(perm=MIS) == ALIGN
    assert gq(codes=MIS) == ALIGN
    # global amax, primitives
    assert L.fp4q_global_amax(A, 4, 64, 24, A, None) == UNSUP
    assert L.fp4q_global_amax(A, 4, 48, 32, A, None) == SHAPE
    assert L.fp4q_global_amax(A, 4, 64, 0, A + 2, None) == ALIGN
    assert L.fp4q_global_amax(None, 4, 64, 0, A, None) == NULL
    assert L.fp4q_e2m1_encode(A, -1, A, None) == SHAPE
    assert L.fp4q_e2m1_encode(MIS, 8, A, None) == ALIGN
    assert L.fp4q_e4m3_encode(A, 8, None, None) == NULL


def test_python_wrapper_rejects_cpu_tensors():
    import torch
    import microscaling_fp4_quantization_bf16_b200 as fp4q
    with pytest.raises(ValueError, match="CUDA"):
        fp4q.quantize(torch.zeros(4, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        fp4q.focus_bwd(torch.zeros(4, 64, dtype=torch.bfloat16),
                       torch.zeros(4, 64, dtype=torch.bfloat16), torch.zeros(4, 8))


def test_gemm_validation(lib):
    L = lib
    assert L.fp4q_gemm(A, A, A, A, A, A, 128, 128, 48, NV, A, A, 0, None) == SHAPE  # K % 32
    assert L.fp4q_gemm(A, A, A, A, A, A, 128, 130, 64, NV, A, A, 0, None) == SHAPE  # N % 4 (fp32)
    assert L.fp4q_gemm(A, A, A, A, A, A, 128, 132, 64, NV, A, A, 1, None) == SHAPE  # N % 8 (bf16)
    assert L.fp4q_gemm(A, A, None, A, A, A, 128, 128, 64, NV, A, A, 0, None) == NULL  # NVFP4 s_g
    assert L.fp4q_gemm(A, A, A, A, A, A, 128, 128, 64, NV, None, A, 0, None) == NULL  # alpha_out
    assert L.fp4q_gemm(MIS, A, A, A, A, A, 128, 128, 64, NV, A, A, 0, None) == ALIGN
    assert L.fp4q_gemm(A, A, A, A, A, A, 128, 128, 64, 2, A, A, 0, None) == UNSUP
    assert L.fp4q_gemm(A, A, A, A, A, A, 128, 128, 64, NV, A, A, 5, None) == UNSUP
    assert L.fp4q_mma_scale_bytes(128, 48, NV) == 512   # 128 rows x 3 blocks, padded to 4
    assert L.fp4q_mma_scale_bytes(300, 64, MX) == 384 * 4  # rows padded to 384, 2 blocks -> 4
    assert L.fp4q_mma_scale_bytes(128, 40, NV) == 0
    assert L.fp4q_scales_to_mma(A, 128, 40, NV, A, None) == SHAPE
    assert L.fp4q_scales_to_mma(None, 128, 64, NV, A, None) == NULL
    qm = lambda **k: L.fp4q_quantize_mma(A, 4, k.get("cols", 64), k.get("fmt", NV), 0, 0, None,
                                         A3, A2, k.get("sc", A), None)
    assert qm(cols=48) == SHAPE      # not a multiple of 32
    assert qm(fmt=3) == UNSUP
    assert qm(sc=None) == NULL
    assert qm(sc=MIS) == ALIGN
    assert qm(fmt=UE) == UNSUP       # the MMA takes E4M3 / E8M0 scales only
    assert L.fp4q_mma_scale_bytes(128, 64, UE) == 0
    assert L.fp4q_scales_to_mma(A, 128, 64, UE, A, None) == UNSUP


def test_header_is_plain_c(tmp_path):
    """include/fp4q.h compiles as ISO C11 (pedantic) and C++17: no torch or C++
    types in the interface."""
    import shutil
    import subprocess
    cuda_inc = "/usr/local/cuda/include"
    if shutil.which("gcc") is None or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime_api.h")):
        pytest.skip("gcc or the CUDA headers are not available")
    src = tmp_path / "h.c"
    src.write_text('#include "fp4q.h"\nint main(void) { return (int)FP4Q_OK; }\n')
    for cc, std, name in (("gcc", "-std=c11", "h.c"), ("g++", "-std=c++17", "h.cpp")):
        f = tmp_path / name
        f.write_text(src.read_text())
        r = subprocess.run([cc, std, "-Wall", "-Wextra", "-pedantic", "-Werror",
                            "-I" + os.path.dirname(HEADER), "-I" + cuda_inc, "-c", str(f),
                            "-o", str(tmp_path / (name + ".o"))], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_injected_cuda_error_every_entry_point(lib):
    """The CUDA-error path, host side only: with fp4q_debug_fail_launches set,
    every entry point that enqueues work validates its (valid) arguments,
    returns FP4Q_ERR_CUDA with the injected code for fp4q_last_cuda_error,
    and touches nothing. Host buffers stand in for the device arrays: no
    kernel, memset or copy may reach them (on a machine without a GPU a
    CUDA call would fail with a different code)."""
    import numpy as np

    bufs = [np.full(1 << 16, 0xA5, np.uint8) for _ in range(12)]
    for b in bufs:
        assert b.ctypes.data % 16 == 0
    p = [b.ctypes.data for b in bufs]
    X, CODES, SCALES, GS, OUT, MSE, C, G, M, V, U, W = p
    NVF, ADAM, F32 = NV, 1, 0
    calls = {
        "fp4q_quantize": lambda: lib.fp4q_quantize(X, 4, 64, NVF, 16, 0, 0, None, GS, CODES, SCALES,
                                                   MSE, OUT, F32, None),
        "fp4q_quantize_mma": lambda: lib.fp4q_quantize_mma(X, 4, 64, NVF, 0, 0, None, GS, CODES,
                                                           SCALES, None),
        "fp4q_dequantize": lambda: lib.fp4q_dequantize(CODES, SCALES, GS, 4, 64, NVF, 16, OUT, F32,
                                                       None),
        "fp4q_dequantize_unrotate": lambda: lib.fp4q_dequantize_unrotate(
            CODES, SCALES, GS, 4, 64, NVF, 16, 32, OUT, F32, None),
        "fp4q_block_mse": lambda: lib.fp4q_block_mse(X, CODES, SCALES, GS, 4, 64, NVF, 16, 0, MSE,
                                                     None),
        "fp4q_focus_fwd": lambda: lib.fp4q_focus_fwd(X, C, 4, 64, NVF, 16, 8, None, GS, OUT, F32,
                                                     None, None, None),
        "fp4q_focus_bwd": lambda: lib.fp4q_focus_bwd(X, G, C, 4, 64, 8, OUT, None),
        "fp4q_focus_update": lambda: lib.fp4q_focus_update(X, G, C, W, M, V, 4, 64, 8, ADAM, 1e-3,
                                                           0.9, 0.999, 1e-8, 1, None),
        "fp4q_focus_step": lambda: lib.fp4q_focus_step(X, 4, 64, NVF, 16, 8, None, GS, C, W, M, V,
                                                       MSE, ADAM, 1e-3, 0.9, 0.999, 1e-8, 1, None),
        "fp4q_gptq": lambda: lib.fp4q_gptq(X, 4, 128, NVF, 16, 16, SCALES, GS, U, None, OUT, CODES,
                                           None),
        "fp4q_global_amax": lambda: lib.fp4q_global_amax(X, 4, 64, 0, GS, None),
        "fp4q_e2m1_encode": lambda: lib.fp4q_e2m1_encode(X, 64, CODES, None),
        "fp4q_e4m3_encode": lambda: lib.fp4q_e4m3_encode(X, 64, CODES, None),
        "fp4q_scales_to_mma": lambda: lib.fp4q_scales_to_mma(SCALES, 4, 64, NVF, OUT, None),
        "fp4q_gemm": lambda: lib.fp4q_gemm(X, SCALES, GS, CODES, U, MSE, 128, 128, 64, NVF, M, OUT,
                                           F32, None),
        "fp4q_gemm_noalloc": lambda: lib.fp4q_gemm_noalloc(X, SCALES, GS, CODES, U, MSE, 128, 128,
                                                           64, NVF, OUT, F32, None),
    }
    # every entry point that can enqueue work is covered
    launching = set(declared_functions()) - {
        "fp4q_status_string", "fp4q_last_cuda_error", "fp4q_device_errors",
        "fp4q_mma_scale_bytes", "fp4q_debug_fail_launches"}
    assert set(calls) == launching
    code = 719  # cudaErrorLaunchFailure
    lib.fp4q_debug_fail_launches(code)
    try:
        for name, call in calls.items():
            lib.fp4q_debug_fail_launches(code + len(name))  # a distinct code per entry point
            assert call() == CUDA, name
            assert lib.fp4q_last_cuda_error() == code + len(name), name
        # validation still comes first
        assert lib.fp4q_quantize(None, 4, 64, NVF, 16, 0, 0, None, GS, CODES, SCALES, None, None,
                                 0, None) == NULL
    finally:
        lib.fp4q_debug_fail_launches(0)
    for b in bufs:
        assert (b == 0xA5).all()
