"""fp4q_gemm_noalloc against fp4q_gemm: the same GEMM with alpha in the
library's scratch float instead of a caller-owned one, so the outputs must be
identical bit for bit. Two calls in a row with different operands (and global
scales), so the second call cannot pass on the first call's alpha."""
import numpy as np
import pytest
import torch

from microscaling_fp4_quantization_bf16_b200 import synth

pytestmark = pytest.mark.gpu


def operands(gpu, fmt, block, M, N, K, seed):
    a = (synth.laplace_outliers(M, K, seed=seed) * (1.0 + seed)).cuda()
    w = synth.gaussian(N, K, seed=seed + 1, std=0.02 * (seed + 1)).cuda()
    qa = gpu.quantize_mma(a, fmt, "absmax", 0)
    qw = gpu.quantize_mma(w, fmt, "absmax", 0)
    return qa, qw


@pytest.mark.parametrize("fmt,block", [("nvfp4", 16), ("mxfp4", 32)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_noalloc_matches_gemm_twice(gpu, fmt, block, out_dtype):
    for seed, (M, N, K) in ((1, (256, 384, 512)), (2, (200, 136, 1024))):
        qa, qw = operands(gpu, fmt, block, M, N, K, seed)
        want = gpu.gemm(qa.codes, qa.scales, qa.global_scale, qw.codes, qw.scales, qw.global_scale,
                        fmt, out_dtype)
        got = gpu.gemm_noalloc(qa.codes, qa.scales, qa.global_scale, qw.codes, qw.scales,
                               qw.global_scale, fmt, out_dtype=out_dtype)
        torch.cuda.synchronize()
        g = got.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32).cpu().numpy()
        w = want.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32).cpu().numpy()
        assert np.array_equal(g, w), f"call with seed {seed}: {np.sum(g != w)} outputs differ"
