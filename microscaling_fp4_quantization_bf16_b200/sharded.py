"""Row-sharded quantization over one process per GPU.

Every block (and rotation chunk) lies inside a row, so a tensor split by rows
across ranks quantizes independently on each rank; the one exchange is the
NVFP4 tensor abs-max behind the FP32 global scale ("Finer is Better (with the
Right Scaling)", 手法 2, hierarchical scaling): each rank takes the abs-max of
its rows with the library kernel, one all-reduce(MAX) of that single float
over the process group (NCCL on GPUs) gives the tensor's, and every rank then
quantizes its rows in one pass with it. MXFP4 and UE5M3 need no exchange.

torch.distributed is the plumbing here; the arithmetic stays in the CUDA
library (fp4q.global_amax and fp4q.quantize).
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist


def global_amax_sharded(x_local: torch.Tensor, rot: int = 0, group=None,
                        local_amax: Optional[Callable] = None) -> torch.Tensor:
    """Abs-max of the whole row-sharded tensor (after the blockwise rotation
    rot), as a float32 [1] tensor on x_local's device. local_amax defaults to
    the library's fp4q.global_amax."""
    if local_amax is None:
        from . import global_amax as local_amax
    a = local_amax(x_local, rot)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(a, op=dist.ReduceOp.MAX, group=group)
    return a


def quantize_sharded(x_local: torch.Tensor, fmt="nvfp4", block: int = 16, strategy="absmax",
                     rot: int = 0, group=None, **kwargs):
    """fp4q.quantize of this rank's rows with the tensor-wide NVFP4 global scale:
    equal, row for row, to quantizing the whole tensor on one GPU."""
    from . import quantize
    ga = global_amax_sharded(x_local, rot, group) if fmt == "nvfp4" else None
    return quantize(x_local, fmt, block, strategy, rot, global_amax=ga, **kwargs)
