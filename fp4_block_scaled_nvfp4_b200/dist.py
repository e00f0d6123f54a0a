"""Quantizing one tensor whose rows are sharded across processes (one per GPU).

Blocks never straddle rows, so every rank quantizes its own rows; the only coupling is the
per-tensor scale S = max|x| / (256*6) (ScaleSweep, gist.science/ko/paper/2606.07618,
Methodology).  Rounding to nearest is monotone, so the largest per-rank
S_r = RN(amax_r / 1536) equals RN(max_r amax_r / 1536), the S of the whole tensor: one
4-byte all-reduce-MAX of S_r gives every rank exactly the scale a single-GPU call would
compute, and the quantized rows are then identical to that call's.  The same holds for IF6's
S = RN(amax / 1920).

A non-finite element makes a rank's S_r NaN; NaN is carried through the MAX as +inf (a
finite tensor cannot produce an infinite S) and turned back into NaN, so every rank's
quantize call reports FP4Q_DEVSTAT_NONFINITE and zero-fills, as the single call would.
"""
from __future__ import annotations


def reduce_global_scale(s_local, group=None):
    """All-reduce-MAX of per-rank tensor scales ([1] float32 tensor, any device the process
    group's backend supports); returns a new tensor holding the whole tensor's S."""
    import torch
    import torch.distributed as dist

    t = torch.nan_to_num(s_local.to(torch.float32), nan=float("inf"), posinf=float("inf")).clone()
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return torch.where(torch.isinf(t), torch.full_like(t, float("nan")), t)


def sharded_quantize(x_local, fmt: str = "nvfp4", objective: str = "sweep_mse", importance=None, group=None,
                     workspace=None, out=None, hadamard16: bool = False):
    """Quantize this rank's rows of a row-sharded tensor with the whole tensor's S.

    Two kernels and one collective per call: the local amax pass (fp4q_global_scale,
    fp4q_hadamard_global_scale for the 16-point rotated blocks, fp4q_if6_global_scale for IF6),
    the 4-byte all-reduce-MAX, then fp4q_quantize with FP4Q_F_GLOBAL_SCALE_GIVEN.  MXFP4 has no
    tensor scale and needs no collective.  Returns (codes, scales, S)."""
    from . import global_scale, new_workspace, quantize

    ws = workspace if workspace is not None else new_workspace(x_local.device)
    if fmt == "mxfp4":
        return quantize(x_local, fmt, objective, out=out, workspace=ws)
    s_all = reduce_global_scale(global_scale(x_local, workspace=ws, hadamard16=hadamard16, fmt=fmt), group)
    return quantize(x_local, fmt, objective, importance=importance, global_scale=s_all, out=out, workspace=ws,
                    hadamard16=hadamard16)


def max_over_ranks(value: float, device="cpu", group=None) -> float:
    """The largest of a per-rank float (timings are reported as the slowest rank's)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
