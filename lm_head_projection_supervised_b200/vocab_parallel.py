"""Vocabulary-parallel (tensor-parallel over V) fused linear cross-entropy.

Each rank of a process group holds one slice [v0, v0 + V_r) of the
vocabulary: rows v0 .. v0 + V_r - 1 of the projection W (and of the bias).
One step is five calls, two of them collectives:

  1. slice forward (CUDA)  per-row partial statistics (m_r, log s_r, t_r, o_r)
  2. all-gather            every rank gets all slices' statistics [P, N, 4]
  3. combine (CUDA)        full-vocabulary m, log s and the loss: the two-state
                           online-softmax merge ("数学基础" maths-basics page,
                           worked example 9.4; "分块交叉熵" §02)
  4. slice backward (CUDA) dW and db of the slice, and the slice's term of dH
  5. all-reduce (sum)      dH = sum over slices

The cross-device aggregation that a sharded vocabulary needs is the remark of
the maths-basics page, §5.9.  Every compute step runs in libflce.so through the
binding; this module only cuts the vocabulary and moves the statistics and dH
between ranks with torch.distributed (NCCL on GPUs).  The exchange is 16 P N
bytes forward (the statistics) and 4 N D bytes backward (dH); W never moves.

`ops` is the object that provides the three compute steps (default: the CUDA
binding).  Passing another one is how the host logic is exercised on CPU
ranks, without a GPU.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import binding


def vocab_slice(V: int, P: int, r: int, align: int = 256) -> Tuple[int, int]:
    """(v0, V_r) of rank r when V vocabulary ids are cut into P slices.

    Slice boundaries fall on multiples of `align` ids (the kernels' vocabulary
    tile) when V >= align * P, so that only the last slice has a ragged tile;
    else on multiples of 8 ids (16 bytes of a 16-bit bias, so that a bias
    slice stays on the TMA's 16-byte grid) when V >= 8 * P; else the plain
    balanced cut.  Slices are contiguous, disjoint, cover [0, V) in rank
    order and are never empty."""
    if P < 1 or not 0 <= r < P:
        raise ValueError("need 0 <= r < P")
    if V < P:
        raise ValueError("fewer vocabulary ids than slices")
    for a in (align, 8, 1):
        if V >= a * P:
            break
    units = V // a
    v0 = (r * units // P) * a
    v1 = V if r == P - 1 else ((r + 1) * units // P) * a
    return v0, v1 - v0


def _group_size_rank(group):
    return dist.get_world_size(group), dist.get_rank(group)


def gather_stats(stats: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of the [N, 4] per-row statistics into [P, N, 4], rank order."""
    P, _ = _group_size_rank(group)
    parts = [torch.empty_like(stats) for _ in range(P)]
    dist.all_gather(parts, stats.contiguous(), group=group)
    return torch.stack(parts)


def forward(H, W_slice, b_slice, labels, mask=None, ignore_index: int = -100, *, V_total: int,
            v0: int, group=None, weight=None, reduction: str = "mean",
            denom: Optional[float] = None, round_logits: bool = False, ops=binding):
    """(loss, m, logs) over the full vocabulary; the same on every rank."""
    stats = ops.shard_forward(H, W_slice, b_slice, labels, mask, ignore_index, v0=v0,
                              V_total=V_total, round_logits=round_logits)
    allstats = gather_stats(stats, group)
    return ops.shard_combine(allstats, labels, mask, ignore_index, weight=weight,
                             reduction=reduction, denom=denom)


def backward(H, W_slice, b_slice, labels, mask, ignore_index: int, m, logs, *, V_total: int,
             v0: int, group=None, lam: float = 1.0, lam_dev=None, weight=None,
             reduction: str = "mean", denom: Optional[float] = None, grad_rows=None,
             round_logits: bool = False, ops=binding):
    """(dH, dW_slice, db_slice): dH summed over the group (all-reduce), the
    slice's dW and db local."""
    dH, dW, db = ops.shard_backward(H, W_slice, b_slice, labels, mask, ignore_index, m, logs,
                                    v0=v0, V_total=V_total, lam=lam, lam_dev=lam_dev,
                                    weight=weight, reduction=reduction, denom=denom,
                                    grad_rows=grad_rows, round_logits=round_logits)
    dist.all_reduce(dH, op=dist.ReduceOp.SUM, group=group)
    return dH, dW, db


class VocabParallelLinearCrossEntropy(torch.autograd.Function):
    """Autograd form: inputs H (replicated), this rank's W and b slices."""

    @staticmethod
    def forward(ctx, H, W_slice, b_slice, labels, mask, ignore_index, V_total, v0, group,
                weight=None, reduction="mean", denom=None, round_logits=False, ops=binding):
        loss, m, logs = forward(H, W_slice, b_slice, labels, mask, ignore_index,
                                V_total=V_total, v0=v0, group=group, weight=weight,
                                reduction=reduction, denom=denom, round_logits=round_logits,
                                ops=ops)
        ctx.save_for_backward(H, W_slice, b_slice, labels, mask, weight, m, logs)
        ctx.cfg = (ignore_index, V_total, v0, group, reduction, denom, round_logits, ops)
        return loss

    @staticmethod
    def backward(ctx, grad_out):
        H, W_slice, b_slice, labels, mask, weight, m, logs = ctx.saved_tensors
        ignore_index, V_total, v0, group, reduction, denom, round_logits, ops = ctx.cfg
        kw = dict(V_total=V_total, v0=v0, group=group, weight=weight, reduction=reduction,
                  denom=denom, round_logits=round_logits, ops=ops)
        if reduction == "none":
            kw["grad_rows"] = grad_out.reshape(-1)
        else:
            kw["lam_dev"] = grad_out
        dH, dW, db = backward(H, W_slice, b_slice, labels, mask, ignore_index, m, logs, **kw)
        return (dH.reshape(H.shape).to(H.dtype), dW.to(W_slice.dtype),
                None if db is None else db.to(b_slice.dtype),
                None, None, None, None, None, None, None, None, None, None, None)


def vocab_parallel_cross_entropy(H, W_slice, labels, *, V_total: int, v0: int, group=None,
                                 b_slice=None, mask=None, ignore_index: int = -100, weight=None,
                                 reduction: str = "mean", denom: Optional[float] = None,
                                 round_logits: bool = False, ops=binding):
    """Loss of the full vocabulary from this rank's slice, differentiable in
    H, W_slice and b_slice.  H: [N, D] (or [..., D]) replicated on the group."""
    D = H.shape[-1]
    loss = VocabParallelLinearCrossEntropy.apply(
        H.reshape(-1, D), W_slice, b_slice, labels.reshape(-1),
        None if mask is None else mask.reshape(-1), ignore_index, V_total, v0, group,
        None if weight is None else weight.reshape(-1), reduction, denom, round_logits, ops)
    return loss.reshape(labels.shape) if reduction == "none" else loss


def run_slices_on_one_device(H, W, b, labels, mask=None, ignore_index: int = -100, P: int = 2,
                             lam: float = 1.0, weight=None, reduction: str = "mean",
                             denom: Optional[float] = None, grad_rows=None,
                             round_logits: bool = False, ws=None, out=None):
    """All P slices' calls on one device, one after the other: the same kernels
    and data as a P-rank step, with the two exchanges done in place (each
    slice writes its statistics into its row of one [P, N, 4] buffer, and adds
    its dH term into one dH with FLCE_FLAG_ACCUMULATE_DH).

    Returns dict(loss, m, logs, dH, dW, db); each slice writes its rows of dW
    and db directly.  ws, when given, is one workspace large enough for the
    widest slice, shared by all calls; out = (stats, dH, dW, db) preallocated
    outputs (db None without bias)."""
    N, D = H.reshape(-1, H.shape[-1]).shape
    V = W.shape[0]
    bounds = [vocab_slice(V, P, r) for r in range(P)]
    if out is None:
        f32 = dict(dtype=torch.float32, device=H.device)
        out = (torch.empty((P, N, 4), **f32), torch.zeros((N, D), **f32),
               torch.empty((V, D), **f32), None if b is None else torch.empty(V, **f32))
    stats, dH, dW, db = out
    for r, (v0, n) in enumerate(bounds):
        binding.shard_forward(H, W[v0:v0 + n], None if b is None else b[v0:v0 + n], labels, mask,
                              ignore_index, v0=v0, V_total=V, ws=ws, round_logits=round_logits,
                              out=stats[r])
    loss, m, logs = binding.shard_combine(stats, labels, mask, ignore_index, weight=weight,
                                          reduction=reduction, denom=denom)
    for r, (v0, n) in enumerate(bounds):
        binding.shard_backward(H, W[v0:v0 + n], None if b is None else b[v0:v0 + n], labels,
                               mask, ignore_index, m, logs, v0=v0, V_total=V, lam=lam,
                               weight=weight, reduction=reduction, denom=denom,
                               grad_rows=grad_rows, round_logits=round_logits, ws=ws,
                               out=(dH, dW[v0:v0 + n], None if db is None else db[v0:v0 + n]),
                               accumulate_dh=r > 0)
    return dict(loss=loss, m=m, logs=logs, dH=dH, dW=dW, db=db)
