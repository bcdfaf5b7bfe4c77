"""CPU binary64 oracle for the vocabulary-sharded form of exact fused linear
cross-entropy.

TEST INFRASTRUCTURE ONLY (the same rule as flce_oracle: imported by the tests,
the smoke check and the benchmark's CPU leg, never by the product path).

The vocabulary [0, V) is cut into disjoint slices [v0, v0 + V_r), one per
rank, each holding the rows W[v0 : v0 + V_r] of the projection (and of the
bias).  A rank can only form the logits of its own slice, so the loss needs
one exchange of per-row statistics; the pages describe the ingredients:

  * the two-state merge of online softmax ("数学基础" maths-basics page,
    §9.4 worked example; "分块交叉熵" §02): for a partition of the columns,
        M = max_r m_r,   S = sum_r s_r exp(m_r - M),   log S = log sum_r exp((m_r - M) + log s_r)
    and this is exact in the reals for any partition;
  * the target logit Z_{i,y_i} lives on exactly one slice (the one that holds
    y_i), so the loss is (M - Z_{i,y_i}) + log S (§02) after the merge;
  * the cross-device aggregation that a tensor-parallel vocabulary needs
    (maths-basics page, §5.9 remark on sharded vocabularies).

The backward needs no further exchange of statistics: with the merged m and
log s every slice forms its own columns of G (§04), so dW and db of the slice
are local and dH = sum_r G_r W_r is a sum over slices.

Per-row partial statistics are four numbers (m_r, log s_r, t_r, o_r): the
slice max, the log of the slice sum, the target logit when the slice holds the
label (else 0) and the ownership flag 1[v0 <= y_i < v0 + V_r].  Unsupervised
rows carry (-inf, -inf, 0, 0), the recurrence's initial state.
"""
from __future__ import annotations

import numpy as np
import torch

from .flce_oracle import (IGNORE_INDEX, REDUCTIONS, _denominator, _f64, _logits,
                          _row_weights, row_scales, supervised_rows)


def _check_global_labels(labels, idx, V_total):
    y = np.asarray(labels, dtype=np.int64)[idx]
    if y.size and (y.min() < 0 or y.max() >= V_total):
        raise ValueError("supervised label outside [0, V)")
    return y


def shard_partials(H, W_r, b_r, labels, mask=None, ignore_index: int = IGNORE_INDEX,
                   v0: int = 0, V_total=None, logits_dtype=None, row_block: int = 512):
    """Partial statistics [N, 4] = (m_r, log s_r, t_r, o_r) of the slice
    [v0, v0 + V_r) whose projection rows are W_r (and bias b_r).  V_total
    (default v0 + V_r) bounds the labels."""
    H, W_r, b_r = _f64(H), _f64(W_r), _f64(b_r)
    N, V_r = H.shape[0], W_r.shape[0]
    V_total = v0 + V_r if V_total is None else int(V_total)
    if v0 < 0 or v0 + V_r > V_total:
        raise ValueError("slice outside [0, V)")
    idx, C = supervised_rows(labels, mask, ignore_index)
    y = _check_global_labels(labels, idx, V_total)
    out = torch.zeros((N, 4), dtype=torch.float64)
    out[:, 0] = -np.inf
    out[:, 1] = -np.inf
    for r0 in range(0, C, row_block):
        r1 = min(C, r0 + row_block)
        rows = torch.as_tensor(idx[r0:r1])
        Z = _logits(H[rows], W_r, b_r, logits_dtype)      # this slice's columns only
        m = Z.max(dim=1).values
        logs = torch.log(torch.exp(Z - m[:, None]).sum(dim=1))
        yl = torch.as_tensor(y[r0:r1] - v0)
        own = (yl >= 0) & (yl < V_r)
        t = torch.zeros(r1 - r0, dtype=torch.float64)
        k = torch.nonzero(own).flatten()
        t[k] = Z[k, yl[k]]
        out[rows, 0], out[rows, 1], out[rows, 2] = m, logs, t
        out[rows, 3] = own.to(torch.float64)
    return out.numpy()


def shard_combine(stats, labels, mask=None, ignore_index: int = IGNORE_INDEX, weight=None,
                  reduction: str = "mean", denom=None):
    """Merge the partial statistics of all slices ([P, N, 4], any order) into
    the full-vocabulary m, log s and the loss.  Every supervised row must be
    owned by exactly one slice (ValueError otherwise).

    Returns dict(loss, loss_vec, m, logs, idx, C) as forward() does."""
    if reduction not in REDUCTIONS:
        raise ValueError(f"reduction must be one of {REDUCTIONS}")
    st = _f64(stats)
    if st.dim() != 3 or st.shape[2] != 4:
        raise ValueError("stats must be [P, N, 4]")
    N = st.shape[1]
    idx, C = supervised_rows(labels, mask, ignore_index)
    m = torch.full((N,), -np.inf, dtype=torch.float64)
    logs = torch.full((N,), -np.inf, dtype=torch.float64)
    rows = torch.as_tensor(idx)
    sr = st[:, rows, :]                                   # [P, C, 4]
    if C:
        owners = sr[:, :, 3].sum(dim=0)
        if not torch.all(owners == 1.0):
            raise ValueError("a supervised label is held by no slice or by several")
    M = sr[:, :, 0].max(dim=0).values
    logS = torch.log(torch.exp((sr[:, :, 0] - M[None, :]) + sr[:, :, 1]).sum(dim=0))
    tgt = (sr[:, :, 2] * sr[:, :, 3]).sum(dim=0)
    loss_rows = (M - tgt) + logS
    m[rows], logs[rows] = M, logS
    w = _row_weights(weight, idx)
    loss_vec = torch.zeros(N, dtype=torch.float64)
    loss_vec[rows] = w * loss_rows
    if reduction == "none":
        loss = None
    elif C == 0:
        loss = 0.0
    else:
        loss = float((w * loss_rows).sum() / _denominator(reduction, C, denom))
    return dict(loss=loss, loss_vec=loss_vec.numpy(), m=m.numpy(), logs=logs.numpy(), idx=idx,
                C=C, loss_rows=loss_rows.numpy())


def shard_backward(H, W_r, b_r, labels, mask=None, ignore_index: int = IGNORE_INDEX,
                   v0: int = 0, V_total=None, lam: float = 1.0, m=None, logs=None,
                   weight=None, reduction: str = "mean", denom=None, grad_rows=None,
                   logits_dtype=None, row_block: int = 512):
    """This slice's share of the gradients (§04): G_r = the columns
    [v0, v0 + V_r) of G, built from the merged full-vocabulary m and log s;
    returns (dH_r = G_r W_r, dW_r = G_r^T H, db_r = column sums of G_r, or
    None without bias).  The full dH is the sum of dH_r over the slices."""
    if m is None or logs is None:
        raise ValueError("the slice backward needs the merged m and log s")
    H, W_r, b_r = _f64(H), _f64(W_r), _f64(b_r)
    N, D, V_r = H.shape[0], H.shape[1], W_r.shape[0]
    V_total = v0 + V_r if V_total is None else int(V_total)
    if v0 < 0 or v0 + V_r > V_total:
        raise ValueError("slice outside [0, V)")
    idx, C = supervised_rows(labels, mask, ignore_index)
    y = _check_global_labels(labels, idx, V_total)
    dH = torch.zeros((N, D), dtype=torch.float64)
    dW = torch.zeros((V_r, D), dtype=torch.float64)
    db = torch.zeros(V_r, dtype=torch.float64) if b_r is not None else None
    if C == 0:
        return dH.numpy(), dW.numpy(), (None if db is None else db.numpy())
    m, logs = _f64(m), _f64(logs)
    scale = row_scales(labels, mask, ignore_index, lam, weight, reduction, denom, grad_rows)
    for r0 in range(0, C, row_block):
        r1 = min(C, r0 + row_block)
        rows = torch.as_tensor(idx[r0:r1])
        Hs = H[rows]
        Z = _logits(Hs, W_r, b_r, logits_dtype)
        P = torch.exp((Z - m[rows][:, None]) - logs[rows][:, None])
        yl = torch.as_tensor(y[r0:r1] - v0)
        k = torch.nonzero((yl >= 0) & (yl < V_r)).flatten()
        P[k, yl[k]] -= 1.0
        G = scale[r0:r1, None] * P
        dH[rows] = G @ W_r
        dW += G.T @ Hs
        if db is not None:
            db += G.sum(dim=0)
    return dH.numpy(), dW.numpy(), (None if db is None else db.numpy())
