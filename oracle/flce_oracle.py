"""CPU oracle for exact fused linear cross-entropy, in binary64.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check of the build
entry point and the CPU-baseline leg of the benchmark may import this module.
The product path (the CUDA library and its binding) never calls it, and this
module shares no code with the product path: it imports only torch (CPU,
float64) and numpy.

What it computes is the plain definition of the pages
("分块交叉熵 / Output projection / exact cross entropy", §01 equation):

    Z_ij = H_i W_j^T + b_j
    a_i  = 1[mask_i] 1[y_i != ignore],   C = sum_i a_i
    L    = (1/C) sum_{i: a_i = 1} ( log sum_j exp(Z_ij) - Z_{i,y_i} ),   C > 0

with the saved statistics of §02 (the per-row max m_i and log s_i, where
s_i = sum_j exp(Z_ij - m_i)), the loss written as (m_i - Z_{i,y_i}) + log s_i
(§02), the C = 0 convention of §01 (zero loss, zero gradients), and the
gradients of §04:

    p_ij = exp((Z_ij - m_i) - log s_i)
    G_ij = (lambda a_i / C) (p_ij - 1[j = y_i])
    dH = G W,   dW = G^T H,   db = sum_i G_i

``forward``/``backward`` take a DENSE full-vocabulary row of Z for each
supervised row (row blocks only bound the memory; every row sees all V
columns at once).  ``chunked`` follows the running-LSE recurrence of §02 and
the tile replay of §04 on the oracle's own (T, B) tiling; it exists to pin
the recurrence against the dense definition (§02: exact in the reals) and to
plant the two fault modes that §04 names, so that the tests can show they are
caught.

Readings where the pages are silent:
  * m and log s of a row with a_i = 0 are the recurrence's initial state:
    m = -inf, s = 0, so log s = -inf.
  * Z is not rounded to the input dtype; it is exact (float64 here).
  * bias absent means b = 0.
  * a label outside [0, V) on a supervised row is an error (ValueError here).

All arguments are numpy arrays (or anything torch.as_tensor accepts); float
inputs are upcast to float64 exactly.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

IGNORE_INDEX = -100


def _f64(x):
    if x is None:
        return None
    return torch.as_tensor(np.asarray(x), dtype=torch.float64)


def supervised_rows(labels, mask, ignore_index: int = IGNORE_INDEX):
    """a_i = 1[mask_i] 1[y_i != ignore] (§01); the supervised rows in
    ascending order and their count C.  mask None means all true."""
    labels = np.asarray(labels, dtype=np.int64)
    a = labels != ignore_index
    if mask is not None:
        a &= np.asarray(mask).astype(bool)
    idx = np.flatnonzero(a).astype(np.int64)
    return idx, int(idx.size)


def _check_labels(labels, idx, V):
    y = np.asarray(labels, dtype=np.int64)[idx]
    if y.size and (y.min() < 0 or y.max() >= V):
        raise ValueError("supervised label outside [0, V)")
    return y


LOGIT_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}


def _logits(Hs, W, b, logits_dtype=None):
    """Z = H W^T + b; with logits_dtype the logits are first rounded to
    float32 and then to the 16-bit model dtype (round to nearest even, torch's
    CPU casts), as a projection that outputs the model dtype does (NeMo
    ``logits_dtype``; the bf16 logits of "ChunkedLinearCrossEntropy")."""
    Z = Hs @ W.T
    if b is not None:
        Z = Z + b
    if logits_dtype is not None:
        Z = Z.to(torch.float32).to(LOGIT_DTYPES[logits_dtype]).to(torch.float64)
    return Z


def _rows_stats(Hs, W, b, y, logits_dtype=None):
    """Dense full-vocabulary statistics of a block of rows.

    Returns Z (rows x V), m, log s, the target logits and the per-row loss
    (m - Z_y) + log s (§02)."""
    Z = _logits(Hs, W, b, logits_dtype)
    m = Z.max(dim=1).values
    s = torch.exp(Z - m[:, None]).sum(dim=1)
    logs = torch.log(s)
    tgt = Z[torch.arange(Z.shape[0]), torch.as_tensor(y)]
    loss_rows = (m - tgt) + logs
    return Z, m, logs, tgt, loss_rows


REDUCTIONS = ("mean", "sum", "none")


def _row_weights(weight, idx):
    """w_i of the supervised rows (1 when no weights are given)."""
    if weight is None:
        return torch.ones(len(idx), dtype=torch.float64)
    return _f64(weight)[torch.as_tensor(idx)]


def _denominator(reduction, C, denom):
    """mean: C (p2 §01); sum: the caller's global count (NeMo num_label_tokens) or 1."""
    if reduction == "mean":
        return float(C)
    if reduction == "sum":
        return float(denom) if denom is not None and denom > 0 else 1.0
    return 1.0


def forward(H, W, b, labels, mask=None, ignore_index: int = IGNORE_INDEX,
            row_block: int = 512, weight=None, reduction: str = "mean", denom=None,
            logits_dtype=None):
    """Loss and saved statistics (§01, §02), dense in the vocabulary.

    reduction "mean" is the objective of p2 §01, (1/C) sum_i w_i l_i; "sum"
    is sum_i w_i l_i / denom and "none" the per-row w_i l_i (the NeMo
    ChunkedCrossEntropy reductions, num_label_tokens and loss_weights).  w_i = 1
    without weights.

    Returns dict(loss, loss_vec[N], m[N], logs[N], idx, C, loss_rows[C]);
    loss_vec holds w_i l_i on supervised rows and 0 elsewhere, loss is None for
    "none".  For C = 0 the loss is the zero sentinel of §01 and m = log s = -inf
    for every row."""
    if reduction not in REDUCTIONS:
        raise ValueError(f"reduction must be one of {REDUCTIONS}")
    H, W, b = _f64(H), _f64(W), _f64(b)
    N, V = H.shape[0], W.shape[0]
    idx, C = supervised_rows(labels, mask, ignore_index)
    y = _check_labels(labels, idx, V)
    m = torch.full((N,), -np.inf, dtype=torch.float64)
    logs = torch.full((N,), -np.inf, dtype=torch.float64)
    loss_rows = torch.zeros(C, dtype=torch.float64)
    for r0 in range(0, C, row_block):
        r1 = min(C, r0 + row_block)
        rows = torch.as_tensor(idx[r0:r1])
        _, mb, lb, _, lr = _rows_stats(H[rows], W, b, y[r0:r1], logits_dtype)
        m[rows], logs[rows], loss_rows[r0:r1] = mb, lb, lr
    w = _row_weights(weight, idx)
    loss_vec = torch.zeros(N, dtype=torch.float64)
    loss_vec[torch.as_tensor(idx)] = w * loss_rows
    if reduction == "none":
        loss = None
    elif C == 0:
        loss = 0.0
    else:
        loss = float((w * loss_rows).sum() / _denominator(reduction, C, denom))
    return dict(loss=loss, loss_vec=loss_vec.numpy(), m=m.numpy(), logs=logs.numpy(), idx=idx,
                C=C, loss_rows=loss_rows.numpy())


def row_scales(labels, mask, ignore_index, lam, weight=None, reduction="mean", denom=None,
               grad_rows=None):
    """s_i of G_ij = s_i (p_ij - 1[j = y_i]) for the supervised rows (§04 with
    lambda a_i / C generalised to the reductions): mean lambda w_i / C, sum
    lambda w_i / denom, none g_i w_i with g the per-row upstream gradient."""
    idx, C = supervised_rows(labels, mask, ignore_index)
    w = _row_weights(weight, idx)
    if reduction == "none":
        if grad_rows is None:
            raise ValueError("reduction 'none' needs grad_rows")
        return _f64(grad_rows)[torch.as_tensor(idx)] * w
    if C == 0:
        return torch.zeros(0, dtype=torch.float64)
    return (lam / _denominator(reduction, C, denom)) * w


def backward(H, W, b, labels, mask=None, ignore_index: int = IGNORE_INDEX,
             lam: float = 1.0, m=None, logs=None, row_block: int = 512, weight=None,
             reduction: str = "mean", denom=None, grad_rows=None, logits_dtype=None):
    """dH, dW, db from the reconstruction of §04, dense in the vocabulary.

    m and logs are the saved statistics (recomputed here when not given).
    db is None when b is None.  See row_scales for the reductions."""
    H, W, bt = _f64(H), _f64(W), _f64(b)
    N, D, V = H.shape[0], H.shape[1], W.shape[0]
    idx, C = supervised_rows(labels, mask, ignore_index)
    y = _check_labels(labels, idx, V)
    dH = torch.zeros((N, D), dtype=torch.float64)
    dW = torch.zeros((V, D), dtype=torch.float64)
    db = torch.zeros(V, dtype=torch.float64) if bt is not None else None
    if C == 0:
        return dH.numpy(), dW.numpy(), (None if db is None else db.numpy())
    if m is None or logs is None:
        st = forward(H.numpy(), W.numpy(), None if bt is None else bt.numpy(), labels, mask,
                     ignore_index, row_block, logits_dtype=logits_dtype)
        m, logs = st["m"], st["logs"]
    m, logs = _f64(m), _f64(logs)
    scale = row_scales(labels, mask, ignore_index, lam, weight, reduction, denom, grad_rows)
    for r0 in range(0, C, row_block):
        r1 = min(C, r0 + row_block)
        rows = torch.as_tensor(idx[r0:r1])
        Hs = H[rows]
        Z = _logits(Hs, W, bt, logits_dtype)  # the rounding passes the gradient through
        P = torch.exp((Z - m[rows][:, None]) - logs[rows][:, None])
        P[torch.arange(r1 - r0), torch.as_tensor(y[r0:r1])] -= 1.0
        G = scale[r0:r1, None] * P
        dH[rows] = G @ W
        dW += G.T @ Hs
        if db is not None:
            db += G.sum(dim=0)
    return dH.numpy(), dW.numpy(), (None if db is None else db.numpy())


def forward_backward(H, W, b, labels, mask=None, ignore_index: int = IGNORE_INDEX,
                     lam: float = 1.0, row_block: int = 512, weight=None,
                     reduction: str = "mean", denom=None, grad_rows=None, logits_dtype=None):
    f = forward(H, W, b, labels, mask, ignore_index, row_block, weight, reduction, denom,
                logits_dtype)
    dH, dW, db = backward(H, W, b, labels, mask, ignore_index, lam, f["m"], f["logs"],
                          row_block, weight, reduction, denom, grad_rows, logits_dtype)
    f.update(dH=dH, dW=dW, db=db)
    return f


# ---------------------------------------------------------------------------
# Sampled outputs for full-size comparisons
# ---------------------------------------------------------------------------

def row_outputs(H, W, b, labels, mask, ignore_index, lam, rows):
    """m, log s, per-row loss and dH of the given supervised rows (§02, §04).

    Each needs only that row's dense statistics and the global count C."""
    H, W, b = _f64(H), _f64(W), _f64(b)
    idx, C = supervised_rows(labels, mask, ignore_index)
    rows = np.asarray(rows, dtype=np.int64)
    y = _check_labels(labels, rows, W.shape[0])
    Z, m, logs, tgt, lr = _rows_stats(H[torch.as_tensor(rows)], W, b, y)
    P = torch.exp((Z - m[:, None]) - logs[:, None])
    P[torch.arange(len(rows)), torch.as_tensor(y)] -= 1.0
    dH = (lam / C) * (P @ W)
    return dict(m=m.numpy(), logs=logs.numpy(), loss_rows=lr.numpy(), dH=dH.numpy())


def vocab_outputs(H, W, b, labels, mask, ignore_index, lam, m, logs, cols,
                  row_block: int = 4096):
    """dW and db of the given vocabulary ids (§04), from the saved statistics
    m, log s of every supervised row (as computed by ``forward``)."""
    H, W, bt = _f64(H), _f64(W), _f64(b)
    idx, C = supervised_rows(labels, mask, ignore_index)
    y = _check_labels(labels, idx, W.shape[0])
    cols = np.asarray(cols, dtype=np.int64)
    ct = torch.as_tensor(cols)
    m, logs = _f64(m), _f64(logs)
    dW = torch.zeros((len(cols), H.shape[1]), dtype=torch.float64)
    db = torch.zeros(len(cols), dtype=torch.float64)
    for r0 in range(0, C, row_block):
        r1 = min(C, r0 + row_block)
        rows = torch.as_tensor(idx[r0:r1])
        Hs = H[rows]
        Z = Hs @ W[ct].T
        if bt is not None:
            Z = Z + bt[ct]
        P = torch.exp((Z - m[rows][:, None]) - logs[rows][:, None])
        P -= torch.as_tensor(y[r0:r1][:, None] == cols[None, :], dtype=torch.float64)
        G = (lam / C) * P
        dW += G.T @ Hs
        db += G.sum(dim=0)
    return dW.numpy(), (db.numpy() if bt is not None else None)


# ---------------------------------------------------------------------------
# The tiled recurrence of §02 / §04 on the oracle's own tiling
# ---------------------------------------------------------------------------

def chunked(H, W, b, labels, mask=None, ignore_index: int = IGNORE_INDEX, lam: float = 1.0,
            T: int = 16, B: int = 64, fault: Optional[str] = None):
    """Forward by the running (m, s) update over vocabulary blocks, target
    captured from the block that holds it; backward by replaying each T x B
    tile (§02, §04).  Tiles are visited rows-outer, vocabulary-inner.

    ``fault`` plants one of the two failure modes of §04 (for tests only):
      "local_norm"   -- each vocabulary block normalised on its own in the
                        backward, so every block carries probability mass 1;
      "dh_overwrite" -- dH of a row block written instead of accumulated
                        across vocabulary blocks.
    """
    H, W, bt = _f64(H), _f64(W), _f64(b)
    N, D, V = H.shape[0], H.shape[1], W.shape[0]
    labels = np.asarray(labels, dtype=np.int64)
    idx, C = supervised_rows(labels, mask, ignore_index)
    a = np.zeros(N, dtype=bool)
    a[idx] = True
    m_all = torch.full((N,), -np.inf, dtype=torch.float64)
    logs_all = torch.full((N,), -np.inf, dtype=torch.float64)
    dH = torch.zeros((N, D), dtype=torch.float64)
    dW = torch.zeros((V, D), dtype=torch.float64)
    db = torch.zeros(V, dtype=torch.float64) if bt is not None else None
    loss_sum = 0.0
    for t0 in range(0, N, T):
        t1 = min(N, t0 + T)
        rows = torch.arange(t0, t1)
        act = torch.as_tensor(a[t0:t1])
        y = labels[t0:t1]
        Ht = H[t0:t1]
        m = torch.full((t1 - t0,), -np.inf, dtype=torch.float64)
        s = torch.zeros(t1 - t0, dtype=torch.float64)
        tgt = torch.zeros(t1 - t0, dtype=torch.float64)
        for v0 in range(0, V, B):
            v1 = min(V, v0 + B)
            Zb = Ht @ W[v0:v1].T
            if bt is not None:
                Zb = Zb + bt[v0:v1]
            m_new = torch.maximum(m, Zb.max(dim=1).values)
            # scale factor of the running sum; defined as 0 on the first block
            factor = torch.where(torch.isinf(m), torch.zeros_like(m), torch.exp(m - m_new))
            s = factor * s + torch.exp(Zb - m_new[:, None]).sum(dim=1)
            m = m_new
            for r in range(t1 - t0):
                if act[r] and v0 <= y[r] < v1:
                    tgt[r] = Zb[r, y[r] - v0]      # local id = global id - block start
        logs = torch.log(s)
        m_all[t0:t1] = torch.where(act, m, m_all[t0:t1])
        logs_all[t0:t1] = torch.where(act, logs, logs_all[t0:t1])
        if act.any():
            loss_sum += float(((m - tgt) + logs)[act].sum())
        if C == 0:
            continue
        for v0 in range(0, V, B):
            v1 = min(V, v0 + B)
            Zb = Ht @ W[v0:v1].T
            if bt is not None:
                Zb = Zb + bt[v0:v1]
            if fault == "local_norm":
                mb = Zb.max(dim=1).values
                e = torch.exp(Zb - mb[:, None])
                P = e / e.sum(dim=1, keepdim=True)
            else:
                P = torch.exp((Zb - m[:, None]) - logs[:, None])
            for r in range(t1 - t0):
                if v0 <= y[r] < v1:
                    P[r, y[r] - v0] -= 1.0
            G = (lam / C) * P * act[:, None].to(torch.float64)
            if fault == "dh_overwrite":
                dH[t0:t1] = G @ W[v0:v1]
            else:
                dH[t0:t1] += G @ W[v0:v1]
            dW[v0:v1] += G.T @ Ht
            if db is not None:
                db[v0:v1] += G.sum(dim=0)
    loss = loss_sum / C if C > 0 else 0.0
    return dict(loss=loss, m=m_all.numpy(), logs=logs_all.numpy(), idx=idx, C=C,
                dH=dH.numpy(), dW=dW.numpy(), db=(None if db is None else db.numpy()))


def objective(H, W, b, labels, mask=None, ignore_index: int = IGNORE_INDEX) -> float:
    """L of §01 as a plain function of H, W, b (for finite differences)."""
    return forward(H, W, b, labels, mask, ignore_index)["loss"]
