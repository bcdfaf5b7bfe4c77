"""CPU oracle for the opt-in gradient filtering of the backward, in binary64.

TEST INFRASTRUCTURE ONLY (the same rule as flce_oracle.py: imported by the
tests, the smoke check and the benchmark's CPU leg, never by the product
path; it shares no code with the CUDA library).

The "分块交叉熵 / Output projection / exact cross entropy" page (§07, on
Apple's Cut Cross-Entropy) describes gradient filtering as an approximation:
blocks of the softmax whose probabilities are all negligible are skipped in
the backward contractions.  This module states that variant on top of the
exact gradient of §04:

    E_ij = p_ij - 1[j = y_i]        p_ij = exp((Z_ij - m_i) - log s_i)
    G_ij = (lambda / C) E_ij

A block is BR consecutive supervised rows (in ascending row order) by BC
consecutive vocabulary ids, aligned to multiples of BR and BC (128 x 64 by
default).  A block is dropped when every |E_ij| in it is below eps; dropped
blocks contribute nothing to dH = G W and dW = G^T H.  db = sum_i G_i keeps
every entry (it costs no contraction).  eps = 0 drops nothing and is the
exact backward.

Readings (the page names the idea, not these details): the test is on the
unscaled E (independent of lambda and C), strict "< eps" drops, padding
columns past V and padding rows past C count as zeros, and the block grid is
the one above.
"""
from __future__ import annotations

import numpy as np
import torch

from .flce_oracle import IGNORE_INDEX, _check_labels, _f64, forward, supervised_rows


def backward_filtered(H, W, b, labels, mask=None, ignore_index: int = IGNORE_INDEX,
                      lam: float = 1.0, m=None, logs=None, eps: float = 2.0 ** -12,
                      block_rows: int = 128, block_cols: int = 64):
    """dH [N, D], dW [V, D] with dropped blocks, exact db [V] (None without a
    bias), and keep [ceil(C / BR), ceil(V / BC)] (True = block kept)."""
    H, W, bt = _f64(H), _f64(W), _f64(b)
    N, D, V = H.shape[0], H.shape[1], W.shape[0]
    idx, C = supervised_rows(labels, mask, ignore_index)
    y = _check_labels(labels, idx, V)
    dH = torch.zeros((N, D), dtype=torch.float64)
    dW = torch.zeros((V, D), dtype=torch.float64)
    db = torch.zeros(V, dtype=torch.float64) if bt is not None else None
    ncb = -(-V // block_cols)
    keep = np.zeros((-(-C // block_rows), ncb), dtype=bool)
    if C == 0:
        return dict(dH=dH.numpy(), dW=dW.numpy(), db=None if db is None else db.numpy(),
                    keep=keep)
    if m is None or logs is None:
        st = forward(H.numpy(), W.numpy(), None if bt is None else bt.numpy(), labels, mask,
                     ignore_index)
        m, logs = st["m"], st["logs"]
    m, logs = _f64(m), _f64(logs)
    scale = lam / C
    for rb, r0 in enumerate(range(0, C, block_rows)):
        r1 = min(C, r0 + block_rows)
        rows = torch.as_tensor(idx[r0:r1])
        Hs = H[rows]
        Z = Hs @ W.T
        if bt is not None:
            Z = Z + bt
        E = torch.exp((Z - m[rows][:, None]) - logs[rows][:, None])
        E[torch.arange(r1 - r0), torch.as_tensor(y[r0:r1])] -= 1.0
        if db is not None:
            db += scale * E.sum(dim=0)
        # the largest |E| of each BC-column block of these rows
        Ep = torch.zeros((r1 - r0, ncb * block_cols), dtype=torch.float64)
        Ep[:, :V] = E.abs()
        bmax = Ep.reshape(r1 - r0, ncb, block_cols).amax(dim=(0, 2))
        kept = (bmax >= eps).numpy()
        keep[rb] = kept
        colmask = torch.as_tensor(np.repeat(kept, block_cols)[:V], dtype=torch.float64)
        G = scale * E * colmask[None, :]
        dH[rows] = G @ W
        dW += G.T @ Hs
    return dict(dH=dH.numpy(), dW=dW.numpy(), db=None if db is None else db.numpy(),
                keep=keep)
