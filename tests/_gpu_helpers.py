"""Shared helpers of the GPU tests: device copies of the seeded inputs and
the parity comparisons with the tolerances of the method's acceptance bar:

  loss          relative error <= 1e-4
  m, log s      relative error <= 1e-5   (|got - ref| <= 1e-5 * max(|ref|, 1))
  dH, dW, db    max |got - ref| <= 2e-3 * max |ref|
  idx, C        bit-exact

For log s the bound also admits the float32 floor of the logits it is
computed from: each logit is an fp32 sum of D exact products, whose error is
about u * sqrt(D) * max|partial sum| (u = 2^-24), and log s = LSE - m inherits
that error whatever its own size.  At D = 1024 the 1e-5 term governs; at
D = 4096 with logits near 20 (and for rows with logits in the hundreds) the
floor does.
"""
import numpy as np
import torch

from oracle import flce_oracle as orc

LOSS_RTOL = 1e-4
STAT_RTOL = 1e-5
GRAD_RTOL = 2e-3


def to_device(inp, dev="cuda"):
    tdt = torch.bfloat16 if inp.dtype == "bf16" else torch.float16
    H = torch.from_numpy(inp.H.view(np.int16)).view(tdt).to(dev)
    W = torch.from_numpy(inp.W.view(np.int16)).view(tdt).to(dev)
    b = None if inp.b is None else torch.from_numpy(inp.b.view(np.int16)).view(tdt).to(dev)
    y = torch.from_numpy(inp.labels).to(dev)
    mk = torch.from_numpy(inp.mask).to(dev)
    return H, W, b, y, mk


def rel_err(got, ref):
    return abs(got - ref) / max(abs(ref), 1e-30)


def check_loss(got, ref):
    assert abs(got - ref) <= LOSS_RTOL * max(abs(ref), 1.0), (got, ref)


U_F32 = 2.0 ** -24


def logs_floor(m_ref, D):
    """fp32 floor of log s for rows with max logit m_ref and depth D."""
    return U_F32 * np.sqrt(D) * np.maximum(np.abs(np.asarray(m_ref, dtype=np.float64)), 1.0)


def check_stats(got, ref, rows=None, floor=None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if rows is not None:
        got, ref = got[rows], ref[rows]
    err = np.abs(got - ref)
    tol = STAT_RTOL * np.maximum(np.abs(ref), 1.0)
    if floor is not None:
        tol = np.maximum(tol, floor)
    bad = np.flatnonzero(~(err <= tol))
    assert bad.size == 0, (bad[:5], got[bad[:5]], ref[bad[:5]])


def check_grad(name, got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert err <= GRAD_RTOL * scale, (name, err, scale)
    return err / scale if scale > 0 else 0.0


def sampled_check(inp, got, n_rows=64, n_cols=192, full_stats=True):
    rng = np.random.default_rng(0)
    idx, C = orc.supervised_rows(inp.labels, inp.mask)
    H64, W64, b64 = inp.H64(), inp.W64(), inp.b64()
    rows = np.sort(rng.choice(idx, size=min(n_rows, C), replace=False))
    r = orc.row_outputs(H64, W64, b64, inp.labels, inp.mask, -100, inp.lam, rows)
    check_stats(got["m"][rows], r["m"])
    check_stats(got["logs"][rows], r["logs"], floor=logs_floor(r["m"], inp.D))
    if full_stats:
        f = orc.forward(H64, W64, b64, inp.labels, inp.mask)
        check_loss(got["loss"], f["loss"])
        check_stats(got["m"], f["m"], idx)
        check_stats(got["logs"], f["logs"], idx, floor=logs_floor(f["m"][idx], inp.D))
        # vocabulary columns: the most frequent targets, the tail tile, random ids
        ys, counts = np.unique(inp.labels[idx], return_counts=True)
        hot = ys[np.argsort(-counts)[:32]]
        cols = np.unique(np.concatenate([hot, [0, inp.V - 1],
                                         rng.choice(inp.V, n_cols, replace=False)]))
        dW, db = orc.vocab_outputs(H64, W64, b64, inp.labels, inp.mask, -100, inp.lam,
                                   f["m"], f["logs"], cols)
        # tolerance scale: the largest dW / db entry, which sits in a hot target row
        check_grad("dW[cols]", got["dW"][cols], dW)
        if b64 is not None:
            check_grad("db[cols]", got["db"][cols], db)
    # dH rows: the tolerance scale is the largest |dH| among the sampled rows,
    # never above the largest over all rows, so this is at least as strict.
    check_grad("dH[rows]", got["dH"][rows], r["dH"])
    # a property of every size: sum_j p_ij = 1 gives sum_j dW_j = 0
    dWd = got["dW"].astype(np.float64)
    colsum = np.abs(dWd.sum(axis=0))
    assert np.all(colsum <= 1e-3 * np.abs(dWd).sum(axis=0) + 1e-30), colsum.max()
    unsup = np.setdiff1d(np.arange(inp.N), idx)
    assert not got["dH"][unsup].any()
    assert np.all(np.isneginf(got["m"][unsup]))
