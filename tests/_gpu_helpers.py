"""Shared helpers of the GPU tests: device copies of the seeded inputs and
the parity comparisons with the tolerances of the method's acceptance bar:

  loss          relative error <= 1e-4
  m, log s      relative error <= 1e-5   (|got - ref| <= 1e-5 * max(|ref|, 1))
  dH, dW, db    max |got - ref| <= 2e-3 * max |ref|
  idx, C        bit-exact

For log s the bound also admits the float32 floor of the logits it is
computed from, on the rows where that floor can exceed the flat bar: each
logit is an fp32 sum of D exact products, whose error is about
u * sqrt(D) * max|partial sum| (u = 2^-24), and log s = LSE - m inherits that
error whatever its own size.  The floor is applied only where it can matter:
depth D >= 4096, or rows whose largest logit has |m| >= 64.  Everywhere else
log s must meet the flat 1e-5 bar.

Every check records its largest error and its bar (and, for log s, the ratio
against the flat bar and how many rows needed the floor).  With the
environment variable FLCE_PARITY_REPORT set to a path, each record is
appended to that file as one JSON line, so that a run of the GPU suite leaves
the error budget of every configuration behind.
"""
import json
import os

import numpy as np
import torch

from oracle import flce_oracle as orc

LOSS_RTOL = 1e-4
STAT_RTOL = 1e-5
GRAD_RTOL = 2e-3
U_F32 = 2.0 ** -24
FLOOR_MIN_D = 4096      # depth from which every row may use the fp32 floor
FLOOR_MIN_ABS_M = 64.0  # rows with a larger |max logit| may use it at any depth

REPORT = []


def _case():
    cur = os.environ.get("PYTEST_CURRENT_TEST", "")
    return cur.split(" ")[0].split("::", 1)[-1] if cur else "?"


def record(quantity, max_err, bar, case=None, **extra):
    """Keeps one error-budget record (and appends it to FLCE_PARITY_REPORT)."""
    bar = float(bar)
    err = float(max_err)
    rec = dict(case=case or _case(), quantity=quantity, max_err=err, bar=bar,
               ratio=(err / bar) if bar > 0 else (0.0 if err == 0 else float("inf")))
    rec.update(extra)
    REPORT.append(rec)
    path = os.environ.get("FLCE_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")
    return rec


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


def check_loss(got, ref, quantity="loss", case=None):
    err = abs(got - ref)
    bar = LOSS_RTOL * max(abs(ref), 1.0)
    record(quantity, err, bar, case)
    assert err <= bar, (got, ref)


def logs_floor(m_ref, D):
    """fp32 floor of log s per row (max logit m_ref, depth D); zero on the
    rows where the flat bar applies (D < 4096 and |m| < 64)."""
    am = np.abs(np.asarray(m_ref, dtype=np.float64))
    fl = U_F32 * np.sqrt(D) * np.maximum(am, 1.0)
    if D >= FLOOR_MIN_D:
        return fl
    return np.where(am >= FLOOR_MIN_ABS_M, fl, 0.0)


def check_stats(got, ref, rows=None, floor=None, quantity="stat", case=None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if rows is not None:
        got, ref = got[rows], ref[rows]
    err = np.abs(got - ref)
    flat = STAT_RTOL * np.maximum(np.abs(ref), 1.0)
    tol = flat if floor is None else np.maximum(flat, floor)
    if err.size:
        worst = int(np.argmax(err / tol))
        rf = err / flat
        record(quantity, err[worst], tol[worst], case, rows=int(err.size),
               ratio_flat=float(np.max(rf)), rows_over_flat=int(np.count_nonzero(rf > 1.0)),
               governing=("flat" if tol[worst] == flat[worst] else "fp32 floor"))
    bad = np.flatnonzero(~(err <= tol))
    assert bad.size == 0, (bad[:5], got[bad[:5]], ref[bad[:5]])


def check_grad(name, got, ref, case=None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    record(name, err, GRAD_RTOL * scale, case)
    assert err <= GRAD_RTOL * scale, (name, err, scale)
    return err / scale if scale > 0 else 0.0


def sampled_check(inp, got, n_rows=64, n_cols=192, full_stats=True, extra_rows=None):
    """Full-size comparison on what the oracle can compute piecewise: m, log s
    and dH of sampled rows (plus `extra_rows`, checked again on their own),
    and with full_stats the loss, m and log s of every supervised row and dW /
    db of the hottest labels, the first and last ids and random ids."""
    rng = np.random.default_rng(0)
    idx, C = orc.supervised_rows(inp.labels, inp.mask)
    H64, W64, b64 = inp.H64(), inp.W64(), inp.b64()
    rows = np.sort(rng.choice(idx, size=min(n_rows, C), replace=False))
    if extra_rows is not None and len(extra_rows):
        rows = np.union1d(rows, np.asarray(extra_rows, dtype=np.int64))
    r = orc.row_outputs(H64, W64, b64, inp.labels, inp.mask, -100, inp.lam, rows)
    check_stats(got["m"][rows], r["m"], quantity="m[sampled rows]")
    check_stats(got["logs"][rows], r["logs"], floor=logs_floor(r["m"], inp.D),
                quantity="logs[sampled rows]")
    if extra_rows is not None and len(extra_rows):
        sel = np.isin(rows, extra_rows)
        check_stats(got["m"][rows[sel]], r["m"][sel], quantity="m[extra rows]")
        check_stats(got["logs"][rows[sel]], r["logs"][sel],
                    floor=logs_floor(r["m"][sel], inp.D), quantity="logs[extra rows]")
        check_grad("dH[extra rows]", got["dH"][rows[sel]], r["dH"][sel])
    if full_stats:
        f = orc.forward(H64, W64, b64, inp.labels, inp.mask)
        check_loss(got["loss"], f["loss"])
        check_stats(got["m"], f["m"], idx, quantity="m[all rows]")
        check_stats(got["logs"], f["logs"], idx, floor=logs_floor(f["m"][idx], inp.D),
                    quantity="logs[all rows]")
        # vocabulary columns: the most frequent targets, the tail tile, random ids
        ys, counts = np.unique(inp.labels[idx], return_counts=True)
        hot = ys[np.argsort(-counts)[:32]]
        cols = np.unique(np.concatenate([hot, [0, inp.V - 1],
                                         np.arange(max(0, inp.V - 8), inp.V),
                                         rng.choice(inp.V, n_cols, replace=False)]))
        dW, db = orc.vocab_outputs(H64, W64, b64, inp.labels, inp.mask, -100, inp.lam,
                                   f["m"], f["logs"], cols)
        # tolerance scale: the largest dW / db entry, which sits in a hot target row
        check_grad("dW[cols]", got["dW"][cols], dW)
        if b64 is not None:
            check_grad("db[cols]", got["db"][cols], db)
    # dH rows: the tolerance scale is the largest |dH| among the sampled rows,
    # never above the largest over all rows, so this is at least as strict.
    check_grad("dH[sampled rows]", got["dH"][rows], r["dH"])
    # a property of every size: sum_j p_ij = 1 gives sum_j dW_j = 0
    dWd = got["dW"].astype(np.float64)
    colsum = np.abs(dWd.sum(axis=0))
    assert np.all(colsum <= 1e-3 * np.abs(dWd).sum(axis=0) + 1e-30), colsum.max()
    del dWd
    unsup = np.setdiff1d(np.arange(inp.N), idx)
    assert not got["dH"][unsup].any()
    assert np.all(np.isneginf(got["m"][unsup]))
