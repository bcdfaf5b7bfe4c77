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
