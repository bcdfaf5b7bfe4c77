"""The stored tiny cases of tests/golden/tiny_cases.json (written by
tests/golden/make_golden.py from the oracle): pinned to closed forms and to
the oracle on CPU, and the CUDA path checked against them on the GPU."""
import json
import math
import os

import numpy as np
import pytest

from oracle import flce_oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))
CASES = json.load(open(os.path.join(HERE, "golden", "tiny_cases.json")))["cases"]
BY_NAME = {c["name"]: c for c in CASES}


def _arr(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def _stats(v):
    return np.array([-np.inf if t is None else t for t in v], dtype=np.float64)


def test_uniform_case_is_log_v():
    """W = 0, b = 0: L = log V, m = 0, log s = log V on every supervised row
    ("数学基础" §5.6, maximum entropy of the uniform distribution)."""
    c = BY_NAME["uniform"]
    V = len(c["W"])
    assert abs(c["loss"] - math.log(V)) < 1e-14
    assert np.all(_stats(c["m"]) == 0.0)
    assert np.max(np.abs(_stats(c["logs"]) - math.log(V))) < 1e-14
    assert not np.any(_arr(c["dH"]))


def test_binary_case_is_mean_softplus():
    """V = 2: each row's loss is softplus(z_other - z_target) ("数学基础" §5.5,
    the two-class cross entropy), computed here from explicit dot products."""
    c = BY_NAME["binary"]
    H, W, y = _arr(c["H"]), _arr(c["W"]), c["labels"]
    total = 0.0
    for i, yi in enumerate(y):
        z = [sum(H[i, d] * W[j, d] for d in range(H.shape[1])) for j in range(2)]
        t = z[1 - yi] - z[yi]
        total += max(t, 0.0) + math.log1p(math.exp(-abs(t)))
    assert abs(c["loss"] - total / len(y)) < 1e-13


def test_none_case_is_the_zero_sentinel():
    c = BY_NAME["none"]
    assert c["loss"] == 0.0
    assert all(v is None for v in c["m"])
    assert not np.any(_arr(c["dH"])) and not np.any(_arr(c["dW"]))


@pytest.mark.parametrize("name", list(BY_NAME))
def test_oracle_reproduces_the_stored_values(name):
    """The stored values are the oracle's: a later change to its arithmetic
    shows up here."""
    c = BY_NAME[name]
    r = orc.forward_backward(_arr(c["H"]), _arr(c["W"]), _arr(c["b"]), c["labels"],
                             np.asarray(c["mask"], np.uint8), lam=c["lam"])
    assert abs(r["loss"] - c["loss"]) <= 1e-13 * max(1.0, abs(c["loss"]))
    idx = r["idx"]
    assert np.max(np.abs(r["m"][idx] - _stats(c["m"])[idx]), initial=0.0) < 1e-13
    for k in ("dH", "dW"):
        assert np.max(np.abs(r[k] - _arr(c[k]))) < 1e-13
    if c["b"] is not None:
        assert np.max(np.abs(r["db"] - _arr(c["db"]))) < 1e-13


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(BY_NAME))
def test_cuda_path_matches_the_stored_values(name, cuda_device):
    import torch

    from lm_head_projection_supervised_b200 import binding, build
    build.build()
    c = BY_NAME[name]
    # the inputs are exact in bf16
    H = torch.tensor(c["H"], dtype=torch.float64).to(torch.bfloat16).cuda()
    W = torch.tensor(c["W"], dtype=torch.float64).to(torch.bfloat16).cuda()
    b = None if c["b"] is None else torch.tensor(c["b"], dtype=torch.float64).to(
        torch.bfloat16).cuda()
    assert torch.equal(H.double().cpu(), torch.tensor(c["H"], dtype=torch.float64))
    y = torch.tensor(c["labels"], dtype=torch.int64).cuda()
    mk = torch.tensor(c["mask"], dtype=torch.uint8).cuda()
    loss, m, logs = binding.forward(H, W, b, y, mk)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=c["lam"])
    assert abs(loss.item() - c["loss"]) <= 1e-4 * max(1.0, abs(c["loss"]))
    ms, ls = _stats(c["m"]), _stats(c["logs"])
    got_m, got_l = m.cpu().numpy().astype(np.float64), logs.cpu().numpy().astype(np.float64)
    sup = np.isfinite(ms)
    assert np.all(np.isneginf(got_m[~sup]))
    assert np.all(np.abs(got_m[sup] - ms[sup]) <= 1e-5 * np.maximum(np.abs(ms[sup]), 1.0))
    assert np.all(np.abs(got_l[sup] - ls[sup]) <= 1e-5 * np.maximum(np.abs(ls[sup]), 1.0))
    for got, ref in ((dH, c["dH"]), (dW, c["dW"]), (db, c["db"])):
        if ref is None:
            continue
        ref = _arr(ref)
        err = np.max(np.abs(got.cpu().numpy().astype(np.float64) - ref))
        assert err <= 2e-3 * max(np.max(np.abs(ref)), 1e-30), err
