"""Pins of the gradient-filtering oracle (oracle/flce_filtered.py) against
what the mathematics fixes: no filtering is the exact backward, total
filtering leaves only db, a pure-Python brute force of the block rule, rows
whose blocks are dropped or kept by construction, and the error bound that
dropping entries below eps implies."""
import itertools
import math

import numpy as np
import pytest

from lm_head_projection_supervised_b200 import workloads as wl
from oracle import flce_filtered as ofl
from oracle import flce_oracle as orc


def _case(seed=3, N=40, D=12, V=300, bias=True):
    return wl.random_case(seed=seed, N=N, D=D, V=V, bias=bias, w_std=0.3)


def test_eps_zero_is_the_exact_backward():
    inp = _case()
    args = (inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask)
    ex = orc.forward_backward(*args, lam=0.7)
    f = ofl.backward_filtered(*args, lam=0.7, eps=0.0, block_rows=8, block_cols=32)
    assert f["keep"].all()
    for k in ("dH", "dW", "db"):
        np.testing.assert_allclose(f[k], ex[k], rtol=0, atol=1e-13)


def test_eps_above_one_drops_every_block_but_keeps_db():
    inp = _case(seed=4)
    args = (inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask)
    ex = orc.forward_backward(*args, lam=1.3)
    f = ofl.backward_filtered(*args, lam=1.3, eps=1.0 + 1e-9)  # |p - onehot| <= 1 always
    assert not f["keep"].any()
    assert not f["dH"].any() and not f["dW"].any()
    np.testing.assert_allclose(f["db"], ex["db"], rtol=0, atol=1e-14)


def test_brute_force_block_rule():
    """Every entry and every block decided by explicit loops."""
    inp = _case(seed=5, N=17, D=5, V=41)
    H, W, b = inp.H64(), inp.W64(), inp.b64()
    y, mk = inp.labels, inp.mask
    BR, BC, eps, lam = 3, 7, 0.05, 0.9
    f = ofl.backward_filtered(H, W, b, y, mk, lam=lam, eps=eps, block_rows=BR, block_cols=BC)
    idx = [i for i in range(len(y)) if y[i] != -100 and mk[i]]
    C, V, D = len(idx), W.shape[0], W.shape[1]
    E = []
    for i in idx:
        z = [sum(H[i, d] * W[j, d] for d in range(D)) + b[j] for j in range(V)]
        mx = max(z)
        s = sum(math.exp(t - mx) for t in z)
        E.append([math.exp(z[j] - mx) / s - (1.0 if j == y[i] else 0.0) for j in range(V)])
    keep = {}
    for rb, cb in itertools.product(range(-(-C // BR)), range(-(-V // BC))):
        vals = [abs(E[r][c]) for r in range(rb * BR, min(C, rb * BR + BR))
                for c in range(cb * BC, min(V, cb * BC + BC))]
        keep[rb, cb] = max(vals) >= eps
        assert f["keep"][rb, cb] == keep[rb, cb]
    assert 0 < sum(keep.values()) < len(keep)  # the case exercises both outcomes
    dW = np.zeros((V, D))
    dH = np.zeros((len(y), D))
    db = np.zeros(V)
    for r, i in enumerate(idx):
        for j in range(V):
            g = lam / C * E[r][j]
            db[j] += g
            if keep[r // BR, j // BC]:
                dW[j] += g * H[i]
                dH[i] += g * W[j]
    np.testing.assert_allclose(f["dW"], dW, rtol=0, atol=1e-12)
    np.testing.assert_allclose(f["dH"], dH, rtol=0, atol=1e-12)
    np.testing.assert_allclose(f["db"], db, rtol=0, atol=1e-12)


def test_blocks_dropped_and_kept_by_construction():
    """W = I (D = V): rows with H = 0 have p = 1/V everywhere (every block
    kept), rows with H = 40 e_y put all mass on the label (|E| < 1e-15, every
    block dropped).  The result is then the exact backward of the kept rows
    alone, with the full row count in lambda / C."""
    V = D = 48
    W = np.eye(V)
    y = np.array([3, 9, 17, 40, 5, 5, 30, 47], dtype=np.int64)
    H = np.zeros((8, D))
    for i in range(4, 8):
        H[i, y[i]] = 40.0
    f = ofl.backward_filtered(H, W, None, y, None, lam=1.0, eps=1e-6, block_rows=4,
                              block_cols=16)
    assert f["keep"][0].all() and not f["keep"][1].any()
    sub = orc.forward_backward(H[:4], W, None, y[:4], None, lam=4.0 / 8.0)
    np.testing.assert_allclose(f["dW"], sub["dW"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(f["dH"][:4], sub["dH"], rtol=0, atol=1e-14)
    assert not f["dH"][4:].any()


@pytest.mark.parametrize("seed,eps", [(6, 5e-3), (7, 1e-2), (8, 5e-2)])
def test_error_is_bounded_by_the_dropped_entries(seed, eps):
    """Dropped entries are below eps, so |dW_f - dW| <= eps (lam/C) sum_i |H_i|
    and |dH_f - dH| <= eps (lam/C) sum_j |W_j| element-wise."""
    inp = _case(seed=seed, N=60, D=10, V=500)
    H, W, b = inp.H64(), inp.W64(), inp.b64()
    ex = orc.forward_backward(H, W, b, inp.labels, inp.mask, lam=1.0)
    f = ofl.backward_filtered(H, W, b, inp.labels, inp.mask, lam=1.0, eps=eps, block_rows=8,
                              block_cols=16)
    idx, C = orc.supervised_rows(inp.labels, inp.mask)
    assert 0 < f["keep"].sum() < f["keep"].size
    bw = eps / C * np.abs(H[idx]).sum(axis=0)
    assert np.all(np.abs(f["dW"] - ex["dW"]) <= bw[None, :] + 1e-15)
    bh = eps / C * np.abs(W).sum(axis=0)
    assert np.all(np.abs(f["dH"] - ex["dH"]) <= bh[None, :] + 1e-15)
