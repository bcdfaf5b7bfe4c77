"""Pins for the vocabulary-sharded oracle: each slice's statistics against
brute force, the merged statistics against the dense oracle (itself pinned in
test_oracle.py) and against scipy, and the slices' gradients reassembled
against the dense gradients.

  [p2] "分块交叉熵 / Output projection / exact cross entropy" (glenzli.com)
  [p5] AIInfraGuide ch.2 "数学基础" (maths basics)
"""
import math

import numpy as np
import pytest
import scipy.special

from oracle import flce_oracle as orc
from oracle import flce_shards as sh


def _case(seed=0, N=17, D=6, V=41, bias=True, ignore=3, mask_false=2):
    rng = np.random.default_rng(seed)
    H = rng.standard_normal((N, D))
    W = 0.8 * rng.standard_normal((V, D))
    b = 0.3 * rng.standard_normal(V) if bias else None
    y = rng.integers(0, V, N)
    y[rng.permutation(N)[:ignore]] = -100
    mask = np.ones(N, dtype=np.uint8)
    mask[rng.permutation(N)[:mask_false]] = 0
    return H, W, b, y, mask


def _bounds(V, sizes):
    assert sum(sizes) == V
    out, v0 = [], 0
    for s in sizes:
        out.append((v0, s))
        v0 += s
    return out


def _partials(H, W, b, y, mask, bounds, **kw):
    V = W.shape[0]
    return np.stack([sh.shard_partials(H, W[v0:v0 + n], None if b is None else b[v0:v0 + n],
                                       y, mask, v0=v0, V_total=V, **kw)
                     for v0, n in bounds])


PARTITIONS = {
    "one": [41],
    "even_ish": [11, 10, 10, 10],
    "uneven": [1, 5, 35],
    "columns": [1] * 41,
}


@pytest.mark.parametrize("name", list(PARTITIONS))
def test_partition_merge_equals_dense(name):
    """The two-state merge is exact in the reals for any partition of the
    columns ([p5] §9.4; [p2] §02): merged m, log s, per-row and mean loss equal
    the dense definition (to the rounding of the logits' dot products, which a
    library matmul may order differently on a slice)."""
    H, W, b, y, mask = _case(1)
    st = _partials(H, W, b, y, mask, _bounds(41, PARTITIONS[name]))
    got = sh.shard_combine(st, y, mask)
    ref = orc.forward(H, W, b, y, mask)
    idx = ref["idx"]
    assert np.max(np.abs(got["m"][idx] - ref["m"][idx])) < 1e-13
    assert np.max(np.abs(got["logs"][idx] - ref["logs"][idx])) < 1e-12
    assert np.all(np.isneginf(np.delete(got["logs"], idx)))
    assert np.all(np.isneginf(np.delete(got["m"], idx)))
    assert abs(got["loss"] - ref["loss"]) < 1e-12
    assert np.max(np.abs(got["loss_vec"] - ref["loss_vec"])) < 1e-12


def test_partials_pure_python_brute_force():
    """Each slice's (m_r, log s_r, t_r, o_r) from explicit dot products and
    math.exp/math.log, no vector library ([p2] §01-§02 on one slice)."""
    H, W, b, y, mask = _case(2, N=7, D=3, V=9, ignore=1, mask_false=1)
    for v0, n in _bounds(9, [4, 2, 3]):
        st = sh.shard_partials(H, W[v0:v0 + n], b[v0:v0 + n], y, mask, v0=v0, V_total=9)
        for i in range(7):
            if y[i] == -100 or mask[i] == 0:
                assert np.isneginf(st[i, 0]) and np.isneginf(st[i, 1])
                assert st[i, 2] == 0.0 and st[i, 3] == 0.0
                continue
            z = [sum(H[i, d] * W[v0 + j, d] for d in range(3)) + b[v0 + j] for j in range(n)]
            mx = max(z)
            ls = math.log(sum(math.exp(t - mx) for t in z))
            own = v0 <= y[i] < v0 + n
            assert st[i, 0] == pytest.approx(mx, abs=1e-13)
            assert st[i, 1] == pytest.approx(ls, abs=1e-13)
            assert st[i, 3] == (1.0 if own else 0.0)
            assert st[i, 2] == pytest.approx(z[y[i] - v0] if own else 0.0, abs=1e-13)


def test_merged_logsumexp_matches_scipy():
    """m + log s of the merge is the full-row logsumexp (scipy's routine)."""
    H, W, b, y, mask = _case(3, N=9, D=5, V=30, bias=False)
    st = _partials(H, W, None, y, mask, _bounds(30, [7, 13, 10]))
    got = sh.shard_combine(st, y, mask)
    idx, _ = orc.supervised_rows(y, mask)
    lse = scipy.special.logsumexp(H[idx] @ W.T, axis=1)
    assert np.max(np.abs(got["m"][idx] + got["logs"][idx] - lse)) < 1e-12


def test_slice_order_does_not_matter():
    H, W, b, y, mask = _case(4)
    st = _partials(H, W, b, y, mask, _bounds(41, [9, 9, 9, 14]))
    a = sh.shard_combine(st, y, mask)
    c = sh.shard_combine(st[::-1].copy(), y, mask)
    assert abs(a["loss"] - c["loss"]) < 1e-13
    idx = a["idx"]
    assert np.max(np.abs(a["logs"][idx] - c["logs"][idx])) < 1e-13


@pytest.mark.parametrize("kw", [
    dict(),
    dict(weight="w", reduction="sum", denom=23.0),
    dict(weight="w", reduction="none", grad_rows="g"),
    dict(logits_dtype="bf16"),
])
def test_slice_gradients_reassemble_dense(kw):
    """dW and db of the slices, stacked, are the dense dW and db; the slices'
    dH_r sum to the dense dH ([p2] §04: G's columns split over the slices)."""
    H, W, b, y, mask = _case(5, N=21, D=7, V=50)
    rng = np.random.default_rng(5)
    kw = dict(kw)
    if kw.get("weight") == "w":
        kw["weight"] = rng.uniform(0.0, 2.0, 21)
    if kw.get("grad_rows") == "g":
        kw["grad_rows"] = rng.standard_normal(21)
    lam = 0.6
    fwd_kw = {k: v for k, v in kw.items() if k in ("weight", "reduction", "denom")}
    bounds = _bounds(50, [13, 20, 17])
    st = _partials(H, W, b, y, mask, bounds, logits_dtype=kw.get("logits_dtype"))
    comb = sh.shard_combine(st, y, mask, **fwd_kw)
    ref = orc.forward_backward(H, W, b, y, mask, lam=lam, **kw)
    if comb["loss"] is not None:
        assert abs(comb["loss"] - ref["loss"]) < 1e-12
    assert np.max(np.abs(comb["loss_vec"] - ref["loss_vec"])) < 1e-12
    dH = np.zeros_like(H)
    dWs, dbs = [], []
    for v0, n in bounds:
        a, c, d = sh.shard_backward(H, W[v0:v0 + n], b[v0:v0 + n], y, mask, v0=v0, V_total=50,
                                    lam=lam, m=comb["m"], logs=comb["logs"], **kw)
        dH += a
        dWs.append(c)
        dbs.append(d)
    assert np.max(np.abs(dH - ref["dH"])) < 1e-12
    assert np.max(np.abs(np.concatenate(dWs) - ref["dW"])) < 1e-12
    assert np.max(np.abs(np.concatenate(dbs) - ref["db"])) < 1e-12


def test_one_slice_is_the_dense_oracle():
    """A single slice covering [0, V) is the unsharded method."""
    H, W, b, y, mask = _case(6)
    st = sh.shard_partials(H, W, b, y, mask)
    ref = orc.forward(H, W, b, y, mask)
    idx = ref["idx"]
    assert np.array_equal(st[idx, 0], ref["m"][idx])
    assert np.max(np.abs(st[idx, 1] - ref["logs"][idx])) < 1e-13
    assert np.all(st[idx, 3] == 1.0)
    dH, dW, db = sh.shard_backward(H, W, b, y, mask, lam=1.3, m=ref["m"], logs=ref["logs"])
    rb = orc.backward(H, W, b, y, mask, lam=1.3, m=ref["m"], logs=ref["logs"])
    for a, c in zip((dH, dW, db), rb):
        assert np.max(np.abs(a - c)) < 1e-13


def test_uncovered_or_doubly_held_labels_are_rejected():
    H, W, b, y, mask = _case(7)
    st = _partials(H, W, b, y, mask, _bounds(41, [20, 21]))
    with pytest.raises(ValueError):
        sh.shard_combine(st[:1], y, mask)                   # second slice missing
    with pytest.raises(ValueError):
        sh.shard_combine(np.concatenate([st, st[1:]]), y, mask)   # a slice twice
    with pytest.raises(ValueError):
        sh.shard_partials(H, W[:20], b[:20], y, mask, v0=30, V_total=41)  # slice past V
    y2 = y.copy()
    y2[0], mask[0] = 41, 1
    with pytest.raises(ValueError):
        sh.shard_partials(H, W[:20], b[:20], y2, mask, v0=0, V_total=41)


def test_no_supervised_rows():
    H, W, b, y, mask = _case(8)
    y[:] = -100
    st = _partials(H, W, b, y, mask, _bounds(41, [40, 1]))
    got = sh.shard_combine(st, y, mask)
    assert got["C"] == 0 and got["loss"] == 0.0
    assert np.all(np.isneginf(got["m"])) and np.all(got["loss_vec"] == 0.0)
    dH, dW, db = sh.shard_backward(H, W[:40], b[:40], y, mask, v0=0, V_total=41,
                                   m=got["m"], logs=got["logs"])
    assert not dH.any() and not dW.any() and not db.any()


def test_unrescaled_merge_would_be_caught():
    """Summing the slices' s_r without the exp(m_r - M) rescale (a plausible
    slip) moves log s by far more than the pins' tolerance on this case, so
    test_partition_merge_equals_dense would fail on it."""
    H, W, b, y, mask = _case(9)
    st = _partials(H, W, b, y, mask, _bounds(41, [11, 10, 10, 10]))
    good = sh.shard_combine(st, y, mask)
    idx = good["idx"]
    wrong = np.log(np.exp(st[:, idx, 1]).sum(axis=0))
    assert np.max(np.abs(wrong - good["logs"][idx])) > 1e-3
