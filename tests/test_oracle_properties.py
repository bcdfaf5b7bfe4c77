"""Property-based pins of the oracle (hypothesis): over random small shapes,
tilings and vocabulary partitions, the identities the pages state hold.

  [p2] "分块交叉熵 / Output projection / exact cross entropy"
  [p5] AIInfraGuide ch. 2 "数学基础" (maths basics)
"""
import numpy as np
import scipy.special
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import flce_oracle as orc
from oracle import flce_shards as sh

# derandomize: the same examples on every run, so that the suite's outcome does
# not depend on the run (a failing example would fail every time)
SETTINGS = dict(max_examples=25, deadline=None, derandomize=True,
                suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])


@st.composite
def problems(draw):
    N = draw(st.integers(1, 12))
    D = draw(st.integers(1, 6))
    V = draw(st.integers(2, 40))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    H = rng.standard_normal((N, D)) * draw(st.sampled_from([0.1, 1.0, 4.0]))
    W = rng.standard_normal((V, D)) * draw(st.sampled_from([0.1, 0.5, 2.0]))
    b = rng.standard_normal(V) * 0.3 if draw(st.booleans()) else None
    y = rng.integers(0, V, N)
    y[rng.random(N) < draw(st.sampled_from([0.0, 0.3, 1.0]))] = -100
    mask = (rng.random(N) > draw(st.sampled_from([0.0, 0.2]))).astype(np.uint8)
    return H, W, b, y, mask


@settings(**SETTINGS)
@given(problems(), st.integers(1, 7), st.integers(1, 45))
def test_tiled_recurrence_equals_dense(prob, T, B):
    """[p2] §02: the running (m, s) update over any tiling reaches the dense
    statistics (exact in the reals)."""
    H, W, b, y, mask = prob
    d = orc.forward_backward(H, W, b, y, mask, lam=0.9)
    c = orc.chunked(H, W, b, y, mask, lam=0.9, T=T, B=B)
    assert abs(c["loss"] - d["loss"]) <= 1e-12 * max(1.0, abs(d["loss"]))
    for k in ("dH", "dW"):
        assert np.max(np.abs(c[k] - d[k]), initial=0.0) <= 1e-12 * max(1.0, np.max(np.abs(d[k])))


@settings(**SETTINGS)
@given(problems())
def test_statistics_are_the_logsumexp(prob):
    """m + log s is scipy's logsumexp of each supervised row ([p5] §5.3)."""
    H, W, b, y, mask = prob
    f = orc.forward(H, W, b, y, mask)
    idx = f["idx"]
    if idx.size == 0:
        assert f["loss"] == 0.0
        return
    Z = H[idx] @ W.T + (0.0 if b is None else b)
    lse = scipy.special.logsumexp(Z, axis=1)
    assert np.max(np.abs(f["m"][idx] + f["logs"][idx] - lse)) <= 1e-12 * max(1.0, np.max(np.abs(lse)))


@settings(**SETTINGS)
@given(problems(), st.data())
def test_any_vocabulary_partition_merges_to_dense(prob, data):
    """[p5] §9.4 / [p2] §02: the slices' statistics of any partition of the
    vocabulary merge to the dense loss, and the slices' gradients reassemble the
    dense ones ([p2] §04)."""
    H, W, b, y, mask = prob
    V = W.shape[0]
    cuts = sorted(set(data.draw(st.lists(st.integers(1, V - 1), max_size=5))))
    bounds = list(zip([0] + cuts, cuts + [V]))
    stats = np.stack([sh.shard_partials(H, W[a:e], None if b is None else b[a:e], y, mask,
                                        v0=a, V_total=V) for a, e in bounds])
    comb = sh.shard_combine(stats, y, mask)
    d = orc.forward_backward(H, W, b, y, mask, lam=1.1)
    assert abs(comb["loss"] - d["loss"]) <= 1e-12 * max(1.0, abs(d["loss"]))
    dH = np.zeros_like(H)
    for a, e in bounds:
        h, w, c = sh.shard_backward(H, W[a:e], None if b is None else b[a:e], y, mask, v0=a,
                                    V_total=V, lam=1.1, m=comb["m"], logs=comb["logs"])
        dH += h
        assert np.max(np.abs(w - d["dW"][a:e]), initial=0.0) <= 1e-12 * max(
            1.0, np.max(np.abs(d["dW"])))
        if b is not None:
            assert np.max(np.abs(c - d["db"][a:e]), initial=0.0) <= 1e-12
    assert np.max(np.abs(dH - d["dH"]), initial=0.0) <= 1e-12 * max(1.0, np.max(np.abs(d["dH"])))


@settings(**SETTINGS)
@given(problems())
def test_gradient_rows_sum_to_zero(prob):
    """sum_j p_ij = 1 ([p5] §5.2), so each supervised row of G sums to 0: db
    sums to 0 and so does every column of dW (sum_j dW_j = sum_i (sum_j G_ij) H_i)."""
    H, W, b, y, mask = prob
    d = orc.forward_backward(H, W, b, y, mask, lam=1.0)
    if b is not None:
        assert abs(np.sum(d["db"])) <= 1e-13 * max(1.0, np.max(np.abs(d["db"])) * W.shape[0])
    assert np.max(np.abs(d["dW"].sum(axis=0)), initial=0.0) <= 1e-12 * max(
        1.0, np.max(np.abs(d["dW"])) * W.shape[0])


@settings(**SETTINGS)
@given(problems(), st.integers(0, 2**31 - 1))
def test_reductions_are_consistent(prob, seed):
    """The NeMo-style reductions of the same per-row losses agree with one
    another: sum over 'none' rows = 'sum'; 'mean' = 'sum' with denom = C; and
    the gradients scale the same way (per-row upstream gradients of 1/C give
    the mean's gradients)."""
    H, W, b, y, mask = prob
    rng = np.random.default_rng(seed)
    w = rng.uniform(0.0, 2.0, H.shape[0])
    none = orc.forward_backward(H, W, b, y, mask, weight=w, reduction="none",
                                grad_rows=np.ones(H.shape[0]))
    summ = orc.forward_backward(H, W, b, y, mask, weight=w, reduction="sum", lam=1.0)
    C = none["C"]
    assert abs(np.sum(none["loss_vec"]) - summ["loss"]) <= 1e-12 * max(1.0, abs(summ["loss"]))
    for k in ("dH", "dW"):
        assert np.max(np.abs(none[k] - summ[k]), initial=0.0) <= 1e-12 * max(
            1.0, np.max(np.abs(summ[k]), initial=0.0))
    if C:
        mean = orc.forward_backward(H, W, b, y, mask, weight=w, reduction="mean", lam=1.0)
        den = orc.forward_backward(H, W, b, y, mask, weight=w, reduction="sum", denom=float(C),
                                   lam=1.0)
        assert abs(mean["loss"] - den["loss"]) <= 1e-13 * max(1.0, abs(mean["loss"]))
        g = orc.forward_backward(H, W, b, y, mask, weight=w, reduction="none",
                                 grad_rows=np.full(H.shape[0], 1.0 / C))
        assert np.max(np.abs(g["dW"] - mean["dW"]), initial=0.0) <= 1e-12 * max(
            1.0, np.max(np.abs(mean["dW"]), initial=0.0))
