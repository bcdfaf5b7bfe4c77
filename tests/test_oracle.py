"""Pins for the CPU oracle, each checked against something other than itself.

Citations name the page and section of the method's sources:
  [p2] "分块交叉熵 / Output projection / exact cross entropy" (glenzli.com)
  [p5] AIInfraGuide ch.2 "数学基础" (maths basics)
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

from oracle import flce_oracle as orc
from lm_head_projection_supervised_b200 import workloads as wl


def _case(seed=0, N=13, D=5, V=37, bias=True, ignore=3, mask_false=2, wstd=0.7):
    rng = np.random.default_rng(seed)
    H = rng.standard_normal((N, D))
    W = wstd * rng.standard_normal((V, D))
    b = 0.3 * rng.standard_normal(V) if bias else None
    y = rng.integers(0, V, N)
    y[rng.permutation(N)[:ignore]] = -100
    mask = np.ones(N, dtype=np.uint8)
    mask[rng.permutation(N)[:mask_false]] = 0
    return H, W, b, y, mask


def _close(a, b, tol=1e-11):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    return float(np.max(np.abs(a - b))) <= tol * scale if a.size else True


# --- closed forms ----------------------------------------------------------

def test_uniform_scores_give_log_v():
    """W = 0, b = 0: every row is uniform, so L = log V (max entropy, [p5] §5.6),
    m = 0, log s = log V, dH = 0, and the gradients have closed forms
    ([p2] §04 with p_ij = 1/V)."""
    H, W, b, y, mask = _case(1, N=11, D=4, V=29)
    W[:] = 0.0
    b = np.zeros(29)
    lam = 0.75
    f = orc.forward_backward(H, W, b, y, mask, lam=lam)
    idx, C = orc.supervised_rows(y, mask)
    assert C > 0
    assert abs(f["loss"] - math.log(29)) < 1e-13
    assert np.all(f["m"][idx] == 0.0)
    assert np.allclose(f["logs"][idx], math.log(29), rtol=0, atol=1e-14)
    assert np.all(f["dH"] == 0.0)
    dW = np.zeros((29, 4))
    db = np.zeros(29)
    for i in idx:
        for j in range(29):
            g = (lam / C) * (1.0 / 29 - (1.0 if y[i] == j else 0.0))
            dW[j] += g * H[i]
            db[j] += g
    assert _close(f["dW"], dW) and _close(f["db"], db)
    # sum_j p_ij = 1  <=>  sum_j db_j = 0
    assert abs(f["db"].sum()) < 1e-14


def test_bias_only_matches_logsumexp():
    """W = 0: l_i = LSE(b) - b_{y_i}; LSE from scipy ([p5] §5.3)."""
    H, W, b, y, mask = _case(2, V=41)
    W[:] = 0.0
    f = orc.forward(H, W, b, y, mask)
    idx, C = orc.supervised_rows(y, mask)
    lse = scipy.special.logsumexp(b)
    want = np.mean([lse - b[y[i]] for i in idx])
    assert abs(f["loss"] - want) < 1e-13
    assert np.allclose(f["m"][idx] + f["logs"][idx], lse, rtol=0, atol=1e-13)


def test_confident_row_has_zero_loss():
    """p_y = 1 gives a zero loss ([p5] §5.5)."""
    H = np.zeros((1, 3))
    W = np.zeros((5, 3))
    b = np.zeros(5)
    b[2] = 1000.0
    f = orc.forward(H, W, b, np.array([2]), None)
    assert f["loss"] == 0.0 and f["m"][0] == 1000.0 and f["logs"][0] == 0.0


def test_large_common_shift_is_stable():
    """Scores near 1e3 would overflow a naive exp; the (m - target) + log s form
    stays finite and equals scipy's logsumexp ([p2] §02, [p5] §5.2)."""
    H, W, b, y, mask = _case(3)
    H[0] *= 2000.0
    f = orc.forward(H, W, b, y, None)
    Z = H @ W.T + b
    assert np.max(np.abs(Z)) > 700
    idx, C = orc.supervised_rows(y, None)
    want = np.mean([scipy.special.logsumexp(Z[i]) - Z[i, y[i]] for i in idx])
    assert np.isfinite(f["loss"]) and abs(f["loss"] - want) < 1e-10 * abs(want)


def test_shift_invariance():
    """b -> b + c leaves L and all gradients unchanged and shifts m by c
    ([p5] §5.1: softmax(z + c) = softmax(z))."""
    H, W, b, y, mask = _case(4)
    f0 = orc.forward_backward(H, W, b, y, mask)
    f1 = orc.forward_backward(H, W, b + 17.25, y, mask)
    idx, _ = orc.supervised_rows(y, mask)
    assert abs(f0["loss"] - f1["loss"]) < 1e-12
    assert np.allclose(f1["m"][idx] - f0["m"][idx], 17.25, rtol=0, atol=1e-12)
    for k in ("dH", "dW", "db"):
        assert _close(f0[k], f1[k], 1e-10)


# --- independent implementations --------------------------------------------

def test_pure_python_brute_force():
    """Loops with math.exp / math.log on a 5x3x7 case ([p2] §01, §04)."""
    H, W, b, y, mask = _case(5, N=5, D=3, V=7, ignore=1, mask_false=1)
    lam = -0.5
    f = orc.forward_backward(H, W, b, y, mask, lam=lam)
    N, D, V = 5, 3, 7
    rows = [i for i in range(N) if mask[i] and y[i] != -100]
    C = len(rows)
    Z = [[sum(H[i][d] * W[j][d] for d in range(D)) + b[j] for j in range(V)] for i in range(N)]
    L = 0.0
    dH = [[0.0] * D for _ in range(N)]
    dW = [[0.0] * D for _ in range(V)]
    db = [0.0] * V
    for i in rows:
        lse = math.log(sum(math.exp(z) for z in Z[i]))
        L += lse - Z[i][y[i]]
        for j in range(V):
            g = lam / C * (math.exp(Z[i][j] - lse) - (1.0 if j == y[i] else 0.0))
            db[j] += g
            for d in range(D):
                dH[i][d] += g * W[j][d]
                dW[j][d] += g * H[i][d]
    assert abs(f["loss"] - L / C) < 1e-13
    assert _close(f["dH"], dH) and _close(f["dW"], dW) and _close(f["db"], db)


def test_matches_torch_cross_entropy_autograd():
    """Textbook special case: torch's float64 cross_entropy with autograd on
    the dense logits, mask folded into the ignored labels ([p5] §6.8)."""
    H, W, b, y, mask = _case(6, N=40, D=9, V=123)
    lam = 1.7
    f = orc.forward_backward(H, W, b, y, mask, lam=lam)
    Ht = torch.tensor(H, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    yy = torch.tensor(np.where(mask.astype(bool), y, -100))
    L = torch.nn.functional.cross_entropy(Ht @ Wt.T + bt, yy, ignore_index=-100)
    (lam * L).backward()
    assert abs(f["loss"] - L.item()) < 1e-12
    assert _close(f["dH"], Ht.grad.numpy()) and _close(f["dW"], Wt.grad.numpy())
    assert _close(f["db"], bt.grad.numpy())


def test_central_finite_differences():
    """Central differences of the full objective on H, W and b
    ([p5] §6.9; [p2] §06 asks for this check on H/W/b)."""
    H, W, b, y, mask = _case(7, N=6, D=3, V=9, ignore=1, mask_false=1)
    f = orc.forward_backward(H, W, b, y, mask, lam=1.0)
    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, X, G in (("H", H, f["dH"]), ("W", W, f["dW"]), ("b", b, f["db"])):
        for flat in rng.choice(X.size, size=min(X.size, 12), replace=False):
            ix = np.unravel_index(flat, X.shape)
            Xp, Xm = X.copy(), X.copy()
            Xp[ix] += eps
            Xm[ix] -= eps
            args_p = dict(H=H, W=W, b=b)
            args_m = dict(H=H, W=W, b=b)
            args_p[name], args_m[name] = Xp, Xm
            fd = (orc.objective(args_p["H"], args_p["W"], args_p["b"], y, mask)
                  - orc.objective(args_m["H"], args_m["W"], args_m["b"], y, mask)) / (2 * eps)
            assert abs(fd - G[ix]) < 1e-8, (name, ix, fd, G[ix])


# --- the recurrence, C = 0, lambda ------------------------------------------

@pytest.mark.parametrize("T,B", [(1, 1), (4, 7), (5, 16), (13, 37), (64, 64), (3, 1000)])
def test_chunked_equals_dense(T, B):
    """The running (m, s) update and the tile replay reach the dense result
    ([p2] §02: identical in the reals; §03 allows T >= N, B >= V)."""
    H, W, b, y, mask = _case(8, N=13, D=5, V=37)
    d = orc.forward_backward(H, W, b, y, mask, lam=0.9)
    c = orc.chunked(H, W, b, y, mask, lam=0.9, T=T, B=B)
    idx, _ = orc.supervised_rows(y, mask)
    assert abs(c["loss"] - d["loss"]) < 1e-12
    assert _close(c["m"][idx], d["m"][idx]) and _close(c["logs"][idx], d["logs"][idx])
    for k in ("dH", "dW", "db"):
        assert _close(c[k], d[k], 1e-11), k


def test_zero_supervised_rows():
    """C = 0: zero sentinel loss and zero gradients ([p2] §01)."""
    H, W, b, y, mask = _case(9)
    y[:] = -100
    f = orc.forward_backward(H, W, b, y, mask, lam=3.0)
    assert f["C"] == 0 and f["loss"] == 0.0
    assert np.all(np.isneginf(f["m"])) and np.all(np.isneginf(f["logs"]))
    assert not f["dH"].any() and not f["dW"].any() and not f["db"].any()
    c = orc.chunked(H, W, b, y, mask, T=4, B=8)
    assert c["loss"] == 0.0 and not c["dW"].any()


def test_mask_false_rows_are_unsupervised():
    H, W, b, y, mask = _case(10)
    mask[:] = 0
    f = orc.forward_backward(H, W, b, y, mask)
    assert f["C"] == 0 and not f["dH"].any()


@pytest.mark.parametrize("lam", [0.0, -1.3, 2.5])
def test_lambda_scales_gradients_only(lam):
    """lambda = dJ/dL scales the gradients and leaves L unchanged ([p2] §04;
    §06 asks for positive, negative and zero upstream gradients)."""
    H, W, b, y, mask = _case(11)
    f1 = orc.forward_backward(H, W, b, y, mask, lam=1.0)
    fl = orc.forward_backward(H, W, b, y, mask, lam=lam)
    assert fl["loss"] == f1["loss"]
    for k in ("dH", "dW", "db"):
        assert _close(fl[k], lam * f1[k], 1e-12)
    if lam == 0.0:
        assert not fl["dH"].any() and not fl["dW"].any()


def test_no_bias_means_zero_bias():
    H, W, b, y, mask = _case(12)
    f0 = orc.forward_backward(H, W, None, y, mask)
    fz = orc.forward_backward(H, W, np.zeros_like(b), y, mask)
    assert f0["db"] is None and f0["loss"] == fz["loss"] and _close(f0["dW"], fz["dW"], 0)


def test_target_in_every_vocab_block():
    """The target captured from whichever block holds it ([p2] §02, §06)."""
    N, V, B = 10, 50, 7
    H, W, b, y, mask = _case(13, N=N, V=V, ignore=0, mask_false=0)
    y[:] = np.arange(N) * B % V  # targets spread over every block, incl. the tail block
    y[-1] = V - 1
    d = orc.forward_backward(H, W, b, y, mask)
    c = orc.chunked(H, W, b, y, mask, T=3, B=B)
    assert abs(c["loss"] - d["loss"]) < 1e-12 and _close(c["dW"], d["dW"])


def test_out_of_range_label_is_rejected():
    H, W, b, y, mask = _case(14)
    y[0] = 37
    mask[0] = 1
    with pytest.raises(ValueError):
        orc.forward(H, W, b, y, mask)


# --- planted faults must be caught ------------------------------------------

def test_local_normalisation_fault_is_caught():
    """Per-block softmax makes each block's mass 1: the forward is still right,
    the gradients are not ([p2] §04, first fault mode)."""
    H, W, b, y, mask = _case(15, N=13, D=5, V=37)
    d = orc.forward_backward(H, W, b, y, mask)
    B = 8
    c = orc.chunked(H, W, b, y, mask, T=4, B=B, fault="local_norm")
    assert abs(c["loss"] - d["loss"]) < 1e-12
    for k in ("dH", "dW", "db"):
        assert not _close(c[k], d[k], 1e-3), k
    # sum_j G_ij = (lambda / C) (#blocks - 1) instead of 0
    idx, C = orc.supervised_rows(y, mask)
    nblocks = -(-37 // B)
    assert abs(c["db"].sum() - (nblocks - 1)) < 1e-9


def test_dh_overwrite_fault_is_caught():
    """Writing dH per vocabulary block keeps only the last block: dH is
    wrong, dW and db are not ([p2] §04, second fault mode)."""
    H, W, b, y, mask = _case(16, N=13, D=5, V=37)
    d = orc.forward_backward(H, W, b, y, mask)
    c = orc.chunked(H, W, b, y, mask, T=4, B=8, fault="dh_overwrite")
    assert not _close(c["dH"], d["dH"], 1e-3)
    assert _close(c["dW"], d["dW"]) and _close(c["db"], d["db"])


# --- sampled outputs used for full-size comparisons ----------------------------

def test_sampled_outputs_equal_full():
    H, W, b, y, mask = _case(17, N=30, D=6, V=55)
    lam = 0.6
    f = orc.forward_backward(H, W, b, y, mask, lam=lam)
    idx, _ = orc.supervised_rows(y, mask)
    rows = idx[::3]
    r = orc.row_outputs(H, W, b, y, mask, -100, lam, rows)
    assert _close(r["m"], f["m"][rows]) and _close(r["logs"], f["logs"][rows])
    assert _close(r["dH"], f["dH"][rows])
    assert abs(np.mean(orc.row_outputs(H, W, b, y, mask, -100, lam, idx)["loss_rows"])
               - f["loss"]) < 1e-13
    cols = np.array([0, 5, int(y[idx[0]]), 54])
    dW, db = orc.vocab_outputs(H, W, b, y, mask, -100, lam, f["m"], f["logs"], cols,
                               row_block=7)
    assert _close(dW, f["dW"][cols]) and _close(db, f["db"][cols])


# --- the seeded workloads (shared input generator) ----------------------------

def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 1.0 + 2**-8 + 2**-20],
                 dtype=np.float32)
    bits = wl.f32_to_bf16_bits(x)
    assert list(bits) == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x3F81]
    assert np.all(wl.bf16_bits_to_f32(bits)[[0, 3]] == x[[0, 3]])


@pytest.mark.parametrize("name,C", [("tiny", 48), ("small", 1228)])
def test_workload_supervised_counts(name, C):
    inp = wl.make_inputs(name)
    assert orc.supervised_rows(inp.labels, inp.mask)[1] == C


def test_packed_layout_counts():
    """8 documents of 2048 tokens, first 614 of each ignored: C = 11472."""
    spec = wl.SPECS["packed"]
    import dataclasses
    inp = wl.make_inputs(dataclasses.replace(spec, V=1024, D=8))
    assert orc.supervised_rows(inp.labels, inp.mask)[1] == 11472
    assert np.all(inp.labels[:614] == -100) and inp.labels[614] >= 0


# --- reductions, per-row weights and per-row upstream gradients ---------------
# (NeMo ChunkedCrossEntropy: reduction 'sum'/'none', num_label_tokens,
#  loss_weights; the page's objective is the 'mean' case)

def _torch_rows(H, W, b, y, mask):
    """Per-row CE of the dense logits from torch (0 for unsupervised rows)."""
    Ht = torch.tensor(H, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    yy = torch.tensor(np.where(mask.astype(bool), y, -100))
    rows = torch.nn.functional.cross_entropy(Ht @ Wt.T + bt, yy, ignore_index=-100,
                                             reduction="none")
    return Ht, Wt, bt, rows


def test_reduction_none_matches_torch_per_row():
    H, W, b, y, mask = _case(18, N=33, D=7, V=90)
    w = np.random.default_rng(1).uniform(0.2, 2.0, 33)
    f = orc.forward(H, W, b, y, mask, weight=w, reduction="none")
    _, _, _, rows = _torch_rows(H, W, b, y, mask)
    assert f["loss"] is None
    assert _close(f["loss_vec"], w * rows.detach().numpy(), 1e-12)


@pytest.mark.parametrize("denom", [None, 37.0])
def test_weighted_sum_matches_torch_autograd(denom):
    H, W, b, y, mask = _case(19, N=30, D=6, V=70)
    w = np.random.default_rng(2).uniform(0.0, 3.0, 30)
    lam = 0.8
    f = orc.forward_backward(H, W, b, y, mask, lam=lam, weight=w, reduction="sum", denom=denom)
    Ht, Wt, bt, rows = _torch_rows(H, W, b, y, mask)
    L = (torch.tensor(w) * rows).sum() / (denom if denom else 1.0)
    (lam * L).backward()
    assert abs(f["loss"] - L.item()) < 1e-12 * max(1.0, abs(L.item()))
    assert _close(f["dH"], Ht.grad.numpy()) and _close(f["dW"], Wt.grad.numpy())
    assert _close(f["db"], bt.grad.numpy())


def test_none_backward_matches_torch_autograd():
    H, W, b, y, mask = _case(20, N=25, D=5, V=60)
    rng = np.random.default_rng(3)
    w = rng.uniform(0.5, 1.5, 25)
    g = rng.standard_normal(25)
    f = orc.forward_backward(H, W, b, y, mask, weight=w, reduction="none", grad_rows=g)
    Ht, Wt, bt, rows = _torch_rows(H, W, b, y, mask)
    (torch.tensor(w) * rows).backward(torch.tensor(g))
    assert _close(f["dH"], Ht.grad.numpy()) and _close(f["dW"], Wt.grad.numpy())
    assert _close(f["db"], bt.grad.numpy())


def test_sum_over_c_equals_mean():
    H, W, b, y, mask = _case(21)
    idx, C = orc.supervised_rows(y, mask)
    a = orc.forward_backward(H, W, b, y, mask, lam=1.3)
    s = orc.forward_backward(H, W, b, y, mask, lam=1.3, reduction="sum", denom=float(C))
    assert abs(a["loss"] - s["loss"]) < 1e-13
    for k in ("dH", "dW", "db"):
        assert _close(a[k], s[k], 1e-13)


def test_weighted_sum_finite_differences():
    H, W, b, y, mask = _case(22, N=6, D=3, V=9, ignore=1, mask_false=1)
    w = np.array([0.5, 2.0, 1.0, 0.0, 3.0, 1.5])
    f = orc.forward_backward(H, W, b, y, mask, weight=w, reduction="sum", denom=4.0)
    eps = 1e-6
    for ix in [(0, 0), (2, 1), (5, 2)]:
        Hp, Hm = H.copy(), H.copy()
        Hp[ix] += eps
        Hm[ix] -= eps
        fd = (orc.forward(Hp, W, b, y, mask, weight=w, reduction="sum", denom=4.0)["loss"]
              - orc.forward(Hm, W, b, y, mask, weight=w, reduction="sum", denom=4.0)["loss"]) / (2 * eps)
        assert abs(fd - f["dH"][ix]) < 1e-8
    for j in [0, 4, 8]:
        bp, bm = b.copy(), b.copy()
        bp[j] += eps
        bm[j] -= eps
        fd = (orc.forward(H, W, bp, y, mask, weight=w, reduction="sum", denom=4.0)["loss"]
              - orc.forward(H, W, bm, y, mask, weight=w, reduction="sum", denom=4.0)["loss"]) / (2 * eps)
        assert abs(fd - f["db"][j]) < 1e-8


# --- logits rounded to the model dtype (opt-in variant) -----------------------

@pytest.mark.parametrize("dt,tdt", [("bf16", torch.bfloat16), ("fp16", torch.float16)])
def test_rounded_logits_match_torch_autograd(dt, tdt):
    """Logits cast to the 16-bit dtype before the loss, gradient passed through
    the cast: torch float64 autograd over an explicit round-trip cast."""
    H, W, b, y, mask = _case(23, N=30, D=8, V=80)
    f = orc.forward_backward(H, W, b, y, mask, lam=1.1, logits_dtype=dt)
    Ht = torch.tensor(H, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    Z = Ht @ Wt.T + bt
    Zr = Z + (Z.detach().to(torch.float32).to(tdt).to(torch.float64) - Z.detach())
    yy = torch.tensor(np.where(mask.astype(bool), y, -100))
    L = torch.nn.functional.cross_entropy(Zr, yy, ignore_index=-100)
    (1.1 * L).backward()
    assert abs(f["loss"] - L.item()) < 1e-12
    assert _close(f["dH"], Ht.grad.numpy()) and _close(f["dW"], Wt.grad.numpy())
    assert _close(f["db"], bt.grad.numpy())
    # the rounding changes the result (the variant is not a no-op)
    assert abs(orc.forward(H, W, b, y, mask)["loss"] - f["loss"]) > 1e-9


def test_rounded_logits_are_exact_16bit_values():
    H, W, b, y, mask = _case(24, N=5, D=4, V=11)
    Z = orc._logits(torch.tensor(H), torch.tensor(W), torch.tensor(b), "bf16")
    Zb = Z.to(torch.bfloat16).to(torch.float64)
    assert torch.equal(Z, Zb)
