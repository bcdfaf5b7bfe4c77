"""GPU parity of the reduction variants (sum with a global label count, per-row
losses, per-row weights and per-row upstream gradients) against the oracle."""
import numpy as np
import pytest
import torch

from lm_head_projection_supervised_b200 import binding
from lm_head_projection_supervised_b200 import workloads as wl
from oracle import flce_oracle as orc

from _gpu_helpers import check_grad, check_loss, check_stats, logs_floor, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from lm_head_projection_supervised_b200 import build
    build.build()
    binding.lib()


CASES = [
    # name, case kwargs, reduction, weights?, denom
    ("sum_denom", dict(seed=31, N=300, D=72, V=9000), "sum", False, 517.0),
    ("sum_weights", dict(seed=32, N=257, D=64, V=5000, bias=False), "sum", True, None),
    ("mean_weights_fp16", dict(seed=33, N=200, D=40, V=3000, dtype="fp16"), "mean", True, None),
    ("none_bf16", dict(seed=34, N=400, D=128, V=9100), "none", True, None),
    ("none_fp16_bias", dict(seed=35, N=129, D=32, V=2000, dtype="fp16"), "none", False, None),
]


@pytest.mark.parametrize("name,kw,reduction,weighted,denom", CASES, ids=[c[0] for c in CASES])
def test_reduction_parity(name, kw, reduction, weighted, denom):
    inp = wl.random_case(**kw)
    rng = np.random.default_rng(kw["seed"])
    w = rng.uniform(0.0, 2.0, inp.N) if weighted else None
    # per-row upstream gradients of both signs, spanning three decades
    g = rng.choice([-1.0, 1.0], inp.N) * 10.0 ** rng.uniform(-2, 1, inp.N)
    lam = 0.7
    H, W, b, y, mk = to_device(inp)
    wt = None if w is None else torch.tensor(w, dtype=torch.float32, device="cuda")
    w32 = None if w is None else wt.cpu().numpy().astype(np.float64)  # the values the GPU sees
    g32 = torch.tensor(g, dtype=torch.float32).numpy().astype(np.float64)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    loss, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws, weight=wt,
                                    reduction=reduction, denom=denom)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=lam, ws=ws, weight=wt,
                                  reduction=reduction, denom=denom,
                                  grad_rows=torch.tensor(g32, dtype=torch.float32,
                                                         device="cuda"))
    assert binding.device_status(ws) == 0
    ref = orc.forward_backward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask, lam=lam,
                               weight=w32, reduction=reduction, denom=denom, grad_rows=g32)
    idx = ref["idx"]
    if reduction == "none":
        got = loss.cpu().numpy().astype(np.float64)
        err = np.abs(got - ref["loss_vec"])
        assert np.all(err <= 1e-4 * np.maximum(np.abs(ref["loss_vec"]), 1.0)), err.max()
        unsup = np.setdiff1d(np.arange(inp.N), idx)
        assert np.all(got[unsup] == 0.0)
    else:
        check_loss(loss.item(), ref["loss"])
    check_stats(m.cpu().numpy(), ref["m"], idx, quantity="m")
    check_stats(logs.cpu().numpy(), ref["logs"], idx, floor=logs_floor(ref["m"][idx], inp.D),
                quantity="logs")
    check_grad("dH", dH.cpu().numpy(), ref["dH"])
    check_grad("dW", dW.cpu().numpy(), ref["dW"])
    if inp.b is not None:
        check_grad("db", db.cpu().numpy(), ref["db"])


def test_mean_reduction_is_the_plain_call():
    """flce_forward/flce_backward are the _ex calls with MEAN and no weights."""
    inp = wl.random_case(seed=36, N=150, D=48, V=1200)
    H, W, b, y, mk = to_device(inp)
    l0, m0, s0 = binding.forward(H, W, b, y, mk)
    g0 = binding.backward(H, W, b, y, mk, -100, m0, s0, lam=1.5)
    l1, m1, s1 = binding.forward(H, W, b, y, mk, weight=torch.ones(inp.N, device="cuda"),
                                 reduction="mean")
    g1 = binding.backward(H, W, b, y, mk, -100, m1, s1, lam=1.5,
                          weight=torch.ones(inp.N, device="cuda"))
    assert torch.equal(l0, l1) and torch.equal(m0, m1)
    for a, c in zip(g0, g1):
        assert torch.equal(a, c)


def test_loss_module_none_with_leading_dims():
    """The nn.Module front end: hidden [2, T, D], per-token losses [2, T], and
    autograd gradients equal to the oracle's for sum_i g_i w_i l_i."""
    inp = wl.random_case(seed=37, N=2 * 96, D=64, V=2500)
    H, W, b, y, mk = to_device(inp)
    rng = np.random.default_rng(37)
    w = rng.uniform(0.5, 1.5, inp.N).astype(np.float32)
    g = rng.standard_normal(inp.N).astype(np.float32)
    Hp = H.reshape(2, 96, inp.D).clone().requires_grad_(True)
    Wp = W.clone().requires_grad_(True)
    crit = binding.LinearCrossEntropyLoss(reduction="none")
    out = crit(Hp, y.reshape(2, 96), Wp, loss_weights=torch.tensor(w, device="cuda").reshape(2, 96),
               mask=mk.reshape(2, 96))
    assert out.shape == (2, 96)
    out.backward(torch.tensor(g, device="cuda").reshape(2, 96))
    ref = orc.forward_backward(inp.H64(), inp.W64(), None, inp.labels, inp.mask,
                               weight=w.astype(np.float64), reduction="none",
                               grad_rows=g.astype(np.float64))
    err = np.abs(out.detach().cpu().numpy().reshape(-1) - ref["loss_vec"])
    assert np.all(err <= 1e-4 * np.maximum(np.abs(ref["loss_vec"]), 1.0))
    # gradients come back in the parameter dtype (bf16): compare at bf16 resolution
    dH = Hp.grad.float().cpu().numpy().reshape(inp.N, inp.D)
    dW = Wp.grad.float().cpu().numpy()
    assert np.max(np.abs(dH - ref["dH"])) <= 1e-2 * np.max(np.abs(ref["dH"]))
    assert np.max(np.abs(dW - ref["dW"])) <= 1e-2 * np.max(np.abs(ref["dW"]))


def ulp16(x, dtype):
    """Spacing of the 16-bit type at |x| (7 fraction bits for bf16, 10 for fp16)."""
    frac = 7 if dtype == "bf16" else 10
    e = np.floor(np.log2(np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -14)))
    return 2.0 ** (e - frac)


@pytest.mark.parametrize("kw", [dict(seed=41, N=300, D=64, V=9000),
                                dict(seed=42, N=200, D=48, V=3000, dtype="fp16")],
                         ids=["bf16", "fp16_bias"])
def test_rounded_logits_parity(kw):
    """Logits rounded to the input dtype (NeMo logits_dtype).  The GPU rounds
    its fp32 logit, the oracle its exact one; a logit within fp32 error of a
    16-bit rounding boundary can round the other way, so m and log s may
    differ by one 16-bit spacing of the row's largest logit."""
    inp = wl.random_case(**kw)
    H, W, b, y, mk = to_device(inp)
    loss, m, logs = binding.forward(H, W, b, y, mk, round_logits=True)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=inp.lam, round_logits=True)
    ref = orc.forward_backward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask,
                               lam=inp.lam, logits_dtype=inp.dtype)
    plain = orc.forward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask)
    idx = ref["idx"]
    check_loss(loss.item(), ref["loss"])
    # the variant is visible: the rounded-logit loss is not the exact one
    assert abs(ref["loss"] - plain["loss"]) > 10 * abs(loss.item() - ref["loss"])
    ulp = ulp16(ref["m"][idx], inp.dtype)
    check_stats(m.cpu().numpy(), ref["m"], idx, floor=ulp, quantity="m")
    check_stats(logs.cpu().numpy(), ref["logs"], idx,
                floor=np.maximum(ulp, logs_floor(ref["m"][idx], inp.D)), quantity="logs")
    check_grad("dH", dH.cpu().numpy(), ref["dH"])
    check_grad("dW", dW.cpu().numpy(), ref["dW"])
    if inp.b is not None:
        check_grad("db", db.cpu().numpy(), ref["db"])


def test_weighted_target_term_of_dh_is_exact():
    """With weights the panel entry s_i/S (p - 1) sigma is rounded to 16 bits
    with up to 2^-8 relative error, and that entry dominates the row's dH.  The
    backward adds the rounding residual back in fp32, so dH's error is left to
    the small off-target entries: far inside the 2e-3 bar (checked at 2e-4)."""
    inp = wl.random_case(seed=55, N=400, D=128, V=12000)
    H, W, b, y, mk = to_device(inp)
    rng = np.random.default_rng(55)
    wt = torch.tensor(rng.uniform(0.0, 2.0, inp.N), dtype=torch.float32, device="cuda")
    loss, m, logs = binding.forward(H, W, b, y, mk, weight=wt, reduction="sum", denom=611.0)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=1.0, weight=wt,
                                  reduction="sum", denom=611.0)
    ref = orc.forward_backward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask,
                               weight=wt.cpu().numpy().astype(np.float64), reduction="sum",
                               denom=611.0)
    got = dH.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - ref["dH"])) <= 2e-4 * np.max(np.abs(ref["dH"]))
    check_grad("dW", dW.cpu().numpy(), ref["dW"])
