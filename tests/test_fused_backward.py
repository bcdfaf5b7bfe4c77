"""GPU parity of the single-kernel backward (D <= 64): the scores, the
gradient of the logits and both contractions per tile in one kernel, dH kept
on chip per row block, dW summed from per-row-block partials ("分块交叉熵"
page, §04).  Each case runs both backward forms on the same inputs and checks
each against the binary64 oracle, then the two against each other."""
import numpy as np
import pytest
import torch

from lm_head_projection_supervised_b200 import binding
from lm_head_projection_supervised_b200 import workloads as wl
from oracle import flce_oracle as orc

from _gpu_helpers import check_grad, check_loss, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from lm_head_projection_supervised_b200 import build
    build.build()
    binding.lib()


def _both_forms(inp, **kw):
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    loss, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws,
                                    round_logits=kw.get("round_logits", False))
    out = {}
    for form, panel in (("fused", False), ("panel", True)):
        dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=inp.lam, ws=ws,
                                      panel_backward=panel, **kw)
        assert binding.device_status(ws) == 0
        out[form] = dict(dH=dH.cpu().numpy(), dW=dW.cpu().numpy(),
                         db=None if db is None else db.cpu().numpy())
    return loss.item(), out


CASES = [
    # several row blocks and vocabulary chunks, ragged C and V
    ("d64_bias", dict(seed=71, N=1100, D=64, V=5000)),
    ("d64_many_chunks", dict(seed=72, N=2000, D=64, V=20011, bias=False)),
    ("d40_fp16", dict(seed=73, N=600, D=40, V=3001, dtype="fp16")),
    ("d24_one_tile", dict(seed=74, N=300, D=24, V=100)),
    ("d8_v1", dict(seed=75, N=70, D=8, V=1)),
    ("d64_one_row", dict(seed=76, N=1, D=64, V=900, ignore_frac=0.0, mask_false_frac=0.0)),
]


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_fused_and_panel_backward_match_the_oracle(name, kw):
    inp = wl.random_case(**kw)
    loss, out = _both_forms(inp)
    ref = orc.forward_backward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask,
                               lam=inp.lam)
    check_loss(loss, ref["loss"])
    for form in ("fused", "panel"):
        g = out[form]
        check_grad(f"dH_{form}", g["dH"], ref["dH"])
        check_grad(f"dW_{form}", g["dW"], ref["dW"])
        if inp.b is not None:
            check_grad(f"db_{form}", g["db"], ref["db"])
    unsup = np.setdiff1d(np.arange(inp.N), ref["idx"])
    assert not out["fused"]["dH"][unsup].any()
    # the two forms differ only by rounding order: well inside the bar
    for q in ("dH", "dW"):
        scale = np.abs(ref[q]).max()
        if scale > 0:
            assert np.abs(out["fused"][q] - out["panel"][q]).max() <= 1e-3 * scale


def test_fused_backward_mixed_row_scales():
    """Per-row upstream gradients that are positive for the first rows and of
    mixed sign (some zero) after them: warps whose rows all have a positive
    scale take it into the exponent, the others scale each entry, and both
    must agree with the oracle."""
    inp = wl.random_case(seed=80, N=700, D=64, V=6000, bias=False, ignore_frac=0.0,
                         mask_false_frac=0.0)
    rng = np.random.default_rng(80)
    g = 10.0 ** rng.uniform(-2, 1, inp.N)
    tail = np.arange(inp.N) >= 256
    g[tail] *= rng.choice([-1.0, 0.0, 1.0], int(tail.sum()))
    g32 = torch.tensor(g, dtype=torch.float32).numpy().astype(np.float64)
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    _, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws, reduction="none")
    grads = torch.tensor(g32, dtype=torch.float32, device="cuda")
    out = {}
    for form, panel in (("fused", False), ("panel", True)):
        dH, dW, _ = binding.backward(H, W, b, y, mk, -100, m, logs, lam=1.0, ws=ws,
                                     reduction="none", grad_rows=grads, panel_backward=panel)
        assert binding.device_status(ws) == 0
        out[form] = (dH.cpu().numpy(), dW.cpu().numpy())
    ref = orc.forward_backward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask, lam=1.0,
                               reduction="none", grad_rows=g32)
    for form in ("fused", "panel"):
        check_grad(f"dH_{form}", out[form][0], ref["dH"])
        check_grad(f"dW_{form}", out[form][1], ref["dW"])
    # rows with a zero upstream gradient get a zero dH row
    zero = np.flatnonzero(g32 == 0.0)
    assert zero.size > 0 and not out["fused"][0][zero].any()


def test_fused_backward_rounded_logits():
    inp = wl.random_case(seed=77, N=500, D=64, V=4000)
    loss, out = _both_forms(inp, round_logits=True)
    ref = orc.forward_backward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask,
                               lam=inp.lam, logits_dtype=inp.dtype)
    check_loss(loss, ref["loss"])
    check_grad("dH", out["fused"]["dH"], ref["dH"])
    check_grad("dW", out["fused"]["dW"], ref["dW"])
    check_grad("db", out["fused"]["db"], ref["db"])


def test_fused_backward_is_deterministic():
    inp = wl.random_case(seed=78, N=1500, D=64, V=12000)
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    _, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws)
    r1 = binding.backward(H, W, b, y, mk, -100, m, logs, lam=1.0, ws=ws)
    r2 = binding.backward(H, W, b, y, mk, -100, m, logs, lam=1.0, ws=ws)
    for a, c in zip(r1, r2):
        assert torch.equal(a, c)


def test_fused_backward_no_supervised_rows():
    inp = wl.random_case(seed=79, N=400, D=64, V=3000)
    inp.labels[:] = -100
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    _, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=1.0, ws=ws)
    assert binding.device_status(ws) == 0
    assert not dH.any() and not dW.any() and not db.any()

