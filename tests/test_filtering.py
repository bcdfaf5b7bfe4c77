"""GPU: the opt-in gradient filtering (flce_backward_filtered) against the
filtering oracle (oracle/flce_filtered.py), how far it lands from the exact
gradient, and that filter_eps = 0 is the exact backward bit for bit."""
import numpy as np
import pytest
import torch

from lm_head_projection_supervised_b200 import binding
from lm_head_projection_supervised_b200 import workloads as wl
from oracle import flce_filtered as ofl
from oracle import flce_oracle as orc

from _gpu_helpers import check_grad, record, to_device

pytestmark = pytest.mark.gpu
EPS = 2.0 ** -12


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from lm_head_projection_supervised_b200 import build
    build.build()
    binding.lib()


def _peaked(seed, N, D, V, dtype="bf16", bias=False):
    spec = wl.dataclasses.replace(wl.SPECS["peaked"], N=N, D=D, V=V, dtype=dtype,
                                  segments=0, prefix_frac=0.0, ignore_frac=0.2,
                                  mask_false_frac=0.05, bias_std=0.05 if bias else None)
    return wl.make_inputs(spec, seed=seed)


# The peaked construction needs D of several hundred (the other logits'
# spread grows as the logits placed on purpose, over sqrt(D)).
CASES = [
    ("peaked_two_panels", dict(seed=31, N=700, D=512, V=9000)),
    ("peaked_fp16_bias", dict(seed=32, N=515, D=520, V=8500, dtype="fp16", bias=True)),
    ("peaked_three_panels", dict(seed=33, N=1100, D=1024, V=20000)),
]


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_filtered_matches_filtering_oracle(name, kw):
    inp = _peaked(**kw)
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    loss, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=inp.lam, ws=ws,
                                  filter_eps=EPS)
    assert binding.device_status(ws) == 0
    args = (inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask)
    f = orc.forward(*args)
    ref = ofl.backward_filtered(*args, lam=inp.lam, m=f["m"], logs=f["logs"], eps=EPS)
    kept = ref["keep"].mean()
    assert 0.0 < kept < 0.5, kept          # the filter drops most blocks here
    check_grad("dH filtered", dH.cpu().numpy(), ref["dH"])
    check_grad("dW filtered", dW.cpu().numpy(), ref["dW"])
    if b is not None:
        check_grad("db filtered", db.cpu().numpy(), ref["db"])
    # how far the approximation lands from the exact gradient (reported only)
    ex = orc.backward(*args, lam=inp.lam, m=f["m"], logs=f["logs"])
    gH, gW = dH.cpu().numpy().astype(np.float64), dW.cpu().numpy().astype(np.float64)
    record("dH filtered vs exact (report)", float(np.max(np.abs(gH - ex[0]))),
           2e-3 * float(np.max(np.abs(ex[0]))), kept_blocks=float(kept))
    record("dW filtered vs exact (report)", float(np.max(np.abs(gW - ex[1]))),
           2e-3 * float(np.max(np.abs(ex[1]))), kept_blocks=float(kept))


def test_filter_eps_zero_is_the_exact_backward():
    inp = _peaked(seed=34, N=400, D=512, V=8300, bias=True)
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    _, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws)
    exact = binding.backward(H, W, b, y, mk, -100, m, logs, lam=0.8, ws=ws)
    outs = [torch.empty_like(t) for t in exact]
    L = binding.lib()
    P = binding._ptr
    st = L.flce_backward_filtered(P(H), P(W), P(b), P(y), P(mk), -100, inp.N, inp.D, inp.V,
                                  binding.dtype_code(H.dtype), P(m), P(logs), None, 0, 0.0, 0,
                                  0.8, None, None, 0.0, P(outs[0]), P(outs[1]), P(outs[2]),
                                  ws.ptr(), ws.nbytes, binding._stream(None))
    assert st == 0
    assert binding.device_status(ws) == 0
    for a, c in zip(exact, outs):
        assert torch.equal(a, c)


def test_filter_eps_rejected_when_negative():
    inp = _peaked(seed=35, N=64, D=32, V=600)
    H, W, b, y, mk = to_device(inp)
    _, m, logs = binding.forward(H, W, b, y, mk)
    with pytest.raises(binding.FlceError):
        binding.backward(H, W, b, y, mk, -100, m, logs, filter_eps=-1e-3)


def test_exact_backward_on_peaked_logits():
    """The exact path on the same peaked inputs: its dH error against the exact
    oracle shows what the 16-bit staging of large non-target probabilities
    costs without any filtering."""
    inp = _peaked(**CASES[0][1])
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    _, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws)
    dH, dW, _ = binding.backward(H, W, b, y, mk, -100, m, logs, lam=inp.lam, ws=ws)
    ex = orc.forward_backward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask, lam=inp.lam)
    check_grad("dH exact, peaked", dH.cpu().numpy(), ex["dH"])
    check_grad("dW exact, peaked", dW.cpu().numpy(), ex["dW"])
