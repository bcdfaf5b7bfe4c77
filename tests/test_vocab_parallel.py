"""GPU parity of the vocabulary-sharded calls (flce_shard_forward,
flce_shard_combine, flce_shard_backward) against the oracle.  All slices run
on one GPU, one after the other, with the two exchanges done in place (the
statistics in one [P, N, 4] buffer, the dH terms summed by the backward's
accumulate flag): the same kernels and data as a multi-rank step."""
import numpy as np
import pytest
import torch

from lm_head_projection_supervised_b200 import binding
from lm_head_projection_supervised_b200 import vocab_parallel as vp
from lm_head_projection_supervised_b200 import workloads as wl
from oracle import flce_oracle as orc
from oracle import flce_shards as sh

from _gpu_helpers import (check_grad, check_loss, check_stats, logs_floor, sampled_check,
                          to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from lm_head_projection_supervised_b200 import build
    build.build()
    binding.lib()


def _np(t):
    return None if t is None else t.cpu().numpy()


def test_slice_statistics_match_the_oracle():
    """Each slice's (m_r, log s_r, t_r, o_r): ownership bit-exact, the rest to
    the statistics' tolerance."""
    inp = wl.random_case(seed=51, N=333, D=96, V=7000)
    H, W, b, y, mk = to_device(inp)
    H64, W64, b64 = inp.H64(), inp.W64(), inp.b64()
    idx, _ = orc.supervised_rows(inp.labels, inp.mask)
    unsup = np.setdiff1d(np.arange(inp.N), idx)
    for r in range(3):
        v0, n = vp.vocab_slice(inp.V, 3, r)
        st = binding.shard_forward(H, W[v0:v0 + n], b[v0:v0 + n], y, mk, v0=v0, V_total=inp.V)
        got = st.cpu().numpy().astype(np.float64)
        ref = sh.shard_partials(H64, W64[v0:v0 + n], b64[v0:v0 + n], inp.labels, inp.mask,
                                v0=v0, V_total=inp.V)
        assert np.array_equal(got[:, 3], ref[:, 3])
        check_stats(got[:, 0], ref[:, 0], idx)
        check_stats(got[:, 1], ref[:, 1], idx, floor=logs_floor(ref[idx, 0], inp.D))
        own = idx[ref[idx, 3] == 1.0]
        check_stats(got[:, 2], ref[:, 2], own)
        assert np.all(got[np.setdiff1d(idx, own), 2] == 0.0)
        assert np.all(np.isneginf(got[unsup, :2])) and not got[unsup, 2:].any()


CASES = [
    # name, case kwargs, P, extra
    ("bf16_bias_p2", dict(seed=52, N=300, D=64, V=9000), 2, {}),
    ("bf16_p3_ragged", dict(seed=53, N=517, D=136, V=20011, bias=False), 3, {}),
    ("fp16_p4", dict(seed=54, N=260, D=40, V=5000, dtype="fp16"), 4, {}),
    ("p8_sum_weights", dict(seed=55, N=400, D=128, V=12000), 8,
     dict(reduction="sum", denom=611.0, weighted=True)),
    ("p5_none", dict(seed=56, N=129, D=32, V=4000, dtype="fp16"), 5,
     dict(reduction="none", weighted=True)),
    ("p3_rounded", dict(seed=57, N=200, D=48, V=3000), 3, dict(round_logits=True)),
    ("p2_tiny_slices", dict(seed=58, N=64, D=16, V=300), 2, {}),   # V < 256 P: unaligned cut
]


@pytest.mark.parametrize("name,kw,P,extra", CASES, ids=[c[0] for c in CASES])
def test_slices_reproduce_the_dense_oracle(name, kw, P, extra):
    inp = wl.random_case(**kw)
    H, W, b, y, mk = to_device(inp)
    rng = np.random.default_rng(kw["seed"])
    reduction = extra.get("reduction", "mean")
    w = rng.uniform(0.0, 2.0, inp.N) if extra.get("weighted") else None
    g = rng.standard_normal(inp.N) if reduction == "none" else None
    wt = None if w is None else torch.tensor(w, dtype=torch.float32, device="cuda")
    gt = None if g is None else torch.tensor(g, dtype=torch.float32, device="cuda")
    w32 = None if wt is None else _np(wt).astype(np.float64)
    g32 = None if gt is None else _np(gt).astype(np.float64)
    rl = extra.get("round_logits", False)
    got = vp.run_slices_on_one_device(H, W, b, y, mk, -100, P=P, lam=inp.lam, weight=wt,
                                      reduction=reduction, denom=extra.get("denom"),
                                      grad_rows=gt, round_logits=rl)
    ref = orc.forward_backward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask,
                               lam=inp.lam, weight=w32, reduction=reduction,
                               denom=extra.get("denom"), grad_rows=g32,
                               logits_dtype=inp.dtype if rl else None)
    idx = ref["idx"]
    if reduction == "none":
        lv = _np(got["loss"]).astype(np.float64)
        assert np.all(np.abs(lv - ref["loss_vec"]) <= 1e-4 * np.maximum(np.abs(ref["loss_vec"]),
                                                                        1.0))
    else:
        check_loss(got["loss"].item(), ref["loss"])
    floor = logs_floor(ref["m"][idx], inp.D)
    if rl:   # one 16-bit spacing of the row max, as for the unsharded rounded variant
        frac = 7 if inp.dtype == "bf16" else 10
        floor = np.maximum(floor, 2.0 ** (np.floor(np.log2(np.maximum(
            np.abs(ref["m"][idx]), 2.0 ** -14))) - frac))
    check_stats(_np(got["m"]), ref["m"], idx, floor=floor if rl else None, quantity="m")
    check_stats(_np(got["logs"]), ref["logs"], idx, floor=floor, quantity="logs")
    check_grad("dH", _np(got["dH"]), ref["dH"])
    check_grad("dW", _np(got["dW"]), ref["dW"])
    if inp.b is not None:
        check_grad("db", _np(got["db"]), ref["db"])


def test_one_slice_equals_the_unsharded_call():
    """P = 1: the slice path and flce_forward/flce_backward agree (the
    combine re-rounds log s through exp/log, so to the statistics' tolerance;
    the gradients to float32 rounding)."""
    inp = wl.random_case(seed=59, N=250, D=64, V=3000)
    H, W, b, y, mk = to_device(inp)
    got = vp.run_slices_on_one_device(H, W, b, y, mk, -100, P=1, lam=inp.lam)
    loss, m, logs = binding.forward(H, W, b, y, mk)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=inp.lam)
    idx, _ = orc.supervised_rows(inp.labels, inp.mask)
    assert torch.equal(got["m"], m)
    check_stats(_np(got["logs"]), _np(logs).astype(np.float64), idx, quantity="logs")
    check_loss(got["loss"].item(), loss.item())
    for a, c in ((got["dH"], dH), (got["dW"], dW), (got["db"], db)):
        assert (a - c).abs().max().item() <= 1e-5 * c.abs().max().item()


def test_combine_reports_a_missing_slice():
    """Stats of only some slices: the combine records FLCE_ERR_SHARD and the
    loss is NaN (an input error turned into a status, no device fault)."""
    inp = wl.random_case(seed=60, N=100, D=32, V=2000)
    H, W, b, y, mk = to_device(inp)
    v0, n = vp.vocab_slice(inp.V, 2, 0)
    st = binding.shard_forward(H, W[v0:v0 + n], b[v0:v0 + n], y, mk, v0=v0, V_total=inp.V)
    cws = binding.CombineWorkspace(inp.N)
    loss, m, logs = binding.shard_combine(st[None], y, mk, ws=cws)
    assert binding.device_status(cws) == binding.STATUS_CODE["FLCE_ERR_SHARD"]
    assert torch.isnan(loss).item()
    # the same slice twice
    loss, _, _ = binding.shard_combine(torch.stack([st, st]), y, mk, ws=cws)
    assert binding.device_status(cws) == binding.STATUS_CODE["FLCE_ERR_SHARD"]


def test_label_outside_the_full_vocabulary_is_reported():
    inp = wl.random_case(seed=61, N=64, D=32, V=1000)
    H, W, b, y, mk = to_device(inp)
    y[3], mk[3] = 1000, 1       # inside no slice of [0, 1000)
    ws = binding.Workspace(inp.N, inp.D, 500, H.dtype)
    binding.shard_forward(H, W[500:], b[500:], y, mk, v0=500, V_total=1000, ws=ws)
    assert binding.device_status(ws) == binding.STATUS_CODE["FLCE_ERR_LABEL"]


def test_packed_workload_eight_slices_sampled():
    """The full 16384 x 1024 x 248320 workload cut into 8 slices, checked on
    sampled rows and vocabulary ids like the unsharded full-size test."""
    inp = wl.make_inputs("packed")
    H, W, b, y, mk = to_device(inp)
    Vmax = max(vp.vocab_slice(inp.V, 8, r)[1] for r in range(8))
    ws = binding.Workspace(inp.N, inp.D, Vmax, H.dtype)
    got = vp.run_slices_on_one_device(H, W, b, y, mk, -100, P=8, lam=inp.lam, ws=ws)
    assert binding.device_status(ws) == 0
    res = dict(loss=got["loss"].item(), m=_np(got["m"]), logs=_np(got["logs"]),
               dH=_np(got["dH"]), dW=_np(got["dW"]), db=_np(got["db"]))
    sampled_check(inp, res, full_stats=True)


def test_accumulate_dh_adds_in_place():
    """FLCE_FLAG_ACCUMULATE_DH: dH += the call's dH; unsupervised rows keep
    what they held."""
    inp = wl.random_case(seed=62, N=300, D=64, V=4000)
    H, W, b, y, mk = to_device(inp)
    loss, m, logs = binding.forward(H, W, b, y, mk)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=inp.lam)
    base = torch.randn(inp.N, inp.D, device="cuda")
    acc = base.clone()
    binding.backward(H, W, b, y, mk, -100, m, logs, lam=inp.lam, accumulate_dh=True,
                     out=(acc, torch.empty_like(dW), torch.empty_like(db)))
    idx, _ = orc.supervised_rows(inp.labels, inp.mask)
    unsup = torch.from_numpy(np.setdiff1d(np.arange(inp.N), idx)).cuda()
    assert torch.equal(acc[unsup], base[unsup])
    assert (acc - (base + dH)).abs().max().item() <= 1e-6 * (base + dH).abs().max().item()


def test_autograd_wrapper_on_a_one_rank_nccl_group():
    """vocab_parallel_cross_entropy with the real NCCL collectives (one rank:
    the whole vocabulary is the slice) equals the unsharded call, through
    torch.autograd."""
    import socket

    import torch.distributed as dist
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        inp = wl.random_case(seed=63, N=200, D=64, V=3000)
        H, W, b, y, mk = to_device(inp)
        Hp = H.clone().requires_grad_(True)
        Wp = W.clone().requires_grad_(True)
        bp = b.clone().requires_grad_(True)
        loss = vp.vocab_parallel_cross_entropy(Hp, Wp, y, V_total=inp.V, v0=0, b_slice=bp,
                                               mask=mk)
        (0.5 * loss).backward()
        ref_loss, m, logs = binding.forward(H, W, b, y, mk)
        dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=0.5)
        check_loss(loss.item(), ref_loss.item())
        for got, ref in ((Hp.grad, dH), (Wp.grad, dW), (bp.grad, db)):
            g = got.float()
            assert (g - ref).abs().max().item() <= 1e-2 * ref.abs().max().item()
    finally:
        dist.destroy_process_group()
