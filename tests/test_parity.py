"""GPU parity: the CUDA path through the C ABI against the binary64 oracle on
the same seeded 16-bit inputs."""
import numpy as np
import pytest
import torch

from lm_head_projection_supervised_b200 import binding
from lm_head_projection_supervised_b200 import workloads as wl
from oracle import flce_oracle as orc

from _gpu_helpers import (check_grad, check_loss, check_stats, logs_floor, sampled_check,
                          to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from lm_head_projection_supervised_b200 import build
    build.build()
    binding.lib()


def run_gpu(inp, lam=None):
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    loss, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs,
                                  lam=inp.lam if lam is None else lam, ws=ws)
    st = binding.device_status(ws)
    return dict(loss=loss.item(), m=m.cpu().numpy(), logs=logs.cpu().numpy(),
                dH=dH.cpu().numpy(), dW=dW.cpu().numpy(),
                db=None if db is None else db.cpu().numpy(), status=st)


def full_check(inp, got):
    ref = orc.forward_backward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask,
                               lam=inp.lam)
    assert got["status"] == 0, binding.status_string(got["status"])
    check_loss(got["loss"], ref["loss"])
    idx = ref["idx"]
    unsup = np.setdiff1d(np.arange(inp.N), idx)
    check_stats(got["m"], ref["m"], idx, quantity="m")
    check_stats(got["logs"], ref["logs"], idx, floor=logs_floor(ref["m"][idx], inp.D),
                quantity="logs")
    assert np.all(np.isneginf(got["m"][unsup])) and np.all(np.isneginf(got["logs"][unsup]))
    assert not got["dH"][unsup].any()
    check_grad("dH", got["dH"], ref["dH"])
    check_grad("dW", got["dW"], ref["dW"])
    if inp.b is not None:
        check_grad("db", got["db"], ref["db"])
    return ref


# --------------------------------------------------------------------------
# the tensor-core GEMM core, every operand layout
# --------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 1), (0, 1), (1, 0)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 296, 136), (384, 520, 1000)])
def test_gemm_core_layouts(dtype, a_mn, b_mn, M, N, K):
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K + 11 * a_mn + 5 * b_mn)
    A = torch.randn(M, K, generator=g).to(dtype)
    B = torch.randn(N, K, generator=g).to(dtype)
    ref = A.double() @ B.double().T
    Ad = (A.T.contiguous() if a_mn else A).cuda()
    Bd = (B.T.contiguous() if b_mn else B).cuda()
    out = binding.diag_gemm(Ad, Bd, M, N, K, bool(a_mn), bool(b_mn), scale=0.5).cpu().double()
    err = (out - 0.5 * ref).abs().max().item()
    assert err <= 1e-4 * 0.5 * ref.abs().max().item() + 1e-5, err


# --------------------------------------------------------------------------
# compaction
# --------------------------------------------------------------------------
@pytest.mark.parametrize("N", [0, 1, 1000, 32768, 100003])
def test_compaction_bit_exact(N):
    rng = np.random.default_rng(N)
    y = rng.integers(0, 50, N)
    y[rng.random(N) < 0.3] = -100
    mask = (rng.random(N) > 0.1).astype(np.uint8)
    idx, C, ws = binding.compact(torch.from_numpy(y).cuda(), torch.from_numpy(mask).cuda(), -100, 50)
    want, Cw = orc.supervised_rows(y, mask)
    assert int(C.item()) == Cw
    assert np.array_equal(idx[:Cw].cpu().numpy(), want)


# --------------------------------------------------------------------------
# parity on small and ragged shapes (several tiles, ragged tails, panels)
# --------------------------------------------------------------------------
CASES = [
    ("tiny", None),
    ("small", None),
    ("ragged_a", dict(seed=1, N=129, D=40, V=257)),
    ("ragged_b", dict(seed=2, N=300, D=72, V=1000, dtype="fp16")),
    ("two_panels", dict(seed=3, N=257, D=136, V=4100)),
    ("three_panels_fp16", dict(seed=4, N=200, D=64, V=8492, dtype="fp16", bias=True)),
    ("no_bias_wide_d", dict(seed=5, N=160, D=520, V=3000, bias=False)),
    ("single_class", dict(seed=6, N=5, D=8, V=1)),
    ("one_row", dict(seed=7, N=1, D=16, V=700, ignore_frac=0.0, mask_false_frac=0.0)),
    # small hidden sizes: one exponential in four on the FMA pipe
    ("small_d64", dict(seed=15, N=700, D=64, V=9000)),
    ("small_d128_fp16", dict(seed=16, N=600, D=128, V=8300, dtype="fp16")),
    # few labels: each label's rows span many windows of the dW target-term sums
    ("few_labels", dict(seed=17, N=1000, D=200, V=12)),
    ("few_labels_d64_fp16", dict(seed=18, N=900, D=64, V=5, dtype="fp16")),
    # size extremes: a vocabulary of a million ids (thousands of tiles; 74 chained panel
    # launches at D = 136) and the largest specified hidden size on a ragged small case
    ("wide_vocab_d64", dict(seed=19, N=300, D=64, V=1000003)),
    ("wide_vocab_panels", dict(seed=20, N=260, D=136, V=600011, dtype="fp16")),
    ("deep_d4096_fp16", dict(seed=21, N=300, D=4096, V=5000, dtype="fp16")),
]


def case_inputs(name, kw):
    if kw is None:
        return wl.make_inputs(name)
    return wl.random_case(**kw)


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_parity(name, kw):
    inp = case_inputs(name, kw)
    full_check(inp, run_gpu(inp))


def test_large_common_shift():
    """Rows scaled far up: m is large, the (m - target) + log s form keeps
    the loss accurate ("分块交叉熵" page §02)."""
    inp = wl.random_case(seed=8, N=96, D=64, V=2000, w_std=0.1)
    H = inp.H.copy()
    Hf = wl.decode_f64(H, "bf16")
    Hf[:8] *= 300.0
    inp.H[:] = wl.encode(Hf.astype(np.float32), "bf16")
    full_check(inp, run_gpu(inp))


def test_zero_supervised_rows():
    inp = wl.random_case(seed=9, N=300, D=32, V=1500)
    inp.labels[:] = -100
    got = run_gpu(inp)
    assert got["status"] == 0 and got["loss"] == 0.0
    assert np.all(np.isneginf(got["m"])) and np.all(np.isneginf(got["logs"]))
    assert not got["dH"].any() and not got["dW"].any() and not got["db"].any()


def test_label_out_of_range_is_reported():
    inp = wl.random_case(seed=10, N=64, D=32, V=500, mask_false_frac=0.0)
    inp.labels[3] = 500
    got = run_gpu(inp)
    assert binding.STATUS[got["status"]] == "FLCE_ERR_LABEL"
    assert np.isnan(got["loss"])


def test_bounded_wait_reports_timeout():
    """A wait nothing completes gives up after its limit; the error word says so."""
    assert binding.STATUS[binding.diag_timeout(20_000_000)] == "FLCE_ERR_TIMEOUT"


def test_backward_is_deterministic():
    inp = wl.random_case(seed=11, N=700, D=128, V=9000)
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    loss, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws)
    r1 = binding.backward(H, W, b, y, mk, -100, m, logs, lam=1.0, ws=ws)
    r2 = binding.backward(H, W, b, y, mk, -100, m, logs, lam=1.0, ws=ws)
    for a, c in zip(r1, r2):
        assert torch.equal(a, c)
    l2, _, _ = binding.forward(H, W, b, y, mk, -100, ws=ws)
    assert torch.equal(loss, l2)


def test_backward_reuses_forward_compaction():
    """FLCE_FLAG_REUSE_FORWARD: the backward on the forward's workspace skips
    the compaction and gather and gives bit-identical gradients."""
    inp = wl.random_case(seed=14, N=900, D=96, V=5000, dtype="fp16")
    H, W, b, y, mk = to_device(inp)
    ws = binding.Workspace(inp.N, inp.D, inp.V, H.dtype)
    _, m, logs = binding.forward(H, W, b, y, mk, -100, ws=ws)
    fresh = binding.backward(H, W, b, y, mk, -100, m, logs, lam=0.7, ws=ws)
    _, m2, logs2 = binding.forward(H, W, b, y, mk, -100, ws=ws)
    reused = binding.backward(H, W, b, y, mk, -100, m2, logs2, lam=0.7, ws=ws,
                              reuse_forward=True)
    assert binding.device_status(ws) == 0
    for a, c in zip(fresh, reused):
        assert torch.equal(a, c)


def test_lambda_on_device_and_sign():
    inp = wl.random_case(seed=12, N=150, D=48, V=1200)
    H, W, b, y, mk = to_device(inp)
    loss, m, logs = binding.forward(H, W, b, y, mk, -100)
    g1 = binding.backward(H, W, b, y, mk, -100, m, logs, lam=1.0)
    gn = binding.backward(H, W, b, y, mk, -100, m, logs,
                          lam_dev=torch.tensor(-0.5, device="cuda"))
    g0 = binding.backward(H, W, b, y, mk, -100, m, logs, lam=0.0)
    for a, c, z in zip(g1, gn, g0):
        assert torch.equal(c, -0.5 * a)
        assert not z.any()


def test_autograd_wrapper_matches_abi():
    inp = wl.random_case(seed=13, N=100, D=32, V=800)
    H, W, b, y, mk = to_device(inp)
    Hp, Wp, bp = (t.clone().requires_grad_(True) for t in (H, W, b))
    loss = binding.fused_linear_cross_entropy(Hp, Wp, y, b=bp, mask=mk)
    (2.0 * loss).backward()
    _, m, logs = binding.forward(H, W, b, y, mk)
    dH, dW, db = binding.backward(H, W, b, y, mk, -100, m, logs, lam=2.0)
    assert torch.equal(Hp.grad, dH.to(H.dtype)) and torch.equal(Wp.grad, dW.to(W.dtype))
    assert torch.equal(bp.grad, db.to(b.dtype))


# --------------------------------------------------------------------------
# full-size workloads, as the benchmark launches them
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["page2", "packed", "packed_d64", "packed_d128", "packed_d256",
                                  "packed_d512"])
def test_full_size_sampled(name):
    inp = wl.make_inputs(name)
    got = run_gpu(inp)
    assert got["status"] == 0
    sampled_check(inp, got, full_stats=True)


def test_stress_full():
    """Stress (N=32768, D=4096, V=248320, 1 % of rows x50): the loss and m, log s
    of every supervised row from the oracle's full forward, dW of the hottest,
    tail and random ids, dH of sampled rows, and every x50 row on its own
    (the large common shifts of the "分块交叉熵" page, §02 and §06)."""
    inp = wl.make_inputs("stress")
    got = run_gpu(inp)
    assert got["status"] == 0
    idx, _ = orc.supervised_rows(inp.labels, inp.mask)
    big = np.intersect1d(inp.big_rows, idx)
    assert big.size > 100
    sampled_check(inp, got, n_rows=48, full_stats=True, extra_rows=big)


def test_stress_all_ignored():
    inp = wl.make_inputs("stress_c0")
    got = run_gpu(inp)
    assert got["status"] == 0 and got["loss"] == 0.0
    assert np.all(np.isneginf(got["m"]))
    assert not got["dH"].any() and not got["dW"].any()
