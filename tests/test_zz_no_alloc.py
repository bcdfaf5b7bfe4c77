"""The forward entry point that allocates nothing (flce_forward_noalloc).

It serves callers that cannot provide device scratch memory -- a plug-in
inside a framework that owns every device allocation, or a latency-critical
path where cudaMalloc's device-wide synchronisation is not acceptable.  Its
scratch is a fixed buffer compiled into the library.  These tests call it
through the C ABI and compare it with flce_forward() run on a caller-owned
workspace, on two calls in a row (the second call finds the first call's
leftovers in the shared buffer), and both with the binary64 oracle.  This file is collected last so that a run
stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

from lm_head_projection_supervised_b200 import binding
from lm_head_projection_supervised_b200 import workloads as wl

NOALLOC_BYTES = 32 << 20


def _noalloc_fn():
    from lm_head_projection_supervised_b200 import build
    build.build()
    f = binding.lib().flce_forward_noalloc
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, ctypes.c_int, vp, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def test_oversized_problem_is_rejected_before_any_gpu_work():
    """Sizes whose workspace exceeds the fixed buffer get FLCE_ERR_WORKSPACE."""
    f = _noalloc_fn()
    fake = ctypes.c_void_p(0x100000)
    N, D, V = 16384, 1024, 248320   # forward scratch ~275 MiB
    st = f(fake, fake, None, fake, None, -100, N, D, V, 0, fake, fake, fake, None)
    assert binding.STATUS[st] == "FLCE_ERR_WORKSPACE"


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "small", "fp16_bias"])
def test_noalloc_forward_matches_workspace_forward(cuda_device, name):
    import torch
    from _gpu_helpers import check_loss, check_stats, logs_floor, to_device
    from oracle import flce_oracle as orc

    f = _noalloc_fn()
    if name == "fp16_bias":
        inp = wl.random_case(seed=21, N=300, D=72, V=1000, dtype="fp16")
    else:
        inp = wl.make_inputs(name)
    H, W, b, y, mk = to_device(inp)
    ref_loss, ref_m, ref_logs = binding.forward(H, W, b, y, mk, -100)
    ref_m, ref_logs = ref_m.cpu().numpy(), ref_logs.cpu().numpy()
    sup = (inp.labels != -100) & (inp.mask != 0)
    exact = orc.forward(inp.H64(), inp.W64(), inp.b64(), inp.labels, inp.mask)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        loss = torch.full((), float("nan"), dtype=torch.float32, device=cuda_device)
        m = torch.full((inp.N,), float("nan"), dtype=torch.float32, device=cuda_device)
        logs = torch.full((inp.N,), float("nan"), dtype=torch.float32, device=cuda_device)
        st = f(ctypes.c_void_p(H.data_ptr()), ctypes.c_void_p(W.data_ptr()),
               None if b is None else ctypes.c_void_p(b.data_ptr()),
               ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(mk.data_ptr()), -100,
               inp.N, inp.D, inp.V, binding.dtype_code(H.dtype),
               ctypes.c_void_p(loss.data_ptr()), ctypes.c_void_p(m.data_ptr()),
               ctypes.c_void_p(logs.data_ptr()), stream)
        assert st == 0, binding.status_string(st)
        torch.cuda.synchronize()
        check_loss(loss.item(), ref_loss.item(), quantity="loss vs flce_forward")
        gm, gl = m.cpu().numpy(), logs.cpu().numpy()
        check_stats(gm[sup], ref_m[sup], quantity="m vs flce_forward")
        check_stats(gl[sup], ref_logs[sup], floor=logs_floor(ref_m[sup], inp.D),
                    quantity="logs vs flce_forward")
        assert np.all(np.isneginf(gm[~sup])) and np.all(np.isneginf(gl[~sup]))
        # and both against the oracle
        check_loss(loss.item(), exact["loss"], quantity="loss vs oracle")
        check_stats(gm[sup], exact["m"][sup], quantity="m vs oracle")
        check_stats(gl[sup], exact["logs"][sup], floor=logs_floor(exact["m"][sup], inp.D),
                    quantity="logs vs oracle")
