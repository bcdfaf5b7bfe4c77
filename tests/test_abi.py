"""Host-only checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before anything reaches a GPU."""
import ctypes
import os
import re

import pytest

from lm_head_projection_supervised_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("flce.h", "flce_diag.h")]


@pytest.fixture(scope="module")
def L():
    from lm_head_projection_supervised_b200 import build
    build.build()
    return binding.lib()


def declared_symbols():
    names = []
    for h in HEADERS:
        names += re.findall(r"FLCE_API\s+[\w\s\*]+?\b(flce_\w+)\s*\(", open(h).read())
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert "flce_forward" in names and "flce_backward" in names and len(names) >= 8
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code, name in binding.STATUS.items():
        assert binding.status_string(code).startswith(name)


def test_workspace_bytes(L):
    a = L.flce_workspace_bytes(2048, 512, 32000, 0)
    b = L.flce_workspace_bytes(4096, 512, 32000, 0)
    assert 0 < a < b
    assert L.flce_workspace_bytes(-1, 512, 32000, 0) == 0
    assert L.flce_workspace_bytes(16, 4, 10, 0) == 0        # D < 8
    assert L.flce_workspace_bytes(16, 8, 10, 7) == 0        # bad dtype
    # no N x V term: doubling V at fixed N grows the workspace far less than N*V*2 bytes
    big = L.flce_workspace_bytes(16384, 1024, 248320, 0)
    assert big < 16384 * 248320 * 2 // 4


P = ctypes.c_void_p
FAKE = 0x100000  # 256-aligned, never dereferenced: validation fails first


def fwd(L, **kw):
    a = dict(H=FAKE, W=FAKE, b=None, labels=FAKE, mask=None, ig=-100, N=64, D=32, V=1000, dt=0,
             loss=FAKE, m=FAKE, logs=FAKE, ws=FAKE, wsb=1 << 40, s=None)
    a.update(kw)
    return L.flce_forward(P(a["H"]), P(a["W"]), P(a["b"]), P(a["labels"]), P(a["mask"]), a["ig"],
                          a["N"], a["D"], a["V"], a["dt"], P(a["loss"]), P(a["m"]), P(a["logs"]),
                          P(a["ws"]), a["wsb"], P(a["s"]))


def bwd(L, **kw):
    a = dict(H=FAKE, W=FAKE, b=None, labels=FAKE, mask=None, ig=-100, N=64, D=32, V=1000, dt=0,
             m=FAKE, logs=FAKE, lam=1.0, lamd=None, dH=FAKE, dW=FAKE, db=None, ws=FAKE,
             wsb=1 << 40, s=None)
    a.update(kw)
    return L.flce_backward(P(a["H"]), P(a["W"]), P(a["b"]), P(a["labels"]), P(a["mask"]),
                           a["ig"], a["N"], a["D"], a["V"], a["dt"], P(a["m"]), P(a["logs"]),
                           a["lam"], P(a["lamd"]), P(a["dH"]), P(a["dW"]), P(a["db"]), P(a["ws"]),
                           a["wsb"], P(a["s"]))


S = binding.STATUS_CODE


@pytest.mark.parametrize("kw,want", [
    (dict(H=None), "FLCE_ERR_NULL"),
    (dict(ws=None), "FLCE_ERR_NULL"),
    (dict(loss=None), "FLCE_ERR_NULL"),
    (dict(dt=2), "FLCE_ERR_DTYPE"),
    (dict(N=-1), "FLCE_ERR_SHAPE"),
    (dict(V=0), "FLCE_ERR_SHAPE"),
    (dict(D=0), "FLCE_ERR_SHAPE"),
    (dict(D=36), "FLCE_ERR_ALIGN"),
    (dict(H=FAKE + 8), "FLCE_ERR_ALIGN"),
    (dict(ws=FAKE + 128), "FLCE_ERR_ALIGN"),
    (dict(b=FAKE + 2), "FLCE_ERR_ALIGN"),
    (dict(wsb=1024), "FLCE_ERR_WORKSPACE"),
])
def test_forward_argument_errors(L, kw, want):
    assert fwd(L, **kw) == S[want]


@pytest.mark.parametrize("kw,want", [
    (dict(dH=None), "FLCE_ERR_NULL"),
    (dict(m=None), "FLCE_ERR_NULL"),
    (dict(b=FAKE, db=None), "FLCE_ERR_NULL"),
    (dict(dt=-1), "FLCE_ERR_DTYPE"),
    (dict(N=1 << 30), "FLCE_ERR_SHAPE"),
    (dict(dW=FAKE + 4), "FLCE_ERR_ALIGN"),
    (dict(D=12), "FLCE_ERR_ALIGN"),
    (dict(wsb=4096), "FLCE_ERR_WORKSPACE"),
])
def test_backward_argument_errors(L, kw, want):
    assert bwd(L, **kw) == S[want]


def test_valid_call_without_gpu_fails_cleanly(L):
    """With no usable device the call reports a CUDA/device error, no crash."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert fwd(L) in (S["FLCE_ERR_CUDA"], S["FLCE_ERR_DEVICE"])


def test_binding_refuses_cpu_tensors(L):
    import torch
    H = torch.zeros(4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.forward(H, torch.zeros(3, 8, dtype=torch.bfloat16), None,
                        torch.zeros(4, dtype=torch.int64))


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "lm_head_projection_supervised_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f


def fwd_ex(L, **kw):
    a = dict(H=FAKE, W=FAKE, b=None, labels=FAKE, mask=None, ig=-100, N=64, D=32, V=1000, dt=0,
             w=None, red=0, den=0.0, fl=0, loss=FAKE, rows=None, m=FAKE, logs=FAKE, ws=FAKE,
             wsb=1 << 40, s=None)
    a.update(kw)
    return L.flce_forward_ex(P(a["H"]), P(a["W"]), P(a["b"]), P(a["labels"]), P(a["mask"]),
                             a["ig"], a["N"], a["D"], a["V"], a["dt"], P(a["w"]), a["red"],
                             a["den"], a["fl"], P(a["loss"]), P(a["rows"]), P(a["m"]),
                             P(a["logs"]),
                             P(a["ws"]), a["wsb"], P(a["s"]))


def bwd_ex(L, **kw):
    a = dict(H=FAKE, W=FAKE, b=None, labels=FAKE, mask=None, ig=-100, N=64, D=32, V=1000, dt=0,
             m=FAKE, logs=FAKE, w=None, red=0, den=0.0, fl=0, lam=1.0, lamd=None, g=None, dH=FAKE,
             dW=FAKE, db=None, ws=FAKE, wsb=1 << 40, s=None)
    a.update(kw)
    return L.flce_backward_ex(P(a["H"]), P(a["W"]), P(a["b"]), P(a["labels"]), P(a["mask"]),
                              a["ig"], a["N"], a["D"], a["V"], a["dt"], P(a["m"]), P(a["logs"]),
                              P(a["w"]), a["red"], a["den"], a["fl"], a["lam"], P(a["lamd"]),
                              P(a["g"]),
                              P(a["dH"]), P(a["dW"]), P(a["db"]), P(a["ws"]), a["wsb"], P(a["s"]))


@pytest.mark.parametrize("kw,want", [
    (dict(red=3), "FLCE_ERR_ARG"),
    (dict(red=-1), "FLCE_ERR_ARG"),
    (dict(fl=2), "FLCE_ERR_ARG"),                    # dH accumulation: backward-only bit
    (dict(fl=4), "FLCE_ERR_ARG"),                    # reuse of a forward: backward-only bit
    (dict(fl=8), "FLCE_ERR_ARG"),                    # panel backward: backward-only bit
    (dict(red=2, rows=None), "FLCE_ERR_NULL"),       # 'none' needs the per-row output
    (dict(red=1, loss=None), "FLCE_ERR_NULL"),       # 'sum' needs the scalar
    (dict(red=0, w=FAKE + 2), "FLCE_ERR_ALIGN"),
    (dict(red=2, loss=None, rows=FAKE, wsb=512), "FLCE_ERR_WORKSPACE"),
])
def test_forward_ex_argument_errors(L, kw, want):
    assert fwd_ex(L, **kw) == S[want]


@pytest.mark.parametrize("kw,want", [
    (dict(red=7), "FLCE_ERR_ARG"),
    (dict(fl=0x80), "FLCE_ERR_ARG"),
    (dict(red=2, g=None), "FLCE_ERR_NULL"),          # 'none' needs per-row upstream gradients
    (dict(red=1, g=FAKE + 1), "FLCE_ERR_ALIGN"),
    (dict(red=2, g=FAKE, wsb=4096), "FLCE_ERR_WORKSPACE"),
])
def test_backward_ex_argument_errors(L, kw, want):
    assert bwd_ex(L, **kw) == S[want]


def sfwd(L, **kw):
    a = dict(H=FAKE, W=FAKE, b=None, labels=FAKE, mask=None, ig=-100, N=64, D=32, V=1000, v0=0,
             Vt=1000, dt=0, fl=0, st=FAKE, ws=FAKE, wsb=1 << 40, s=None)
    a.update(kw)
    return L.flce_shard_forward(P(a["H"]), P(a["W"]), P(a["b"]), P(a["labels"]), P(a["mask"]),
                                a["ig"], a["N"], a["D"], a["V"], a["v0"], a["Vt"], a["dt"],
                                a["fl"], P(a["st"]), P(a["ws"]), a["wsb"], P(a["s"]))


def scomb(L, **kw):
    a = dict(st=FAKE, Pn=2, labels=FAKE, mask=None, ig=-100, N=64, w=None, red=0, den=0.0,
             loss=FAKE, rows=None, m=FAKE, logs=FAKE, ws=FAKE, wsb=1 << 40, s=None)
    a.update(kw)
    return L.flce_shard_combine(P(a["st"]), a["Pn"], P(a["labels"]), P(a["mask"]), a["ig"],
                                a["N"], P(a["w"]), a["red"], a["den"], P(a["loss"]),
                                P(a["rows"]), P(a["m"]), P(a["logs"]), P(a["ws"]), a["wsb"],
                                P(a["s"]))


def sbwd(L, **kw):
    a = dict(H=FAKE, W=FAKE, b=None, labels=FAKE, mask=None, ig=-100, N=64, D=32, V=1000, v0=0,
             Vt=1000, dt=0, m=FAKE, logs=FAKE, w=None, red=0, den=0.0, fl=0, lam=1.0, lamd=None,
             g=None, dH=FAKE, dW=FAKE, db=None, ws=FAKE, wsb=1 << 40, s=None)
    a.update(kw)
    return L.flce_shard_backward(P(a["H"]), P(a["W"]), P(a["b"]), P(a["labels"]), P(a["mask"]),
                                 a["ig"], a["N"], a["D"], a["V"], a["v0"], a["Vt"], a["dt"],
                                 P(a["m"]), P(a["logs"]), P(a["w"]), a["red"], a["den"], a["fl"],
                                 a["lam"], P(a["lamd"]), P(a["g"]), P(a["dH"]), P(a["dW"]),
                                 P(a["db"]), P(a["ws"]), a["wsb"], P(a["s"]))


@pytest.mark.parametrize("kw,want", [
    (dict(st=None), "FLCE_ERR_NULL"),
    (dict(W=None), "FLCE_ERR_NULL"),
    (dict(v0=-1), "FLCE_ERR_SHAPE"),
    (dict(v0=1, Vt=1000), "FLCE_ERR_SHAPE"),          # slice runs past V_total
    (dict(Vt=(1 << 24) + 1, v0=(1 << 24) - 999), "FLCE_ERR_SHAPE"),
    (dict(st=FAKE + 8), "FLCE_ERR_ALIGN"),            # float4 rows need 16 bytes
    (dict(fl=4), "FLCE_ERR_ARG"),
    (dict(fl=2), "FLCE_ERR_ARG"),                    # dH accumulation: backward-only bit
    (dict(dt=5), "FLCE_ERR_DTYPE"),
    (dict(wsb=2048), "FLCE_ERR_WORKSPACE"),
])
def test_shard_forward_argument_errors(L, kw, want):
    assert sfwd(L, **kw) == S[want]


@pytest.mark.parametrize("kw,want", [
    (dict(st=None), "FLCE_ERR_NULL"),
    (dict(m=None), "FLCE_ERR_NULL"),
    (dict(red=2, rows=None), "FLCE_ERR_NULL"),
    (dict(red=4), "FLCE_ERR_ARG"),
    (dict(Pn=0), "FLCE_ERR_SHAPE"),
    (dict(N=-3), "FLCE_ERR_SHAPE"),
    (dict(st=FAKE + 4), "FLCE_ERR_ALIGN"),
    (dict(wsb=256), "FLCE_ERR_WORKSPACE"),
])
def test_shard_combine_argument_errors(L, kw, want):
    assert scomb(L, **kw) == S[want]


@pytest.mark.parametrize("kw,want", [
    (dict(dW=None), "FLCE_ERR_NULL"),
    (dict(b=FAKE, db=None), "FLCE_ERR_NULL"),
    (dict(v0=4, Vt=1004, wsb=4096), "FLCE_ERR_WORKSPACE"),
    (dict(v0=10, Vt=1004), "FLCE_ERR_SHAPE"),
    (dict(fl=16), "FLCE_ERR_ARG"),
])
def test_shard_backward_argument_errors(L, kw, want):
    assert sbwd(L, **kw) == S[want]


def test_workspace_holds_the_fused_backward_partials(L):
    """D <= 64: the workspace carries the single-kernel backward's partial
    sums (8 dW slabs of V rows, 160 dH slabs of N rows), sharing space with the
    panel buffers; at the packed shape that is about a sixth of one 16-bit
    copy of the N x V logits."""
    N, V = 16384, 248320
    Vp, Np = (V + 127) // 128 * 128, (N + 255) // 256 * 256
    for D in (8, 40, 64):
        ws = L.flce_workspace_bytes(N, D, V, 0)
        assert ws >= (8 * Vp + 160 * Np) * D * 4
        assert ws < N * V * 2 / 5
    # D > 64 has no partials
    d72 = L.flce_workspace_bytes(N, 72, V, 0)
    assert d72 < (8 * Vp + 160 * Np) * 72 * 4


def test_shard_combine_workspace_bytes(L):
    assert L.flce_shard_combine_workspace_bytes(-1) == 0
    a = L.flce_shard_combine_workspace_bytes(1000)
    assert a >= 2 * 1000 * 4 and a < L.flce_shard_combine_workspace_bytes(100000)


def test_mask_conversion_keeps_every_nonzero_entry():
    """Any nonzero mask value means "takes part", also for integer masks whose
    values do not fit in a byte (a plain uint8 cast would wrap 256 to 0)."""
    import torch
    from lm_head_projection_supervised_b200.binding import _mask_u8
    m = _mask_u8(torch.tensor([0, 1, 256, -3, 7]))
    assert m.dtype == torch.uint8 and m.tolist() == [0, 1, 1, 1, 1]
    assert _mask_u8(torch.tensor([True, False])).tolist() == [1, 0]
    assert _mask_u8(None) is None
