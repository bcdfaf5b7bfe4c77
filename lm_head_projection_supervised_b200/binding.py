"""ctypes binding of libflce.so.

Argument marshalling only: every step of the loss runs in the library's CUDA
kernels.  torch provides device memory (inputs, outputs, workspace) and the
current stream.  There is no fallback: when the library is missing or the
device is not sm_100, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libflce.so")

FLCE_BF16, FLCE_FP16 = 0, 1
STATUS = {0: "FLCE_OK", 1: "FLCE_ERR_NULL", 2: "FLCE_ERR_SHAPE", 3: "FLCE_ERR_DTYPE",
          4: "FLCE_ERR_ALIGN", 5: "FLCE_ERR_WORKSPACE", 6: "FLCE_ERR_CUDA", 7: "FLCE_ERR_LABEL",
          8: "FLCE_ERR_TIMEOUT", 9: "FLCE_ERR_NONFINITE", 10: "FLCE_ERR_DEVICE",
          11: "FLCE_ERR_ARG", 12: "FLCE_ERR_SHARD"}
REDUCTIONS = {"mean": 0, "sum": 1, "none": 2}
FLAG_ROUND_LOGITS = 1
FLAG_ACCUMULATE_DH = 2
FLAG_REUSE_FORWARD = 4
FLAG_PANEL_BACKWARD = 8
STATUS_CODE = {v: k for k, v in STATUS.items()}

_lib = None


class FlceError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}" if where else status_string(status))


def lib() -> ctypes.CDLL:
    """Load libflce.so (built in-tree); raises if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built: run "
                           "`python -m lm_head_projection_supervised_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, \
        ctypes.c_float
    L.flce_workspace_bytes.argtypes = [i64, i64, i64, i32]
    L.flce_workspace_bytes.restype = sz
    L.flce_status_string.argtypes = [i32]
    L.flce_status_string.restype = ctypes.c_char_p
    L.flce_compact.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, sz, vp]
    L.flce_compact.restype = i32
    L.flce_forward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, vp, vp, vp, vp, sz,
                               vp]
    L.flce_forward.restype = i32
    L.flce_backward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, vp, vp, f32, vp, vp,
                                vp, vp, vp, sz, vp]
    L.flce_backward.restype = i32
    u32 = ctypes.c_uint
    L.flce_forward_ex.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, vp, i32, f32, u32,
                                  vp, vp, vp, vp, vp, sz, vp]
    L.flce_forward_ex.restype = i32
    L.flce_backward_ex.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, vp, vp, vp, i32,
                                   f32, u32, f32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.flce_backward_ex.restype = i32
    L.flce_backward_filtered.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, vp, vp, vp,
                                         i32, f32, u32, f32, vp, vp, f32, vp, vp, vp, vp, sz, vp]
    L.flce_backward_filtered.restype = i32
    L.flce_shard_forward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i32, u32,
                                     vp, vp, sz, vp]
    L.flce_shard_forward.restype = i32
    L.flce_shard_combine_workspace_bytes.argtypes = [i64]
    L.flce_shard_combine_workspace_bytes.restype = sz
    L.flce_shard_combine.argtypes = [vp, i32, vp, vp, i64, i64, vp, i32, f32, vp, vp, vp, vp, vp,
                                     sz, vp]
    L.flce_shard_combine.restype = i32
    L.flce_shard_backward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i32, vp,
                                      vp, vp, i32, f32, u32, f32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.flce_shard_backward.restype = i32
    L.flce_device_status.argtypes = [vp, vp]
    L.flce_device_status.restype = i32
    L.flce_diag_gemm.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, i32, f32, vp, sz, vp]
    L.flce_diag_gemm.restype = i32
    L.flce_diag_exp2.argtypes = [vp, vp, vp, i64, vp]
    L.flce_diag_exp2.restype = i32
    L.flce_diag_timeout.argtypes = [vp, sz, ctypes.c_uint64, vp]
    L.flce_diag_timeout.restype = i32
    L.flce_diag_profile_begin.argtypes = []
    L.flce_diag_profile_begin.restype = i32
    L.flce_diag_profile_end.argtypes = [ctypes.POINTER(ctypes.c_double),
                                        ctypes.POINTER(ctypes.c_int64), i32]
    L.flce_diag_profile_end.restype = i32
    _lib = L
    return L


def status_string(status: int) -> str:
    try:
        return lib().flce_status_string(int(status)).decode()
    except RuntimeError:
        return STATUS.get(int(status), f"status {status}")


def _check(status: int, where: str):
    if status != 0:
        raise FlceError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return FLCE_BF16
    if dt == torch.float16:
        return FLCE_FP16
    raise TypeError(f"H and W must be bfloat16 or float16, got {dt}")


def workspace_bytes(N: int, D: int, V: int, dtype: torch.dtype = torch.bfloat16) -> int:
    return int(lib().flce_workspace_bytes(N, D, V, dtype_code(dtype)))


class Workspace:
    """Caller-owned device scratch of flce_workspace_bytes() bytes."""

    def __init__(self, N: int, D: int, V: int, dtype: torch.dtype, device=None):
        n = workspace_bytes(N, D, V, dtype)
        if n == 0:
            raise FlceError(STATUS_CODE["FLCE_ERR_SHAPE"], "workspace_bytes")
        self.nbytes = n
        self.buf = torch.empty(n, dtype=torch.uint8, device=device or "cuda")

    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


def _prep(H, W, b, labels, mask):
    if not (H.is_cuda and W.is_cuda and labels.is_cuda):
        raise ValueError("H, W and labels must be CUDA tensors")
    if H.dtype != W.dtype or (b is not None and b.dtype != H.dtype):
        raise TypeError("H, W and b must share one dtype")
    D = H.shape[-1]
    H2 = H.reshape(-1, D)
    if not H2.is_contiguous():
        H2 = H2.contiguous()
    if W.dim() != 2 or W.shape[1] != D:
        raise ValueError(f"W must be [V, {D}]")
    W2 = W if W.is_contiguous() else W.contiguous()
    y = labels.reshape(-1)
    if y.dtype != torch.int64:
        y = y.to(torch.int64)
    if y.numel() != H2.shape[0]:
        raise ValueError("labels must have one entry per row of H")
    y = y.contiguous()
    b2 = None if b is None else b.contiguous()
    if b2 is not None and b2.data_ptr() % 16:
        b2 = b2.clone()  # a vocabulary slice of a bias can start off the 16-byte grid
    return H2, W2, b2, y, _mask_u8(mask)


def _mask_u8(mask):
    """uint8 contiguous [N] view of a mask (nonzero = takes part), or None."""
    if mask is None:
        return None
    mk = mask.reshape(-1)
    if mk.dtype == torch.bool:
        mk = mk.view(torch.uint8)
    elif mk.dtype != torch.uint8:
        mk = (mk != 0).view(torch.uint8)
    return mk.contiguous()


def _flags(round_logits=False, accumulate_dh=False, reuse_forward=False,
           panel_backward=False) -> int:
    return (FLAG_ROUND_LOGITS if round_logits else 0) | \
        (FLAG_ACCUMULATE_DH if accumulate_dh else 0) | \
        (FLAG_REUSE_FORWARD if reuse_forward else 0) | \
        (FLAG_PANEL_BACKWARD if panel_backward else 0)


def _vec(t, N, device):
    """float32 contiguous [N] device vector (or None)."""
    if t is None:
        return None
    t = t.reshape(-1).to(device=device, dtype=torch.float32).contiguous()
    if t.numel() != N:
        raise ValueError("per-row vectors must have one entry per row of H")
    return t


def forward(H, W, b, labels, mask=None, ignore_index: int = -100, ws: Optional[Workspace] = None,
            stream=None, weight=None, reduction: str = "mean", denom: Optional[float] = None,
            round_logits: bool = False):
    """(loss, m [N], logs [N]) -- flce_forward_ex().

    loss is a 0-d float32 for "mean" and "sum", and the per-row losses [N] for
    "none"; weight ([N], optional) multiplies each row's loss; denom divides
    the "sum" (e.g. a global label count); round_logits rounds each logit to
    the input dtype before the loss."""
    H2, W2, b2, y, mk = _prep(H, W, b, labels, mask)
    N, D = H2.shape
    V = W2.shape[0]
    red = REDUCTIONS[reduction]
    if ws is None:
        ws = Workspace(N, D, V, H2.dtype, H2.device)
    wt = _vec(weight, N, H2.device)
    loss = torch.empty((), dtype=torch.float32, device=H2.device)
    rows = torch.empty(N, dtype=torch.float32, device=H2.device) if reduction == "none" else None
    m = torch.empty(N, dtype=torch.float32, device=H2.device)
    logs = torch.empty(N, dtype=torch.float32, device=H2.device)
    st = lib().flce_forward_ex(_ptr(H2), _ptr(W2), _ptr(b2), _ptr(y), _ptr(mk), ignore_index, N,
                               D, V, dtype_code(H2.dtype), _ptr(wt), red,
                               float(denom or 0.0), FLAG_ROUND_LOGITS if round_logits else 0,
                               _ptr(loss), _ptr(rows), _ptr(m), _ptr(logs),
                               ws.ptr(), ws.nbytes, _stream(stream))
    _check(st, "flce_forward_ex")
    return (rows if reduction == "none" else loss), m, logs


def backward(H, W, b, labels, mask, ignore_index: int, m, logs, lam: float = 1.0, lam_dev=None,
             ws: Optional[Workspace] = None, out=None, stream=None, weight=None,
             reduction: str = "mean", denom: Optional[float] = None, grad_rows=None,
             round_logits: bool = False, accumulate_dh: bool = False,
             reuse_forward: bool = False, filter_eps: float = 0.0, panel_backward: bool = False):
    """dH [N, D], dW [V, D], db [V] or None (float32) -- flce_backward_ex(), or
    flce_backward_filtered() when filter_eps > 0 (gradient filtering: 128-row x
    64-id blocks whose |p - onehot| are all below filter_eps are left out of
    dH and dW; an approximation).

    For reduction "none", grad_rows [N] is the upstream gradient of each row's
    loss; otherwise lam (or the device scalar lam_dev) is dJ/dL.  With
    accumulate_dh the call adds its dH to out[0] instead of overwriting it.
    reuse_forward: `ws` holds the compaction of a forward() on the same
    inputs, untouched since; the backward skips redoing it.  panel_backward:
    the panel form of the backward even where the single-kernel form applies
    (D <= 64)."""
    H2, W2, b2, y, mk = _prep(H, W, b, labels, mask)
    N, D = H2.shape
    V = W2.shape[0]
    red = REDUCTIONS[reduction]
    if ws is None:
        ws = Workspace(N, D, V, H2.dtype, H2.device)
    if out is None:
        dH = torch.empty((N, D), dtype=torch.float32, device=H2.device)
        dW = torch.empty((V, D), dtype=torch.float32, device=H2.device)
        db = None if b2 is None else torch.empty(V, dtype=torch.float32, device=H2.device)
    else:
        dH, dW, db = out
    if lam_dev is not None:
        lam_dev = lam_dev.reshape(()).to(torch.float32).contiguous()
    wt = _vec(weight, N, H2.device)
    gr = _vec(grad_rows, N, H2.device)
    common = (_ptr(H2), _ptr(W2), _ptr(b2), _ptr(y), _ptr(mk), ignore_index, N, D, V,
              dtype_code(H2.dtype), _ptr(m), _ptr(logs), _ptr(wt), red, float(denom or 0.0),
              _flags(round_logits, accumulate_dh, reuse_forward, panel_backward), float(lam),
              _ptr(lam_dev),
              _ptr(gr))
    tail = (_ptr(dH), _ptr(dW), _ptr(db), ws.ptr(), ws.nbytes, _stream(stream))
    if filter_eps:
        st = lib().flce_backward_filtered(*common, float(filter_eps), *tail)
        _check(st, "flce_backward_filtered")
    else:
        st = lib().flce_backward_ex(*common, *tail)
        _check(st, "flce_backward_ex")
    return dH, dW, db


class CombineWorkspace:
    """Device scratch of flce_shard_combine_workspace_bytes(N) bytes."""

    def __init__(self, N: int, device=None):
        n = int(lib().flce_shard_combine_workspace_bytes(N))
        if n == 0:
            raise FlceError(STATUS_CODE["FLCE_ERR_SHAPE"], "shard_combine_workspace_bytes")
        self.nbytes = n
        self.buf = torch.empty(n, dtype=torch.uint8, device=device or "cuda")

    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


def shard_forward(H, W_slice, b_slice, labels, mask=None, ignore_index: int = -100, v0: int = 0,
                  V_total: Optional[int] = None, ws: Optional[Workspace] = None, stream=None,
                  round_logits: bool = False, out=None):
    """Per-row partial statistics [N, 4] float32 (m_r, log s_r, t_r, o_r) of
    the vocabulary slice [v0, v0 + V_slice) -- flce_shard_forward().  out: an
    optional contiguous float32 [N, 4] device tensor to write them to."""
    H2, W2, b2, y, mk = _prep(H, W_slice, b_slice, labels, mask)
    N, D = H2.shape
    Vs = W2.shape[0]
    V_total = v0 + Vs if V_total is None else int(V_total)
    if ws is None:
        ws = Workspace(N, D, Vs, H2.dtype, H2.device)
    stats = torch.empty((N, 4), dtype=torch.float32, device=H2.device) if out is None else out
    if stats.shape != (N, 4) or stats.dtype != torch.float32 or not stats.is_contiguous():
        raise ValueError("out must be a contiguous float32 [N, 4] tensor")
    st = lib().flce_shard_forward(_ptr(H2), _ptr(W2), _ptr(b2), _ptr(y), _ptr(mk), ignore_index,
                                  N, D, Vs, int(v0), V_total, dtype_code(H2.dtype),
                                  FLAG_ROUND_LOGITS if round_logits else 0, _ptr(stats),
                                  ws.ptr(), ws.nbytes, _stream(stream))
    _check(st, "flce_shard_forward")
    return stats


def shard_combine(stats_all, labels, mask=None, ignore_index: int = -100, weight=None,
                  reduction: str = "mean", denom: Optional[float] = None,
                  ws: Optional[CombineWorkspace] = None, stream=None):
    """(loss, m [N], logs [N]) of the full vocabulary from the slices' stats
    stacked as [P, N, 4] -- flce_shard_combine().  loss as in forward()."""
    if not (stats_all.is_cuda and labels.is_cuda):
        raise ValueError("stats and labels must be CUDA tensors")
    if stats_all.dim() != 3 or stats_all.shape[2] != 4 or stats_all.dtype != torch.float32:
        raise ValueError("stats_all must be float32 [P, N, 4]")
    P, N = int(stats_all.shape[0]), int(stats_all.shape[1])
    st_all = stats_all.contiguous()
    y = labels.reshape(-1).to(torch.int64).contiguous()
    if y.numel() != N:
        raise ValueError("labels must have one entry per row")
    mk = _mask_u8(mask)
    dev = st_all.device
    if ws is None:
        ws = CombineWorkspace(N, dev)
    wt = _vec(weight, N, dev)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    rows = torch.empty(N, dtype=torch.float32, device=dev) if reduction == "none" else None
    m = torch.empty(N, dtype=torch.float32, device=dev)
    logs = torch.empty(N, dtype=torch.float32, device=dev)
    st = lib().flce_shard_combine(_ptr(st_all), P, _ptr(y), _ptr(mk), ignore_index, N, _ptr(wt),
                                  REDUCTIONS[reduction], float(denom or 0.0), _ptr(loss),
                                  _ptr(rows), _ptr(m), _ptr(logs), ws.ptr(), ws.nbytes,
                                  _stream(stream))
    _check(st, "flce_shard_combine")
    return (rows if reduction == "none" else loss), m, logs


def shard_backward(H, W_slice, b_slice, labels, mask, ignore_index: int, m, logs, v0: int = 0,
                   V_total: Optional[int] = None, lam: float = 1.0, lam_dev=None,
                   ws: Optional[Workspace] = None, out=None, stream=None, weight=None,
                   reduction: str = "mean", denom: Optional[float] = None, grad_rows=None,
                   round_logits: bool = False, accumulate_dh: bool = False,
                   panel_backward: bool = False):
    """(dH_r [N, D], dW_slice [V_slice, D], db_slice [V_slice] or None),
    float32 -- flce_shard_backward().  dH_r is this slice's term of dH (added
    to out[0] with accumulate_dh)."""
    H2, W2, b2, y, mk = _prep(H, W_slice, b_slice, labels, mask)
    N, D = H2.shape
    Vs = W2.shape[0]
    V_total = v0 + Vs if V_total is None else int(V_total)
    if ws is None:
        ws = Workspace(N, D, Vs, H2.dtype, H2.device)
    if out is None:
        dH = torch.empty((N, D), dtype=torch.float32, device=H2.device)
        dW = torch.empty((Vs, D), dtype=torch.float32, device=H2.device)
        db = None if b2 is None else torch.empty(Vs, dtype=torch.float32, device=H2.device)
    else:
        dH, dW, db = out
    if lam_dev is not None:
        lam_dev = lam_dev.reshape(()).to(torch.float32).contiguous()
    wt = _vec(weight, N, H2.device)
    gr = _vec(grad_rows, N, H2.device)
    st = lib().flce_shard_backward(_ptr(H2), _ptr(W2), _ptr(b2), _ptr(y), _ptr(mk), ignore_index,
                                   N, D, Vs, int(v0), V_total, dtype_code(H2.dtype), _ptr(m),
                                   _ptr(logs), _ptr(wt), REDUCTIONS[reduction],
                                   float(denom or 0.0),
                                   _flags(round_logits, accumulate_dh,
                                          panel_backward=panel_backward),
                                   float(lam), _ptr(lam_dev), _ptr(gr), _ptr(dH), _ptr(dW),
                                   _ptr(db), ws.ptr(), ws.nbytes, _stream(stream))
    _check(st, "flce_shard_backward")
    return dH, dW, db


def device_status(ws: Workspace, stream=None) -> int:
    return int(lib().flce_device_status(ws.ptr(), _stream(stream)))


def compact(labels, mask, ignore_index: int, V: int, stream=None):
    """idx (int32, first C valid) and C (int32 device scalar) -- flce_compact()."""
    y = labels.reshape(-1).to(torch.int64).contiguous()
    mk = _mask_u8(mask)
    N = y.numel()
    idx = torch.empty(max(N, 1), dtype=torch.int32, device=y.device)
    C = torch.empty((), dtype=torch.int32, device=y.device)
    ws = torch.empty(256, dtype=torch.uint8, device=y.device)
    st = lib().flce_compact(_ptr(y), _ptr(mk), ignore_index, N, V, _ptr(idx), _ptr(C),
                            _ptr(ws), 256, _stream(stream))
    _check(st, "flce_compact")
    return idx, C, ws


def diag_gemm(A, B, M: int, N: int, K: int, a_mn: bool, b_mn: bool, scale: float = 1.0,
              stream=None):
    out = torch.empty((M, N), dtype=torch.float32, device=A.device)
    ws = torch.zeros(256, dtype=torch.uint8, device=A.device)
    st = lib().flce_diag_gemm(_ptr(A), _ptr(B), _ptr(out), M, N, K, dtype_code(A.dtype),
                              int(a_mn), int(b_mn), float(scale), _ptr(ws), 256, _stream(stream))
    _check(st, "flce_diag_gemm")
    s2 = lib().flce_device_status(_ptr(ws), _stream(stream))
    _check(s2, "flce_diag_gemm (device)")
    return out


def diag_exp2(x: torch.Tensor, stream=None):
    """(ex2_poly(x), ex2.approx(x)) element-wise, float32 -- flce_diag_exp2()."""
    x = x.to(torch.float32).contiguous()
    yp, ys = torch.empty_like(x), torch.empty_like(x)
    _check(lib().flce_diag_exp2(_ptr(x), _ptr(yp), _ptr(ys), x.numel(), _stream(stream)),
           "flce_diag_exp2")
    return yp, ys


def diag_timeout(limit_ns: int, device="cuda", stream=None) -> int:
    ws = torch.zeros(256, dtype=torch.uint8, device=device)
    _check(lib().flce_diag_timeout(_ptr(ws), 256, int(limit_ns), _stream(stream)),
           "flce_diag_timeout")
    return int(lib().flce_device_status(_ptr(ws), _stream(stream)))


PROFILE_KINDS = ("fwd_gemm", "bwd_gemm", "plain_gemm", "aux")


def profile_begin():
    _check(lib().flce_diag_profile_begin(), "flce_diag_profile_begin")


def profile_end():
    """Per kernel kind: (total ms, launches) recorded since profile_begin()."""
    ms = (ctypes.c_double * 4)()
    n = (ctypes.c_int64 * 4)()
    _check(lib().flce_diag_profile_end(ms, n, 4), "flce_diag_profile_end")
    return {k: (ms[i], int(n[i])) for i, k in enumerate(PROFILE_KINDS)}


class FusedLinearCrossEntropy(torch.autograd.Function):
    """L = reduce_i w_i CE(H W^T + b, y)_i over the supervised rows; gradients
    from the library's backward, with the upstream gradient kept on the
    device (no host round trip).  One workspace serves both passes: the
    forward's compaction and gathered rows are kept in it for the backward."""

    @staticmethod
    def forward(ctx, H, W, b, labels, mask, ignore_index, weight=None, reduction="mean",
                denom=None, round_logits=False):
        H2 = H.reshape(-1, H.shape[-1])
        ws = Workspace(H2.shape[0], H2.shape[1], W.shape[0], H.dtype, H.device)
        loss, m, logs = forward(H, W, b, labels, mask, ignore_index, ws=ws, weight=weight,
                                reduction=reduction, denom=denom, round_logits=round_logits)
        ctx.save_for_backward(H, W, b, labels, mask, m, logs, weight)
        ctx.ignore_index, ctx.reduction, ctx.denom = ignore_index, reduction, denom
        ctx.round_logits = round_logits
        ctx.ws = ws
        return loss

    @staticmethod
    def backward(ctx, grad_out):
        H, W, b, labels, mask, m, logs, weight = ctx.saved_tensors
        ws, ctx.ws = ctx.ws, None
        g = grad_out.detach()
        common = dict(weight=weight, round_logits=ctx.round_logits, ws=ws, reuse_forward=True)
        if ctx.reduction == "none":
            dH, dW, db = backward(H, W, b, labels, mask, ctx.ignore_index, m, logs,
                                  reduction="none", grad_rows=g, **common)
        else:
            dH, dW, db = backward(H, W, b, labels, mask, ctx.ignore_index, m, logs, lam_dev=g,
                                  reduction=ctx.reduction, denom=ctx.denom, **common)
        return (dH.reshape(H.shape).to(H.dtype), dW.to(W.dtype),
                None if db is None else db.to(b.dtype), None, None, None, None, None, None, None)


def fused_linear_cross_entropy(H, W, labels, b=None, mask=None, ignore_index: int = -100,
                               weight=None, reduction: str = "mean", denom=None,
                               round_logits: bool = False):
    return FusedLinearCrossEntropy.apply(H, W, b, labels, mask, ignore_index, weight, reduction,
                                         denom, round_logits)


class LinearCrossEntropyLoss(torch.nn.Module):
    """Loss module over final hidden states and the projection weight, with
    the reductions of a chunked linear cross-entropy loss ("mean", "sum",
    "none"), an optional global label count for "sum" and optional per-token
    loss weights.  Hidden states may have any leading token dimensions.
    round_logits rounds the logits to the input dtype before the loss (a
    projection that outputs the model dtype)."""

    def __init__(self, ignore_index: int = -100, reduction: str = "mean",
                 round_logits: bool = False):
        super().__init__()
        if reduction not in REDUCTIONS:
            raise ValueError(f"reduction must be one of {tuple(REDUCTIONS)}")
        self.ignore_index = ignore_index
        self.reduction = reduction
        self.round_logits = round_logits

    def forward(self, hidden_states, labels, lm_weight, bias=None, num_label_tokens=None,
                loss_weights=None, mask=None):
        lead = hidden_states.shape[:-1]
        out = fused_linear_cross_entropy(hidden_states, lm_weight, labels, b=bias, mask=mask,
                                         ignore_index=self.ignore_index, weight=loss_weights,
                                         reduction=self.reduction, denom=num_label_tokens,
                                         round_logits=self.round_logits)
        return out.reshape(lead) if self.reduction == "none" else out
