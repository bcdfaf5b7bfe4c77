"""Seeded synthetic inputs for exact fused linear cross-entropy.

This module only draws random numbers and rounds them to the 16-bit input
dtype.  It holds none of the loss arithmetic: both the CUDA path and the CPU
oracle take their inputs from here, and nothing here depends on either.

Workloads follow the shapes and value distributions of the pages
("分块交叉熵 / Output projection / exact cross entropy", §01 problem statement:
H in R^{NxD}, W in R^{VxD}, optional b in R^V, labels with ignore = -100 and a
boolean mask) and of the long-sequence training story of
"ChunkedLinearCrossEntropy (Qwen3.5 training memory peak)" (16k packed rows,
vocabulary 248320).  No dataset or trained weights are involved.

Arrays are returned as numpy arrays.  16-bit tensors are returned as their raw
bit patterns (``uint16``) so that the same bits can be handed to the GPU and
upcast exactly to float64 for the oracle.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

IGNORE_INDEX = -100
SEED_BASE = 20261202


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    name: str
    k: int                      # seed offset
    N: int
    D: int
    V: int
    dtype: str                  # "bf16" | "fp16"
    w_std: float
    h_scale: float = 1.0
    bias_std: Optional[float] = None
    label_dist: str = "uniform"  # "uniform" | "zipf"
    zipf_s: float = 1.1
    # supervision layout
    segments: int = 0           # >0: N split into equal segments, prefix of each ignored
    prefix_frac: float = 0.0    # fraction of each segment ignored (rounded half-up)
    ignore_frac: float = 0.0    # exact count round(frac*N) chosen by permutation
    mask_false_frac: float = 0.0
    all_ignored: bool = False
    big_row_frac: float = 0.0   # rows scaled by big_row_scale before rounding
    big_row_scale: float = 1.0
    lam: float = 1.0
    # peaked logits (0 = off): each hidden row gets the direction of its label's
    # weight row scaled so that the label's logit is about `peak_logit`, and of
    # `n_comp` competitor ids (Zipf-distributed, frequent ids first) with logits
    # drawn uniformly from `comp_logits`; h_scale then sets the noise level
    peak_logit: float = 0.0
    n_comp: int = 0
    comp_logits: tuple = (0.0, 0.0)


SPECS = {
    "tiny": WorkloadSpec("tiny", 0, N=64, D=32, V=1000, dtype="bf16", w_std=0.1,
                         bias_std=0.1, ignore_frac=0.25),
    "small": WorkloadSpec("small", 1, N=2048, D=512, V=32000, dtype="bf16", w_std=0.02,
                          segments=4, prefix_frac=0.4),
    "page2": WorkloadSpec("page2", 2, N=8192, D=2048, V=131072, dtype="fp16", w_std=0.02,
                          bias_std=0.01, ignore_frac=0.10, mask_false_frac=0.05, lam=0.5),
    "packed": WorkloadSpec("packed", 3, N=16384, D=1024, V=248320, dtype="bf16", w_std=0.02,
                           label_dist="zipf", segments=8, prefix_frac=0.3),
    # the packed recipe at the two smaller hidden sizes the method is compared on
    # (w_std scaled by sqrt(1024 / D) so that the logits keep the same spread)
    "packed_d256": WorkloadSpec("packed_d256", 5, N=16384, D=256, V=248320, dtype="bf16",
                                w_std=0.04, label_dist="zipf", segments=8, prefix_frac=0.3),
    "packed_d512": WorkloadSpec("packed_d512", 6, N=16384, D=512, V=248320, dtype="bf16",
                                w_std=0.02 * 2 ** 0.5, label_dist="zipf", segments=8,
                                prefix_frac=0.3),
    "packed_d128": WorkloadSpec("packed_d128", 8, N=16384, D=128, V=248320, dtype="bf16",
                                w_std=0.02 * 8 ** 0.5, label_dist="zipf", segments=8,
                                prefix_frac=0.3),
    "packed_d64": WorkloadSpec("packed_d64", 9, N=16384, D=64, V=248320, dtype="bf16",
                               w_std=0.08, label_dist="zipf", segments=8, prefix_frac=0.3),
    # the packed recipe with a few dominant logits per row (a trained model's
    # shape of softmax), for the opt-in gradient filtering
    "peaked": WorkloadSpec("peaked", 7, N=16384, D=1024, V=248320, dtype="bf16", w_std=0.02,
                           h_scale=0.5, label_dist="zipf", segments=8, prefix_frac=0.3,
                           peak_logit=16.0, n_comp=8, comp_logits=(6.0, 12.0)),
    "stress": WorkloadSpec("stress", 4, N=32768, D=4096, V=248320, dtype="bf16", w_std=0.02,
                           h_scale=4.0, big_row_frac=0.01, big_row_scale=50.0,
                           ignore_frac=0.5),
    "stress_c0": WorkloadSpec("stress_c0", 4, N=32768, D=4096, V=248320, dtype="bf16",
                              w_std=0.02, h_scale=4.0, big_row_frac=0.01,
                              big_row_scale=50.0, all_ignored=True),
}


def round_half_up(x: float) -> int:
    return int(np.floor(x + 0.5))


# ---------------------------------------------------------------------------
# 16-bit encodings (round to nearest even), and exact decodings
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round to nearest even.  In 32-bit arithmetic: for finite inputs the
    sum stays below 2^32 (the draws here are always finite)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_fp16_bits(x: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def fp16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return bits.view(np.float16).astype(np.float32)


def encode(x: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x) if dtype == "bf16" else f32_to_fp16_bits(x)


def decode_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    f = bf16_bits_to_f32(bits) if dtype == "bf16" else fp16_bits_to_f32(bits)
    return f.astype(np.float64)


# ---------------------------------------------------------------------------
# Inputs
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Inputs:
    spec: WorkloadSpec
    H: np.ndarray                 # uint16 bits [N, D]
    W: np.ndarray                 # uint16 bits [V, D]
    b: Optional[np.ndarray]       # uint16 bits [V] or None
    labels: np.ndarray            # int64 [N]
    mask: np.ndarray              # uint8 [N] (1 = supervised position)
    ignore_index: int = IGNORE_INDEX
    big_rows: Optional[np.ndarray] = None  # rows scaled by big_row_scale (ascending), if any

    @property
    def N(self):
        return self.H.shape[0]

    @property
    def D(self):
        return self.H.shape[1]

    @property
    def V(self):
        return self.W.shape[0]

    @property
    def dtype(self):
        return self.spec.dtype

    @property
    def lam(self):
        return self.spec.lam

    def H64(self):
        return decode_f64(self.H, self.dtype)

    def W64(self):
        return decode_f64(self.W, self.dtype)

    def b64(self):
        return None if self.b is None else decode_f64(self.b, self.dtype)


def _normal_bits(rng: np.random.Generator, shape, std: float, dtype: str,
                 row_scale: Optional[np.ndarray] = None, chunk_rows: int = 8192):
    """N(0, std) draws in float32, optionally scaled per row, rounded to 16 bits.

    Drawn in row chunks so that the float32 staging buffer stays small.
    """
    rows, cols = shape if len(shape) == 2 else (shape[0], 1)
    out = np.empty((rows, cols), dtype=np.uint16)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
        x *= np.float32(std)
        if row_scale is not None:
            x *= row_scale[r0:r1, None].astype(np.float32)
        out[r0:r1] = encode(x, dtype)
    return out.reshape(shape)


def _zipf_labels(rng: np.random.Generator, n: int, V: int, s: float) -> np.ndarray:
    """P(id = k) proportional to (k+1)^-s on [0, V); inverse CDF on the table."""
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    return np.minimum(np.searchsorted(cdf, u, side="right"), V - 1).astype(np.int64)


def _peaked_hidden(rng: np.random.Generator, H_bits: np.ndarray, W_bits: np.ndarray,
                   labels: np.ndarray, spec: "WorkloadSpec", chunk_rows: int = 2048):
    """Adds to each (noise) hidden row a / |w|^2 times the weight row w of its
    label (a = peak_logit) and of n_comp Zipf-drawn competitor ids (a drawn
    from comp_logits), so that those logits sit near a; re-rounded to 16 bits."""
    N, D = H_bits.shape
    V = W_bits.shape[0]
    comp = _zipf_labels(rng, N * spec.n_comp, V, spec.zipf_s).reshape(N, spec.n_comp)
    lo, hi = spec.comp_logits
    amp = rng.uniform(lo, hi, size=(N, spec.n_comp))
    out = np.empty_like(H_bits)
    for r0 in range(0, N, chunk_rows):
        r1 = min(N, r0 + chunk_rows)
        h = decode_f64(H_bits[r0:r1], spec.dtype).astype(np.float32)
        ids = np.concatenate([labels[r0:r1, None], comp[r0:r1]], axis=1)
        a = np.concatenate([np.full((r1 - r0, 1), spec.peak_logit), amp[r0:r1]], axis=1)
        w = decode_f64(W_bits[ids.reshape(-1)], spec.dtype).astype(np.float32)
        w = w.reshape(r1 - r0, ids.shape[1], D)
        coef = (a / np.maximum((w.astype(np.float64) ** 2).sum(axis=2), 1e-30)).astype(np.float32)
        h += np.einsum("rk,rkd->rd", coef, w)
        out[r0:r1] = encode(h, spec.dtype)
    return out


def make_inputs(name_or_spec, seed: Optional[int] = None, **overrides) -> Inputs:
    """Build the seeded inputs of a named workload (or of a spec).

    ``overrides`` replace spec fields (e.g. N, V) to derive scaled-down cases
    with the same recipe.
    """
    spec = SPECS[name_or_spec] if isinstance(name_or_spec, str) else name_or_spec
    if overrides:
        spec = dataclasses.replace(spec, **overrides)
    rng = np.random.Generator(np.random.PCG64(SEED_BASE + spec.k if seed is None else seed))
    N, D, V = spec.N, spec.D, spec.V

    row_scale = np.full(N, spec.h_scale, dtype=np.float64)
    big = None
    if spec.big_row_frac > 0:
        nb = round_half_up(spec.big_row_frac * N)
        big = rng.permutation(N)[:nb]
        row_scale[big] *= spec.big_row_scale
    H = _normal_bits(rng, (N, D), 1.0, spec.dtype, row_scale=row_scale)
    W = _normal_bits(rng, (V, D), spec.w_std, spec.dtype)
    b = None
    if spec.bias_std is not None:
        b = _normal_bits(rng, (V,), spec.bias_std, spec.dtype)

    if spec.label_dist == "zipf":
        labels = _zipf_labels(rng, N, V, spec.zipf_s)
    else:
        labels = rng.integers(0, V, size=N, dtype=np.int64)
    if spec.peak_logit > 0:
        H = _peaked_hidden(rng, H, W, labels, spec)

    if spec.all_ignored:
        labels[:] = IGNORE_INDEX
    elif spec.segments > 0:
        seg = N // spec.segments
        pre = round_half_up(spec.prefix_frac * seg)
        for s in range(spec.segments):
            labels[s * seg: s * seg + pre] = IGNORE_INDEX
    if spec.ignore_frac > 0 and not spec.all_ignored:
        ni = round_half_up(spec.ignore_frac * N)
        labels[rng.permutation(N)[:ni]] = IGNORE_INDEX

    mask = np.ones(N, dtype=np.uint8)
    if spec.mask_false_frac > 0:
        nm = round_half_up(spec.mask_false_frac * N)
        mask[rng.permutation(N)[:nm]] = 0

    return Inputs(spec=spec, H=H, W=W, b=b, labels=labels, mask=mask,
                  big_rows=None if big is None else np.sort(big))


def random_case(seed: int, N: int, D: int, V: int, dtype: str = "bf16", bias: bool = True,
                ignore_frac: float = 0.25, mask_false_frac: float = 0.1, w_std: float = 0.05,
                lam: float = 1.0, h_scale: float = 1.0) -> Inputs:
    """A small seeded case of arbitrary shape (for ragged-tile parity tests)."""
    spec = WorkloadSpec(f"case{N}x{D}x{V}", 0, N=N, D=D, V=V, dtype=dtype, w_std=w_std,
                        h_scale=h_scale, bias_std=(0.1 if bias else None),
                        ignore_frac=ignore_frac, mask_false_frac=mask_false_frac, lam=lam)
    return make_inputs(spec, seed=seed)
