"""GPU: the polynomial 2^x the epilogues evaluate on the FMA pipe for small
hidden sizes (ex2_poly), against 2^x in binary64 and beside the special-
function unit's ex2.approx on the same arguments.

Bound: the degree-5 polynomial of best relative approximation of 2^f on
[-1/2, 1/2] has relative error 1.55e-7 once its coefficients are rounded to
float32 (exp2_poly_fit.py); evaluating it in float32 adds at most one rounding
of 2^-24 relative per fused multiply-add (five) and none for the exponent
insertion, so |ex2_poly(x) / 2^x - 1| <= 1.55e-7 + 5 * 2^-24 < 4.5e-7 for
x in [-125, 16]."""
import numpy as np
import pytest
import torch

from lm_head_projection_supervised_b200 import binding

from _gpu_helpers import record

pytestmark = pytest.mark.gpu
BOUND = 1.55e-7 + 5 * 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from lm_head_projection_supervised_b200 import build
    build.build()
    binding.lib()


def test_ex2_poly_relative_error():
    rng = np.random.default_rng(0)
    grid = np.linspace(-125.0, 16.0, 4_000_001, dtype=np.float64)
    edges = np.arange(-125, 17, dtype=np.float64)
    near = np.concatenate([edges + d for d in (-0.5, -0.5 + 1e-6, 0.5 - 1e-6, 0.0, 1e-7)])
    x32 = np.concatenate([grid, near, rng.uniform(-30, 0, 1_000_000)]).astype(np.float32)
    x32 = x32[(x32 >= -125.0) & (x32 <= 16.0)]
    yp, ys = binding.diag_exp2(torch.from_numpy(x32).cuda())
    ref = np.exp2(x32.astype(np.float64))
    rp = np.abs(yp.cpu().numpy().astype(np.float64) / ref - 1.0)
    rs = np.abs(ys.cpu().numpy().astype(np.float64) / ref - 1.0)
    ok = ref >= 2.0 ** -126  # ex2.approx flushes subnormal results; compare normal ones
    record("ex2_poly relative error", float(rp.max()), BOUND,
           sfu_max_relative_error=float(rs[ok].max()))
    assert rp.max() <= BOUND, float(rp.max())


def test_ex2_poly_below_range_is_tiny_and_nonnegative():
    x = torch.tensor([-125.0, -126.0, -200.0, -1e30, float("-inf")], device="cuda")
    yp, _ = binding.diag_exp2(x)
    y = yp.cpu().numpy()
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -124)
