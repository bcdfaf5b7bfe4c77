"""Writes tests/golden/tiny_cases.json: four tiny cases whose expected values
come from the CPU oracle (oracle.flce_oracle.forward_backward) and nothing
else.  Two of them also have closed forms that tests/test_golden.py checks
the stored values against:

  uniform   W = 0, b = 0: every row is uniform, L = log V, m = 0, log s = log V
            (maximum entropy, "数学基础" maths-basics page §5.6);
  binary    V = 2: L = mean_i softplus(z_other - z_target) (the two-class case
            of the cross entropy, maths-basics page §5.5);
  mixed     bias, a false mask entry and an ignored label (the supervised-row
            filter a_i of "分块交叉熵" §01);
  none      every label ignored: the zero sentinel of §01.

Inputs are small multiples of powers of two, exact in bf16, so the CUDA path
sees the same values.  Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
from oracle import flce_oracle as orc  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_cases.json")


def _grid(rng, shape, lo, hi, step):
    """Values k * step with k uniform in [lo, hi]: exact in bf16 for small k."""
    return rng.integers(lo, hi + 1, size=shape).astype(np.float64) * step


def cases():
    rng = np.random.default_rng(7)
    out = []
    # uniform: W = 0, b = 0
    H = _grid(rng, (5, 8), -8, 8, 0.125)
    out.append(dict(name="uniform", H=H, W=np.zeros((10, 8)), b=np.zeros(10),
                    labels=np.array([0, 3, 9, 4, 7]), mask=np.ones(5, np.uint8), lam=1.0))
    # binary: V = 2, no bias
    H = _grid(rng, (6, 8), -8, 8, 0.125)
    W = _grid(rng, (2, 8), -8, 8, 0.0625)
    out.append(dict(name="binary", H=H, W=W, b=None, labels=np.array([0, 1, 1, 0, 1, 0]),
                    mask=np.ones(6, np.uint8), lam=1.0))
    # mixed: bias, a false mask entry, an ignored label, lambda != 1
    H = _grid(rng, (7, 16), -8, 8, 0.125)
    W = _grid(rng, (37, 16), -8, 8, 0.0625)
    b = _grid(rng, (37,), -8, 8, 0.03125)
    out.append(dict(name="mixed", H=H, W=W, b=b, labels=np.array([5, -100, 36, 0, 12, 12, 30]),
                    mask=np.array([1, 1, 1, 0, 1, 1, 1], np.uint8), lam=0.75))
    # none supervised
    H = _grid(rng, (4, 8), -8, 8, 0.125)
    W = _grid(rng, (9, 8), -8, 8, 0.0625)
    out.append(dict(name="none", H=H, W=W, b=None, labels=np.full(4, -100),
                    mask=np.ones(4, np.uint8), lam=1.0))
    return out


def _list(a):
    return None if a is None else np.asarray(a, dtype=np.float64).tolist()


def main():
    rows = []
    for c in cases():
        r = orc.forward_backward(c["H"], c["W"], c["b"], c["labels"], c["mask"], lam=c["lam"])
        rows.append(dict(
            name=c["name"],
            source="oracle.flce_oracle.forward_backward (tests/golden/make_golden.py)",
            H=_list(c["H"]), W=_list(c["W"]), b=_list(c["b"]),
            labels=np.asarray(c["labels"]).tolist(), mask=np.asarray(c["mask"]).tolist(),
            lam=c["lam"], loss=r["loss"],
            m=[None if not np.isfinite(v) else float(v) for v in r["m"]],
            logs=[None if not np.isfinite(v) else float(v) for v in r["logs"]],
            dH=_list(r["dH"]), dW=_list(r["dW"]), db=_list(r["db"])))
    with open(OUT, "w") as f:
        json.dump({"cases": rows}, f, indent=1)
    print(OUT)


if __name__ == "__main__":
    main()
