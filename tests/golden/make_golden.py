"""Writes tests/golden/tiny_case.json from the oracle alone.

The fixture locks the oracle's arithmetic on one tiny packed, causal input
(two segments plus a padding token, RoPE theta 1e4).  It is a regression
guard, not a pin: the pins are the tests in tests/test_oracle.py.
Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
from oracle import attention_backward  # noqa: E402


def main():
    rng = np.random.default_rng(20240213)
    B, S, H, D = 1, 9, 2, 4
    q, k, v, do = (np.round(rng.standard_normal((B, S, H, D)), 3) for _ in range(4))
    seg = np.array([[0, 0, 0, 0, 1, 1, 1, 1, -1]])
    theta, causal = 1e4, True
    res = attention_backward(q, k, v, do, seg, causal=causal, theta=theta)
    fix = lambda a: np.where(np.isfinite(a), a, None).tolist()
    out = {
        "source": "oracle only (tests/golden/make_golden.py); packing mask per the LWM research note, section 训练方法, Masked Sequence Packing",
        "causal": causal, "theta": theta,
        "inputs": {"q": q.tolist(), "k": k.tolist(), "v": v.tolist(), "do": do.tolist(),
                   "seg": seg.tolist()},
        "expected": {key: fix(res[key]) for key in ("o", "lse", "dq", "dk", "dv")},
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_case.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
