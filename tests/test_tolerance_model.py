"""Where the bf16 parity bounds come from (CPU only).

The device rounds the rotated q and k to bf16 before the tensor-core MMAs;
the oracle rotates the exact inputs in float64.  This test applies exactly
that one extra rounding on the CPU (oracle on bf16-rounded rotated q, k, no
further rotation, gradients turned back with R^T) and checks that the error
it alone causes stays inside the bounds the GPU parity tests use: the stated
bf16 bound for the named workloads' score scales, the derived sharp bound
for sigma 2 stress inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import TOL
from workloads import Workload, make_tensors


def _bf16(a):
    return torch.tensor(a).float().bfloat16().double().numpy()


@pytest.mark.parametrize("sigma,S,tol", [(0.5, 129, "bf16"), (1.0, 129, "bf16"),
                                         (2.0, 129, "bf16_sharp"), (2.0, 640, "bf16_sharp")])
def test_rotated_operand_rounding_fits_bounds(sigma, S, tol):
    theta = 1e7
    w = Workload("model", 1, S, 2, 128, "bf16", theta, sigma=sigma)
    t = make_tensors(w, seed=7, device="cpu", with_grad_out=True)
    q, k, v, do = (t[n].double().numpy() for n in ("q", "k", "v", "do"))
    ref = oracle.attention_backward(q, k, v, do, None, theta=theta)
    qr = _bf16(oracle.rope_apply(q, theta))
    kr = _bf16(oracle.rope_apply(k, theta))
    mod = oracle.attention_backward(qr, kr, v, do, None, theta=0.0)
    mod["dq"] = oracle.rope_apply(mod["dq"], theta, inverse=True)
    mod["dk"] = oracle.rope_apply(mod["dk"], theta, inverse=True)
    mx, mean = TOL[tol]
    for key in ("o", "lse", "dq", "dk", "dv"):
        d = np.abs(mod[key] - ref[key])
        # leave room for the outputs' own bf16 rounding on top of the model
        assert d.max() <= 0.75 * mx and d.mean() <= 0.75 * mean, (key, d.max(), d.mean())
