"""GPU parity of the RoPE entry points against the float64 oracle, element
by element: lwm_rope_apply and lwm_rope_apply_at, forward and inverse, bf16
and fp32, out of place and in place, positions from 0 and from an offset,
and positions up to 2^20 at theta 5e7, where the angle p * w_t is formed and
reduced in fp64 (an fp32 angle would be off by ~0.06 rad there).

Bounds: the oracle rotates the exact input in float64.  A bf16 result is
that value rounded once (half an ulp: 2^-9 relative) after an fp32 rotation;
an fp32 result differs by the fp32 rotation only.  So each element must lie
within 2^-8 |y| + 1e-6 (bf16) or 1e-5 (fp32, unit-variance inputs) of the
oracle, well inside the stated parity bounds (2e-2 / 2e-3 and 1e-4), which
are asserted too.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import assert_close, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lwm():
    import long_context_causal_attention_b200 as m
    return m


def _x(shape, dtype, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda").to(dtype)


def _check(got, want, dtype):
    got = to64(got)
    err = np.abs(got - want)
    if dtype == torch.bfloat16:
        assert np.all(err <= 2.0 ** -8 * np.abs(want) + 1e-6), float((err - 2.0 ** -8 * np.abs(want)).max())
        assert_close("rope", got, want, "bf16")
    else:
        assert float(err.max()) <= 1e-5, float(err.max())
        assert_close("rope", got, want, "fp32")


CASES = [
    # B, S, H, D, dtype, theta, offset
    (2, 300, 3, 128, torch.bfloat16, 1e4, 0),
    (1, 257, 2, 64, torch.float32, 1e6, 0),
    (1, 128, 4, 128, torch.float32, 1e7, 12345),
    (2, 200, 2, 64, torch.bfloat16, 5e7, 999_000),
    (1, 64, 2, 128, torch.bfloat16, 5e7, (1 << 20) - 64),   # last positions of a 1M row
    (1, 64, 2, 128, torch.float32, 5e7, (1 << 20) - 64),
    (1, 32, 1, 16, torch.float32, 1e4, 0),                  # small head size
]


@pytest.mark.parametrize("inverse", [False, True])
@pytest.mark.parametrize("case", CASES, ids=[f"{c[4]}-S{c[1]}-D{c[3]}-off{c[6]}" for c in CASES])
def test_rope_matches_oracle(lwm, case, inverse):
    B, S, H, D, dtype, theta, off = case
    x = _x((B, S, H, D), dtype, seed=S + D + off % 1000)
    want = oracle.rope_apply(to64(x), theta, inverse=inverse, position_offset=off)
    if off == 0:
        got = lwm.lwm_rope_apply(x, theta, inverse=inverse)
        torch.cuda.synchronize()
        _check(got, want, dtype)
    got = lwm.lwm_rope_apply_at(x, theta, off, inverse=inverse)
    torch.cuda.synchronize()
    _check(got, want, dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_rope_in_place_and_round_trip(lwm, dtype):
    """out = x works (in place), and the inverse undoes the forward up to the
    output rounding."""
    theta, off = 5e7, 700_000
    x = _x((2, 333, 2, 128), dtype, seed=5)
    x0 = to64(x)
    want = oracle.rope_apply(x0, theta, position_offset=off)
    lwm.lwm_rope_apply_at(x, theta, off, out=x)
    torch.cuda.synchronize()
    _check(x, want, dtype)
    back = lwm.lwm_rope_apply_at(x, theta, off, inverse=True)
    torch.cuda.synchronize()
    tol = 2.0 ** -7 if dtype == torch.bfloat16 else 1e-5
    assert float(np.abs(to64(back) - x0).max()) <= tol * max(1.0, float(np.abs(x0).max()))


def test_rope_theta_zero_copies(lwm):
    """theta <= 0 disables the rotation: the output equals the input."""
    x = _x((1, 100, 2, 128), torch.bfloat16, seed=8)
    got = lwm.lwm_rope_apply(x, 0.0)
    torch.cuda.synchronize()
    assert torch.equal(got, x)
