"""GPU parity of the decode step (lwm_attn_decode) against the float64 oracle.

New tokens are the last T positions of each row; the cache holds the
rotated keys, built on the GPU with lwm_rope_apply from the seeded
un-rotated keys, which are what the oracle receives.  Cases cover one and
several new tokens (each kernel variant: 1, 2 and groups of 4), packed
segments with padding among the new tokens (chunks of other segments are
skipped unread), both mask modes, no rotation, a one-token cache, and the
million-token cache with theta 5e7 on sampled heads.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import assert_close, to64
from workloads import packed_video_text_row, random_segments

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lwm():
    import long_context_causal_attention_b200 as m
    return m


def draw(B, S, T, H, D, seed, sigma=0.5):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    q = (torch.randn((B, T, H, D), generator=g, device="cuda") * sigma).to(torch.bfloat16)
    k = (torch.randn((B, S, H, D), generator=g, device="cuda") * sigma).to(torch.bfloat16)
    v = (torch.randn((B, S, H, D), generator=g, device="cuda") * sigma).to(torch.bfloat16)
    return q, k, v


def run_decode(lwm, q, k, v, seg, causal, theta):
    seg_d = None if seg is None else torch.as_tensor(seg, dtype=torch.int32, device="cuda")
    k_cache = lwm.lwm_rope_apply(k, theta) if theta > 0 else k
    o, lse = lwm.lwm_attn_decode(q, k_cache, v, seg_d, causal=causal, rope_theta=theta,
                                 check_status=True)
    torch.cuda.synchronize()
    return o, lse


CASES = [
    # name, B, S, H, T, theta, causal, segments
    ("t1_packed_pad", 2, 1000, 4, 1, 1e6, True, "random_pad"),
    ("t2_packed", 2, 1000, 4, 2, 1e6, True, "random"),
    ("t3_single", 1, 777, 3, 3, 1e7, True, "single"),
    ("t16_packed_pad", 2, 1300, 2, 16, 1e6, True, "random_pad"),
    ("t5_noncausal", 2, 600, 2, 5, 1e4, False, "random"),
    ("t4_no_rope", 1, 513, 2, 4, 0.0, True, "single"),
    ("s1_t1", 1, 1, 2, 1, 1e4, True, "single"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_decode_small(lwm, case):
    name, B, S, H, T, theta, causal, segs = case
    q, k, v = draw(B, S, T, H, 128, seed=len(name) * 7 + S)
    rng = np.random.default_rng(S + T)
    seg = None
    if segs.startswith("random"):
        seg = random_segments(rng, B, S, 20, 300, pad_tail=2 if segs.endswith("pad") else 0)
    o, lse = run_decode(lwm, q, k, v, seg, causal, theta)
    o_ref, lse_ref = oracle.attention_decode(to64(q), to64(k), to64(v), seg, causal=causal,
                                             theta=theta)
    assert_close("o", to64(o), o_ref, "bf16")
    assert_close("lse", to64(lse), lse_ref, "bf16")


def test_decode_packed_video_text_64k(lwm):
    """Packed 64K rows of the video/text mix; new tokens sit in the last
    segment, so most cache chunks belong to other segments and are skipped."""
    B, S, H, T = 2, 65536, 4, 4
    rng = np.random.default_rng(3)
    seg = np.stack([packed_video_text_row(rng, S) for _ in range(B)])
    assert len(np.unique(seg[0])) > 10
    q, k, v = draw(B, S, T, H, 128, seed=11)
    o, lse = run_decode(lwm, q, k, v, seg, True, 1e6)
    o_ref, lse_ref = oracle.attention_decode(to64(q), to64(k), to64(v), seg, theta=1e6)
    assert_close("o", to64(o), o_ref, "bf16")
    assert_close("lse", to64(lse), lse_ref, "bf16")


def test_decode_million_token_cache(lwm):
    """One new token against a 2^20-token cache, theta 5e7, all 32 heads on
    the GPU; the oracle checks two of them in full (every key)."""
    B, S, H, T = 1, 1 << 20, 32, 1
    q, k, v = draw(B, S, T, H, 128, seed=5)
    o, lse = run_decode(lwm, q, k, v, None, True, 5e7)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    for h in (0, 19):  # one head at a time keeps the float64 copies at ~1 GB each
        o_ref, lse_ref = oracle.attention_decode(to64(q[:, :, h:h + 1]), to64(k[:, :, h:h + 1]),
                                                 to64(v[:, :, h:h + 1]), None, theta=5e7)
        assert_close("o", to64(o[:, :, h:h + 1]), o_ref, "bf16")
        assert_close("lse", to64(lse[:, h:h + 1]), lse_ref, "bf16")


def test_decode_matches_forward_last_rows(lwm):
    """Same inputs through lwm_attn_fwd: its last T rows are the decode step."""
    B, S, H, T, theta = 1, 900, 2, 3, 1e6
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    q, k, v = ((torch.randn((B, S, H, 128), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
               for _ in range(3))
    rng = np.random.default_rng(9)
    seg = random_segments(rng, B, S, 100, 400)
    seg_d = torch.as_tensor(seg, dtype=torch.int32, device="cuda")
    o_f, lse_f = lwm.lwm_attn_fwd(q, k, v, seg_d, True, theta, check_status=True)
    o_d, lse_d = run_decode(lwm, q[:, S - T:].contiguous(), k, v, seg, True, theta)
    assert_close("o", to64(o_d), to64(o_f[:, S - T:]), "bf16")
    assert_close("lse", to64(lse_d), to64(lse_f[:, :, S - T:]), "bf16")
