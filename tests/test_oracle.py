"""Pins for the float64 oracle, CPU only.

Each test checks the oracle against something that is not the oracle: torch's
own float64 attention and autograd, a scalar brute force, finite differences,
closed forms and the invariants the method fixes (exact softmax rows, relative
positions of rotary embeddings, and the packing equivalence the LWM research
note states in section "训练方法", Masked Sequence Packing).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A
from workloads import WORKLOADS, segment_ids, random_segments, THETA_SCHEDULE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape, sigma=1.0):
    return rng.standard_normal(shape) * sigma


# ----------------------------------------------------------------------------
# independent formulations used as pins
# ----------------------------------------------------------------------------

def rope_complex(x, theta, offset=0):
    """RoPE as complex multiplication: pair (x[2i], x[2i+1]) is the complex
    number x[2i] + 1j x[2i+1], multiplied by exp(1j p w_i).  Frequencies are
    built as a geometric sequence starting at 1 with ratio theta**(-2/D)."""
    x = torch.as_tensor(x, dtype=torch.float64)
    B, S, H, D = x.shape
    ratio = float(theta) ** (-2.0 / D)
    w = torch.tensor([ratio ** i for i in range(D // 2)], dtype=torch.float64)
    p = torch.arange(S, dtype=torch.float64) + offset
    rot = torch.polar(torch.ones(S, D // 2, dtype=torch.float64), p[:, None] * w[None, :])
    z = torch.view_as_complex(x.reshape(B, S, H, D // 2, 2).contiguous())
    z = z * rot[None, :, None, :]
    return torch.view_as_real(z).reshape(B, S, H, D)


def torch_attention(q, k, v, seg, causal, theta, scale=None):
    """torch float64 attention with RoPE by complex multiplication and an
    explicit boolean mask, through scaled_dot_product_attention."""
    q = torch.as_tensor(q, dtype=torch.float64)
    k = torch.as_tensor(k, dtype=torch.float64)
    v = torch.as_tensor(v, dtype=torch.float64)
    B, S, H, D = q.shape
    if theta and theta > 0:
        q, k = rope_complex(q, theta), rope_complex(k, theta)
    seg = torch.as_tensor(np.asarray(seg), dtype=torch.int64)
    mask = (seg[:, :, None] == seg[:, None, :]) & (seg[:, :, None] >= 0)
    if causal:
        mask = mask & torch.ones(S, S, dtype=torch.bool).tril()[None]
    sc = scale if scale else 1.0 / math.sqrt(D)
    out = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2),
        attn_mask=mask[:, None], scale=sc)
    scores = torch.einsum("bqhd,bkhd->bhqk", q, k) * sc
    lse = torch.logsumexp(scores.masked_fill(~mask[:, None], -math.inf), dim=-1)
    return out.transpose(1, 2), lse


def brute_force(q, k, v, d_o, seg, causal, theta, scale):
    """Scalar triple loops in plain Python floats (tiny inputs only)."""
    B, S, H, D = q.shape
    o = np.zeros((B, S, H, D)); lse = np.full((B, H, S), -np.inf)
    dq = np.zeros_like(o); dk = np.zeros_like(o); dv = np.zeros_like(o)

    def rot(vec, pos, sign):
        out = [0.0] * D
        for i in range(D // 2):
            a = pos * (theta ** (-2.0 * i / D)) if theta > 0 else 0.0
            c, s = math.cos(a), sign * math.sin(a)
            out[2 * i] = vec[2 * i] * c - vec[2 * i + 1] * s
            out[2 * i + 1] = vec[2 * i] * s + vec[2 * i + 1] * c
        return out

    for b in range(B):
        for h in range(H):
            qt = [rot(list(q[b, i, h]), i, 1.0) for i in range(S)]
            kt = [rot(list(k[b, j, h]), j, 1.0) for j in range(S)]
            dkt = [[0.0] * D for _ in range(S)]
            for i in range(S):
                ok = [j for j in range(S) if seg[b][i] >= 0 and seg[b][j] == seg[b][i]
                      and (not causal or j <= i)]
                if not ok:
                    continue
                s = {j: scale * sum(qt[i][d] * kt[j][d] for d in range(D)) for j in ok}
                m = max(s.values())
                z = sum(math.exp(s[j] - m) for j in ok)
                L = m + math.log(z)
                lse[b, h, i] = L
                P = {j: math.exp(s[j] - L) for j in ok}
                for d in range(D):
                    o[b, i, h, d] = sum(P[j] * v[b, j, h, d] for j in ok)
                dP = {j: sum(d_o[b, i, h, d] * v[b, j, h, d] for d in range(D)) for j in ok}
                Dsum = sum(P[j] * dP[j] for j in ok)
                dS = {j: P[j] * (dP[j] - Dsum) for j in ok}
                dqt = [scale * sum(dS[j] * kt[j][d] for j in ok) for d in range(D)]
                dq[b, i, h] = rot(dqt, i, -1.0)
                for j in ok:
                    for d in range(D):
                        dkt[j][d] += scale * dS[j] * qt[i][d]
                        dv[b, j, h, d] += P[j] * d_o[b, i, h, d]
            for j in range(S):
                dk[b, j, h] = rot(dkt[j], j, -1.0)
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


def _case(seed=0, B=2, S=40, H=3, D=8, sigma=1.0, seg=None, pad_tail=0):
    rng = np.random.default_rng(seed)
    q, k, v, do = (_rand(rng, B, S, H, D, sigma=sigma) for _ in range(4))
    if seg is None:
        seg = random_segments(rng, B, S, 1, 15, pad_tail=pad_tail)
    return q, k, v, do, seg


def _close(a, b, tol=1e-10):
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin)
    return np.allclose(a[fin], b[fin], atol=tol, rtol=tol)


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("theta", [1e4, 1e6, 5e7])
def test_rope_matches_complex_multiplication(theta):
    rng = np.random.default_rng(1)
    x = _rand(rng, 2, 33, 3, 16)
    y = A.rope_apply(x, theta)
    assert np.allclose(y, rope_complex(x, theta).numpy(), atol=1e-12)
    # inverse undoes, norms of each pair are kept
    assert np.allclose(A.rope_apply(y, theta, inverse=True), x, atol=1e-12)
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    assert np.allclose(n0, n1, atol=1e-12)


def test_rope_frequency_geometric_sequence():
    for theta, D in [(1e4, 128), (5e7, 128), (1e6, 64)]:
        w = A.rope_frequencies(D, theta)
        assert w[0] == 1.0
        assert np.allclose(w[1:] / w[:-1], theta ** (-2.0 / D), rtol=1e-13)
        # the sequence would reach exactly 1/theta one step past its end
        assert math.isclose(w[-1] * theta ** (-2.0 / D), 1.0 / theta, rel_tol=1e-12)


def test_rope_large_position_angles_are_reduced_exactly():
    # at p ~ 1e6 the angle for w_0 = 1 is p itself: cos must match math.cos(p)
    x = np.zeros((1, 1, 1, 4)); x[..., 0] = 1.0
    p = 1048575
    y = A.rope_apply(x, 5e7, position_offset=p)
    assert math.isclose(y[0, 0, 0, 0], math.cos(p), abs_tol=1e-12)
    assert math.isclose(y[0, 0, 0, 1], math.sin(p), abs_tol=1e-12)


def test_rope_disabled_is_identity():
    rng = np.random.default_rng(2)
    x = _rand(rng, 1, 5, 2, 8)
    assert np.array_equal(A.rope_apply(x, 0.0), x)


# ----------------------------------------------------------------------------
# forward and backward against torch float64
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("theta", [0.0, 1e4, 1e7])
def test_forward_matches_torch_sdpa(causal, theta):
    q, k, v, _, seg = _case(seed=3)
    o, lse = A.attention_forward(q, k, v, seg, causal=causal, theta=theta)
    to, tl = torch_attention(q, k, v, seg, causal, theta)
    assert np.allclose(o, to.numpy(), atol=1e-12)
    assert np.allclose(lse, tl.numpy(), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_matches_torch_autograd(causal):
    q, k, v, do, seg = _case(seed=4, S=36)
    theta = 1e4
    res = A.attention_backward(q, k, v, do, seg, causal=causal, theta=theta)
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    to, _ = torch_attention(tq, tk, tv, seg, causal, theta)
    (to * torch.tensor(do)).sum().backward()
    assert np.allclose(res["dq"], tq.grad.numpy(), atol=1e-11)
    assert np.allclose(res["dk"], tk.grad.numpy(), atol=1e-11)
    assert np.allclose(res["dv"], tv.grad.numpy(), atol=1e-11)


def test_backward_matches_finite_differences_of_forward():
    q, k, v, do, seg = _case(seed=5, B=1, S=10, H=1, D=4)
    theta = 100.0
    res = A.attention_backward(q, k, v, do, seg, causal=True, theta=theta)

    def loss(qq, kk, vv):
        o, _ = A.attention_forward(qq, kk, vv, seg, causal=True, theta=theta)
        return float(np.sum(o * do))

    eps = 1e-6
    for name, arr, grad in (("q", q, res["dq"]), ("k", k, res["dk"]), ("v", v, res["dv"])):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a1 = arr.copy(); a1[idx] += eps
            a2 = arr.copy(); a2[idx] -= eps
            args1 = {"q": (a1, k, v), "k": (q, a1, v), "v": (q, k, a1)}[name]
            args2 = {"q": (a2, k, v), "k": (q, a2, v), "v": (q, k, a2)}[name]
            num[idx] = (loss(*args1) - loss(*args2)) / (2 * eps)
        assert np.allclose(grad, num, atol=1e-7), name


def test_brute_force_tiny_with_padding():
    q, k, v, do, seg = _case(seed=6, B=2, S=12, H=2, D=4, pad_tail=2)
    seg[1, :5] = -1  # padding at the front of one row too
    theta, scale = 50.0, 0.7
    bf = brute_force(q, k, v, do, seg, True, theta, scale)
    res = A.attention_backward(q, k, v, do, seg, causal=True, theta=theta, scale=scale)
    for key in ("o", "lse", "dq", "dk", "dv"):
        assert _close(res[key], bf[key], 1e-11), key
    # padding rows: O = 0, LSE = -inf, gradients 0
    assert np.all(res["o"][1, :5] == 0) and np.all(np.isneginf(res["lse"][1, :, :5]))
    assert np.all(res["dq"][1, :5] == 0) and np.all(res["dk"][1, :5] == 0)


# ----------------------------------------------------------------------------
# invariants the method fixes
# ----------------------------------------------------------------------------

def test_softmax_rows_sum_to_one():
    q, k, v, _, seg = _case(seed=7, sigma=3.0)
    o, _ = A.attention_forward(q, k, np.ones_like(v), seg, theta=1e6)
    assert np.allclose(o, 1.0, atol=1e-12)


def test_relative_position_invariance():
    q, k, v, do, seg = _case(seed=8)
    r0 = A.attention_backward(q, k, v, do, seg, theta=1e4)
    r1 = A.attention_backward(q, k, v, do, seg, theta=1e4, position_offset=777777)
    for key in ("o", "lse", "dq", "dk", "dv"):
        assert _close(r0[key], r1[key], 1e-9), key


def test_closed_form_head_dim_two():
    # D = 2: w_0 = 1 and s_ij = scale |q_i| |k_j| cos(a_i + i - b_j - j)
    rng = np.random.default_rng(9)
    S = 20
    q = _rand(rng, 1, S, 1, 2); k = _rand(rng, 1, S, 1, 2); v = _rand(rng, 1, S, 1, 2)
    _, lse = A.attention_forward(q, k, v, None, causal=True, theta=123.0, scale=0.9)
    rq = np.hypot(q[0, :, 0, 0], q[0, :, 0, 1]); aq = np.arctan2(q[0, :, 0, 1], q[0, :, 0, 0])
    rk = np.hypot(k[0, :, 0, 0], k[0, :, 0, 1]); ak = np.arctan2(k[0, :, 0, 1], k[0, :, 0, 0])
    for i in range(S):
        s = [0.9 * rq[i] * rk[j] * math.cos(aq[i] + i - ak[j] - j) for j in range(i + 1)]
        assert math.isclose(lse[0, 0, i], math.log(sum(math.exp(x) for x in s)), abs_tol=1e-12)


def test_packing_equals_each_segment_alone():
    q, k, v, do, seg = _case(seed=10, B=1, S=48, H=2, D=8)
    seg[0] = np.repeat(np.arange(4), [7, 20, 1, 20])
    theta = 1e4
    packed = A.attention_backward(q, k, v, do, seg, theta=theta)
    start = 0
    for L in (7, 20, 1, 20):
        sl = slice(start, start + L)
        alone = A.attention_backward(q[:, sl], k[:, sl], v[:, sl], do[:, sl], None, theta=theta)
        for key in ("o", "dq", "dk", "dv"):
            assert np.allclose(packed[key][:, sl], alone[key], atol=1e-11), key
        assert np.allclose(packed["lse"][:, :, sl], alone["lse"], atol=1e-11)
        start += L


def test_first_token_of_segment_returns_its_value():
    q, k, v, _, seg = _case(seed=11)
    o, lse = A.attention_forward(q, k, v, seg, theta=1e5)
    B, S, H, D = q.shape
    qt, kt = A.rope_apply(q, 1e5), A.rope_apply(k, 1e5)
    for b in range(B):
        for i in range(S):
            if seg[b, i] >= 0 and (i == 0 or seg[b, i - 1] != seg[b, i]):
                assert np.allclose(o[b, i], v[b, i], atol=1e-12)
                sii = np.sum(qt[b, i] * kt[b, i], axis=-1) / math.sqrt(D)
                assert np.allclose(lse[b, :, i], sii, atol=1e-12)


def test_gradient_sums_per_segment():
    q, k, v, do, seg = _case(seed=12)
    theta = 1e6
    res = A.attention_backward(q, k, v, do, seg, theta=theta)
    dkt = A.rope_apply(res["dk"], theta)  # back to rotated space
    for b in range(seg.shape[0]):
        for sid in np.unique(seg[b]):
            m = seg[b] == sid
            assert np.allclose(res["dv"][b, m].sum(0), do[b, m].sum(0), atol=1e-11)
            assert np.allclose(dkt[b, m].sum(0), 0.0, atol=1e-11)


def test_key_shift_without_rotation_moves_only_lse():
    """theta disabled: adding one vector c to every key adds scale q_i.c to
    every score of row i, a per-row constant the softmax removes.  O, dQ, dK
    and dV stay (dQ because each row of dS sums to zero) and LSE moves by
    exactly scale q_i.c."""
    q, k, v, do, seg = _case(seed=21, pad_tail=3)
    c = np.random.default_rng(22).standard_normal(q.shape[-1])
    scale = 1.0 / math.sqrt(q.shape[-1])
    r0 = A.attention_backward(q, k, v, do, seg, theta=0.0)
    r1 = A.attention_backward(q, k + c, v, do, seg, theta=0.0)
    for key in ("o", "dq", "dk", "dv"):
        assert _close(r1[key], r0[key], 1e-9), key
    shift = scale * np.einsum("bshd,d->bhs", q, c)
    assert _close(r1["lse"], r0["lse"] + shift, 1e-9)


def test_value_shift_moves_output_by_the_same_vector():
    """Adding c to every value adds c to every output row that attends to
    anything (softmax rows sum to one) and leaves all three gradients: dP
    moves by a per-row constant that D_i absorbs."""
    q, k, v, do, seg = _case(seed=23, pad_tail=2)
    c = np.random.default_rng(24).standard_normal(q.shape[-1])
    r0 = A.attention_backward(q, k, v, do, seg, theta=1e6)
    r1 = A.attention_backward(q, k, v + c, do, seg, theta=1e6)
    live = (seg >= 0)[:, :, None, None]
    assert _close(r1["o"], r0["o"] + np.where(live, c, 0.0), 1e-9)
    for key in ("lse", "dq", "dk", "dv"):
        assert _close(r1[key], r0[key], 1e-9), key


def test_rows_and_tail_agree_with_full():
    q, k, v, do, seg = _case(seed=13, B=2, S=64)
    full = A.attention_backward(q, k, v, do, seg, theta=1e7)
    samples = [(0, 1, 0), (1, 2, 63), (1, 0, 31), (0, 2, 17)]
    rows = A.attention_rows(q, k, v, do, samples, seg, theta=1e7)
    for r, (b, h, i) in enumerate(samples):
        assert np.allclose(rows["o"][r], full["o"][b, i, h], atol=1e-12)
        assert np.allclose(rows["lse"][r], full["lse"][b, h, i], atol=1e-12)
        assert np.allclose(rows["dq"][r], full["dq"][b, i, h], atol=1e-12)
    tail = A.attention_backward(q, k, v, do, seg, theta=1e7, row_start=40)
    for key in ("dk", "dv", "dq", "o"):
        assert np.allclose(tail[key][:, 40:], full[key][:, 40:], atol=1e-11), key


def test_kept_pairs_counts_mask():
    w = WORKLOADS["tiny_packed_fp32"]
    seg = segment_ids(w)
    assert A.kept_pairs(seg) == 5050 + 12246 == 17296
    rng = np.random.default_rng(14)
    seg2 = random_segments(rng, 3, 50, 1, 9, pad_tail=3)
    S = 50
    brute = sum(int(A.allowed_mask(seg2[b], np.arange(S), np.arange(S), True).sum())
                for b in range(3))
    assert A.kept_pairs(seg2) == brute


# ----------------------------------------------------------------------------
# planted mistakes: each plausible error in the oracle fails a pin above
# ----------------------------------------------------------------------------

def test_planted_mistakes_are_caught(monkeypatch):
    q, k, v, do, seg = _case(seed=15, S=24)
    theta = 1e4
    to, tl = torch_attention(q, k, v, seg, True, theta)
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    o2, _ = torch_attention(tq, tk, tv, seg, True, theta)
    (o2 * torch.tensor(do)).sum().backward()

    def fails(fn):
        res = fn()
        ok = (np.allclose(res["o"], to.numpy(), atol=1e-9)
              and np.allclose(res["lse"], tl.numpy(), atol=1e-9)
              and np.allclose(res["dq"], tq.grad.numpy(), atol=1e-9)
              and np.allclose(res["dk"], tk.grad.numpy(), atol=1e-9)
              and np.allclose(res["dv"], tv.grad.numpy(), atol=1e-9))
        return not ok

    run = lambda: A.attention_backward(q, k, v, do, seg, causal=True, theta=theta)
    assert not fails(run)

    orig_rope = A.rope_apply
    # 1. wrong sign of the rotation
    monkeypatch.setattr(A, "rope_apply", lambda x, th, inverse=False, position_offset=0:
                        orig_rope(x, th, not inverse, position_offset))
    assert fails(run)
    monkeypatch.setattr(A, "rope_apply", orig_rope)

    # 2. rotate-half pairing instead of interleaved pairs
    def rope_half(x, th, inverse=False, position_offset=0):
        x = np.asarray(x, dtype=np.float64)
        D = x.shape[-1]
        perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])
        inv = np.argsort(perm)
        return orig_rope(x[..., inv], th, inverse, position_offset)[..., perm]
    monkeypatch.setattr(A, "rope_apply", rope_half)
    assert fails(run)
    monkeypatch.setattr(A, "rope_apply", orig_rope)

    # 3. dropped softmax scale
    assert fails(lambda: A.attention_backward(q, k, v, do, seg, causal=True, theta=theta, scale=1.0))

    # 4. segment mask dropped (packing ignored)
    assert fails(lambda: A.attention_backward(q, k, v, do, None, causal=True, theta=theta))

    # 5. log-sum-exp in base 2 instead of the natural log
    orig_soft = A._softmax_rows
    def lse_base2(s, allowed):
        lse, p = orig_soft(s, allowed)
        return lse / np.log(2.0), p
    monkeypatch.setattr(A, "_softmax_rows", lse_base2)
    assert fails(run)
    monkeypatch.setattr(A, "_softmax_rows", orig_soft)

    # 6. causal mask off by one (each row also sees key i + 1)
    orig_allowed = A.allowed_mask
    def off_by_one(seg_row, qi, ki, causal):
        m = orig_allowed(seg_row, qi, ki, False)
        if causal:
            m &= np.asarray(ki)[None, :] < np.asarray(qi)[:, None] + 2
        return m
    monkeypatch.setattr(A, "allowed_mask", off_by_one)
    assert fails(run)
    monkeypatch.setattr(A, "allowed_mask", orig_allowed)


# ----------------------------------------------------------------------------
# golden fixtures
# ----------------------------------------------------------------------------

def test_theta_schedule_matches_pages():
    with open(os.path.join(GOLDEN, "theta_schedule.json")) as f:
        g = json.load(f)
    for row in g["stages"]:
        assert THETA_SCHEDULE[row["seq_len"]] == row["theta"]
    assert WORKLOADS["fwd_32k"].theta == THETA_SCHEDULE[32768]
    assert WORKLOADS["long_128k"].theta == THETA_SCHEDULE[131072]
    assert WORKLOADS["million_1m"].theta == THETA_SCHEDULE[1048576]


def test_golden_tiny_case_regression():
    """Values written by tests/golden/make_golden.py (oracle only); any change
    to the oracle's arithmetic shows up here and must name its reason."""
    with open(os.path.join(GOLDEN, "tiny_case.json")) as f:
        g = json.load(f)
    q, k, v, do = (np.array(g["inputs"][n]) for n in ("q", "k", "v", "do"))
    seg = np.array(g["inputs"]["seg"])
    res = A.attention_backward(q, k, v, do, seg, causal=g["causal"], theta=g["theta"])
    for key in ("o", "lse", "dq", "dk", "dv"):
        assert _close(res[key], np.array(g["expected"][key], dtype=np.float64), 1e-12), key


# ----------------------------------------------------------------- decode step
def test_decode_equals_the_last_rows_of_the_forward():
    """A decode step is the forward pass's last T rows: same positions, same
    mask, same softmax (causal prefix property).  The decode oracle is a
    separate restatement, pinned here against the pinned forward oracle."""
    rng = np.random.default_rng(31)
    B, S, H, D, T = 2, 70, 3, 8, 5
    q = rng.standard_normal((B, S, H, D))
    k = rng.standard_normal((B, S, H, D))
    v = rng.standard_normal((B, S, H, D))
    seg = np.stack([np.repeat([0, 1, 2], [30, 25, 15]), np.repeat([0, 1], [66, 4])])
    seg[1, -2] = -1  # a padding token among the new ones
    for causal in (True, False):
        o_f, lse_f = oracle.attention_forward(q, k, v, seg, causal=causal, theta=500.0)
        o_d, lse_d = oracle.attention_decode(q[:, S - T:], k, v, seg, causal=causal, theta=500.0)
        np.testing.assert_allclose(o_d, o_f[:, S - T:], atol=1e-12)
        np.testing.assert_array_equal(np.isneginf(lse_d), np.isneginf(lse_f[:, :, S - T:]))
        fin = np.isfinite(lse_d)
        np.testing.assert_allclose(lse_d[fin], lse_f[:, :, S - T:][fin], atol=1e-12)


def test_decode_no_rope_matches_torch_sdpa():
    """theta disabled, one segment: each new query is plain softmax attention
    over the keys up to its position (torch fp64 SDPA with an explicit mask)."""
    import torch
    rng = np.random.default_rng(32)
    B, S, H, D, T = 2, 40, 2, 16, 4
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, S, H, D))
    v = rng.standard_normal((B, S, H, D))
    o, lse = oracle.attention_decode(q, k, v, None, theta=0.0)
    mask = torch.arange(S)[None, :] <= torch.arange(S - T, S)[:, None]
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    s = torch.einsum("bhtd,bhsd->bhts", tq, tk) / np.sqrt(D)
    ref_lse = torch.logsumexp(s.masked_fill(~mask, -float("inf")), dim=-1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), atol=1e-12)


def test_decode_oracle_catches_a_position_shift(monkeypatch):
    """Planted mistake: rotating the new queries as if they started at 0
    breaks the equality with the forward rows."""
    rng = np.random.default_rng(33)
    B, S, H, D, T = 1, 50, 1, 8, 3
    q, k, v = (rng.standard_normal((B, S, H, D)) for _ in range(3))
    o_f, _ = oracle.attention_forward(q, k, v, None, theta=100.0)
    real = oracle.attention.rope_apply

    def shifted(x, theta, inverse=False, position_offset=0):
        return real(x, theta, inverse, 0)
    monkeypatch.setattr(oracle.attention, "rope_apply", shifted)
    o_d, _ = oracle.attention_decode(q[:, S - T:], k, v, None, theta=100.0)
    assert np.abs(o_d - o_f[:, S - T:]).max() > 1e-3


# ------------------------------------------------- packed loss re-weighting
def test_packed_loss_equals_unpacked_per_sample_mean():
    """The pages' claim: with the re-weighting, packed training equals
    training on the samples one by one with padding, i.e. the mean over
    samples of each sample's own mean token loss (computed here per sample,
    with torch's cross-entropy)."""
    import torch
    rng = np.random.default_rng(41)
    B, S, V = 2, 40, 11
    seg = np.stack([np.repeat([0, 1, 2, -1], [12, 5, 20, 3]), np.repeat([0, 1], [33, 7])])
    targets = rng.integers(0, V, size=(B, S))
    targets[0, :4] = -1          # prompt tokens without loss
    targets[1, 33:] = -1         # a sample with no loss token at all
    targets[0, 37:] = -1         # padding
    z = rng.standard_normal((B, S, V))
    loss, d = oracle.packed_cross_entropy(z, targets, seg)
    per_sample = []
    for b in range(B):
        for s, e in oracle.sample_runs(seg[b]):
            keep = targets[b, s:e] >= 0
            if keep.any():
                zz = torch.from_numpy(z[b, s:e][keep])
                yy = torch.from_numpy(targets[b, s:e][keep])
                per_sample.append(torch.nn.functional.cross_entropy(zz, yy).item())
    assert len(per_sample) == 4
    assert abs(loss - np.mean(per_sample)) < 1e-12
    w = oracle.packed_loss_weights(seg, targets)
    assert abs(w.sum() - 1.0) < 1e-12 and np.all(w[targets < 0] == 0)
    # naive packing (token mean) differs: short samples weigh less there
    naive = np.mean([torch.nn.functional.cross_entropy(
        torch.from_numpy(z[b][targets[b] >= 0]), torch.from_numpy(targets[b][targets[b] >= 0]),
        reduction="sum").item() for b in range(B)]) * B / np.count_nonzero(targets >= 0)
    assert abs(naive - loss) > 1e-3


def test_packed_loss_out_of_vocabulary_targets_carry_no_loss():
    """A target outside [0, V) marks a token without loss, like a negative
    one: the loss is the mean over samples of torch's per-sample mean
    cross-entropy over the in-vocabulary targets only, and such tokens get a
    zero gradient row."""
    import torch
    rng = np.random.default_rng(43)
    B, S, V = 2, 30, 9
    seg = np.stack([np.repeat([0, 1, 2], [10, 6, 14]), np.repeat([3, -1], [26, 4])])
    targets = rng.integers(0, V, size=(B, S))
    targets[0, 10:16] = V + rng.integers(0, 5, size=6)   # the whole of sample 1
    targets[0, [2, 20, 21]] = V                          # a few inside other samples
    targets[1, 5] = 2 ** 30
    z = rng.standard_normal((B, S, V))
    loss, d = oracle.packed_cross_entropy(z, targets, seg)
    keep_all = (targets >= 0) & (targets < V)
    per_sample = []
    for b in range(B):
        for s, e in oracle.sample_runs(seg[b]):
            keep = keep_all[b, s:e]
            if keep.any():
                zz = torch.from_numpy(z[b, s:e][keep])
                yy = torch.from_numpy(targets[b, s:e][keep])
                per_sample.append(torch.nn.functional.cross_entropy(zz, yy).item())
    assert len(per_sample) == 3   # sample 1 of row 0 has no in-vocabulary target
    assert abs(loss - np.mean(per_sample)) < 1e-12
    assert np.all(d[~keep_all] == 0)
    w = oracle.packed_loss_weights(seg, targets, vocab=V)
    assert abs(w.sum() - 1.0) < 1e-12 and np.all(w[~keep_all] == 0)


def test_packed_loss_gradient_matches_autograd():
    import torch
    rng = np.random.default_rng(42)
    B, S, V = 2, 17, 7
    seg = np.stack([np.repeat([0, 1], [9, 8]), np.repeat([4, -1], [15, 2])])
    targets = rng.integers(0, V, size=(B, S))
    targets[1, 15:] = -1
    z = rng.standard_normal((B, S, V))
    loss, d = oracle.packed_cross_entropy(z, targets, seg)
    w = torch.from_numpy(oracle.packed_loss_weights(seg, targets))
    zt = torch.from_numpy(z).requires_grad_(True)
    y = torch.from_numpy(np.where(targets >= 0, targets, 0))
    ce = torch.nn.functional.cross_entropy(zt.reshape(-1, V), y.reshape(-1), reduction="none")
    tl = (ce.reshape(B, S) * w).sum()
    tl.backward()
    assert abs(tl.item() - loss) < 1e-12
    np.testing.assert_allclose(d, zt.grad.numpy(), atol=1e-14)


def test_sample_runs_split_equal_ids_in_separate_runs():
    assert oracle.sample_runs([0, 0, 1, 1, 0, -1, -1, 2]) == [(0, 2), (2, 4), (4, 5), (7, 8)]
