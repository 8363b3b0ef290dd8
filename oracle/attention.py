"""Float64 CPU oracle: exact causal softmax attention with RoPE and packing mask.

TEST INFRASTRUCTURE ONLY (see the package docstring).  The product path never
imports this module.

What it computes, step by step, and where each step comes from:

1. RoPE frequencies  w_i = theta ** (-2 i / D),  i = 0 .. D/2-1.
   LWM research note, section "模型架构" (model architecture): "standard RoPE";
   the RoFormer entry of the paper card's reference list fixes the form.
   theta is the per-stage value of the note's section "训练方法" (32K: 1e6,
   128K: 1e7, 256K: 1e7, 512K: 2.5e7, 1M: 5e7).
2. Rotation of query and key vectors by angle p * w_i on the interleaved
   pairs (x[2i], x[2i+1]), p = position of the token in its row.
3. Scores  s_ij = scale * <q~_i, k~_j>.
4. Mask  allowed(i, j) = seg_i == seg_j  and  seg_i >= 0  and  (j <= i if
   causal).  Research note, section "训练方法", Masked Sequence Packing: each
   packed sample attends only to itself.
5. Exact softmax (paper card, Summary: "without approximation"):
   LSE_i = ln sum_{allowed j} exp(s_ij),  P_ij = exp(s_ij - LSE_i) on allowed
   pairs and 0 elsewhere,  O_i = sum_j P_ij v_j.
6. Backward (the gradients that training through this layer needs; the
   FlashAttention entry of the reference list recomputes P from LSE, which is
   the same arithmetic):  dP_ij = <dO_i, v_j>,  D_i = sum_j P_ij dP_ij,
   dS_ij = P_ij (dP_ij - D_i),  dq~_i = scale sum_j dS_ij k~_j,
   dk~_j = scale sum_i dS_ij q~_i,  dv_j = sum_i P_ij dO_i,
   dq = R(p)^T dq~,  dk = R(p)^T dk~.

Scores are materialised one block of query rows at a time so memory stays
bounded; there is no other blocking, fusion or reordering.

7. Packed loss re-weighting (same section, Masked Sequence Packing: packed
   training made numerically equal to unpacked training with padding): a
   sample is a contiguous run of one segment id; each loss token of a sample
   with n loss tokens weighs 1 / (n * number of samples with a loss token),
   so the packed loss is the mean over samples of each sample's mean token
   cross-entropy.  packed_cross_entropy returns that loss and d loss / d
   logits.
"""

from __future__ import annotations

import numpy as np

# Readings of points the pages leave open.  Each one is also listed in the
# design notes of the repository.
READINGS = {
    "rope_pairing": "interleaved pairs (x[2i], x[2i+1]) as in the RoFormer formulation",
    "rope_frequency": "w_i = theta ** (-2 i / D)",
    "rope_positions": "p = index of the token in its row, continuing across packed segments "
                      "(attention output and gradients are unchanged by a per-segment restart, "
                      "since rotary scores depend only on i - j)",
    "rope_disabled": "theta <= 0 disables the rotation",
    "scale": "1/sqrt(D) unless given",
    "padding": "segment id < 0 marks padding: O = 0, LSE = -inf, all gradients 0",
    "lse_base": "natural log of the scaled scores",
    "grad_wrt": "dq, dk are gradients with respect to the un-rotated inputs",
}


def rope_frequencies(head_dim: int, theta: float) -> np.ndarray:
    """w_i = theta ** (-2 i / D) for i < D/2 (RoFormer form; LWM note, "模型架构")."""
    if head_dim % 2:
        raise ValueError("head_dim must be even for rotary pairs")
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * i / head_dim)


def rope_angles(positions, head_dim: int, theta: float) -> np.ndarray:
    """Angles p * w_i in float64, shape [len(positions), D/2]."""
    p = np.asarray(positions, dtype=np.float64)
    return np.multiply.outer(p, rope_frequencies(head_dim, theta))


def rope_apply(x, theta: float, inverse: bool = False, position_offset: int = 0) -> np.ndarray:
    """Rotate x of shape [B, S, H, D] by R(p), or by R(p)^T when ``inverse``.

    Position p of token t is ``t + position_offset``.  Interleaved pairs
    (x[2i], x[2i+1]) turn by angle p * w_i:
        y[2i]   = x[2i] cos - x[2i+1] sin
        y[2i+1] = x[2i] sin + x[2i+1] cos
    theta <= 0 returns x unchanged (as float64).
    """
    x = np.asarray(x, dtype=np.float64)
    if theta is None or theta <= 0:
        return x.copy()
    B, S, H, D = x.shape
    ang = rope_angles(np.arange(S) + position_offset, D, theta)  # [S, D/2]
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    if inverse:
        s = -s
    xe = x[..., 0::2]
    xo = x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = xe * c - xo * s
    y[..., 1::2] = xe * s + xo * c
    return y


def allowed_mask(seg_row, q_idx, k_idx, causal: bool) -> np.ndarray:
    """Boolean [len(q_idx), len(k_idx)]: same segment, not padding, causal order."""
    seg_row = np.asarray(seg_row)
    sq = seg_row[np.asarray(q_idx)][:, None]
    sk = seg_row[np.asarray(k_idx)][None, :]
    m = (sq == sk) & (sq >= 0)
    if causal:
        m &= np.asarray(k_idx)[None, :] <= np.asarray(q_idx)[:, None]
    return m


def _seg_or_default(seg, B, S):
    if seg is None:
        return np.zeros((B, S), dtype=np.int64)
    seg = np.asarray(seg).astype(np.int64)
    if seg.shape != (B, S):
        raise ValueError(f"segment ids must be [B, S] = {(B, S)}, got {seg.shape}")
    return seg


def _scale(scale, D):
    return 1.0 / np.sqrt(D) if (scale is None or scale <= 0) else float(scale)


def _softmax_rows(s, allowed):
    """LSE per row and P, exact in float64; rows with nothing allowed give LSE=-inf, P=0."""
    sm = np.where(allowed, s, -np.inf)
    m = np.max(sm, axis=1, initial=-np.inf)
    has = np.isfinite(m)
    m_safe = np.where(has, m, 0.0)
    e = np.where(allowed, np.exp(s - m_safe[:, None]), 0.0)
    tot = e.sum(axis=1)
    lse = np.where(has, m_safe + np.log(np.where(has, tot, 1.0)), -np.inf)
    p = np.where(allowed, np.exp(s - np.where(has, lse, 0.0)[:, None]), 0.0)
    return lse, p


def _rows_per_block(S):
    return int(min(512, max(1, (1 << 24) // max(S, 1))))


def attention_forward(q, k, v, seg=None, causal=True, theta=1e4, scale=None,
                      position_offset=0):
    """O [B,S,H,D] and LSE [B,H,S] in float64 (steps 1-5 of the module docstring)."""
    out = attention_backward(q, k, v, None, seg=seg, causal=causal, theta=theta,
                             scale=scale, position_offset=position_offset)
    return out["o"], out["lse"]


def attention_backward(q, k, v, d_o, seg=None, causal=True, theta=1e4, scale=None,
                       row_start=0, position_offset=0):
    """Forward plus (when ``d_o`` is given) backward, in float64.

    Query rows ``[row_start, S)`` of every (batch, head) are processed.  The
    returned ``o``, ``lse`` and ``dq`` are exact for those rows (other rows are
    left at 0 / -inf).  ``dk`` and ``dv`` hold the contributions of those rows
    only; with a causal mask that is the exact gradient of every key at
    position >= row_start, which is how long inputs are checked on their last
    rows without the full quadratic cost.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, S, H, D = q.shape
    seg = _seg_or_default(seg, B, S)
    sc = _scale(scale, D)
    qt = rope_apply(q, theta, position_offset=position_offset)
    kt = rope_apply(k, theta, position_offset=position_offset)
    want_bwd = d_o is not None
    if want_bwd:
        d_o = np.asarray(d_o, dtype=np.float64)

    o = np.zeros((B, S, H, D))
    lse = np.full((B, H, S), -np.inf)
    dqt = np.zeros((B, S, H, D)) if want_bwd else None
    dkt = np.zeros((B, S, H, D)) if want_bwd else None
    dv = np.zeros((B, S, H, D)) if want_bwd else None
    blk = _rows_per_block(S)

    for b in range(B):
        for h in range(H):
            Q, K, V = qt[b, :, h, :], kt[b, :, h, :], v[b, :, h, :]
            for r0 in range(row_start, S, blk):
                r1 = min(S, r0 + blk)
                kend = r1 if causal else S
                rows = np.arange(r0, r1)
                keys = np.arange(kend)
                s = sc * (Q[r0:r1] @ K[:kend].T)
                allowed = allowed_mask(seg[b], rows, keys, causal)
                l, P = _softmax_rows(s, allowed)
                lse[b, h, r0:r1] = l
                o[b, r0:r1, h, :] = P @ V[:kend]
                if want_bwd:
                    dO = d_o[b, r0:r1, h, :]
                    dP = dO @ V[:kend].T
                    Di = np.sum(P * dP, axis=1)
                    dS = P * (dP - Di[:, None])
                    dqt[b, r0:r1, h, :] = sc * (dS @ K[:kend])
                    dkt[b, :kend, h, :] += sc * (dS.T @ Q[r0:r1])
                    dv[b, :kend, h, :] += P.T @ dO

    res = {"o": o, "lse": lse}
    if want_bwd:
        res["dq"] = rope_apply(dqt, theta, inverse=True, position_offset=position_offset)
        res["dk"] = rope_apply(dkt, theta, inverse=True, position_offset=position_offset)
        res["dv"] = dv
    return res


def attention_rows(q, k, v, d_o, samples, seg=None, causal=True, theta=1e4, scale=None):
    """Exact O row, LSE and dq row for sampled query rows.

    ``samples`` is a sequence of (b, h, i).  Each row needs only its own keys,
    so this scales to any sequence length.  ``d_o`` may be None (no dq).
    Returns dict of arrays: o [n, D], lse [n], dq [n, D] (when d_o given).
    """
    q = np.asarray(q)
    B, S, H, D = q.shape
    seg = _seg_or_default(seg, B, S)
    sc = _scale(scale, D)
    n = len(samples)
    o = np.zeros((n, D))
    lse = np.full(n, -np.inf)
    dq = np.zeros((n, D)) if d_o is not None else None
    use_rope = theta is not None and theta > 0
    # group the samples by (b, h) so each head's keys are rotated once
    groups = {}
    for r, (b, h, i) in enumerate(samples):
        groups.setdefault((int(b), int(h)), []).append((r, int(i)))
    for (b, h), items in groups.items():
        kmax = max(i for _, i in items) + 1 if causal else S
        Kall = np.asarray(k[b, :kmax, h, :], dtype=np.float64)
        if use_rope:
            Kall = rope_apply(Kall.reshape(1, kmax, 1, D), theta).reshape(kmax, D)
        Vall = np.asarray(v[b, :kmax, h, :], dtype=np.float64)
        for r, i in items:
            kend = i + 1 if causal else S
            keys = np.arange(kend)
            K, V = Kall[:kend], Vall[:kend]
            qi = np.asarray(q[b, i, h, :], dtype=np.float64)
            if use_rope:
                qi = rope_apply(qi.reshape(1, 1, 1, D), theta, position_offset=i).reshape(D)
            s = sc * (K @ qi)
            allowed = allowed_mask(seg[b], np.array([i]), keys, causal)
            l, P = _softmax_rows(s[None, :], allowed)
            lse[r] = l[0]
            o[r] = P[0] @ V
            if d_o is not None:
                dOi = np.asarray(d_o[b, i, h, :], dtype=np.float64)
                dP = V @ dOi
                Di = np.sum(P[0] * dP)
                dS = P[0] * (dP - Di)
                dqt = sc * (dS @ K)
                if use_rope:
                    dqt = rope_apply(dqt.reshape(1, 1, 1, D), theta, inverse=True,
                                     position_offset=i).reshape(D)
                dq[r] = dqt
    res = {"o": o, "lse": lse}
    if dq is not None:
        res["dq"] = dq
    return res


def attention_decode(q_new, k, v, seg=None, causal=True, theta=1e4, scale=None, heads=None):
    """Decode step: T new query tokens against a cache of S tokens, in float64.

    The new tokens are the last T positions of each row (their own keys and
    values are already the last T entries of ``k``/``v``), the generation
    setting of the research note's sections "模型架构" and "Infra"
    (inference over a million-token context).  Query t sits at position
    p_t = S - T + t and attends exactly as row p_t of ``attention_forward``:
    rotated by R(p_t), keys rotated by R(j), the same mask and softmax.

    q_new [B, T, H, D]; k, v [B, S, H, D] un-rotated; seg [B, S] or None.
    ``heads`` limits the computation to those heads (others stay NaN).
    Returns o [B, T, H, D] and lse [B, H, T].
    """
    q_new = np.asarray(q_new)
    B, T, H, D = q_new.shape
    S = np.asarray(k).shape[1]
    if T > S:
        raise ValueError("more new tokens than cache entries")
    seg = _seg_or_default(seg, B, S)
    sc = _scale(scale, D)
    use_rope = theta is not None and theta > 0
    o = np.full((B, T, H, D), np.nan)
    lse = np.full((B, H, T), np.nan)
    pos = np.arange(S - T, S)
    keys = np.arange(S)
    for b in range(B):
        allowed = allowed_mask(seg[b], pos, keys, causal)  # [T, S]
        for h in (range(H) if heads is None else heads):
            K = np.asarray(k[b, :, h, :], dtype=np.float64)
            Q = np.asarray(q_new[b, :, h, :], dtype=np.float64)
            if use_rope:
                K = rope_apply(K.reshape(1, S, 1, D), theta).reshape(S, D)
                Q = rope_apply(Q.reshape(1, T, 1, D), theta,
                               position_offset=S - T).reshape(T, D)
            s = sc * (Q @ K.T)
            l, P = _softmax_rows(s, allowed)
            lse[b, h] = l
            o[b, :, h, :] = P @ np.asarray(v[b, :, h, :], dtype=np.float64)
    return o, lse


def kept_pairs(seg, causal=True) -> int:
    """Number of allowed (i, j) pairs summed over rows: sum over segments of
    L(L+1)/2 when causal, L^2 otherwise (each id's tokens counted together)."""
    seg = np.asarray(seg)
    total = 0
    for row in seg.reshape(-1, seg.shape[-1]):
        ids, counts = np.unique(row[row >= 0], return_counts=True)
        if causal:
            # causal within a segment counts pairs j <= i that share the id
            total += int(sum(c * (c + 1) // 2 for c in counts))
        else:
            total += int(sum(c * c for c in counts))
    return total


def sample_runs(seg_row):
    """Samples of one packed row: maximal runs of equal non-negative segment
    id, as (start, end) index pairs (research note, "训练方法": each packed
    sample is a contiguous piece of the row)."""
    seg_row = np.asarray(seg_row)
    runs, start = [], 0
    for t in range(1, len(seg_row) + 1):
        if t == len(seg_row) or seg_row[t] != seg_row[t - 1]:
            if seg_row[start] >= 0:
                runs.append((start, t))
            start = t
    return runs


def packed_loss_weights(seg, targets, vocab=None):
    """Per-token loss weights that make packed training equal to unpacked
    training with padding (research note, "训练方法", Masked Sequence
    Packing, and the ablation of section "评测": naive packing down-weights
    short samples).  Unpacked training averages each sample's loss over its
    own loss tokens, then averages over the samples of the batch; so a loss
    token of a sample with n loss tokens weighs 1 / (n * number of samples
    that have a loss token).  A token carries a loss iff its target is a
    class index: 0 <= y (and y < vocab when the vocabulary size is given);
    any other target marks a token without loss (prompts, padding)."""
    seg = np.asarray(seg)
    targets = np.asarray(targets)
    has_loss = targets >= 0
    if vocab is not None:
        has_loss &= targets < vocab
    w = np.zeros(seg.shape, dtype=np.float64)
    samples = []
    for b in range(seg.shape[0]):
        for s, e in sample_runs(seg[b]):
            n = int(np.count_nonzero(has_loss[b, s:e]))
            if n:
                samples.append((b, s, e, n))
    for b, s, e, n in samples:
        w[b, s:e] = np.where(has_loss[b, s:e], 1.0 / (n * len(samples)), 0.0)
    return w


def packed_cross_entropy(logits, targets, seg):
    """Re-weighted cross-entropy of a packed batch and its gradient, float64.

    logits [B, S, V], targets [B, S] (outside [0, V): no loss), seg [B, S].
    Returns (loss, dlogits): loss = sum_t w_t * (logsumexp(z_t) - z_t[y_t]),
    dlogits_t = w_t * (softmax(z_t) - onehot(y_t))."""
    z = np.asarray(logits, dtype=np.float64)
    targets = np.asarray(targets)
    V = z.shape[-1]
    w = packed_loss_weights(seg, targets, vocab=V)
    m = z.max(axis=-1, keepdims=True)
    lse = m[..., 0] + np.log(np.exp(z - m).sum(axis=-1))
    y = np.where((targets >= 0) & (targets < V), targets, 0)
    picked = np.take_along_axis(z, y[..., None], axis=-1)[..., 0]
    loss = float(np.sum(w * (lse - picked)))
    g = np.exp(z - lse[..., None])
    onehot = np.zeros_like(z)
    np.put_along_axis(onehot, y[..., None], 1.0, axis=-1)
    d = w[..., None] * (g - onehot)
    return loss, d
