"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no attention arithmetic: it only names the workloads and
draws their inputs.  Both the CUDA path's callers and the oracle's callers use
it, so the two sides always see the same tensors.

Workloads (shapes follow the Large World Model pages: LLaMA-2-7B heads,
32 x 128; context lengths and RoPE theta from the research note's training
tables, section "训练方法"; packed vision/text rows from the note's section
"数据" (16x16 VQ tokens per frame plus an <eof>/<eov> marker, packed with text
into one sequence)):

  tiny_packed_fp32  B1 H1 D64 fp32, S=256, segments 100 + 156, theta 1e4, fwd
  fwd_32k           B1 H32 D128 bf16, S=32768, one segment, theta 1e6, fwd
  packed_8k         B4 H32 D128 bf16, S=8192 packed video/text, theta 1e6, fwd+bwd
  long_128k         B1 H32 D128 bf16, S=131072, one segment, theta 1e7, fwd+bwd
  million_1m        B1 H32 D128 bf16, S=1048576, one segment, theta 5e7, fwd+bwd
  decode_1m         B1 H32 D128 bf16, one new token against a 1048576-token
                    cache (the new token's own key and value included), theta 5e7
  fp32_8k           B1 H32 D128 fp32, S=8192, one segment, theta 1e6, fwd+bwd
  packed_loss_8k    packed_8k's rows, bf16 logits over a 32000-token vocabulary,
                    re-weighted cross-entropy and its gradient
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

FRAME_TOKENS = 257  # 16 x 16 VQ codes + one <eof>/<eov> marker


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    heads: int
    head_dim: int
    dtype: str            # "bf16" or "fp32"
    theta: float
    causal: bool = True
    sigma: float = 0.5    # std of q, k, v
    segments: str = "single"   # "single", "two_100_156", "packed_video_text"
    backward: bool = True
    scale: float = 0.0    # <= 0 means 1/sqrt(head_dim)
    extra: dict = field(default_factory=dict)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_packed_fp32": Workload("tiny_packed_fp32", 1, 256, 1, 64, "fp32", 1e4,
                                 sigma=1.0, segments="two_100_156", backward=False),
    "fwd_32k": Workload("fwd_32k", 1, 32768, 32, 128, "bf16", 1e6, backward=False),
    "packed_8k": Workload("packed_8k", 4, 8192, 32, 128, "bf16", 1e6,
                          segments="packed_video_text"),
    "long_128k": Workload("long_128k", 1, 131072, 32, 128, "bf16", 1e7),
    "million_1m": Workload("million_1m", 1, 1048576, 32, 128, "bf16", 5e7),
    # profiling case: same head shape, 16K tokens (each tensor 128 MiB, above L2)
    "prof_16k": Workload("prof_16k", 1, 16384, 32, 128, "bf16", 1e6),
    # decode step: n_new new tokens, the cache of `seqlen` tokens includes them
    "decode_1m": Workload("decode_1m", 1, 1048576, 32, 128, "bf16", 5e7, backward=False,
                          extra={"n_new": 1}),
    # fp32 end to end (the pages train in fp32) at 8K tokens: the split-precision
    # tensor-core path (LWM_ATTN_FP32_SIMT=1: the CUDA-core kernels)
    "fp32_8k": Workload("fp32_8k", 1, 8192, 32, 128, "fp32", 1e6),
    # packed loss re-weighting: the packed_8k rows, LLaMA vocabulary (32000)
    "packed_loss_8k": Workload("packed_loss_8k", 4, 8192, 32, 128, "bf16", 1e6,
                               segments="packed_video_text", backward=False,
                               extra={"vocab": 32000}),
    # decode profiling case: 128K-token cache (2 GiB of keys and values, above L2)
    "prof_decode_128k": Workload("prof_decode_128k", 1, 131072, 32, 128, "bf16", 1e7,
                                 backward=False, extra={"n_new": 1}),
}
ORDER = ["tiny_packed_fp32", "fwd_32k", "packed_8k", "long_128k", "million_1m"]


def packed_video_text_row(rng: np.random.Generator, seqlen: int) -> np.ndarray:
    """One packed row: alternate a video segment of 257*k tokens (k uniform in
    1..30) and a text segment of uniform 32..1024 tokens, starting with video,
    the last segment cut so the row holds exactly ``seqlen`` tokens.  Segment
    ids count up from 0."""
    ids = np.empty(seqlen, dtype=np.int32)
    pos, sid, video = 0, 0, True
    while pos < seqlen:
        if video:
            n = FRAME_TOKENS * int(rng.integers(1, 31))
        else:
            n = int(rng.integers(32, 1025))
        n = min(n, seqlen - pos)
        ids[pos:pos + n] = sid
        pos += n
        sid += 1
        video = not video
    return ids


def segment_ids(w: Workload, seed: int = 0) -> np.ndarray:
    """int32 [B, S] segment ids for a workload (numpy default_rng(seed))."""
    if w.segments == "single":
        return np.zeros((w.batch, w.seqlen), dtype=np.int32)
    if w.segments == "two_100_156":
        assert w.seqlen == 256
        row = np.concatenate([np.zeros(100, np.int32), np.ones(156, np.int32)])
        return np.tile(row, (w.batch, 1))
    if w.segments == "packed_video_text":
        rng = np.random.default_rng(seed)
        return np.stack([packed_video_text_row(rng, w.seqlen) for _ in range(w.batch)])
    raise ValueError(w.segments)


def random_segments(rng: np.random.Generator, batch: int, seqlen: int, min_len=1,
                    max_len=300, pad_tail=0) -> np.ndarray:
    """Contiguous runs of random lengths with increasing ids; optional padding
    (id -1) on the last ``pad_tail`` tokens of each row (edge-case inputs)."""
    out = np.empty((batch, seqlen), dtype=np.int32)
    for b in range(batch):
        pos, sid = 0, 0
        while pos < seqlen:
            n = min(int(rng.integers(min_len, max_len + 1)), seqlen - pos)
            out[b, pos:pos + n] = sid
            pos += n
            sid += 1
        if pad_tail:
            out[b, seqlen - pad_tail:] = -1
    return out


def torch_dtype(name: str):
    import torch
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_tensors(w: Workload, seed: int = 0, device="cpu", with_grad_out=None):
    """Draw q, k, v (and dO) in that order from one seeded torch generator.

    q, k, v ~ N(0, 1) * sigma and dO ~ N(0, 1), drawn in float32 and rounded
    to the workload dtype (round to nearest even).  Layout [B, S, H, D]."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    shape = (w.batch, w.seqlen, w.heads, w.head_dim)
    dt = torch_dtype(w.dtype)
    out = {}
    for name in ("q", "k", "v"):
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        out[name] = (t * w.sigma).to(dt)
    if with_grad_out if with_grad_out is not None else w.backward:
        out["do"] = torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dt)
    return out


THETA_SCHEDULE = {32768: 1e6, 131072: 1e7, 262144: 1e7, 524288: 2.5e7, 1048576: 5e7}
