"""Reference oracle for blockwise causal attention with RoPE and masked packing.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It is a plain, slow, float64 CPU restatement of
what the method computes, written from the method's description and never
from the CUDA code.  It shares no code, tables or constants with the CUDA
path.

Sources (the pages describing Large World Model):

* LWM research note (zhao9797.github.io), section "模型架构" (model
  architecture): exact blockwise RingAttention fused with FlashAttention,
  "standard RoPE" with a scaled theta.
* Same note, section "训练方法" (training method): the theta schedule per
  context length and "Masked Sequence Packing" (each packed pair attends only
  to itself; numerically equal to unpacked training with padding).
* Paper card "World Model on Million-Length Video And Language With
  Blockwise RingAttention" (research.elamur.ai), Summary: attention over very
  long sequences "without approximation"; reference list entries RoFormer
  (rotary embedding) and FlashAttention (blockwise exact softmax).

Every function states which of these it follows.  Readings of points the
pages leave open are listed in ``oracle.attention.READINGS``.

Parity pins: every function here is pinned by ``tests/test_oracle.py``
against something other than itself (torch fp64 SDPA and autograd, a scalar
brute force, closed forms, invariants).  No function is "parity unpinned".
"""

from .attention import (  # noqa: F401
    READINGS,
    rope_frequencies,
    rope_angles,
    rope_apply,
    allowed_mask,
    attention_forward,
    attention_backward,
    attention_rows,
    attention_decode,
    sample_runs,
    packed_loss_weights,
    packed_cross_entropy,
    kept_pairs,
)
