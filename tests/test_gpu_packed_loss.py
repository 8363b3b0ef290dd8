"""GPU parity of the packed, re-weighted cross-entropy against the oracle.

Rows of packed samples (random segment lengths, padding at the end, tokens
without loss), with and without segment ids, bf16 and fp32 logits.  Row
lengths below and above the 256 chunks of the run-counting kernel make
samples cross chunk edges (the stitching of run totals).  The loss must
match to 1e-4 relative; the gradient within 2e-2 (bf16) or 1e-4 (fp32) of
its largest magnitude, since its values scale with the per-token weights.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import random_segments

pytestmark = pytest.mark.gpu


def run_case(B, S, V, dtype, packed, seed, no_loss_frac=0.2, out_of_vocab_frac=0.0):
    import long_context_causal_attention_b200 as lwm
    rng = np.random.default_rng(seed)
    seg = random_segments(rng, B, S, 5, max(6, S // 4), pad_tail=3) if packed else None
    targets = rng.integers(0, V, size=(B, S)).astype(np.int32)
    targets[rng.random((B, S)) < no_loss_frac] = -1   # tokens without loss (prompts)
    oov = rng.random((B, S)) < out_of_vocab_frac        # targets >= V: no loss either
    targets[oov] = V + rng.integers(0, 3 * V, size=int(oov.sum()))
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    logits = (torch.randn((B, S, V), generator=g, device="cuda") * 2.0).to(dtype)
    t_d = torch.as_tensor(targets, device="cuda")
    s_d = torch.as_tensor(seg, dtype=torch.int32, device="cuda") if packed else None
    loss, d = lwm.lwm_packed_cross_entropy(logits, t_d, s_d, check_status=True)
    torch.cuda.synchronize()
    z = logits.double().cpu().numpy()
    ref_loss, ref_d = oracle.packed_cross_entropy(z, targets,
                                                  seg if packed else np.zeros((B, S), np.int32))
    assert abs(loss.item() - ref_loss) <= 1e-4 * abs(ref_loss), (loss.item(), ref_loss)
    scale = np.abs(ref_d).max()
    err = np.abs(d.double().cpu().numpy() - ref_d).max()
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    assert err <= tol * scale, (err, scale)


@pytest.mark.parametrize("B,S,V,dtype,packed", [
    (3, 700, 1000, torch.bfloat16, True),
    (2, 700, 1000, torch.float32, True),
    (2, 513, 776, torch.bfloat16, False),
    (1, 5000, 2048, torch.bfloat16, True),
    (1, 2048, 32000, torch.bfloat16, True),
    (1, 600, 32768, torch.bfloat16, True),    # largest bf16 row: 64 KB, three ring stages
    (1, 400, 16384, torch.float32, True),     # largest fp32 row
    (2, 3000, 8, torch.bfloat16, True),       # 16-byte rows: sixteen stages, many rows per CTA
    (1, 5, 64, torch.float32, False),         # fewer rows than SMs
])
def test_packed_cross_entropy(B, S, V, dtype, packed):
    run_case(B, S, V, dtype, packed, seed=B * 1000 + S)


def test_packed_cross_entropy_no_loss_rows():
    """Long stretches of rows without a loss pass through the row ring with
    no data: most rows here carry none."""
    run_case(2, 1500, 1024, torch.bfloat16, True, seed=77, no_loss_frac=0.9)


def test_packed_cross_entropy_out_of_vocabulary_targets():
    """Targets >= V carry no loss: they must not count towards their
    sample's token count n nor make a sample count, in the run-counting
    kernel as in the loss kernel."""
    run_case(2, 900, 504, torch.bfloat16, True, seed=91, out_of_vocab_frac=0.3)
    run_case(1, 300, 64, torch.float32, True, seed=92, no_loss_frac=0.0, out_of_vocab_frac=0.6)
