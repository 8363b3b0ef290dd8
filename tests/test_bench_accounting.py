"""Host-side accounting of bench.py, CPU only: the algorithmic pair count
behind every TFLOP/s figure and the tile-pair count reported with the
roofline, each against a brute-force count over the mask itself."""
import numpy as np
import pytest

import bench
from workloads import WORKLOADS, random_segments, segment_ids


def brute_pairs(seg, causal):
    total = 0
    for row in seg:
        ok = (row[:, None] == row[None, :]) & (row[:, None] >= 0)
        if causal:
            ok &= np.tril(np.ones((len(row), len(row)), dtype=bool))
        total += int(ok.sum())
    return total


@pytest.mark.parametrize("causal", [True, False])
def test_kept_pairs_equals_mask_count(causal):
    rng = np.random.default_rng(5)
    seg = random_segments(rng, 3, 300, 1, 60, pad_tail=7)
    seg[1, 10:20] = -1                      # padding inside a row
    seg[2, 250:260] = seg[2, 5]             # an id that comes back later
    assert bench.kept_pairs(seg, causal) == brute_pairs(seg, causal)


def brute_tile_pairs(seg, heads, tile=128):
    total = 0
    for row in seg:
        n = (len(row) + tile - 1) // tile
        ids = [set(row[t * tile:(t + 1) * tile][row[t * tile:(t + 1) * tile] >= 0].tolist())
               for t in range(n)]
        total += sum(1 for qt in range(n) for kt in range(qt + 1) if ids[qt] & ids[kt])
    return total * heads


def test_tile_pairs_of_packed_rows_equal_tiles_sharing_an_id():
    """For ids in contiguous runs (what packing produces) two tiles' id ranges
    meet exactly when the tiles share an id, and every causal pair of such
    tiles then holds an allowed (query, key) pair."""
    w = WORKLOADS["packed_8k"]
    seg = segment_ids(w, seed=3)
    assert bench.tile_pairs(seg, heads=2) == brute_tile_pairs(seg, heads=2)


def test_single_segment_counts_are_the_causal_triangle():
    S, heads, tile = 131072, 32, 128
    seg = np.zeros((1, S), np.int32)
    assert bench.kept_pairs(seg) == S * (S + 1) // 2
    n = S // tile
    assert bench.tile_pairs(seg, heads) == heads * n * (n + 1) // 2


def test_loss_bytes_count_only_the_logit_rows_read():
    """Packed-loss bytes: logits of loss tokens (target in [0, V), segment id
    >= 0) read once, every gradient row written once, targets and segment
    ids read once; counted token by token here."""
    rng = np.random.default_rng(9)
    B, S, V, elt = 2, 50, 40, 2
    seg = random_segments(rng, B, S, 3, 15, pad_tail=4)
    targets = rng.integers(-1, V + 5, size=(B, S)).astype(np.int32)
    read = 0
    for b in range(B):
        for t in range(S):
            if 0 <= targets[b, t] < V and seg[b, t] >= 0:
                read += V * elt
    want = read + B * S * V * elt + B * S * 8
    assert bench.loss_bytes(V, elt, targets, seg) == want
