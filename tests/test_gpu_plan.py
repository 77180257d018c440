"""The attention kernel's work plan against a plain restatement of its rule,
on the GPU's own block masks.

With 64-token blocks two query blocks share a 128-row tile.  The planner
pairs them: rounds of mutual-best-partner matching among blocks at most 32
positions apart, weighted by the number of KV blocks both keep (ties to the
nearer, then the lower index), at most 6 rounds or until a round forms no
pair; the blocks left over are paired in index order (an odd one out is a
tile of its own).  Tiles of each (batch, head) are ordered by decreasing
union size (the union counted exactly for partners within the window, as
the sum of the two counts beyond it), ties in any order.  With 128-token
blocks every block is a tile, ordered by its count.

The plan decides only the schedule, never the result (the parity tests
cover that); this test pins the schedule itself: the same tiles, each block
in exactly one, in an order of non-increasing size.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_fractal_b200 import synth

from _util import lists_to_keep, small

pytestmark = pytest.mark.gpu

WINDOW = 32
ROUNDS = 6

CASES = [
    synth.WORKLOADS["tiny"],
    small("plan_ragged64_odd", 1, 3, 20, 28, 2, 128, 64, 8, 0.15),     # nb = 27
    small("plan_batch2", 2, 2, 16, 24, 2, 64, 64, 8, 0.25),
    small("plan_hybrid", 1, 4, 24, 24, 2, 128, 64, 8, 0.2, sta=(1, 1, 1)),
    small("plan_ragged128", 1, 2, 13, 37, 3, 64, 128, 4, 0.3),
    synth.WORKLOADS["wan480p"],
]


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as m
    return m


def expected_tiles(keep: np.ndarray, paired: bool) -> dict:
    """{(first block, second block or -1): union size} of one (batch, head)."""
    nb = keep.shape[0]
    cnt = keep.sum(axis=1).astype(np.int64)
    if not paired:
        return {(r, -1): int(min(max(cnt[r], 1), nb)) for r in range(nb)}
    k = keep.astype(np.int64)
    overlap = k @ k.T
    partner = [-1] * nb
    for _ in range(ROUNDS):
        choice = [-1] * nb
        for r in range(nb):
            if partner[r] >= 0:
                continue
            best, bestw = -1, -1
            for off in range(1, WINDOW + 1):
                lo, hi = r - off, r + off
                if lo >= 0 and partner[lo] < 0 and overlap[lo, r] > bestw:
                    best, bestw = lo, overlap[lo, r]
                if hi < nb and partner[hi] < 0 and overlap[r, hi] > bestw:
                    best, bestw = hi, overlap[r, hi]
            choice[r] = best
        formed = False
        for r in range(nb):
            j = choice[r]
            if partner[r] < 0 and j >= 0 and choice[j] == r:
                partner[r] = j
                formed = True
        if not formed:
            break
    left = [r for r in range(nb) if partner[r] < 0]
    for i in range(0, len(left), 2):
        a = left[i]
        b = left[i + 1] if i + 1 < len(left) else a
        partner[a], partner[b] = b, a
    tiles = {}
    for r in range(nb):
        p = partner[r]
        if p < r:
            continue
        if p == r:
            u = cnt[r]
        else:
            u = cnt[r] + cnt[p] - (overlap[r, p] if p - r <= WINDOW else 0)
        tiles[(r, p if p != r else -1)] = int(min(max(u, 1), nb))
    return tiles


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_plan_matches_the_rule(bsa, w):
    q, k, v = synth.make_qkv(w)
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    plan = bsa.NablaAttention(s)
    plan.reorder_inputs(q.cuda(), k.cuda(), v.cuda())
    plan.join_side()
    plan.mask_step(w.thr, w.sta)
    plan.attention_step()
    torch.cuda.synchronize()
    assert plan.status() == 0
    nb = plan.nb
    paired = w.block == 64
    per_bh = -(-nb // 2) if paired else nb
    n = w.B * w.heads * per_bh
    off = bsa.plan_items_offset(s)
    items = plan.ws[off:off + 8 * n].view(torch.int32).view(w.B * w.heads, per_bh, 2).cpu().numpy()
    keep = lists_to_keep(plan.kv_count, plan.kv_idx, nb).reshape(-1, nb, nb)
    for bh in range(w.B * w.heads):
        want = expected_tiles(keep[bh], paired)
        got = [(int(a), int(b)) for a, b in items[bh]]
        assert sorted(got) == sorted(want), f"head {bh}: tiles differ"
        sizes = [want[t] for t in got]
        assert all(x >= y for x, y in zip(sizes, sizes[1:])), f"head {bh}: tiles not in decreasing size"
        blocks = [b for t in got for b in t if b >= 0]
        assert sorted(blocks) == list(range(nb)), f"head {bh}: not a partition of the blocks"
