"""GPU parity of bsa_attn_fwd_fine (AB-Attention article, "Los tres recursos
de AB-Attention": 4-token KV blocks gathered by index, SIP inclusion weights)
against the fp64 oracle, oracle.fine_attention:

* small shapes, every row: ragged lists (empty ones, exactly one tile, one
  entry past a tile, several tiles per softmax group), a last 4-token block
  that straddles N, d = 64 and 128, with and without weights, repeated and
  unsorted entries: O within max-abs 2e-2 / mean-abs 2e-3 and the LSE within
  2e-3 (the attention tolerances);
* the Wan-480p shape (12 heads, 32760 tokens) with 10.8 % of the 4-token
  blocks per query block, weighted, in the launch configuration the bench
  times: sampled query blocks (the last, ragged one included) row by row;
* invalid entries (an index past the sequence, a weight <= 0) are skipped
  and reported as BSA_ERR_DEVICE_INDEX; the forced-timeout hook reports
  BSA_ERR_TIMEOUT and the next call computes normally.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_fractal_b200 import synth

from _util import LSE_ABS, MAX_ABS, MEAN_ABS, compare_outputs, small, to64

pytestmark = pytest.mark.gpu

KB = 4   # tokens of a KV block


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as m
    return m


def _inputs(w):
    """q, k, v as bf16 [B, heads, Npad, d] (token order as drawn, rows >= N zero)."""
    out = []
    for x in synth.make_qkv(w):
        y = torch.zeros(w.B, w.heads, w.Npad, w.d, dtype=torch.bfloat16)
        y[:, :, :w.N] = x.permute(0, 2, 1, 3)
        out.append(y)
    return out


def _run(bsa, w, q, k, v, off, idx, wt, lse=True):
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    ws = torch.zeros(bsa.attn_fine_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    o = torch.full((w.B, w.heads, w.Npad, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    l = torch.full((w.B, w.heads, w.Npad), float("nan"), dtype=torch.float32, device="cuda") if lse else None
    bsa.attn_fwd_fine(s, q.cuda(), k.cuda(), v.cuda(), off.cuda(), idx.cuda(),
                      None if wt is None else wt.cuda(), 0.0, o, l, ws)
    status = bsa.check_device_status(ws)
    return o, l, status


def _check_all(w, q, k, v, off, idx, wt, o, l):
    O_ref, lse_ref = oracle.fine_attention(to64(q), to64(k), to64(v), off.numpy(), idx.numpy(),
                                           None if wt is None else wt.numpy().astype(np.float64), w.N)
    O = to64(o)
    assert not np.isnan(O).any()
    assert np.all(O[:, :, w.N:] == 0)
    mx, mean = compare_outputs(O[:, :, :w.N], O_ref[:, :, :w.N])
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    if l is not None:
        L = to64(l)
        assert np.abs(L[:, :, :w.N] - lse_ref[:, :, :w.N]).max() <= LSE_ABS
        assert np.all(L[:, :, w.N:] == 0)


# (workload, fraction of the 4-token blocks, ragged list lengths, weighted)
CASES = [
    (small("fine_ragged", 1, 3, 11, 17, 2, 128, 128, 8, 0.0, seed=41), 0.2, True, True),
    (small("fine_ragged_unweighted", 1, 3, 11, 17, 2, 128, 128, 8, 0.0, seed=42), 0.2, True, False),
    (small("fine_d64", 2, 2, 13, 20, 2, 64, 128, 8, 0.0, seed=43), 0.3, True, True),
    (small("fine_long", 1, 4, 16, 16, 2, 128, 128, 8, 0.0, seed=44), 0.9, False, True),
    (small("fine_d64_long", 1, 5, 16, 13, 3, 64, 128, 8, 0.0, seed=45), 0.7, True, False),
]


@pytest.mark.parametrize("w,frac,ragged,weighted", CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_fine_attention_matches_oracle(bsa, w, frac, ragged, weighted):
    q, k, v = _inputs(w)
    nq, nkb = w.Npad // 128, -(-w.N // KB)
    off, idx, wt = synth.random_fine_lists(w.B, w.heads, nq, nkb, frac, w.seed, ragged=ragged)
    if not weighted:
        wt = None
    o, l, status = _run(bsa, w, q, k, v, off, idx, wt)
    assert status == 0
    _check_all(w, q, k, v, off, idx, wt, o, l)


def test_list_lengths_around_a_tile(bsa):
    """Lists of 0 to 200 entries around the tile boundaries (32 entries a
    tile), each ending on the 4-token block that straddles N."""
    w = small("fine_tile_edges", 1, 7, 11, 17, 1, 128, 128, 8, 0.0, seed=46)   # N = 1309 = 4 * 327 + 1
    q, k, v = _inputs(w)
    nq, nkb = w.Npad // 128, -(-w.N // KB)
    lens = [0, 1, 31, 32, 33, 63, 64, 65, 96, 97, 200]
    assert len(lens) == nq and w.N % KB != 0
    g = torch.Generator().manual_seed(7)
    rows = []
    for r, n in enumerate(lens):
        row = torch.sort(torch.randperm(nkb - 1, generator=g)[:n]).values
        if n:
            row[-1] = nkb - 1      # the block holding keys >= N
        rows.append(row)
    off = torch.zeros(nq + 1, dtype=torch.int64)
    off[1:] = torch.cumsum(torch.tensor([len(x) for x in rows]), 0)
    idx = torch.cat(rows).to(torch.int32)
    wt = (1.0 + 3.0 * torch.rand(idx.numel(), generator=g)).to(torch.float32)
    o, l, status = _run(bsa, w, q, k, v, off, idx, wt)
    assert status == 0
    _check_all(w, q, k, v, off, idx, wt, o, l)
    assert np.all(to64(o)[0, 0, :128] == 0) and np.all(to64(l)[0, 0, :128] == 0)   # the empty list


def test_repeated_and_unsorted_entries(bsa):
    """Entries in any order; a repeated entry counts once more (the oracle's
    definition), i.e. like a weight of 2."""
    w = small("fine_repeat", 1, 2, 16, 16, 2, 128, 128, 8, 0.0, seed=47)
    q, k, v = _inputs(w)
    nq, nkb = w.Npad // 128, -(-w.N // KB)
    off, idx, wt = synth.random_fine_lists(w.B, w.heads, nq, nkb, 0.25, w.seed)
    g = torch.Generator().manual_seed(8)
    rows, wrows = [], []
    for r in range(off.numel() - 1):
        lo, hi = int(off[r]), int(off[r + 1])
        perm = torch.randperm(hi - lo, generator=g)
        extra = perm[: (hi - lo) // 4]
        rows.append(torch.cat([idx[lo:hi][perm], idx[lo:hi][extra]]))
        wrows.append(torch.cat([wt[lo:hi][perm], wt[lo:hi][extra]]))
    off2 = torch.zeros_like(off)
    off2[1:] = torch.cumsum(torch.tensor([len(x) for x in rows]), 0)
    idx2, wt2 = torch.cat(rows), torch.cat(wrows)
    o, l, status = _run(bsa, w, q, k, v, off2, idx2, wt2)
    assert status == 0
    _check_all(w, q, k, v, off2, idx2, wt2, o, l)


def test_whole_blocks_give_block_sparse_attention(bsa):
    """Selecting every 4-token block of the kept 128-token blocks, unweighted,
    is the block-sparse attention of those blocks: both kernels against the
    same oracle, and against each other."""
    w = small("fine_vs_block", 1, 3, 16, 20, 2, 128, 128, 8, 0.0, seed=48)
    q, k, v = _inputs(w)
    nq = w.Npad // 128
    kv_count, kv_idx = synth.random_block_lists(w.B, w.heads, nq, 0.5, w.seed)
    rows = []
    for r in range(w.B * w.heads * nq):
        blocks = kv_idx.view(-1, nq)[r, : int(kv_count.view(-1)[r])]
        rows.append(torch.cat([torch.arange(int(J) * 32, min((int(J) + 1) * 32, -(-w.N // KB))) for J in blocks]))
    off = torch.zeros(len(rows) + 1, dtype=torch.int64)
    off[1:] = torch.cumsum(torch.tensor([len(x) for x in rows]), 0)
    idx = torch.cat(rows).to(torch.int32)
    o, l, status = _run(bsa, w, q, k, v, off, idx, None)
    assert status == 0
    keep = np.zeros((w.B, w.heads, nq, nq), dtype=bool)
    cnt, kvi = kv_count.numpy().reshape(-1), kv_idx.numpy().reshape(-1, nq)
    for r in range(cnt.size):
        keep.reshape(-1, nq)[r, kvi[r, :cnt[r]]] = True
    O_ref, lse_ref = oracle.masked_attention(to64(q), to64(k), to64(v), keep, w.N, 128)
    mx, mean = compare_outputs(to64(o)[:, :, :w.N], O_ref[:, :, :w.N])
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    assert np.abs(to64(l)[:, :, :w.N] - lse_ref[:, :, :w.N]).max() <= LSE_ABS
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    ws = torch.zeros(bsa.workspace_bytes(s), dtype=torch.uint8, device="cuda")
    o2 = torch.empty_like(o)
    bsa.attn_fwd(s, q.cuda(), k.cuda(), v.cuda(), kv_count.cuda(), kv_idx.cuda(), 0.0, o2, None, ws)
    assert bsa.check_device_status(ws) == 0
    mx, _ = compare_outputs(to64(o2)[:, :, :w.N], to64(o)[:, :, :w.N])
    assert mx <= 2 * MAX_ABS


def test_invalid_entries_are_skipped_and_reported(bsa):
    w = small("fine_invalid", 1, 2, 16, 16, 2, 128, 128, 8, 0.0, seed=49)
    q, k, v = _inputs(w)
    nq, nkb = w.Npad // 128, -(-w.N // KB)
    off, idx, wt = synth.random_fine_lists(w.B, w.heads, nq, nkb, 0.3, w.seed)
    for bad_idx, bad_w in ((True, False), (False, True)):
        idx2, wt2 = idx.clone(), wt.clone()
        pos = int(off[1]) + 3
        if bad_idx:
            idx2[pos] = nkb + 5
        if bad_w:
            wt2[pos] = -1.0
        o, l, status = _run(bsa, w, q, k, v, off, idx2, wt2)
        assert status == 4                        # BSA_ERR_DEVICE_INDEX
        # the same as the list without that entry
        keep = torch.ones(idx.numel(), dtype=torch.bool)
        keep[pos] = False
        off3 = off.clone()
        off3[2:] -= 1
        _check_all(w, q, k, v, off3, idx[keep], wt[keep], o, l)


def test_forced_timeout_is_reported_and_the_next_call_computes(bsa, monkeypatch):
    w = small("fine_timeout", 1, 2, 16, 16, 2, 128, 128, 8, 0.0, seed=50)
    q, k, v = _inputs(w)
    nq, nkb = w.Npad // 128, -(-w.N // KB)
    off, idx, wt = synth.random_fine_lists(w.B, w.heads, nq, nkb, 0.3, w.seed)
    monkeypatch.setenv("BSA_TEST_FORCE_TIMEOUT", "1")
    _, _, status = _run(bsa, w, q, k, v, off, idx, wt)
    assert status == 5                            # BSA_ERR_TIMEOUT
    monkeypatch.delenv("BSA_TEST_FORCE_TIMEOUT")
    o, l, status = _run(bsa, w, q, k, v, off, idx, wt)
    assert status == 0
    _check_all(w, q, k, v, off, idx, wt, o, l)


def test_wan480p_sampled_query_blocks(bsa):
    """The Wan-480p shape at the page's budget (10.8 % of the keys), weighted,
    in the bench's launch configuration; 16 query blocks checked row by row
    against the oracle, the last (120 valid rows) among them."""
    base = synth.WORKLOADS["wan480p"]
    w = synth.Workload("wan480p_fine", base.B, base.T, base.H, base.W, base.heads, base.d, 128, base.patch, 0.0,
                       None, base.alpha, base.seed)
    q, k, v = _inputs(w)
    nq, nkb = w.Npad // 128, -(-w.N // KB)
    off, idx, wt = synth.random_fine_lists(w.B, w.heads, nq, nkb, 0.108, w.seed)
    o, l, status = _run(bsa, w, q, k, v, off, idx, wt)
    assert status == 0
    rng = np.random.default_rng(5)
    picks = {(0, w.heads - 1, nq - 1)} | {(0, int(h), int(I)) for h, I in
                                          zip(rng.integers(0, w.heads, 15), rng.integers(0, nq, 15))}
    O, L = o.float().cpu(), l.cpu()
    for (b, h, I) in sorted(picks):
        r = (b * w.heads + h) * nq + I
        lo, hi = I * 128, min((I + 1) * 128, w.N)
        e0, e1 = int(off[r]), int(off[r + 1])
        O_ref, lse_ref = oracle.fine_attention_block(
            to64(q[b, h, lo:hi]), to64(k[b, h]), to64(v[b, h]), idx[e0:e1].numpy(),
            wt[e0:e1].numpy().astype(np.float64), w.N)
        mx, mean = compare_outputs(O[b, h, lo:hi].double().numpy(), O_ref)
        assert mx <= MAX_ABS and mean <= MEAN_ABS, ((b, h, I), mx, mean)
        assert np.abs(L[b, h, lo:hi].double().numpy() - lse_ref).max() <= LSE_ABS


def test_weights_past_the_unchecked_range(bsa):
    """Entries of every tile after the first two weighted 2^70: each group's
    logits jump by 70 (log2 units) after its first tile, past the range the
    kernel accepts without a max pass, so every query block redoes a tile with
    a new max (O, sums and stored weights rescaled)."""
    w = small("fine_jump", 1, 4, 16, 16, 2, 128, 128, 8, 0.0, seed=51)
    q, k, v = _inputs(w)
    nq, nkb = w.Npad // 128, -(-w.N // KB)
    off, idx, wt = synth.random_fine_lists(w.B, w.heads, nq, nkb, 0.6, w.seed)
    wt = torch.ones_like(wt)
    for r in range(off.numel() - 1):
        lo, hi = int(off[r]), int(off[r + 1])
        wt[lo + 64:hi] = 2.0 ** 70
    o, l, status = _run(bsa, w, q, k, v, off, idx, wt)
    assert status == 0
    _check_all(w, q, k, v, off, idx, wt, o, l)
