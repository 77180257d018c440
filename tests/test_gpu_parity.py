"""GPU parity: every C-ABI call against the fp64 oracle on the same seeded inputs.

* reorder / inverse reorder: bit-exact;
* block mask: bit-exact except blocks the oracle flags as ambiguous (prefix
  mass within 1e-6 of 1 - thr, or a near-tie with the boundary block), which
  are counted;
* attention, with the oracle's mask fed to the kernel: max-abs <= 2e-2 and
  mean-abs <= 2e-3 on the valid rows, LSE within 2e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_fractal_b200 import synth

from _util import LSE_ABS, MAX_ABS, MEAN_ABS, compare_outputs, lists_to_keep, small, to64

pytestmark = pytest.mark.gpu

SMALL = [
    synth.WORKLOADS["tiny"],
    small("ragged64", 1, 3, 20, 28, 2, 128, 64, 8, 0.15),
    small("ragged128_d64", 1, 2, 13, 37, 3, 64, 128, 4, 0.3),
    small("batch2_d64", 2, 2, 16, 24, 2, 64, 64, 8, 0.25),
    small("hybrid_small", 1, 4, 24, 24, 2, 128, 64, 8, 0.2, sta=(1, 1, 1)),
    small("dense_thr0", 1, 2, 12, 20, 2, 128, 128, 4, 0.0),
    small("one_block", 1, 1, 5, 7, 2, 64, 64, 8, 0.1),
    small("sharp", 1, 3, 16, 16, 2, 128, 64, 8, 0.05, alpha=2.0),
]

# Larger values than the pages' workloads: |O| reaches 8 and more, where one
# bf16 ulp (1/16) already exceeds the absolute bound.  Checked against the
# bound plus half a bf16 ulp of the reference value.
HOT = small("hot", 1, 3, 16, 16, 2, 128, 64, 8, 0.05, alpha=3.0)


def _half_ulp_bf16(x):
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 0.5 * 2.0 ** (np.floor(np.log2(ax)) - 7)


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as m
    return m


def _shape(bsa, w):
    return bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)


def _run_mask(bsa, w, plan, q, k, fused=True):
    """The block mask of q, k (model order) into the plan's lists: the fused
    path (Q/K reorder with the block means, then the mask from those means)
    or the separate one (reorder, then pooling and mask from the reordered
    tensors)."""
    if fused:
        bsa.reorder_qk_pooled(plan.shape, q, k, plan.q, plan.k, plan.ws)
        plan.mask_step(w.thr, w.sta)
    else:
        bsa.reorder(plan.shape, q, plan.q)
        bsa.reorder(plan.shape, k, plan.k)
        bsa.build_block_mask(plan.shape, plan.q, plan.k, w.thr, w.sta, plan.kv_count, plan.kv_idx, plan.mask,
                             plan.ws)
    torch.cuda.synchronize()


def _reorder_all(bsa, plan, q, k, v):
    bsa.reorder_qk_pooled(plan.shape, q.cuda(), k.cuda(), plan.q, plan.k, plan.ws)
    bsa.reorder(plan.shape, v.cuda(), plan.v)


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_reorder_bit_exact(bsa, w):
    q, _, _ = synth.make_qkv(w)
    s = _shape(bsa, w)
    Npad = bsa.padded_len(s)
    qd = q.cuda()
    y = torch.full((w.B, w.heads, Npad, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    bsa.reorder(s, qd, y)
    want = oracle.reorder(to64(q), w.T, w.H, w.W, w.patch, w.block)
    assert np.array_equal(to64(y), want)
    back = torch.full_like(qd, float("nan"))
    bsa.inverse_reorder(s, y, back)
    assert torch.equal(back, qd)
    assert np.array_equal(to64(back), oracle.inverse_reorder(want, w.T, w.H, w.W, w.patch))


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_fused_qk_reorder_and_block_means(bsa, w):
    """bsa_reorder_qk_pooled: both reorders bit-exact, and the block means it
    leaves in the workspace equal the oracle's (sums of bf16 values in double
    are exact here, so the means agree to the last bit)."""
    q, k, _ = synth.make_qkv(w)
    s = _shape(bsa, w)
    Npad, nb = bsa.padded_len(s), bsa.num_blocks(s)
    yq = torch.full((w.B, w.heads, Npad, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    yk = torch.full_like(yq, float("nan"))
    ws = torch.full(((bsa.workspace_bytes(s) + 15) // 16 * 16,), 0xFF, dtype=torch.uint8, device="cuda")
    bsa.workspace_init(ws)
    bsa.reorder_qk_pooled(s, q.cuda(), k.cuda(), yq, yk, ws)
    torch.cuda.synchronize()
    want_q = oracle.reorder(to64(q), w.T, w.H, w.W, w.patch, w.block)
    want_k = oracle.reorder(to64(k), w.T, w.H, w.W, w.patch, w.block)
    assert np.array_equal(to64(yq), want_q) and np.array_equal(to64(yk), want_k)
    n = w.B * w.heads * nb * w.d
    means = ws[256:256 + 16 * n].view(torch.float64).cpu().numpy()
    qbar = means[:n].reshape(w.B, w.heads, nb, w.d)
    kbar = means[n:].reshape(w.B, w.heads, w.d, nb).swapaxes(-1, -2)
    assert np.array_equal(qbar, oracle.block_means(want_q, w.N, w.block))
    assert np.array_equal(kbar, oracle.block_means(want_k, w.N, w.block))


@pytest.mark.parametrize("fused", [True, False], ids=["fused_pool", "separate_pool"])
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_block_mask_matches_oracle(bsa, w, fused):
    q, k, _ = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w), with_mask=True)
    _run_mask(bsa, w, plan, q.cuda(), k.cuda(), fused)
    assert plan.status() == 0
    keep_ref, amb = oracle.block_mask(to64(plan.q), to64(plan.k), w.T, w.H, w.W, w.patch, w.block, w.thr, w.sta)
    keep = lists_to_keep(plan.kv_count, plan.kv_idx, plan.nb)
    assert np.array_equal(keep, plan.mask.cpu().numpy().astype(bool))
    mismatch = (keep != keep_ref) & ~amb
    assert not mismatch.any(), f"{int(mismatch.sum())} unambiguous blocks differ"
    assert amb.sum() <= max(2, 0.01 * amb.size)


@pytest.mark.parametrize("baseline", [False, True], ids=["tcgen05", "mma_sync"])
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_attention_matches_oracle_with_oracle_mask(bsa, w, baseline):
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w), with_lse=True)
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder(plan.shape, src.cuda(), dst)
    q64, k64, v64 = to64(plan.q), to64(plan.k), to64(plan.v)
    keep, _ = oracle.block_mask(q64, k64, w.T, w.H, w.W, w.patch, w.block, w.thr, w.sta)
    cnt, idx = oracle.mask_to_lists(keep)
    plan.kv_count.copy_(torch.from_numpy(cnt))
    plan.kv_idx.copy_(torch.from_numpy(idx))
    plan.attention_step(baseline=baseline)
    torch.cuda.synchronize()
    assert plan.status() == 0
    O_ref, lse_ref = oracle.masked_attention(q64, k64, v64, keep, w.N, w.block)
    O = to64(plan.o)
    mx, mean = compare_outputs(O[:, :, :w.N], O_ref[:, :, :w.N])
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    assert np.all(O[:, :, w.N:] == 0)
    lse = to64(plan.lse)
    assert np.abs(lse[:, :, :w.N] - lse_ref[:, :, :w.N]).max() <= LSE_ABS
    assert np.all(lse[:, :, w.N:] == 0)


@pytest.mark.parametrize("w", [SMALL[0], SMALL[1], SMALL[4]], ids=lambda w: w.name)
def test_whole_path_matches_oracle(bsa, w):
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w))
    out = plan(q.cuda(), k.cuda(), v.cuda(), w.thr, w.sta)
    torch.cuda.synchronize()
    assert plan.status() == 0
    O_ref, keep_ref, amb = oracle.nabla_attention(to64(q), to64(k), to64(v), w.T, w.H, w.W, w.patch, w.block,
                                                  w.thr, w.sta)
    assert not amb.any()
    mx, mean = compare_outputs(to64(out), O_ref)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


def test_random_lists_any_density(bsa):
    """Arbitrary (seeded random) lists, as an external mask would give them."""
    w = small("random_lists", 1, 2, 16, 40, 3, 128, 64, 8, 0.0, iid=True)
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w))
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder(plan.shape, src.cuda(), dst)
    q64, k64, v64 = to64(plan.q), to64(plan.k), to64(plan.v)
    for dens in (0.05, 0.3, 1.0):
        cnt, idx = synth.random_block_lists(w.B, w.heads, plan.nb, dens, seed=7)
        plan.kv_count.copy_(cnt)
        plan.kv_idx.copy_(idx)
        plan.attention_step()
        torch.cuda.synchronize()
        keep = lists_to_keep(cnt, idx, plan.nb)
        O_ref, _ = oracle.masked_attention(q64, k64, v64, keep, w.N, w.block)
        mx, mean = compare_outputs(to64(plan.o)[:, :, :w.N], O_ref[:, :, :w.N])
        assert mx <= MAX_ABS and mean <= MEAN_ABS, (dens, mx, mean)


def test_bad_lists_set_the_device_error_word(bsa):
    w = small("bad_lists", 1, 1, 16, 16, 2, 64, 64, 8, 0.0)
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w))
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder(plan.shape, src.cuda(), dst)
    nb = plan.nb
    plan.kv_count.fill_(1)
    plan.kv_idx.zero_()
    plan.kv_idx[0, 1, 2, 0] = nb + 5            # out of range: skipped, flagged
    plan.attention_step()
    assert plan.status() == 4
    assert plan.status() == 0                    # cleared on read
    plan.kv_idx[0, 1, 2, 0] = 0
    plan.kv_count[0, 0, 1] = nb + 1              # count out of range: clamped, flagged
    plan.attention_step()
    assert plan.status() == 4
    plan.kv_count[0, 0, 1] = 0
    plan.attention_step()
    assert plan.status() == 4
    assert torch.all(plan.o[0, 0, w.block:2 * w.block] == 0)   # empty row -> zero output


def test_attention_large_values_within_bf16_resolution(bsa):
    w = HOT
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w))
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder(plan.shape, src.cuda(), dst)
    q64, k64, v64 = to64(plan.q), to64(plan.k), to64(plan.v)
    keep, _ = oracle.block_mask(q64, k64, w.T, w.H, w.W, w.patch, w.block, w.thr, w.sta)
    cnt, idx = oracle.mask_to_lists(keep)
    plan.kv_count.copy_(torch.from_numpy(cnt))
    plan.kv_idx.copy_(torch.from_numpy(idx))
    plan.attention_step()
    torch.cuda.synchronize()
    O_ref, _ = oracle.masked_attention(q64, k64, v64, keep, w.N, w.block)
    got, want = to64(plan.o)[:, :, :w.N], O_ref[:, :, :w.N]
    assert np.abs(want).max() > 8.0
    assert np.all(np.abs(got - want) <= MAX_ABS + _half_ulp_bf16(want))


# Edge cases: the largest nb the kernels accept (1024 blocks of 64 tokens), a
# threshold close to 1 (about one block per row), batch 2 with 128-token blocks.
EDGE = [
    small("max_blocks", 1, 1, 256, 256, 1, 64, 64, 8, 0.3, alpha=2.0, seed=21),
    small("thr_near_one", 1, 3, 16, 24, 2, 128, 64, 8, 0.995, seed=22),
    small("batch2_b128", 2, 2, 24, 24, 2, 128, 128, 8, 0.2, seed=23),
]


@pytest.mark.parametrize("w", EDGE, ids=lambda w: w.name)
def test_edge_shapes_mask_and_attention(bsa, w):
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w), with_mask=True, with_lse=True)
    assert plan.nb <= 1024
    _run_mask(bsa, w, plan, q.cuda(), k.cuda())
    bsa.reorder(plan.shape, v.cuda(), plan.v)
    assert plan.status() == 0
    q64, k64, v64 = to64(plan.q), to64(plan.k), to64(plan.v)
    keep_ref, amb = oracle.block_mask(q64, k64, w.T, w.H, w.W, w.patch, w.block, w.thr, w.sta)
    keep = lists_to_keep(plan.kv_count, plan.kv_idx, plan.nb)
    mismatch = (keep != keep_ref) & ~amb
    assert not mismatch.any(), f"{int(mismatch.sum())} unambiguous blocks differ"
    if w.thr > 0.99:
        assert keep_ref.sum(axis=-1).mean() < 2.0          # about one block per row
    # attention with the oracle's mask, sampled rows (the largest case has 1024 blocks)
    cnt, idx = oracle.mask_to_lists(keep_ref)
    plan.kv_count.copy_(torch.from_numpy(cnt))
    plan.kv_idx.copy_(torch.from_numpy(idx))
    plan.attention_step()
    torch.cuda.synchronize()
    assert plan.status() == 0
    rng = np.random.default_rng(5)
    picks = {(w.B - 1, w.heads - 1, plan.nb - 1), (0, 0, 0)}
    while len(picks) < min(12, w.B * w.heads * plan.nb):
        picks.add((int(rng.integers(w.B)), int(rng.integers(w.heads)), int(rng.integers(plan.nb))))
    O_ref, lse_ref = oracle.masked_attention(q64, k64, v64, keep_ref, w.N, w.block, blocks=sorted(picks))
    O, lse = to64(plan.o), to64(plan.lse)
    for (b, h, I) in sorted(picks):
        lo, hi = I * w.block, min((I + 1) * w.block, w.N)
        mx, mean = compare_outputs(O[b, h, lo:hi], O_ref[b, h, lo:hi])
        assert mx <= MAX_ABS and mean <= MEAN_ABS, ((b, h, I), mx, mean)
        assert np.abs(lse[b, h, lo:hi] - lse_ref[b, h, lo:hi]).max() <= LSE_ABS


def test_forced_timeout_is_reported_and_the_context_stays_usable(bsa, monkeypatch):
    """The bounded-wait failure path: with the test hook set, the attention
    kernel's first wait runs out (2 ms, nothing arrives), BSA_ERR_TIMEOUT comes
    back through the error word, and the next call computes normally."""
    w = small("forced_timeout", 1, 2, 16, 16, 2, 128, 64, 8, 0.2, seed=31)
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w))
    _reorder_all(bsa, plan, q, k, v)
    plan.mask_step(w.thr, w.sta)
    monkeypatch.setenv("BSA_TEST_FORCE_TIMEOUT", "1")
    plan.attention_step()
    assert plan.status() == 5                     # BSA_ERR_TIMEOUT
    monkeypatch.delenv("BSA_TEST_FORCE_TIMEOUT")
    plan.attention_step()
    torch.cuda.synchronize()
    assert plan.status() == 0
    keep = lists_to_keep(plan.kv_count, plan.kv_idx, plan.nb)
    O_ref, _ = oracle.masked_attention(to64(plan.q), to64(plan.k), to64(plan.v), keep, w.N, w.block)
    mx, mean = compare_outputs(to64(plan.o)[:, :, :w.N], O_ref[:, :, :w.N])
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


def test_a_timeout_left_by_an_earlier_call_does_not_cut_the_next_call_short(bsa):
    """The error word is sticky until bsa_check_device_status reads it.  A
    timeout bit and an abort mark left in the workspace by an earlier call
    must not make the next mask or attention call give up: its output is the
    oracle's, and the stale bit is still reported (then cleared) afterwards."""
    w = small("stale_timeout", 1, 2, 16, 16, 2, 128, 64, 8, 0.2, seed=33)
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w))
    _reorder_all(bsa, plan, q, k, v)
    torch.cuda.synchronize()
    ctrl = plan.ws[:256].view(torch.int32)
    ctrl[0] = 4                      # kErrTimeout, as an earlier timed-out call leaves it
    ctrl[4:5].fill_(-1)              # an abort mark of an earlier launch
    plan.o.fill_(float("nan"))
    # the separate pooling path: its bulk-copy waits and the attention's both run
    bsa.build_block_mask(plan.shape, plan.q, plan.k, w.thr, w.sta, plan.kv_count, plan.kv_idx, None, plan.ws)
    plan.attention_step()
    torch.cuda.synchronize()
    assert plan.status() == 5        # the stale bit is reported once ...
    assert plan.status() == 0        # ... and cleared
    keep_ref, amb = oracle.nabla.block_mask(to64(plan.q), to64(plan.k), w.T, w.H, w.W, w.patch, w.block, w.thr)
    keep = lists_to_keep(plan.kv_count, plan.kv_idx, plan.nb)
    assert not ((keep != keep_ref) & ~amb).any()
    O_ref, _ = oracle.masked_attention(to64(plan.q), to64(plan.k), to64(plan.v), keep, w.N, w.block)
    mx, mean = compare_outputs(to64(plan.o)[:, :, :w.N], O_ref[:, :, :w.N])
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


# Keys whose scale grows along the key blocks: each row's running max keeps
# rising as the kernel walks its ascending list, so the lazy rescale of O (a
# max that grows by more than 8 in log2 units) runs many times per row, in
# both tile layouts (two 64-token blocks per 128-row tile, and 128-token
# blocks).
GROWTH = [
    small("growth64", 1, 3, 16, 24, 2, 128, 64, 8, 0.0, seed=31),
    small("growth128_d64", 1, 2, 16, 32, 2, 64, 128, 8, 0.0, seed=32),
]


@pytest.mark.parametrize("w", GROWTH, ids=lambda w: w.name)
def test_running_max_growth_rescales(bsa, w):
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w), with_lse=True)
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder(plan.shape, src.cuda(), dst)
    nb = plan.nb
    blk = torch.arange(plan.k.shape[2], device=plan.k.device) // w.block
    ramp = 1.0 + 2.0 * blk.float() / nb
    plan.k.copy_((plan.k.float() * ramp[None, None, :, None]).to(torch.bfloat16))
    q64, k64, v64 = to64(plan.q), to64(plan.k), to64(plan.v)
    # the case is meaningful only if many rows' max grows by more than 8
    # (log2 units) after their first key block
    s = np.einsum("bhnd,bhmd->bhnm", q64[:, :, :w.N], k64[:, :, :w.N]) / math.sqrt(w.d) / math.log(2.0)
    first = s[..., :w.block].max(axis=-1)
    assert np.mean(s.max(axis=-1) - first > 8.0) > 0.2
    for dens in (1.0, 0.4):
        cnt, idx = synth.random_block_lists(w.B, w.heads, nb, dens, seed=9)
        plan.kv_count.copy_(cnt)
        plan.kv_idx.copy_(idx)
        plan.attention_step()
        torch.cuda.synchronize()
        assert plan.status() == 0
        keep = lists_to_keep(cnt, idx, nb)
        O_ref, lse_ref = oracle.masked_attention(q64, k64, v64, keep, w.N, w.block)
        got, want = to64(plan.o)[:, :, :w.N], O_ref[:, :, :w.N]
        assert np.all(np.abs(got - want) <= MAX_ABS + _half_ulp_bf16(want)), dens
        assert np.abs(got - want).mean() <= MEAN_ABS, dens
        lse = to64(plan.lse)[:, :, :w.N]
        assert np.abs(lse - lse_ref[:, :, :w.N]).max() <= LSE_ABS * max(1.0, np.abs(lse_ref).max() / 16.0), dens


@pytest.mark.parametrize("w", GROWTH, ids=lambda w: w.name)
def test_running_max_jump_past_the_unchecked_range(bsa, w):
    """After a row's first kept tile the kernel skips the max pass and checks
    each 32-key chunk's weights instead; scores that exceed the running max by
    64 or more (log2 units) make the warp redo the tile from that chunk with a
    new max, rescaling O, the sums and the weights already stored.  Keys
    scaled up steeply along the blocks force that path on most rows: O, LSE and
    (dense lists, the warm-up pass) the entropy against the oracle."""
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(_shape(bsa, w), with_lse=True)
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder(plan.shape, src.cuda(), dst)
    nb = plan.nb
    blk = torch.arange(plan.k.shape[2], device=plan.k.device) // w.block
    ramp = 1.0 + 40.0 * (blk.float() / nb) ** 2
    plan.k.copy_((plan.k.float() * ramp[None, None, :, None]).to(torch.bfloat16))
    q64, k64, v64 = to64(plan.q), to64(plan.k), to64(plan.v)
    s = np.einsum("bhnd,bhmd->bhnm", q64[:, :, :w.N], k64[:, :, :w.N]) / math.sqrt(w.d) / math.log(2.0)
    first = s[..., :2 * w.block].max(axis=-1)
    assert np.mean(s.max(axis=-1) - first > 64.0) > 0.2
    cnt, idx = synth.random_block_lists(w.B, w.heads, nb, 1.0, seed=9)
    plan.kv_count.copy_(cnt)
    plan.kv_idx.copy_(idx)
    keep = lists_to_keep(cnt, idx, nb)
    O_ref, lse_ref = oracle.masked_attention(q64, k64, v64, keep, w.N, w.block)
    want, lse_want = O_ref[:, :, :w.N], lse_ref[:, :, :w.N]
    lse_tol = LSE_ABS * max(1.0, np.abs(lse_want).max() / 16.0)
    plan.attention_step()
    torch.cuda.synchronize()
    assert plan.status() == 0
    got = to64(plan.o)[:, :, :w.N]
    assert np.all(np.abs(got - want) <= MAX_ABS + _half_ulp_bf16(want))
    assert np.abs(got - want).mean() <= MEAN_ABS
    assert np.abs(to64(plan.lse)[:, :, :w.N] - lse_want).max() <= lse_tol
    ent = torch.full_like(plan.lse, float("nan"))
    bsa.attn_fwd_entropy(plan.shape, plan.q, plan.k, plan.v, plan.kv_count, plan.kv_idx, 0.0, plan.o, plan.lse, ent,
                         plan.ws)
    torch.cuda.synchronize()
    assert plan.status() == 0
    got = to64(plan.o)[:, :, :w.N]
    assert np.all(np.abs(got - want) <= MAX_ABS + _half_ulp_bf16(want))
    assert np.abs(to64(plan.lse)[:, :, :w.N] - lse_want).max() <= lse_tol
    H_ref = oracle.attention_entropy(q64, k64, w.N)[:, :, :w.N]
    assert np.abs(to64(ent)[:, :, :w.N] - H_ref).max() <= 2e-3
