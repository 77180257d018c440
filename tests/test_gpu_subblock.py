"""GPU parity of the alternative order and estimator (DFSAttn explainer,
sections 1 and 2) against the fp64 oracle:

* bsa_hilbert_order: bit-exact against oracle.hilbert_order;
* bsa_reorder_perm / bsa_inverse_reorder_perm / bsa_reorder_qk_pooled_perm with
  that order: bit-exact data movement, exact block means;
* bsa_build_block_mask_subblock: masks bit-exact against
  oracle.block_mask_subblock except blocks the oracle flags as ambiguous;
* the whole path in Hilbert order (reorder, sub-block mask, attention with the
  oracle's mask, inverse reorder) within the attention tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import nabla
from block_sparse_attention_fractal_b200 import synth

from _util import MAX_ABS, MEAN_ABS, compare_outputs, lists_to_keep, small, to64

pytestmark = pytest.mark.gpu

ORDER_SHAPES = [(2, 2, 2), (3, 5, 6), (4, 16, 16), (21, 30, 52), (33, 45, 80)]

SUB_CASES = [
    (synth.WORKLOADS["tiny"], 16),
    (small("sub_ragged64", 1, 3, 20, 28, 2, 128, 64, 8, 0.15), 16),
    (small("sub_ragged64_s32", 1, 3, 20, 28, 2, 128, 64, 8, 0.15), 32),
    (small("sub_ragged128_d64", 1, 2, 13, 37, 3, 64, 128, 4, 0.3), 32),
    (small("sub_batch2_d64", 2, 2, 16, 24, 2, 64, 64, 8, 0.25), 16),
    (small("sub_equal_block", 1, 2, 12, 20, 2, 128, 64, 4, 0.2), 64),
]


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as m
    return m


def _order(bsa, s, N):
    order = torch.full((N,), -1, dtype=torch.int32, device="cuda")
    ws = torch.zeros((bsa.hilbert_workspace_bytes(s) + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    bsa.hilbert_order(s, order, ws)
    torch.cuda.synchronize()
    return order


@pytest.mark.parametrize("T,H,W", ORDER_SHAPES)
def test_hilbert_order_matches_oracle(bsa, T, H, W):
    s = bsa.make_shape(1, T, H, W, 1, 64, 64, 8)
    order = _order(bsa, s, T * H * W)
    assert np.array_equal(order.cpu().numpy(), oracle.hilbert_order(T, H, W))


@pytest.mark.parametrize("w,sub", SUB_CASES[:3], ids=lambda x: getattr(x, "name", str(x)))
def test_reorder_by_table_bit_exact(bsa, w, sub):
    q, k, _ = synth.make_qkv(w)
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    order = _order(bsa, s, w.N)
    o64 = order.cpu().numpy().astype(np.int64)
    Npad = bsa.padded_len(s)
    y = torch.full((w.B, w.heads, Npad, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    bsa.reorder_perm(s, order, q.cuda(), y)
    want = nabla.reorder_by(to64(q), o64, w.block)
    assert np.array_equal(to64(y), want)
    back = torch.full_like(q.cuda(), float("nan"))
    bsa.inverse_reorder_perm(s, order, y, back)
    assert torch.equal(back.cpu(), q)
    # the fused Q/K pass with the table: both reorders and the exact block means
    yq, yk = torch.empty_like(y), torch.empty_like(y)
    ws = torch.zeros((bsa.workspace_bytes(s) + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    bsa.reorder_qk_pooled_perm(s, order, q.cuda(), k.cuda(), yq, yk, ws)
    torch.cuda.synchronize()
    want_k = nabla.reorder_by(to64(k), o64, w.block)
    assert np.array_equal(to64(yq), want) and np.array_equal(to64(yk), want_k)
    nb, n = bsa.num_blocks(s), w.B * w.heads * bsa.num_blocks(s) * w.d
    means = ws[256:256 + 16 * n].view(torch.float64).cpu().numpy()
    assert np.array_equal(means[:n].reshape(w.B, w.heads, nb, w.d), oracle.block_means(want, w.N, w.block))


@pytest.mark.parametrize("w,sub", SUB_CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_subblock_mask_matches_oracle(bsa, w, sub):
    q, k, _ = synth.make_qkv(w)
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    order = _order(bsa, s, w.N)
    Npad, nb = bsa.padded_len(s), bsa.num_blocks(s)
    yq = torch.empty((w.B, w.heads, Npad, w.d), dtype=torch.bfloat16, device="cuda")
    yk = torch.empty_like(yq)
    bsa.reorder_perm(s, order, q.cuda(), yq)
    bsa.reorder_perm(s, order, k.cuda(), yk)
    cnt = torch.empty((w.B, w.heads, nb), dtype=torch.int32, device="cuda")
    idx = torch.empty((w.B, w.heads, nb, nb), dtype=torch.int32, device="cuda")
    mask = torch.empty((w.B, w.heads, nb, nb), dtype=torch.uint8, device="cuda")
    ws = torch.zeros((bsa.subblock_workspace_bytes(s, sub) + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    bsa.workspace_init(ws)
    bsa.build_block_mask_subblock(s, yq, yk, sub, w.thr, cnt, idx, mask, ws)
    torch.cuda.synchronize()
    assert bsa.check_device_status(ws) == 0
    keep = lists_to_keep(cnt, idx, nb)
    assert np.array_equal(keep, mask.cpu().numpy().astype(bool))
    keep_ref, amb = oracle.block_mask_subblock(to64(yq), to64(yk), w.N, w.block, sub, w.thr)
    mismatch = (keep != keep_ref) & ~amb
    assert not mismatch.any(), f"{int(mismatch.sum())} unambiguous blocks differ"
    assert amb.sum() <= max(2, 0.01 * amb.size)
    if sub == w.block:   # one sub-block per block: NABLA's mask
        keep_nabla, amb_n = oracle.block_mask(to64(yq), to64(yk), w.T, w.H, w.W, w.patch, w.block, w.thr)
        assert not ((keep != keep_nabla) & ~amb_n & ~amb).any()


@pytest.mark.parametrize("w,sub", [SUB_CASES[1], SUB_CASES[3]], ids=lambda x: getattr(x, "name", str(x)))
def test_hilbert_subblock_path_matches_oracle(bsa, w, sub):
    """Reorder by the Hilbert order, sub-block mask, block-sparse attention,
    inverse reorder: against the oracle's composition of the same steps."""
    q, k, v = synth.make_qkv(w)
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    order = _order(bsa, s, w.N)
    plan = bsa.NablaAttention(s, with_lse=True)
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder_perm(s, order, src.cuda(), dst)
    ws = torch.zeros((bsa.subblock_workspace_bytes(s, sub) + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    bsa.build_block_mask_subblock(s, plan.q, plan.k, sub, w.thr, plan.kv_count, plan.kv_idx, None, ws)
    plan.attention_step()
    out = torch.empty_like(q.cuda())
    bsa.inverse_reorder_perm(s, order, plan.o, out)
    torch.cuda.synchronize()
    assert plan.status() == 0 and bsa.check_device_status(ws) == 0
    o64 = oracle.hilbert_order(w.T, w.H, w.W)
    yq, yk, yv = (nabla.reorder_by(to64(x), o64, w.block) for x in (q, k, v))
    keep_ref, amb = oracle.block_mask_subblock(yq, yk, w.N, w.block, sub, w.thr)
    assert not amb.any()
    O_ref, _ = oracle.masked_attention(yq, yk, yv, keep_ref, w.N, w.block)
    want = np.zeros_like(to64(q))
    for p in range(w.N):
        want[:, o64[p]] = O_ref[:, :, p]
    mx, mean = compare_outputs(to64(out), want)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
