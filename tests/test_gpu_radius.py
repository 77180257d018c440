"""GPU parity of the token-radius mask chain (TRA summary, section 2) against
the fp64 oracle:

* bsa_attn_fwd_entropy over dense lists (the warm-up pass): per-row entropy
  within 2e-3 nats of oracle.attention_entropy, and the output and LSE within
  the attention tolerances;
* bsa_build_block_mask_radius fed the same float32 entropies as the oracle:
  the block mask bit-exact against oracle.radius_block_mask (radii and
  comparisons in double on both sides).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_fractal_b200 import synth

from _util import LSE_ABS, MAX_ABS, MEAN_ABS, compare_outputs, lists_to_keep, small, to64

pytestmark = pytest.mark.gpu

ENT_ABS = 2e-3

CASES = [
    (synth.WORKLOADS["tiny"], 0.05, 0.5, 1),
    (small("rad_ragged64", 1, 3, 20, 28, 2, 128, 64, 8, 0.0), 0.02, 0.3, 1),
    (small("rad_ragged64_vote", 1, 3, 20, 28, 2, 128, 64, 8, 0.0), 0.05, 0.8, 8),
    (small("rad_ragged128_d64", 1, 2, 13, 37, 3, 64, 128, 4, 0.0), 0.1, 0.0, 1),
    (small("rad_batch2_d64", 2, 2, 16, 24, 2, 64, 64, 8, 0.0), 0.03, 1.0, 2),
]


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as m
    return m


def _warmup(bsa, w):
    q, k, v = synth.make_qkv(w)
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    plan = bsa.NablaAttention(s, with_lse=True)
    plan.reorder_inputs(q.cuda(), k.cuda(), v.cuda())
    plan.join_side()
    bsa.dense_lists(s, plan.kv_count, plan.kv_idx)
    ent = torch.full_like(plan.lse, float("nan"))
    bsa.attn_fwd_entropy(s, plan.q, plan.k, plan.v, plan.kv_count, plan.kv_idx, 0.0, plan.o, plan.lse, ent, plan.ws)
    torch.cuda.synchronize()
    assert plan.status() == 0
    return plan, ent


@pytest.mark.parametrize("w,tau,gamma,vote", CASES[:2] + CASES[3:4], ids=lambda x: getattr(x, "name", str(x)))
def test_dense_warmup_entropy_matches_oracle(bsa, w, tau, gamma, vote):
    plan, ent = _warmup(bsa, w)
    assert lists_to_keep(plan.kv_count, plan.kv_idx, plan.nb).all()
    q64, k64, v64 = to64(plan.q), to64(plan.k), to64(plan.v)
    H = oracle.attention_entropy(q64, k64, w.N)
    e = to64(ent)
    assert np.abs(e[:, :, :w.N] - H[:, :, :w.N]).max() <= ENT_ABS
    assert np.all(e[:, :, w.N:] == 0)
    keep = np.ones((w.B, w.heads, plan.nb, plan.nb), dtype=bool)
    O_ref, lse_ref = oracle.masked_attention(q64, k64, v64, keep, w.N, w.block)
    mx, mean = compare_outputs(to64(plan.o)[:, :, :w.N], O_ref[:, :, :w.N])
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    assert np.abs(to64(plan.lse)[:, :, :w.N] - lse_ref[:, :, :w.N]).max() <= LSE_ABS


@pytest.mark.parametrize("w,tau,gamma,vote", CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_radius_mask_matches_oracle(bsa, w, tau, gamma, vote):
    plan, ent = _warmup(bsa, w)
    mask = torch.empty((w.B, w.heads, plan.nb, plan.nb), dtype=torch.uint8, device="cuda")
    bsa.build_block_mask_radius(plan.shape, ent, tau, gamma, vote, plan.kv_count, plan.kv_idx, mask)
    torch.cuda.synchronize()
    keep = lists_to_keep(plan.kv_count, plan.kv_idx, plan.nb)
    assert np.array_equal(keep, mask.cpu().numpy().astype(bool))
    # the oracle from the same float32 entropies
    t_of = oracle.fractal_order(w.T, w.H, w.W, w.patch) // (w.H * w.W)
    r = oracle.token_radius(to64(ent), t_of, w.T, tau, gamma, w.N)
    keep_ref = oracle.radius_block_mask(r, w.T, w.H, w.W, w.patch, w.block, gamma, vote)
    assert np.array_equal(keep, keep_ref), int((keep != keep_ref).sum())
    assert keep.diagonal(axis1=-2, axis2=-1).all()     # every block holds its own query tokens' positions
    print(f"{w.name}: radius mask density {keep.mean():.3f}")
