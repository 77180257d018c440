"""GPU parity of the block-sparse attention backward (bsa_attn_bwd) against
the fp64 oracle's gradients (oracle.masked_attention_backward), on the same
seeded inputs and the oracle's own block mask.

The kernels round P and dS to bf16 for the tensor-core products (as the
forward rounds P) and write bf16 gradients; the bound is relative to each
gradient's own scale: max-abs error <= 2e-2 * max|ref| and mean-abs error
<= 1e-2 * mean|ref| per tensor (the derivation is in the design notes:
bf16 rounding of P, dS and the output, about 2^-9 relative each).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_fractal_b200 import synth

from _util import small, to64

pytestmark = pytest.mark.gpu

MAX_REL = 2e-2
MEAN_REL = 1e-2

CASES = [
    synth.WORKLOADS["tiny"],
    small("bwd_ragged64", 1, 3, 20, 28, 2, 128, 64, 8, 0.15),
    small("bwd_ragged128_d64", 1, 2, 13, 37, 3, 64, 128, 4, 0.3),
    small("bwd_batch2_d64", 2, 2, 16, 24, 2, 64, 64, 8, 0.25),
    small("bwd_dense", 1, 2, 12, 20, 2, 128, 128, 4, 0.0),
    small("bwd_one_block", 1, 1, 5, 7, 2, 64, 64, 8, 0.1),
]


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as m
    return m


def _run(bsa, w, seed=7):
    q, k, v = synth.make_qkv(w)
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    plan = bsa.NablaAttention(s, with_lse=True)
    plan.reorder_inputs(q.cuda(), k.cuda(), v.cuda())
    plan.join_side()
    plan.mask_step(w.thr, w.sta)
    plan.attention_step()
    g = torch.Generator().manual_seed(seed)
    dO = torch.randn(plan.o.shape, generator=g).to(torch.bfloat16)
    dO[:, :, w.N:] = 0
    dO = dO.cuda()
    dq, dk, dv = (torch.full_like(plan.q, float("nan")) for _ in range(3))
    ws = torch.zeros((bsa.attn_bwd_workspace_bytes(s) + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    bsa.attn_bwd(s, plan.q, plan.k, plan.v, plan.o, dO, plan.lse, plan.kv_count, plan.kv_idx, 0.0, dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert bsa.check_device_status(ws) == 0
    assert plan.status() == 0
    return plan, dO, dq, dk, dv


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_matches_oracle(bsa, w):
    plan, dO, dq, dk, dv = _run(bsa, w)
    keep = np.zeros((w.B, w.heads, plan.nb, plan.nb), dtype=bool)
    cnt, idx = plan.kv_count.cpu().numpy(), plan.kv_idx.cpu().numpy()
    for b in range(w.B):
        for h in range(w.heads):
            for I in range(plan.nb):
                keep[b, h, I, idx[b, h, I, :cnt[b, h, I]]] = True
    # the gradient of the kernel's own forward output O: the oracle recomputes
    # O from the same Q, K, V and mask
    ref = oracle.masked_attention_backward(to64(plan.q), to64(plan.k), to64(plan.v), keep, to64(dO), w.N, w.block)
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        g64 = to64(got)
        assert np.all(g64[:, :, w.N:] == 0), name
        err = np.abs(g64[:, :, :w.N] - want[:, :, :w.N])
        scale_max = np.abs(want[:, :, :w.N]).max()
        scale_mean = np.abs(want[:, :, :w.N]).mean()
        print(f"{w.name} {name}: max-abs {err.max():.3e} (ref max {scale_max:.3e}), "
              f"mean-abs {err.mean():.3e} (ref mean {scale_mean:.3e})")
        assert err.max() <= MAX_REL * scale_max, (name, err.max(), scale_max)
        assert err.mean() <= MEAN_REL * scale_mean, (name, err.mean(), scale_mean)
