"""GPU parity at the full workload sizes, in the launch configuration the bench
times (NablaAttention: reorder x3, mask, attention, inverse reorder).

* reorder: bit-exact on the whole tensor (checked against the oracle's order);
* block masks: compared in full, head by head, against the oracle;
* attention: the oracle's mask is fed to the kernel; outputs are compared on
  a seeded sample of query blocks (always including the ragged last block);
* density sweep: seeded random lists at every density, sampled blocks.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_fractal_b200 import synth

from _util import MAX_ABS, MEAN_ABS, compare_outputs, lists_to_keep, to64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as m
    return m


def _plan(bsa, w):
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    return bsa.NablaAttention(s, with_mask=True)


def _sample_blocks(w, nb, n, seed):
    rng = np.random.default_rng(seed)
    picks = {(0, 0, nb - 1), (0, w.heads - 1, 0)}
    while len(picks) < n:
        picks.add((int(rng.integers(w.B)), int(rng.integers(w.heads)), int(rng.integers(nb))))
    return sorted(picks)


def _check_reorder(plan, w, x_dev, y):
    order = torch.from_numpy(oracle.fractal_order(w.T, w.H, w.W, w.patch)).cuda()
    want = x_dev.permute(0, 2, 1, 3)[:, :, order, :]
    assert torch.equal(y[:, :, :w.N], want)
    assert torch.all(y[:, :, w.N:] == 0)


def _attention_sample(plan, w, keep, blocks):
    for (b, h, I) in blocks:
        q64 = to64(plan.q[b:b + 1, h:h + 1])
        k64 = to64(plan.k[b:b + 1, h:h + 1])
        v64 = to64(plan.v[b:b + 1, h:h + 1])
        O_ref, _ = oracle.masked_attention(q64, k64, v64, keep[b:b + 1, h:h + 1], w.N, w.block,
                                           blocks=[(0, 0, I)])
        lo, hi = I * w.block, min((I + 1) * w.block, w.N)
        got = to64(plan.o[b, h, lo:hi])
        mx, mean = compare_outputs(got, O_ref[0, 0, lo:hi])
        assert mx <= MAX_ABS and mean <= MEAN_ABS, ((b, h, I), mx, mean)


@pytest.mark.parametrize("name", ["wan480p", "hybrid_wan480p", "hunyuan720p"])
def test_full_size_workload(bsa, name):
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(w)
    plan = _plan(bsa, w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    del q, k, v
    out = plan(qd, kd, vd, w.thr, w.sta)
    torch.cuda.synchronize()
    assert plan.status() == 0
    _check_reorder(plan, w, qd, plan.q)
    _check_reorder(plan, w, kd, plan.k)
    _check_reorder(plan, w, vd, plan.v)
    # the inverse reorder of the kernel's own output
    order = torch.from_numpy(oracle.fractal_order(w.T, w.H, w.W, w.patch)).cuda()
    assert torch.equal(out[:, order].permute(0, 2, 1, 3), plan.o[:, :, :w.N])

    gpu_keep = lists_to_keep(plan.kv_count, plan.kv_idx, plan.nb)
    assert np.array_equal(gpu_keep, plan.mask.cpu().numpy().astype(bool))
    keep = np.zeros_like(gpu_keep)
    n_amb = 0
    for b in range(w.B):
        for h in range(w.heads):
            kr, amb = oracle.block_mask(to64(plan.q[b:b + 1, h:h + 1]), to64(plan.k[b:b + 1, h:h + 1]),
                                        w.T, w.H, w.W, w.patch, w.block, w.thr, w.sta)
            keep[b, h] = kr[0, 0]
            bad = (gpu_keep[b, h] != kr[0, 0]) & ~amb[0, 0]
            assert not bad.any(), (b, h, int(bad.sum()))
            n_amb += int(amb.sum())
    print(f"{name}: density {keep.mean():.4f}, ambiguous blocks {n_amb}")

    # attention with the oracle's mask
    cnt, idx = oracle.mask_to_lists(keep)
    plan.kv_count.copy_(torch.from_numpy(cnt))
    plan.kv_idx.copy_(torch.from_numpy(idx))
    plan.attention_step()
    torch.cuda.synchronize()
    assert plan.status() == 0
    _attention_sample(plan, w, keep, _sample_blocks(w, plan.nb, 12, seed=1))


def test_density_sweep(bsa):
    w = synth.WORKLOADS["density_sweep"]
    q, k, v = synth.make_qkv(w)
    plan = _plan(bsa, w)
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder(plan.shape, src.cuda(), dst)
    del q, k, v
    for dens in w.densities:
        cnt, idx = synth.random_block_lists(w.B, w.heads, plan.nb, dens, seed=w.seed)
        plan.kv_count.copy_(cnt)
        plan.kv_idx.copy_(idx)
        plan.attention_step()
        torch.cuda.synchronize()
        assert plan.status() == 0
        keep = lists_to_keep(cnt, idx, plan.nb)
        _attention_sample(plan, w, keep, _sample_blocks(w, plan.nb, 4, seed=int(dens * 100)))
