"""GPU parity at the full workload sizes, in the launch configuration the bench
times (NablaAttention: reorder x3, mask, attention, inverse reorder).

* reorder: bit-exact on the whole tensor (checked against the oracle's order);
* block masks: compared in full, every head, against the oracle's; blocks the
  oracle flags as ambiguous are counted and reported, every other block must
  match;
* attention: the oracle's mask is fed to the kernel, and the output and LSE
  are compared element by element with the oracle's -- every query block of
  every head on Wan-480p and the NABLA u STA hybrid, a sample on Hunyuan-720p
  (every head, the ragged last block) and on the density sweep (every head,
  plus a run of consecutive blocks so both halves of many paired tiles are
  covered).  The oracle runs on the host cores through oracle.parallel.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.parallel import OraclePool
from block_sparse_attention_fractal_b200 import synth

from _util import LSE_ABS, MAX_ABS, MEAN_ABS, lists_to_keep

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as m
    return m


def _plan(bsa, w):
    s = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    return bsa.NablaAttention(s, with_mask=True, with_lse=True)


def _check_reorder(w, x_dev, y):
    order = torch.from_numpy(oracle.fractal_order(w.T, w.H, w.W, w.patch)).cuda()
    want = x_dev.permute(0, 2, 1, 3)[:, :, order, :]
    assert torch.equal(y[:, :, :w.N], want)
    assert torch.all(y[:, :, w.N:] == 0)


def _sampled_items(w, per_head, seed, run=0):
    """(b, h, blocks): `per_head` random blocks of every head (the ragged last
    block in head 0), plus `run` consecutive blocks of one head."""
    rng = np.random.default_rng(seed)
    items = []
    for b in range(w.B):
        for h in range(w.heads):
            blocks = set(int(x) for x in rng.choice(w.nb, size=per_head, replace=False))
            if h == 0:
                blocks.add(w.nb - 1)
            items.append((b, h, sorted(blocks)))
    if run:
        h = int(rng.integers(w.heads))
        lo = int(rng.integers(0, max(1, w.nb - run)))
        items.append((0, h, list(range(lo, min(w.nb, lo + run)))))
    return items


def _check_attention(pool, plan, items):
    mx, mean, n, lmx, pad = pool.check_attention(plan.o.cpu(), plan.lse.cpu(), items)
    print(f"  attention vs oracle: {n} elements, max-abs {mx:.3e}, mean-abs {mean:.3e}, LSE max {lmx:.3e}")
    assert n > 0
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    assert lmx <= LSE_ABS, lmx
    assert pad == 0


@pytest.mark.parametrize("name", ["wan480p", "hybrid_wan480p", "hunyuan720p"])
def test_full_size_workload(bsa, name):
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(w)
    plan = _plan(bsa, w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out = plan(qd, kd, vd, w.thr, w.sta)
    torch.cuda.synchronize()
    assert plan.status() == 0
    _check_reorder(w, qd, plan.q)
    _check_reorder(w, kd, plan.k)
    _check_reorder(w, vd, plan.v)
    # the inverse reorder of the kernel's own output
    order = torch.from_numpy(oracle.fractal_order(w.T, w.H, w.W, w.patch)).cuda()
    assert torch.equal(out[:, order].permute(0, 2, 1, 3), plan.o[:, :, :w.N])
    del qd, kd, vd, out

    gpu_keep = lists_to_keep(plan.kv_count, plan.kv_idx, plan.nb)
    assert np.array_equal(gpu_keep, plan.mask.cpu().numpy().astype(bool))
    with OraclePool(w, q, k, v) as pool:
        pool.reorder(pool.pairs())
        keep, amb, _ = pool.masks(pool.pairs())
        mismatch = int(((gpu_keep != keep) & ~amb).sum())
        n_amb = int(amb.sum())
        print(f"{name}: density {keep.mean():.4f}, ambiguous blocks {n_amb}, unambiguous mismatches {mismatch}")
        assert mismatch == 0
        assert n_amb <= max(2, amb.size // 1000)

        # attention with the oracle's mask
        cnt, idx = oracle.mask_to_lists(keep)
        plan.kv_count.copy_(torch.from_numpy(cnt))
        plan.kv_idx.copy_(torch.from_numpy(idx))
        plan.attention_step()
        torch.cuda.synchronize()
        assert plan.status() == 0
        if name == "hunyuan720p":
            items = _sampled_items(w, per_head=3, seed=1)
        else:
            items = [(b, h, range(w.nb)) for (b, h) in pool.pairs()]
        _check_attention(pool, plan, items)


def test_density_sweep(bsa):
    w = synth.WORKLOADS["density_sweep"]
    q, k, v = synth.make_qkv(w)
    plan = _plan(bsa, w)
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder(plan.shape, src.cuda(), dst)
    with OraclePool(w, q, k, v) as pool:
        pool.reorder(pool.pairs())
        for i, dens in enumerate(w.densities):
            cnt, idx = synth.random_block_lists(w.B, w.heads, plan.nb, dens, seed=w.seed)
            plan.kv_count.copy_(cnt)
            plan.kv_idx.copy_(idx)
            plan.attention_step()
            torch.cuda.synchronize()
            assert plan.status() == 0
            keep = lists_to_keep(cnt, idx, plan.nb)
            pool.set_keep(keep)
            print(f"density {dens}:")
            _check_attention(pool, plan, _sampled_items(w, per_head=2, seed=100 + i, run=48))


def test_full_size_backward_wan480p(bsa):
    """The backward pass at the Wan-480p size: every element of dQ, dK and dV
    of every head against the oracle's gradients (oracle mask of the GPU's
    forward lists), within the bounds of tests/test_gpu_backward.py."""
    from test_gpu_backward import MAX_REL, MEAN_REL
    w = synth.WORKLOADS["wan480p"]
    q, k, v = synth.make_qkv(w)
    plan = _plan(bsa, w)
    plan(q.cuda(), k.cuda(), v.cuda(), w.thr, w.sta)
    g = torch.Generator().manual_seed(17)
    dO = torch.randn(plan.o.shape, generator=g).to(torch.bfloat16)
    dO[:, :, w.N:] = 0
    dOd = dO.cuda()
    dq, dk, dv = (torch.full_like(plan.q, float("nan")) for _ in range(3))
    ws = torch.zeros((bsa.attn_bwd_workspace_bytes(plan.shape) + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    bsa.attn_bwd(plan.shape, plan.q, plan.k, plan.v, plan.o, dOd, plan.lse, plan.kv_count, plan.kv_idx, 0.0,
                 dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert bsa.check_device_status(ws) == 0 and plan.status() == 0
    keep = lists_to_keep(plan.kv_count, plan.kv_idx, plan.nb)
    with OraclePool(w, q, k, v) as pool:
        pool.reorder(pool.pairs())
        pool.set_keep(keep)
        rep = pool.check_backward(dO, dq.cpu(), dk.cpu(), dv.cpu(), pool.pairs())
    for name, (mx, mean, refmax, refmean, pad) in rep.items():
        print(f"  {name}: max-abs {mx:.3e} (ref max {refmax:.3e}), mean-abs {mean:.3e} (ref mean {refmean:.3e})")
        assert pad == 0, name
        assert mx <= MAX_REL * refmax and mean <= MEAN_REL * refmean, name
