"""oracle.parallel (the host process pool the full-size GPU tests and the bench's
oracle legs use) gives exactly what the serial oracle gives.  CPU only."""
import numpy as np
import torch

import oracle
from oracle.parallel import OraclePool
from block_sparse_attention_fractal_b200 import synth

from _util import small


def _serial(w, q, k, v):
    f64 = lambda t: t.to(torch.float64).numpy()
    yq = oracle.reorder(f64(q), w.T, w.H, w.W, w.patch, w.block)
    yk = oracle.reorder(f64(k), w.T, w.H, w.W, w.patch, w.block)
    yv = oracle.reorder(f64(v), w.T, w.H, w.W, w.patch, w.block)
    keep, amb = oracle.block_mask(yq, yk, w.T, w.H, w.W, w.patch, w.block, w.thr, w.sta)
    O, lse = oracle.masked_attention(yq, yk, yv, keep, w.N, w.block)
    return keep, amb, O, lse


def test_pool_equals_the_serial_oracle():
    w = small("pool_small", 2, 2, 9, 14, 3, 64, 64, 4, 0.2, sta=(1, 1, 1))
    q, k, v = synth.make_qkv(w)
    keep_s, amb_s, O_s, lse_s = _serial(w, q, k, v)
    with OraclePool(w, q, k, v, workers=3) as pool:
        pool.reorder(pool.pairs())
        keep, amb, _ = pool.masks(pool.pairs())
        assert np.array_equal(keep, keep_s) and np.array_equal(amb, amb_s)
        # a "GPU output" equal to the oracle's, rounded to bf16: within half a bf16 ulp
        o_bf = torch.from_numpy(O_s).to(torch.bfloat16)
        lse32 = torch.from_numpy(lse_s).to(torch.float32)
        items = [(b, h, range(w.nb)) for (b, h) in pool.pairs()]
        mx, mean, n, lmx, pad = pool.check_attention(o_bf, lse32, items)
        assert n == w.B * w.heads * w.N * w.d
        assert mx <= 2.0 ** -8 * np.abs(O_s).max() and lmx < 1e-5 and pad == 0
        # one planted error in one element of one head is found
        o_bad = o_bf.clone()
        o_bad[1, 2, w.N - 1, 5] += 0.5
        mx2, _, _, _, _ = pool.check_attention(o_bad, lse32, items)
        assert mx2 > 0.4
        # a nonzero padded row is found
        o_pad = o_bf.clone()
        o_pad[0, 1, w.N, 0] = 1.0
        assert pool.check_attention(o_pad, lse32, items)[4] == 1
        # the attention and inverse stages run and time themselves
        assert pool.attention(0, 1, range(w.nb)) > 0 and pool.inverse() > 0
        # backward: the serial oracle's gradients, rounded to bf16, pass; a planted error is found
        f64 = lambda t: t.to(torch.float64).numpy()
        yq, yk, yv = (oracle.reorder(f64(x), w.T, w.H, w.W, w.patch, w.block) for x in (q, k, v))
        dO = torch.randn(o_bf.shape, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
        dO[:, :, w.N:] = 0
        grads = oracle.masked_attention_backward(yq, yk, yv, keep_s, f64(dO), w.N, w.block)
        gb = [torch.from_numpy(g).to(torch.bfloat16) for g in grads]
        rep = pool.check_backward(dO, *gb, pool.pairs())
        for name, (mx_, mean_, refmax, refmean, pad_) in rep.items():
            assert mx_ <= 2.0 ** -8 * refmax and pad_ == 0, name
        gb[1][1, 0, 5, 3] += 1.0
        assert pool.check_backward(dO, *gb, pool.pairs())["dk"][0] > 0.9
