"""Pins for the fp64 oracle against facts that do not come from the oracle itself:
hand-derived values (tests/golden), closed forms, brute force over all subsets,
special cases that reduce to a library routine (torch SDPA in float64), and
invariants.  CPU only.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import nabla


def _read_golden(path):
    kv = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            kv[key] = [int(v) for v in vals]
    return kv


# ------------------------------------------------------------------ reorder

def test_fractal_order_matches_hand_derivation(golden_dir):
    g = _read_golden(os.path.join(golden_dir, "fractal_order_T2_H3_W5_P2.txt"))
    T, H, W, P = g["T"][0], g["H"][0], g["W"][0], g["P"][0]
    assert oracle.fractal_order(T, H, W, P).tolist() == g["order"]


def test_fractal_order_landmarks():
    o = oracle.fractal_order(1, 16, 16, 8)
    # second patch of the first patch row starts with token (t=0, h=0, w=8)
    assert o[64] == 8
    # second patch row starts with token (0, 8, 0)
    assert o[128] == 8 * 16
    # inside a patch: row-major
    assert o[:10].tolist() == [0, 1, 2, 3, 4, 5, 6, 7, 16, 17]


@pytest.mark.parametrize("T,H,W,P", [(4, 16, 16, 8), (2, 24, 40, 8)])
def test_aligned_blocks_are_single_patches(T, H, W, P):
    o = oracle.fractal_order(T, H, W, P)
    bs = P * P
    for I in range(len(o) // bs):
        toks = o[I * bs:(I + 1) * bs]
        t = toks // (H * W)
        h = (toks % (H * W)) // W
        w = toks % W
        assert len(set(t.tolist())) == 1
        assert len(set((h // P).tolist())) == 1 and len(set((w // P).tolist())) == 1
        assert sorted(set(h.tolist())) == list(range(h.min(), h.min() + P))


@pytest.mark.parametrize("T,H,W,P,bs", [(1, 3, 5, 2, 4), (2, 7, 9, 4, 16), (3, 10, 13, 8, 64), (2, 8, 8, 8, 64)])
def test_reorder_is_a_bijection(T, H, W, P, bs):
    rng = np.random.default_rng(0)
    N = T * H * W
    o = oracle.fractal_order(T, H, W, P)
    assert sorted(o.tolist()) == list(range(N))
    x = rng.standard_normal((2, N, 3, 4))
    y = oracle.reorder(x, T, H, W, P, bs)
    assert y.shape == (2, 3, nabla.padded_len(N, bs), 4)
    assert np.all(y[:, :, N:, :] == 0.0)
    assert np.array_equal(oracle.inverse_reorder(y, T, H, W, P), x)
    # reorder moves whole token rows: position p holds the token the order names
    p = N // 2
    assert np.array_equal(y[1, 2, p], x[1, o[p], 2])


# ------------------------------------------------------------------ pooling

def test_block_means_closed_forms():
    # constant -> the constant; ramp value = position -> midpoint of valid positions
    N, bs, d = 70, 64, 3
    Npad = nabla.padded_len(N, bs)
    y = np.zeros((1, 1, Npad, d))
    y[0, 0, :N, 0] = 2.5
    y[0, 0, :N, 1] = np.arange(N)
    y[0, 0, N:, :] = 1e9        # padding must not leak into the means
    m = oracle.block_means(y, N, bs)
    assert m.shape == (1, 1, 2, d)
    assert np.allclose(m[0, 0, :, 0], 2.5, rtol=0, atol=1e-15)
    assert m[0, 0, 0, 1] == (0 + 63) / 2
    assert m[0, 0, 1, 1] == (64 + 69) / 2
    assert np.all(m[0, 0, :, 2] == 0.0)


# --------------------------------------------------------- reduced attention

def test_reduced_attention_closed_forms():
    # equal pooled keys -> uniform rows
    kb = np.tile(np.array([[0.3, -1.0, 2.0, 0.5]]), (5, 1))
    qb = np.random.default_rng(1).standard_normal((5, 4))
    A = oracle.reduced_attention(qb, kb)
    assert np.allclose(A, 1 / 5, atol=1e-15)
    # two blocks, d = 2: s = (q.k0, q.k1)/sqrt(2) = (sqrt(2), 0) -> logistic
    qb = np.array([[1.0, 0.0]])
    kb = np.array([[2.0, 0.0], [0.0, 0.0]])
    A = oracle.reduced_attention(qb, kb)
    want0 = 1.0 / (1.0 + math.exp(-math.sqrt(2.0)))
    assert abs(A[0, 0] - want0) < 1e-15 and abs(A[0, 1] - (1 - want0)) < 1e-15
    # a transposed operand would break the asymmetric case: q only sees its own row
    qb = np.array([[1.0, 0.0], [0.0, 0.0]])
    kb = np.array([[0.0, 0.0], [3.0, 0.0]])
    A = oracle.reduced_attention(qb, kb)
    assert A[0, 1] > 0.8 and np.allclose(A[1], 0.5)


def test_reduced_attention_rows_are_distributions():
    rng = np.random.default_rng(2)
    A = oracle.reduced_attention(rng.standard_normal((3, 40, 16)) * 4, rng.standard_normal((3, 40, 16)) * 4)
    assert np.all(A > 0)
    assert np.allclose(A.sum(-1), 1.0, atol=1e-12)
    # against torch's softmax in float64 (a different library routine)
    qb = rng.standard_normal((40, 16))
    kb = rng.standard_normal((40, 16))
    ref = torch.softmax(torch.from_numpy(qb @ kb.T / 4.0), dim=-1).numpy()
    assert np.allclose(oracle.reduced_attention(qb, kb), ref, rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------ CDF threshold

def test_cdf_matches_hand_examples(golden_dir):
    with open(os.path.join(golden_dir, "cdf_threshold_examples.txt")) as f:
        rows = [l for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 5
    for line in rows:
        thr, probs, kept = [p.strip() for p in line.split("|")]
        A = np.array([float(x) for x in probs.split()])[None]
        keep, _ = oracle.cdf_keep(A, float(thr))
        assert np.nonzero(keep[0])[0].tolist() == [int(x) for x in kept.split()], line


def test_cdf_is_minimal_by_brute_force():
    rng = np.random.default_rng(3)
    for trial in range(300):
        nb = int(rng.integers(1, 11))
        A = rng.dirichlet(np.full(nb, float(rng.choice([0.3, 1.0, 3.0]))))[None]
        thr = float(rng.uniform(0.0, 0.95))
        keep, amb = oracle.cdf_keep(A, thr)
        if amb.any():
            continue
        target = 1.0 - thr
        best_k, best_mass = None, -1.0
        for k in range(1, nb + 1):
            masses = [sum(A[0, list(c)]) for c in itertools.combinations(range(nb), k)]
            if max(masses) >= target - 1e-12:
                best_k, best_mass = k, max(masses)
                break
        if thr == 0.0:
            best_k = nb
        assert keep.sum() == best_k, (A, thr)
        # the kept set carries the largest mass among sets of that size
        assert abs(A[0, keep[0]].sum() - best_mass) < 1e-12


def test_cdf_extremes():
    rng = np.random.default_rng(4)
    A = rng.dirichlet(np.ones(30), size=4)
    keep, _ = oracle.cdf_keep(A, 0.0)
    assert keep.all()
    keep, _ = oracle.cdf_keep(A, 1.0 - 1e-12)
    assert np.array_equal(keep, A == A.max(axis=1, keepdims=True))
    with pytest.raises(ValueError):
        oracle.cdf_keep(A, 1.0)


def test_cdf_flags_blocks_near_the_threshold():
    # ranked: 0.4 (J0), 0.25 (J3), 0.2 (J1), 0.15 (J2); prefix mass ahead of each:
    # J0 0, J3 0.4, J1 0.65, J2 0.85.  Target 0.6000005 is far from all of them.
    A = np.array([[0.4, 0.2, 0.15, 0.25]])
    keep, amb = oracle.cdf_keep(A, 1.0 - 0.6000005)
    assert not amb.any()
    A = np.array([[0.4, 0.2, 0.15, 0.25]])
    keep, amb = oracle.cdf_keep(A, 1.0 - 0.65 + 4e-7)   # target 0.6499996 ~ prefix 0.65 before J1
    assert amb[0, 1] and not amb[0, 0]


def test_cdf_flags_an_exact_tie_at_the_boundary():
    # target 0.65: ranked 0.4 (J0), 0.3 (J1), 0.3 (J2); the tie J1/J2 decides
    # which block is the last kept one, so both are ambiguous; J0 is not.
    A = np.array([[0.4, 0.3, 0.3]])
    keep, amb = oracle.cdf_keep(A, 0.35)
    assert keep[0].tolist() == [True, True, False]
    assert amb[0].tolist() == [False, True, True]


def test_cdf_does_not_flag_a_tie_away_from_the_boundary():
    # target 0.8: ranked 0.3 (J0), 0.3 (J1), 0.25 (J2), 0.15 (J3); the tie J0/J1
    # lies inside the kept set and the boundary block J2 has no near-equal peer.
    A = np.array([[0.3, 0.3, 0.25, 0.15]])
    keep, amb = oracle.cdf_keep(A, 0.2)
    assert keep[0].tolist() == [True, True, True, False]
    assert not amb.any()


def test_cdf_near_tie_window_is_relative_1e9():
    # the boundary block J1 and J2 differ by 2e-12 relative: flagged; by 2e-6: not.
    for rel, flagged in ((1e-12, True), (1e-6, False)):
        A = np.array([[0.4, 0.3 * (1 + rel), 0.3 * (1 - rel)]])
        keep, amb = oracle.cdf_keep(A, 0.35)
        assert keep[0].tolist() == [True, True, False]
        assert amb[0].tolist() == [False, flagged, flagged], rel


def test_pins_catch_a_dropped_tie_rule(monkeypatch):
    orig = nabla.cdf_keep

    def no_tie_rule(A, thr):   # only the prefix-mass rule flags blocks
        keep, _ = orig(A, thr)
        amb = np.zeros_like(keep)
        flat_a, flat_m = A.reshape(-1, A.shape[-1]), amb.reshape(-1, A.shape[-1])
        for r in range(flat_a.shape[0]):
            order = np.argsort(-flat_a[r], kind="stable")
            before = np.concatenate([[0.0], np.cumsum(flat_a[r][order])[:-1]])
            flat_m[r, order[np.abs(before - (1.0 - thr)) <= nabla.AMBIGUITY_MASS]] = True
        return keep, amb
    monkeypatch.setattr(oracle, "cdf_keep", no_tie_rule)
    with pytest.raises(AssertionError):
        test_cdf_flags_an_exact_tie_at_the_boundary()


def test_pins_catch_a_tie_window_that_is_too_wide(monkeypatch):
    monkeypatch.setattr(nabla, "AMBIGUITY_TIE_REL", 0.5)
    with pytest.raises(AssertionError):
        test_cdf_does_not_flag_a_tie_away_from_the_boundary()


# ----------------------------------------------------------------- STA

def test_sta_on_aligned_grid_is_the_tile_window():
    T, H, W, P = 3, 24, 24, 8
    bs = P * P
    nPr, nPc = H // P, W // P
    m = oracle.sta_mask(T, H, W, P, bs, (1, 1, 1))
    nb = T * nPr * nPc
    assert m.shape == (nb, nb)
    for I in range(nb):
        tI, rI, cI = I // (nPr * nPc), (I // nPc) % nPr, I % nPc
        for J in range(nb):
            tJ, rJ, cJ = J // (nPr * nPc), (J // nPc) % nPr, J % nPc
            want = abs(tI - tJ) <= 1 and abs(rI - rJ) <= 1 and abs(cI - cJ) <= 1
            assert m[I, J] == want
    # an interior block sees exactly 27 tiles; a corner block 8
    assert m[1 * nPr * nPc + 1 * nPc + 1].sum() == 27
    assert m[0].sum() == 2 * 2 * 2


def _sta_golden(golden_dir):
    return _read_golden(os.path.join(golden_dir, "sta_tiles_T2_H5_W7_P4_bs8.txt"))


def _sta_golden_mismatches(g):
    """Differences between the oracle's tiles / windows and the hand-derived
    file (empty when they agree).  Looks the functions up on the module at
    call time, so a planted mistake is seen."""
    T, H, W, P, bs = g["T"][0], g["H"][0], g["W"][0], g["P"][0], g["block"][0]
    bad = []
    tiles = nabla.block_tiles(T, H, W, P, bs)
    nb = tiles.shape[0]
    if nb != len(g["first"]):
        return [("nb", nb)]
    for I in range(nb):
        if tiles[I].tolist() != g[f"tile{I}"]:
            bad.append(("tile", I, tiles[I].tolist(), g[f"tile{I}"]))
    for half, key in (((0, 0, 0), "w000"), ((1, 0, 0), "w100"), ((0, 0, 1), "w001")):
        m = nabla.sta_mask(T, H, W, P, bs, half)
        for I in range(nb):
            if np.nonzero(m[I])[0].tolist() != g[f"{key}_{I}"]:
                bad.append((key, I, np.nonzero(m[I])[0].tolist(), g[f"{key}_{I}"]))
    return bad


def test_sta_on_ragged_grid_matches_hand_derivation(golden_dir):
    g = _sta_golden(golden_dir)
    o = oracle.fractal_order(g["T"][0], g["H"][0], g["W"][0], g["P"][0])
    # the first token of each block is the position the file names
    assert [8 * I for I in range(len(g["first"]))] == g["first"]
    assert o.size == 70
    assert _sta_golden_mismatches(g) == []


def _tiles_of(token_of_block):
    """block_tiles with another choice of the block's representative token."""
    def tiles(T, H, W, P, block):
        N = T * H * W
        order = nabla.fractal_order(T, H, W, P)
        nb = nabla.num_blocks(N, block)
        out = np.zeros((nb, 3), dtype=np.int64)
        for I in range(nb):
            n = int(token_of_block(order, I, block, N))
            t, rem = divmod(n, H * W)
            h, w = divmod(rem, W)
            out[I] = (t, h // P, w // P)
        return out
    return tiles


@pytest.mark.parametrize("mistake", ["last_token", "majority_tile", "position_as_token"])
def test_pins_catch_a_wrong_block_tile(monkeypatch, golden_dir, mistake):
    if mistake == "last_token":
        bad = _tiles_of(lambda order, I, bs, N: order[min((I + 1) * bs, N) - 1])
    elif mistake == "position_as_token":
        bad = _tiles_of(lambda order, I, bs, N: I * bs)
    else:
        def bad(T, H, W, P, block):
            N = T * H * W
            order = nabla.fractal_order(T, H, W, P)
            nb = nabla.num_blocks(N, block)
            out = np.zeros((nb, 3), dtype=np.int64)
            for I in range(nb):
                toks = order[I * block:min((I + 1) * block, N)]
                t = toks // (H * W)
                h = (toks % (H * W)) // W
                w = toks % W
                keys, counts = np.unique(np.stack([t, h // P, w // P], 1), axis=0, return_counts=True)
                out[I] = keys[np.argmax(counts)]
            return out
    monkeypatch.setattr(nabla, "block_tiles", bad)
    assert _sta_golden_mismatches(_sta_golden(golden_dir)) != []


def test_hybrid_mask_contains_both_parts():
    rng = np.random.default_rng(5)
    T, H, W, P, bs = 2, 12, 20, 4, 16
    N = T * H * W
    q = oracle.reorder(rng.standard_normal((1, N, 2, 8)), T, H, W, P, bs)
    k = oracle.reorder(rng.standard_normal((1, N, 2, 8)), T, H, W, P, bs)
    keep_a, _ = oracle.block_mask(q, k, T, H, W, P, bs, 0.3)
    keep_h, _ = oracle.block_mask(q, k, T, H, W, P, bs, 0.3, sta=(1, 1, 1))
    sta = oracle.sta_mask(T, H, W, P, bs, (1, 1, 1))
    assert np.array_equal(keep_h, keep_a | sta[None, None])


# ------------------------------------------------------------- attention

def _sdpa_rows(q, k, v, keymask, scale):
    """torch SDPA in float64 with a boolean mask (True = take part)."""
    out = F.scaled_dot_product_attention(torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
                                         torch.from_numpy(v)[None, None],
                                         attn_mask=torch.from_numpy(keymask)[None, None], scale=scale)
    return out[0, 0].numpy()


@pytest.mark.parametrize("N,bs", [(96, 32), (100, 32)])
def test_masked_attention_equals_library_attention(N, bs):
    rng = np.random.default_rng(6)
    d, heads = 16, 2
    Npad = nabla.padded_len(N, bs)
    nb = Npad // bs
    q = rng.standard_normal((1, heads, Npad, d)) * 2
    k = rng.standard_normal((1, heads, Npad, d)) * 2
    v = rng.standard_normal((1, heads, Npad, d))
    keep = rng.random((1, heads, nb, nb)) < 0.5
    keep[..., np.arange(nb), np.arange(nb)] = True
    O, lse = oracle.masked_attention(q, k, v, keep, N, bs)
    scale = 1 / math.sqrt(d)
    for h in range(heads):
        tokmask = np.kron(keep[0, h], np.ones((bs, bs), dtype=bool))[:N, :N]
        ref = _sdpa_rows(q[0, h, :N], k[0, h, :N], v[0, h, :N], tokmask, scale)
        assert np.allclose(O[0, h, :N], ref, rtol=1e-12, atol=1e-12)
        s = (q[0, h, :N] @ k[0, h, :N].T) * scale
        s[~tokmask] = -np.inf
        ref_lse = torch.logsumexp(torch.from_numpy(s), dim=-1).numpy()
        assert np.allclose(lse[0, h, :N], ref_lse, rtol=1e-12, atol=1e-12)
    assert np.all(O[:, :, N:] == 0) and np.all(lse[:, :, N:] == 0)


def test_attention_special_cases():
    rng = np.random.default_rng(7)
    N, bs, d = 120, 32, 8
    Npad = nabla.padded_len(N, bs)
    nb = Npad // bs
    q = rng.standard_normal((1, 1, Npad, d))
    k = rng.standard_normal((1, 1, Npad, d))
    # V constant -> output is that constant
    v = np.full((1, 1, Npad, d), -0.75)
    keep = rng.random((1, 1, nb, nb)) < 0.6
    keep[..., np.arange(nb), np.arange(nb)] = True
    O, _ = oracle.masked_attention(q, k, v, keep, N, bs)
    assert np.allclose(O[0, 0, :N], -0.75, atol=1e-14)
    # a single kept block whose keys are identical -> mean of that block's valid V
    J = nb - 1                                   # the ragged last block (24 valid keys)
    k2 = k.copy()
    k2[0, 0, J * bs:] = k[0, 0, J * bs]
    v2 = rng.standard_normal((1, 1, Npad, d))
    keep2 = np.zeros((1, 1, nb, nb), dtype=bool)
    keep2[..., J] = True
    O2, _ = oracle.masked_attention(q, k2, v2, keep2, N, bs)
    assert np.allclose(O2[0, 0, :N], v2[0, 0, J * bs:N].mean(axis=0), atol=1e-13)


def test_thr_zero_pipeline_is_dense_attention_in_model_order():
    """thr = 0 keeps every block; reorder -> attention -> inverse must then equal
    dense attention applied directly to the model-order tokens."""
    rng = np.random.default_rng(8)
    T, H, W, P, bs = 2, 6, 10, 4, 16
    N, heads, d = T * H * W, 2, 8
    q = rng.standard_normal((1, N, heads, d))
    k = rng.standard_normal((1, N, heads, d))
    v = rng.standard_normal((1, N, heads, d))
    O, keep, amb = oracle.nabla_attention(q, k, v, T, H, W, P, bs, 0.0)
    assert keep.all() and not amb.any()
    for h in range(heads):
        ref = _sdpa_rows(q[0, :, h], k[0, :, h], v[0, :, h], np.ones((N, N), dtype=bool), 1 / math.sqrt(d))
        assert np.allclose(O[0, :, h], ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- backward

@pytest.mark.parametrize("N,bs", [(96, 32), (100, 32)])
def test_backward_equals_library_autograd(N, bs):
    """The oracle's gradients equal torch autograd (float64) through the
    library attention (scaled_dot_product_attention) with the expanded mask."""
    rng = np.random.default_rng(11)
    d, heads = 16, 2
    Npad = nabla.padded_len(N, bs)
    nb = Npad // bs
    q = rng.standard_normal((1, heads, Npad, d)) * 1.5
    k = rng.standard_normal((1, heads, Npad, d)) * 1.5
    v = rng.standard_normal((1, heads, Npad, d))
    dO = rng.standard_normal((1, heads, Npad, d))
    keep = rng.random((1, heads, nb, nb)) < 0.5
    keep[..., np.arange(nb), np.arange(nb)] = True
    dq, dk, dv = oracle.masked_attention_backward(q, k, v, keep, dO, N, bs)
    scale = 1 / math.sqrt(d)
    for h in range(heads):
        tokmask = torch.from_numpy(np.kron(keep[0, h], np.ones((bs, bs), dtype=bool))[:N, :N])
        tq, tk, tv = (torch.from_numpy(x[0, h, :N].copy()).requires_grad_() for x in (q, k, v))
        out = F.scaled_dot_product_attention(tq[None, None], tk[None, None], tv[None, None],
                                             attn_mask=tokmask[None, None], scale=scale)[0, 0]
        out.backward(torch.from_numpy(dO[0, h, :N].copy()))
        assert np.allclose(dq[0, h, :N], tq.grad.numpy(), rtol=1e-11, atol=1e-12)
        assert np.allclose(dk[0, h, :N], tk.grad.numpy(), rtol=1e-11, atol=1e-12)
        assert np.allclose(dv[0, h, :N], tv.grad.numpy(), rtol=1e-11, atol=1e-12)
    for g in (dq, dk, dv):
        assert np.all(g[:, :, N:] == 0)


def test_backward_matches_central_differences():
    """d<O, dO>/dx by central differences (step 1e-6) at a few entries of
    q, k and v, on a tiny masked problem with a ragged last block."""
    rng = np.random.default_rng(12)
    N, bs, d = 40, 16, 4
    Npad = nabla.padded_len(N, bs)
    nb = Npad // bs
    x = {n: rng.standard_normal((1, 1, Npad, d)) for n in ("q", "k", "v")}
    dO = rng.standard_normal((1, 1, Npad, d))
    keep = np.array([[[[True, False, True], [True, True, False], [False, True, True]]]])
    grads = dict(zip(("q", "k", "v"), oracle.masked_attention_backward(x["q"], x["k"], x["v"], keep, dO, N, bs)))

    def loss(xx):
        O, _ = oracle.masked_attention(xx["q"], xx["k"], xx["v"], keep, N, bs)
        return float((O[:, :, :N] * dO[:, :, :N]).sum())

    eps = 1e-6
    for name in ("q", "k", "v"):
        for (row, col) in ((0, 0), (17, 2), (N - 1, 3), (33, 1)):
            xp = {n: a.copy() for n, a in x.items()}
            xm = {n: a.copy() for n, a in x.items()}
            xp[name][0, 0, row, col] += eps
            xm[name][0, 0, row, col] -= eps
            fd = (loss(xp) - loss(xm)) / (2 * eps)
            assert abs(fd - grads[name][0, 0, row, col]) < 1e-7 * max(1.0, abs(fd)), (name, row, col)


def test_pins_catch_a_backward_without_the_softmax_jacobian_term(monkeypatch):
    def bad(q, k, v, keep, dO, N, block, scale=None):   # dS = P * dP: the rowsum(dO * O) term dropped
        B, heads, Npad, d = q.shape
        scale = 1.0 / math.sqrt(d) if scale is None else scale
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        for h in range(heads):
            for I in range(Npad // block):
                lo, hi = I * block, min((I + 1) * block, N)
                cols = np.concatenate([np.arange(J * block, min((J + 1) * block, N))
                                       for J in np.nonzero(keep[0, h, I])[0]])
                s_ = (q[0, h, lo:hi] @ k[0, h, cols].T) * scale
                P = np.exp(s_ - s_.max(1, keepdims=True))
                P /= P.sum(1, keepdims=True)
                dS = P * (dO[0, h, lo:hi] @ v[0, h, cols].T)
                dv[0, h, cols] += P.T @ dO[0, h, lo:hi]
                dq[0, h, lo:hi] += scale * dS @ k[0, h, cols]
                dk[0, h, cols] += scale * dS.T @ q[0, h, lo:hi]
        return dq, dk, dv
    monkeypatch.setattr(oracle, "masked_attention_backward", bad)
    with pytest.raises(AssertionError):
        test_backward_equals_library_autograd(96, 32)


# ------------------------------------------------- Hilbert order, sub-blocks

def test_hilbert_2x2x2_matches_hand_derivation(golden_dir):
    g = _read_golden(os.path.join(golden_dir, "hilbert_order_2x2x2.txt"))
    assert oracle.hilbert_order(2, 2, 2).tolist() == g["order"]
    assert [oracle.hilbert_index((n // 4, (n // 2) % 2, n % 2), 1) for n in range(8)] == g["index"]


def _hilbert_curve_properties(bits):
    """The cube's points in curve order, checked for the properties that
    define a Hilbert curve: a bijection onto [0, 8^bits), consecutive points
    one step apart, and every aligned sub-cube of side 2^k visited as one
    contiguous run of 8^k points."""
    side = 1 << bits
    pts = [(t, h, w) for t in range(side) for h in range(side) for w in range(side)]
    idx = [nabla.hilbert_index(p, bits) for p in pts]
    if sorted(idx) != list(range(side ** 3)):
        return False
    path = [p for _, p in sorted(zip(idx, pts))]
    if any(sum(abs(a - b) for a, b in zip(path[i], path[i + 1])) != 1 for i in range(len(path) - 1)):
        return False
    for k in range(1, bits):
        runs = {}
        for pos, p in enumerate(path):
            runs.setdefault(tuple(c >> k for c in p), []).append(pos)
        for positions in runs.values():
            if positions != list(range(positions[0], positions[0] + 8 ** k)):
                return False
    return path[0] == (0, 0, 0)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_hilbert_curve_is_continuous_and_hierarchical(bits):
    assert _hilbert_curve_properties(bits)


def test_pins_catch_a_hilbert_curve_without_the_gray_encoding(monkeypatch):
    def bad(coords, bits):          # interleaves the raw coordinate bits (a Z-order curve)
        h = 0
        for b in range(bits - 1, -1, -1):
            for c in coords:
                h = (h << 1) | ((int(c) >> b) & 1)
        return h
    monkeypatch.setattr(nabla, "hilbert_index", bad)
    assert not _hilbert_curve_properties(2)


def test_hilbert_order_of_a_ragged_grid_is_the_cube_order_restricted():
    T, H, W = 3, 5, 6
    o = oracle.hilbert_order(T, H, W)
    assert sorted(o.tolist()) == list(range(T * H * W))
    bits = oracle.hilbert_bits(T, H, W)
    keys = [nabla.hilbert_index((n // (H * W), (n // W) % H, n % W), bits) for n in o]
    assert keys == sorted(keys)
    # a reorder by it is a bijection of the token rows, zero tail
    x = np.random.default_rng(13).standard_normal((1, T * H * W, 2, 3))
    y = nabla.reorder_by(x, o, 16)
    assert np.all(y[:, :, T * H * W:] == 0)
    assert np.array_equal(y[0, 1, 7], x[0, o[7], 1])


def test_subblock_scores_with_one_subblock_per_block_is_the_reduced_map():
    rng = np.random.default_rng(14)
    N, bs, d = 100, 32, 8
    q = rng.standard_normal((1, 2, nabla.padded_len(N, bs), d))
    k = rng.standard_normal((1, 2, nabla.padded_len(N, bs), d))
    q[:, :, N:] = 0
    k[:, :, N:] = 0
    want = oracle.reduced_attention(oracle.block_means(q, N, bs), oracle.block_means(k, N, bs))
    assert np.allclose(oracle.subblock_scores(q, k, N, bs, bs), want, rtol=0, atol=1e-15)


def test_subblock_scores_closed_forms():
    rng = np.random.default_rng(15)
    N, bs, sub, d = 100, 32, 8, 4       # 13 valid sub-blocks: 4 + 4 + 4 + 1
    Npad = nabla.padded_len(N, bs)
    q = rng.standard_normal((1, 1, Npad, d))
    # identical key sub-blocks: every query sub-block spreads its mass evenly,
    # so block J's importance is its share of the valid key sub-blocks
    k = np.tile(rng.standard_normal((1, 1, 1, d)), (1, 1, Npad, 1))
    M = oracle.subblock_scores(q, k, N, bs, sub)
    assert np.allclose(M[0, 0], np.array([4, 4, 4, 1]) / 13.0, rtol=0, atol=1e-15)
    # rows are distributions for any input
    k = rng.standard_normal((1, 1, Npad, d)) * 3
    M = oracle.subblock_scores(q, k, N, bs, sub)
    assert np.all(M >= 0) and np.allclose(M.sum(-1), 1.0, atol=1e-12)


def test_pins_catch_subblock_scores_that_average_instead_of_summing(monkeypatch):
    orig = nabla.subblock_scores

    def bad(q, k, N, block, sub, scale=None):
        per = block // sub
        return orig(q, k, N, block, sub, scale) / per
    monkeypatch.setattr(oracle, "subblock_scores", bad)
    with pytest.raises(AssertionError):
        test_subblock_scores_closed_forms()


# ------------------------------------------------------------ radius masks

def test_attention_entropy_against_library_and_closed_forms():
    rng = np.random.default_rng(21)
    N, bs, d = 50, 16, 8
    Npad = nabla.padded_len(N, bs)
    q = rng.standard_normal((1, 2, Npad, d)) * 2
    k = rng.standard_normal((1, 2, Npad, d)) * 2
    H = oracle.attention_entropy(q, k, N)
    for h in range(2):
        logits = torch.from_numpy(q[0, h, :N] @ k[0, h, :N].T / math.sqrt(d))
        ref = torch.distributions.Categorical(logits=logits).entropy().numpy()
        assert np.allclose(H[0, h, :N], ref, rtol=1e-12, atol=1e-12)
    assert np.all(H[:, :, N:] == 0)
    # identical keys: a uniform distribution over the N valid keys
    k_eq = np.tile(k[:, :, :1], (1, 1, Npad, 1))
    assert np.allclose(oracle.attention_entropy(q, k_eq, N)[:, :, :N], math.log(N), atol=1e-12)


def test_token_radius_closed_form():
    T, N = 3, 30
    t_of = np.repeat(np.arange(T), N // T)
    H = np.full((1, 1, N), math.log(12.0))
    r = oracle.token_radius(H, t_of, T, 2.0, 0.5, N)
    # budget 2 * 12 = 24 tokens; a query in frame 0 has disks of area pi r^2 (1 + e^-1 + e^-2)
    assert abs(r[0, 0, 0] - math.sqrt(24.0 / (math.pi * (1 + math.exp(-1) + math.exp(-2))))) < 1e-12
    # frame 1 (middle): 1 + 2 e^-1
    assert abs(r[0, 0, 10] - math.sqrt(24.0 / (math.pi * (1 + 2 * math.exp(-1))))) < 1e-12
    # the budget is clamped to [1, N]
    r = oracle.token_radius(np.full((1, 1, N), 50.0), t_of, 1, 1.0, 0.0, N)
    assert abs(r[0, 0, 0] - math.sqrt(N / math.pi)) < 1e-12


def _radius_mask_brute(r_tok, T, H, W, P, bs, gamma, vote):
    """Token-level support by explicit loops over original (t, h, w)
    coordinates, blocks through the inverse of the fractal order."""
    N = T * H * W
    pos = np.empty(N, dtype=np.int64)
    pos[oracle.fractal_order(T, H, W, P)] = np.arange(N)       # token -> position
    nb = nabla.num_blocks(N, bs)
    votes = np.zeros((nb, nb), dtype=np.int64)
    for ti in range(T):
        for hi in range(H):
            for wi in range(W):
                i = ti * H * W + hi * W + wi
                hit = set()
                for tj in range(T):
                    rad = r_tok[i] * math.exp(-gamma * abs(tj - ti))
                    for hj in range(H):
                        for wj in range(W):
                            if (hj - hi) ** 2 + (wj - wi) ** 2 <= rad * rad:
                                hit.add(pos[tj * H * W + hj * W + wj] // bs)
                for J in hit:
                    votes[pos[i] // bs, J] += 1
    return votes >= vote


@pytest.mark.parametrize("gamma,vote", [(0.0, 1), (0.7, 1), (0.7, 3)])
def test_radius_block_mask_by_brute_force(gamma, vote):
    rng = np.random.default_rng(22)
    T, H, W, P, bs = 3, 5, 7, 4, 8
    N = T * H * W
    r_tok = rng.uniform(0.0, 2.5, N)                      # radius per token (model order)
    order = oracle.fractal_order(T, H, W, P)
    r_pos = np.zeros((1, 1, nabla.padded_len(N, bs)))
    r_pos[0, 0, :N] = r_tok[order]
    got = oracle.radius_block_mask(r_pos, T, H, W, P, bs, gamma, vote)[0, 0]
    assert np.array_equal(got, _radius_mask_brute(r_tok, T, H, W, P, bs, gamma, vote))


def test_radius_zero_is_the_same_position_in_every_frame():
    """r = 0, no decay: a query's support is its own (h, w) in every frame; on
    an aligned grid (blocks = patches) that is the STA window (T, 0, 0)."""
    T, H, W, P = 3, 16, 16, 8
    bs = P * P
    r = np.zeros((1, 1, T * H * W))
    keep = oracle.radius_block_mask(r, T, H, W, P, bs, 0.0, 1)[0, 0]
    assert np.array_equal(keep, oracle.sta_mask(T, H, W, P, bs, (T, 0, 0)))


def test_pins_catch_a_radius_mask_without_temporal_decay(monkeypatch):
    orig = nabla.radius_block_mask

    def bad(r, T, H, W, P, block, gamma, vote=1):
        return orig(r, T, H, W, P, block, 0.0, vote)
    monkeypatch.setattr(oracle, "radius_block_mask", bad)
    with pytest.raises(AssertionError):
        test_radius_block_mask_by_brute_force(0.7, 1)


def test_subblock_mask_with_whole_blocks_is_the_nabla_mask():
    """Sub-blocks as large as the blocks: the sub-block mask is NABLA's block
    mask (reduced map of the block means + CDF rule), reached by another route."""
    rng = np.random.default_rng(16)
    T, H, W, P, bs, d = 2, 6, 10, 4, 16, 8
    N = T * H * W
    Npad = nabla.padded_len(N, bs)
    q = rng.standard_normal((1, 2, Npad, d)) * 1.5
    k = rng.standard_normal((1, 2, Npad, d)) * 1.5
    q[:, :, N:] = 0
    k[:, :, N:] = 0
    keep_sub, amb_sub = oracle.block_mask_subblock(q, k, N, bs, bs, 0.2)
    keep_nabla, amb_nabla = oracle.block_mask(q, k, T, H, W, P, bs, 0.2)
    assert np.array_equal(keep_sub, keep_nabla) and np.array_equal(amb_sub, amb_nabla)


def test_radius_chain_against_library_entropy_and_brute_force():
    """The whole chain on reordered Q, K: entropies from torch's categorical
    entropy, radii from the closed form, the mask by brute force over the
    original coordinates."""
    rng = np.random.default_rng(23)
    T, H, W, P, bs, d = 3, 5, 7, 4, 8, 8
    N = T * H * W
    Npad = nabla.padded_len(N, bs)
    q = rng.standard_normal((1, 1, Npad, d)) * 1.5
    k = rng.standard_normal((1, 1, Npad, d)) * 1.5
    q[:, :, N:] = 0
    k[:, :, N:] = 0
    tau, gamma = 0.3, 0.6
    got = oracle.radius_mask_from_qk(q, k, T, H, W, P, bs, tau, gamma, vote=2)[0, 0]
    logits = torch.from_numpy(q[0, 0, :N] @ k[0, 0, :N].T / math.sqrt(d))
    ent = torch.distributions.Categorical(logits=logits).entropy().numpy()   # per position
    order = oracle.fractal_order(T, H, W, P)
    r_tok = np.zeros(N)
    for p_ in range(N):
        n = order[p_]
        t = n // (H * W)
        budget = min(max(tau * math.exp(ent[p_]), 1.0), float(N))
        area = math.pi * sum(math.exp(-2 * gamma * abs(tt - t)) for tt in range(T))
        r_tok[n] = math.sqrt(budget / area)
    assert np.array_equal(got, _radius_mask_brute(r_tok, T, H, W, P, bs, gamma, 2))


def test_density_and_attention_flops_closed_forms():
    keep = np.zeros((1, 2, 4, 4), dtype=bool)
    keep[0, 0, :, 0] = True
    keep[0, 1] = True
    assert oracle.density(keep) == (4 + 16) / 32
    assert oracle.attention_flops(1000, 64, 3, 2, 0.25) == 4.0 * 1000 * 1000 * 64 * 3 * 2 * 0.25


# ----------------------------------------------- fine-grained KV selection

def _fine_lists(keep_blocks, per):
    """CSR lists of 4-token blocks covering the kept 64-token blocks (nq x nb bool)."""
    off, idx = [0], []
    for row in keep_blocks:
        for J in np.nonzero(row)[0]:
            idx.extend(range(J * per, (J + 1) * per))
        off.append(len(idx))
    return np.asarray(off), np.asarray(idx)


def test_fine_attention_with_whole_blocks_is_block_sparse_attention():
    rng = np.random.default_rng(31)
    N, qb, d = 250, 128, 16
    Npad = nabla.padded_len(N, qb)
    q, k, v = (rng.standard_normal((1, 1, Npad, d)) for _ in range(3))
    keep = rng.random((1, 1, Npad // qb, Npad // qb)) < 0.6
    keep[..., np.arange(Npad // qb), np.arange(Npad // qb)] = True
    off, idx = _fine_lists(keep[0, 0], qb // 4)
    O, lse = oracle.fine_attention(q, k, v, off, idx, None, N)
    O_ref, lse_ref = oracle.masked_attention(q, k, v, keep, N, qb)
    assert np.allclose(O, O_ref, atol=1e-13) and np.allclose(lse, lse_ref, atol=1e-13)


def test_fine_attention_weights_against_library_attention():
    """Weights as an additive log mask in torch SDPA (float64); a uniform
    weight changes nothing (the softmax is shift invariant); a weight of 3 on a
    block acts as three copies of it."""
    rng = np.random.default_rng(32)
    N, d = 100, 8
    Npad = nabla.padded_len(N, 128)
    q, k, v = (rng.standard_normal((1, 1, Npad, d)) for _ in range(3))
    idx = np.sort(rng.choice(N // 4, size=9, replace=False))
    w = rng.uniform(1.0, 6.0, idx.size)
    off = np.array([0, idx.size])
    O, _ = oracle.fine_attention(q, k, v, off, idx, w, N)
    cols = np.concatenate([np.arange(4 * b, 4 * b + 4) for b in idx])
    bias = torch.from_numpy(np.repeat(np.log(w), 4))[None, :].expand(N, -1).contiguous()
    ref = F.scaled_dot_product_attention(torch.from_numpy(q[0, 0, :N])[None, None],
                                         torch.from_numpy(k[0, 0, cols])[None, None],
                                         torch.from_numpy(v[0, 0, cols])[None, None],
                                         attn_mask=bias[None, None], scale=1 / math.sqrt(d))[0, 0].numpy()
    assert np.allclose(O[0, 0, :N], ref, rtol=1e-12, atol=1e-12)
    O1, _ = oracle.fine_attention(q, k, v, off, idx, np.full(idx.size, 2.5), N)
    O0, _ = oracle.fine_attention(q, k, v, off, idx, None, N)
    assert np.allclose(O1, O0, atol=1e-13)
    # weight 3 on block idx[0] == that block listed three times with weight 1
    w3 = np.ones(idx.size)
    w3[0] = 3.0
    O3, _ = oracle.fine_attention(q, k, v, off, idx, w3, N)
    idx_rep = np.concatenate([[idx[0], idx[0]], idx])
    Orep, _ = oracle.fine_attention(q, k, v, np.array([0, idx_rep.size]), idx_rep, None, N)
    assert np.allclose(O3, Orep, atol=1e-13)


def test_fine_attention_block_against_library_attention():
    """One query block alone: rows of a head over the listed 4-token blocks
    (one straddling N), weights as an additive log mask in torch SDPA."""
    rng = np.random.default_rng(33)
    N, d, n = 91, 16, 37
    kh, vh = rng.standard_normal((96, d)), rng.standard_normal((96, d))
    qr = rng.standard_normal((n, d))
    idx = np.array([22, 3, 17, 9])          # block 22 holds keys 88-91: 91 is >= N
    w = np.array([1.0, 4.0, 1.5, 2.0])
    O, lse = oracle.fine_attention_block(qr, kh, vh, idx, w, N)
    cols = np.array([c for b in idx for c in range(4 * b, min(4 * b + 4, N))])
    wcol = np.array([w[e] for e, b in enumerate(idx) for c in range(4 * b, min(4 * b + 4, N))])
    s = qr @ kh[cols].T / math.sqrt(d) + np.log(wcol)[None, :]
    ref = F.scaled_dot_product_attention(torch.from_numpy(qr)[None, None], torch.from_numpy(kh[cols])[None, None],
                                         torch.from_numpy(vh[cols])[None, None],
                                         attn_mask=torch.from_numpy(np.log(wcol))[None, :].expand(n, -1)[None, None],
                                         scale=1 / math.sqrt(d))[0, 0].numpy()
    assert np.allclose(O, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, np.log(np.exp(s).sum(axis=1)), rtol=1e-12, atol=1e-12)
    # an empty list: zeros
    O0, lse0 = oracle.fine_attention_block(qr, kh, vh, np.array([], dtype=np.int64), None, N)
    assert np.all(O0 == 0) and np.all(lse0 == 0)


def test_pins_catch_weights_applied_to_the_numerator_only(monkeypatch):
    orig = nabla.fine_attention

    def bad(q, k, v, off, idx, w, N, qblock=128, kblock=4, scale=None):
        O, lse = orig(q, k, v, off, idx, None, N, qblock, kblock, scale)
        if w is None:
            return O, lse
        return O * float(np.mean(w)), lse
    monkeypatch.setattr(oracle, "fine_attention", bad)
    with pytest.raises(AssertionError):
        test_fine_attention_weights_against_library_attention()


def test_lists_roundtrip():
    rng = np.random.default_rng(9)
    keep = rng.random((2, 3, 7, 7)) < 0.4
    cnt, idx = oracle.mask_to_lists(keep)
    assert np.array_equal(oracle.lists_to_mask(cnt, idx, 7), keep)
    for r in range(cnt.size):
        row = idx.reshape(-1, 7)[r]
        c = cnt.reshape(-1)[r]
        assert np.all(np.diff(row[:c]) > 0) and np.all(row[c:] == -1)


# ------------------------------------------------ planted mistakes are caught

def test_pins_catch_an_off_by_one_cdf(monkeypatch):
    def bad(A, thr):  # keeps one block too few
        keep, amb = orig(A, thr)
        for r in np.ndindex(keep.shape[:-1]):
            js = np.nonzero(keep[r])[0]
            if len(js) > 1:
                weakest = js[np.argmin(A[r][js])]
                keep[r + (weakest,)] = False
        return keep, amb
    orig = nabla.cdf_keep
    monkeypatch.setattr(oracle, "cdf_keep", bad)
    with pytest.raises(AssertionError):
        test_cdf_is_minimal_by_brute_force()


def test_pins_catch_a_transposed_patch_order(monkeypatch, golden_dir):
    def bad(T, H, W, P):  # patches column-major instead of row-major
        order = []
        for t in range(T):
            for pc in range(-(-W // P)):
                for pr in range(-(-H // P)):
                    for h in range(pr * P, min((pr + 1) * P, H)):
                        for w in range(pc * P, min((pc + 1) * P, W)):
                            order.append(t * H * W + h * W + w)
        return np.asarray(order)
    monkeypatch.setattr(oracle, "fractal_order", bad)
    with pytest.raises(AssertionError):
        test_fractal_order_matches_hand_derivation(golden_dir)
