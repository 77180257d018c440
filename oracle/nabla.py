"""Plain fp64 CPU oracle of NABLA-style block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
and reference legs of ``bench.py`` use it.  It shares no code with the CUDA
path.

Every function writes out a definition from the NABLA technical summary
("NABLA - Atencion de Bloque Adaptativa al Vecindario para la Generacion
Eficiente de Video", gist.science/es/paper/2507.13546), cited below as
"NABLA summary" plus the section.  Arithmetic is float64 throughout, applied to
the exact float64 values of the bf16 inputs.  Library primitives (a matmul, a
stable argsort, a cumulative sum, exp) serve as single steps; there is no
blocking or fusion beyond what each definition states.

Readings taken where the page is silent or garbled:

* fractal order: one level of P x P grouping, time outermost, patches in
  row-major order, tokens inside a patch in row-major order; edge patches are
  clipped to H and W; the sequence is then zero-padded at its end to a
  multiple of the block size;
* pooling divides by the number of valid (non-padding) tokens of the block;
* softmax scale is 1/sqrt(d) in both the reduced map and the attention;
* CDF rule: sort a row by descending probability (ties: lower block index
  first) and keep the shortest prefix whose mass reaches 1 - thr; thr == 0
  keeps every block; if rounding leaves every prefix short of 1 - thr, every
  block is kept;
* STA: block I sits at the tile (t, h // P, w // P) of its first token in the
  fractal order; blocks I, J are in the window when the tile coordinates
  differ by at most the half-widths in each of t, h, w;
* padded keys take part in nothing; padded query rows output 0 (LSE 0).

Parity pins (tests/test_oracle_pins.py): a hand-derived permutation, the
bijection, closed forms for pooling and the reduced map, brute force over all
subsets for the CDF rule, hand-worked threshold rows including exact and
near ties at the boundary, a hand-derived tile grid for STA on a ragged grid
(blocks straddling patches and frames) and on an aligned one, and a library
attention (torch scaled_dot_product_attention in float64) for the masked
softmax.  The pages print no worked example of the whole path; each
function is pinned on its own, and the composition is pinned at thr = 0,
where reorder -> mask -> attention -> inverse reorder must equal dense
attention on the model-order tokens.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

AMBIGUITY_MASS = 1e-6      # prefix-mass window around 1 - thr
AMBIGUITY_TIE_REL = 1e-9   # relative near-tie window around the boundary block's probability


# ---------------------------------------------------------------- shapes

def padded_len(N: int, block: int) -> int:
    return -(-N // block) * block


def num_blocks(N: int, block: int) -> int:
    return padded_len(N, block) // block


# ------------------------------------------------------- fractal reorder

def fractal_order(T: int, H: int, W: int, P: int) -> np.ndarray:
    """Position p of the reordered sequence -> original token n = t*H*W + h*W + w.

    NABLA summary, Metodologia 1 ("Reordenamiento de Tokens (Aplanamiento
    Fractal)"): tokens of each P x P spatial patch become contiguous and the
    temporal order is kept.
    """
    order = []
    for t in range(T):
        for pr in range(-(-H // P)):
            for pc in range(-(-W // P)):
                for h in range(pr * P, min((pr + 1) * P, H)):
                    for w in range(pc * P, min((pc + 1) * P, W)):
                        order.append(t * H * W + h * W + w)
    return np.asarray(order, dtype=np.int64)


def reorder(x_bnhd: np.ndarray, T: int, H: int, W: int, P: int, block: int) -> np.ndarray:
    """[B, N, heads, d] in model order -> [B, heads, Npad, d] in fractal order, zero tail."""
    B, N, heads, d = x_bnhd.shape
    assert N == T * H * W
    order = fractal_order(T, H, W, P)
    y = np.zeros((B, heads, padded_len(N, block), d), dtype=np.float64)
    for p in range(N):
        y[:, :, p, :] = x_bnhd[:, order[p], :, :]
    return y


def inverse_reorder(y_bhnd: np.ndarray, T: int, H: int, W: int, P: int) -> np.ndarray:
    """Undo ``reorder``: [B, heads, Npad, d] -> [B, N, heads, d], padding dropped."""
    B, heads, _, d = y_bhnd.shape
    N = T * H * W
    order = fractal_order(T, H, W, P)
    x = np.zeros((B, N, heads, d), dtype=np.float64)
    for p in range(N):
        x[:, order[p], :, :] = y_bhnd[:, :, p, :]
    return x


# ------------------------------------------------------------- pooling

def block_means(y_bhnd: np.ndarray, N: int, block: int) -> np.ndarray:
    """Mean of the valid tokens of every block: [B, heads, Npad, d] -> [B, heads, nb, d].

    NABLA summary, Metodologia 2, "Submuestreo": Q and K are averaged over
    blocks of tokens.
    """
    B, heads, Npad, d = y_bhnd.shape
    nb = Npad // block
    out = np.zeros((B, heads, nb, d), dtype=np.float64)
    for I in range(nb):
        lo = I * block
        hi = min((I + 1) * block, N)
        if hi > lo:                       # a block past the last token has no mean (left 0)
            out[:, :, I, :] = y_bhnd[:, :, lo:hi, :].sum(axis=2) / float(hi - lo)
    return out


# ---------------------------------------------------- reduced attention

def reduced_attention(qbar: np.ndarray, kbar: np.ndarray, scale: Optional[float] = None) -> np.ndarray:
    """Row softmax of the pooled scores: [.., nb, d] x [.., nb, d] -> [.., nb, nb].

    NABLA summary, Metodologia 2, "Atencion Reducida": a full attention map over
    the pooled block representations.
    """
    d = qbar.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = np.matmul(qbar, np.swapaxes(kbar, -1, -2)) * scale
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


# ------------------------------------------------------- CDF threshold

def cdf_keep(A: np.ndarray, thr: float) -> Tuple[np.ndarray, np.ndarray]:
    """Binary block mask from a reduced map, plus the ambiguous blocks.

    NABLA summary, Metodologia 2, "Umbralizacion CDF": per row, the blocks are
    taken in decreasing probability and the shortest prefix whose cumulative
    mass reaches 1 - thr is kept.

    Returns ``(keep, ambiguous)``, both bool with the shape of ``A``.  A block is
    ambiguous when the mass of the blocks ranked before it lies within
    ``AMBIGUITY_MASS`` of 1 - thr (its decision flips under rounding), or when
    its probability is within ``AMBIGUITY_TIE_REL`` (relative) of the last kept
    block's (a near-tie can swap which of the two is kept).
    """
    if not (0.0 <= thr < 1.0):
        raise ValueError("thr must lie in [0, 1)")
    lead = A.shape[:-1]
    nb = A.shape[-1]
    rows = A.reshape(-1, nb)
    keep = np.zeros(rows.shape, dtype=bool)
    amb = np.zeros(rows.shape, dtype=bool)
    target = 1.0 - thr
    for r in range(rows.shape[0]):
        a = rows[r]
        if thr == 0.0:
            keep[r, :] = True
            continue
        order = np.argsort(-a, kind="stable")          # descending, ties -> lower J first
        c = np.cumsum(a[order])                         # c[k-1] = mass of the first k blocks
        reach = np.nonzero(c >= target)[0]
        kstar = int(reach[0]) + 1 if reach.size else nb
        keep[r, order[:kstar]] = True
        before = np.concatenate([[0.0], c[:-1]])        # mass ranked ahead of each block
        amb[r, order[np.abs(before - target) <= AMBIGUITY_MASS]] = True
        vb = a[order[kstar - 1]]
        near = np.abs(a - vb) <= AMBIGUITY_TIE_REL * vb
        if near.sum() > 1:
            amb[r, near] = True
    return keep.reshape(A.shape), amb.reshape(A.shape)


# ------------------------------------------------------------ STA union

def block_tiles(T: int, H: int, W: int, P: int, block: int) -> np.ndarray:
    """(t, h // P, w // P) of the first token of every block in the fractal order: [nb, 3]."""
    N = T * H * W
    order = fractal_order(T, H, W, P)
    nb = num_blocks(N, block)
    tiles = np.zeros((nb, 3), dtype=np.int64)
    for I in range(nb):
        n = int(order[I * block])
        t, rem = divmod(n, H * W)
        h, w = divmod(rem, W)
        tiles[I] = (t, h // P, w // P)
    return tiles


def sta_mask(T: int, H: int, W: int, P: int, block: int, half: Tuple[int, int, int]) -> np.ndarray:
    """Static sliding-tile window over blocks: [nb, nb] bool.

    NABLA summary, Metodologia 3 ("Integracion Hibrida con STA"): the final mask
    is the union of the adaptive mask and a static window mask.
    """
    tiles = block_tiles(T, H, W, P, block)
    nb = tiles.shape[0]
    m = np.zeros((nb, nb), dtype=bool)
    for I in range(nb):
        for J in range(nb):
            m[I, J] = all(abs(int(tiles[I, a]) - int(tiles[J, a])) <= half[a] for a in range(3))
    return m


# ----------------------------------------------------------- block mask

def block_mask(q_bhnd: np.ndarray, k_bhnd: np.ndarray, T: int, H: int, W: int, P: int, block: int,
               thr: float, sta: Optional[Tuple[int, int, int]] = None,
               scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Reduced map -> CDF mask (-> union with STA).  Returns ``(keep, ambiguous)`` [B, heads, nb, nb].

    Blocks that the STA window keeps are never ambiguous: the union keeps them
    whatever the CDF rule decides.
    """
    N = T * H * W
    qbar = block_means(q_bhnd, N, block)
    kbar = block_means(k_bhnd, N, block)
    A = reduced_attention(qbar, kbar, scale)
    keep, amb = cdf_keep(A, thr)
    if sta is not None:
        m = sta_mask(T, H, W, P, block, sta)
        keep = keep | m[None, None]
        amb = amb & ~m[None, None]
    return keep, amb


def mask_to_lists(keep: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Bool [.., nb, nb] -> (kv_count [.., nb] int32, kv_idx [.., nb, nb] int32 ascending, -1 tail)."""
    nb = keep.shape[-1]
    flat = keep.reshape(-1, nb)
    count = flat.sum(axis=1).astype(np.int32)
    idx = np.full(flat.shape, -1, dtype=np.int32)
    for r in range(flat.shape[0]):
        js = np.nonzero(flat[r])[0]
        idx[r, :js.size] = js
    return count.reshape(keep.shape[:-1]), idx.reshape(keep.shape)


def lists_to_mask(kv_count: np.ndarray, kv_idx: np.ndarray, nb: int) -> np.ndarray:
    """Inverse of ``mask_to_lists`` (entries past ``kv_count`` are ignored)."""
    cnt = kv_count.reshape(-1)
    idx = kv_idx.reshape(-1, kv_idx.shape[-1])
    keep = np.zeros((cnt.size, nb), dtype=bool)
    for r in range(cnt.size):
        keep[r, idx[r, :cnt[r]]] = True
    return keep.reshape(kv_count.shape + (nb,))


# ------------------------------------------------- block-sparse attention

def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, keep: np.ndarray, N: int, block: int,
                     scale: Optional[float] = None,
                     blocks: Optional[Iterable[Tuple[int, int, int]]] = None
                     ) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention restricted to the kept N x N tiles.

    NABLA summary, Metodologia 2, "Expansion": the block mask, expanded to
    tokens, says which attention tiles are computed; a query in block I attends
    to every valid key of every kept block J, with a softmax over exactly those
    keys.

    ``q, k, v``: [B, heads, Npad, d] (fractal order).  ``keep``: [B, heads, nb, nb].
    ``blocks``: optional iterable of (b, head, I) to compute; others stay 0.
    Returns ``(O [B, heads, Npad, d], lse [B, heads, Npad])`` (natural log);
    padded query rows have O = 0 and lse = 0.
    """
    B, heads, Npad, d = q.shape
    nb = Npad // block
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros_like(q, dtype=np.float64)
    lse = np.zeros((B, heads, Npad), dtype=np.float64)
    if blocks is None:
        blocks = [(b, h, I) for b in range(B) for h in range(heads) for I in range(nb)]
    for (b, h, I) in blocks:
        qlo, qhi = I * block, min((I + 1) * block, N)
        if qhi <= qlo:
            continue
        cols = []
        for J in np.nonzero(keep[b, h, I])[0]:
            klo, khi = int(J) * block, min((int(J) + 1) * block, N)
            cols.extend(range(klo, khi))
        cols = np.asarray(cols, dtype=np.int64)
        if cols.size == 0:
            continue
        s = (q[b, h, qlo:qhi, :] @ k[b, h, cols, :].T) * scale
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        O[b, h, qlo:qhi, :] = (e @ v[b, h, cols, :]) / z
        lse[b, h, qlo:qhi] = (m + np.log(z))[:, 0]
    return O, lse


# --------------------------------------- Hilbert-curve order, sub-block scoring

def hilbert_index(coords: Sequence[int], bits: int) -> int:
    """Index of a point along the n-dimensional Hilbert curve of side 2^bits.

    DFSAttn explainer, section 1 ("El barajado de la Curva de Hilbert"): tokens
    are ordered along a 3-D Hilbert curve so that neighbours in the sequence
    are neighbours in space and time.  The page does not say which Hilbert
    curve; this is J. Skilling's construction ("Programming the Hilbert
    curve", AIP Conf. Proc. 707, 2004), written from its description: the
    coordinates are turned into the curve's "transposed" index by undoing the
    excess work of the reflected Gray code level by level (from the top bit
    down, an axis with the current bit set flips the lower bits of axis 0,
    otherwise axes 0 and i exchange their lower bits), Gray-encoding across
    the axes, and a final fix-up; the index interleaves the transposed words
    from the top bit down, axis 0 first.
    """
    x = [int(c) for c in coords]
    n = len(x)
    top = 1 << (bits - 1)
    q = top
    while q > 1:
        low = q - 1
        for i in range(n):
            if x[i] & q:
                x[0] ^= low
            else:
                t = (x[0] ^ x[i]) & low
                x[0] ^= t
                x[i] ^= t
        q >>= 1
    for i in range(1, n):
        x[i] ^= x[i - 1]
    t = 0
    q = top
    while q > 1:
        if x[n - 1] & q:
            t ^= q - 1
        q >>= 1
    for i in range(n):
        x[i] ^= t
    h = 0
    for b in range(bits - 1, -1, -1):
        for i in range(n):
            h = (h << 1) | ((x[i] >> b) & 1)
    return h


def hilbert_bits(T: int, H: int, W: int) -> int:
    """Bits per axis of the smallest power-of-two cube that holds the grid."""
    return max(1, int(math.ceil(math.log2(max(T, H, W)))))


def hilbert_order(T: int, H: int, W: int) -> np.ndarray:
    """Position p -> original token n = t*H*W + h*W + w along the 3-D Hilbert
    curve of the smallest power-of-two cube holding the T x H x W grid, axes
    (t, h, w) in that order, points outside the grid skipped (the plainest
    reading for grids that are not a power-of-two cube)."""
    bits = hilbert_bits(T, H, W)
    keys = []
    for t in range(T):
        for h in range(H):
            for w in range(W):
                keys.append(hilbert_index((t, h, w), bits))
    return np.argsort(np.asarray(keys, dtype=np.int64), kind="stable").astype(np.int64)


def reorder_by(x_bnhd: np.ndarray, order: np.ndarray, block: int) -> np.ndarray:
    """[B, N, heads, d] -> [B, heads, Npad, d] with position p holding token
    order[p], zero tail (the layout change of ``reorder`` for any order)."""
    B, N, heads, d = x_bnhd.shape
    y = np.zeros((B, heads, padded_len(N, block), d), dtype=np.float64)
    for p in range(N):
        y[:, :, p, :] = x_bnhd[:, order[p], :, :]
    return y


def subblock_scores(q_bhnd: np.ndarray, k_bhnd: np.ndarray, N: int, block: int, sub: int,
                    scale: Optional[float] = None) -> np.ndarray:
    """Hierarchical block importance from sub-block scores: [.., nb, nb], rows sum to 1.

    DFSAttn explainer, section 2 ("La puntuacion de Sub-bloque"): instead of
    judging a block by its average, blocks are split into smaller sub-blocks
    and their finer scores are added up.  Reading: Q and K are mean-pooled over
    sub-blocks of `sub` tokens (valid tokens only; `sub` divides the block
    size), the reduced attention is taken at sub-block resolution (a row
    softmax over all key sub-blocks), and block I's importance for block J is
    the mass its query sub-blocks give to J's key sub-blocks, summed over J's
    sub-blocks and averaged over I's valid query sub-blocks.  With sub ==
    block this is NABLA's reduced map.
    """
    assert block % sub == 0
    qs = block_means(q_bhnd, N, sub)           # [.., ns, d]
    ks = block_means(k_bhnd, N, sub)
    ns_valid = -(-N // sub)                    # sub-blocks holding at least one valid token
    qs, ks = qs[..., :ns_valid, :], ks[..., :ns_valid, :]
    A = reduced_attention(qs, ks, scale)       # [.., ns_valid, ns_valid]
    per = block // sub
    nb = padded_len(N, block) // block
    out = np.zeros(A.shape[:-2] + (nb, nb), dtype=np.float64)
    for I in range(nb):
        a_rows = [a for a in range(I * per, (I + 1) * per) if a < ns_valid]
        for J in range(nb):
            b_cols = [b for b in range(J * per, (J + 1) * per) if b < ns_valid]
            if b_cols:
                out[..., I, J] = A[..., a_rows, :][..., :, b_cols].sum(axis=(-1, -2)) / len(a_rows)
    return out


def block_mask_subblock(q_bhnd: np.ndarray, k_bhnd: np.ndarray, N: int, block: int, sub: int, thr: float,
                        scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Sub-block importance -> the same CDF rule as NABLA.  Returns (keep, ambiguous)."""
    return cdf_keep(subblock_scores(q_bhnd, k_bhnd, N, block, sub, scale), thr)


# ------------------------------------------------------ token-radius masks

def attention_entropy(q: np.ndarray, k: np.ndarray, N: int, scale: Optional[float] = None) -> np.ndarray:
    """Entropy (nats) of each query row of the dense attention: [B, heads, Npad] (0 for padded rows).

    TRA summary, section 2 ("Entropia-a-Presupuesto"): in a dense warm-up pass
    the entropy of each query's attention distribution is computed,
    H_i = -sum_j p_ij ln p_ij with p_i = softmax_j(scale q_i . k_j) over the
    valid keys.
    """
    B, heads, Npad, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    H = np.zeros((B, heads, Npad), dtype=np.float64)
    for b in range(B):
        for h in range(heads):
            s = (q[b, h, :N] @ k[b, h, :N].T) * scale
            s = s - s.max(axis=1, keepdims=True)
            e = np.exp(s)
            p = e / e.sum(axis=1, keepdims=True)
            H[b, h, :N] = -(p * np.log(p, where=p > 0, out=np.zeros_like(p))).sum(axis=1)
    return H


def token_radius(H: np.ndarray, t_of: np.ndarray, T: int, tau: float, gamma: float, N: int) -> np.ndarray:
    """Base radius of each query token from its entropy: [.., Npad] (0 for padded rows).

    TRA summary, section 2 ("Entropia-a-Presupuesto", "Presupuesto-a-Radio"):
    the token budget is tau * exp(H_i) keys (clamped to [1, N]); the support
    of the query in frame t is a 2-D disk of radius r_i * phi(|t - t_i|), with
    phi(delta) = exp(-gamma * delta), and r_i makes the disks' total area the
    budget: sum_t pi (r_i phi(|t - t_i|))^2 = budget.  `t_of`: the frame of the
    token at each position.
    """
    out = np.zeros(H.shape, dtype=np.float64)
    for p in range(N):
        ti = int(t_of[p])
        area = sum(math.pi * math.exp(-2.0 * gamma * abs(t - ti)) for t in range(T))
        budget = np.clip(tau * np.exp(H[..., p]), 1.0, float(N))
        out[..., p] = np.sqrt(budget / area)
    return out


def radius_block_mask(r: np.ndarray, T: int, H: int, W: int, P: int, block: int, gamma: float,
                      vote: int = 1) -> np.ndarray:
    """Block mask from token-radius supports: [B, heads, nb, nb] bool.

    TRA summary, section 2 ("Ejecucion Eficiente"): tokens in the tile-major
    (here: the fractal P x P) order; key token j is in query token i's support
    when (h_j - h_i)^2 + (w_j - w_i)^2 <= (r_i phi(|t_j - t_i|))^2; a query
    token votes for a key block when the block holds a key of its support, and
    block I keeps block J when at least `vote` of I's valid query tokens vote
    for J (the token-level masks made into regular block masks).
    `r`: [B, heads, Npad] base radii by position.
    """
    N = T * H * W
    order = fractal_order(T, H, W, P)
    nb = num_blocks(N, block)
    t = order // (H * W)
    hh = (order % (H * W)) // W
    ww = order % W
    lead = r.shape[:-1]
    keep = np.zeros(lead + (nb, nb), dtype=bool)
    for idx in np.ndindex(*lead):
        for I in range(nb):
            qs = range(I * block, min((I + 1) * block, N))
            votes = np.zeros(nb, dtype=np.int64)
            for i in qs:
                rad = r[idx + (i,)] * np.exp(-gamma * np.abs(t - t[i]))
                inside = (hh - hh[i]) ** 2 + (ww - ww[i]) ** 2 <= rad ** 2
                hit = np.zeros(nb, dtype=bool)
                hit[np.nonzero(inside)[0] // block] = True
                votes += hit
            keep[idx + (I,)] = votes >= vote
    return keep


def radius_mask_from_qk(q: np.ndarray, k: np.ndarray, T: int, H: int, W: int, P: int, block: int, tau: float,
                        gamma: float, vote: int = 1, scale: Optional[float] = None) -> np.ndarray:
    """The whole chain on reordered Q, K: entropy -> budget -> radius -> block mask."""
    N = T * H * W
    Hn = attention_entropy(q, k, N, scale)
    t_of = fractal_order(T, H, W, P) // (H * W)
    r = token_radius(Hn, t_of, T, tau, gamma, N)
    return radius_block_mask(r, T, H, W, P, block, gamma, vote)


# --------------------------------------------- fine-grained KV selection

def fine_attention_block(qr: np.ndarray, kh: np.ndarray, vh: np.ndarray, idx: np.ndarray,
                         w: Optional[np.ndarray], N: int, kblock: int = 4,
                         scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """One query block of fine_attention: rows ``qr`` [n, d] of one head over
    the keys of the 4-token blocks ``idx`` (weights ``w`` or None) of that
    head's ``kh``, ``vh`` [Npad, d].  Returns (O [n, d], lse [n]); both zero
    when the list holds no valid key."""
    n, d = qr.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    cols, shift = [], []
    for e, blk in enumerate(np.asarray(idx, dtype=np.int64)):
        lw = 0.0 if w is None else math.log(float(w[e]))
        for key in range(int(blk) * kblock, min((int(blk) + 1) * kblock, N)):
            cols.append(key)
            shift.append(lw)
    if not cols:
        return np.zeros((n, d)), np.zeros(n)
    cols = np.asarray(cols, dtype=np.int64)
    s = (qr @ kh[cols, :].T) * scale + np.asarray(shift)[None, :]
    m = s.max(axis=1, keepdims=True)
    e_ = np.exp(s - m)
    z = e_.sum(axis=1, keepdims=True)
    return (e_ @ vh[cols, :]) / z, (m + np.log(z))[:, 0]


def fine_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, sel_offsets: np.ndarray, sel_idx: np.ndarray,
                   sel_w: Optional[np.ndarray], N: int, qblock: int = 128, kblock: int = 4,
                   scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Attention over per-query-block lists of small KV blocks, with optional
    inclusion weights.

    AB-Attention article, "Los tres recursos de AB-Attention": KV blocks of
    only 4 tokens, chosen per query block (of 128 tokens) and gathered by
    index (the fine selection on coarse hardware); and SIP: each chosen block
    counts with the inverse of its inclusion probability w (Horvitz-Thompson),
    as a logit shift ln w in both the numerator and the normalisation of the
    softmax:
        O_q = sum_k w_b(k) e^(s_qk) v_k / sum_k w_b(k) e^(s_qk),  s = scale q.k
    over the valid keys k of the chosen blocks.  Lists are CSR: query block r
    of head (b, h) (r = (b * heads + h) * nq + I) uses entries
    sel_offsets[r] .. sel_offsets[r + 1] of sel_idx (block indices, 4-token
    units) and sel_w (None: all 1).  Returns (O, lse) like masked_attention
    (lse includes the shifts; rows >= N and rows with no valid key are 0).
    """
    B, heads, Npad, d = q.shape
    nq = Npad // qblock
    O = np.zeros_like(q, dtype=np.float64)
    lse = np.zeros((B, heads, Npad), dtype=np.float64)
    for b in range(B):
        for h in range(heads):
            for I in range(nq):
                r = (b * heads + h) * nq + I
                qlo, qhi = I * qblock, min((I + 1) * qblock, N)
                if qhi <= qlo:
                    continue
                lo, hi = int(sel_offsets[r]), int(sel_offsets[r + 1])
                O[b, h, qlo:qhi], lse[b, h, qlo:qhi] = fine_attention_block(
                    q[b, h, qlo:qhi], k[b, h], v[b, h], sel_idx[lo:hi], None if sel_w is None else sel_w[lo:hi],
                    N, kblock, scale)
    return O, lse


# ------------------------------------------ block-sparse attention backward

def masked_attention_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, keep: np.ndarray, dO: np.ndarray,
                              N: int, block: int, scale: Optional[float] = None
                              ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients of ``masked_attention`` with respect to q, k and v, given the
    gradient dO of its output.

    NABLA summary, "Contribuciones Clave" ("Aceleracion de Doble Fase"): the
    block-sparse attention also runs in pre-training and fine-tuning, so its
    backward pass follows the same block mask.  Per query block I, with the
    valid keys of its kept blocks as columns:

        P  = softmax(scale * Q_I K^T)           (as in the forward pass)
        dV += P^T dO_I
        dP = dO_I V^T
        dS = P * (dP - rowsum(dO_I * O_I))     (O_I = P V: the softmax Jacobian)
        dQ_I = scale * dS K,    dK += scale * dS^T Q_I

    Padded query rows take part in nothing (their dO is ignored, their dQ is
    0); padded keys are never columns.  Returns (dq, dk, dv) [B, heads, Npad, d].
    """
    B, heads, Npad, d = q.shape
    nb = Npad // block
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros_like(k, dtype=np.float64)
    dv = np.zeros_like(v, dtype=np.float64)
    for b in range(B):
        for h in range(heads):
            for I in range(nb):
                qlo, qhi = I * block, min((I + 1) * block, N)
                if qhi <= qlo:
                    continue
                cols = []
                for J in np.nonzero(keep[b, h, I])[0]:
                    klo, khi = int(J) * block, min((int(J) + 1) * block, N)
                    cols.extend(range(klo, khi))
                cols = np.asarray(cols, dtype=np.int64)
                if cols.size == 0:
                    continue
                qI, kc, vc, dOI = q[b, h, qlo:qhi], k[b, h, cols], v[b, h, cols], dO[b, h, qlo:qhi]
                s = (qI @ kc.T) * scale
                e = np.exp(s - s.max(axis=1, keepdims=True))
                P = e / e.sum(axis=1, keepdims=True)
                OI = P @ vc
                dv[b, h, cols] += P.T @ dOI
                dP = dOI @ vc.T
                dS = P * (dP - (dOI * OI).sum(axis=1, keepdims=True))
                dq[b, h, qlo:qhi] += scale * (dS @ kc)
                dk[b, h, cols] += scale * (dS.T @ qI)
    return dq, dk, dv


# ------------------------------------------------------------ full path

def nabla_attention(q_bnhd: np.ndarray, k_bnhd: np.ndarray, v_bnhd: np.ndarray,
                    T: int, H: int, W: int, P: int, block: int, thr: float,
                    sta: Optional[Tuple[int, int, int]] = None,
                    scale: Optional[float] = None):
    """The whole path on model-order inputs: reorder, mask, attention, inverse reorder.

    Returns ``(O [B, N, heads, d], keep, ambiguous)``.
    """
    N = T * H * W
    q = reorder(q_bnhd, T, H, W, P, block)
    k = reorder(k_bnhd, T, H, W, P, block)
    v = reorder(v_bnhd, T, H, W, P, block)
    keep, amb = block_mask(q, k, T, H, W, P, block, thr, sta, scale)
    O, _ = masked_attention(q, k, v, keep, N, block, scale)
    return inverse_reorder(O, T, H, W, P), keep, amb


def density(keep: np.ndarray) -> float:
    return float(keep.sum()) / float(keep.size)


def attention_flops(N: int, d: int, heads: int, B: int, dens: float) -> float:
    """Effective FLOPs of one block-sparse call: 4 * N^2 * d * heads * B * density."""
    return 4.0 * N * N * d * heads * B * dens
