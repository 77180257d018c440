"""Seeded synthetic inputs shaped like the video-DiT workloads of the NABLA method.

This module only *draws* inputs; it contains none of the method's arithmetic
(no reorder, pooling, softmax, thresholding or attention).  Both the fp64
oracle (``oracle/``) and the CUDA path consume what it returns, so the two
sides always see identical bytes.

Recipe (the pages give no input distribution; this is the stand-in for the
Wan 2.1 / HunyuanVideo latents the NABLA, AB-Attention and TRA summaries
measure on):

* Q, K, V have the model layout ``[B, N, heads, d]`` with ``N = T*H*W`` and
  token ``n = t*H*W + h*W + w`` (row-major video latent).
* ``X = noise + alpha * field`` where ``noise ~ N(0, 1)`` i.i.d. per tensor and
  ``field[n, head] = G_head @ phi(t, h, w)``:
  ``phi`` stacks ``sin`` and ``cos`` of ``omega_f . (t, h, w)`` for 16
  frequency vectors ``omega_f`` with components ~ U(-0.5, 0.5) rad per latent
  step, and ``G_head`` is a ``d x 32`` matrix with entries ~ N(0, 1/32).
  Q, K and V share the field (so nearby tokens attend to each other) and have
  independent noise.  The result is rounded to bf16 (round-to-nearest-even).
* Density-sweep masks: for every (b, head, query block I) keep
  ``k = max(1, round(rho * nb))`` blocks: the diagonal block I plus ``k - 1``
  others drawn uniformly without replacement.

* Fine selections (AB-Attention): for every (b, head, query block of 128)
  a list of ``k`` distinct 4-token KV blocks drawn uniformly without
  replacement (``k = round(frac * nkb)``, or, for ragged lists, ``k`` drawn
  uniformly from ``[0, 2 * round(frac * nkb)]``), in ascending order; the
  weights are 1 for half of the entries (blocks always taken) and ``1 / pi``
  with ``pi ~ U(0.05, 1)`` for the others.

Random numbers come from ``torch.Generator`` (CPU, Mersenne twister) in fixed
chunks of ``_CHUNK`` elements, each chunk seeded from (seed, stream, chunk
index); chunks are drawn on a thread pool, so the values do not depend on the
number of threads.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field as dc_field
from typing import Optional, Tuple

import torch

_CHUNK = 1 << 24


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: the video latent grid, attention shape and the
    NABLA hyper-parameters used on it."""
    name: str
    B: int
    T: int
    H: int
    W: int
    heads: int
    d: int
    block: int
    patch: int
    thr: float
    sta: Optional[Tuple[int, int, int]]  # STA half-widths (t, h, w) in block-tile units, or None
    alpha: float                         # positional-field scale
    seed: int
    iid: bool = False                    # Q, K, V i.i.d. N(0,1) (density sweep)
    densities: Tuple[float, ...] = dc_field(default_factory=tuple)

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def Npad(self) -> int:
        return -(-self.N // self.block) * self.block

    @property
    def nb(self) -> int:
        return self.Npad // self.block


# The five workloads: a tiny case the oracle finishes in seconds, the Wan-480p
# and Hunyuan-720p latent shapes, the NABLA u STA hybrid and a density sweep.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 16, 16, 2, 64, 64, 8, 0.1, None, 1.5, 1),
    "wan480p": Workload("wan480p", 1, 21, 30, 52, 12, 128, 64, 8, 0.2, None, 1.5, 2),
    "hunyuan720p": Workload("hunyuan720p", 1, 33, 45, 80, 24, 128, 128, 8, 0.1, None, 2.0, 3),
    "hybrid_wan480p": Workload("hybrid_wan480p", 1, 21, 30, 52, 12, 128, 64, 8, 0.2, (1, 1, 1), 1.5, 2),
    "density_sweep": Workload("density_sweep", 1, 21, 30, 52, 24, 128, 64, 8, 0.0, None, 0.0, 5,
                              iid=True, densities=(0.05, 0.10, 0.20, 0.35, 0.50, 1.00)),
}


def _mix(*parts: int) -> int:
    """SplitMix64-style mixing of integers into one 63-bit seed."""
    x = 0x9E3779B97F4A7C15
    for p in parts:
        x = (x ^ (p & 0xFFFFFFFFFFFFFFFF)) & 0xFFFFFFFFFFFFFFFF
        x = (x + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
        x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
        x ^= x >> 31
    return x & 0x7FFFFFFFFFFFFFFF


def _randn_chunked(numel: int, seed: int, stream: int, dtype=torch.float32) -> torch.Tensor:
    out = torch.empty(numel, dtype=dtype)
    nchunks = -(-numel // _CHUNK)

    def fill(i: int) -> None:
        g = torch.Generator().manual_seed(_mix(seed, stream, i))
        lo, hi = i * _CHUNK, min(numel, (i + 1) * _CHUNK)
        out[lo:hi] = torch.randn(hi - lo, generator=g, dtype=dtype)

    workers = max(1, min(nchunks, os.cpu_count() or 1))
    if workers == 1:
        for i in range(nchunks):
            fill(i)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def positional_field(T: int, H: int, W: int, heads: int, d: int, seed: int) -> torch.Tensor:
    """``G_head @ phi(t, h, w)`` for every token and head: float32 [N, heads, d]."""
    g = torch.Generator().manual_seed(_mix(seed, 0xF1E1D))
    omega = torch.rand(16, 3, generator=g, dtype=torch.float64) - 0.5
    G = torch.randn(heads, d, 32, generator=g, dtype=torch.float64) / math.sqrt(32.0)
    t = torch.arange(T, dtype=torch.float64).view(T, 1, 1).expand(T, H, W)
    h = torch.arange(H, dtype=torch.float64).view(1, H, 1).expand(T, H, W)
    w = torch.arange(W, dtype=torch.float64).view(1, 1, W).expand(T, H, W)
    pos = torch.stack([t, h, w], dim=-1).reshape(-1, 3)          # [N, 3], n = t*H*W + h*W + w
    ang = pos @ omega.T                                           # [N, 16]
    phi = torch.cat([torch.sin(ang), torch.cos(ang)], dim=1)      # [N, 32]
    out = torch.empty(pos.shape[0], heads, d, dtype=torch.float32)
    for hd in range(heads):
        out[:, hd, :] = (phi @ G[hd].T).to(torch.float32)
    return out


def make_qkv(w: Workload) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q, K, V as bf16 CPU tensors [B, N, heads, d] for workload ``w``."""
    shape = (w.B, w.N, w.heads, w.d)
    numel = w.B * w.N * w.heads * w.d
    fld = None
    if not w.iid and w.alpha != 0.0:
        fld = positional_field(w.T, w.H, w.W, w.heads, w.d, w.seed).unsqueeze(0)
        fld.mul_(w.alpha)
    outs = []
    for stream in range(3):
        x = _randn_chunked(numel, w.seed, 1 + stream).view(shape)
        if fld is not None:
            x.add_(fld)
        outs.append(x.to(torch.bfloat16))
        del x
    return outs[0], outs[1], outs[2]


def random_block_lists(B: int, heads: int, nb: int, density: float, seed: int):
    """Seeded random block masks as ascending KV index lists.

    Returns ``(kv_count [B, heads, nb] int32, kv_idx [B, heads, nb, nb] int32)``;
    row (b, h, I) keeps the diagonal block I plus ``k - 1`` blocks drawn
    uniformly without replacement, ``k = max(1, round(density * nb))``; unused
    tail entries of ``kv_idx`` are -1.
    """
    k = max(1, min(nb, int(round(density * nb))))
    g = torch.Generator().manual_seed(_mix(seed, 0x5EED, int(round(density * 1e6))))
    keys = torch.rand(B, heads, nb, nb, generator=g)
    diag = torch.arange(nb)
    keys[:, :, diag, diag] = -1.0                                   # diagonal always drawn first
    chosen = torch.argsort(keys, dim=-1)[..., :k]
    chosen, _ = torch.sort(chosen, dim=-1)
    kv_idx = torch.full((B, heads, nb, nb), -1, dtype=torch.int32)
    kv_idx[..., :k] = chosen.to(torch.int32)
    kv_count = torch.full((B, heads, nb), k, dtype=torch.int32)
    return kv_count, kv_idx


def random_fine_lists(B: int, heads: int, nq: int, nkb: int, frac: float, seed: int, ragged: bool = False):
    """Seeded fine selections as CSR lists.

    Returns ``(sel_offsets [B*heads*nq + 1] int64, sel_idx [n_sel] int32,
    sel_w [n_sel] float32)``: row r = (b*heads + h)*nq + I holds entries
    ``sel_offsets[r] .. sel_offsets[r+1]`` (see the module docstring for the
    draw).
    """
    rows = B * heads * nq
    k0 = max(1, min(nkb, int(round(frac * nkb))))
    g = torch.Generator().manual_seed(_mix(seed, 0xF1E5, int(round(frac * 1e6)), int(ragged)))
    if ragged:
        counts = torch.randint(0, min(nkb, 2 * k0) + 1, (rows,), generator=g)
    else:
        counts = torch.full((rows,), k0, dtype=torch.int64)
    offsets = torch.zeros(rows + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(counts, 0)
    idx = torch.empty(int(offsets[-1]), dtype=torch.int32)
    step = max(1, (1 << 24) // max(1, nkb))          # rows per batch of draws
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        order = torch.argsort(torch.rand(r1 - r0, nkb, generator=g), dim=1)
        for r in range(r0, r1):
            c = int(counts[r])
            if c:
                idx[int(offsets[r]):int(offsets[r]) + c] = torch.sort(order[r - r0, :c]).values.to(torch.int32)
    always = torch.rand(idx.numel(), generator=g) < 0.5
    pi = 0.05 + 0.95 * torch.rand(idx.numel(), generator=g)
    w = torch.where(always, torch.ones_like(pi), 1.0 / pi).to(torch.float32)
    return offsets, idx, w
