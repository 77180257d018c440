"""Runs the fp64 oracle over work items on a pool of host processes.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline and reference legs of
``bench.py`` use it; the product path never imports it.

It does no arithmetic of its own.  Every task calls one function of
``oracle.nabla`` (``reorder``, ``block_mask``, ``masked_attention``,
``inverse_reorder``) on one attention head, or on a list of query blocks of
one head, and the parent gathers what the tasks return.  The work items are
(b, head) for the reorder and the mask, and (b, head, list of query blocks)
for the attention, so every host core the process may run on takes part.

Data travels through memory-mapped files in a private temporary directory:
the model-order inputs as their bf16 bit patterns, the reordered tensors as
float32 (which holds every bf16 value exactly); a task converts its slice to
float64 before the oracle touches it.  Workers are started with the "spawn"
method, so a pool may be created after CUDA has been initialised in the
parent, and each worker limits BLAS to one thread: the parallelism is the
pool's.
"""
from __future__ import annotations

import os
import shutil
import tempfile
import time
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _bf16_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> their exact values (the top half of a float32)."""
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ worker side

_S: Dict = {}


def _open(meta, name, mode="r+"):
    dtype, shape = meta["files"][name]
    return np.memmap(os.path.join(meta["dir"], name), dtype=dtype, mode=mode, shape=tuple(shape))


def _init_worker(meta):
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    import oracle  # noqa: F401  (imported once here, not inside the first timed task)
    _S.clear()
    _S["meta"] = meta
    _S["mm"] = {}


def _mm(name):
    mm = _S["mm"]
    if name not in mm:
        mm[name] = _open(_S["meta"], name)
    return mm[name]


def _dims():
    m = _S["meta"]
    return m["T"], m["H"], m["W"], m["P"], m["block"], m["N"], m["Npad"], m["nb"]


def _head(t, b, h):
    """Reordered tensor t (0 = Q, 1 = K, 2 = V) of one head as float64 [1, 1, Npad, d]."""
    return np.asarray(_mm("xre")[t, b, h], dtype=np.float64)[None, None]


def _task(args):
    import oracle
    kind = args[0]
    T, H, W, P, block, N, Npad, nb = _dims()
    t0 = time.perf_counter()
    if kind == "reorder":                      # ("reorder", tensor, b, h)
        _, t, b, h = args
        x = _bf16_bits_to_f64(np.asarray(_mm("xin")[t, b, :, h, :]))[None, :, None, :]
        y = oracle.reorder(x, T, H, W, P, block)
        _mm("xre")[t, b, h] = y[0, 0].astype(np.float32)
        return time.perf_counter() - t0
    if kind == "mask":                         # ("mask", b, h)
        _, b, h = args
        m = _S["meta"]
        keep, amb = oracle.block_mask(_head(0, b, h), _head(1, b, h), T, H, W, P, block, m["thr"],
                                      m["sta"])
        _mm("keep")[b, h] = keep[0, 0]
        return amb[0, 0].copy(), time.perf_counter() - t0
    if kind in ("attn", "check"):              # (kind, b, h, blocks[, slot])
        b, h, blocks = args[1], args[2], list(args[3])
        keep = np.asarray(_mm("keep")[b, h], dtype=bool)[None, None]
        O, lse = oracle.masked_attention(_head(0, b, h), _head(1, b, h), _head(2, b, h), keep, N, block,
                                         blocks=[(0, 0, I) for I in blocks])
        if kind == "attn":
            slot = args[4]
            o64 = _mm("o64")
            for I in blocks:
                o64[slot, I * block:(I + 1) * block] = O[0, 0, I * block:(I + 1) * block]
            return time.perf_counter() - t0
        # compare with the GPU output of the same head, element by element
        ogpu, lgpu = _mm("ogpu"), _mm("lsegpu")
        mx, sm, n, lmx, pad_nonzero = 0.0, 0.0, 0, 0.0, 0
        for I in blocks:
            lo, hi = I * block, min((I + 1) * block, N)
            got = _bf16_bits_to_f64(np.asarray(ogpu[b, h, lo:hi]))
            err = np.abs(got - O[0, 0, lo:hi])
            mx = max(mx, float(err.max()))
            sm += float(err.sum())
            n += err.size
            lmx = max(lmx, float(np.abs(np.asarray(lgpu[b, h, lo:hi], dtype=np.float64) - lse[0, 0, lo:hi]).max()))
            if hi < (I + 1) * block:           # padded rows of the last block must be 0
                pad_nonzero += int(np.count_nonzero(np.asarray(ogpu[b, h, hi:(I + 1) * block])))
        return mx, sm, n, lmx, pad_nonzero
    if kind == "bwd_check":                    # ("bwd_check", b, h)
        b, h = args[1], args[2]
        keep = np.asarray(_mm("keep")[b, h], dtype=bool)[None, None]
        dO = _bf16_bits_to_f64(np.asarray(_mm("dogpu")[b, h]))[None, None]
        grads = oracle.masked_attention_backward(_head(0, b, h), _head(1, b, h), _head(2, b, h), keep, dO, N, block)
        out = []
        for i, name in enumerate(("dqgpu", "dkgpu", "dvgpu")):
            got = _bf16_bits_to_f64(np.asarray(_mm(name)[b, h]))
            want = grads[i][0, 0]
            err = np.abs(got[:N] - want[:N])
            out.append((float(err.max()), float(err.sum()), err.size, float(np.abs(want[:N]).max()),
                        float(np.abs(want[:N]).sum()), int(np.count_nonzero(got[N:]))))
        return out
    if kind == "inverse":                      # ("inverse", slot)
        slot = args[1]
        x = oracle.inverse_reorder(np.asarray(_mm("o64")[slot])[None, None], T, H, W, P)
        return float(x[0, 0, 0, 0]), time.perf_counter() - t0
    raise ValueError(kind)


# ------------------------------------------------------------------ parent side

class OraclePool:
    """The oracle on one workload, spread over host processes.

    ``q, k, v``: bf16 CPU tensors [B, N, heads, d] in model order (the same
    bytes the CUDA path receives).  ``slots``: heads whose float64 attention
    output can be held at once (for ``attention`` and ``inverse``).
    """

    def __init__(self, w, q, k, v, workers: Optional[int] = None, slots: int = 1):
        import torch
        import multiprocessing as mp
        self.w = w
        self.B, self.heads, self.d = w.B, w.heads, w.d
        self.N, self.Npad, self.nb, self.block = w.N, w.Npad, w.nb, w.block
        self.dir = tempfile.mkdtemp(prefix="oracle_pool_")
        files = {
            "xin": ("uint16", (3, w.B, w.N, w.heads, w.d)),
            "xre": ("float32", (3, w.B, w.heads, w.Npad, w.d)),
            "keep": ("uint8", (w.B, w.heads, w.nb, w.nb)),
            "o64": ("float64", (max(1, slots), w.Npad, w.d)),
            "ogpu": ("uint16", (w.B, w.heads, w.Npad, w.d)),
            "lsegpu": ("float32", (w.B, w.heads, w.Npad)),
            "dogpu": ("uint16", (w.B, w.heads, w.Npad, w.d)),
            "dqgpu": ("uint16", (w.B, w.heads, w.Npad, w.d)),
            "dkgpu": ("uint16", (w.B, w.heads, w.Npad, w.d)),
            "dvgpu": ("uint16", (w.B, w.heads, w.Npad, w.d)),
        }
        self.meta = {"dir": self.dir, "files": files, "T": w.T, "H": w.H, "W": w.W, "P": w.patch,
                     "block": w.block, "N": w.N, "Npad": w.Npad, "nb": w.nb, "thr": w.thr,
                     "sta": tuple(w.sta) if w.sta else None}
        for name, (dt, shape) in files.items():
            np.memmap(os.path.join(self.dir, name), dtype=dt, mode="w+", shape=shape).flush()
        xin = _open(self.meta, "xin")
        for i, x in enumerate((q, k, v)):
            xin[i] = x.contiguous().view(torch.int16).numpy().view(np.uint16)
        xin.flush()
        del xin
        self.workers = max(1, min(workers or host_cores(), 64))
        saved = {k_: os.environ.get(k_) for k_ in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k_ in saved:
            os.environ[k_] = "1"
        try:
            self.pool = mp.get_context("spawn").Pool(self.workers, initializer=_init_worker, initargs=(self.meta,))
        finally:
            for k_, v_ in saved.items():
                if v_ is None:
                    os.environ.pop(k_, None)
                else:
                    os.environ[k_] = v_

    # -- plumbing
    def close(self) -> None:
        if getattr(self, "pool", None) is not None:
            self.pool.terminate()
            self.pool.join()
            self.pool = None
        shutil.rmtree(self.dir, ignore_errors=True)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def _map(self, tasks: List[tuple]):
        t0 = time.perf_counter()
        out = self.pool.map(_task, tasks, chunksize=1) if tasks else []
        return out, time.perf_counter() - t0

    def pairs(self) -> List[Tuple[int, int]]:
        return [(b, h) for b in range(self.B) for h in range(self.heads)]

    # -- stages; each returns its wall time in seconds
    def reorder(self, pairs: Iterable[Tuple[int, int]], tensors: Sequence[int] = (0, 1, 2)) -> float:
        _, t = self._map([("reorder", tt, b, h) for (b, h) in pairs for tt in tensors])
        return t

    def masks(self, pairs: Iterable[Tuple[int, int]]):
        """oracle.block_mask of each (b, h) (Q and K must be reordered).  Sets
        the mask the attention uses; returns (keep, ambiguous, wall seconds),
        both bool [B, heads, nb, nb] (rows of other heads are False)."""
        pairs = list(pairs)
        res, t = self._map([("mask", b, h) for (b, h) in pairs])
        amb = np.zeros((self.B, self.heads, self.nb, self.nb), dtype=bool)
        for (b, h), (a, _) in zip(pairs, res):
            amb[b, h] = a
        keep = np.asarray(_open(self.meta, "keep", "r"), dtype=bool).copy()
        return keep, amb, t

    def set_keep(self, keep: np.ndarray) -> None:
        """The block mask the attention uses, bool [B, heads, nb, nb]."""
        mm = _open(self.meta, "keep")
        mm[:] = keep.astype(np.uint8)
        mm.flush()

    def attention(self, b: int, h: int, blocks: Sequence[int], slot: int = 0, chunk: int = 8) -> float:
        """oracle.masked_attention of the given query blocks of head (b, h), in
        chunks of `chunk` blocks; the float64 rows land in output slot `slot`."""
        blocks = list(blocks)
        _, t = self._map([("attn", b, h, blocks[i:i + chunk], slot) for i in range(0, len(blocks), chunk)])
        return t

    def inverse(self, slot: int = 0) -> float:
        _, t = self._map([("inverse", slot)])
        return t

    def check_backward(self, dO, dq, dk, dv, pairs: Iterable[Tuple[int, int]]):
        """Element-by-element comparison of GPU gradients with the oracle's
        (oracle.masked_attention_backward, one task per (b, head), under the
        mask set by ``masks`` or ``set_keep``).  All tensors bf16 CPU
        [B, heads, Npad, d].  Returns, per gradient name, (max-abs error,
        mean-abs error, max |ref|, mean |ref|, nonzero padded elements)."""
        import torch
        for name, t in (("dogpu", dO), ("dqgpu", dq), ("dkgpu", dk), ("dvgpu", dv)):
            mm = _open(self.meta, name)
            mm[:] = t.contiguous().view(torch.int16).numpy().view(np.uint16)
            mm.flush()
        res, _ = self._map([("bwd_check", b, h) for (b, h) in pairs])
        out = {}
        for i, name in enumerate(("dq", "dk", "dv")):
            rows = [r[i] for r in res]
            n = sum(r[2] for r in rows)
            out[name] = (max(r[0] for r in rows), sum(r[1] for r in rows) / max(1, n),
                         max(r[3] for r in rows), sum(r[4] for r in rows) / max(1, n), sum(r[5] for r in rows))
        return out

    def check_attention(self, o_gpu, lse_gpu, items: Iterable[Tuple[int, int, Sequence[int]]], chunk: int = 16):
        """Element-by-element comparison of the GPU output with the oracle's.

        ``o_gpu``: bf16 CPU tensor [B, heads, Npad, d]; ``lse_gpu``: float32
        [B, heads, Npad] or None; ``items``: (b, h, query blocks).  Returns
        (max-abs error, mean-abs error, elements compared, max LSE error,
        nonzero padded output elements)."""
        import torch
        og = _open(self.meta, "ogpu")
        og[:] = o_gpu.contiguous().view(torch.int16).numpy().view(np.uint16)
        og.flush()
        lg = _open(self.meta, "lsegpu")
        lg[:] = 0.0 if lse_gpu is None else lse_gpu.numpy()
        lg.flush()
        tasks = []
        for (b, h, blocks) in items:
            blocks = list(blocks)
            tasks += [("check", b, h, blocks[i:i + chunk]) for i in range(0, len(blocks), chunk)]
        res, _ = self._map(tasks)
        mx = max((r[0] for r in res), default=0.0)
        n = sum(r[2] for r in res)
        mean = sum(r[1] for r in res) / max(1, n)
        lmx = max((r[3] for r in res), default=0.0)
        pad = sum(r[4] for r in res)
        return mx, mean, n, lmx, pad
