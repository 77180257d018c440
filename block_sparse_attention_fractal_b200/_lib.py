"""ctypes binding of libbsa.so: argument marshalling only.

Every function takes torch tensors (device memory owned by the caller), passes
their raw pointers, sizes and the current CUDA stream to the C ABI declared in
include/bsa.h, and raises ``BsaError`` on a non-OK status.  The library is
loaded on the first call (so that importing the package, e.g. for its input
generator, maps nothing); there is no fallback: if libbsa.so is missing, that
first call raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

BSA_OK = 0
STATUS_NAMES = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_UNSUPPORTED", 3: "BSA_ERR_CUDA",
                4: "BSA_ERR_DEVICE_INDEX", 5: "BSA_ERR_TIMEOUT"}


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class Shape(ctypes.Structure):
    """bsa_shape: B, T, H, W, heads, d, block, patch."""
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "T", "H", "W", "heads", "d", "block", "patch")]

    def __repr__(self) -> str:
        return "Shape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbsa.so not built ({LIB_PATH}); run python -m block_sparse_attention_fractal_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    S = ctypes.POINTER(Shape)
    st = ctypes.c_int
    sig = {
        "bsa_validate_shape": (st, [S]),
        "bsa_seq_len": (ctypes.c_int64, [S]),
        "bsa_padded_len": (ctypes.c_int64, [S]),
        "bsa_num_blocks": (ctypes.c_int64, [S]),
        "bsa_workspace_bytes": (ctypes.c_size_t, [S]),
        "bsa_workspace_init": (st, [P, ctypes.c_size_t, P]),
        "bsa_plan_items_offset": (ctypes.c_int64, [S]),
        "bsa_reorder": (st, [S, P, P, P]),
        "bsa_inverse_reorder": (st, [S, P, P, P]),
        "bsa_build_block_mask": (st, [S, P, P, ctypes.c_float, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      P, P, P, P, ctypes.c_size_t, P]),
        "bsa_reorder_qk_pooled": (st, [S, P, P, P, P, P, ctypes.c_size_t, P]),
        "bsa_build_block_mask_pooled": (st, [S, ctypes.c_float, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                             P, P, P, P, ctypes.c_size_t, P]),
        "bsa_attn_fwd": (st, [S, P, P, P, P, P, ctypes.c_float, P, P, P, ctypes.c_size_t, P]),
        "bsa_attn_fwd_baseline": (st, [S, P, P, P, P, P, ctypes.c_float, P, P, P, ctypes.c_size_t, P]),
        "bsa_attn_fwd_entropy": (st, [S, P, P, P, P, P, ctypes.c_float, P, P, P, P, ctypes.c_size_t, P]),
        "bsa_dense_lists": (st, [S, P, P, P]),
        "bsa_build_block_mask_radius": (st, [S, P, ctypes.c_float, ctypes.c_float, ctypes.c_int32, P, P, P, P]),
        "bsa_hilbert_workspace_bytes": (ctypes.c_size_t, [S]),
        "bsa_hilbert_order": (st, [S, P, P, ctypes.c_size_t, P]),
        "bsa_reorder_perm": (st, [S, P, P, P, P]),
        "bsa_inverse_reorder_perm": (st, [S, P, P, P, P]),
        "bsa_reorder_qk_pooled_perm": (st, [S, P, P, P, P, P, P, ctypes.c_size_t, P]),
        "bsa_subblock_workspace_bytes": (ctypes.c_size_t, [S, ctypes.c_int32]),
        "bsa_build_block_mask_subblock": (st, [S, P, P, ctypes.c_int32, ctypes.c_float, P, P, P, P, ctypes.c_size_t,
                                               P]),
        "bsa_attn_bwd_workspace_bytes": (ctypes.c_size_t, [S]),
        "bsa_attn_bwd": (st, [S, P, P, P, P, P, P, P, P, ctypes.c_float, P, P, P, P, ctypes.c_size_t, P]),
        "bsa_attn_fine_workspace_bytes": (ctypes.c_size_t, [S]),
        "bsa_attn_fwd_fine": (st, [S, P, P, P, P, P, P, ctypes.c_int64, ctypes.c_float, P, P, P, ctypes.c_size_t, P]),
        "bsa_check_device_status": (st, [P, P]),
        "bsa_status_string": (ctypes.c_char_p, [st]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_LIB = None


def get_lib() -> ctypes.CDLL:
    """libbsa.so, loaded on first use; ImportError if it has not been built."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "lib":
        return get_lib()
    raise AttributeError(name)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libbsa must be contiguous")
    return t.data_ptr()


def _stream(device: Optional[torch.device] = None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(status: int, where: str) -> None:
    if status != BSA_OK:
        raise BsaError(status, where)


def make_shape(B: int, T: int, H: int, W: int, heads: int, d: int, block: int, patch: int) -> Shape:
    return Shape(B, T, H, W, heads, d, block, patch)


def validate_shape(s: Shape) -> int:
    return get_lib().bsa_validate_shape(ctypes.byref(s))


def seq_len(s: Shape) -> int:
    return get_lib().bsa_seq_len(ctypes.byref(s))


def padded_len(s: Shape) -> int:
    return get_lib().bsa_padded_len(ctypes.byref(s))


def num_blocks(s: Shape) -> int:
    return get_lib().bsa_num_blocks(ctypes.byref(s))


def workspace_bytes(s: Shape) -> int:
    return get_lib().bsa_workspace_bytes(ctypes.byref(s))


def plan_items_offset(s: Shape) -> int:
    """Byte offset of the attention work plan (int2 per 128-row tile) in the workspace."""
    return get_lib().bsa_plan_items_offset(ctypes.byref(s))


def workspace_init(ws: torch.Tensor) -> None:
    _check(get_lib().bsa_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(ws.device)),
           "bsa_workspace_init")


def reorder(s: Shape, x_bnhd: torch.Tensor, y_bhnd: torch.Tensor) -> None:
    _check(get_lib().bsa_reorder(ctypes.byref(s), _ptr(x_bnhd), _ptr(y_bhnd), _stream(x_bnhd.device)), "bsa_reorder")


def inverse_reorder(s: Shape, y_bhnd: torch.Tensor, x_bnhd: torch.Tensor) -> None:
    _check(get_lib().bsa_inverse_reorder(ctypes.byref(s), _ptr(y_bhnd), _ptr(x_bnhd), _stream(y_bhnd.device)),
           "bsa_inverse_reorder")


def build_block_mask(s: Shape, q_bhnd: torch.Tensor, k_bhnd: torch.Tensor, thr: float,
                     sta: Optional[Tuple[int, int, int]], kv_count: torch.Tensor, kv_idx: torch.Tensor,
                     mask: Optional[torch.Tensor], ws: torch.Tensor) -> None:
    st_t, st_h, st_w = sta if sta is not None else (-1, -1, -1)
    _check(get_lib().bsa_build_block_mask(ctypes.byref(s), _ptr(q_bhnd), _ptr(k_bhnd), float(thr), st_t, st_h, st_w,
                                    _ptr(kv_count), _ptr(kv_idx), _ptr(mask), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(q_bhnd.device)),
           "bsa_build_block_mask")


def reorder_qk_pooled(s: Shape, q_bnhd: torch.Tensor, k_bnhd: torch.Tensor, q_bhnd: torch.Tensor,
                      k_bhnd: torch.Tensor, ws: torch.Tensor) -> None:
    _check(get_lib().bsa_reorder_qk_pooled(ctypes.byref(s), _ptr(q_bnhd), _ptr(k_bnhd), _ptr(q_bhnd), _ptr(k_bhnd),
                                           _ptr(ws), ws.numel() * ws.element_size(), _stream(q_bnhd.device)),
           "bsa_reorder_qk_pooled")


def build_block_mask_pooled(s: Shape, thr: float, sta: Optional[Tuple[int, int, int]], kv_count: torch.Tensor,
                            kv_idx: torch.Tensor, mask: Optional[torch.Tensor], ws: torch.Tensor) -> None:
    st_t, st_h, st_w = sta if sta is not None else (-1, -1, -1)
    _check(get_lib().bsa_build_block_mask_pooled(ctypes.byref(s), float(thr), st_t, st_h, st_w, _ptr(kv_count),
                                                 _ptr(kv_idx), _ptr(mask), _ptr(ws), ws.numel() * ws.element_size(),
                                                 _stream(kv_count.device)),
           "bsa_build_block_mask_pooled")


def attn_fwd(s: Shape, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, kv_count: torch.Tensor,
             kv_idx: torch.Tensor, scale: float, o: torch.Tensor, lse: Optional[torch.Tensor],
             ws: torch.Tensor) -> None:
    _check(get_lib().bsa_attn_fwd(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(kv_count), _ptr(kv_idx),
                            float(scale), _ptr(o), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(),
                            _stream(q.device)),
           "bsa_attn_fwd")


def attn_fwd_baseline(s: Shape, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, kv_count: torch.Tensor,
                      kv_idx: torch.Tensor, scale: float, o: torch.Tensor, lse: Optional[torch.Tensor],
                      ws: torch.Tensor) -> None:
    """The legacy mma.sync kernel with the same contract (the measured baseline)."""
    _check(get_lib().bsa_attn_fwd_baseline(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(kv_count), _ptr(kv_idx),
                                     float(scale), _ptr(o), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(q.device)),
           "bsa_attn_fwd_baseline")


def attn_fwd_entropy(s: Shape, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, kv_count: torch.Tensor,
                     kv_idx: torch.Tensor, scale: float, o: torch.Tensor, lse: torch.Tensor, entropy: torch.Tensor,
                     ws: torch.Tensor) -> None:
    _check(get_lib().bsa_attn_fwd_entropy(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(kv_count), _ptr(kv_idx),
                                          float(scale), _ptr(o), _ptr(lse), _ptr(entropy), _ptr(ws),
                                          ws.numel() * ws.element_size(), _stream(q.device)),
           "bsa_attn_fwd_entropy")


def dense_lists(s: Shape, kv_count: torch.Tensor, kv_idx: torch.Tensor) -> None:
    _check(get_lib().bsa_dense_lists(ctypes.byref(s), _ptr(kv_count), _ptr(kv_idx), _stream(kv_count.device)),
           "bsa_dense_lists")


def build_block_mask_radius(s: Shape, entropy: torch.Tensor, tau: float, gamma: float, vote: int,
                            kv_count: torch.Tensor, kv_idx: torch.Tensor, mask: Optional[torch.Tensor]) -> None:
    _check(get_lib().bsa_build_block_mask_radius(ctypes.byref(s), _ptr(entropy), float(tau), float(gamma), int(vote),
                                                 _ptr(kv_count), _ptr(kv_idx), _ptr(mask), _stream(entropy.device)),
           "bsa_build_block_mask_radius")


def hilbert_workspace_bytes(s: Shape) -> int:
    return get_lib().bsa_hilbert_workspace_bytes(ctypes.byref(s))


def hilbert_order(s: Shape, order: torch.Tensor, ws: torch.Tensor) -> None:
    _check(get_lib().bsa_hilbert_order(ctypes.byref(s), _ptr(order), _ptr(ws), ws.numel() * ws.element_size(),
                                       _stream(order.device)), "bsa_hilbert_order")


def reorder_perm(s: Shape, order: torch.Tensor, x_bnhd: torch.Tensor, y_bhnd: torch.Tensor) -> None:
    _check(get_lib().bsa_reorder_perm(ctypes.byref(s), _ptr(order), _ptr(x_bnhd), _ptr(y_bhnd),
                                      _stream(x_bnhd.device)), "bsa_reorder_perm")


def inverse_reorder_perm(s: Shape, order: torch.Tensor, y_bhnd: torch.Tensor, x_bnhd: torch.Tensor) -> None:
    _check(get_lib().bsa_inverse_reorder_perm(ctypes.byref(s), _ptr(order), _ptr(y_bhnd), _ptr(x_bnhd),
                                              _stream(y_bhnd.device)), "bsa_inverse_reorder_perm")


def reorder_qk_pooled_perm(s: Shape, order: torch.Tensor, q_bnhd: torch.Tensor, k_bnhd: torch.Tensor,
                           q_bhnd: torch.Tensor, k_bhnd: torch.Tensor, ws: torch.Tensor) -> None:
    _check(get_lib().bsa_reorder_qk_pooled_perm(ctypes.byref(s), _ptr(order), _ptr(q_bnhd), _ptr(k_bnhd),
                                                _ptr(q_bhnd), _ptr(k_bhnd), _ptr(ws), ws.numel() * ws.element_size(),
                                                _stream(q_bnhd.device)), "bsa_reorder_qk_pooled_perm")


def subblock_workspace_bytes(s: Shape, sub: int) -> int:
    return get_lib().bsa_subblock_workspace_bytes(ctypes.byref(s), int(sub))


def build_block_mask_subblock(s: Shape, q_bhnd: torch.Tensor, k_bhnd: torch.Tensor, sub: int, thr: float,
                              kv_count: torch.Tensor, kv_idx: torch.Tensor, mask: Optional[torch.Tensor],
                              ws: torch.Tensor) -> None:
    _check(get_lib().bsa_build_block_mask_subblock(ctypes.byref(s), _ptr(q_bhnd), _ptr(k_bhnd), int(sub), float(thr),
                                                   _ptr(kv_count), _ptr(kv_idx), _ptr(mask), _ptr(ws),
                                                   ws.numel() * ws.element_size(), _stream(q_bhnd.device)),
           "bsa_build_block_mask_subblock")


def attn_bwd_workspace_bytes(s: Shape) -> int:
    return get_lib().bsa_attn_bwd_workspace_bytes(ctypes.byref(s))


def attn_bwd(s: Shape, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, dO: torch.Tensor,
             lse: torch.Tensor, kv_count: torch.Tensor, kv_idx: torch.Tensor, scale: float, dq: torch.Tensor,
             dk: torch.Tensor, dv: torch.Tensor, ws: torch.Tensor) -> None:
    _check(get_lib().bsa_attn_bwd(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                                  _ptr(kv_count), _ptr(kv_idx), float(scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(q.device)),
           "bsa_attn_bwd")


def attn_fine_workspace_bytes(s: Shape) -> int:
    return get_lib().bsa_attn_fine_workspace_bytes(ctypes.byref(s))


def attn_fwd_fine(s: Shape, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, sel_offsets: torch.Tensor,
                  sel_idx: torch.Tensor, sel_w: Optional[torch.Tensor], scale: float, o: torch.Tensor,
                  lse: Optional[torch.Tensor], ws: torch.Tensor) -> None:
    """Attention over per-query-block lists of 4-token KV blocks (int64 CSR
    offsets, int32 block indices, optional float32 inclusion weights)."""
    if sel_offsets.dtype != torch.int64 or sel_idx.dtype != torch.int32:
        raise TypeError("sel_offsets must be int64 and sel_idx int32")
    if sel_w is not None and (sel_w.dtype != torch.float32 or sel_w.numel() != sel_idx.numel()):
        raise TypeError("sel_w must be float32 with one weight per entry")
    n_sel = sel_idx.numel()
    _check(get_lib().bsa_attn_fwd_fine(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(sel_offsets),
                                       _ptr(sel_idx) if n_sel else None, _ptr(sel_w) if n_sel else None, n_sel,
                                       float(scale), _ptr(o), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(),
                                       _stream(q.device)),
           "bsa_attn_fwd_fine")


def check_device_status(ws: torch.Tensor) -> int:
    """Synchronises the current stream; returns the device status (0 = OK) and clears it."""
    return get_lib().bsa_check_device_status(_ptr(ws), _stream(ws.device))
