"""B200-native NABLA-style block-sparse attention for video diffusion transformers.

The compute path is libbsa.so (hand-written CUDA for sm_100a, C ABI in
include/bsa.h); this package only marshals torch tensors into it.

    import block_sparse_attention_fractal_b200 as bsa
    shape = bsa.make_shape(B, T, H, W, heads, d, block, patch)
    plan = bsa.NablaAttention(shape, device="cuda")
    out = plan(q, k, v, thr=0.2)            # q, k, v: [B, T*H*W, heads, d] bf16

The four steps can also be called one by one: ``reorder``,
``build_block_mask``, ``attn_fwd``, ``inverse_reorder``.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from ._lib import (BsaError, Shape, attn_bwd, attn_bwd_workspace_bytes, attn_fwd, attn_fwd_baseline,  # noqa: F401
                   attn_fwd_fine, attn_fine_workspace_bytes, plan_items_offset,
                   build_block_mask, build_block_mask_pooled, build_block_mask_subblock, hilbert_order,
                   hilbert_workspace_bytes, inverse_reorder_perm, reorder_perm, reorder_qk_pooled_perm,
                   subblock_workspace_bytes, attn_fwd_entropy, dense_lists, build_block_mask_radius,
                   check_device_status, inverse_reorder, reorder_qk_pooled, get_lib, make_shape, num_blocks, padded_len, reorder, seq_len, validate_shape, workspace_bytes,
                   workspace_init, LIB_PATH)

def __getattr__(name):
    # ``lib`` (the ctypes handle of libbsa.so) is loaded on first access
    if name == "lib":
        return get_lib()
    raise AttributeError(name)


__all__ = ["BsaError", "Shape", "make_shape", "NablaAttention", "reorder", "inverse_reorder", "build_block_mask",
           "reorder_qk_pooled", "build_block_mask_pooled", "attn_bwd", "attn_bwd_workspace_bytes",
           "hilbert_order", "hilbert_workspace_bytes", "reorder_perm", "inverse_reorder_perm",
           "reorder_qk_pooled_perm", "build_block_mask_subblock", "subblock_workspace_bytes",
           "attn_fwd_entropy", "dense_lists", "build_block_mask_radius", "attn_fwd_fine", "attn_fine_workspace_bytes",
           "plan_items_offset",
           "attn_fwd", "attn_fwd_baseline", "check_device_status", "workspace_bytes", "workspace_init", "padded_len", "num_blocks",
           "seq_len", "validate_shape", "get_lib", "LIB_PATH"]


class NablaAttention:
    """Owns the device buffers of one shape and runs the whole path: reorder
    Q and K with their block means -> block mask -> block-sparse attention ->
    inverse reorder, ordered on the current stream.  V's reorder runs on a
    side stream after the Q/K reorder, concurrently with the block mask (which
    needs only Q and K); the attention waits for both.  Buffers are allocated
    once (torch) and reused."""

    def __init__(self, shape: Shape, device="cuda", with_mask: bool = False, with_lse: bool = False):
        st = validate_shape(shape)
        if st != 0:
            raise BsaError(st, "bsa_validate_shape")
        self.shape = shape
        dev = torch.device(device)
        B, heads, d = shape.B, shape.heads, shape.d
        Npad, nb = padded_len(shape), num_blocks(shape)
        self.N, self.Npad, self.nb = seq_len(shape), Npad, nb
        kw = dict(device=dev)
        self.q = torch.empty(B, heads, Npad, d, dtype=torch.bfloat16, **kw)
        self.k = torch.empty_like(self.q)
        self.v = torch.empty_like(self.q)
        self.o = torch.empty_like(self.q)
        self.kv_count = torch.empty(B, heads, nb, dtype=torch.int32, **kw)
        self.kv_idx = torch.empty(B, heads, nb, nb, dtype=torch.int32, **kw)
        self.mask = torch.empty(B, heads, nb, nb, dtype=torch.uint8, **kw) if with_mask else None
        self.lse = torch.empty(B, heads, Npad, dtype=torch.float32, **kw) if with_lse else None
        ws_bytes = workspace_bytes(shape)
        self.ws = torch.empty((ws_bytes + 15) // 16 * 16, dtype=torch.uint8, **kw)
        workspace_init(self.ws)
        self.side = torch.cuda.Stream(device=dev)

    def reorder_inputs(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> None:
        """Q and K in one launch on the current stream, with their block means
        kept in the workspace for mask_step; V on the side stream (joined by
        join_side before the attention)."""
        main = torch.cuda.current_stream(q.device)
        reorder_qk_pooled(self.shape, q, k, self.q, self.k, self.ws)
        # V after the Q/K launch: its reorder then overlaps the (compute-bound)
        # mask kernel rather than sharing HBM with the Q/K pass
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            reorder(self.shape, v, self.v)

    def join_side(self) -> None:
        torch.cuda.current_stream(self.q.device).wait_stream(self.side)

    def mask_step(self, thr: float, sta: Optional[Tuple[int, int, int]] = None) -> None:
        """The block mask from the block means reorder_inputs left in the workspace."""
        build_block_mask_pooled(self.shape, thr, sta, self.kv_count, self.kv_idx, self.mask, self.ws)

    def attention_step(self, scale: float = 0.0, baseline: bool = False) -> None:
        fn = attn_fwd_baseline if baseline else attn_fwd
        fn(self.shape, self.q, self.k, self.v, self.kv_count, self.kv_idx, scale, self.o, self.lse, self.ws)

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, thr: float,
                 sta: Optional[Tuple[int, int, int]] = None, scale: float = 0.0,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
        self.reorder_inputs(q, k, v)
        self.mask_step(thr, sta)
        self.join_side()
        self.attention_step(scale)
        if out is None:
            out = torch.empty_like(q)
        inverse_reorder(self.shape, self.o, out)
        return out

    def status(self) -> int:
        return check_device_status(self.ws)
