"""bsa_attn_fwd_noalloc: attention for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc where they run attention (a fixed memory
budget handed out up front, a plug-in inside a host program that owns every
allocation).  bsa_attn_fwd_noalloc takes no workspace: its scratch is a static
device array inside libbsa.so.  These tests call it through the C ABI and check
that it gives the same output as bsa_attn_fwd, call after call, that it
reports device errors in the caller's error word, and that it refuses shapes
whose scratch would not fit.

This file is collected last, so a run that stops at the first failure has run
every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_fractal_b200 import synth

from _util import MAX_ABS, MEAN_ABS, compare_outputs, small, to64

NOALLOC_SCRATCH_BYTES = 4 << 20   # BSA_NOALLOC_SCRATCH_BYTES in include/bsa.h


def _fn(lib):
    fn = lib.bsa_attn_fwd_noalloc
    P = ctypes.c_void_p
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, P, P, P, P, P, ctypes.c_float, P, P, P, P]
    return fn


def test_too_large_shape_is_refused_before_any_launch():
    import block_sparse_attention_fractal_b200 as bsa
    fn = _fn(bsa.lib)
    # 1024 heads x 1024 query tiles of 128 rows: 8 MiB of plan, beyond the 4 MiB array.
    s = bsa.make_shape(1, 1, 256, 512, 1024, 128, 128, 8)
    assert bsa.validate_shape(s) == 0
    assert 256 + 8 * 1024 * bsa.num_blocks(s) > NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)   # aligned and never dereferenced: the call must return first
    st = fn(ctypes.addressof(s), fake, fake, fake, fake, fake, 0.0, fake, None, None, None)
    assert st == 2   # BSA_ERR_UNSUPPORTED
    st = fn(ctypes.addressof(s), None, fake, fake, fake, fake, 0.0, fake, None, None, None)
    assert st == 1   # BSA_ERR_INVALID_ARG comes first for a missing pointer


@pytest.mark.gpu
@pytest.mark.parametrize("w", [small("noalloc_b64", 1, 3, 20, 28, 2, 128, 64, 8, 0.15),
                               small("noalloc_b128_d64", 1, 2, 13, 37, 3, 64, 128, 4, 0.3)],
                         ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point_twice_in_a_row(w):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as bsa
    fn = _fn(bsa.lib)
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch), with_lse=True)
    bsa.reorder_qk_pooled(plan.shape, q.cuda(), k.cuda(), plan.q, plan.k, plan.ws)
    bsa.reorder(plan.shape, v.cuda(), plan.v)
    plan.mask_step(w.thr, w.sta)
    plan.attention_step()                     # the workspace entry point: the expected output
    torch.cuda.synchronize()
    assert plan.status() == 0
    want_o, want_lse = to64(plan.o), to64(plan.lse)

    err = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full_like(plan.o, float("nan"))
        lse = torch.full_like(plan.lse, float("nan"))
        st = fn(ctypes.addressof(plan.shape), plan.q.data_ptr(), plan.k.data_ptr(), plan.v.data_ptr(),
                plan.kv_count.data_ptr(), plan.kv_idx.data_ptr(), 0.0, o.data_ptr(), lse.data_ptr(),
                err.data_ptr(), stream)
        assert st == 0, (call, st)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, (call, int(err.item()))
        got = to64(o)
        mx, mean = compare_outputs(got[:, :, :w.N], want_o[:, :, :w.N])
        assert mx <= MAX_ABS and mean <= MEAN_ABS, (call, mx, mean)
        assert np.all(got[:, :, w.N:] == 0)
        assert np.abs(to64(lse)[:, :, :w.N] - want_lse[:, :, :w.N]).max() <= 2e-3


@pytest.mark.gpu
def test_noalloc_reports_device_errors_per_call():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_attention_fractal_b200 as bsa
    fn = _fn(bsa.lib)
    w = small("noalloc_err", 1, 1, 16, 16, 2, 64, 64, 8, 0.0)
    q, k, v = synth.make_qkv(w)
    plan = bsa.NablaAttention(bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch))
    for src, dst in ((q, plan.q), (k, plan.k), (v, plan.v)):
        bsa.reorder(plan.shape, src.cuda(), dst)
    plan.kv_count.fill_(1)
    plan.kv_idx.zero_()
    plan.kv_idx[0, 1, 2, 0] = plan.nb + 5      # out of range: skipped by the kernel and flagged
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    args = lambda: (ctypes.addressof(plan.shape), plan.q.data_ptr(), plan.k.data_ptr(), plan.v.data_ptr(),
                    plan.kv_count.data_ptr(), plan.kv_idx.data_ptr(), 0.0, plan.o.data_ptr(), None,
                    err.data_ptr(), stream)
    assert fn(*args()) == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 1                 # BSA_ERR_DEVICE_INDEX bit
    plan.kv_idx[0, 1, 2, 0] = 0
    assert fn(*args()) == 0                     # the next call starts from a clear error word
    torch.cuda.synchronize()
    assert int(err.item()) == 0
