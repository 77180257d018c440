"""The C ABI library loads here (no GPU) and exports every symbol the header
declares; host-side shape arithmetic and argument checks need no device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^BSA_API\s+[\w\s\*]+?\b(bsa_\w+)\s*\(", text, flags=re.M))
    return sorted(names)


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_fractal_b200 as m
    return m


def test_header_declares_the_path():
    names = _declared_symbols()
    for want in ("bsa_reorder", "bsa_build_block_mask", "bsa_attn_fwd", "bsa_inverse_reorder",
                 "bsa_check_device_status", "bsa_workspace_bytes"):
        assert want in names


def test_library_exports_every_declared_symbol(bsa):
    lib = ctypes.CDLL(bsa.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name


def test_shape_arithmetic(bsa):
    s = bsa.make_shape(1, 21, 30, 52, 12, 128, 64, 8)
    assert bsa.seq_len(s) == 32760
    assert bsa.padded_len(s) == 32768
    assert bsa.num_blocks(s) == 512
    # control block | q and k block means (double) | reduced scores (double) | attention
    # plan (one int2 per 128-row tile, then pairing weights of 32 neighbours (uint16) and
    # a count (int32) per block row, then a 256-byte slot for the work counter of the
    # attention kernel)
    assert bsa.workspace_bytes(s) == (256 + 2 * 12 * 512 * 128 * 8 + 12 * 512 * 512 * 8 + 12 * 256 * 8
                                      + 12 * 512 * 64 + 12 * 512 * 4 + 256)
    s = bsa.make_shape(1, 33, 45, 80, 24, 128, 128, 8)
    assert (bsa.seq_len(s), bsa.padded_len(s), bsa.num_blocks(s)) == (118800, 118912, 929)
    assert bsa.validate_shape(s) == 0


@pytest.mark.parametrize("field,value", [("d", 96), ("block", 32), ("patch", 0), ("B", 0), ("heads", 0)])
def test_invalid_shapes_are_rejected(bsa, field, value):
    s = bsa.make_shape(1, 4, 16, 16, 2, 64, 64, 8)
    setattr(s, field, value)
    assert bsa.validate_shape(s) == 1
    assert bsa.padded_len(s) == -1 and bsa.workspace_bytes(s) == 0


def test_too_many_blocks_is_unsupported(bsa):
    s = bsa.make_shape(1, 1, 256, 257, 1, 64, 64, 8)   # nb = 1028
    assert bsa.num_blocks(s) == 1028
    assert bsa.validate_shape(s) == 2


def test_argument_errors_return_before_any_cuda_call(bsa):
    lib = bsa.lib
    s = bsa.make_shape(1, 4, 16, 16, 2, 64, 64, 8)
    ref = ctypes.byref(s)
    fake = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced: every call below fails its checks
    odd = ctypes.c_void_p((1 << 20) + 4)     # misaligned
    assert lib.bsa_reorder(ref, None, fake, None) == 1
    assert lib.bsa_reorder(ref, odd, fake, None) == 1
    assert lib.bsa_reorder(ref, fake, fake, None) == 1          # in place is refused
    assert lib.bsa_inverse_reorder(None, fake, fake, None) == 1
    ws = bsa.workspace_bytes(s)
    for thr in (-0.1, 1.0, float("nan")):
        assert lib.bsa_build_block_mask(ref, fake, fake, thr, -1, -1, -1, fake, fake, None, fake, ws, None) == 1
    assert lib.bsa_build_block_mask(ref, fake, fake, 0.1, -1, -1, -1, fake, fake, None, fake, ws - 16, None) == 1
    assert lib.bsa_attn_fwd(ref, fake, fake, fake, fake, fake, float("inf"), fake, None, fake, ws, None) == 1
    assert lib.bsa_attn_fwd(ref, fake, fake, None, fake, fake, 0.0, fake, None, fake, ws, None) == 1
    assert lib.bsa_workspace_init(None, 1024, None) == 1
    assert lib.bsa_status_string(4) == b"BSA_ERR_DEVICE_INDEX"
