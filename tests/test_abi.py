"""The C-ABI library loads, exports every entry point include/bra.h declares, and
rejects bad arguments before touching CUDA (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

from vision_transformer_sparse_b200 import bra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "bra.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bra_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    assert set(names) == set(bra.SYMBOLS), names


def test_library_exports_every_declared_symbol(bra_lib):
    for name in declared_functions():
        assert hasattr(bra_lib, name), name
    assert bra_lib.bra_version() >> 16 == 1
    for code in range(9):
        assert bra.status_string(code) != "unknown status"


FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: checks fail first
ODD = ctypes.c_void_p(0x10008)


def fwd(shape, ptrs=None):
    p = [FAKE] * 5 if ptrs is None else ptrs[:5]
    o = [FAKE] * 3 if ptrs is None else ptrs[5:]
    return bra.raw_call("bra_forward", *p, *shape, *o, None)


@pytest.mark.parametrize("shape,code", [
    ((1, 56, 56, 64, 3, 7, 1, 1), 2),    # C % heads
    ((1, 56, 56, 96, 2, 7, 1, 1), 2),    # d = 48
    ((1, 56, 56, 64, 2, 7, 0, 1), 2),    # topk = 0
    ((1, 56, 56, 64, 2, 7, 50, 1), 2),   # topk > S^2
    ((1, 68, 68, 64, 2, 17, 1, 1), 2),   # S^2 > 256
    ((1, 56, 56, 64, 2, 0, 1, 1), 2),    # S = 0
    ((-1, 56, 56, 64, 2, 7, 1, 1), 2),   # N < 0
    ((1, 56, 56, 64, 2, 7, 1, 7), 4),    # dtype
    ((1, 1032, 1032, 64, 2, 4, 1, 1), 2),  # region wider than 128
    ((1, 64, 1025, 64, 2, 8, 1, 1), 2),    # padded region wider than 128 (ceil(1025/8) = 129)
])
def test_bad_shapes_rejected(bra_lib, shape, code):
    assert fwd(shape) == code
    assert bra.raw_call("bra_route", FAKE, FAKE, *shape, FAKE, FAKE, None) == code
    assert bra.raw_call("bra_attend", *[FAKE] * 5, *shape, FAKE, FAKE, None) == code
    assert bra.raw_call("bra_forward_host", *[FAKE] * 5, *shape, *[FAKE] * 3, None) == code
    assert bra.raw_call("bra_forward_noalloc", *[FAKE] * 5, *shape, *[FAKE] * 3, None) == code


def test_null_and_alignment_rejected(bra_lib):
    shape = (1, 56, 56, 64, 2, 7, 1, 1)
    for i in range(8):
        ptrs = [FAKE] * 8
        ptrs[i] = None
        assert fwd(shape, ptrs) == 1
    for i in (0, 1, 2, 5):   # q, k, v, out need 16 bytes
        ptrs = [FAKE] * 8
        ptrs[i] = ODD
        assert fwd(shape, ptrs) == 3
    ptrs = [FAKE] * 8
    ptrs[6] = ctypes.c_void_p(0x10002)   # r_idx needs 4 bytes
    assert fwd(shape, ptrs) == 3
    assert bra.raw_call("bra_route", None, FAKE, *shape, FAKE, FAKE, None) == 1
    assert bra.raw_call("bra_attend", *[FAKE] * 5, *shape, None, FAKE, None) == 1


def test_empty_batch_is_a_no_op(bra_lib):
    shape = (0, 56, 56, 64, 2, 7, 1, 1)
    assert fwd(shape, [None] * 8) == 0
    assert bra.raw_call("bra_route", None, None, *shape, None, None, None) == 0


# ---------------------------------------------------------------- projections and the layer

def lin(M, K, Nout, dtype, x=FAKE, w=FAKE, b=FAKE, y=FAKE):
    return bra.raw_call("bra_linear", x, w, b, M, K, Nout, dtype, y, None)


@pytest.mark.parametrize("M,K,Nout,dtype,code", [
    (10, 64, 64, 7, 4),       # dtype
    (-1, 64, 64, 1, 2),       # M < 0
    (10, 0, 64, 1, 2),        # K = 0
    (10, 48, 64, 1, 2),       # bf16 K not a multiple of 32
    (10, 64, 48, 1, 2),       # bf16 Nout not a multiple of 32
    (10, 8192, 64, 1, 2),     # K above 4096
    (10, 64, 8192, 0, 2),     # Nout above 4096
])
def test_linear_bad_shapes_rejected(bra_lib, M, K, Nout, dtype, code):
    assert lin(M, K, Nout, dtype) == code


def test_linear_nulls_alignment_and_empty(bra_lib):
    for i in range(4):
        ptrs = [FAKE] * 4
        ptrs[i] = None
        assert lin(10, 64, 64, 1, *ptrs) == 1
    for i in (0, 1, 3):   # x, w, y need 16 bytes
        ptrs = [FAKE] * 4
        ptrs[i] = ODD
        assert lin(10, 64, 64, 1, *ptrs) == 3
    assert lin(10, 64, 64, 1, b=ctypes.c_void_p(0x10001)) == 3   # bias aligned to its element
    assert lin(0, 64, 64, 1, None, None, None, None) == 0        # nothing to do
    assert lin(0, 48, 40, 0, None, None, None, None) == 0        # float32 takes any K, Nout


def test_qkv_rejects_before_cuda(bra_lib):
    call = lambda M, C, dt, *p: bra.raw_call("bra_qkv", *(p[:3] if p else [FAKE] * 3), M, C, dt,
                                             *(p[3:] if p else [FAKE] * 3), None)
    assert call(10, 48, 1) == 2          # each third must be a multiple of 32 in bf16
    assert call(10, 2000, 1) == 2        # 3C above 4096
    assert call(10, 64, 9) == 4
    assert call(10, 64, 1, FAKE, FAKE, FAKE, FAKE, None, FAKE) == 1
    assert call(10, 64, 1, FAKE, FAKE, FAKE, FAKE, FAKE, ODD) == 3
    assert call(0, 64, 1, None, None, None, None, None, None) == 0


@pytest.mark.parametrize("shape,code", [
    ((1, 56, 56, 96, 2, 7, 1, 1), 2),    # d = 48
    ((1, 56, 56, 64, 2, 7, 50, 1), 2),   # topk > S^2
    ((1, 56, 56, 64, 2, 7, 1, 7), 4),    # dtype
])
def test_layer_bad_shapes_rejected(bra_lib, shape, code):
    assert bra.raw_call("bra_attention_layer", *[FAKE] * 7, *shape, *[FAKE] * 3, None) == code


def test_layer_nulls_and_alignment(bra_lib):
    shape = (1, 56, 56, 64, 2, 7, 1, 1)
    for i in range(10):
        ptrs = [FAKE] * 10
        ptrs[i] = None
        assert bra.raw_call("bra_attention_layer", *ptrs[:7], *shape, *ptrs[7:], None) == 1
    for i in (0, 1, 3, 7):   # x, w_qkv, w_o, out need 16 bytes
        ptrs = [FAKE] * 10
        ptrs[i] = ODD
        assert bra.raw_call("bra_attention_layer", *ptrs[:7], *shape, *ptrs[7:], None) == 3
    assert bra.raw_call("bra_attention_layer", *[None] * 7, 0, 56, 56, 64, 2, 7, 1, 1, *[None] * 3, None) == 0


def test_backward_rejects_before_cuda(bra_lib):
    shape = (1, 56, 56, 64, 2, 7, 1, 1)
    call = lambda ptrs, shp=shape: bra.raw_call("bra_backward", *ptrs[:6], *shp, *ptrs[6:], None)
    assert call([FAKE] * 11, (1, 57, 56, 64, 2, 7, 1, 1)) == 2      # H % S
    assert call([FAKE] * 11, (1, 56, 56, 64, 2, 7, 1, 7)) == 4      # dtype
    for i in range(11):
        ptrs = [FAKE] * 11
        ptrs[i] = None
        assert call(ptrs) == 1
    for i in (0, 1, 2, 3, 5):   # bf16 maps and weight: 2-byte alignment
        ptrs = [FAKE] * 11
        ptrs[i] = ctypes.c_void_p(0x10001)
        assert call(ptrs) == 3
    for i in (4, 6, 7, 8, 9, 10):   # r_idx and the float32 outputs: 4 bytes
        ptrs = [FAKE] * 11
        ptrs[i] = ctypes.c_void_p(0x10002)
        assert call(ptrs) == 3


@pytest.mark.parametrize("shape", [
    (0, 57, 56, 64, 2, 7, 1, 1),     # H not a multiple of S
    (0, 56, 50, 64, 2, 7, 1, 1),     # W not a multiple of S
    (0, 30, 30, 64, 2, 7, 3, 1),     # a whole region row and column of padding
    (0, 250, 250, 64, 2, 16, 1, 1),  # 250 -> 256: the padded grid of 16 x 16 regions
])
def test_padded_grid_shapes_accepted(bra_lib, shape):
    """H or W not a multiple of S is the padded grid: accepted by every forward entry
    point (N = 0 launches nothing), refused by the no-allocation entry point (its static
    array cannot hold the padded copies) and by the backward."""
    assert fwd(shape, [None] * 8) == 0
    assert bra.raw_call("bra_route", None, None, *shape, None, None, None) == 0
    assert bra.raw_call("bra_attend", *[None] * 5, *shape, None, None, None) == 0
    assert bra.raw_call("bra_forward_host", *[None] * 5, *shape, *[None] * 3, None) == 0
    assert bra.raw_call("bra_attention_layer", *[None] * 7, *shape, *[None] * 3, None) == 0
    one = (1,) + shape[1:]
    assert bra.raw_call("bra_forward_noalloc", *[FAKE] * 5, *one, *[FAKE] * 3, None) == 7
    assert bra.raw_call("bra_backward", *[FAKE] * 6, *one, *[FAKE] * 5, None) == 2
