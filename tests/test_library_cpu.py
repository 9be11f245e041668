"""Host-side checks of libbsattn.so that need no GPU.

The library must load on a machine without a GPU driver, export every entry
point declared in include/bsattn.h, and reject bad arguments before touching
the device.
"""
import ctypes
import os
import re

import pytest

import block_sparse_attention_49_b200 as bsa
from block_sparse_attention_49_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return bsa.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "bsattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_binding_names():
    assert _declared() == sorted(bsa.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert bsa.bsa_version().startswith("bsattn")


def _create(lib, *args):
    h = ctypes.c_void_p()
    st = lib.bsa_plan_create(ctypes.byref(h), *args)
    return st, h


@pytest.mark.parametrize("args,status", [
    ((1, 2, 96, 8, 8, 8, 0, 0, 0, 64), 2),      # head dim 96 unsupported
    ((1, 2, 64, 8, 8, 8, 0, 0, 0, 96), 2),      # block must divide 128
    ((1, 2, 64, 8, 8, 8, 0, 0, 0, 256), 2),     # blocks above 128 slots
    ((1, 2, 64, 8, 8, 8, 1, 2, 3, 4), 1),       # pool_h * pool_w != block
    ((1, 2, 64, 8, 8, 8, 1, 0, 2, 4), 1),       # pool sizes must be positive
    ((0, 2, 64, 8, 8, 8, 0, 0, 0, 64), 1),      # empty batch
    ((1, 2, 64, 8, 8, 8, 7, 0, 0, 64), 1),      # unknown layout
    ((1, 2, 64, 8, 65536, 65536, 0, 0, 0, 64), 2),        # H * W beyond 32 bits
    ((1, 2, 64, 8, 8, 8, 1, 65536, 65536, 64), 1),        # pool_h * pool_w beyond 32 bits
    ((1, 2, 64, 8, 8, 8, 1, 128, 33554433, 128), 1),      # product wraps to 128 in 32 bits
])
def test_plan_create_rejects_bad_geometry_on_host(lib, args, status):
    st, h = _create(lib, *args)
    assert st == status
    assert not h.value
    assert bsa.bsa_last_error()


def test_null_plan_is_rejected(lib):
    assert lib.bsa_padded_tokens(None) == -1
    assert lib.bsa_lvsa_mask(None, 4, 4, 0, None, None, None, None) == 1
    assert lib.bsa_attn_fwd(None, None, None, None, None, None, 0, 1.0, None, None, None) == 1
    assert lib.bsa_poll_status(None, None) == 1
    assert lib.bsa_plan_set_lvsa_variant(None, 0, 0) == 1
    assert lib.bsa_plan_set_draft_pooling(None, 0) == 1
    assert lib.bsa_plan_set_draft_precision(None, 0) == 1
    assert lib.bsa_plan_set_reorder_pads(None, 0) == 1
    assert lib.bsa_lvsa_attn_fwd(None, 4, 4, 0, None, None, None, 1.0, None, None, None) == 1
    assert lib.bsa_attn_fwd_natural(None, None, None, None, None, None, 1, 1.0, None, None,
                                    None) == 1
    assert lib.bsa_draft_mask(None, None, None, 90, None, None, None, None, 0, None) == 1
    assert lib.bsa_draft_mask_natural(None, None, None, 90, None, None, None, None, 0, None) == 1
    assert lib.bsa_draft_mask_noalloc(None, None, None, 90, None, None, None, None) == 1
    assert lib.bsa_quantize_e4m3(None, None, None, None, None, None, None, None, None) == 1
    assert lib.bsa_draft_mask_natural_e4m3(None, None, None, None, 90, None, None, None, None, 0,
                                           None, None, None, None, None) == 1
    assert lib.bsa_attn_fwd_natural_e4m3(None, None, None, None, None, None, None, 1, 1.0, None,
                                         None, None) == 1
    assert lib.bsa_reorder_fwd(None, None, None, None, None, None, None, None) == 1
    assert lib.bsa_reorder_inv(None, None, None, None) == 1
    assert lib.bsa_lvsa_nnz(None, 4) == -1
    assert lib.bsa_draft_keep_count(None, 90) == -1
    assert lib.bsa_draft_workspace_bytes(None) == 0


def test_no_cpu_fallback_path():
    # the binding only marshals arguments: a CPU tensor is refused before any call
    import torch
    with pytest.raises(ValueError):
        bsa._ptr(torch.zeros(4))
