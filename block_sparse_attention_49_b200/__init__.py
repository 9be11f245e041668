"""Python binding of libbsattn.so: block-sparse attention over [t,h,w] video
tokens on NVIDIA B200 (sm_100a).

Argument marshalling only: every computation runs in the library's CUDA
kernels.  The binding passes device pointers (`tensor.data_ptr()`) and the
current torch CUDA stream, and raises BsaError on any non-OK status.  If the
library is missing, importing the binding's functions raises; there is no
fallback of any kind.

Entry points keep the C names (bsa_plan_create, bsa_lvsa_mask,
bsa_draft_mask, bsa_reorder_fwd, bsa_reorder_inv, bsa_attn_fwd,
bsa_poll_status, ...); see include/bsattn.h for their exact contracts.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "BsaError", "Plan", "LAYOUT_FRAME", "LAYOUT_TILE", "lib_path", "load",
    "ANCHORS_ROTATING", "ANCHORS_FIXED", "ANCHORS_NONE", "WINDOW_DISTANCE", "WINDOW_ALTERNATE",
    "POOL_MEAN", "POOL_MAX", "DRAFT_FP64", "DRAFT_FP32", "PADS_WRITE", "PADS_KEEP",
    "bsa_plan_create", "bsa_plan_destroy", "bsa_plan_set_lvsa_variant",
    "bsa_plan_set_draft_pooling", "bsa_plan_set_draft_precision", "bsa_plan_set_reorder_pads",
    "bsa_padded_tokens",
    "bsa_num_blocks",
    "bsa_block_size", "bsa_lvsa_mask", "bsa_lvsa_nnz", "bsa_draft_keep_count",
    "bsa_draft_workspace_bytes", "bsa_draft_mask", "bsa_draft_mask_noalloc",
    "bsa_draft_noalloc_max_scratch_bytes", "bsa_reorder_fwd", "bsa_reorder_inv",
    "bsa_attn_fwd", "bsa_attn_fwd_natural", "bsa_draft_mask_natural", "bsa_quantize_e4m3",
    "bsa_attn_fwd_natural_e4m3", "bsa_draft_mask_natural_e4m3", "bsa_lvsa_attn_fwd", "bsa_poll_status", "bsa_set_wait_limit_ns", "bsa_selftest_timeout",
    "bsa_last_error", "bsa_version", "EXPORTED_SYMBOLS",
]

LAYOUT_FRAME = 0
LAYOUT_TILE = 1
ANCHORS_ROTATING, ANCHORS_FIXED, ANCHORS_NONE = 0, 1, 2
WINDOW_DISTANCE, WINDOW_ALTERNATE = 0, 1
POOL_MEAN, POOL_MAX = 0, 1
DRAFT_FP64, DRAFT_FP32 = 0, 1
PADS_WRITE, PADS_KEEP = 0, 1

STATUS = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_UNSUPPORTED",
          3: "BSA_ERR_ALIGNMENT", 4: "BSA_ERR_CUDA", 5: "BSA_ERR_TIMEOUT",
          6: "BSA_ERR_BAD_BLOCKLIST"}

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libbsattn.so")

_c_int, _c_i64, _c_sz, _c_p, _c_u64 = (ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                                       ctypes.c_void_p, ctypes.c_uint64)

# name -> (restype, argtypes)
_SIGS = {
    "bsa_plan_create": (_c_int, [ctypes.POINTER(_c_p)] + [_c_int] * 10),
    "bsa_plan_destroy": (_c_int, [_c_p]),
    "bsa_plan_set_lvsa_variant": (_c_int, [_c_p, _c_int, _c_int]),
    "bsa_plan_set_draft_pooling": (_c_int, [_c_p, _c_int]),
    "bsa_plan_set_draft_precision": (_c_int, [_c_p, _c_int]),
    "bsa_plan_set_reorder_pads": (_c_int, [_c_p, _c_int]),
    "bsa_padded_tokens": (_c_i64, [_c_p]),
    "bsa_num_blocks": (_c_i64, [_c_p]),
    "bsa_block_size": (_c_int, [_c_p]),
    "bsa_lvsa_mask": (_c_int, [_c_p, _c_int, _c_int, _c_int, _c_p, _c_p, _c_p, _c_p]),
    "bsa_lvsa_nnz": (_c_i64, [_c_p, _c_int]),
    "bsa_draft_keep_count": (_c_int, [_c_p, _c_int]),
    "bsa_draft_workspace_bytes": (_c_sz, [_c_p]),
    "bsa_draft_mask": (_c_int, [_c_p, _c_p, _c_p, _c_int, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "bsa_draft_mask_noalloc": (_c_int, [_c_p, _c_p, _c_p, _c_int, _c_p, _c_p, _c_p, _c_p]),
    "bsa_draft_noalloc_max_scratch_bytes": (_c_sz, []),
    "bsa_reorder_fwd": (_c_int, [_c_p] * 8),
    "bsa_reorder_inv": (_c_int, [_c_p, _c_p, _c_p, _c_p]),
    "bsa_attn_fwd": (_c_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_int, ctypes.c_float, _c_p,
                              _c_p, _c_p]),
    "bsa_attn_fwd_natural": (_c_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_int, ctypes.c_float, _c_p,
                              _c_p, _c_p]),
    "bsa_draft_mask_natural": (_c_int, [_c_p, _c_p, _c_p, _c_int, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "bsa_quantize_e4m3": (_c_int, [_c_p] * 9),
    "bsa_draft_mask_natural_e4m3": (_c_int, [_c_p, _c_p, _c_p, _c_p, _c_int, _c_p, _c_p, _c_p, _c_p,
                                             _c_sz, _c_p, _c_p, _c_p, _c_p, _c_p]),
    "bsa_attn_fwd_natural_e4m3": (_c_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_int,
                                           ctypes.c_float, _c_p, _c_p, _c_p]),
    "bsa_lvsa_attn_fwd": (_c_int, [_c_p, _c_int, _c_int, _c_int, _c_p, _c_p, _c_p, ctypes.c_float,
                                   _c_p, _c_p, _c_p]),
    "bsa_poll_status": (_c_int, [_c_p, _c_p]),
    "bsa_set_wait_limit_ns": (_c_int, [_c_p, _c_u64]),
    "bsa_selftest_timeout": (_c_int, [_c_p, _c_u64, _c_p]),
    "bsa_last_error": (ctypes.c_char_p, []),
    "bsa_version": (ctypes.c_char_p, []),
}
EXPORTED_SYMBOLS = tuple(_SIGS)

_lib = None


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")
        self.status = status


def load():
    """Load libbsattn.so (building nothing) and return the ctypes handle."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise ImportError(f"libbsattn.so not built ({lib_path}); run "
                              "python -m block_sparse_attention_49_b200._build")
        lib = ctypes.CDLL(lib_path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(st: int, where: str):
    if st != 0:
        raise BsaError(st, where, load().bsa_last_error().decode())


def _ptr(t) -> Optional[int]:
    """Device address of a tensor (or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _need(what: str, t, nbytes: int):
    """Rejects a tensor smaller than the plan implies: the kernels take every
    size from the plan, so a short buffer would be read or written past its
    end.  None and raw integer addresses pass unchecked."""
    if t is None or isinstance(t, int):
        return
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise ValueError(f"{what}: {have} bytes, the plan needs {nbytes}")


def _natural(plan, elem: int = 2) -> int:
    """Bytes of one natural-layout tensor [B, N, Hh, D]."""
    return plan.B * plan.T * plan.H * plan.W * plan.Hh * plan.D * elem


def _slots(plan, elem: int = 2) -> int:
    """Bytes of one slot-layout tensor [B, Hh, Npad, D]."""
    return plan.B * plan.Hh * plan.Npad * plan.D * elem


def _need_lists(plan, per_head_lists: bool, row_ptr):
    lists = plan.B * plan.Hh if per_head_lists else 1
    _need("row_ptr", row_ptr, (lists * plan.nblocks + 1) * 4)


def _need_draft_outputs(plan, sparsity_pct: int, row_ptr, kv_idx, draft_map):
    if not 0 <= sparsity_pct < 100:
        return  # rejected by the library
    rows = plan.B * plan.Hh * plan.nblocks
    keep = plan.keep_count(sparsity_pct)
    _need("kv_idx", kv_idx, rows * keep * 4)
    _need("row_ptr", row_ptr, (rows + 1) * 4)
    _need("draft_map", draft_map, rows * plan.nblocks * 4)


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


class Plan:
    """Owns a bsa_plan_t; geometry of one attention problem."""

    def __init__(self, B, Hh, D, T, H, W, layout, pool_h=0, pool_w=0, block=128):
        self.B, self.Hh, self.D, self.T, self.H, self.W = B, Hh, D, T, H, W
        self.layout, self.pool_h, self.pool_w = layout, pool_h, pool_w
        h = _c_p()
        _check(load().bsa_plan_create(ctypes.byref(h), B, Hh, D, T, H, W, layout, pool_h,
                                      pool_w, block), "bsa_plan_create")
        self.handle = h
        self.Npad = int(load().bsa_padded_tokens(h))
        self.nblocks = int(load().bsa_num_blocks(h))
        self.block = int(load().bsa_block_size(h))

    def keep_count(self, sparsity_pct: int) -> int:
        """Blocks kept per draft row at `sparsity_pct` (bsa_draft_keep_count)."""
        k = int(load().bsa_draft_keep_count(self.handle, int(sparsity_pct)))
        if k < 0:
            raise BsaError(1, "bsa_draft_keep_count", load().bsa_last_error().decode())
        return k

    def close(self):
        if getattr(self, "handle", None):
            _check(load().bsa_plan_destroy(self.handle), "bsa_plan_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def bsa_plan_create(B, Hh, D, T, H, W, layout, pool_h=0, pool_w=0, block=128) -> Plan:
    return Plan(B, Hh, D, T, H, W, layout, pool_h, pool_w, block)


def bsa_plan_destroy(plan: Plan):
    plan.close()


def bsa_padded_tokens(plan: Plan) -> int:
    return int(load().bsa_padded_tokens(plan.handle))


def bsa_num_blocks(plan: Plan) -> int:
    return int(load().bsa_num_blocks(plan.handle))


def bsa_block_size(plan: Plan) -> int:
    return int(load().bsa_block_size(plan.handle))


def bsa_lvsa_nnz(plan: Plan, C: int) -> int:
    return int(load().bsa_lvsa_nnz(plan.handle, C))


def bsa_lvsa_mask(plan: Plan, C: int, T_per: int, s: int, frame_sets, row_ptr, col_idx,
                  stream=None):
    if C > 0:
        _need("frame_sets", frame_sets, plan.T * C * 4)
        _need("col_idx", col_idx, plan.nblocks * C * (plan.nblocks // plan.T) * 4)
    _need("row_ptr", row_ptr, (plan.nblocks + 1) * 4)
    _check(load().bsa_lvsa_mask(plan.handle, C, T_per, s, _ptr(frame_sets), _ptr(row_ptr),
                                _ptr(col_idx), _stream(stream)), "bsa_lvsa_mask")


def bsa_draft_keep_count(plan: Plan, sparsity_pct: int) -> int:
    return int(load().bsa_draft_keep_count(plan.handle, sparsity_pct))


def bsa_draft_workspace_bytes(plan: Plan) -> int:
    return int(load().bsa_draft_workspace_bytes(plan.handle))


def bsa_draft_mask(plan: Plan, q_slots, k_slots, sparsity_pct: int, row_ptr, kv_idx,
                   draft_map, workspace, stream=None):
    _need("q_slots", q_slots, _slots(plan))
    _need("k_slots", k_slots, _slots(plan))
    _need_draft_outputs(plan, sparsity_pct, row_ptr, kv_idx, draft_map)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().bsa_draft_mask(plan.handle, _ptr(q_slots), _ptr(k_slots), sparsity_pct,
                                 _ptr(row_ptr), _ptr(kv_idx), _ptr(draft_map), _ptr(workspace),
                                 nbytes, _stream(stream)), "bsa_draft_mask")


def bsa_draft_mask_noalloc(plan: Plan, q_slots, k_slots, sparsity_pct: int, row_ptr, kv_idx,
                           draft_map, stream=None):
    """bsa_draft_mask without a caller workspace (scratch inside the library)."""
    _need("q_slots", q_slots, _slots(plan))
    _need("k_slots", k_slots, _slots(plan))
    _need_draft_outputs(plan, sparsity_pct, row_ptr, kv_idx, draft_map)
    _check(load().bsa_draft_mask_noalloc(plan.handle, _ptr(q_slots), _ptr(k_slots), sparsity_pct,
                                         _ptr(row_ptr), _ptr(kv_idx), _ptr(draft_map),
                                         _stream(stream)), "bsa_draft_mask_noalloc")


def bsa_draft_noalloc_max_scratch_bytes() -> int:
    return int(load().bsa_draft_noalloc_max_scratch_bytes())


def bsa_reorder_fwd(plan: Plan, x0, y0, x1=None, y1=None, x2=None, y2=None, stream=None):
    for i, (x, y) in enumerate(((x0, y0), (x1, y1), (x2, y2))):
        _need(f"x{i}", x, _natural(plan))
        _need(f"y{i}", y, _slots(plan))
    _check(load().bsa_reorder_fwd(plan.handle, _ptr(x0), _ptr(y0), _ptr(x1), _ptr(y1),
                                  _ptr(x2), _ptr(y2), _stream(stream)), "bsa_reorder_fwd")


def bsa_reorder_inv(plan: Plan, x_slots, x_nat, stream=None):
    _need("x_slots", x_slots, _slots(plan))
    _need("x_nat", x_nat, _natural(plan))
    _check(load().bsa_reorder_inv(plan.handle, _ptr(x_slots), _ptr(x_nat), _stream(stream)),
           "bsa_reorder_inv")


def bsa_attn_fwd(plan: Plan, q, k, v, row_ptr, col_idx, per_head_lists: bool, scale: float,
                 o, lse=None, stream=None):
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _need(name, t, _slots(plan))
    _need("lse", lse, plan.B * plan.Hh * plan.Npad * 4)
    _need_lists(plan, per_head_lists, row_ptr)
    _check(load().bsa_attn_fwd(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr),
                               _ptr(col_idx), int(bool(per_head_lists)), float(scale), _ptr(o),
                               _ptr(lse), _stream(stream)), "bsa_attn_fwd")


def bsa_attn_fwd_natural(plan: Plan, q, k, v, row_ptr, col_idx, per_head_lists: bool,
                         scale: float, o, lse=None, stream=None):
    """bsa_attn_fwd on natural-layout [B, N, Hh, D] tensors (TILE plan, 128-slot tiles)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _need(name, t, _natural(plan))
    _need("lse", lse, _natural(plan, 4) // plan.D)
    _need_lists(plan, per_head_lists, row_ptr)
    _check(load().bsa_attn_fwd_natural(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr),
                                       _ptr(col_idx), int(bool(per_head_lists)), float(scale),
                                       _ptr(o), _ptr(lse), _stream(stream)), "bsa_attn_fwd_natural")


def bsa_draft_mask_natural(plan: Plan, q, k, sparsity_pct: int, row_ptr, kv_idx, draft_map,
                           workspace, stream=None):
    """bsa_draft_mask reading natural-layout q, k directly."""
    _need("q", q, _natural(plan))
    _need("k", k, _natural(plan))
    _need_draft_outputs(plan, sparsity_pct, row_ptr, kv_idx, draft_map)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().bsa_draft_mask_natural(plan.handle, _ptr(q), _ptr(k), sparsity_pct,
                                         _ptr(row_ptr), _ptr(kv_idx), _ptr(draft_map),
                                         _ptr(workspace), nbytes, _stream(stream)),
           "bsa_draft_mask_natural")


def bsa_quantize_e4m3(plan: Plan, q, k, v, q8, k8, v8, scales, stream=None):
    """e4m3 copies of natural-layout q, k, v (uint8 tensors) and their
    per-(tensor, batch, head) scales (float32 [3, B, Hh])."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(name, t, _natural(plan))
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _need(name, t, _natural(plan, 1))
    _need("scales", scales, 3 * plan.B * plan.Hh * 4)
    _check(load().bsa_quantize_e4m3(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8),
                                    _ptr(v8), _ptr(scales), _stream(stream)), "bsa_quantize_e4m3")


def bsa_draft_mask_natural_e4m3(plan: Plan, q, k, v, sparsity_pct: int, row_ptr, kv_idx,
                                draft_map, workspace, q8, k8, v8, scales, stream=None):
    """bsa_draft_mask_natural and bsa_quantize_e4m3 in one call (the pooling
    also takes the maxima of q and k)."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(name, t, _natural(plan))
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _need(name, t, _natural(plan, 1))
    _need("scales", scales, 3 * plan.B * plan.Hh * 4)
    _need_draft_outputs(plan, sparsity_pct, row_ptr, kv_idx, draft_map)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().bsa_draft_mask_natural_e4m3(plan.handle, _ptr(q), _ptr(k), _ptr(v), sparsity_pct,
                                              _ptr(row_ptr), _ptr(kv_idx), _ptr(draft_map),
                                              _ptr(workspace), nbytes, _ptr(q8), _ptr(k8), _ptr(v8),
                                              _ptr(scales), _stream(stream)),
           "bsa_draft_mask_natural_e4m3")


def bsa_attn_fwd_natural_e4m3(plan: Plan, q8, k8, v8, scales, row_ptr, col_idx,
                              per_head_lists: bool, scale: float, o, lse=None, stream=None):
    """bsa_attn_fwd_natural on e4m3 inputs from bsa_quantize_e4m3 (8-bit MMAs)."""
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _need(name, t, _natural(plan, 1))
    _need("o", o, _natural(plan))
    _need("scales", scales, 3 * plan.B * plan.Hh * 4)
    _need("lse", lse, _natural(plan, 4) // plan.D)
    _need_lists(plan, per_head_lists, row_ptr)
    _check(load().bsa_attn_fwd_natural_e4m3(plan.handle, _ptr(q8), _ptr(k8), _ptr(v8),
                                            _ptr(scales), _ptr(row_ptr), _ptr(col_idx),
                                            int(bool(per_head_lists)), float(scale), _ptr(o),
                                            _ptr(lse), _stream(stream)),
           "bsa_attn_fwd_natural_e4m3")


def bsa_lvsa_attn_fwd(plan: Plan, C: int, T_per: int, s: int, q, k, v, scale: float, o,
                      lse=None, stream=None):
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _need(name, t, _natural(plan))
    _need("lse", lse, _natural(plan, 4) // plan.D)
    _check(load().bsa_lvsa_attn_fwd(plan.handle, C, T_per, s, _ptr(q), _ptr(k), _ptr(v),
                                    float(scale), _ptr(o), _ptr(lse), _stream(stream)),
           "bsa_lvsa_attn_fwd")


def bsa_poll_status(plan: Plan, stream=None):
    _check(load().bsa_poll_status(plan.handle, _stream(stream)), "bsa_poll_status")


def bsa_plan_set_lvsa_variant(plan: Plan, anchors: int, window_order: int):
    _check(load().bsa_plan_set_lvsa_variant(plan.handle, int(anchors), int(window_order)),
           "bsa_plan_set_lvsa_variant")


def bsa_plan_set_draft_pooling(plan: Plan, pooling: int):
    _check(load().bsa_plan_set_draft_pooling(plan.handle, int(pooling)),
           "bsa_plan_set_draft_pooling")


def bsa_plan_set_draft_precision(plan: Plan, precision: int):
    _check(load().bsa_plan_set_draft_precision(plan.handle, int(precision)),
           "bsa_plan_set_draft_precision")


def bsa_plan_set_reorder_pads(plan: Plan, pads: int):
    _check(load().bsa_plan_set_reorder_pads(plan.handle, int(pads)), "bsa_plan_set_reorder_pads")


def bsa_set_wait_limit_ns(plan: Plan, ns: int):
    _check(load().bsa_set_wait_limit_ns(plan.handle, int(ns)), "bsa_set_wait_limit_ns")


def bsa_selftest_timeout(plan: Plan, limit_ns: int, stream=None):
    _check(load().bsa_selftest_timeout(plan.handle, int(limit_ns), _stream(stream)),
           "bsa_selftest_timeout")


def bsa_last_error() -> str:
    return load().bsa_last_error().decode()


def bsa_version() -> str:
    return load().bsa_version().decode()
