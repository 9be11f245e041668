"""Ready-made call sequences over the C ABI, with buffers from torch.

LVSA attention ("LVSA: Training-Free Sparse Attention for Long Video
Diffusion", section 2): lvsa_mask(s) -> reorder_fwd(Q,K,V) -> attn_fwd ->
reorder_inv(O), or the one-kernel lvsa_attn_fwd.  Draft attention (Draft
Attention article): reorder_fwd(Q,K,V) -> draft_mask -> attn_fwd ->
reorder_inv(O), or draft_mask_natural -> attn_fwd_natural with no reorder.

torch only allocates device memory and supplies the stream; every step runs
in libbsattn.so.
"""
from __future__ import annotations

import math

import torch

from . import (ANCHORS_ROTATING, DRAFT_FP64, LAYOUT_FRAME, LAYOUT_TILE, PADS_KEEP, PADS_WRITE,
               POOL_MEAN, WINDOW_ALTERNATE, Plan,
               bsa_attn_fwd, bsa_attn_fwd_natural, bsa_attn_fwd_natural_e4m3,
               bsa_draft_keep_count, bsa_draft_mask, bsa_draft_mask_natural,
               bsa_draft_mask_natural_e4m3,
               bsa_draft_workspace_bytes, bsa_quantize_e4m3,
               bsa_lvsa_attn_fwd, bsa_lvsa_mask, bsa_lvsa_nnz, bsa_plan_set_draft_pooling,
               bsa_plan_set_draft_precision, bsa_plan_set_reorder_pads,
               bsa_plan_set_lvsa_variant, bsa_reorder_fwd, bsa_reorder_inv)


class _Base:
    def _alloc_slots(self, device):
        p = self.plan
        shape = (p.B, p.Hh, p.Npad, p.D)
        mk = lambda: torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.q_s, self.k_s, self.v_s, self.o_s = mk(), mk(), mk(), mk()
        self.lse = torch.empty((p.B, p.Hh, p.Npad), dtype=torch.float32, device=device)
        self._pads_zero = False  # the empty slots of q_s, k_s, v_s hold zeros

    def attend(self, per_head: bool):
        bsa_attn_fwd(self.plan, self.q_s, self.k_s, self.v_s, self.row_ptr, self.col_idx,
                     per_head, self.scale, self.o_s, self.lse)

    def gather(self, q, k, v):
        # the slot buffers' empty slots are zeroed by the first gather; later
        # ones write only the tokens (nothing else writes those slots)
        bsa_plan_set_reorder_pads(self.plan, PADS_KEEP if self._pads_zero else PADS_WRITE)
        try:
            bsa_reorder_fwd(self.plan, q, self.q_s, k, self.k_s, v, self.v_s)
        finally:
            bsa_plan_set_reorder_pads(self.plan, PADS_WRITE)
        self._pads_zero = True

    def scatter(self, out):
        bsa_reorder_inv(self.plan, self.o_s, out)
        return out


class LvsaAttention(_Base):
    """LVSA block-sparse attention on the frame layout.  `anchors` and
    `window_order` select a mask variant (bsa_plan_set_lvsa_variant)."""

    def __init__(self, B, Hh, D, T, H, W, C, T_per, block=128, device="cuda", scale=None,
                 anchors=ANCHORS_ROTATING, window_order=WINDOW_ALTERNATE):
        self.plan = Plan(B, Hh, D, T, H, W, LAYOUT_FRAME, block=block)
        bsa_plan_set_lvsa_variant(self.plan, anchors, window_order)
        self.C, self.T_per = C, T_per
        self.scale = scale if scale is not None else 1.0 / math.sqrt(D)
        nnz = bsa_lvsa_nnz(self.plan, C)
        self.frame_sets = torch.empty(T * C, dtype=torch.int32, device=device)
        self.row_ptr = torch.empty(self.plan.nblocks + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(nnz, dtype=torch.int32, device=device)
        self._alloc_slots(device)

    def mask(self, s: int):
        bsa_lvsa_mask(self.plan, self.C, self.T_per, s, self.frame_sets, self.row_ptr,
                      self.col_idx)

    def __call__(self, q, k, v, s: int, out=None):
        out = torch.empty_like(q) if out is None else out
        self.mask(s)
        self.gather(q, k, v)
        self.attend(per_head=False)
        return self.scatter(out)

    def fused(self, q, k, v, s: int, out=None, lse=None):
        """The same attention in one kernel on the natural layout."""
        out = torch.empty_like(q) if out is None else out
        bsa_lvsa_attn_fwd(self.plan, self.C, self.T_per, s, q, k, v, self.scale, out, lse)
        return out


class DraftAttention(_Base):
    """Draft-mask block-sparse attention on the tile layout.  `pooling`:
    POOL_MEAN (the article's average) or POOL_MAX; `precision`: DRAFT_FP64
    or DRAFT_FP32 draft logits."""

    def __init__(self, B, Hh, D, T, H, W, pool_h, pool_w, sparsity_pct, device="cuda",
                 scale=None, want_map=False, pooling=POOL_MEAN, precision=DRAFT_FP64):
        self.plan = Plan(B, Hh, D, T, H, W, LAYOUT_TILE, pool_h, pool_w, pool_h * pool_w)
        bsa_plan_set_draft_pooling(self.plan, pooling)
        bsa_plan_set_draft_precision(self.plan, precision)
        self.sparsity = sparsity_pct
        self.scale = scale if scale is not None else 1.0 / math.sqrt(D)
        self.keep = bsa_draft_keep_count(self.plan, sparsity_pct)
        rows = B * Hh * self.plan.nblocks
        self.row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(rows * self.keep, dtype=torch.int32, device=device)
        self.draft_map = (torch.empty(rows * self.plan.nblocks, dtype=torch.float32,
                                      device=device) if want_map else None)
        nbytes = bsa_draft_workspace_bytes(self.plan)
        self.workspace = torch.empty((nbytes + 7) // 8, dtype=torch.float64, device=device)
        self._alloc_slots(device)

    def mask(self):
        bsa_draft_mask(self.plan, self.q_s, self.k_s, self.sparsity, self.row_ptr, self.col_idx,
                       self.draft_map, self.workspace)

    def __call__(self, q, k, v, out=None):
        out = torch.empty_like(q) if out is None else out
        self.gather(q, k, v)
        self.mask()
        self.attend(per_head=True)
        return self.scatter(out)

    def fused(self, q, k, v, out=None, lse=None):
        """The same attention with no reorder: the draft mask pools the
        natural layout in place and the attention reads and writes it
        through tile-shaped tensor maps (pool_h * pool_w must be 128)."""
        out = torch.empty_like(q) if out is None else out
        bsa_draft_mask_natural(self.plan, q, k, self.sparsity, self.row_ptr, self.col_idx,
                               self.draft_map, self.workspace)
        bsa_attn_fwd_natural(self.plan, q, k, v, self.row_ptr, self.col_idx, True, self.scale,
                             out, lse)
        return out

    def _e4m3_buffers(self, q):
        if getattr(self, "q8", None) is None or self.q8.shape != q.shape:
            self.q8, self.k8, self.v8 = (torch.empty(q.shape, dtype=torch.uint8, device=q.device)
                                         for _ in range(3))
            p = self.plan
            self.fp8_scales = torch.empty((3, p.B, p.Hh), dtype=torch.float32, device=q.device)

    def quantize(self, q, k, v):
        """e4m3 copies of q, k, v and their per-(tensor, batch, head) scales."""
        self._e4m3_buffers(q)
        bsa_quantize_e4m3(self.plan, q, k, v, self.q8, self.k8, self.v8, self.fp8_scales)

    def mask_and_quantize(self, q, k, v):
        """The draft mask from the bf16 Q and K and the e4m3 copies of Q, K, V
        in one call (the pooling also takes the maxima of Q and K)."""
        self._e4m3_buffers(q)
        bsa_draft_mask_natural_e4m3(self.plan, q, k, v, self.sparsity, self.row_ptr, self.col_idx,
                                    self.draft_map, self.workspace, self.q8, self.k8, self.v8,
                                    self.fp8_scales)

    def fused_e4m3(self, q, k, v, out=None, lse=None):
        """fused() with 8-bit attention: the draft mask from the bf16 Q and K,
        Q, K, V quantized to e4m3, then attended with 8-bit MMAs."""
        out = torch.empty_like(q) if out is None else out
        self.mask_and_quantize(q, k, v)
        bsa_attn_fwd_natural_e4m3(self.plan, self.q8, self.k8, self.v8, self.fp8_scales,
                                  self.row_ptr, self.col_idx, True, self.scale, out, lse)
        return out


class StreamedSteps:
    """Runs attention steps whose inputs and outputs live in pinned host
    memory, overlapping transfers with compute: step i+1's host-to-device
    copies and step i-1's device-to-host read run on their own streams while
    step i computes.  Two device buffer sets; every step still moves all of
    its inputs in and its output out.

        steps = StreamedSteps(shape, torch.bfloat16)
        steps.run(lambda q, k, v, out, i: att.fused(q, k, v, i, out),
                  host_inputs=(hq, hk, hv), host_output=ho, n=10)
    """

    def __init__(self, shape, dtype, device="cuda"):
        mk = lambda: torch.empty(shape, dtype=dtype, device=device)
        self.bufs = [[mk() for _ in range(4)] for _ in range(2)]  # q, k, v, out per set
        self.h2d = torch.cuda.Stream(device)
        self.d2h = torch.cuda.Stream(device)

    def run(self, fn, host_inputs, host_output, n: int):
        """Enqueue n steps; returns (start, end) CUDA events around all of them.
        host_inputs: pinned (q, k, v) copied in for every step; host_output:
        pinned tensor that receives every step's output."""
        compute = torch.cuda.current_stream()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of a set copied
        ev_done = [torch.cuda.Event() for _ in range(2)]   # step on a set computed
        ev_out = [torch.cuda.Event() for _ in range(2)]    # output of a set read back
        start.record(compute)
        self.h2d.wait_event(start)
        self.d2h.wait_event(start)
        for i in range(n):
            b = i % 2
            q, k, v, out = self.bufs[b]
            with torch.cuda.stream(self.h2d):
                if i >= 2:
                    self.h2d.wait_event(ev_done[b])        # inputs of step i-2 consumed
                for dst, src in zip((q, k, v), host_inputs):
                    dst.copy_(src, non_blocking=True)
                ev_in[b].record(self.h2d)
            compute.wait_event(ev_in[b])
            if i >= 2:
                compute.wait_event(ev_out[b])              # output of step i-2 read back
            fn(q, k, v, out, i)
            ev_done[b].record(compute)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(ev_done[b])
                host_output.copy_(out, non_blocking=True)
                ev_out[b].record(self.d2h)
        compute.wait_stream(self.d2h)
        end.record(compute)
        return start, end
