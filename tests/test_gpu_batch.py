"""Batch size 2 through every path (the five workloads all have B = 1).

The natural-layout kernels address batch b through the token row b*N + n
and the frame b*T + t of their tensor maps; the slot-layout kernels through
(b*Hh + h)*Npad; the block lists through b*Hh + h.  Each path is compared
with the fp64 oracle (within max-abs 2e-2 / mean-abs 2e-3; 3e-2 / 3e-3 for
the 8-bit path) and, where a batch is just two independent problems, with
the same call on each batch alone (bit for bit).
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_49_b200 as bsa
import oracle
from block_sparse_attention_49_b200 import _build
from block_sparse_attention_49_b200.pipeline import DraftAttention, LvsaAttention
from synth import CONFIGS, make_qkv, small_workload

from gpu_util import to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    bsa.load()


def _check(got, ref, max_abs=2e-2, mean_abs=2e-3):
    m = np.isfinite(ref)
    assert m.any()
    err = np.abs(to_np64(got)[m] - ref[m])
    assert err.max() <= max_abs and err.mean() <= mean_abs, (err.max(), err.mean())


def _lvsa_ref(w, C, T_per, s, q, k, v):
    perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, 128)
    A = oracle.lvsa_frame_sets(w.T, C, T_per, s)
    rp, ci = oracle.lvsa_block_csr(A, -(-w.P // 128))
    O, _ = oracle.masked_attention(*(oracle.reorder_fwd(to_np64(x), perm, Np) for x in (q, k, v)),
                                   oracle.slot_valid(perm, Np), 128, rp, ci, False,
                                   1 / math.sqrt(w.D))
    return oracle.reorder_inv(O, perm)


def test_lvsa_fused_and_four_kernel_batch_of_two():
    w = small_workload(CONFIGS[1], B=2, T=6, H=9, W=15, Hh=2, D=64)
    q, k, v = make_qkv(w, device="cuda")
    att = LvsaAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, 4, 3, block=128)
    ref = _lvsa_ref(w, 4, 3, 1, q, k, v)
    fused = att.fused(q, k, v, 1)
    four = att(q, k, v, 1)
    bsa.bsa_poll_status(att.plan)
    _check(fused, ref)
    _check(four, ref)
    # batch 1 alone gives the same bits as inside the batch of two
    one = LvsaAttention(1, w.Hh, w.D, w.T, w.H, w.W, 4, 3, block=128).fused(
        q[1:].contiguous(), k[1:].contiguous(), v[1:].contiguous(), 1)
    assert torch.equal(one.view(torch.int16), fused[1:].view(torch.int16))


def _draft_ref(w, q, k, v, kv):
    ph, pw = w.draft_ph, w.draft_pw
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, ph, pw)
    rp, ci = oracle.fixed_k_csr(kv)
    O, _ = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Np) for x in (q, k, v)),
                                   oracle.slot_valid(perm, Np), ph * pw, rp, ci, True,
                                   1 / math.sqrt(w.D))
    return oracle.reorder_inv(O, perm)


def test_draft_paths_batch_of_two():
    w = small_workload(CONFIGS[2], B=2, T=2, H=13, W=37, Hh=2, field_grid=(2, 4, 7))
    q, k, v = make_qkv(w, device="cuda")
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    slots = att(q, k, v)
    kv_slots = att.col_idx.clone()
    nat = att.fused(q, k, v)
    bsa.bsa_poll_status(att.plan)
    assert torch.equal(att.col_idx, kv_slots)
    qn, kn, vn = (to_np64(x) for x in (q, k, v))
    kv = oracle.draft_blocks(qn, kn, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    nb = kv.shape[2]
    np.testing.assert_array_equal(att.col_idx.view(w.B, w.Hh, nb, -1).cpu().numpy(), kv)
    ref = _draft_ref(w, qn, kn, vn, kv)
    _check(nat, ref)
    _check(slots, ref)
    # batch 1 alone gives the same bits as inside the batch of two
    one = DraftAttention(1, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    nat1 = one.fused(q[1:].contiguous(), k[1:].contiguous(), v[1:].contiguous())
    bsa.bsa_poll_status(one.plan)
    assert torch.equal(nat1.view(torch.int16), nat[1:].view(torch.int16))


def test_e4m3_path_batch_of_two():
    w = small_workload(CONFIGS[2], B=2, T=2, H=13, W=37, Hh=2, field_grid=(2, 4, 7))
    q0, k0, v = make_qkv(w, device="cuda")
    # different scales per batch with the same attention: Q x 4 and K / 4 in
    # batch 1 (exact in bf16, so the scores are unchanged)
    q = torch.cat([q0[:1], q0[1:] * 4.0])
    k = torch.cat([k0[:1], k0[1:] * 0.25])
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    out8 = att.fused_e4m3(q, k, v)
    bsa.bsa_poll_status(att.plan)
    sc = att.fp8_scales.cpu().numpy()
    for i, x in enumerate((q, k, v)):
        np.testing.assert_array_equal(sc[i], oracle.fp8_scales(to_np64(x)))
    # batch 1's codes are those of its unscaled data (the scales moved by 4)
    plan1 = bsa.Plan(1, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, w.draft_ph, w.draft_pw,
                     w.draft_ph * w.draft_pw)
    x1 = [q0[1:].contiguous(), k0[1:].contiguous(), v[1:].contiguous()]
    y1 = [torch.empty(x.shape, dtype=torch.uint8, device="cuda") for x in x1]
    s1 = torch.empty((3, 1, w.Hh), dtype=torch.float32, device="cuda")
    bsa.bsa_quantize_e4m3(plan1, *x1, *y1, s1)
    bsa.bsa_poll_status(plan1)
    assert torch.equal(y1[0], att.q8[1:]) and torch.equal(y1[1], att.k8[1:])
    deq = [oracle.fp8_dequantize(x8.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy(),
                                 sc[i]) for i, x8 in enumerate((att.q8, att.k8, att.v8))]
    nb = att.plan.nblocks
    kv = att.col_idx.view(w.B, w.Hh, nb, -1).cpu().numpy()
    _check(out8, _draft_ref(w, *deq, kv), 3e-2, 3e-3)
