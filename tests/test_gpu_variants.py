"""Parity of the mask variants with the fp64 oracle.

LVSA ("LVSA: Training-Free Sparse Attention for Long Video Diffusion",
section 2): fixed-grid anchors and no anchors (sliding window) beside the
rotating grid, and the alternating growth order of the extended window beside
the distance order.  Draft Attention article: max pooling beside average
pooling.  Frame sets, block lists, pooled values and kept blocks: bit-exact.
Attention: max-abs <= 2e-2, mean-abs <= 2e-3, LSE within 2e-3 against fp64.
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

from gpu_util import LSE_ABS, MAX_ABS, MEAN_ABS, sample_blocks, to_np64

pytestmark = pytest.mark.gpu

ANCHORS = {"rotating": bsa.ANCHORS_ROTATING, "fixed": bsa.ANCHORS_FIXED, "none": bsa.ANCHORS_NONE}
ORDERS = {"distance": bsa.WINDOW_DISTANCE, "alternate": bsa.WINDOW_ALTERNATE}
VARIANTS = [("fixed", "distance"), ("none", "distance"), ("rotating", "alternate"),
            ("fixed", "alternate"), ("none", "alternate")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    bsa.load()


# ------------------------------------------------------------------ masks
@pytest.mark.parametrize("cid", [1, 3, 4])
@pytest.mark.parametrize("anchors,order", VARIANTS)
def test_lvsa_mask_variants_bit_exact(cid, anchors, order):
    w = CONFIGS[cid]
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=w.lvsa_block)
    bsa.bsa_plan_set_lvsa_variant(plan, ANCHORS[anchors], ORDERS[order])
    nbf = -(-w.P // w.lvsa_block)
    fs = torch.empty(w.T * w.lvsa_C, dtype=torch.int32, device="cuda")
    rp = torch.empty(plan.nblocks + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty(bsa.bsa_lvsa_nnz(plan, w.lvsa_C), dtype=torch.int32, device="cuda")
    for s in (0, 1, w.lvsa_T_per - 1, w.lvsa_T_per + 2):
        bsa.bsa_lvsa_mask(plan, w.lvsa_C, w.lvsa_T_per, s, fs, rp, ci)
        bsa.bsa_poll_status(plan)
        A = oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, s, anchors, order)
        rpo, cio = oracle.lvsa_block_csr(A, nbf)
        np.testing.assert_array_equal(fs.cpu().numpy().reshape(w.T, w.lvsa_C), A)
        np.testing.assert_array_equal(rp.cpu().numpy(), rpo)
        np.testing.assert_array_equal(ci.cpu().numpy(), cio)


def test_lvsa_mask_variants_small_grids_every_budget():
    # every feasible C on short videos, both orders, all anchor modes: the
    # closed forms in the kernel against the oracle's loops
    for T in (1, 2, 5, 9, 13):
        plan = bsa.Plan(1, 1, 64, T, 1, 64, bsa.LAYOUT_FRAME, block=64)
        for anchors, order in VARIANTS + [("rotating", "distance")]:
            bsa.bsa_plan_set_lvsa_variant(plan, ANCHORS[anchors], ORDERS[order])
            for T_per in (1, 3, 4):
                for s in range(T_per):
                    base = len(oracle.lvsa_anchors(T, T_per, s, anchors))
                    for C in range(1, T + 1):
                        if base + (base < T) > C:
                            continue
                        fs = torch.empty(T * C, dtype=torch.int32, device="cuda")
                        rp = torch.empty(T + 1, dtype=torch.int32, device="cuda")
                        ci = torch.empty(T * C, dtype=torch.int32, device="cuda")
                        bsa.bsa_lvsa_mask(plan, C, T_per, s, fs, rp, ci)
                        A = oracle.lvsa_frame_sets(T, C, T_per, s, anchors, order)
                        np.testing.assert_array_equal(fs.cpu().numpy().reshape(T, C), A,
                                                      err_msg=f"{T} {C} {T_per} {s} {anchors} {order}")
        bsa.bsa_poll_status(plan)


def test_variant_setters_reject_unknown_values():
    plan = bsa.Plan(1, 1, 64, 8, 8, 8, bsa.LAYOUT_FRAME, block=64)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_plan_set_lvsa_variant(plan, 3, 0)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_plan_set_lvsa_variant(plan, 0, 2)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_plan_set_draft_pooling(plan, 2)


def test_window_only_accepts_budgets_that_rotating_anchors_rule_out():
    # 8 frames, T_per 4: rotating anchors need C >= 3; with no anchors C = 1 works
    plan = bsa.Plan(1, 1, 64, 8, 8, 8, bsa.LAYOUT_FRAME, block=64)
    rp = torch.empty(9, dtype=torch.int32, device="cuda")
    ci = torch.empty(8, dtype=torch.int32, device="cuda")
    with pytest.raises(bsa.BsaError):
        bsa.bsa_lvsa_mask(plan, 1, 4, 0, None, rp, ci)
    bsa.bsa_plan_set_lvsa_variant(plan, bsa.ANCHORS_NONE, bsa.WINDOW_DISTANCE)
    fs = torch.empty(8, dtype=torch.int32, device="cuda")
    bsa.bsa_lvsa_mask(plan, 1, 4, 0, fs, rp, ci)
    bsa.bsa_poll_status(plan)
    assert fs.cpu().tolist() == list(range(8))
    assert ci.cpu().tolist() == list(range(8)) and rp.cpu().tolist() == list(range(9))


# ------------------------------------------------------------------ fused LVSA attention
def _fused(w, C, T_per, s, q, k, v, anchors, order):
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=128)
    bsa.bsa_plan_set_lvsa_variant(plan, ANCHORS[anchors], ORDERS[order])
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.Hh, w.N), float("nan"), dtype=torch.float32, device="cuda")
    bsa.bsa_lvsa_attn_fwd(plan, C, T_per, s, q, k, v, 1 / math.sqrt(w.D), o, lse)
    bsa.bsa_poll_status(plan)
    return o, lse


def _oracle_natural(w, C, T_per, s, q, k, v, heads, anchors, order, q_blocks=None):
    blk = 128
    nbf = -(-w.P // blk)
    perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, blk)
    valid = oracle.slot_valid(perm, Np)
    rp, ci = oracle.lvsa_block_csr(oracle.lvsa_frame_sets(w.T, C, T_per, s, anchors, order), nbf)
    sub = lambda x: oracle.reorder_fwd(to_np64(x[:, :, heads]), perm, Np)
    O, L = oracle.masked_attention(sub(q), sub(k), sub(v), valid, blk, rp, ci, False,
                                   1 / math.sqrt(w.D), q_blocks=q_blocks)
    return oracle.reorder_inv(O, perm), L[:, :, perm]


def _check(o, lse, On, Ln, heads):
    got = to_np64(o[:, :, heads])
    m = np.isfinite(On)
    assert m.any()
    err = np.abs(got[m] - On[m])
    assert err.max() <= MAX_ABS, err.max()
    assert err.mean() <= MEAN_ABS, err.mean()
    lg = lse[:, heads].double().cpu().numpy()
    fin = np.isfinite(Ln)
    assert np.abs(lg[fin] - Ln[fin]).max() <= LSE_ABS


@pytest.mark.parametrize("anchors,order", VARIANTS)
def test_fused_variants_tiny_all_tokens(anchors, order):
    w = CONFIGS[1]
    q, k, v = (x.cuda() for x in make_qkv(w))
    heads = list(range(w.Hh))
    for s in (0, 3):
        o, lse = _fused(w, w.lvsa_C, w.lvsa_T_per, s, q, k, v, anchors, order)
        On, Ln = _oracle_natural(w, w.lvsa_C, w.lvsa_T_per, s, q, k, v, heads, anchors, order)
        _check(o, lse, On, Ln, heads)


@pytest.mark.parametrize("anchors,order", [("rotating", "alternate"), ("none", "distance")])
def test_fused_variants_ragged_frames(anchors, order):
    # 63-token frames and key tiles that overhang into the next run of frames
    w = small_workload(CONFIGS[1], T=9, H=7, W=9, Hh=2, D=64)
    q, k, v = (x.cuda() for x in make_qkv(w))
    for s in (0, 1):
        o, lse = _fused(w, 5, 3, s, q, k, v, anchors, order)
        On, Ln = _oracle_natural(w, 5, 3, s, q, k, v, [0, 1], anchors, order)
        _check(o, lse, On, Ln, [0, 1])


@pytest.mark.parametrize("anchors,order,s", [("rotating", "alternate", 5), ("fixed", "distance", 7),
                                             ("none", "alternate", 0)])
def test_fused_variants_full_size_sampled(anchors, order, s):
    w = CONFIGS[3]
    q, k, v = make_qkv(w, device="cuda")
    o, lse = _fused(w, w.lvsa_C, w.lvsa_T_per, s, q, k, v, anchors, order)
    nb = w.T * -(-w.P // 128)
    heads = [0, w.Hh - 1]
    On, Ln = _oracle_natural(w, w.lvsa_C, w.lvsa_T_per, s, q, k, v, heads, anchors, order,
                             q_blocks=sample_blocks(nb, 6, seed=s + 11))
    _check(o, lse, On, Ln, heads)
    assert torch.isfinite(o).all()


def test_unfused_pipeline_variant_matches_fused():
    w = small_workload(CONFIGS[3], T=20, Hh=2, field_grid=(20, 4, 7))
    q, k, v = make_qkv(w, device="cuda")
    att = LvsaAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, 9, 6, block=128,
                        anchors=bsa.ANCHORS_ROTATING, window_order=bsa.WINDOW_ALTERNATE)
    a = att(q, k, v, 2)
    b = att.fused(q, k, v, 2)
    bsa.bsa_poll_status(att.plan)
    d = (a.float() - b.float()).abs()
    assert d.max().item() <= 3e-2 and d.mean().item() <= 1e-3


# ------------------------------------------------------------------ draft max pooling
def _slots_gpu(x_nat, perm, Npad):
    B, N, Hh, D = x_nat.shape
    out = torch.zeros((B, Hh, Npad, D), dtype=x_nat.dtype, device="cuda")
    out[:, :, torch.from_numpy(perm).cuda()] = x_nat.cuda().permute(0, 2, 1, 3)
    return out


@pytest.mark.parametrize("over", [dict(cid=1), dict(cid=2),
                                  dict(cid=1, T=3, H=5, W=7, Hh=3, D=128, qk="iid", draft_ph=4,
                                       draft_pw=4, draft_sparsity=70)])
@pytest.mark.parametrize("noalloc", [False, True])
def test_draft_max_pool_bit_exact(over, noalloc):
    over = dict(over)
    w = small_workload(CONFIGS[over.pop("cid")], **over)
    ph, pw, sp = w.draft_ph, w.draft_pw, w.draft_sparsity
    q, k, _ = make_qkv(w)
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, ph, pw, ph * pw)
    bsa.bsa_plan_set_draft_pooling(plan, bsa.POOL_MAX)
    perm, _ = oracle.tile_layout_perm(w.T, w.H, w.W, ph, pw)
    qs, ks = _slots_gpu(q, perm, plan.Npad), _slots_gpu(k, perm, plan.Npad)
    keep = bsa.bsa_draft_keep_count(plan, sp)
    nb = plan.nblocks
    rows = w.B * w.Hh * nb
    rp = torch.empty(rows + 1, dtype=torch.int32, device="cuda")
    kv = torch.empty(rows * keep, dtype=torch.int32, device="cuda")
    qn, kn = to_np64(q), to_np64(k)
    qbar = oracle.draft_pool(qn, w.T, w.H, w.W, ph, pw, "max")
    kbar = oracle.draft_pool(kn, w.T, w.H, w.W, ph, pw, "max")
    if noalloc:
        bsa.bsa_draft_mask_noalloc(plan, qs, ks, sp, rp, kv, None)
    else:
        ws = torch.full(((bsa.bsa_draft_workspace_bytes(plan) + 7) // 8,), float("nan"),
                        dtype=torch.float64, device="cuda")
        bsa.bsa_draft_mask(plan, qs, ks, sp, rp, kv, None, ws)
        got = ws.cpu().numpy()[:2 * rows * w.D].reshape(2, w.B, w.Hh, nb, w.D)
        np.testing.assert_array_equal(got[0], qbar)
        np.testing.assert_array_equal(got[1], kbar)
    bsa.bsa_poll_status(plan)
    ref = oracle.draft_topk(oracle.draft_logits(qbar, kbar), oracle.draft_keep_count(nb, sp))
    np.testing.assert_array_equal(kv.cpu().numpy().reshape(w.B, w.Hh, nb, keep), ref)


def test_draft_pipeline_max_pool_tiny():
    w = CONFIGS[1]
    q, k, v = make_qkv(w)
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity,
                         pooling=bsa.POOL_MAX)
    out = att(q.cuda(), k.cuda(), v.cuda())
    bsa.bsa_poll_status(att.plan)
    ph, pw = w.draft_ph, w.draft_pw
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, ph, pw)
    valid = oracle.slot_valid(perm, Np)
    qn, kn, vn = (to_np64(x) for x in (q, k, v))
    kv = oracle.draft_blocks(qn, kn, w.T, w.H, w.W, ph, pw, w.draft_sparsity, "max")
    nb = Np // (ph * pw)
    np.testing.assert_array_equal(att.col_idx.view(w.B, w.Hh, nb, -1).cpu().numpy(), kv)
    # max pooling keeps different blocks than the mean on this input
    assert not np.array_equal(kv, oracle.draft_blocks(qn, kn, w.T, w.H, w.W, ph, pw,
                                                      w.draft_sparsity))
    rp, ci = oracle.fixed_k_csr(kv)
    O, _ = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Np) for x in (qn, kn, vn)),
                                   valid, ph * pw, rp, ci, True, 1 / math.sqrt(w.D))
    ref = oracle.reorder_inv(O, perm)
    err = np.abs(to_np64(out) - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS
