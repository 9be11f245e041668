"""The draft path on the natural layout (no reorder): bsa_draft_mask_natural
and bsa_attn_fwd_natural.

Draft Attention article: pooled Q and K give the draft map and the kept
blocks; the reorder that makes the kept blocks contiguous is fused into the
attention's tile loads and stores here.  Pooled values and kept blocks:
bit-exact against the oracle.  Attention: within max-abs 2e-2 / mean-abs
2e-3 of the fp64 oracle (LSE within 2e-3), on grids whose edges leave
partial tiles (the kernel packs those key tiles several to an MMA tile) and
on lists too long to pack; it is identical, bit for bit, to the reorder +
attn_fwd + reorder_inv path, whose attention packs the same tiles.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_49_b200 as bsa
import oracle
from block_sparse_attention_49_b200 import _build
from block_sparse_attention_49_b200.pipeline import DraftAttention
from synth import CONFIGS, make_qkv, small_workload

from gpu_util import MAX_ABS, MEAN_ABS, sample_blocks, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    bsa.load()


CASES = [
    dict(cid=2),                                                        # 30 x 52 grid, 8 x 16 tiles
    dict(cid=5, Hh=6),                                                  # 40-head workload, 6 heads
    dict(cid=2, T=3, H=13, W=37, Hh=3, field_grid=(3, 4, 7)),          # ragged edges both ways
    dict(cid=2, T=2, H=20, W=12, Hh=2, D=64, draft_ph=16, draft_pw=8,  # transposed tile, D = 64
         field_grid=(2, 4, 7)),
    dict(cid=2, T=2, H=9, W=70, Hh=2, draft_ph=4, draft_pw=32, draft_sparsity=70,
         field_grid=(2, 4, 7)),
]


@pytest.mark.parametrize("over", CASES)
@pytest.mark.parametrize("pooling", [bsa.POOL_MEAN, bsa.POOL_MAX])
@pytest.mark.parametrize("precision", [bsa.DRAFT_FP64, bsa.DRAFT_FP32])
def test_draft_mask_natural_bit_exact(over, pooling, precision):
    over = dict(over)
    w = small_workload(CONFIGS[over.pop("cid")], **over)
    ph, pw, sp = w.draft_ph, w.draft_pw, w.draft_sparsity
    q, k, _ = make_qkv(w, device="cuda")
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, ph, pw, ph * pw)
    bsa.bsa_plan_set_draft_pooling(plan, pooling)
    bsa.bsa_plan_set_draft_precision(plan, precision)
    keep = bsa.bsa_draft_keep_count(plan, sp)
    nb = plan.nblocks
    rows = w.B * w.Hh * nb
    rp = torch.empty(rows + 1, dtype=torch.int32, device="cuda")
    kv = torch.empty(rows * keep, dtype=torch.int32, device="cuda")
    dt, npdt = ((torch.float64, np.float64) if precision == bsa.DRAFT_FP64
                else (torch.float32, np.float32))
    nbytes = bsa.bsa_draft_workspace_bytes(plan)
    # fp32: the pooled values; fp64: the pooled values, their fp32 copies
    # and one norm per pooled vector
    assert nbytes == (2 * rows * w.D * 4 if precision == bsa.DRAFT_FP32
                      else 2 * rows * w.D * 12 + 2 * rows * 4)
    ws = torch.full((nbytes // np.dtype(npdt).itemsize,), float("nan"), dtype=dt, device="cuda")
    bsa.bsa_draft_mask_natural(plan, q, k, sp, rp, kv, None, ws)
    bsa.bsa_poll_status(plan)
    mode = "max" if pooling == bsa.POOL_MAX else "mean"
    qbar = oracle.draft_pool(to_np64(q), w.T, w.H, w.W, ph, pw, mode)
    kbar = oracle.draft_pool(to_np64(k), w.T, w.H, w.W, ph, pw, mode)
    got = ws.cpu().numpy()[:2 * rows * w.D].reshape(2, w.B, w.Hh, nb, w.D)
    # the fp64 sum and division, rounded once to fp32 in FP32 precision
    np.testing.assert_array_equal(got[0], qbar.astype(npdt))
    np.testing.assert_array_equal(got[1], kbar.astype(npdt))
    prec = "fp64" if precision == bsa.DRAFT_FP64 else "fp32"
    ref = oracle.draft_topk(oracle.draft_logits(qbar, kbar, prec), oracle.draft_keep_count(nb, sp))
    np.testing.assert_array_equal(kv.cpu().numpy().reshape(w.B, w.Hh, nb, keep), ref)


def _oracle_natural(w, q, k, v, kv_gpu, heads, q_blocks=None):
    """fp64 oracle attention on the natural layout for the given heads (and
    query blocks), with the kept blocks the GPU chose (checked separately)."""
    ph, pw = w.draft_ph, w.draft_pw
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, ph, pw)
    valid = oracle.slot_valid(perm, Np)
    qn, kn, vn = (to_np64(x[:, :, heads]) for x in (q, k, v))
    rp, ci = oracle.fixed_k_csr(kv_gpu[:, heads])
    O, LSE = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Np) for x in (qn, kn, vn)),
                                     valid, ph * pw, rp, ci, True, 1 / math.sqrt(w.D),
                                     q_blocks=q_blocks)
    return (oracle.reorder_inv(np.nan_to_num(O, nan=np.inf), perm),
            np.nan_to_num(LSE, nan=np.inf)[:, :, perm])


@pytest.mark.parametrize("over", CASES)
def test_attn_natural_matches_oracle_and_reorder_path(over):
    # grids with partial edge tiles: both paths pack the kept edge key
    # tiles several to an MMA tile, in the same order (the reorder path's
    # attention loads the valid slots of each piece from the slot tensors),
    # so besides matching the oracle they agree bit for bit
    over = dict(over)
    w = small_workload(CONFIGS[over.pop("cid")], **over)
    q, k, v = make_qkv(w, device="cuda")
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    a = att(q, k, v)
    kv_a = att.col_idx.clone()
    b = torch.full_like(q, float("nan"))
    lse_nat = torch.full((w.B, w.Hh, w.N), float("nan"), dtype=torch.float32, device="cuda")
    att.fused(q, k, v, b, lse_nat)
    bsa.bsa_poll_status(att.plan)
    assert torch.equal(att.col_idx, kv_a)                        # same kept blocks
    nb = att.plan.nblocks
    kv = att.col_idx.view(w.B, w.Hh, nb, -1).cpu().numpy()
    heads = sorted({0, w.Hh - 1})
    small = w.N * w.Hh <= 200_000
    ref, ref_lse = _oracle_natural(w, q, k, v, kv, heads,
                                   None if small else sample_blocks(nb, 6, seed=w.N))
    got = to_np64(b[:, :, heads])
    m = np.isfinite(ref)
    err = np.abs(got[m] - ref[m])
    assert m.any() and err.max() <= MAX_ABS and err.mean() <= MEAN_ABS
    lse = lse_nat[:, heads].cpu().numpy().astype(np.float64)
    ml = np.isfinite(ref_lse)
    assert np.abs(lse[ml] - ref_lse[ml]).max() <= 2e-3
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))  # the two GPU paths agree
    perm, _ = oracle.tile_layout_perm(w.T, w.H, w.W, w.draft_ph, w.draft_pw)
    assert torch.equal(att.lse[:, :, torch.from_numpy(perm).cuda()], lse_nat)


def test_attn_natural_equals_reorder_path_bitwise_without_edge_tiles():
    # 8 x 16 tiles dividing a 16 x 32 grid: no partial tiles, nothing to
    # pack, so the natural-layout kernel does the reorder path's arithmetic
    # on the same tiles: the same bits on every token
    w = small_workload(CONFIGS[2], T=3, H=16, W=32, Hh=2, field_grid=(3, 4, 7))
    q, k, v = make_qkv(w, device="cuda")
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, 8, 16, 50)
    a = att(q, k, v)
    lse_slots = att.lse.clone()
    b = torch.full_like(q, float("nan"))
    lse_nat = torch.full((w.B, w.Hh, w.N), float("nan"), dtype=torch.float32, device="cuda")
    att.fused(q, k, v, b, lse_nat)
    bsa.bsa_poll_status(att.plan)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    perm, _ = oracle.tile_layout_perm(w.T, w.H, w.W, 8, 16)
    assert torch.equal(lse_slots[:, :, torch.from_numpy(perm).cuda()], lse_nat)


def test_attn_natural_long_lists_run_unpacked():
    # 792 key blocks, all kept (sparsity 0): lists longer than a CTA packs
    # run tile by tile; sampled query blocks against the oracle
    w = small_workload(CONFIGS[2], T=11, H=90, W=90, Hh=1, D=64, draft_sparsity=0,
                       field_grid=(11, 4, 7))
    q, k, v = make_qkv(w, device="cuda")
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, 8, 16, 0)
    assert att.plan.nblocks == 792 and att.keep == 792
    out = att.fused(q, k, v)
    bsa.bsa_poll_status(att.plan)
    kv = att.col_idx.view(1, 1, 792, -1).cpu().numpy()
    assert (kv == np.arange(792)).all()
    ref, _ = _oracle_natural(w, q, k, v, kv, [0], q_blocks=[0, 71, 400, 791])
    got = to_np64(out)
    m = np.isfinite(ref)
    err = np.abs(got[m] - ref[m])
    assert m.any() and err.max() <= MAX_ABS and err.mean() <= MEAN_ABS


@pytest.mark.parametrize("T", [256, 300])
def test_attn_natural_lists_at_and_past_the_bin_limit(T):
    # a 6 x 10 frame is one corner tile of 60 tokens (8 x 16 tiles): two
    # pieces fit a 128-row MMA tile, so a list keeping every block of T
    # frames needs T / 2 packed tiles - 128 at T = 256, the most a list
    # buffer holds, and 150 at T = 300, where the list runs unpacked
    w = small_workload(CONFIGS[2], T=T, H=6, W=10, Hh=1, D=64, draft_sparsity=0,
                       field_grid=(16, 2, 3))
    q, k, v = make_qkv(w, device="cuda")
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, 8, 16, 0)
    assert att.plan.nblocks == T and att.keep == T
    out = att.fused(q, k, v)
    bsa.bsa_poll_status(att.plan)
    kv = att.col_idx.view(1, 1, T, -1).cpu().numpy()
    assert (kv == np.arange(T)).all()
    ref, _ = _oracle_natural(w, q, k, v, kv, [0], q_blocks=[0, 1, T // 2, T - 1])
    got = to_np64(out)
    m = np.isfinite(ref)
    err = np.abs(got[m] - ref[m])
    assert m.any() and err.max() <= MAX_ABS and err.mean() <= MEAN_ABS


@pytest.mark.parametrize("cid", [2, 5])
def test_attn_natural_full_size_sampled_vs_oracle(cid):
    w = CONFIGS[cid]
    q, k, v = make_qkv(w, device="cuda")
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    out = att.fused(q, k, v)
    bsa.bsa_poll_status(att.plan)
    ph, pw = w.draft_ph, w.draft_pw
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, ph, pw)
    valid = oracle.slot_valid(perm, Np)
    nb = Np // (ph * pw)
    heads = [0, w.Hh - 1]
    qn, kn, vn = (to_np64(x[:, :, heads]) for x in (q, k, v))
    kv = oracle.draft_blocks(qn, kn, w.T, w.H, w.W, ph, pw, w.draft_sparsity)
    np.testing.assert_array_equal(att.col_idx.view(w.B, w.Hh, nb, -1)[:, heads].cpu().numpy(), kv)
    rp, ci = oracle.fixed_k_csr(kv)
    O, _ = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Np) for x in (qn, kn, vn)),
                                   valid, ph * pw, rp, ci, True, 1 / math.sqrt(w.D),
                                   q_blocks=sample_blocks(nb, 6, seed=cid))
    ref = oracle.reorder_inv(np.nan_to_num(O, nan=np.inf), perm)
    got = to_np64(out[:, :, heads])
    m = np.isfinite(ref)
    err = np.abs(got[m] - ref[m])
    assert m.any() and err.max() <= MAX_ABS and err.mean() <= MEAN_ABS


def test_attn_natural_rejects_unsupported_plans():
    x = torch.zeros((1, 512, 1, 64), dtype=torch.bfloat16, device="cuda")
    buf = torch.zeros(4096, dtype=torch.int32, device="cuda")
    fplan = bsa.Plan(1, 1, 64, 8, 8, 8, bsa.LAYOUT_FRAME, block=64)
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_attn_fwd_natural(fplan, x, x, x, buf, buf, True, 0.125, x)
    assert ei.value.status == 1
    tplan = bsa.Plan(1, 1, 64, 8, 8, 8, bsa.LAYOUT_TILE, 2, 2, 4)     # 4-token tiles
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_attn_fwd_natural(tplan, x, x, x, buf, buf, True, 0.125, x)
    assert ei.value.status == 2


@pytest.mark.parametrize("precision", [bsa.DRAFT_FP64, bsa.DRAFT_FP32])
def test_draft_mask_many_blocks_takes_the_shared_memory_selection(precision):
    # 2 x 64 x 64 grid with 2 x 2 tiles: 2048 blocks per row, more than the
    # register-held logits of the scorer, so the shared-memory kernel runs
    # (in the plan's precision); the draft map is checked too
    w = small_workload(CONFIGS[1], T=2, H=64, W=64, Hh=1, D=64, qk="iid", draft_ph=2, draft_pw=2,
                       draft_sparsity=95)
    q, k, _ = make_qkv(w, device="cuda")
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, 2, 2, 4)
    bsa.bsa_plan_set_draft_precision(plan, precision)
    nb = plan.nblocks
    assert nb == 2048
    keep = bsa.bsa_draft_keep_count(plan, 95)
    kv = torch.empty(nb * keep, dtype=torch.int32, device="cuda")
    dm = torch.empty(nb * nb, dtype=torch.float32, device="cuda")
    ws = torch.empty(bsa.bsa_draft_workspace_bytes(plan), dtype=torch.uint8, device="cuda")
    bsa.bsa_draft_mask_natural(plan, q, k, 95, None, kv, dm, ws)
    bsa.bsa_poll_status(plan)
    prec = "fp64" if precision == bsa.DRAFT_FP64 else "fp32"
    qbar = oracle.draft_pool(to_np64(q), w.T, w.H, w.W, 2, 2)
    kbar = oracle.draft_pool(to_np64(k), w.T, w.H, w.W, 2, 2)
    L = oracle.draft_logits(qbar, kbar, prec)
    ref = oracle.draft_topk(L, keep)
    np.testing.assert_array_equal(kv.cpu().numpy().reshape(1, 1, nb, keep), ref)
    np.testing.assert_allclose(dm.cpu().numpy().reshape(1, 1, nb, nb), oracle.draft_map(L, w.D),
                               rtol=1e-5, atol=1e-7)
