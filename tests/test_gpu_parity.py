"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Masks, block lists, permutations and pooled values: bit-exact.  Attention
output: max-abs <= 2e-2 and mean-abs <= 2e-3 against fp64 on bf16 inputs;
LSE within 2e-3.  Small workloads are compared on every element; the full
workloads (in the launch configuration the benchmark times) on sampled query
blocks that the oracle computes one by one.
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

from gpu_util import compare_attention, padded, perm_of, sample_blocks, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    bsa.load()


def _slots_gpu(x_nat: torch.Tensor, perm: np.ndarray, Npad: int) -> torch.Tensor:
    """Slot tensor built with torch indexing from the oracle's permutation."""
    B, N, Hh, D = x_nat.shape
    out = torch.zeros((B, Hh, Npad, D), dtype=x_nat.dtype, device="cuda")
    out[:, :, torch.from_numpy(perm).cuda()] = x_nat.cuda().permute(0, 2, 1, 3)
    return out


def _run_attn(plan, qs, ks, vs, row_ptr, col_idx, per_head, scale):
    o = torch.full_like(qs, float("nan"))
    lse = torch.full(qs.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    bsa.bsa_attn_fwd(plan, qs, ks, vs, torch.as_tensor(row_ptr).cuda(),
                     torch.as_tensor(col_idx).cuda(), per_head, scale, o, lse)
    bsa.bsa_poll_status(plan)
    return o, lse


# ------------------------------------------------------------------ LVSA mask
@pytest.mark.parametrize("cid", [1, 3, 4])
def test_lvsa_mask_bit_exact(cid):
    w = CONFIGS[cid]
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=w.lvsa_block)
    nbf = -(-w.P // w.lvsa_block)
    nnz = bsa.bsa_lvsa_nnz(plan, w.lvsa_C)
    fs = torch.empty(w.T * w.lvsa_C, dtype=torch.int32, device="cuda")
    rp = torch.empty(plan.nblocks + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty(nnz, dtype=torch.int32, device="cuda")
    for s in list(w.lvsa_steps) + [w.lvsa_T_per + 3]:     # a step past one period too
        bsa.bsa_lvsa_mask(plan, w.lvsa_C, w.lvsa_T_per, s, fs, rp, ci)
        bsa.bsa_poll_status(plan)
        A = oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, s)
        rpo, cio = oracle.lvsa_block_csr(A, nbf)
        np.testing.assert_array_equal(fs.cpu().numpy().reshape(w.T, w.lvsa_C), A)
        np.testing.assert_array_equal(rp.cpu().numpy(), rpo)
        np.testing.assert_array_equal(ci.cpu().numpy(), cio)


def test_lvsa_mask_rejects_infeasible_budget():
    plan = bsa.Plan(1, 1, 64, 8, 8, 8, bsa.LAYOUT_FRAME, block=64)
    buf = torch.empty(1024, dtype=torch.int32, device="cuda")
    with pytest.raises(bsa.BsaError):
        bsa.bsa_lvsa_mask(plan, 2, 4, 0, None, buf, buf)   # 2 anchors + t > C = 2
    with pytest.raises(bsa.BsaError):
        bsa.bsa_lvsa_mask(plan, 9, 4, 0, None, buf, buf)   # C > T


# ------------------------------------------------------------------ reorder
REORDER_CASES = [
    # (workload overrides, layout, pool/block)
    (dict(cid=1), "frame", 64),
    (dict(cid=1), "tile", (2, 2)),
    (dict(cid=2, Hh=3), "tile", (8, 16)),
    (dict(cid=2, Hh=3), "frame", 128),
    (dict(cid=1, T=3, H=5, W=7, Hh=3, D=128, qk="iid"), "tile", (4, 4)),
    (dict(cid=1, T=3, H=5, W=7, Hh=2, D=64, qk="iid"), "frame", 32),
]


@pytest.mark.parametrize("over,layout,blk", REORDER_CASES)
def test_reorder_bit_exact(over, layout, blk):
    over = dict(over)
    base = CONFIGS[over.pop("cid")]
    w = small_workload(base, **over)
    q, k, v = make_qkv(w)
    if layout == "frame":
        plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=blk)
        perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, blk)
    else:
        plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, blk[0], blk[1],
                        blk[0] * blk[1])
        perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, *blk)
    assert plan.Npad == padded(Np)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    outs = [torch.full((w.B, w.Hh, plan.Npad, w.D), 7.0, dtype=torch.bfloat16, device="cuda")
            for _ in range(3)]
    bsa.bsa_reorder_fwd(plan, qg, outs[0], kg, outs[1], vg, outs[2])
    for x, y in zip((q, k, v), outs):
        ref = oracle.reorder_fwd(x.view(torch.int16).numpy(), perm, Np)   # raw bits
        got = y.cpu().view(torch.int16).numpy()
        np.testing.assert_array_equal(got[:, :, :Np], ref)
        assert (got[:, :, Np:] == 0).all()
    back = torch.full_like(qg, 3.0)
    bsa.bsa_reorder_inv(plan, outs[1], back)
    assert torch.equal(back.cpu().view(torch.int16), k.view(torch.int16))


@pytest.mark.parametrize("layout", ["frame", "tile"])
def test_reorder_keep_pads_writes_only_token_slots(layout):
    # BSA_PADS_KEEP: the slots holding tokens get the tokens bit for bit;
    # every empty slot keeps what the buffer held (here 7.0)
    w = small_workload(CONFIGS[2], T=3, H=13, W=37, Hh=2, field_grid=(3, 4, 7))
    q, _, _ = make_qkv(w)
    if layout == "frame":
        plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=128)
        perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, 128)
    else:
        plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, 8, 16, 128)
        perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, 8, 16)
    bsa.bsa_plan_set_reorder_pads(plan, bsa.PADS_KEEP)
    y = torch.full((w.B, w.Hh, plan.Npad, w.D), 7.0, dtype=torch.bfloat16, device="cuda")
    bsa.bsa_reorder_fwd(plan, q.cuda(), y)
    bsa.bsa_poll_status(plan)
    valid = np.zeros(plan.Npad, dtype=bool)
    valid[:Np] = oracle.slot_valid(perm, Np)
    ref = oracle.reorder_fwd(q.view(torch.int16).numpy(), perm, Np)
    got = y.cpu().view(torch.int16).numpy()
    np.testing.assert_array_equal(got[:, :, :Np][:, :, valid[:Np]], ref[:, :, valid[:Np]])
    seven = torch.tensor(7.0, dtype=torch.bfloat16).view(torch.int16).item()
    assert (got[:, :, ~valid] == seven).all() and (~valid).any()
    # WRITE (the default) zeroes them again
    bsa.bsa_plan_set_reorder_pads(plan, bsa.PADS_WRITE)
    bsa.bsa_reorder_fwd(plan, q.cuda(), y)
    assert (y.cpu().view(torch.int16).numpy()[:, :, ~valid] == 0).all()


def test_reorder_rejects_a_third_pair_without_the_second():
    plan = bsa.Plan(1, 1, 64, 8, 8, 8, bsa.LAYOUT_FRAME, block=64)
    x = torch.zeros((1, 512, 1, 64), dtype=torch.bfloat16, device="cuda")
    y = [torch.full((1, 1, plan.Npad, 64), 7.0, dtype=torch.bfloat16, device="cuda")
         for _ in range(3)]
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_reorder_fwd(plan, x, y[0], None, None, x, y[2])
    assert ei.value.status == 1
    # rejected on the host: nothing was written
    assert all((t == 7.0).all() for t in y)
    bsa.bsa_reorder_fwd(plan, x, y[0], x, y[1], x, y[2])
    bsa.bsa_poll_status(plan)
    assert all((t == 0).all() for t in y)


@pytest.mark.parametrize("cid,layout", [(3, "frame"), (4, "frame"), (5, "tile")])
def test_reorder_round_trip_full_size(cid, layout):
    w = CONFIGS[cid]
    g = torch.Generator(device="cuda").manual_seed(cid)
    x = torch.randn((w.B, w.N, w.Hh, w.D), generator=g, device="cuda").to(torch.bfloat16)
    if layout == "frame":
        plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=128)
        perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, 128)
    else:
        plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, w.draft_ph, w.draft_pw,
                        w.draft_ph * w.draft_pw)
        perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, w.draft_ph, w.draft_pw)
    ys = torch.empty((w.B, w.Hh, plan.Npad, w.D), dtype=torch.bfloat16, device="cuda")
    bsa.bsa_reorder_fwd(plan, x, ys)
    back = torch.empty_like(x)
    bsa.bsa_reorder_inv(plan, ys, back)
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))
    # sampled tokens land in the oracle's slots
    idx = torch.randint(0, w.N, (4096,), generator=torch.Generator().manual_seed(1))
    slots = torch.from_numpy(perm[idx.numpy()]).cuda()
    assert torch.equal(ys[0, :, slots].view(torch.int16),
                       x[0, idx.cuda()].permute(1, 0, 2).view(torch.int16))
    valid = torch.from_numpy(oracle.slot_valid(perm, Np)).cuda()
    assert (ys[:, :, :Np][:, :, ~valid] == 0).all()


# ------------------------------------------------------------------ draft mask
DRAFT_CASES = [
    dict(cid=1),
    dict(cid=2),
    dict(cid=1, T=3, H=5, W=7, Hh=3, D=128, qk="iid", draft_ph=4, draft_pw=4, draft_sparsity=70),
    dict(cid=5),
    # rows of exactly 32 blocks (no padded keys): keep = the whole row, where
    # the threshold search is settled before its first bit, and keep = 1
    dict(cid=1, T=2, H=16, W=32, Hh=2, D=128, qk="iid", draft_ph=4, draft_pw=8, draft_sparsity=0),
    dict(cid=1, T=2, H=16, W=32, Hh=2, D=128, qk="iid", draft_ph=4, draft_pw=8, draft_sparsity=97),
    # 64 blocks, half kept, head dim 64
    dict(cid=1, T=4, H=16, W=32, Hh=2, D=64, qk="iid", draft_ph=4, draft_pw=8, draft_sparsity=50),
]


@pytest.mark.parametrize("over", DRAFT_CASES)
@pytest.mark.parametrize("precision", [bsa.DRAFT_FP64, bsa.DRAFT_FP32])
def test_draft_mask_bit_exact(over, precision):
    over = dict(over)
    w = small_workload(CONFIGS[over.pop("cid")], **over)
    ph, pw, sp = w.draft_ph, w.draft_pw, w.draft_sparsity
    q, k, _ = make_qkv(w)
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, ph, pw, ph * pw)
    bsa.bsa_plan_set_draft_precision(plan, precision)
    npdt = np.float64 if precision == bsa.DRAFT_FP64 else np.float32
    prec = "fp64" if precision == bsa.DRAFT_FP64 else "fp32"
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, ph, pw)
    qs, ks = _slots_gpu(q, perm, plan.Npad), _slots_gpu(k, perm, plan.Npad)
    keep = bsa.bsa_draft_keep_count(plan, sp)
    nb = plan.nblocks
    rows = w.B * w.Hh * nb
    rp = torch.empty(rows + 1, dtype=torch.int32, device="cuda")
    kv = torch.empty(rows * keep, dtype=torch.int32, device="cuda")
    want_map = w.Hh * nb * nb <= 4_000_000
    dm = torch.empty(rows * nb, dtype=torch.float32, device="cuda") if want_map else None
    ws = torch.full((bsa.bsa_draft_workspace_bytes(plan) // np.dtype(npdt).itemsize,),
                    float("nan"), dtype=torch.from_numpy(np.zeros(1, npdt)).dtype, device="cuda")
    bsa.bsa_draft_mask(plan, qs, ks, sp, rp, kv, dm, ws)
    bsa.bsa_poll_status(plan)

    qn, kn = to_np64(q), to_np64(k)
    qbar = oracle.draft_pool(qn, w.T, w.H, w.W, ph, pw)
    kbar = oracle.draft_pool(kn, w.T, w.H, w.W, ph, pw)
    got_pool = ws.cpu().numpy()[:2 * rows * w.D].reshape(2, w.B, w.Hh, nb, w.D)
    np.testing.assert_array_equal(got_pool[0], qbar.astype(npdt))   # bit-exact
    np.testing.assert_array_equal(got_pool[1], kbar.astype(npdt))
    L = oracle.draft_logits(qbar, kbar, prec)
    ref = oracle.draft_topk(L, oracle.draft_keep_count(nb, sp))
    np.testing.assert_array_equal(kv.cpu().numpy().reshape(w.B, w.Hh, nb, keep), ref)
    np.testing.assert_array_equal(rp.cpu().numpy(), np.arange(rows + 1) * keep)
    if want_map:
        np.testing.assert_allclose(dm.cpu().numpy().reshape(w.B, w.Hh, nb, nb),
                                   oracle.draft_map(L, w.D), rtol=1e-5, atol=1e-7)
    # diagnostic: the selection margin between the k-th and (k+1)-th logit
    if keep < nb:
        srt = -np.sort(-L, axis=-1)
        assert np.isfinite(srt[..., keep - 1] - srt[..., keep]).all()


def test_draft_mask_logits_equal_in_fp32_but_not_in_fp64():
    # Eight 2 x 2 tiles in one row of a 2 x 16 grid, one head, D = 64.  Every
    # query tile pools to q = (1, 2^-20, 0, ...); key tile j to (a_j, d_j, 0,
    # ...), so L[i][j] = a_j + 2^-20 d_j exactly in fp64:
    #   L = 0.5, 2, 1, 3, 1 + 2^-39, 1 + 2^-40, 4, 0.125.
    # Keeping 5 of 8 takes blocks 1, 3, 6 and two of the three logits that
    # round to 1.0 in fp32.  fp64 ranks them by value (blocks 4, 5); fp32
    # sees a tie and takes the lower indices (blocks 2, 4).
    T, H, W, D, ph, pw = 1, 2, 16, 64, 2, 2
    a = [0.5, 2.0, 1.0, 3.0, 1.0, 1.0, 4.0, 0.125]
    d = [0.0, 0.0, 0.0, 0.0, 2.0 ** -19, 2.0 ** -20, 0.0, 0.0]
    q = torch.zeros((1, T * H * W, 1, D), dtype=torch.bfloat16)
    k = torch.zeros_like(q)
    for y in range(H):
        for x in range(W):
            n, j = y * W + x, x // pw
            q[0, n, 0, 0], q[0, n, 0, 1] = 1.0, 2.0 ** -20
            k[0, n, 0, 0], k[0, n, 0, 1] = a[j], d[j]
    qn, kn = to_np64(q), to_np64(k)
    qbar = oracle.draft_pool(qn, T, H, W, ph, pw)
    kbar = oracle.draft_pool(kn, T, H, W, ph, pw)
    L64 = oracle.draft_logits(qbar, kbar)
    assert L64[0, 0, 0, 5] == 1.0 + 2.0 ** -40 and L64[0, 0, 0, 4] == 1.0 + 2.0 ** -39
    want = {bsa.DRAFT_FP64: [1, 3, 4, 5, 6], bsa.DRAFT_FP32: [1, 2, 3, 4, 6]}
    for precision, prec in ((bsa.DRAFT_FP64, "fp64"), (bsa.DRAFT_FP32, "fp32")):
        ref = oracle.draft_topk(oracle.draft_logits(qbar, kbar, prec), 5)
        assert (ref == np.array(want[precision])).all()
        plan = bsa.Plan(1, 1, D, T, H, W, bsa.LAYOUT_TILE, ph, pw, ph * pw)
        bsa.bsa_plan_set_draft_precision(plan, precision)
        assert bsa.bsa_draft_keep_count(plan, 40) == 5
        perm, Np = oracle.tile_layout_perm(T, H, W, ph, pw)
        qs, ks = _slots_gpu(q, perm, plan.Npad), _slots_gpu(k, perm, plan.Npad)
        rp = torch.empty(9, dtype=torch.int32, device="cuda")
        kv = torch.empty(8 * 5, dtype=torch.int32, device="cuda")
        ws = torch.empty(bsa.bsa_draft_workspace_bytes(plan), dtype=torch.uint8, device="cuda")
        bsa.bsa_draft_mask(plan, qs, ks, 40, rp, kv, None, ws)
        bsa.bsa_poll_status(plan)
        got = kv.cpu().numpy().reshape(8, 5)
        assert (got == np.array(want[precision])[None, :]).all(), (precision, got)


def test_draft_mask_fp32_overflow_decided_in_fp64():
    # pooled values 2^66 and 2^66 (1 + j/64): every product overflows fp32,
    # so the fp32 logits are all +inf and tie, while the fp64 ones are
    # distinct.  The fp64 lists then come from the fp64 logits of every
    # block (the overflow path of the certification): blocks 8..15; fp32
    # precision keeps the lowest indices, 0..7.
    T, H, W, D, ph, pw = 1, 4, 16, 64, 2, 2
    q = torch.full((1, T * H * W, 1, D), 2.0 ** 66, dtype=torch.bfloat16)
    k = torch.zeros_like(q)
    for y in range(H):
        for x in range(W):
            j = (y // ph) * (W // pw) + x // pw
            k[0, y * W + x, 0, :] = 2.0 ** 66 * (1 + j / 64)
    qbar = oracle.draft_pool(to_np64(q), T, H, W, ph, pw)
    kbar = oracle.draft_pool(to_np64(k), T, H, W, ph, pw)
    L64 = oracle.draft_logits(qbar, kbar)
    with np.errstate(over="ignore"):
        L32 = oracle.draft_logits(qbar, kbar, "fp32")
    assert np.isinf(L32).all() and np.isfinite(L64).all()
    for precision, L, want in ((bsa.DRAFT_FP64, L64, np.arange(8, 16)),
                               (bsa.DRAFT_FP32, L32, np.arange(8))):
        ref = oracle.draft_topk(L, 8)
        assert (ref == want).all()
        plan = bsa.Plan(1, 1, D, T, H, W, bsa.LAYOUT_TILE, ph, pw, ph * pw)
        bsa.bsa_plan_set_draft_precision(plan, precision)
        assert plan.nblocks == 16 and bsa.bsa_draft_keep_count(plan, 50) == 8
        perm, Np = oracle.tile_layout_perm(T, H, W, ph, pw)
        qs, ks = _slots_gpu(q, perm, plan.Npad), _slots_gpu(k, perm, plan.Npad)
        rp = torch.empty(17, dtype=torch.int32, device="cuda")
        kv = torch.empty(16 * 8, dtype=torch.int32, device="cuda")
        dm = (torch.empty(16 * 16, dtype=torch.float32, device="cuda")
              if precision == bsa.DRAFT_FP64 else None)
        ws = torch.empty(bsa.bsa_draft_workspace_bytes(plan), dtype=torch.uint8, device="cuda")
        bsa.bsa_draft_mask(plan, qs, ks, 50, rp, kv, dm, ws)
        bsa.bsa_poll_status(plan)
        np.testing.assert_array_equal(kv.cpu().numpy().reshape(1, 1, 16, 8), ref)
        if dm is not None:
            np.testing.assert_allclose(dm.cpu().numpy().reshape(1, 1, 16, 16),
                                       oracle.draft_map(L64, D), rtol=1e-6, atol=1e-12)


@pytest.mark.parametrize("precision", [bsa.DRAFT_FP64, bsa.DRAFT_FP32])
def test_draft_mask_all_logits_equal(precision):
    # constant Q and K: every logit of a row is the same, so the kept blocks
    # are the lowest indices (in fp64 every block of the row is within the
    # fp32 error bound of the k-th and gets its fp64 logit)
    T, H, W, D, ph, pw = 1, 4, 8, 64, 2, 2
    q = torch.full((1, T * H * W, 1, D), 0.5, dtype=torch.bfloat16)
    k = torch.full_like(q, -0.25)
    plan = bsa.Plan(1, 1, D, T, H, W, bsa.LAYOUT_TILE, ph, pw, ph * pw)
    bsa.bsa_plan_set_draft_precision(plan, precision)
    keep = bsa.bsa_draft_keep_count(plan, 60)
    nb = plan.nblocks
    perm, Np = oracle.tile_layout_perm(T, H, W, ph, pw)
    qs, ks = _slots_gpu(q, perm, plan.Npad), _slots_gpu(k, perm, plan.Npad)
    rp = torch.empty(nb + 1, dtype=torch.int32, device="cuda")
    kv = torch.empty(nb * keep, dtype=torch.int32, device="cuda")
    dm = torch.empty(nb * nb, dtype=torch.float32, device="cuda")
    ws = torch.empty(bsa.bsa_draft_workspace_bytes(plan), dtype=torch.uint8, device="cuda")
    bsa.bsa_draft_mask(plan, qs, ks, 60, rp, kv, dm, ws)
    bsa.bsa_poll_status(plan)
    prec = "fp64" if precision == bsa.DRAFT_FP64 else "fp32"
    qbar = oracle.draft_pool(to_np64(q), T, H, W, ph, pw)
    kbar = oracle.draft_pool(to_np64(k), T, H, W, ph, pw)
    ref = oracle.draft_topk(oracle.draft_logits(qbar, kbar, prec), keep)
    assert (ref == np.arange(keep)).all()
    np.testing.assert_array_equal(kv.cpu().numpy().reshape(1, 1, nb, keep), ref)
    np.testing.assert_allclose(dm.cpu().numpy(), 1.0 / nb, rtol=1e-6)


# ------------------------------------------------------------------ attention
def _attn_case(w, layout, blk, rp, ci, per_head, q_blocks=None, heads=None, scale=None):
    """Run bsattn on slot tensors built from the oracle's permutation and
    compare with the oracle on the given query blocks / heads."""
    q, k, v = make_qkv(w)
    if layout == "frame":
        plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=blk)
        perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, blk)
    else:
        plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, blk[0], blk[1],
                        blk[0] * blk[1])
        perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, *blk)
        blk = blk[0] * blk[1]
    scale = scale if scale is not None else 1.0 / math.sqrt(w.D)
    qs, ks, vs = (_slots_gpu(x, perm, plan.Npad) for x in (q, k, v))
    o, lse = _run_attn(plan, qs, ks, vs, rp, ci, per_head, scale)
    valid = oracle.slot_valid(perm, Np)
    nqb = Np // blk
    qbs = list(range(nqb)) if q_blocks is None else q_blocks
    hs = [(b, h) for b in range(w.B) for h in range(w.Hh)] if heads is None else heads
    hsel = sorted({h for _, h in hs})
    # oracle on the selected heads only (keeps host memory small at full size)
    sub = lambda x: oracle.reorder_fwd(to_np64(x[:, :, hsel]), perm, Np)
    if per_head:
        nbk = nqb
        rp_np, ci_np = np.asarray(rp), np.asarray(ci)
        lists = []
        for hh in hsel:
            lists.append(ci_np[rp_np[hh * nbk]:rp_np[(hh + 1) * nbk]])
        k_each = np.diff(rp_np)[0]
        rp_sub = (np.arange(len(hsel) * nbk + 1) * k_each).astype(np.int32)
        ci_sub = np.concatenate(lists)
    else:
        rp_sub, ci_sub = rp, ci
    O, L = oracle.masked_attention(sub(q), sub(k), sub(v), valid, blk, rp_sub, ci_sub, per_head,
                                   scale, q_blocks=qbs,
                                   heads=[(0, i) for i in range(len(hsel))])
    og = o[:, hsel]
    lg = lse[:, hsel]
    res = compare_attention(og, lg, O, L, valid, blk, qbs, [(0, i) for i in range(len(hsel))])
    # slots past the oracle's padding are empty: zero output
    if plan.Npad > Np:
        assert (o[:, :, Np:] == 0).all()
    return res


def test_attn_tiny_dense_frame_blocks():
    w = CONFIGS[1]
    rp, ci = oracle.dense_block_csr(8)
    _attn_case(w, "frame", 64, rp, ci, False)


@pytest.mark.parametrize("s", [0, 1, 2, 3])
def test_attn_tiny_lvsa(s):
    w = CONFIGS[1]
    A = oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, s)
    rp, ci = oracle.lvsa_block_csr(A, 1)
    _attn_case(w, "frame", 64, rp, ci, False)


def test_attn_tiny_draft_4_token_blocks():
    w = CONFIGS[1]
    q, k, _ = make_qkv(w)
    kv = oracle.draft_blocks(to_np64(q), to_np64(k), w.T, w.H, w.W, 2, 2, 50)
    rp, ci = oracle.fixed_k_csr(kv)
    _attn_case(w, "tile", (2, 2), rp, ci, True)


@pytest.mark.parametrize("D", [64, 128])
def test_attn_ragged_tiles_dense_and_random_mask(D):
    # 30 x 52 grid in 8 x 16 tiles: edge tiles are partly empty
    w = small_workload(CONFIGS[2], T=2, Hh=2, D=D, field_grid=(2, 4, 7))
    nb = 2 * 16
    rp, ci = oracle.dense_block_csr(nb)
    _attn_case(w, "tile", (8, 16), rp, ci, False)
    rng = np.random.default_rng(D)
    rows = []
    for _ in range(w.B * w.Hh * nb):
        n = int(rng.integers(1, nb + 1))
        rows.append(np.sort(rng.choice(nb, size=n, replace=False)).astype(np.int32))
    rp2 = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    # varying row lengths: per-head lists in one CSR
    _attn_case_var(w, rp2, np.concatenate(rows))


def _attn_case_var(w, rp, ci):
    q, k, v = make_qkv(w)
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, 8, 16, 128)
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, 8, 16)
    qs, ks, vs = (_slots_gpu(x, perm, plan.Npad) for x in (q, k, v))
    scale = 1.0 / math.sqrt(w.D)
    o, lse = _run_attn(plan, qs, ks, vs, rp, ci, True, scale)
    valid = oracle.slot_valid(perm, Np)
    O, L = oracle.masked_attention(*(oracle.reorder_fwd(to_np64(x), perm, Np) for x in (q, k, v)),
                                   valid, 128, rp, ci, True, scale)
    compare_attention(o, lse, O, L, valid, 128, list(range(Np // 128)),
                      [(b, h) for b in range(w.B) for h in range(w.Hh)])


@pytest.mark.parametrize("T", [315, 330])
def test_attn_shared_list_at_and_past_4096_blocks(T):
    # 13 blocks a frame: 4095 blocks run on the paired kernel, 4290 on the
    # block-list kernel (the paired kernel's union holds 4096).  Rows 0 and 1
    # name every block, so their union is the whole plan.
    w = small_workload(CONFIGS[2], T=T, Hh=1, D=64, field_grid=(8, 4, 7))
    nb = T * 13
    rng = np.random.default_rng(T)
    rows = [np.arange(nb), np.arange(nb)]
    rows += [np.unique(np.concatenate([[r], rng.choice(nb, size=2, replace=False)]))
             for r in range(2, nb)]
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    _attn_case(w, "frame", 128, rp, ci, False, q_blocks=[0, 1, 2, 2000, nb - 1])


def test_attn_per_head_lists_frame_layout():
    # per-head lists of 128-slot blocks on the frame layout (each frame's
    # last block is partly empty): the persistent kernel's slot mode
    w = small_workload(CONFIGS[2], T=3, Hh=2, D=128, field_grid=(3, 4, 7))
    nb = 3 * 13
    rng = np.random.default_rng(7)
    k = 9
    rows = [np.sort(rng.choice(nb, size=k, replace=False)) for _ in range(w.B * w.Hh * nb)]
    rp = (np.arange(len(rows) + 1) * k).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    _attn_case(w, "frame", 128, rp, ci, True)


@pytest.mark.parametrize("per_head", [False, True])
def test_attn_empty_rows_and_out_of_range_blocks(per_head):
    # one (batch, head): the same CSR serves as a shared list (the paired
    # kernel) and as per-head lists (the persistent kernel's slot mode)
    w = small_workload(CONFIGS[2], T=1, Hh=1, D=128, field_grid=(1, 4, 7))
    q, k, v = make_qkv(w)
    plan = bsa.Plan(1, 1, 128, 1, 30, 52, bsa.LAYOUT_TILE, 8, 16, 128)
    perm, Np = oracle.tile_layout_perm(1, 30, 52, 8, 16)
    qs, ks, vs = (_slots_gpu(x, perm, plan.Npad) for x in (q, k, v))
    # 16 rows: row 3 empty, row 5 names block 99 (out of range) besides block 0
    lists = [[0, 1, 2]] * 16
    lists = [list(r) for r in lists]
    lists[3] = []
    lists[5] = [0, 99]
    rp = np.concatenate([[0], np.cumsum([len(r) for r in lists])]).astype(np.int32)
    ci = np.array([c for r in lists for c in r], dtype=np.int32)
    o = torch.empty_like(qs)
    lse = torch.empty(qs.shape[:3], dtype=torch.float32, device="cuda")
    bsa.bsa_attn_fwd(plan, qs, ks, vs, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(),
                     per_head, 1 / math.sqrt(128), o, lse)
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_poll_status(plan)
    assert ei.value.status == 6
    assert (o[0, 0, 3 * 128:4 * 128] == 0).all()
    assert torch.isneginf(lse[0, 0, 3 * 128:4 * 128]).all()
    # row 5 equals the row that lists block 0 alone
    valid = oracle.slot_valid(perm, Np)
    ci_ok = np.array([c if c != 99 else 0 for c in ci], dtype=np.int32)
    lists_ok = [list(r) for r in lists]
    lists_ok[5] = [0]
    rp_ok = np.concatenate([[0], np.cumsum([len(r) for r in lists_ok])]).astype(np.int32)
    ci_ok = np.array([c for r in lists_ok for c in r], dtype=np.int32)
    O, L = oracle.masked_attention(*(oracle.reorder_fwd(to_np64(x), perm, Np) for x in (q, k, v)),
                                   valid, 128, rp_ok, ci_ok, per_head, 1 / math.sqrt(128))
    compare_attention(o, lse, O, L, valid, 128, list(range(16)), [(0, 0)])
    bsa.bsa_poll_status(plan)   # status was cleared by the previous poll


def test_attn_dense_native_wan_shape_sampled():
    w = CONFIGS[2]
    nb = w.T * 13
    rp, ci = oracle.dense_block_csr(nb)
    _attn_case(w, "frame", 128, rp, ci, False, q_blocks=sample_blocks(nb, 5),
               heads=[(0, 0), (0, 11)])


@pytest.mark.parametrize("cid,s", [(3, 0), (3, 11), (4, 0), (4, 9)])
def test_attn_lvsa_full_size_sampled(cid, s):
    w = CONFIGS[cid]
    nbf = -(-w.P // 128)
    A = oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, s)
    rp, ci = oracle.lvsa_block_csr(A, nbf)
    nb = w.T * nbf
    _attn_case(w, "frame", 128, rp, ci, False, q_blocks=sample_blocks(nb, 6, seed=s),
               heads=[(0, 0), (0, w.Hh - 1)])


# ------------------------------------------------------------------ end to end
def test_pipeline_lvsa_tiny_natural_order():
    w = CONFIGS[1]
    q, k, v = make_qkv(w)
    att = LvsaAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.lvsa_C, w.lvsa_T_per, block=64)
    perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, 64)
    valid = oracle.slot_valid(perm, Np)
    for s in range(4):
        out = att(q.cuda(), k.cuda(), v.cuda(), s)
        bsa.bsa_poll_status(att.plan)
        rp, ci = oracle.lvsa_block_csr(oracle.lvsa_frame_sets(w.T, 4, 4, s), 1)
        O, _ = oracle.masked_attention(*(oracle.reorder_fwd(to_np64(x), perm, Np) for x in (q, k, v)),
                                       valid, 64, rp, ci, False, 1 / 8.0)
        ref = oracle.reorder_inv(O, perm)
        err = np.abs(to_np64(out) - ref)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3


@pytest.mark.parametrize("cid", [1, 5])
def test_pipeline_draft_natural_order(cid):
    w = CONFIGS[cid]
    q, k, v = make_qkv(w)
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    out = att(q.cuda(), k.cuda(), v.cuda())
    bsa.bsa_poll_status(att.plan)
    ph, pw = w.draft_ph, w.draft_pw
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, ph, pw)
    valid = oracle.slot_valid(perm, Np)
    blk = ph * pw
    nb = Np // blk
    heads = [0, w.Hh - 1] if w.Hh > 2 else list(range(w.Hh))
    qn, kn, vn = (to_np64(x[:, :, heads]) for x in (q, k, v))
    kv = oracle.draft_blocks(qn, kn, w.T, w.H, w.W, ph, pw, w.draft_sparsity)
    np.testing.assert_array_equal(
        att.col_idx.view(w.B, w.Hh, nb, -1)[:, heads].cpu().numpy(), kv)
    rp, ci = oracle.fixed_k_csr(kv)
    qbs = list(range(nb)) if nb <= 128 else sample_blocks(nb, 6)
    O, L = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Np) for x in (qn, kn, vn)),
                                   valid, blk, rp, ci, True, 1 / math.sqrt(w.D), q_blocks=qbs)
    got = to_np64(out[:, :, heads])
    ref_nat = oracle.reorder_inv(np.nan_to_num(O, nan=np.inf), perm)   # unsampled rows -> inf
    m = np.isfinite(ref_nat)
    err = np.abs(got[m] - ref_nat[m])
    assert m.any() and err.max() <= 2e-2 and err.mean() <= 2e-3


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_times_out_and_context_survives():
    plan = bsa.Plan(1, 1, 64, 8, 8, 8, bsa.LAYOUT_FRAME, block=64)
    bsa.bsa_selftest_timeout(plan, 2_000_000)     # 2 ms limit, nobody arrives
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_poll_status(plan)
    assert ei.value.status == 5
    # the context is still usable: a normal call succeeds afterwards
    test_attn_tiny_dense_frame_blocks()
