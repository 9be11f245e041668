"""Parity of the one-pass LVSA attention (bsa_lvsa_attn_fwd, natural layout)
with the fp64 oracle.

The oracle computes on its frame layout and maps the result back to natural
token order; the kernel never builds that layout.  Tolerance as for the
other attention tests: max-abs <= 2e-2, mean-abs <= 2e-3, LSE within 2e-3.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_49_b200 as bsa
import oracle
from block_sparse_attention_49_b200 import _build
from synth import CONFIGS, make_qkv, small_workload

from gpu_util import LSE_ABS, MAX_ABS, MEAN_ABS, sample_blocks, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    bsa.load()


def _fused(w, C, T_per, s, q, k, v):
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=128)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.Hh, w.N), float("nan"), dtype=torch.float32, device="cuda")
    bsa.bsa_lvsa_attn_fwd(plan, C, T_per, s, q, k, v, 1 / math.sqrt(w.D), o, lse)
    bsa.bsa_poll_status(plan)
    return o, lse


def _oracle_natural(w, C, T_per, s, q, k, v, heads, q_blocks=None):
    """Oracle output in natural order for the chosen heads (NaN where not computed)."""
    blk = 128
    nbf = -(-w.P // blk)
    perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, blk)
    valid = oracle.slot_valid(perm, Np)
    rp, ci = oracle.lvsa_block_csr(oracle.lvsa_frame_sets(w.T, C, T_per, s), nbf)
    sub = lambda x: oracle.reorder_fwd(to_np64(x[:, :, heads]), perm, Np)
    O, L = oracle.masked_attention(sub(q), sub(k), sub(v), valid, blk, rp, ci, False,
                                   1 / math.sqrt(w.D), q_blocks=q_blocks)
    On = oracle.reorder_inv(O, perm)                         # [B, N, h, D]
    Ln = np.transpose(L[:, :, perm], (0, 1, 2))              # [B, h, N]
    return On, Ln


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
    return float(err.max()), float(err.mean())


@pytest.mark.parametrize("s", [0, 1, 2, 3, 7])
def test_fused_tiny_all_tokens(s):
    # 64-token frames: one 256-token query pair spans four frames
    w = CONFIGS[1]
    q, k, v = (x.cuda() for x in make_qkv(w))
    o, lse = _fused(w, w.lvsa_C, w.lvsa_T_per, s, q, k, v)
    On, Ln = _oracle_natural(w, w.lvsa_C, w.lvsa_T_per, s, q, k, v, list(range(w.Hh)))
    _check(o, lse, On, Ln, list(range(w.Hh)))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("s", [0, 1])
def test_fused_ragged_frames(D, s):
    # 63-token frames, N = 315 (not a multiple of the 256-token query pair)
    w = small_workload(CONFIGS[1], T=5, H=7, W=9, Hh=3, D=D)
    q, k, v = (x.cuda() for x in make_qkv(w))
    o, lse = _fused(w, 4, 3, s, q, k, v)
    On, Ln = _oracle_natural(w, 4, 3, s, q, k, v, list(range(w.Hh)))
    _check(o, lse, On, Ln, list(range(w.Hh)))


@pytest.mark.parametrize("H,W,s", [(7, 9, 0), (9, 7, 0), (7, 9, 2), (5, 13, 1)])
def test_fused_runs_whose_tiles_overhang_the_next_run(H, W, s):
    # odd frame sizes: a run's last key tile reaches into the frames after it,
    # where another run of the union may begin; those keys belong to one tile only
    w = small_workload(CONFIGS[1], T=5, H=H, W=W, Hh=2, D=64)
    q, k, v = (x.cuda() for x in make_qkv(w))
    o, lse = _fused(w, 4, 3, s, q, k, v)
    On, Ln = _oracle_natural(w, 4, 3, s, q, k, v, [0, 1])
    _check(o, lse, On, Ln, [0, 1])


def test_fused_frames_longer_than_a_pair():
    # 30 x 52 frames (1560 tokens): pairs inside a frame and pairs straddling two
    w = small_workload(CONFIGS[3], T=6, Hh=2, field_grid=(6, 4, 7))
    q, k, v = (x.cuda() for x in make_qkv(w))
    for s in (0, 3):
        o, lse = _fused(w, 3, 4, s, q, k, v)
        On, Ln = _oracle_natural(w, 3, 4, s, q, k, v, [0, 1])
        _check(o, lse, On, Ln, [0, 1])


@pytest.mark.parametrize("cid,s", [(3, 0), (3, 11), (4, 0), (4, 13)])
def test_fused_full_size_sampled(cid, s):
    w = CONFIGS[cid]
    q, k, v = make_qkv(w, device="cuda")
    o, lse = _fused(w, w.lvsa_C, w.lvsa_T_per, s, q, k, v)
    nb = w.T * -(-w.P // 128)
    heads = [0, w.Hh - 1]
    On, Ln = _oracle_natural(w, w.lvsa_C, w.lvsa_T_per, s, q, k, v, heads,
                             q_blocks=sample_blocks(nb, 6, seed=s))
    _check(o, lse, On, Ln, heads)
    assert torch.isfinite(o).all()


def test_fused_matches_unfused_path_full_size():
    from block_sparse_attention_49_b200.pipeline import LvsaAttention
    w = CONFIGS[3]
    q, k, v = make_qkv(w, device="cuda")
    att = LvsaAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.lvsa_C, w.lvsa_T_per, block=128)
    a = att(q, k, v, 5)
    b = att.fused(q, k, v, 5)
    bsa.bsa_poll_status(att.plan)
    d = (a.float() - b.float()).abs()
    assert d.max().item() <= 3e-2 and d.mean().item() <= 1e-3


def test_fused_rejects_unsupported_geometry():
    plan = bsa.Plan(1, 1, 64, 4, 4, 8, bsa.LAYOUT_FRAME, block=32)   # 32-token frames
    x = torch.zeros((1, 128, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_lvsa_attn_fwd(plan, 3, 2, 0, x, x, x, 0.125, x)
    assert ei.value.status == 2
    tplan = bsa.Plan(1, 1, 64, 4, 8, 8, bsa.LAYOUT_TILE, 2, 2, 4)
    y = torch.zeros((1, 256, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_lvsa_attn_fwd(tplan, 3, 2, 0, y, y, y, 0.125, y)
    assert ei.value.status == 1


def test_streamed_steps_match_direct_calls():
    # host inputs copied in and the output read back every step, overlapped
    # with the neighbouring steps' compute: the last step's output equals the
    # direct call's, bit for bit
    from block_sparse_attention_49_b200.pipeline import LvsaAttention, StreamedSteps
    w = small_workload(CONFIGS[3], T=12, Hh=2, field_grid=(12, 4, 7))
    q, k, v = make_qkv(w)
    hq, hk, hv = (x.pin_memory() for x in (q, k, v))
    ho = torch.empty_like(hq).pin_memory()
    att = LvsaAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, 5, 4, block=128)
    streamed = StreamedSteps(q.shape, q.dtype)
    streamed.run(lambda a, b, c, out, i: att.fused(a, b, c, i, out), (hq, hk, hv), ho, 3)
    torch.cuda.synchronize()
    direct = att.fused(q.cuda(), k.cuda(), v.cuda(), 2)
    bsa.bsa_poll_status(att.plan)
    assert torch.equal(ho.view(torch.int16), direct.cpu().view(torch.int16))
