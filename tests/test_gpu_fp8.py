"""The 8-bit draft attention (Draft Attention article, closing paragraph:
quantization as the next step; the reading taken is e4m3 Q, K, V with one
scale per (tensor, batch, head), P rounded to e4m3 on the way into the PV
product, fp32 accumulation).

* bsa_quantize_e4m3: codes and scales bit-exact against the oracle.
* bsa_draft_mask_natural_e4m3 (the draft mask and the quantization in one
  call, the maxima of Q and K taken by the pooling): every output identical,
  bit for bit, to the two separate calls.
* bsa_attn_fwd_natural_e4m3: against the fp64 oracle run on the dequantized
  inputs.  What is left is mostly the e4m3 rounding of P: a relative error
  of at most 2^-4 per weight, of either sign, so it largely cancels in the
  weighted sum over thousands of keys.  Bound used: max-abs 3e-2, mean-abs
  3e-3 (the bf16 path's bound is 2e-2 / 2e-3).
* Quality against the bf16 path: relative RMS difference below 8 %.  That
  difference is the quantization itself, not the kernel: an e4m3 value
  carries a relative rounding error uniform in +-2^-4 (RMS 2^-4/sqrt(3),
  about 3.6 %), and Q, K, V and P each pass through it.  Measured: 5.3 % at
  the Wan-1.3B-shape draft workload.
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

from gpu_util import LSE_ABS, sample_blocks, to_np64

pytestmark = pytest.mark.gpu

MAX_ABS_E4M3 = 3e-2
MEAN_ABS_E4M3 = 3e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    bsa.load()


def _codes_to_values(x8: torch.Tensor) -> np.ndarray:
    return x8.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()


@pytest.mark.parametrize("over", [dict(cid=5, Hh=4), dict(cid=2, T=3, H=13, W=37, Hh=3,
                                                             field_grid=(3, 4, 7)),
                                  dict(cid=1, qk="iid", D=64)])
def test_quantize_e4m3_bit_exact(over):
    over = dict(over)
    w = small_workload(CONFIGS[over.pop("cid")], **over)
    q, k, v = make_qkv(w, device="cuda")
    v = v * 3.0                                   # a different range per tensor
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_FRAME, block=128)
    q8, k8, v8 = (torch.empty(x.shape, dtype=torch.uint8, device="cuda") for x in (q, k, v))
    scales = torch.full((3, w.B, w.Hh), float("nan"), dtype=torch.float32, device="cuda")
    bsa.bsa_quantize_e4m3(plan, q, k, v, q8, k8, v8, scales)
    bsa.bsa_poll_status(plan)
    for i, (x, x8) in enumerate(((q, q8), (k, k8), (v, v8))):
        xn = to_np64(x)
        s_ref = oracle.fp8_scales(xn)
        np.testing.assert_array_equal(scales[i].cpu().numpy(), s_ref)
        np.testing.assert_array_equal(_codes_to_values(x8), oracle.fp8_quantize(xn, s_ref))


@pytest.mark.parametrize("over", [dict(cid=5, Hh=4),
                                  dict(cid=2, T=3, H=13, W=37, Hh=3, field_grid=(3, 4, 7)),
                                  dict(cid=1, qk="iid", D=64),
                                  dict(cid=2, T=2, H=20, W=12, Hh=2, D=64, draft_ph=16,
                                       draft_pw=8, field_grid=(2, 4, 7))])
@pytest.mark.parametrize("pooling", [bsa.POOL_MEAN, bsa.POOL_MAX])
def test_draft_mask_and_quantize_in_one_call_equal_the_two_calls(over, pooling):
    over = dict(over)
    w = small_workload(CONFIGS[over.pop("cid")], **over)
    q, k, v = make_qkv(w, device="cuda")
    v = v * 3.0
    ph, pw, sp = w.draft_ph, w.draft_pw, w.draft_sparsity
    plan = bsa.Plan(w.B, w.Hh, w.D, w.T, w.H, w.W, bsa.LAYOUT_TILE, ph, pw, ph * pw)
    bsa.bsa_plan_set_draft_pooling(plan, pooling)
    keep = bsa.bsa_draft_keep_count(plan, sp)
    rows = w.B * w.Hh * plan.nblocks

    def outputs():
        rp = torch.full((rows + 1,), -1, dtype=torch.int32, device="cuda")
        kv = torch.full((rows * keep,), -1, dtype=torch.int32, device="cuda")
        dm = torch.full((rows * plan.nblocks,), float("nan"), dtype=torch.float32, device="cuda")
        ws = torch.empty(((bsa.bsa_draft_workspace_bytes(plan) + 7) // 8,), dtype=torch.float64,
                         device="cuda")
        x8 = [torch.full(x.shape, 0x7f, dtype=torch.uint8, device="cuda") for x in (q, k, v)]
        sc = torch.full((3, w.B, w.Hh), float("nan"), dtype=torch.float32, device="cuda")
        return rp, kv, dm, ws, x8, sc

    rp, kv, dm, ws, x8, sc = outputs()
    bsa.bsa_draft_mask_natural(plan, q, k, sp, rp, kv, dm, ws)
    bsa.bsa_quantize_e4m3(plan, q, k, v, *x8, sc)
    rp1, kv1, dm1, ws1, y8, sc1 = outputs()
    bsa.bsa_draft_mask_natural_e4m3(plan, q, k, v, sp, rp1, kv1, dm1, ws1, *y8, sc1)
    bsa.bsa_poll_status(plan)
    assert torch.equal(rp, rp1) and torch.equal(kv, kv1) and torch.equal(dm, dm1)
    assert torch.equal(sc, sc1)
    for a, b in zip(x8, y8):
        assert torch.equal(a, b)


def _e4m3_case(w, q_blocks=None, heads=None):
    q, k, v = make_qkv(w, device="cuda")
    att = DraftAttention(w.B, w.Hh, w.D, w.T, w.H, w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    lse = torch.full((w.B, w.Hh, w.N), float("nan"), dtype=torch.float32, device="cuda")
    out8 = att.fused_e4m3(q, k, v, None, lse)
    bsa.bsa_poll_status(att.plan)
    heads = list(range(w.Hh)) if heads is None else heads
    ph, pw = w.draft_ph, w.draft_pw
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, ph, pw)
    valid = oracle.slot_valid(perm, Np)
    nb = Np // (ph * pw)
    # the oracle on the values the 8-bit kernel computes with
    sc = att.fp8_scales.cpu().numpy()
    deq = [oracle.fp8_dequantize(_codes_to_values(x8), sc[i])[:, :, heads]
           for i, x8 in enumerate((att.q8, att.k8, att.v8))]
    kv = att.col_idx.view(w.B, w.Hh, nb, -1)[:, heads].cpu().numpy()
    rp, ci = oracle.fixed_k_csr(kv)
    O, L = oracle.masked_attention(*(oracle.reorder_fwd(x, perm, Np) for x in deq), valid,
                                   ph * pw, rp, ci, True, 1 / math.sqrt(w.D), q_blocks=q_blocks)
    ref = oracle.reorder_inv(np.nan_to_num(O, nan=np.inf), perm)
    got = to_np64(out8[:, :, heads])
    m = np.isfinite(ref)
    assert m.any()
    err = np.abs(got[m] - ref[m])
    # the log-sum-exp of the scores on the dequantized values (S * sq * sk
    # times the softmax scale): P's rounding does not enter it
    lref = np.nan_to_num(L, nan=np.inf)[:, :, perm]
    lgot = lse[:, heads].double().cpu().numpy()
    ml = np.isfinite(lref)
    assert ml.any()
    assert np.abs(lgot[ml] - lref[ml]).max() <= LSE_ABS
    return q, k, v, att, out8, err


@pytest.mark.parametrize("over", [dict(cid=2, T=3, H=13, W=37, Hh=3, field_grid=(3, 4, 7)),
                                  dict(cid=2, T=2, H=9, W=70, Hh=2, draft_ph=4, draft_pw=32,
                                       draft_sparsity=70, field_grid=(2, 4, 7))])
def test_attn_e4m3_small_all_tokens(over):
    over = dict(over)
    w = small_workload(CONFIGS[over.pop("cid")], **over)
    *_, err = _e4m3_case(w)
    assert err.max() <= MAX_ABS_E4M3, err.max()
    assert err.mean() <= MEAN_ABS_E4M3, err.mean()


@pytest.mark.parametrize("T", [256, 300])
def test_attn_e4m3_lists_at_and_past_the_bin_limit(T):
    # 6 x 10 frames: one 60-token corner tile each, two to a packed MMA tile;
    # every block kept: 128 packed tiles (the most a list buffer holds) at
    # T = 256, and an unpacked list at T = 300
    w = small_workload(CONFIGS[2], T=T, H=6, W=10, Hh=1, draft_sparsity=0, field_grid=(16, 2, 3))
    *_, err = _e4m3_case(w, q_blocks=[0, 1, T // 2, T - 1])
    assert err.max() <= MAX_ABS_E4M3, err.max()
    assert err.mean() <= MEAN_ABS_E4M3, err.mean()


@pytest.mark.parametrize("cid", [2, 5])
def test_attn_e4m3_full_size_sampled(cid):
    w = CONFIGS[cid]
    nb = w.T * -(-w.H // w.draft_ph) * -(-w.W // w.draft_pw)
    q, k, v, att, out8, err = _e4m3_case(w, q_blocks=sample_blocks(nb, 6, seed=cid),
                                         heads=[0, w.Hh - 1])
    assert err.max() <= MAX_ABS_E4M3, err.max()
    assert err.mean() <= MEAN_ABS_E4M3, err.mean()
    # quality against the bf16 path on every token
    ref16 = att.fused(q, k, v).float()
    rel = ((out8.float() - ref16).pow(2).mean() / ref16.pow(2).mean()).sqrt().item()
    assert rel < 0.08, rel


def test_attn_e4m3_rejects_unsupported_plans():
    x = torch.zeros((1, 512, 1, 64), dtype=torch.uint8, device="cuda")
    o = torch.zeros((1, 512, 1, 64), dtype=torch.bfloat16, device="cuda")
    sc = torch.ones(3, dtype=torch.float32, device="cuda")
    buf = torch.zeros(4096, dtype=torch.int32, device="cuda")
    p64 = bsa.Plan(1, 1, 64, 2, 16, 16, bsa.LAYOUT_TILE, 8, 16, 128)    # D = 64
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_attn_fwd_natural_e4m3(p64, x, x, x, sc, buf, buf, True, 0.125, o)
    assert ei.value.status == 2
