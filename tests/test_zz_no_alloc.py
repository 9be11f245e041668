"""bsa_draft_mask_noalloc: the draft mask for callers that cannot allocate.

Some callers cannot allocate device memory of their own (a plugin whose host
program owns every allocation and passes only input and output buffers; a
caller on a fixed memory budget).  bsa_draft_mask_noalloc computes what
bsa_draft_mask computes, with its scratch in a fixed 48 MiB array inside the
library instead of a caller workspace.  Here it is called through the C ABI
twice in a row, on two different problems, and each time its outputs must
equal those of bsa_draft_mask on the same inputs (block lists bit for bit,
draft map within the tolerance the other draft tests use).  This file is
named so that pytest collects it last.
"""
import pytest
import torch

import block_sparse_attention_49_b200 as bsa
from block_sparse_attention_49_b200 import _build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    bsa.load()


def _case(T, H, W, Hh, D, ph, pw, sparsity, seed):
    plan = bsa.Plan(1, Hh, D, T, H, W, bsa.LAYOUT_TILE, ph, pw, ph * pw)
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = (1, Hh, plan.Npad, D)
    q = torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)
    return plan, q, k, sparsity


def _outputs(plan, keep):
    rows = plan.B * plan.Hh * plan.nblocks
    rp = torch.full((rows + 1,), -1, dtype=torch.int32, device="cuda")
    kv = torch.full((rows * keep,), -1, dtype=torch.int32, device="cuda")
    dm = torch.full((rows * plan.nblocks,), float("nan"), dtype=torch.float32, device="cuda")
    return rp, kv, dm


@pytest.mark.parametrize("precision", [bsa.DRAFT_FP64, bsa.DRAFT_FP32])
def test_noalloc_matches_workspace_version_on_two_calls_in_a_row(precision):
    cases = [_case(21, 30, 52, 12, 128, 8, 16, 90, seed=1),   # Wan-1.3B-like native grid
             _case(3, 20, 36, 4, 64, 4, 8, 75, seed=2)]       # smaller, other head dim
    for plan, _, _, _ in cases:
        bsa.bsa_plan_set_draft_precision(plan, precision)
    got = []
    for plan, q, k, sp in cases:
        keep = bsa.bsa_draft_keep_count(plan, sp)
        rp, kv, dm = _outputs(plan, keep)
        bsa.bsa_draft_mask_noalloc(plan, q, k, sp, rp, kv, dm)
        got.append((rp, kv, dm))
    torch.cuda.synchronize()
    for (plan, q, k, sp), (rp, kv, dm) in zip(cases, got):
        bsa.bsa_poll_status(plan)
        keep = bsa.bsa_draft_keep_count(plan, sp)
        rp0, kv0, dm0 = _outputs(plan, keep)
        ws = torch.empty(((bsa.bsa_draft_workspace_bytes(plan) + 7) // 8,), dtype=torch.float64,
                         device="cuda")
        bsa.bsa_draft_mask(plan, q, k, sp, rp0, kv0, dm0, ws)
        bsa.bsa_poll_status(plan)
        assert torch.equal(kv, kv0)
        assert torch.equal(rp, rp0)
        assert torch.equal(dm, dm0)          # same kernels on the same inputs: same bits
        assert (kv >= 0).all() and (kv < plan.nblocks).all()


def test_noalloc_rejects_problems_above_its_scratch():
    cap = bsa.bsa_draft_noalloc_max_scratch_bytes()
    assert cap == 48 << 20
    # 40 heads on a 21 x 60 x 104 grid in 8 x 16 tiles: 1344 blocks, 165 MB of scratch
    plan = bsa.Plan(1, 40, 128, 21, 60, 104, bsa.LAYOUT_TILE, 8, 16, 128)
    assert bsa.bsa_draft_workspace_bytes(plan) > cap
    buf = torch.empty(16, dtype=torch.int32, device="cuda")
    x = torch.empty(8, dtype=torch.bfloat16, device="cuda")
    # raw addresses: the binding's size checks pass them through, so the
    # library's own scratch-size check is the one that answers
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_draft_mask_noalloc(plan, x.data_ptr(), x.data_ptr(), 90, buf.data_ptr(),
                                   buf.data_ptr(), None)
    assert ei.value.status == 2
    assert "48 MiB" in bsa.bsa_last_error()
