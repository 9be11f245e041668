"""Statistics of the masks on the synthetic workloads, recomputed from the
oracle (CPU).  They explain the executed-versus-attended work of the
attention kernels; they are not parity evidence.

* Draft lists (Wan-1.3B-shape draft workload, 12 heads, 34 of 336 blocks
  kept per row): a query block shares few kept blocks with its neighbours
  (6.7 with the right one, 8.4 with the lower one, 10.3 with its best partner
  in the frame), so two query tiles sharing K/V would execute far more MMAs.
* The top-k favours partly empty edge blocks (57.5 % of the kept blocks
  against 43.8 % of all blocks): a kept key block is 65 % full on average,
  and 49.6 % of the executed attention work is attended.
* The one-kernel LVSA tiling (256 queries per CTA; the runs of consecutive
  frames of the union of the CTA's frame sets laid end to end at 8-row
  boundaries and cut into 128-row key tiles) at the Wan-1.3B 6x workload:
  99.3 % of the multiplied pairs are attended, CTAs straddling two frames
  cost 0.6 points.  With each run starting on a whole key tile, the share
  was 96.0 % at steps 0-5 and 96.4 % at steps 6-11 (run tail tiles 3.4 and
  3.0 points with 11 and 10 anchors).
* The two readings of the window's growth order (alternating pointers, the
  default, and distance order) differ on 5 of 32 rows of
  the tiny workload, 570 of 1512 at Wan-1.3B 6x and 3 of 1040 at
  HunyuanVideo 2x.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import CONFIGS, make_qkv


@pytest.fixture(scope="module")
def draft_case():
    w = CONFIGS[2]
    q, k, _ = make_qkv(w)
    kv = oracle.draft_blocks(q.to(torch.float64).numpy(), k.to(torch.float64).numpy(), w.T, w.H,
                             w.W, w.draft_ph, w.draft_pw, w.draft_sparsity)
    return w, kv


def _grid(w):
    return -(-w.H // w.draft_ph), -(-w.W // w.draft_pw)


def test_draft_lists_of_neighbouring_query_blocks_share_few_blocks(draft_case):
    w, kv = draft_case
    TH, TW = _grid(w)
    _, Hh, nb, keep = kv.shape
    assert keep == 34 and nb == 336
    right, below, best = [], [], []
    for h in range(Hh):
        for blk in range(nb):
            t, r = divmod(blk, TH * TW)
            i, j = divmod(r, TW)
            own = kv[0, h, blk]
            if j + 1 < TW:
                right.append(len(np.intersect1d(own, kv[0, h, blk + 1])))
            if i + 1 < TH:
                below.append(len(np.intersect1d(own, kv[0, h, blk + TW])))
            f0 = t * TH * TW
            best.append(max(len(np.intersect1d(own, kv[0, h, o]))
                            for o in range(f0, f0 + TH * TW) if o != blk))
    assert np.mean(right) == pytest.approx(6.7, abs=0.1)
    assert np.mean(below) == pytest.approx(8.4, abs=0.1)
    assert np.mean(best) == pytest.approx(10.3, abs=0.1)


def test_top_k_favours_partly_empty_edge_blocks(draft_case):
    w, kv = draft_case
    TH, TW = _grid(w)
    ph, pw = w.draft_ph, w.draft_pw
    nvalid = np.array([min(ph, w.H - i * ph) * min(pw, w.W - j * pw)
                       for _ in range(w.T) for i in range(TH) for j in range(TW)])
    kept = nvalid[kv]
    assert (kept < 128).mean() == pytest.approx(0.575, abs=0.005)
    assert (nvalid < 128).mean() == pytest.approx(0.438, abs=0.001)
    assert kept.mean() / 128 == pytest.approx(0.65, abs=0.005)
    attended = (nvalid[None, None, :, None] * kept).sum()
    assert attended / (128 * 128 * kv.size) == pytest.approx(0.496, abs=0.002)


def _lvsa_tiling(w, s, pack=True):
    """Multiplied and attended pairs of the one-kernel LVSA tiling: 256
    queries per CTA; the runs of consecutive frames of the union of their
    frame sets laid end to end, each starting on the next 8-row boundary
    (pack) or on the next 128-row boundary, cut into 128-row key tiles."""
    T, P = w.T, w.H * w.W
    N = T * P
    A = [set(int(f) for f in r) for r in oracle.lvsa_frame_sets(T, w.lvsa_C, w.lvsa_T_per, s)]
    executed = attended = tails = straddle = 0
    for q0 in range(0, N, 256):
        rows = range(q0, min(q0 + 256, N))
        U = set().union(*(A[t] for t in {n // P for n in rows}))
        runs = []
        for f in sorted(U):
            if runs and runs[-1][1] == f - 1:
                runs[-1][1] = f
            else:
                runs.append([f, f])
        align = 8 if pack else 128
        v = 0
        for a, b in runs:
            v = -(-(v + (b - a + 1) * P) // align) * align
        keys = -(-v // 128) * 128
        executed += 256 * keys
        attended += sum(len(A[n // P]) * P for n in rows)
        tails += 256 * (keys - len(U) * P)
        straddle += sum((len(U) - len(A[n // P])) * P for n in rows)
    return attended / executed, tails / executed, straddle / executed


def test_lvsa_one_kernel_tiling_attends_99_percent():
    w = CONFIGS[3]
    for s in (0, 5, 6, 11):
        frac, tails, straddle = _lvsa_tiling(w, s)
        assert frac == pytest.approx(0.993, abs=0.001)
        assert tails == pytest.approx(0.0007, abs=0.0002)
        assert straddle == pytest.approx(0.006, abs=0.001)
    # runs starting on whole key tiles: each run's last tile is partly empty
    early = [_lvsa_tiling(w, s, pack=False) for s in (0, 5)]   # 11 anchors
    late = [_lvsa_tiling(w, s, pack=False) for s in (6, 11)]   # 10 anchors
    for frac, tails, _ in early:
        assert frac == pytest.approx(0.960, abs=0.001)
        assert tails == pytest.approx(0.034, abs=0.001)
    for frac, tails, _ in late:
        assert frac == pytest.approx(0.964, abs=0.001)
        assert tails == pytest.approx(0.030, abs=0.001)


def test_the_two_window_readings_differ_on_the_stated_rows():
    # rows (t, s) where reading A (distance order) and reading B (alternating
    # pointers) give different frame sets, over one anchor period
    expect = {1: (5, 32), 3: (570, 1512), 4: (3, 1040)}
    for cid, (n_diff, n_rows) in expect.items():
        w = CONFIGS[cid]
        diff = rows = 0
        for s in range(w.lvsa_T_per):
            a = oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, s, order="distance")
            b = oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, s, order="alternate")
            diff += int((a != b).any(axis=1).sum())
            rows += w.T
        assert (diff, rows) == (n_diff, n_rows)
