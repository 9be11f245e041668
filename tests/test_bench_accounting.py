"""The attended-FLOP counts bench.py divides by: 4*D per (valid query,
valid key) pair, checked against the oracle's pair count over the block
lists (CPU only)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from synth import CONFIGS, small_workload  # noqa: E402


def test_lvsa_attended_flops_match_pair_count():
    for w in (CONFIGS[1], small_workload(CONFIGS[3], T=14, H=5, W=29, Hh=3, lvsa_C=5,
                                         lvsa_T_per=4)):
        perm, Np = oracle.frame_layout_perm(w.T, w.H, w.W, 128)
        valid = oracle.slot_valid(perm, Np)
        for s in (0, 1):
            rp, ci = oracle.lvsa_block_csr(oracle.lvsa_frame_sets(w.T, w.lvsa_C, w.lvsa_T_per, s),
                                           -(-w.P // 128))
            pairs = oracle.attended_pairs(valid, 128, rp, ci)
            assert bench.attended_flops(w) == 4.0 * w.D * pairs * w.Hh * w.B


def test_draft_attended_flops_match_pair_count():
    w = small_workload(CONFIGS[2], B=2, T=2, H=13, W=37, Hh=3)
    ph, pw = w.draft_ph, w.draft_pw
    perm, Np = oracle.tile_layout_perm(w.T, w.H, w.W, ph, pw)
    valid = oracle.slot_valid(perm, Np)
    nb = Np // (ph * pw)
    keep = 4
    rng = np.random.default_rng(8)
    kv = np.sort(np.stack([rng.choice(nb, keep, replace=False)
                           for _ in range(w.B * w.Hh * nb)]), axis=1)
    kv = kv.reshape(w.B, w.Hh, nb, keep).astype(np.int32)
    rp, ci = oracle.fixed_k_csr(kv)
    pairs = oracle.attended_pairs(valid, ph * pw, rp, ci, nlists=w.B * w.Hh)
    assert bench.draft_attended_flops(w, kv.reshape(-1), keep) == 4.0 * w.D * pairs
