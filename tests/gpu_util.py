"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

# attention output tolerance against fp64 (bf16 inputs, fp32 accumulation)
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 2e-3


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def perm_of(w, layout: str, block: int | None = None):
    if layout == "frame":
        return oracle.frame_layout_perm(w.T, w.H, w.W, block)
    return oracle.tile_layout_perm(w.T, w.H, w.W, w.draft_ph, w.draft_pw)


def padded(Npad_oracle: int) -> int:
    return (Npad_oracle + 127) // 128 * 128


def sample_blocks(nb: int, n: int = 6, seed: int = 0):
    rng = np.random.default_rng(seed)
    pick = {0, 1, nb // 2, nb - 1}
    pick |= set(int(x) for x in rng.integers(0, nb, size=max(0, n - 4)))
    return sorted(b for b in pick if 0 <= b < nb)


def compare_attention(O_gpu: torch.Tensor, L_gpu: torch.Tensor | None, O_ref, L_ref, valid,
                      block: int, q_blocks, heads):
    """Element-wise check of the CUDA output against the oracle on the rows
    of the sampled query blocks / heads; pad slots must be 0 / -inf."""
    errs = []
    for b, h in heads:
        for qb in q_blocks:
            rows = np.arange(qb * block, (qb + 1) * block)
            og = to_np64(O_gpu[b, h, rows[0]:rows[-1] + 1])
            orf = O_ref[b, h, rows]
            vr = valid[rows]
            assert np.isfinite(og).all()
            assert (og[~vr] == 0).all(), "pad query slots must be zero"
            errs.append(np.abs(og[vr] - orf[vr]).reshape(-1))
            if L_gpu is not None:
                lg = L_gpu[b, h, rows[0]:rows[-1] + 1].double().cpu().numpy()
                lr = LSE_ref = L_ref[b, h, rows]
                assert np.isneginf(lg[~vr]).all()
                fin = np.isfinite(lr) & vr
                assert (np.isneginf(lg[vr & ~np.isfinite(LSE_ref)])).all()
                if fin.any():
                    assert np.abs(lg[fin] - lr[fin]).max() <= LSE_ABS, np.abs(lg[fin] - lr[fin]).max()
    e = np.concatenate(errs) if errs else np.zeros(1)
    assert e.max() <= MAX_ABS, f"max abs err {e.max()}"
    assert e.mean() <= MEAN_ABS, f"mean abs err {e.mean()}"
    return float(e.max()), float(e.mean())
