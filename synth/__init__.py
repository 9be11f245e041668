"""Seeded synthetic workloads shared by the CPU oracle and the CUDA path.

This module holds the five workload configurations (shapes, mask parameters)
and the generator of the bf16 Q/K/V tensors.  It contains none of the method's
arithmetic: no masks, no pooling, no attention.  Both sides of every parity
check consume the very same tensors produced here.

Workloads stand in for the video-DiT attention inputs the pages measure on
(Wan 2.1 1.3B/14B latent grids at native and 6x length, HunyuanVideo 1.5 at
2x length: "LVSA: Training-Free Sparse Attention for Long Video Diffusion",
section 4 "Computational efficiency"; Draft Attention article, experiments at
90% sparsity).  No model weights or datasets are used: Q and K are a smooth
random field plus noise so that the draft map has real structure, V is noise.

Natural layout of every tensor: [B, N, Hh, D] bf16, token n = (t*H + y)*W + x.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Tuple

import torch

__all__ = ["Workload", "CONFIGS", "make_qkv", "seed_of"]


@dataclass(frozen=True)
class Workload:
    cid: int
    name: str
    B: int
    Hh: int
    D: int
    T: int
    H: int
    W: int
    # "iid": Q, K, V i.i.d. N(0,1).  "field": Q, K = rmsnorm(0.7*up(field)+0.3*noise)
    qk: str = "field"
    field_grid: Optional[Tuple[int, int, int]] = None
    # LVSA frame mask: budget C, rotation period T_per, KV block size (tokens)
    lvsa_C: Optional[int] = None
    lvsa_T_per: Optional[int] = None
    lvsa_block: Optional[int] = None
    # draft mask: pooling tile and sparsity (percent of blocks dropped)
    draft_ph: Optional[int] = None
    draft_pw: Optional[int] = None
    draft_sparsity: Optional[int] = None
    # full dense mask (parity with dense attention), on the frame layout
    dense: bool = False
    dense_block: int = 128

    @property
    def P(self) -> int:
        return self.H * self.W

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def lvsa_steps(self) -> range:
        return range(self.lvsa_T_per) if self.lvsa_T_per else range(0)


CONFIGS = {
    1: Workload(1, "tiny 1x2x64, grid 8x8x8", B=1, Hh=2, D=64, T=8, H=8, W=8, qk="iid",
                lvsa_C=4, lvsa_T_per=4, lvsa_block=64,
                draft_ph=2, draft_pw=2, draft_sparsity=50),
    2: Workload(2, "Wan2.1-1.3B-like native, 12x128, grid 21x30x52", B=1, Hh=12, D=128,
                T=21, H=30, W=52, field_grid=(21, 4, 7),
                draft_ph=8, draft_pw=16, draft_sparsity=90, dense=True),
    3: Workload(3, "Wan2.1-1.3B-like 6x length LVSA, 12x128, grid 126x30x52", B=1, Hh=12,
                D=128, T=126, H=30, W=52, field_grid=(126, 4, 7),
                lvsa_C=21, lvsa_T_per=12, lvsa_block=128),
    4: Workload(4, "HunyuanVideo-1.5-like 2x length LVSA, 16x128, grid 65x45x80", B=1,
                Hh=16, D=128, T=65, H=45, W=80, field_grid=(65, 6, 10),
                lvsa_C=33, lvsa_T_per=16, lvsa_block=128),
    5: Workload(5, "Wan2.1-14B-like native draft, 40x128, grid 21x30x52", B=1, Hh=40,
                D=128, T=21, H=30, W=52, field_grid=(21, 4, 7),
                draft_ph=8, draft_pw=16, draft_sparsity=90),
}

# sub-stream numbers of the per-config seed
_STREAM = {"q": 0, "k": 1, "v": 2, "qfield": 3, "kfield": 4}


def seed_of(cid: int, stream: str) -> int:
    """Seed of one sub-stream: base seed 49000 + config number."""
    return (49000 + cid) * 16 + _STREAM[stream]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, seed: int, device) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(seed, device), device=device,
                       dtype=torch.float32)


def _field_tokens(w: Workload, seed: int, device, h0: int, h1: int) -> torch.Tensor:
    """Trilinear upsample of an N(0,1) field on the coarse grid, heads [h0,h1).

    Returns float32 [B, N, h1-h0, D].  The coarse field for all heads is drawn at
    once from the seed, so any head range gives the same values.
    """
    Tc, Hc, Wc = w.field_grid
    coarse = _randn((w.B, w.Hh * w.D, Tc, Hc, Wc), seed, device)
    c = coarse[:, h0 * w.D:h1 * w.D]
    up = torch.nn.functional.interpolate(c, size=(w.T, w.H, w.W), mode="trilinear",
                                         align_corners=False)
    # [B, (h d), T, H, W] -> [B, N, h, d]
    up = up.reshape(w.B, h1 - h0, w.D, w.N).permute(0, 3, 1, 2)
    return up


def _rmsnorm_bf16(x: torch.Tensor) -> torch.Tensor:
    """Per (token, head) RMS normalisation over D in fp32, then bf16 (RNE)."""
    x = x / torch.sqrt(x.pow(2).mean(dim=-1, keepdim=True) + 1e-6)
    return x.to(torch.bfloat16)


def make_qkv(w: Workload, device="cpu", heads_per_chunk: int = 4):
    """Generate Q, K, V in natural layout [B, N, Hh, D] bf16 on `device`.

    Deterministic for a given device type: the same (config, device type)
    always yields the same bytes.  The head-chunk size is part of that: the
    field is the same under any chunking, but the fp32 RMS reduction's order
    follows the chunk's shape, so another chunk size can move a few elements
    by one bf16 rounding step.  Every parity check hands the very same
    tensors to both sides, so this never enters a comparison.
    """
    dev = torch.device(device)
    shape = (w.B, w.N, w.Hh, w.D)
    out = []
    for name in ("q", "k"):
        if w.qk == "iid":
            out.append(_randn(shape, seed_of(w.cid, name), dev).to(torch.bfloat16))
            continue
        noise = _randn(shape, seed_of(w.cid, name), dev)
        t = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        for h0 in range(0, w.Hh, heads_per_chunk):
            h1 = min(w.Hh, h0 + heads_per_chunk)
            f = _field_tokens(w, seed_of(w.cid, name + "field"), dev, h0, h1)
            t[:, :, h0:h1] = _rmsnorm_bf16(0.7 * f + 0.3 * noise[:, :, h0:h1])
            del f
        del noise
        out.append(t)
    out.append(_randn(shape, seed_of(w.cid, "v"), dev).to(torch.bfloat16))
    return tuple(out)


def small_workload(base: Workload, **over) -> Workload:
    """A copy of `base` with some fields replaced (for reduced-size tests)."""
    d = {f: getattr(base, f) for f in base.__dataclass_fields__}
    d.update(over)
    return Workload(**d)
