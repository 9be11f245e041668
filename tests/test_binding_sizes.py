"""The binding rejects tensors smaller than the plan implies, before any
call into the library (the kernels take every size from the plan).

CPU-only: a stand-in plan carries the geometry, and CPU tensors of exactly
the required sizes must get past the size checks to the device check
("must live on a CUDA device"), while one element fewer in any one tensor
must be refused for its size.  Sizes: natural layout [B, N, Hh, D], slot
layout [B, Hh, Npad, D]; bf16 2 bytes, e4m3 1 byte, int32 / fp32 4 bytes.
"""
import types

import pytest
import torch

import block_sparse_attention_49_b200 as bsa
from block_sparse_attention_49_b200 import _build


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    bsa.load()

# FRAME-like geometry: 3 frames of 5 x 7 tokens, 32-token blocks -> 2 blocks
# per frame, 6 blocks, 256 slots
P = types.SimpleNamespace(B=2, Hh=3, D=64, T=3, H=5, W=7, Npad=256, nblocks=6, handle=None,
                         keep_count=lambda sp: -(-6 * (100 - sp) // 100))
N = P.T * P.H * P.W
NAT = (P.B, N, P.Hh, P.D)
SLOT = (P.B, P.Hh, P.Npad, P.D)
ROWS = P.B * P.Hh * P.nblocks


def bf(shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def u8(shape):
    return torch.zeros(shape, dtype=torch.uint8)


def i32(n):
    return torch.zeros(n, dtype=torch.int32)


def f32(n):
    return torch.zeros(n, dtype=torch.float32)


def _keep(sp):
    return -(-P.nblocks * (100 - sp) // 100)


# (wrapper, positional args with exact sizes, names of the tensor arguments to shorten)
CASES = {
    "lvsa_mask": (bsa.bsa_lvsa_mask,
                  lambda: [P, 2, 4, 0, i32(P.T * 2), i32(P.nblocks + 1), i32(P.nblocks * 2 * 2)],
                  [4, 5, 6]),
    "draft_mask": (bsa.bsa_draft_mask,
                   lambda: [P, bf(SLOT), bf(SLOT), 50, i32(ROWS + 1), i32(ROWS * _keep(50)),
                            f32(ROWS * P.nblocks), torch.zeros(1, dtype=torch.float64)],
                   [1, 2, 4, 5, 6]),
    "draft_mask_noalloc": (bsa.bsa_draft_mask_noalloc,
                           lambda: [P, bf(SLOT), bf(SLOT), 90, i32(ROWS + 1),
                                    i32(ROWS * _keep(90)), None],
                           [1, 2, 4, 5]),
    "draft_mask_natural": (bsa.bsa_draft_mask_natural,
                           lambda: [P, bf(NAT), bf(NAT), 90, None, i32(ROWS * _keep(90)),
                                    f32(ROWS * P.nblocks), torch.zeros(1, dtype=torch.float64)],
                           [1, 2, 5, 6]),
    "reorder_fwd": (bsa.bsa_reorder_fwd,
                    lambda: [P, bf(NAT), bf(SLOT), bf(NAT), bf(SLOT), bf(NAT), bf(SLOT)],
                    [1, 2, 3, 4, 5, 6]),
    "reorder_inv": (bsa.bsa_reorder_inv, lambda: [P, bf(SLOT), bf(NAT)], [1, 2]),
    "attn_fwd_shared": (bsa.bsa_attn_fwd,
                        lambda: [P, bf(SLOT), bf(SLOT), bf(SLOT), i32(P.nblocks + 1), i32(1),
                                 False, 0.125, bf(SLOT), f32(P.B * P.Hh * P.Npad)],
                        [1, 2, 3, 4, 8, 9]),
    "attn_fwd_per_head": (bsa.bsa_attn_fwd,
                          lambda: [P, bf(SLOT), bf(SLOT), bf(SLOT), i32(ROWS + 1), i32(1), True,
                                   0.125, bf(SLOT), None],
                          [4]),
    "attn_fwd_natural": (bsa.bsa_attn_fwd_natural,
                         lambda: [P, bf(NAT), bf(NAT), bf(NAT), i32(ROWS + 1), i32(1), True,
                                  0.125, bf(NAT), f32(P.B * P.Hh * N)],
                         [1, 2, 3, 4, 8, 9]),
    "quantize_e4m3": (bsa.bsa_quantize_e4m3,
                      lambda: [P, bf(NAT), bf(NAT), bf(NAT), u8(NAT), u8(NAT), u8(NAT),
                               f32(3 * P.B * P.Hh)],
                      [1, 2, 3, 4, 5, 6, 7]),
    "attn_fwd_natural_e4m3": (bsa.bsa_attn_fwd_natural_e4m3,
                              lambda: [P, u8(NAT), u8(NAT), u8(NAT), f32(3 * P.B * P.Hh),
                                       i32(ROWS + 1), i32(1), True, 0.125, bf(NAT),
                                       f32(P.B * P.Hh * N)],
                              [1, 2, 3, 4, 5, 9, 10]),
    "lvsa_attn_fwd": (bsa.bsa_lvsa_attn_fwd,
                      lambda: [P, 2, 4, 0, bf(NAT), bf(NAT), bf(NAT), 0.125, bf(NAT),
                               f32(P.B * P.Hh * N)],
                      [4, 5, 6, 8, 9]),
}


def _short(t):
    return t.reshape(-1)[1:].clone()


@pytest.mark.parametrize("name", list(CASES))
def test_exact_sizes_pass_the_size_checks(name):
    fn, make, _ = CASES[name]
    with pytest.raises(ValueError, match="CUDA device"):
        fn(*make())


@pytest.mark.parametrize("name", list(CASES))
def test_one_element_short_is_refused(name):
    fn, make, idx = CASES[name]
    for i in idx:
        args = make()
        args[i] = _short(args[i])
        with pytest.raises(ValueError, match="the plan needs"):
            fn(*args)
