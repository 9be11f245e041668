"""The seeded input generator follows its stated recipe (CPU).

Q, K = RMSnorm(0.7 * up(F) + 0.3 * N(0,1)) per (token, head) over D, then
bf16; F an N(0,1) field on a coarse grid, upsampled trilinearly; V and the
tiny workload's Q, K i.i.d. N(0,1).  Checked: shapes and dtype, determinism,
the head chunking (the field bit for bit, the values within one bf16
rounding step), the per-(token, head) RMS, the moments of
the i.i.d. tensors, the spatial correlation the field gives (and its absence
for i.i.d. inputs), and that Q and K are drawn independently.
"""
import math

import torch

from synth import CONFIGS, _field_tokens, make_qkv, seed_of, small_workload

W_FIELD = small_workload(CONFIGS[2], T=3, H=12, W=16, Hh=3, field_grid=(3, 4, 7))
W_IID = CONFIGS[1]


def _f(x):
    return x.to(torch.float64)


def test_shapes_dtype_and_determinism():
    for w in (W_FIELD, W_IID):
        a = make_qkv(w)
        b = make_qkv(w)
        for x, y in zip(a, b):
            assert x.shape == (w.B, w.N, w.Hh, w.D) and x.dtype == torch.bfloat16
            assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_head_chunking_keeps_the_field_and_moves_at_most_one_rounding_step():
    # the coarse field of all heads is drawn at once: any head range gives
    # the same field values, bit for bit
    seed = seed_of(W_FIELD.cid, "qfield")
    whole = _field_tokens(W_FIELD, seed, "cpu", 0, W_FIELD.Hh)
    parts = torch.cat([_field_tokens(W_FIELD, seed, "cpu", h, h + 1) for h in range(W_FIELD.Hh)],
                      dim=2)
    assert torch.equal(whole, parts)
    # the normalised bf16 values: the same up to one bf16 step in a few places
    a = make_qkv(W_FIELD, heads_per_chunk=1)
    b = make_qkv(W_FIELD, heads_per_chunk=4)
    for x, y in zip(a, b):
        d = (_f(x) - _f(y)).abs()
        step = _f(y).abs().clamp_min(2 ** -126) * 2 ** -7
        assert (d <= step).all()
        assert (d > 0).double().mean().item() < 1e-3


def test_field_inputs_are_rms_normalised_per_token_and_head():
    q, k, _ = make_qkv(W_FIELD)
    for x in (q, k):
        rms = _f(x).pow(2).mean(dim=-1).sqrt()
        # bf16 rounding moves each element by at most 2^-8 relative
        assert (rms - 1).abs().max().item() < 2 ** -7


def test_iid_tensors_have_unit_normal_moments():
    q, k, v = make_qkv(W_IID)
    _, _, v2 = make_qkv(W_FIELD)
    for x in (q, k, v, v2):
        x = _f(x).flatten()
        n = x.numel()
        assert abs(x.mean().item()) < 5 / math.sqrt(n)
        assert abs(x.var().item() - 1) < 5 * math.sqrt(2 / n)


def _neighbour_cosine(x, w):
    # cosine of each token's head vector with its right neighbour in the row
    g = _f(x).reshape(w.B, w.T, w.H, w.W, w.Hh, w.D)
    a, b = g[:, :, :, :-1], g[:, :, :, 1:]
    cos = (a * b).sum(-1) / (a.norm(dim=-1) * b.norm(dim=-1))
    return cos.mean().item()


def test_field_gives_spatial_correlation_and_iid_does_not():
    q, k, v = make_qkv(W_FIELD)
    # the field carries 0.49 / 0.58 of the variance and neighbouring tokens
    # see nearly the same field value (7 coarse points over 16 columns here)
    assert _neighbour_cosine(q, W_FIELD) > 0.4
    assert _neighbour_cosine(k, W_FIELD) > 0.4
    assert abs(_neighbour_cosine(v, W_FIELD)) < 0.05
    qi, _, _ = make_qkv(W_IID)
    assert abs(_neighbour_cosine(qi, W_IID)) < 0.05


def test_q_and_k_are_drawn_independently():
    q, k, _ = make_qkv(W_FIELD)
    cos = (_f(q) * _f(k)).sum(-1) / (_f(q).norm(dim=-1) * _f(k).norm(dim=-1))
    assert abs(cos.mean().item()) < 0.05
