"""The e4m3 conversion behind bsa_quantize_e4m3 multiplies by the reciprocal
of the scale and divides only near e4m3 rounding boundaries.  This checks the
claim that makes that exact, with IEEE fp32 arithmetic on the host: wherever
y = x * fp32(1/s) lies in [2^-6, 448] and at least 4 units in the last place
from every e4m3 midpoint, y rounds to the same e4m3 value as the correctly
rounded quotient fp32(x / s).  Rounding to e4m3 is the oracle's.

The kernel's test on y is restated here (the 20 fp32 mantissa bits below the
three e4m3 ones read 0x80000 at a midpoint); the GPU tests then compare the
kernel's codes with the oracle's bit for bit.
"""
import numpy as np
import torch

import oracle


def _safe(y: np.ndarray) -> np.ndarray:
    a = y.view(np.uint32) & np.uint32(0x7FFFFFFF)
    d = (a & np.uint32(0xFFFFF)).astype(np.int64) - 0x80000
    return (a >= 0x3C800000) & (a <= 0x43E00000) & (np.abs(d) >= 4)


def _codes(v: np.ndarray) -> np.ndarray:
    return oracle.e4m3_round(v.astype(np.float64))


def _both(x: np.ndarray, s: np.ndarray):
    x = x.astype(np.float32)
    s = s.astype(np.float32)
    r = np.float32(1.0) / s                  # fp32(1/s), correctly rounded
    y = x * r                                # the product, rounded to fp32
    f = x / s                                # the quotient, rounded to fp32
    return y, f, _safe(y)


def _bf16(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).float().numpy()


def test_shortcut_agrees_on_gaussian_heads():
    g = torch.Generator().manual_seed(49101)
    for sigma in (1e-3, 0.37, 1.0, 25.0):
        x = _bf16(torch.randn(64, 4096, generator=g) * sigma)
        amax = np.abs(x).max(axis=1, keepdims=True).astype(np.float32)
        s = np.broadcast_to(amax / np.float32(448.0), x.shape)
        y, f, ok = _both(x, s)
        np.testing.assert_array_equal(_codes(y[ok]), _codes(f[ok]))
        # almost every value takes the product (exact quotients that are
        # midpoints, frequent for a head whose maximum is a power of two,
        # take the division)
        assert ok.mean() > 0.98, ok.mean()


def test_shortcut_agrees_next_to_every_midpoint():
    # quotients placed within 12 units in the last place of every e4m3
    # midpoint of the normal range: the cases the test on y exists for
    g = torch.Generator().manual_seed(49102)
    mids = []
    for e in range(-6, 9):
        for m in range(8):
            v = (1.0 + (m + 0.5) / 8.0) * 2.0 ** e
            if v < 448.0:
                mids.append(v)
    mids = np.array(mids)
    x = _bf16(torch.rand(len(mids), 200, generator=g) * 8.0 + 0.5)
    k = np.arange(-12, 13)
    xs, ss = [], []
    for i, mv in enumerate(mids):
        ulp = 2.0 ** (np.floor(np.log2(mv)) - 23)
        target = mv + k[None, :] * ulp                     # [1, 25]
        s = (x[i][:, None].astype(np.float64) / target).astype(np.float32)
        xs.append(np.broadcast_to(x[i][:, None], s.shape))
        ss.append(s)
    y, f, ok = _both(np.concatenate(xs).ravel(), np.concatenate(ss).ravel())
    cy, cf = _codes(y), _codes(f)
    np.testing.assert_array_equal(cy[ok], cf[ok])
    # the product alone would be wrong on some of these (the test has teeth),
    # and every such case is one the kernel divides
    wrong = cy != cf
    assert wrong.any()
    assert not (wrong & ok).any()
    assert ok.any() and (~ok).any()


def test_shortcut_bound_is_tight_enough():
    # the 3-unit bound behind the threshold: |y - f| never exceeds 3 units in
    # the last place of f's binade over a wide sweep of x and s
    g = torch.Generator().manual_seed(49103)
    x = _bf16(torch.randn(400_000, generator=g) * 3.0)
    s = (torch.rand(400_000, generator=g).numpy() * 0.05 + 1e-4).astype(np.float32)
    y, f, _ = _both(x, s)
    m = (np.abs(f) >= 2.0 ** -6) & np.isfinite(f)
    ulp = np.ldexp(1.0, np.frexp(np.abs(f[m]).astype(np.float64))[1] - 24)
    assert (np.abs(y[m].astype(np.float64) - f[m]) <= 3 * ulp).all()
