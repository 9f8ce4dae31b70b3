"""The arithmetic behind the E4M3 token operand of moe_forward_w8, checked on the
CPU over every bf16 value: a row scaled by 2^s (s = 7 - the exponent of its
largest magnitude) and split into hi = e4m3(v) and lo = e4m3(v - hi), both
rounded to nearest, gives hi + lo = v exactly for every entry at least 2^-9 of
the row's maximum, and within 2^-10 (scaled units) below that; hi never
saturates.  torch's float8_e4m3fn conversion is the rounding (round to nearest
even), independent of the CUDA code.
"""
import numpy as np
import pytest
import torch


def all_bf16_below(limit_exp):
    """Every finite bf16 value with |v| < 2^limit_exp, as float32."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f)]
    return f[np.abs(f) < 2.0 ** limit_exp]


def split(v):
    t = torch.from_numpy(v)
    hi = t.to(torch.float8_e4m3fn).to(torch.float32)
    lo = (t - hi).to(torch.float8_e4m3fn).to(torch.float32)
    return hi.numpy(), lo.numpy()


@pytest.mark.parametrize("e", [-20, -3, 0, 5, 30])
def test_two_e4m3_terms_represent_a_scaled_bf16_row(e):
    # a row whose largest magnitude has exponent e: its entries are bf16 values
    # below 2^(e + 1); the kernel scales them by 2^(7 - e)
    x = all_bf16_below(e + 1)
    s = 7 - e
    v = (x.astype(np.float64) * 2.0 ** s).astype(np.float32)
    big = np.abs(x) >= 2.0 ** (e - 9)
    # scaling is exact for these (far below, fp32 may underflow: within the bound below)
    assert np.all(v[big].astype(np.float64) == x[big].astype(np.float64) * 2.0 ** s)
    hi, lo = split(v)
    assert np.all(np.abs(hi) <= 256.0)  # no saturation at 448
    assert np.all(hi[big] + lo[big] == v[big])
    err = np.abs((hi + lo).astype(np.float64) - x.astype(np.float64) * 2.0 ** s)
    assert err.max() <= 2.0 ** -10
    # the pair is not trivially exact: some entries need lo
    assert np.any(lo[big] != 0)


def test_one_e4m3_term_is_not_enough():
    """A single E4M3 term of a scaled bf16 row errs by up to 2^-4 relative (the
    reason the operand takes two)."""
    x = all_bf16_below(1)
    v = x * 2.0 ** 7
    hi, _ = split(v)
    big = np.abs(v) >= 1.0
    rel = np.abs(hi[big] - v[big]) / np.abs(v[big])
    assert rel.max() > 2.0 ** -5
