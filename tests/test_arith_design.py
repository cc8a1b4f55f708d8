"""CPU checks of arithmetic identities behind the kernels and the oracle (no GPU).

The oracle rounds the exact sum of two 16-bit values once (add16).  An
independent route to the same value: the IEEE fp32 sum (numpy) followed by a
library RNE conversion, which equals the correctly rounded exact sum because
fp32 carries at least 2p + 1 significand bits for p = 8 (bf16) and p = 11
(fp16) -- the double-rounding condition of Figueroa ("When is double rounding
innocuous?").  Compared on pairs that cover every exponent gap.  The kernels
form the same sum with the packed 16-bit FMA (one rounding of the exact
value), checked against the oracle on the GPU.
"""
import numpy as np
import pytest
import torch

import oracle


def _pairs(n, rng, bits_range):
    a = rng.integers(bits_range[0], bits_range[1], size=n).astype(np.uint16)
    # the second operand's exponent is offset by 0..30 binades from the first
    b = a.astype(np.int64) - (rng.integers(0, 31, size=n) << (10 if bits_range[1] == 0x7C00 else 7))
    b = np.where(b < 1, rng.integers(1, 0x0400, size=n), b).astype(np.uint16)
    b |= (rng.integers(0, 2, size=n) << 15).astype(np.uint16)   # both signs
    b ^= rng.integers(0, 8, size=n).astype(np.uint16)           # vary the low mantissa bits
    return a, b


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_fp32_sum_rounded_to_16bit_is_the_exact_rounding(dt):
    rng = np.random.default_rng(5)
    hi = 0x7C00 if dt == "f16" else 0x7F80
    a, b = _pairs(40000, rng, (0x0001, hi))
    a2, b2 = rng.integers(0, hi, size=(2, 20000)).astype(np.uint16)
    a = np.concatenate([a, a2])
    b = np.concatenate([b, b2 | (rng.integers(0, 2, size=20000) << 15).astype(np.uint16)])
    if dt == "f16":
        fa, fb = a.view(np.float16).astype(np.float32), b.view(np.float16).astype(np.float32)
    else:
        fa = (a.astype(np.uint32) << 16).view(np.float32)
        fb = (b.astype(np.uint32) << 16).view(np.float32)
    ok = np.isfinite(fa) & np.isfinite(fb)
    fa, fb, a, b = fa[ok], fb[ok], a[ok], b[ok]
    s32 = fa + fb                                   # IEEE fp32, round to nearest even
    if dt == "f16":
        with np.errstate(over="ignore"):
            got = s32.astype(np.float16).view(np.uint16)
    else:
        got = torch.from_numpy(s32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    want = np.array([oracle.add16(x, y, dt) for x, y in zip(a, b)], dtype=np.uint16)
    zero = (got & 0x7FFF) == 0                      # +0 / -0 of exact cancellation: compare values only
    np.testing.assert_array_equal(got[~zero], want[~zero])
    assert (want[zero] & 0x7FFF == 0).all()


def test_products_of_16bit_values_are_exact_in_fp32():
    # h * w for 16-bit h, w has at most 2 * 11 significand bits: exact in fp32
    rng = np.random.default_rng(6)
    for dt in ("f16", "bf16"):
        bits = rng.integers(0x0400, 0x7000, size=(2, 20000)).astype(np.uint16)
        if dt == "f16":
            x, y = bits[0].view(np.float16), bits[1].view(np.float16)
        else:
            x = torch.from_numpy(bits[0].view(np.int16)).view(torch.bfloat16).float().numpy()
            y = torch.from_numpy(bits[1].view(np.int16)).view(torch.bfloat16).float().numpy()
        p32 = x.astype(np.float32) * y.astype(np.float32)
        p64 = x.astype(np.float64) * y.astype(np.float64)
        ok = np.isfinite(p64) & (np.abs(p64) > 2.0 ** -126) & (np.abs(p64) < 3e38)
        np.testing.assert_array_equal(p32[ok].astype(np.float64), p64[ok])

