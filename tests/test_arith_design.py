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



def _rn32(x):
    """Round an exact rational to the nearest fp32 (ties to even)."""
    from fractions import Fraction
    f = np.float32(float(x))            # within one ulp (the float() step may double-round)
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - x), int(np.array(c).view(np.uint32)) & 1))
    return best


def test_markstein_block_scale_is_the_correctly_rounded_quotient():
    """The block-128 scale RN(amax / 448) formed as q = RN(amax * RN(1/448)),
    r = amax - 448 q (exact), RN(q + r * RN(1/448)) -- Markstein's correction
    with the correctly rounded reciprocal -- equals the IEEE fp32 quotient, on
    random values, values next to quotient rounding midpoints and every binade."""
    from fractions import Fraction
    rng = np.random.default_rng(9)
    inv = np.float32(1.0) / np.float32(448.0)
    vals = [np.float32(v) for v in rng.uniform(1.0, 2.0, 3000) * 2.0 ** rng.integers(-90, 100, 3000)]
    # amax just beside 448 * (a quotient rounding midpoint)
    for k in rng.integers(1 << 23, 1 << 24, 600):
        mid = Fraction(int(k) * 2 + 1, 2) * Fraction(448) * Fraction(2) ** -23
        for d in (-1, 0, 1):
            v = np.float32(float(mid))
            vals.append(v if d == 0 else np.nextafter(v, np.float32(d * np.inf)))
    vals += [np.float32(2.0 ** e) for e in range(-99, 127)]
    for a in vals:
        q = np.float32(a * inv)
        r = Fraction(float(a)) - 448 * Fraction(float(q))
        assert Fraction(float(np.float32(float(r)))) == r          # the residual is an fp32 number
        got = _rn32(Fraction(float(q)) + r * Fraction(float(inv)))   # one FMA: exact value rounded once
        want = np.float32(a) / np.float32(448.0)                     # IEEE fp32 division
        assert got == want, (a, got, want)
