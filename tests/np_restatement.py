"""Second, independent restatement of the three ops for tiny inputs.

Deliberately built differently from the C++ oracle so that a slip in one does
not repeat in the other:
  * 16-bit and FP8 rounding are done by brute-force nearest search over every
    finite code of the format (ties -> the code with an even last bit), on
    exact rationals (``fractions.Fraction``);
  * the residual sum is formed exactly with rationals;
  * RMSNorm uses numpy's vectorised mean; RoPE is a complex multiplication.
Only meant for inputs of a few dozen elements.
"""
from fractions import Fraction
import bisect
import math

import numpy as np


def _decode_f16(b):
    return float(np.array([b], dtype=np.uint16).view(np.float16)[0])


def _decode_bf16(b):
    return float(np.array([int(b) << 16], dtype=np.uint32).view(np.float32)[0])


DECODE = {"f16": _decode_f16, "bf16": _decode_bf16}


def _grid(dt):
    """Sorted (value, code) over all finite non-negative codes of the format."""
    out = []
    for b in range(0x8000):
        v = DECODE[dt](b)
        if math.isfinite(v):
            out.append((Fraction(v), b))
    out.sort()
    return out


_GRIDS = {}


def round16_exact(v: Fraction, dt: str) -> int:
    """Nearest 16-bit code to the rational v, ties to the even code."""
    if dt not in _GRIDS:
        g = _grid(dt)
        _GRIDS[dt] = ([x for x, _ in g], [c for _, c in g])
    vals, codes = _GRIDS[dt]
    sign = 0x8000 if v < 0 else 0
    a = -v if v < 0 else v
    k = bisect.bisect_left(vals, a)
    if k == len(vals):
        # beyond the largest finite value: rounds to inf past the midpoint
        # towards the next binade (max + half an ulp of max)
        top = vals[-1]
        ulp = top - vals[-2]
        if a >= top + ulp / 2:
            return sign | (0x7C00 if dt == "f16" else 0x7F80)
        return sign | codes[-1]
    if vals[k] == a:
        return sign | codes[k]
    lo, hi = k - 1, k
    dlo, dhi = a - vals[lo], vals[hi] - a
    if dlo < dhi:
        return sign | codes[lo]
    if dhi < dlo:
        return sign | codes[hi]
    return sign | (codes[lo] if codes[lo] % 2 == 0 else codes[hi])


def e4m3_value(c: int) -> float:
    s = -1.0 if c & 0x80 else 1.0
    e, m = (c >> 3) & 0xF, c & 7
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1 + m / 8) * 2.0 ** (e - 7)


_E4 = sorted((Fraction(e4m3_value(c)), c) for c in range(0x7F))  # 0x00..0x7E, all >= 0


def e4m3_exact(v: Fraction, negative: bool) -> int:
    """Nearest e4m3 code to |v| by search, ties to even, saturating at 448;
    ``negative`` carries the sign (so that -0 maps to 0x80)."""
    a = abs(v)
    sign = 0x80 if negative else 0
    if a >= 448:
        return sign | 0x7E
    best = None
    for val, c in _E4:
        d = abs(val - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return sign | best[1]


def residual_rmsnorm_fp8(x, r, w, eps, dt, quant, static_scale=None):
    M, D = x.shape
    dec = DECODE[dt]
    h_bits = np.zeros((M, D), dtype=np.uint16)
    q = np.zeros((M, D), dtype=np.uint8)
    nb = (D + 127) // 128
    scales = np.zeros((M, nb))
    for i in range(M):
        for j in range(D):
            a, b = dec(x[i, j]), dec(r[i, j])
            if a == 0.0 and b == 0.0:  # IEEE: the sum of zeros is -0 only for (-0) + (-0)
                neg = math.copysign(1.0, a) < 0 and math.copysign(1.0, b) < 0
                h_bits[i, j] = 0x8000 if neg else 0
            else:
                h_bits[i, j] = round16_exact(Fraction(a) + Fraction(b), dt)
        h = np.array([dec(b) for b in h_bits[i]])
        ww = np.ones(D) if w is None else np.array([dec(b) for b in w])
        y = h / np.sqrt(np.mean(h * h) + eps) * ww
        _quant_row(y, quant, static_scale, q[i], scales[i])
    return h_bits, q, scales


def _code_fp32(yj, s32):
    """FP8 decision taken in fp32: fp32(y) / fp32(s) in numpy float32, then the
    exact nearest-code search on that quotient."""
    v = np.float32(yj) / np.float32(s32)
    return e4m3_exact(Fraction(float(v)), math.copysign(1.0, float(v)) < 0)


def _quant_row(y, quant, static_scale, q_row, sc_row):
    n = y.size
    if quant == "static":
        for j in range(n):
            q_row[j] = _code_fp32(float(y[j]), static_scale)
        return
    for b in range(0, n, 128):
        blk = y[b:b + 128]
        amax = float(np.max(np.abs(blk)))
        sc_row[b // 128] = amax / 448.0 if amax > 0 else 1.0
        s32 = np.float32(amax) / np.float32(448.0) if amax > 0 else np.float32(1.0)
        for j in range(blk.size):
            q_row[b + j] = _code_fp32(float(blk[j]), s32)


def qkv_norm_rope(qkv, qw, kw, cos, sin, pos, Hq, Hkv, hd, eps, dt):
    """Returns (q [M,Hq,hd], k [M,Hkv,hd], v_bits [M,Hkv,hd]) per row (no cache)."""
    dec = DECODE[dt]
    M = qkv.shape[0]
    half = hd // 2
    q = np.zeros((M, Hq, hd))
    k = np.zeros((M, Hkv, hd))
    v = np.zeros((M, Hkv, hd), dtype=np.uint16)
    for i in range(M):
        p = int(pos[i])
        rot = cos[p].astype(np.float64) + 1j * sin[p].astype(np.float64)
        for h in range(Hq + Hkv):
            vec = np.array([dec(b) for b in qkv[i, h * hd:(h + 1) * hd]])
            nw = qw if h < Hq else kw
            if nw is not None:
                wv = np.array([dec(b) for b in nw])
                vec = vec / np.sqrt(np.mean(vec * vec) + eps) * wv
            z = (vec[:half] + 1j * vec[half:]) * rot
            out = np.concatenate([z.real, z.imag])
            if h < Hq:
                q[i, h] = out
            else:
                k[i, h - Hq] = out
        for g in range(Hkv):
            o = (Hq + Hkv + g) * hd
            v[i, g] = qkv[i, o:o + hd]
    return q, k, v


def act(name, g):
    if name == "relu2":
        return max(g, 0.0) ** 2
    if name == "silu":
        return g * (1.0 / (1.0 + math.exp(-g)))
    # tanh-approximated GELU
    return g * 0.5 * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (g + 0.044715 * g ** 3)))


def gate_act_fp8(gu, act_name, dt, quant, static_scale=None):
    dec = DECODE[dt]
    M, two_i = gu.shape
    I = two_i // 2
    q = np.zeros((M, I), dtype=np.uint8)
    nb = (I + 127) // 128
    scales = np.zeros((M, nb))
    a = np.zeros((M, I))
    for i in range(M):
        g = np.array([dec(b) for b in gu[i, 0::2]])
        u = np.array([dec(b) for b in gu[i, 1::2]])
        a[i] = np.array([act(act_name, float(gg)) for gg in g]) * u
        _quant_row(a[i], quant, static_scale, q[i], scales[i])
    return q, scales, a


def gate_residual_adarms_fp8(x, gate, r, scale, shift, eps, dt, quant, rows_per_cond, static_scale=None):
    """NEXT-1 restated: exact rational residual r + g * x rounded by search,
    numpy fp64 RMS and modulation, fp32 FP8 decisions."""
    M, D = x.shape
    dec = DECODE[dt]
    h_bits = np.zeros((M, D), dtype=np.uint16)
    q = np.zeros((M, D), dtype=np.uint8)
    scales = np.zeros((M, (D + 127) // 128))
    for i in range(M):
        c = i // rows_per_cond
        for j in range(D):
            g = Fraction(dec(gate[c, j])) if gate is not None else Fraction(1)
            v = Fraction(dec(r[i, j])) + g * Fraction(dec(x[i, j]))
            h_bits[i, j] = round16_exact(v, dt) if v != 0 else (h_bits[i, j] & 0)
        h = np.array([dec(b) for b in h_bits[i]])
        y = h / np.sqrt(np.mean(h * h) + eps)
        sc = np.array([dec(b) for b in scale[c]]) if scale is not None else np.zeros(D)
        sh = np.array([dec(b) for b in shift[c]]) if shift is not None else np.zeros(D)
        y = y * (1.0 + sc) + sh
        _quant_row(y, quant, static_scale, q[i], scales[i])
    return h_bits, q, scales
