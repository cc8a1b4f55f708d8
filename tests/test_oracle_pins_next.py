"""Pins for the oracle of the NEXT ops (CPU only).

NEXT-1, gated residual + AdaRMSNorm modulation + FP8 ("FlashRT kernel
fusion", §三, gate_res_adarms_fp8_static): reduction to op (a) when the gate is
one and the modulation zero, a zero gate, a closed form on constant rows, the
condition-row mapping, and the brute-force rational restatement on 4 x 8."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import np_restatement as npr
from memory_bound_non_b200 import workloads as W


def _inputs(M, D, dt, seed, ncond):
    g = W.generator(seed)
    x = W.bits16(W.normal16((M, D), dt, g))
    r = W.bits16(W.normal16((M, D), dt, g, scale=2.0))
    gate = W.bits16(W.normal16((ncond, D), dt, g, scale=0.5))
    sc = W.bits16(W.normal16((ncond, D), dt, g, scale=0.2))
    sh = W.bits16(W.normal16((ncond, D), dt, g, scale=0.2))
    return x, r, gate, sc, sh


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("quant", ["static", "block128"])
def test_adarms_reduces_to_op_a_with_unit_gate_and_no_modulation(dt, quant):
    x, r, _, _, _ = _inputs(6, 384, dt, 1, 1)
    a = oracle.gate_residual_adarms_fp8(x, None, r, None, None, 1e-6, dt, quant, 6, static_scale=0.01, want_y=True)
    b = oracle.residual_rmsnorm_fp8(x, r, None, 1e-6, dt, quant, static_scale=0.01, want_y=True)
    np.testing.assert_array_equal(a["residual_out"], b["residual_out"])
    np.testing.assert_array_equal(a["y"], b["y"])
    np.testing.assert_array_equal(a["out_fp8"], b["out_fp8"])


def test_adarms_zero_gate_keeps_the_residual():
    x, r, gate, sc, sh = _inputs(4, 256, "bf16", 2, 1)
    zero = np.zeros_like(gate)
    o = oracle.gate_residual_adarms_fp8(x, zero, r, sc, sh, 1e-6, "bf16", "static", 4, static_scale=0.01)
    same = (r & 0x7FFF) != 0   # -0 + 0 gives +0: compare the non-zero residuals bitwise
    np.testing.assert_array_equal(o["residual_out"][same], r[same])


def test_adarms_constant_row_closed_form():
    D = 128
    r = W.bits16(torch.full((2, D), -3.0, dtype=torch.bfloat16))
    x = np.zeros((2, D), dtype=np.uint16)
    g = W.generator(3)
    sc = W.bits16(W.normal16((1, D), "bf16", g, scale=0.3))
    sh = W.bits16(W.normal16((1, D), "bf16", g, scale=0.3))
    o = oracle.gate_residual_adarms_fp8(x, None, r, sc, sh, 0.0, "bf16", "block128", 2, want_y=True)
    s = oracle.decode16(sc[0], "bf16")
    t = oracle.decode16(sh[0], "bf16")
    np.testing.assert_allclose(o["y"][0], -1.0 * (1 + s) + t, rtol=1e-15, atol=1e-15)


def test_adarms_condition_rows_map_to_row_groups():
    M, D, rpc = 6, 256, 2
    x, r, gate, sc, sh = _inputs(M, D, "bf16", 4, 3)
    o = oracle.gate_residual_adarms_fp8(x, gate, r, sc, sh, 1e-6, "bf16", "static", rpc, static_scale=0.02,
                                        want_y=True)
    for i in range(M):
        c = i // rpc
        h = oracle.decode16(o["residual_out"][i], "bf16")
        ref = torch.nn.functional.rms_norm(torch.from_numpy(h), (D,), None, float(np.float32(1e-6))).numpy()
        ref = ref * (1 + oracle.decode16(sc[c], "bf16")) + oracle.decode16(sh[c], "bf16")
        np.testing.assert_allclose(o["y"][i], ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("quant", ["static", "block128"])
def test_adarms_bruteforce_4x8(dt, quant):
    x, r, gate, sc, sh = _inputs(4, 8, dt, 5, 2)
    o = oracle.gate_residual_adarms_fp8(x, gate, r, sc, sh, 1e-6, dt, quant, 2, static_scale=0.0078125)
    h, q, bs = npr.gate_residual_adarms_fp8(x, gate, r, sc, sh, float(np.float32(1e-6)), dt, quant, 2,
                                            static_scale=0.0078125)
    np.testing.assert_array_equal(o["residual_out"], h)
    np.testing.assert_array_equal(o["out_fp8"], q)
    if quant == "block128":
        np.testing.assert_allclose(o["block_scales"], bs, rtol=1e-13)


def test_adarms_residual_is_the_exactly_rounded_gated_sum():
    # wide dynamic range, both formats: the oracle's h is RN16(r + g x) exactly
    for dt in ("bf16", "f16"):
        rng = np.random.default_rng(6)
        hi = 0x7800 if dt == "f16" else 0x7F00
        x = rng.integers(0, hi, size=(1, 64)).astype(np.uint16)
        r = rng.integers(0, hi, size=(1, 64)).astype(np.uint16) | 0x8000 * rng.integers(0, 2, (1, 64)).astype(np.uint16)
        gate = rng.integers(0x3000, 0x3C00 if dt == "f16" else 0x3F80, size=(1, 64)).astype(np.uint16)
        o = oracle.gate_residual_adarms_fp8(x, gate, r, None, None, 1e-6, dt, "block128", 1)
        h, _, _ = npr.gate_residual_adarms_fp8(x, gate, r, None, None, 1e-6, dt, "block128", 1)
        ok = np.isfinite(oracle.decode16(o["residual_out"], dt))
        np.testing.assert_array_equal(o["residual_out"][ok], h[ok])


# ------------------------------------------------------------------ NEXT-2 --
# Op (b) with the attention's Q preparation (softmax-scale pre-multiply,
# head-major layout) and an optional e4m3 KV cache with static scales (the
# "5060 Ti" port's step 10, FA2 prepare_q fused into RoPE; "FlashRT kernel
# fusion", §2.2).

def _qkv_inputs(M=5, Hq=4, Hkv=2, hd=16, dt="bf16", seed=7, qk_norm=True):
    g = W.generator(seed)
    H = Hq + 2 * Hkv
    qkv = W.bits16(W.normal16((M, H * hd), dt, g))
    qw = W.bits16(W.norm_weight(hd, dt, g)) if qk_norm else None
    kw = W.bits16(W.norm_weight(hd, dt, g)) if qk_norm else None
    cos, sin = W.rope_tables(64, hd, 1e4)
    pos = np.arange(3, 3 + M, dtype=np.int32)
    return qkv, qw, kw, cos.numpy(), sin.numpy(), pos


def _nearest_e4m3(y):
    """Brute force: the finite e4m3 code nearest to y (ties to the even code,
    |y| beyond 448 saturating), by scanning the whole code table."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    out = np.empty(y.shape, dtype=np.uint8)
    for idx, v in np.ndenumerate(y):
        v = float(np.clip(v, -448.0, 448.0))
        d = np.abs(vals - v)
        best = np.flatnonzero(d == d.min())
        best = [c for c in codes[best] if not (v >= 0) ^ (c < 0x80)] or list(codes[best])
        even = [c for c in best if (c & 1) == 0]
        out[idx] = (even or best)[0]
    return out


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("qk_norm", [True, False])
def test_prepq_defaults_reduce_to_op_b(dt, qk_norm):
    qkv, qw, kw, cos, sin, pos = _qkv_inputs(dt=dt, qk_norm=qk_norm)
    a = oracle.qkv_norm_rope_prepq_kvcache(qkv, qw, kw, cos, sin, pos, 4, 2, 16, 16, 1e-6, dt)
    b = oracle.qkv_norm_rope_kvcache(qkv, qw, kw, cos, sin, pos, 4, 2, 16, 16, 1e-6, dt)
    np.testing.assert_array_equal(a["q_out"], b["q_out"])
    np.testing.assert_array_equal(a["k_cache"], b["k_cache"])
    np.testing.assert_array_equal(a["v_cache"], b["v_cache"])


def test_prepq_head_major_is_the_transpose_and_power_of_two_scale_is_exact():
    qkv, qw, kw, cos, sin, pos = _qkv_inputs()
    base = oracle.qkv_norm_rope_kvcache(qkv, qw, kw, cos, sin, pos, 4, 2, 16, 16, 1e-6, "bf16")["q_out"]
    o = oracle.qkv_norm_rope_prepq_kvcache(qkv, qw, kw, cos, sin, pos, 4, 2, 16, 16, 1e-6, "bf16", q_scale=0.125,
                                           q_layout="head")
    assert o["q_out"].shape == (4, 5, 16)
    np.testing.assert_array_equal(o["q_out"], 0.125 * base.transpose(1, 0, 2))


def test_prepq_softmax_scale():
    qkv, qw, kw, cos, sin, pos = _qkv_inputs(hd=16)
    base = oracle.qkv_norm_rope_kvcache(qkv, qw, kw, cos, sin, pos, 4, 2, 16, 16, 1e-6, "bf16")["q_out"]
    sc = float(np.float32(1.0 / math.sqrt(16.0) * 1.4426950408889634))   # 1/sqrt(hd) * log2(e), as fp32
    o = oracle.qkv_norm_rope_prepq_kvcache(qkv, qw, kw, cos, sin, pos, 4, 2, 16, 16, 1e-6, "bf16", q_scale=sc)
    np.testing.assert_allclose(o["q_out"], base * sc, rtol=1e-15, atol=0)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_prepq_fp8_cache_codes_are_the_nearest_codes(dt):
    qkv, qw, kw, cos, sin, pos = _qkv_inputs(dt=dt)
    base = oracle.qkv_norm_rope_kvcache(qkv, qw, kw, cos, sin, pos, 4, 2, 16, 16, 1e-6, dt)
    ks, vs = 0.0078125, 0.00390625 * 3      # K: power of two; V: 3/256 (an inexact quotient)
    o = oracle.qkv_norm_rope_prepq_kvcache(qkv, qw, kw, cos, sin, pos, 4, 2, 16, 16, 1e-6, dt, kv="e4m3",
                                           k_scale=ks, v_scale=vs)
    rows = pos
    k = base["k_cache"][rows].astype(np.float32).astype(np.float64)       # the fp32 value the decision uses
    np.testing.assert_array_equal(o["k_cache"][rows], _nearest_e4m3(k / ks))
    v = oracle.decode16(base["v_cache"][rows], dt)
    vq = (v.astype(np.float32) / np.float32(vs)).astype(np.float64)       # fp32 quotient, as the reading says
    np.testing.assert_array_equal(o["v_cache"][rows], _nearest_e4m3(vq))
    untouched = np.setdiff1d(np.arange(16), rows)
    assert (o["k_cache"][untouched] == 0x7E).all() and (o["v_cache"][untouched] == 0x7E).all()


def test_prepq_fp8_cache_saturates_and_keeps_sign():
    qkv, qw, kw, cos, sin, pos = _qkv_inputs(qk_norm=False)
    o = oracle.qkv_norm_rope_prepq_kvcache(qkv, None, None, cos, sin, pos, 4, 2, 16, 16, 1e-6, "bf16", kv="e4m3",
                                           k_scale=1e-4, v_scale=1e-4)
    v = oracle.decode16(qkv[:, 6 * 16:].reshape(5, 2, 16), "bf16")
    codes = o["v_cache"][pos]
    big = np.abs(v) / 1e-4 > 464                       # beyond the last rounding boundary of 448
    assert big.any()
    assert (codes[big & (v > 0)] == 0x7E).all() and (codes[big & (v < 0)] == 0xFE).all()


def test_prepq_bad_positions_skip_rows():
    qkv, qw, kw, cos, sin, pos = _qkv_inputs()
    pos = pos.copy()
    pos[1] = -1
    pos[3] = 64                                         # == max_pos
    o = oracle.qkv_norm_rope_prepq_kvcache(qkv, qw, kw, cos, sin, pos, 4, 2, 16, 80, 1e-6, "bf16", kv="e4m3",
                                           k_scale=0.01, v_scale=0.01, q_layout="head")
    assert o["status"] & 1
    assert np.isnan(o["q_out"][:, [1, 3]]).all() and np.isfinite(o["q_out"][:, [0, 2, 4]]).all()
    assert (o["k_cache"][64] == 0x7E).all()


# ------------------------------------------------------------------ NEXT-3 --
# NVFP4 outputs of ops (a) and (c) (the pages' "residual_add_rms_norm_to_nvfp4"
# and "silu_mul_merged_grouped32" NVFP4 producers): e2m1 codes, 16-element
# blocks with e4m3 scale factors and a per-tensor fp32 global scale.

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # the format's magnitudes, code = index (+8 for negative)


def test_e2m1_codes_and_round_trip():
    for c in range(16):
        v = E2M1[c & 7] * (-1 if c & 8 else 1)
        assert oracle.e2m1_decode(c) == v
        assert oracle.e2m1_encode(oracle.e2m1_decode(c)) == c, c
    assert math.copysign(1.0, oracle.e2m1_decode(8)) < 0


def test_e2m1_ties_to_even_and_saturation():
    for lo, hi in zip(E2M1[:-1], E2M1[1:]):
        mid = (lo + hi) / 2
        want = E2M1.index(lo) if E2M1.index(lo) % 2 == 0 else E2M1.index(hi)
        assert oracle.e2m1_encode(mid) == want, mid
        assert oracle.e2m1_encode(-mid) == want | 8
        assert oracle.e2m1_encode(np.nextafter(mid, 0)) == E2M1.index(lo)
        assert oracle.e2m1_encode(np.nextafter(mid, 10)) == E2M1.index(hi)
    assert oracle.e2m1_encode(6.0) == 7 and oracle.e2m1_encode(1e30) == 7 and oracle.e2m1_encode(-7.5) == 15


def _round_f32(q):
    """The fp32 value nearest the rational q (ties to the even significand),
    by brute force over the fp32 neighbours of a first guess, with exact
    rational distances."""
    f = np.float32(float(q))
    cands = {f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))}
    cands = [c for c in cands if np.isfinite(c)]
    best = min(abs(Fraction(float(c)) - q) for c in cands)
    near = [c for c in cands if abs(Fraction(float(c)) - q) == best]
    if len(near) > 1:
        near = [c for c in near if (int(np.array(c, dtype=np.float32).view(np.uint32)) & 1) == 0]
    return float(near[0])


def _nvfp4_brute(y, gs):
    """The NVFP4 reading restated with exact rational quotients: the block
    scale is the e4m3 code nearest fp32(amax / (6 gs)) and each element the
    e2m1 code nearest fp32(y / (sf gs)), every quotient exact and then rounded
    once to fp32 (found by brute force), nearest codes found by searching the
    whole e4m3 table and the 8 e2m1 magnitudes (ties to the even code)."""
    y32 = np.asarray(y, dtype=np.float32)
    g = Fraction(float(np.float32(gs)))
    packed, sfs = [], []
    for b in range(len(y32) // 16):
        blk = y32[16 * b:16 * b + 16]
        amax = Fraction(float(np.max(np.abs(blk))))
        sf = int(_nearest_e4m3(np.array([_round_f32(amax / (6 * g))]))[0])
        eff = Fraction(oracle.e4m3_decode(sf)) * g
        codes = []
        for v in blk:
            if eff == 0:
                codes.append(0)
                continue
            t = _round_f32(Fraction(float(v)) / eff)
            a = min(abs(t), 6.0)
            d = [abs(m - a) for m in E2M1]
            best = [k for k in range(8) if d[k] == min(d)]
            k = [k for k in best if k % 2 == 0][0] if len(best) > 1 else best[0]
            codes.append(k | (8 if math.copysign(1.0, t) < 0 or (t == 0 and math.copysign(1.0, float(v)) < 0)
                              else 0))
        sfs.append(sf)
        packed += [codes[2 * j] | (codes[2 * j + 1] << 4) for j in range(8)]
    return np.array(packed, dtype=np.uint8), np.array(sfs, dtype=np.uint8)


@pytest.mark.parametrize("gs", [1.0, 0.0123, 3.7e-4])
def test_nvfp4_row_matches_brute_force(gs):
    g = W.generator(11)
    y = torch.randn(96, generator=g, dtype=torch.float64).numpy() * 2.5
    y[16:32] *= 1e-3                          # a small block
    y[32:48] = 0.0                            # an all-zero block
    packed, sf = oracle.quant_nvfp4_row(y, gs)
    bp, bsf = _nvfp4_brute(y, gs)
    np.testing.assert_array_equal(sf, bsf)
    np.testing.assert_array_equal(packed, bp)
    assert sf[2] == 0 and (packed[16:24] == 0).all()


def _e2m1_nearest(t):
    a = min(abs(t), 6.0)
    d = [abs(m - a) for m in E2M1]
    best = [k for k in range(8) if d[k] == min(d)]
    return [k for k in best if k % 2 == 0][0] if len(best) > 1 else best[0]


def _reciprocal_form_codes(blk, gs):
    """Scaling by rounded reciprocals instead of quotients (a plausible
    alternative the oracle must not be): sf = e4m3(RN(amax RN(1/RN(6 gs)))),
    code = e2m1(RN(y RN(1/RN(sf gs)))), in numpy fp32."""
    gs = np.float32(gs)
    blk = np.asarray(blk, dtype=np.float32)
    rden = np.float32(np.float32(1.0) / (np.float32(6.0) * gs))
    sf = int(oracle.e4m3_encode(float(np.float32(np.max(np.abs(blk)) * rden))))
    eff = np.float32(np.float32(oracle.e4m3_decode(sf)) * gs)
    reff = np.float32(np.float32(1.0) / eff)
    return sf, [_e2m1_nearest(float(np.float32(v * reff))) for v in blk]


def _neighbours(v, n):
    out, a, b = [np.float32(v)], np.float32(v), np.float32(v)
    for _ in range(n):
        a, b = np.nextafter(a, np.float32(np.inf)), np.nextafter(b, np.float32(-np.inf))
        out += [a, b]
    return out


@pytest.mark.parametrize("gs", [1.0 / 3.0, 0.0123])
def test_nvfp4_decisions_are_quotients_not_reciprocal_products(gs):
    """Blocks built so that scaling by rounded reciprocals decides a different
    scale factor or element code than the quotient definition: the oracle must
    follow the definition (the exact-rational brute force) on every one."""
    g32 = Fraction(float(np.float32(gs)))
    blocks = []
    # element codes: amax fixes sf; the other values sit next to e2m1 midpoints
    for sf_code in (0x38, 0x3B, 0x45):
        eff = Fraction(oracle.e4m3_decode(sf_code)) * g32
        amax = np.float32(float(6 * eff))
        for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
            for v in _neighbours(float(m * eff), 12):
                blk = np.zeros(16, dtype=np.float32)
                blk[0], blk[1], blk[2] = amax, v, -v
                sf_r, codes_r = _reciprocal_form_codes(blk, gs)
                t = _round_f32(Fraction(float(v)) / (Fraction(oracle.e4m3_decode(sf_r)) * g32))
                if sf_r == sf_code and codes_r[1] != _e2m1_nearest(t):
                    blocks.append(blk)
    # scale factors: amax next to (e4m3 midpoint) * 6 gs
    for c in range(0x10, 0x70, 5):
        mid = (Fraction(oracle.e4m3_decode(c)) + Fraction(oracle.e4m3_decode(c + 1))) / 2
        for a in _neighbours(float(mid * 6 * g32), 6):
            want = int(_nearest_e4m3(np.array([_round_f32(Fraction(float(a)) / (6 * g32))]))[0])
            blk = np.zeros(16, dtype=np.float32)
            blk[0] = a
            if _reciprocal_form_codes(blk, gs)[0] != want:
                blocks.append(blk)
    assert len(blocks) >= 8, "too few discriminating blocks (%d)" % len(blocks)
    y = np.concatenate(blocks).astype(np.float64)
    packed, sf = oracle.quant_nvfp4_row(y, gs)
    bp, bsf = _nvfp4_brute(y, gs)
    np.testing.assert_array_equal(sf, bsf)
    np.testing.assert_array_equal(packed, bp)


def test_nvfp4_exact_block_closed_form_and_nibble_order():
    # gs = 1: den = 6; a block whose amax is 6 * 2^k has sf = 2^k exactly and
    # every value k-scaled e2m1 magnitude quantises to its own code
    k = -3
    vals = np.array([E2M1[j % 8] * (-1 if j >= 8 else 1) for j in range(16)]) * 2.0 ** k
    vals[0] = 6.0 * 2.0 ** k                  # amax (code 7) in element 0
    packed, sf = oracle.quant_nvfp4_row(vals, 1.0)
    assert oracle.e4m3_decode(int(sf[0])) == 2.0 ** k
    codes = [int(packed[j // 2] >> (4 * (j % 2))) & 0xF for j in range(16)]
    want = [oracle.e2m1_encode(v / 2.0 ** k) for v in vals]
    assert codes == want and codes[0] == 7   # element 0 in the low nibble of byte 0


def test_nvfp4_dequantisation_error_bound():
    g = W.generator(12)
    y = torch.randn(16 * 64, generator=g, dtype=torch.float64).numpy()
    gs = 0.002
    packed, sf = oracle.quant_nvfp4_row(y, gs)
    codes = np.stack([packed & 0xF, packed >> 4], axis=1).ravel()
    for b in range(64):
        eff = oracle.e4m3_decode(int(sf[b])) * np.float32(gs)
        amax = np.max(np.abs(y[16 * b:16 * b + 16]))
        assert abs(eff * 6 - amax) <= amax * 2.0 ** -3                 # e4m3 scale: within half a step (2^-4) + fp32
        for j in range(16):
            v = y[16 * b + j]
            dq = oracle.e2m1_decode(int(codes[16 * b + j])) * eff
            t = min(abs(v) / eff, 6.0)
            spacing = 0.5 if t < 2 else (1.0 if t < 4 else 2.0)
            assert abs(abs(dq) - min(abs(v), 6 * eff)) <= spacing / 2 * eff * (1 + 1e-6) + 1e-12


def test_nvfp4_ops_reuse_op_a_and_op_c():
    x, r, _, _, _ = _inputs(3, 256, "bf16", 13, 1)
    g = W.generator(13)
    w = W.bits16(W.norm_weight(256, "bf16", g))
    a = oracle.residual_rmsnorm_nvfp4(x, r, w, 1e-6, "bf16", 0.004, want_y=True)
    b = oracle.residual_rmsnorm_fp8(x, r, w, 1e-6, "bf16", "static", static_scale=0.01, want_y=True)
    np.testing.assert_array_equal(a["residual_out"], b["residual_out"])
    np.testing.assert_array_equal(a["y"], b["y"])
    for i in range(3):
        p, s = oracle.quant_nvfp4_row(a["y"][i], 0.004)
        np.testing.assert_array_equal(a["out_fp4"][i], p)
        np.testing.assert_array_equal(a["sf"][i], s)
    gu = W.bits16(W.normal16((2, 2 * 128), "bf16", g))
    c = oracle.gate_act_nvfp4(gu, "silu", "bf16", 0.003, want_a=True)
    d = oracle.gate_act_fp8(gu, "silu", "bf16", "static", static_scale=0.01, want_a=True)
    np.testing.assert_array_equal(c["a"], d["a"])
    for i in range(2):
        p, s = oracle.quant_nvfp4_row(c["a"][i], 0.003)
        np.testing.assert_array_equal(c["out_fp4"][i], p)


def _torch_to_blocked():
    """PyTorch's to_blocked (and its ceil_div) taken from the installed
    torch/testing/_internal/common_quantized.py source: the module itself
    imports test-only packages this image lacks, so the two functions are
    compiled alone from their source text, unchanged."""
    import ast
    import importlib.util
    path = os.path.join(os.path.dirname(importlib.util.find_spec("torch").origin), "testing", "_internal",
                        "common_quantized.py")
    with open(path) as f:
        tree = ast.parse(f.read())
    fns = [n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name in ("ceil_div", "to_blocked")]
    assert sorted(n.name for n in fns) == ["ceil_div", "to_blocked"]
    ns = {"torch": torch}
    exec(compile(ast.Module(body=fns, type_ignores=[]), path, "exec"), ns)
    return ns["to_blocked"]


@pytest.mark.parametrize("rows,cols", [(1, 1), (128, 4), (130, 10), (300, 7), (256, 64), (77, 256)])
def test_sf_swizzle_matches_torch_to_blocked(rows, cols):
    """The swizzled scale-factor layout pinned to an implementation outside
    this repository: PyTorch's own test helper for block-scaled matmul,
    torch.testing._internal.common_quantized.to_blocked, which rearranges an
    [rows, cols] scale matrix into the cuBLAS 1-D block-scaling-factor layout
    (128 x 4 tiles of 512 bytes).  Position p of its flattened output holds
    element (r, c) exactly when the oracle's offset of (r, c) is p; a
    transposed reading (4 k + 16 i) or a column-major tile order fails."""
    to_blocked = _torch_to_blocked()
    idx = torch.arange(1, rows * cols + 1, dtype=torch.int64).reshape(rows, cols)
    flat = to_blocked(idx).numpy()
    n_cols = cols
    assert flat.size == ((rows + 127) // 128) * 128 * ((cols + 3) // 4) * 4
    seen = 0
    for p in np.flatnonzero(flat):
        r, c = divmod(int(flat[p]) - 1, cols)
        assert oracle.sf_swizzle_offset(r, c, n_cols) == p, (r, c, p)
        seen += 1
    assert seen == rows * cols
    # and the oracle's whole-matrix helper places every element the same way
    sf = (np.arange(rows * cols, dtype=np.int64) % 251 + 1).astype(np.uint8).reshape(rows, cols)
    want = to_blocked(torch.from_numpy(sf.astype(np.int64))).numpy().astype(np.uint8)
    got = oracle.sf_swizzle(sf)
    written = want != 0
    np.testing.assert_array_equal(got[written], want[written])


def test_sf_swizzle_layout():
    C = 10
    atoms = (C + 3) // 4
    assert oracle.sf_swizzle_offset(0, 0, C) == 0
    assert oracle.sf_swizzle_offset(1, 0, C) == 16
    assert oracle.sf_swizzle_offset(31, 0, C) == 496
    assert oracle.sf_swizzle_offset(32, 0, C) == 4
    assert oracle.sf_swizzle_offset(97, 3, C) == 16 * 1 + 4 * 3 + 3
    assert oracle.sf_swizzle_offset(0, 4, C) == 512
    assert oracle.sf_swizzle_offset(128, 0, C) == atoms * 512
    M = 300
    offs = {oracle.sf_swizzle_offset(r, c, C) for r in range(((M + 127) // 128) * 128) for c in range(atoms * 4)}
    assert offs == set(range(((M + 127) // 128) * 128 * atoms * 4))   # a bijection onto the padded array


# ------------------------------------------------------------------ NEXT-4 --
# LayerNorm variants: the ViT add + LayerNorm producer (op (a) with LayerNorm)
# and the Chameleon LayerNorm(Q) + LayerNorm(K) + RoPE kernel ("FlashRT kernel
# fusion", §2.2 second bullet).

def test_layernorm_closed_form_and_invariants():
    np.testing.assert_allclose(oracle.layernorm(np.array([1.0, 2.0, 3.0, 4.0]), eps=0.0),
                               np.array([-3, -1, 1, 3]) / math.sqrt(5.0), rtol=1e-15)
    g = W.generator(21)
    h = torch.randn(512, generator=g, dtype=torch.float64).numpy() * 3 + 7
    y = oracle.layernorm(h, eps=0.0)
    assert abs(y.mean()) < 1e-14 and abs((y * y).mean() - 1.0) < 1e-13
    np.testing.assert_allclose(oracle.layernorm(h + 1000.0, eps=0.0), y, atol=1e-10)     # shift invariance
    np.testing.assert_allclose(oracle.layernorm(h * 0.25, eps=0.0), y, rtol=1e-13, atol=1e-14)


def test_layernorm_matches_torch():
    g = W.generator(22)
    h = torch.randn(4, 384, generator=g, dtype=torch.float64)
    w = torch.randn(384, generator=g, dtype=torch.float64)
    b = torch.randn(384, generator=g, dtype=torch.float64)
    ref = torch.nn.functional.layer_norm(h, (384,), w, b, eps=1e-5).numpy()
    for i in range(4):
        np.testing.assert_allclose(oracle.layernorm(h[i].numpy(), w.numpy(), b.numpy(), 1e-5), ref[i], rtol=1e-12,
                                   atol=1e-12)
    ref = torch.nn.functional.layer_norm(h, (384,), None, None, eps=1e-5).numpy()
    np.testing.assert_allclose(oracle.layernorm(h[0].numpy(), eps=1e-5), ref[0], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("quant", ["static", "block128", "nvfp4"])
def test_residual_layernorm_composes_op_a_pieces(quant):
    x, r, _, _, _ = _inputs(3, 256, "bf16", 23, 1)
    g = W.generator(23)
    w = W.bits16(W.norm_weight(256, "bf16", g))
    b = W.bits16(W.normal16((256,), "bf16", g, scale=0.1))
    o = oracle.residual_layernorm(x, r, w, b, 1e-6, "bf16", quant, static_scale=0.01, global_scale=0.002,
                                  want_y=True)
    a = oracle.residual_rmsnorm_fp8(x, r, None, 1e-6, "bf16", "static", static_scale=0.01)
    np.testing.assert_array_equal(o["residual_out"], a["residual_out"])
    h = oracle.decode16(o["residual_out"], "bf16")
    for i in range(3):
        y = torch.nn.functional.layer_norm(torch.from_numpy(h[i]), (256,),
                                           torch.from_numpy(oracle.decode16(w, "bf16")),
                                           torch.from_numpy(oracle.decode16(b, "bf16")),
                                           eps=float(np.float32(1e-6))).numpy()
        np.testing.assert_allclose(o["y"][i], y, rtol=1e-12, atol=1e-12)
        if quant == "nvfp4":
            p, s = oracle.quant_nvfp4_row(o["y"][i], 0.002)
            np.testing.assert_array_equal(o["out"][i], p)
            np.testing.assert_array_equal(o["sf"][i], s)
        elif quant == "static":
            np.testing.assert_array_equal(o["out"][i], oracle.quant_static(o["y"][i], 0.01))


def test_qkv_layernorm_per_head_affine_and_rope():
    M, Hq, Hkv, hd = 3, 4, 2, 16
    qkv, _, _, cos, sin, pos = _qkv_inputs(M=M, Hq=Hq, Hkv=Hkv, hd=hd, qk_norm=False)
    g = W.generator(24)
    qw = W.bits16(W.normal16((Hq, hd), "bf16", g))
    qb = W.bits16(W.normal16((Hq, hd), "bf16", g, scale=0.1))
    kw = W.bits16(W.normal16((Hkv, hd), "bf16", g))
    o = oracle.qkv_layernorm_rope_kvcache(qkv, qw, qb, kw, None, cos, sin, pos, Hq, Hkv, hd, 16, 1e-6, "bf16")
    v = oracle.decode16(qkv, "bf16").reshape(M, Hq + 2 * Hkv, hd)
    for i in range(M):
        for h in range(Hq + Hkv):
            is_q = h < Hq
            w = oracle.decode16((qw if is_q else kw)[h if is_q else h - Hq], "bf16")
            bb = oracle.decode16(qb[h], "bf16") if is_q else None
            y = torch.nn.functional.layer_norm(torch.from_numpy(v[i, h]), (hd,), torch.from_numpy(w),
                                               None if bb is None else torch.from_numpy(bb),
                                               eps=float(np.float32(1e-6))).numpy()
            y = oracle.rope_rotate_half(y, cos[pos[i]], sin[pos[i]])
            got = o["q_out"][i, h] if is_q else o["k_cache"][pos[i], h - Hq]
            np.testing.assert_allclose(got, y, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(o["v_cache"][pos], qkv.reshape(M, Hq + 2 * Hkv, hd)[:, Hq + Hkv:])
