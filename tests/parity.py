"""Agreement checks between the CUDA path and the oracle, and the oracle-side
helpers the GPU tests share (static-scale calibration, the chain replay).

Tolerances (element by element):
  * residual h, V cache, slot placement, untouched slots: bit-exact;
  * 16-bit outputs (Q staging, K cache), against the unrounded fp64 oracle
    value o: |g - o| <= 2e-3 * max(|o|, 2^-6) + ulp16(o) / 2, i.e. a relative
    error of 2e-3 for the arithmetic on top of the final rounding to 16 bits
    (a correctly rounded bf16 alone is up to 2^-8 ~ 3.9e-3 from o, so a bare
    2e-3 bound cannot hold for any bf16 output); and at least 99% of the
    elements must be the correctly rounded value itself (|g - o| <= ulp/2);
  * FP8 codes: equal (+0 == -0), else one code step apart with the same sign,
    on at most 0.1% of the elements;
  * block scales: relative error <= 1e-6 against the fp64 amax / 448;
  * NVFP4 (the same rule for 4-bit codes): e4m3 scale factors equal or one
    code step apart on at most 0.1% of the blocks; e2m1 codes equal (+0 ==
    -0) or one step apart with the same sign, on at most 0.1% of the elements
    plus the 16 elements of each block whose scale factor differs.
"""
import numpy as np
import torch

import oracle
from memory_bound_non_b200 import workloads as W

REL_16 = 2e-3
FLOOR_16 = 2.0 ** -6
FP8_MAX_FRAC = 1e-3
SCALE_REL = 1e-6


def np16(t):
    """uint16 numpy bits of a 16-bit tensor (any device)."""
    return W.bits16(t.detach().cpu())


def decode16(t):
    """float64 numpy values of a 16-bit tensor (exact)."""
    return t.detach().cpu().double().numpy()


def assert_fp8_codes(gpu, ref, max_frac=FP8_MAX_FRAC, what="fp8"):
    g = np.asarray(gpu, dtype=np.uint8).ravel()
    o = np.asarray(ref, dtype=np.uint8).ravel()
    assert g.shape == o.shape
    gm, om = g & 0x7F, o & 0x7F
    same = (g == o) | ((gm == 0) & (om == 0))
    diff = ~same
    n = int(diff.sum())
    if n:
        # every mismatch: same sign, adjacent magnitude code
        gs, os_ = g[diff] >> 7, o[diff] >> 7
        step = np.abs(gm[diff].astype(np.int32) - om[diff].astype(np.int32))
        bad = (step != 1) | ((gs != os_) & (gm[diff] != 0) & (om[diff] != 0))
        assert not bad.any(), "%s: %d codes differ by more than one step; first at %d: gpu 0x%02x oracle 0x%02x" % (
            what, int(bad.sum()), int(np.flatnonzero(diff)[np.argmax(bad)]), g[diff][bad][0], o[diff][bad][0])
    assert n <= max_frac * g.size, "%s: %d of %d codes one step off (> %.2g%%)" % (what, n, g.size, 100 * max_frac)
    return n


def unpack_e2m1(packed):
    """[..., n] bytes -> [..., 2n] e2m1 codes, element 2j from the low nibble."""
    p = np.asarray(packed, dtype=np.uint8)
    return np.stack([p & 0xF, p >> 4], axis=-1).reshape(*p.shape[:-1], p.shape[-1] * 2)


def assert_nvfp4(gpu_codes, gpu_sf, ref_codes, ref_sf, what="nvfp4"):
    """NVFP4 agreement: gpu_codes / ref_codes packed e2m1 bytes [rows, n/2],
    gpu_sf / ref_sf row-major e4m3 scale factors [rows, n/16].  Returns the
    number of differing scale factors and codes."""
    sg = np.asarray(gpu_sf, dtype=np.int32).reshape(np.shape(ref_sf))
    so = np.asarray(ref_sf, dtype=np.int32)
    sdiff = sg != so
    n_sf = int(sdiff.sum())
    assert (np.abs(sg - so) <= 1).all(), "%s: a scale factor differs by more than one code step" % what
    assert n_sf <= FP8_MAX_FRAC * so.size, "%s: %d of %d scale factors one step off" % (what, n_sf, so.size)
    g = unpack_e2m1(np.asarray(gpu_codes).reshape(np.shape(ref_codes))).astype(np.int32)
    o = unpack_e2m1(ref_codes).astype(np.int32)
    gm, om = g & 7, o & 7
    diff = ~((g == o) | ((gm == 0) & (om == 0)))
    n = int(diff.sum())
    if n:
        bad = (np.abs(gm[diff] - om[diff]) != 1) | ((((g[diff] ^ o[diff]) & 8) != 0) & (gm[diff] != 0) &
                                                  (om[diff] != 0))
        assert not bad.any(), "%s: %d codes differ by more than one step" % (what, int(bad.sum()))
    allow = FP8_MAX_FRAC * g.size + 16 * n_sf
    assert n <= allow, "%s: %d of %d codes one step off (allowance %.1f)" % (what, n, g.size, allow)
    return n_sf, n


# significand bits and smallest normal exponent of the 16-bit formats
_FMT16 = {"bf16": (8, -126), "f16": (11, -14)}
MAX_OFF_ROUNDING = 0.01


def ulp16(o, dt):
    """Spacing of the 16-bit format at |o| (the binade of o; subnormal spacing
    below the smallest normal)."""
    p, emin = _FMT16[dt]
    a = np.abs(o)
    e = np.floor(np.log2(np.where(a > 0, a, 2.0 ** emin)))
    e = np.maximum(e, emin)
    return np.ldexp(1.0, (e - (p - 1)).astype(np.int64))


def assert_16bit_close(gpu_vals, ref, what="16-bit", dt="bf16"):
    g = np.asarray(gpu_vals, dtype=np.float64).ravel()
    o = np.asarray(ref, dtype=np.float64).ravel()
    assert g.shape == o.shape
    assert np.isfinite(o).all(), what + ": oracle has non-finite values"
    half = ulp16(o, dt) / 2
    bar = REL_16 * np.maximum(np.abs(o), FLOOR_16) + half
    err = np.abs(g - o)
    k = int(np.argmax(err / bar))
    assert err[k] <= bar[k], "%s: |g-o| %.3g > bar %.3g at %d (gpu %r oracle %r)" % (what, err[k], bar[k], k,
                                                                                      g[k], o[k])
    off = int((err > half * (1 + 1e-12)).sum())
    assert off <= MAX_OFF_ROUNDING * g.size, "%s: %d of %d not the correctly rounded value" % (what, off, g.size)
    return off


def assert_scales_close(gpu, ref, what="block scales"):
    g = np.asarray(gpu, dtype=np.float64).ravel()
    o = np.asarray(ref, dtype=np.float64).ravel()
    assert np.isfinite(g).all(), what + ": unwritten (NaN) or non-finite scale"
    rel = np.abs(g - o) / np.abs(o)
    k = int(np.argmax(rel))
    assert rel[k] <= SCALE_REL, "%s: rel err %.3g at %d (gpu %r oracle %r)" % (what, rel[k], k, g[k], o[k])


def f32(x):
    return float(np.float32(x))


# ----------------------------------------------------- oracle-side helpers --
def calibrate_a(x, r, w, eps, dt):
    """Static scale of op (a): amax/448 of the oracle's y (as fp32)."""
    o = oracle.residual_rmsnorm_fp8(x, r, w, eps, dt, "block128", want_y=True)
    return f32(np.abs(o["y"]).max() / 448.0), o


def calibrate_c(gu, act, dt):
    o = oracle.gate_act_fp8(gu, act, dt, "block128", want_a=True)
    return f32(np.abs(o["a"]).max() / 448.0)


def chain_scales(wl, inp):
    """The three static scales of the chain, calibrated by the oracle on the
    first invocation (attention norm, FFN norm after it, gate activation)."""
    L = inp.layers[0]
    r0 = W.bits16(inp.residual)
    s_attn, o = calibrate_a(W.bits16(L.x_attn), r0, None if L.w_attn is None else W.bits16(L.w_attn),
                            wl.eps, wl.dt)
    s_ffn, _ = calibrate_a(W.bits16(L.x_ffn), o["residual_out"], None if L.w_ffn is None else W.bits16(L.w_ffn),
                           wl.eps, wl.dt)
    s_act = calibrate_c(W.bits16(L.gate_up), wl.act, wl.dt)
    return s_attn, s_ffn, s_act


def oracle_chain(wl, inp, scales, steps):
    """Replay steps x layers invocations on the oracle (residual in place).
    Returns the final residual bits and each layer's last outputs."""
    r = W.bits16(inp.residual).copy()
    out = []
    for _ in range(steps):
        out = []
        for L in inp.layers:
            wa = None if L.w_attn is None else W.bits16(L.w_attn)
            wf = None if L.w_ffn is None else W.bits16(L.w_ffn)
            a1 = oracle.residual_rmsnorm_fp8(W.bits16(L.x_attn), r, wa, wl.eps, wl.dt, wl.quant,
                                             static_scale=scales[0])
            r = a1["residual_out"]
            b = oracle.qkv_norm_rope_kvcache(
                W.bits16(L.qkv), None if L.q_norm_w is None else W.bits16(L.q_norm_w),
                None if L.k_norm_w is None else W.bits16(L.k_norm_w), inp.cos.numpy(), inp.sin.numpy(),
                inp.positions.numpy(), wl.Hq, wl.Hkv, wl.hd, wl.capacity, wl.eps, wl.dt,
                v_cache=W.bits16(L.v_cache))
            a2 = oracle.residual_rmsnorm_fp8(W.bits16(L.x_ffn), r, wf, wl.eps, wl.dt, wl.quant,
                                             static_scale=scales[1])
            r = a2["residual_out"]
            c = oracle.gate_act_fp8(W.bits16(L.gate_up), wl.act, wl.dt, wl.quant, static_scale=scales[2])
            out.append(dict(a1=a1, b=b, a2=a2, c=c))
    return r, out
