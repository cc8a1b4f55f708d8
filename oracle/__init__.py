"""CPU oracle for the fused non-GEMM layer ops -- TEST INFRASTRUCTURE.

Thin numpy/ctypes wrapper over ``frt_oracle.cpp`` (plain fp64 C++).  Only the
tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package; the CUDA library never does, and the two share no code.

16-bit tensors are passed as ``np.uint16`` bit patterns; ``dt`` is ``"f16"``
or ``"bf16"``.  Every function returns freshly allocated numpy arrays.  The
ops' ``eps`` is rounded to fp32 first: that is the value the kernels receive.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_DT = {"f16": 0, "bf16": 1}
_QM = {"static": 0, "block128": 1}
_ACT = {"gelu_tanh": 0, "silu": 1, "relu2": 2}

_lib = None


def _f32(x):
    return float(np.float32(x))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c = ctypes
        L.oracle_f16_decode.argtypes = [c.c_uint16]
        L.oracle_f16_decode.restype = c.c_double
        L.oracle_bf16_decode.argtypes = [c.c_uint16]
        L.oracle_bf16_decode.restype = c.c_double
        L.oracle_f16_round.argtypes = [c.c_double, c.c_double]
        L.oracle_f16_round.restype = c.c_uint16
        L.oracle_bf16_round.argtypes = [c.c_double, c.c_double]
        L.oracle_bf16_round.restype = c.c_uint16
        L.oracle_e4m3_encode.argtypes = [c.c_double]
        L.oracle_e4m3_encode.restype = c.c_uint8
        L.oracle_e4m3_decode.argtypes = [c.c_uint8]
        L.oracle_e4m3_decode.restype = c.c_double
        L.oracle_act.argtypes = [c.c_int, c.c_double]
        L.oracle_act.restype = c.c_double
        L.oracle_add16.argtypes = [c.c_uint16, c.c_uint16, c.c_int]
        L.oracle_add16.restype = c.c_uint16
        L.oracle_quant_static.argtypes = [c.c_void_p, c.c_int64, c.c_double, c.c_void_p]
        L.oracle_quant_static.restype = None
        L.oracle_quant_block128.argtypes = [c.c_void_p, c.c_int64, c.c_void_p, c.c_void_p]
        L.oracle_quant_block128.restype = None
        L.oracle_rmsnorm.argtypes = [c.c_void_p, c.c_int64, c.c_void_p, c.c_double, c.c_void_p]
        L.oracle_rmsnorm.restype = None
        L.oracle_rope_rotate_half.argtypes = [c.c_void_p, c.c_int, c.c_void_p, c.c_void_p]
        L.oracle_rope_rotate_half.restype = None
        L.oracle_residual_rmsnorm_fp8.argtypes = [c.c_void_p] * 5 + [c.c_double, c.c_void_p, c.c_void_p,
                                                                     c.c_int64, c.c_int64, c.c_double,
                                                                     c.c_int, c.c_int]
        L.oracle_residual_rmsnorm_fp8.restype = c.c_int
        L.oracle_qkv_norm_rope_kvcache.argtypes = [c.c_void_p] * 11 + [c.c_int64] * 6 + [c.c_double, c.c_int]
        L.oracle_qkv_norm_rope_kvcache.restype = c.c_int
        L.oracle_gate_act_fp8.argtypes = [c.c_void_p, c.c_void_p, c.c_double, c.c_void_p, c.c_void_p,
                                          c.c_int64, c.c_int64, c.c_int, c.c_int, c.c_int]
        L.oracle_gate_act_fp8.restype = c.c_int
        L.oracle_gate_residual_adarms_fp8.argtypes = [c.c_void_p] * 7 + [c.c_double, c.c_void_p, c.c_void_p,
                                                                          c.c_int64, c.c_int64, c.c_int64,
                                                                          c.c_double, c.c_int, c.c_int]
        L.oracle_gate_residual_adarms_fp8.restype = c.c_int
        L.oracle_qkv_norm_rope_prepq_kvcache.argtypes = ([c.c_void_p] * 13 + [c.c_int64] * 6 +
                                                         [c.c_double, c.c_int, c.c_double, c.c_int, c.c_int,
                                                          c.c_double, c.c_double])
        L.oracle_qkv_norm_rope_prepq_kvcache.restype = c.c_int
        L.oracle_e2m1_encode.argtypes = [c.c_double]
        L.oracle_e2m1_encode.restype = c.c_uint8
        L.oracle_e2m1_decode.argtypes = [c.c_uint8]
        L.oracle_e2m1_decode.restype = c.c_double
        L.oracle_sf_swizzle_offset.argtypes = [c.c_int64, c.c_int64, c.c_int64]
        L.oracle_sf_swizzle_offset.restype = c.c_int64
        L.oracle_quant_nvfp4_row.argtypes = [c.c_void_p, c.c_int64, c.c_float, c.c_void_p, c.c_void_p]
        L.oracle_quant_nvfp4_row.restype = None
        L.oracle_residual_rmsnorm_nvfp4.argtypes = [c.c_void_p] * 6 + [c.c_double, c.c_void_p, c.c_int64,
                                                                       c.c_int64, c.c_double, c.c_int]
        L.oracle_residual_rmsnorm_nvfp4.restype = c.c_int
        L.oracle_gate_act_nvfp4.argtypes = [c.c_void_p] * 3 + [c.c_double, c.c_void_p, c.c_int64, c.c_int64,
                                                               c.c_int, c.c_int]
        L.oracle_gate_act_nvfp4.restype = c.c_int
        L.oracle_layernorm.argtypes = [c.c_void_p, c.c_int64, c.c_void_p, c.c_void_p, c.c_double, c.c_void_p]
        L.oracle_layernorm.restype = None
        L.oracle_residual_layernorm_quant.argtypes = ([c.c_void_p] * 6 + [c.c_double, c.c_void_p, c.c_void_p,
                                                       c.c_double, c.c_void_p, c.c_int64, c.c_int64, c.c_double,
                                                       c.c_int, c.c_int])
        L.oracle_residual_layernorm_quant.restype = c.c_int
        L.oracle_qkv_layernorm_rope_kvcache.argtypes = [c.c_void_p] * 13 + [c.c_int64] * 6 + [c.c_double, c.c_int]
        L.oracle_qkv_layernorm_rope_kvcache.restype = c.c_int
        _lib = L
    return _lib


# ----------------------------------------------------------------- scalars --
def decode16(bits, dt):
    f = lib().oracle_bf16_decode if dt == "bf16" else lib().oracle_f16_decode
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([f(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)


def round16(hi, lo, dt):
    f = lib().oracle_bf16_round if dt == "bf16" else lib().oracle_f16_round
    return int(f(float(hi), float(lo)))


def add16(x_bits, r_bits, dt):
    return int(lib().oracle_add16(int(x_bits), int(r_bits), _DT[dt]))


def e4m3_encode(v):
    return int(lib().oracle_e4m3_encode(float(v)))


def e4m3_decode(c):
    return float(lib().oracle_e4m3_decode(int(c)))


def act(name, g):
    return float(lib().oracle_act(_ACT[name], float(g)))


# ------------------------------------------------------------- components --
def quant_static(y, s):
    y = np.ascontiguousarray(y, dtype=np.float64)
    q = np.empty(y.size, dtype=np.uint8)
    lib().oracle_quant_static(_p(y), y.size, float(s), _p(q))
    return q.reshape(y.shape)


def quant_block128(y):
    y = np.ascontiguousarray(y, dtype=np.float64).ravel()
    q = np.empty(y.size, dtype=np.uint8)
    sc = np.empty((y.size + 127) // 128, dtype=np.float64)
    lib().oracle_quant_block128(_p(y), y.size, _p(q), _p(sc))
    return q, sc


def rmsnorm(h, w, eps):
    h = np.ascontiguousarray(h, dtype=np.float64)
    w = None if w is None else np.ascontiguousarray(w, dtype=np.float64)
    y = np.empty_like(h)
    lib().oracle_rmsnorm(_p(h), h.size, _p(w), float(eps), _p(y))
    return y


def rope_rotate_half(v, c, s):
    v = np.array(v, dtype=np.float64, copy=True)
    c = np.ascontiguousarray(c, dtype=np.float32)
    s = np.ascontiguousarray(s, dtype=np.float32)
    lib().oracle_rope_rotate_half(_p(v), v.size, _p(c), _p(s))
    return v


# -------------------------------------------------------------------- ops --
def residual_rmsnorm_fp8(x, residual_in, weight, eps, dt, quant, static_scale=None, want_y=False):
    """Op (a). x, residual_in: uint16 [M, D]; weight: uint16 [D] or None."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    r = np.ascontiguousarray(residual_in, dtype=np.uint16)
    M, D = x.shape
    w = None if weight is None else np.ascontiguousarray(weight, dtype=np.uint16)
    r_out = np.empty_like(r)
    q = np.empty((M, D), dtype=np.uint8)
    nb = (D + 127) // 128
    sc = np.empty((M, nb), dtype=np.float64) if quant == "block128" else None
    y = np.empty((M, D), dtype=np.float64) if want_y else None
    s = float(static_scale) if quant == "static" else 0.0
    rc = lib().oracle_residual_rmsnorm_fp8(_p(x), _p(r), _p(r_out), _p(w), _p(q), s, _p(sc), _p(y),
                                           M, D, _f32(eps), _DT[dt], _QM[quant])
    if rc != 0:
        raise ValueError("oracle_residual_rmsnorm_fp8: bad argument")
    return {"residual_out": r_out, "out_fp8": q, "block_scales": sc, "y": y}


def qkv_norm_rope_kvcache(qkv, q_norm_w, k_norm_w, cos_tab, sin_tab, positions, Hq, Hkv, hd, capacity,
                          eps, dt, slots=None, k_cache=None, v_cache=None):
    """Op (b). Returns q_out (fp64 [M,Hq,hd]), k_cache (fp64 [cap,Hkv,hd]),
    v_cache (uint16 [cap,Hkv,hd]) and the status word.  Cache rows that are
    not written keep their initial contents (NaN / the given arrays)."""
    qkv = np.ascontiguousarray(qkv, dtype=np.uint16)
    M = qkv.shape[0]
    cos_tab = np.ascontiguousarray(cos_tab, dtype=np.float32)
    sin_tab = np.ascontiguousarray(sin_tab, dtype=np.float32)
    max_pos = cos_tab.shape[0]
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    sl = None if slots is None else np.ascontiguousarray(slots, dtype=np.int64)
    qw = None if q_norm_w is None else np.ascontiguousarray(q_norm_w, dtype=np.uint16)
    kw = None if k_norm_w is None else np.ascontiguousarray(k_norm_w, dtype=np.uint16)
    q_out = np.full((M, Hq, hd), np.nan, dtype=np.float64)
    kc = (np.full((capacity, Hkv, hd), np.nan, dtype=np.float64) if k_cache is None
          else np.array(k_cache, dtype=np.float64, copy=True))
    vc = (np.zeros((capacity, Hkv, hd), dtype=np.uint16) if v_cache is None
          else np.array(v_cache, dtype=np.uint16, copy=True))
    status = np.zeros(1, dtype=np.int32)
    rc = lib().oracle_qkv_norm_rope_kvcache(_p(qkv), _p(qw), _p(kw), _p(cos_tab), _p(sin_tab), _p(pos), _p(sl),
                                            _p(q_out), _p(kc), _p(vc), _p(status), M, Hq, Hkv, hd, max_pos,
                                            capacity, _f32(eps), _DT[dt])
    if rc != 0:
        raise ValueError("oracle_qkv_norm_rope_kvcache: bad argument")
    return {"q_out": q_out, "k_cache": kc, "v_cache": vc, "status": int(status[0])}


def qkv_norm_rope_prepq_kvcache(qkv, q_norm_w, k_norm_w, cos_tab, sin_tab, positions, Hq, Hkv, hd, capacity,
                                eps, dt, q_scale=1.0, q_layout="token", kv="16", k_scale=None, v_scale=None,
                                k_cache=None, v_cache=None, slots=None):
    """NEXT-2 op.  q_out is fp64 [M, Hq, hd] (q_layout "token") or [Hq, M, hd]
    ("head"); with kv "16" the caches are as op (b) (fp64 K, uint16 V), with
    kv "e4m3" both are uint8 codes (initial contents: the given arrays or
    0x7E sentinels)."""
    qkv = np.ascontiguousarray(qkv, dtype=np.uint16)
    M = qkv.shape[0]
    cos_tab = np.ascontiguousarray(cos_tab, dtype=np.float32)
    sin_tab = np.ascontiguousarray(sin_tab, dtype=np.float32)
    max_pos = cos_tab.shape[0]
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    qw = None if q_norm_w is None else np.ascontiguousarray(q_norm_w, dtype=np.uint16)
    kw = None if k_norm_w is None else np.ascontiguousarray(k_norm_w, dtype=np.uint16)
    sl = None if slots is None else np.ascontiguousarray(slots, dtype=np.int64)
    head = {"token": 0, "head": 1}[q_layout]
    fp8 = {"16": 0, "e4m3": 1}[kv]
    q_out = np.full((Hq, M, hd) if head else (M, Hq, hd), np.nan, dtype=np.float64)
    kc = vc = kc8 = vc8 = None
    if fp8:
        kc8 = (np.full((capacity, Hkv, hd), 0x7E, dtype=np.uint8) if k_cache is None
               else np.array(k_cache, dtype=np.uint8, copy=True))
        vc8 = (np.full((capacity, Hkv, hd), 0x7E, dtype=np.uint8) if v_cache is None
               else np.array(v_cache, dtype=np.uint8, copy=True))
    else:
        kc = (np.full((capacity, Hkv, hd), np.nan, dtype=np.float64) if k_cache is None
              else np.array(k_cache, dtype=np.float64, copy=True))
        vc = (np.zeros((capacity, Hkv, hd), dtype=np.uint16) if v_cache is None
              else np.array(v_cache, dtype=np.uint16, copy=True))
    status = np.zeros(1, dtype=np.int32)
    rc = lib().oracle_qkv_norm_rope_prepq_kvcache(
        _p(qkv), _p(qw), _p(kw), _p(cos_tab), _p(sin_tab), _p(pos), _p(sl), _p(q_out), _p(kc), _p(vc), _p(kc8), _p(vc8),
        _p(status), M, Hq, Hkv, hd, max_pos, capacity, _f32(eps), _DT[dt], float(q_scale), head, fp8,
        float(k_scale or 0.0), float(v_scale or 0.0))
    if rc != 0:
        raise ValueError("oracle_qkv_norm_rope_prepq_kvcache: bad argument")
    return {"q_out": q_out, "k_cache": kc8 if fp8 else kc, "v_cache": vc8 if fp8 else vc,
            "status": int(status[0])}


def gate_act_fp8(gate_up, act_name, dt, quant, static_scale=None, want_a=False):
    """Op (c). gate_up: uint16 [M, 2I] interleaved (g0,u0,g1,u1,...)."""
    gu = np.ascontiguousarray(gate_up, dtype=np.uint16)
    M, two_i = gu.shape
    I = two_i // 2
    q = np.empty((M, I), dtype=np.uint8)
    nb = (I + 127) // 128
    sc = np.empty((M, nb), dtype=np.float64) if quant == "block128" else None
    a = np.empty((M, I), dtype=np.float64) if want_a else None
    s = float(static_scale) if quant == "static" else 0.0
    rc = lib().oracle_gate_act_fp8(_p(gu), _p(q), s, _p(sc), _p(a), M, I, _ACT[act_name], _DT[dt], _QM[quant])
    if rc != 0:
        raise ValueError("oracle_gate_act_fp8: bad argument")
    return {"out_fp8": q, "block_scales": sc, "a": a}


def gate_residual_adarms_fp8(x, gate, residual_in, scale, shift, eps, dt, quant, rows_per_cond, static_scale=None,
                             want_y=False):
    """NEXT-1 op.  x, residual_in: uint16 [M, D]; gate / scale / shift: uint16
    [ceil(M / rows_per_cond), D] or None."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    r = np.ascontiguousarray(residual_in, dtype=np.uint16)
    M, D = x.shape
    g, sc, sh = (None if a is None else np.ascontiguousarray(a, dtype=np.uint16) for a in (gate, scale, shift))
    r_out = np.empty_like(r)
    q = np.empty((M, D), dtype=np.uint8)
    nb = (D + 127) // 128
    bs = np.empty((M, nb), dtype=np.float64) if quant == "block128" else None
    y = np.empty((M, D), dtype=np.float64) if want_y else None
    s = float(static_scale) if quant == "static" else 0.0
    rc = lib().oracle_gate_residual_adarms_fp8(_p(x), _p(g), _p(r), _p(r_out), _p(sc), _p(sh), _p(q), s, _p(bs),
                                               _p(y), M, D, int(rows_per_cond), _f32(eps), _DT[dt], _QM[quant])
    if rc != 0:
        raise ValueError("oracle_gate_residual_adarms_fp8: bad argument")
    return {"residual_out": r_out, "out_fp8": q, "block_scales": bs, "y": y}


# ------------------------------------------------------------------ NEXT-3 --
def e2m1_encode(v):
    return int(lib().oracle_e2m1_encode(float(v)))


def e2m1_decode(c):
    return float(lib().oracle_e2m1_decode(int(c)))


def sf_swizzle_offset(r, c, n_cols):
    return int(lib().oracle_sf_swizzle_offset(int(r), int(c), int(n_cols)))


def quant_nvfp4_row(y, global_scale):
    """One row (length a multiple of 16) -> (packed uint8 [n/2], sf uint8 [n/16])."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    n = y.shape[0]
    packed = np.empty(n // 2, dtype=np.uint8)
    sf = np.empty(n // 16, dtype=np.uint8)
    lib().oracle_quant_nvfp4_row(_p(y), n, float(global_scale), _p(packed), _p(sf))
    return packed, sf


def residual_rmsnorm_nvfp4(x, residual_in, weight, eps, dt, global_scale, want_y=False):
    """Op (a) with an NVFP4 output: residual_out, out_fp4 [M, D/2], sf [M, D/16]."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    r = np.ascontiguousarray(residual_in, dtype=np.uint16)
    M, D = x.shape
    w = None if weight is None else np.ascontiguousarray(weight, dtype=np.uint16)
    r_out = np.empty_like(r)
    q = np.empty((M, D // 2), dtype=np.uint8)
    sf = np.empty((M, D // 16), dtype=np.uint8)
    y = np.empty((M, D), dtype=np.float64) if want_y else None
    rc = lib().oracle_residual_rmsnorm_nvfp4(_p(x), _p(r), _p(r_out), _p(w), _p(q), _p(sf), float(global_scale),
                                             _p(y), M, D, _f32(eps), _DT[dt])
    if rc != 0:
        raise ValueError("oracle_residual_rmsnorm_nvfp4: bad argument")
    return {"residual_out": r_out, "out_fp4": q, "sf": sf, "y": y}


def gate_act_nvfp4(gate_up, act_name, dt, global_scale, want_a=False):
    """Op (c) with an NVFP4 output: out_fp4 [M, I/2], sf [M, I/16]."""
    gu = np.ascontiguousarray(gate_up, dtype=np.uint16)
    M, two_i = gu.shape
    I = two_i // 2
    q = np.empty((M, I // 2), dtype=np.uint8)
    sf = np.empty((M, I // 16), dtype=np.uint8)
    a = np.empty((M, I), dtype=np.float64) if want_a else None
    rc = lib().oracle_gate_act_nvfp4(_p(gu), _p(q), _p(sf), float(global_scale), _p(a), M, I, _ACT[act_name],
                                     _DT[dt])
    if rc != 0:
        raise ValueError("oracle_gate_act_nvfp4: bad argument")
    return {"out_fp4": q, "sf": sf, "a": a}


def sf_swizzle(sf_rowmajor):
    """Row-major scale factors [M, C] -> the 128x4-swizzled byte array
    (padded to 128-row / 4-column atoms; padding bytes 0)."""
    M, C = sf_rowmajor.shape
    out = np.zeros(((M + 127) // 128) * 128 * ((C + 3) // 4) * 4, dtype=np.uint8)
    for r in range(M):
        for c in range(C):
            out[sf_swizzle_offset(r, c, C)] = sf_rowmajor[r, c]
    return out


# ------------------------------------------------------------------ NEXT-4 --
def layernorm(h, w=None, b=None, eps=1e-6):
    h = np.ascontiguousarray(h, dtype=np.float64)
    y = np.empty_like(h)
    wv = None if w is None else np.ascontiguousarray(w, dtype=np.float64)
    bv = None if b is None else np.ascontiguousarray(b, dtype=np.float64)
    lib().oracle_layernorm(_p(h), h.shape[0], _p(wv), _p(bv), float(eps), _p(y))
    return y


def residual_layernorm(x, residual_in, weight, bias, eps, dt, quant, static_scale=None, global_scale=None,
                       want_y=False):
    """Op (a) with LayerNorm.  quant: "static" / "block128" (FP8, out [M, D])
    or "nvfp4" (out [M, D/2] + sf [M, D/16])."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    r = np.ascontiguousarray(residual_in, dtype=np.uint16)
    M, D = x.shape
    w = None if weight is None else np.ascontiguousarray(weight, dtype=np.uint16)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
    mode = {"static": 0, "block128": 1, "nvfp4": 2}[quant]
    r_out = np.empty_like(r)
    q = np.empty((M, D // 2) if mode == 2 else (M, D), dtype=np.uint8)
    bs = np.empty((M, (D + 127) // 128), dtype=np.float64) if mode == 1 else None
    sf = np.empty((M, D // 16), dtype=np.uint8) if mode == 2 else None
    y = np.empty((M, D), dtype=np.float64) if want_y else None
    rc = lib().oracle_residual_layernorm_quant(_p(x), _p(r), _p(r_out), _p(w), _p(b), _p(q),
                                               float(static_scale or 0.0), _p(bs), _p(sf), float(global_scale or 0.0),
                                               _p(y), M, D, _f32(eps), _DT[dt], mode)
    if rc != 0:
        raise ValueError("oracle_residual_layernorm_quant: bad argument")
    return {"residual_out": r_out, "out": q, "block_scales": bs, "sf": sf, "y": y}


def qkv_layernorm_rope_kvcache(qkv, q_w, q_b, k_w, k_b, cos_tab, sin_tab, positions, Hq, Hkv, hd, capacity, eps, dt,
                               slots=None, v_cache=None):
    """Op (b) with per-head LayerNorm ([Hq, hd] / [Hkv, hd] affine, each
    optional).  Returns q_out (fp64), k_cache (fp64), v_cache (uint16), status."""
    qkv = np.ascontiguousarray(qkv, dtype=np.uint16)
    M = qkv.shape[0]
    cos_tab = np.ascontiguousarray(cos_tab, dtype=np.float32)
    sin_tab = np.ascontiguousarray(sin_tab, dtype=np.float32)
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    sl = None if slots is None else np.ascontiguousarray(slots, dtype=np.int64)
    prm = [None if a is None else np.ascontiguousarray(a, dtype=np.uint16) for a in (q_w, q_b, k_w, k_b)]
    q_out = np.full((M, Hq, hd), np.nan, dtype=np.float64)
    kc = np.full((capacity, Hkv, hd), np.nan, dtype=np.float64)
    vc = (np.zeros((capacity, Hkv, hd), dtype=np.uint16) if v_cache is None
          else np.array(v_cache, dtype=np.uint16, copy=True))
    status = np.zeros(1, dtype=np.int32)
    rc = lib().oracle_qkv_layernorm_rope_kvcache(_p(qkv), *[_p(a) for a in prm], _p(cos_tab), _p(sin_tab), _p(pos),
                                                 _p(sl), _p(q_out), _p(kc), _p(vc), _p(status), M, Hq, Hkv, hd,
                                                 cos_tab.shape[0], capacity, _f32(eps), _DT[dt])
    if rc != 0:
        raise ValueError("oracle_qkv_layernorm_rope_kvcache: bad argument")
    return {"q_out": q_out, "k_cache": kc, "v_cache": vc, "status": int(status[0])}
