"""Fused non-GEMM transformer-layer ops for B200: Python binding of libfrt.so.

Argument marshalling only.  Every op runs in the CUDA kernels of libfrt.so;
there is no CPU or PyTorch fallback: if the library is missing or a call
fails, a ``FrtError`` is raised.  PyTorch supplies device memory and streams.

Functions carry the C names of ``include/frt.h``:

    frt_residual_rmsnorm_fp8(x, residual_in, residual_out, weight, out_fp8, ...)
    frt_qkv_norm_rope_kvcache(qkv, q_norm_w, k_norm_w, cos, sin, positions, ...)
    frt_gate_act_fp8(gate_up, out_fp8, ...)
    frt_qkv_norm_rope_prepq_kvcache(...)   (NEXT-2)
    frt_gate_residual_adarms_fp8(...)      (NEXT-1)
    frt_noop(grid, block), frt_copy_rows(src, dst)      (launch-floor probes)
    frt_set_pdl / frt_get_pdl, frt_set_wait_polls / frt_get_wait_polls

``load_debug()`` opens the bounds-checked build (libfrt_debug.so,
include/frt_debug.h); ``using_library(load_debug())`` routes these functions
through it and ``bounds_violations()`` reads and clears its counter.
"""
import contextlib
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfrt.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "libfrt_debug.so")

FRT_OK, FRT_ERR_INVALID_ARG, FRT_ERR_UNSUPPORTED, FRT_ERR_CUDA = 0, 1, 2, 3
DTYPE = {torch.float16: 0, torch.bfloat16: 1}
QUANT = {"static": 0, "block128": 1}
ACT = {"gelu_tanh": 0, "silu": 1, "relu2": 2}

# C entry points declared in include/frt.h
EXPORTS = ("frt_residual_rmsnorm_fp8", "frt_qkv_norm_rope_kvcache", "frt_gate_act_fp8",
           "frt_chain_persistent", "frt_residual_layernorm_fp8", "frt_residual_layernorm_nvfp4",
           "frt_qkv_layernorm_rope_kvcache",
           "frt_residual_rmsnorm_nvfp4", "frt_gate_act_nvfp4", "frt_qkv_norm_rope_prepq_kvcache",
           "frt_gate_residual_adarms_fp8", "frt_noop", "frt_copy_rows", "frt_set_pdl", "frt_get_pdl", "frt_set_wait_polls",
           "frt_get_wait_polls", "frt_status_string")


class FrtError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__("%s failed: %s" % (fn, msg))
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfrt.so (once) and declare its C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = _open(path)
    return _lib


_debug_lib = None


def load_debug(path: str = DEBUG_LIB_PATH) -> ctypes.CDLL:
    """Load the bounds-checked build libfrt_debug.so (once): the same entry
    points plus frt_debug_bounds_violations (include/frt_debug.h).  Use it
    through ``using_library``."""
    global _debug_lib
    if _debug_lib is None:
        L = _open(path)
        L.frt_debug_bounds_violations.argtypes = [ctypes.c_void_p]
        L.frt_debug_bounds_violations.restype = ctypes.c_int
        _debug_lib = L
    return _debug_lib


def bounds_violations() -> int:
    """Out-of-range accesses the bounds-checked build skipped since the last
    call (synchronises the device; resets the count)."""
    n = ctypes.c_uint(0)
    _check("frt_debug_bounds_violations", load_debug().frt_debug_bounds_violations(ctypes.byref(n)))
    return int(n.value)


@contextlib.contextmanager
def using_library(L):
    """Route this module's calls through the library handle L (e.g. the
    bounds-checked build) inside the block."""
    global _lib
    prev = load()
    _lib = L
    try:
        yield L
    finally:
        _lib = prev


def _open(path):
    if not os.path.exists(path):
        raise FrtError("load", -1, "%s is missing; build it with `python -m memory_bound_non_b200.build`" % path)
    L = ctypes.CDLL(path)
    c = ctypes
    vp, i32, f32 = c.c_void_p, c.c_int, c.c_float
    L.frt_residual_rmsnorm_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, f32, i32, i32, vp]
    L.frt_residual_rmsnorm_fp8.restype = i32
    L.frt_qkv_norm_rope_kvcache.argtypes = [vp] * 10 + [i32] * 6 + [f32, i32, vp]
    L.frt_qkv_norm_rope_kvcache.restype = i32
    L.frt_qkv_norm_rope_prepq_kvcache.argtypes = [vp] * 10 + [i32] * 6 + [f32, f32, i32, i32, vp, i32, vp]
    L.frt_qkv_norm_rope_prepq_kvcache.restype = i32
    L.frt_chain_persistent.argtypes = [vp, i32, i32] + [vp] * 6 + [i32] * 8 + [f32, i32, i32, i32, vp]
    L.frt_chain_persistent.restype = i32
    L.frt_residual_layernorm_fp8.argtypes = [vp] * 8 + [i32, i32, f32, i32, i32, vp]
    L.frt_residual_layernorm_fp8.restype = i32
    L.frt_residual_layernorm_nvfp4.argtypes = [vp] * 8 + [i32, i32, f32, i32, i32, vp]
    L.frt_residual_layernorm_nvfp4.restype = i32
    L.frt_qkv_layernorm_rope_kvcache.argtypes = [vp] * 12 + [i32] * 6 + [f32, i32, vp]
    L.frt_qkv_layernorm_rope_kvcache.restype = i32
    L.frt_residual_rmsnorm_nvfp4.argtypes = [vp] * 7 + [i32, i32, f32, i32, i32, vp]
    L.frt_residual_rmsnorm_nvfp4.restype = i32
    L.frt_gate_act_nvfp4.argtypes = [vp] * 4 + [i32, i32, i32, i32, i32, vp]
    L.frt_gate_act_nvfp4.restype = i32
    L.frt_gate_act_fp8.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]
    L.frt_gate_act_fp8.restype = i32
    L.frt_gate_residual_adarms_fp8.argtypes = [vp] * 9 + [i32, i32, i32, f32, i32, i32, vp]
    L.frt_gate_residual_adarms_fp8.restype = i32
    L.frt_noop.argtypes = [i32, i32, vp]
    L.frt_noop.restype = i32
    L.frt_copy_rows.argtypes = [vp, vp, i32, i32, vp]
    L.frt_copy_rows.restype = i32
    L.frt_set_pdl.argtypes = [i32]
    L.frt_set_pdl.restype = None
    L.frt_get_pdl.argtypes = []
    L.frt_get_pdl.restype = i32
    L.frt_set_wait_polls.argtypes = [i32]
    L.frt_set_wait_polls.restype = i32
    L.frt_get_wait_polls.argtypes = []
    L.frt_get_wait_polls.restype = i32
    L.frt_status_string.argtypes = [i32]
    L.frt_status_string.restype = c.c_char_p
    return L


def status_string(status: int) -> str:
    return load().frt_status_string(int(status)).decode()


def _check(fn, status):
    if status != FRT_OK:
        raise FrtError(fn, status, status_string(status))


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise FrtError("marshal", FRT_ERR_INVALID_ARG, "tensor is not on a CUDA device")
    if not t.is_contiguous():
        raise FrtError("marshal", FRT_ERR_INVALID_ARG, "tensor is not contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def frt_residual_rmsnorm_fp8(x, residual_in, residual_out, weight, out_fp8, static_scale=None,
                             block_scales=None, eps=1e-6, quant="static", stream=None):
    """Op (a): residual add + RMSNorm (+ weight) + FP8 e4m3.  x, residual_*: [M, D]
    fp16/bf16; weight [D] or None; out_fp8 [M, D] uint8; static_scale fp32[1]
    (static) or block_scales fp32 [M, ceil(D/128)] (block128)."""
    M, D = x.shape
    st = load().frt_residual_rmsnorm_fp8(
        _ptr(x), _ptr(residual_in), _ptr(residual_out), _ptr(weight), _ptr(out_fp8), _ptr(static_scale),
        _ptr(block_scales), M, D, float(eps), DTYPE[x.dtype], QUANT[quant], _stream(stream))
    _check("frt_residual_rmsnorm_fp8", st)


def frt_qkv_norm_rope_kvcache(qkv, q_norm_w, k_norm_w, cos_tab, sin_tab, positions, q_out, k_cache, v_cache,
                              Hq, Hkv, hd, status=None, eps=1e-6, stream=None):
    """Op (b): QKV split + q/k RMSNorm + rotate-half RoPE + Q staging + KV write.
    qkv [M, (Hq+2Hkv)*hd]; cos/sin fp32 [max_pos, hd/2]; positions int32 [M];
    q_out [M, Hq, hd]; caches [capacity, Hkv, hd]; status int32[1] or None."""
    M = qkv.shape[0]
    max_pos = cos_tab.shape[0]
    capacity = k_cache.shape[0]
    st = load().frt_qkv_norm_rope_kvcache(
        _ptr(qkv), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(cos_tab), _ptr(sin_tab), _ptr(positions), _ptr(q_out),
        _ptr(k_cache), _ptr(v_cache), _ptr(status), M, Hq, Hkv, hd, max_pos, capacity, float(eps),
        DTYPE[qkv.dtype], _stream(stream))
    _check("frt_qkv_norm_rope_kvcache", st)


SF_LAYOUT = {"rows": 0, "swizzled": 1}


def nvfp4_sf_bytes(rows, n, layout="rows"):
    """Bytes of the scale-factor array of an [rows, n] NVFP4 output."""
    if layout == "rows":
        return rows * (n // 16)
    return ((rows + 127) // 128) * 128 * ((n // 16 + 3) // 4) * 4


def frt_residual_rmsnorm_nvfp4(x, residual_in, residual_out, weight, out_fp4, out_sf, global_scale, eps=1e-6,
                               sf_layout="rows", stream=None):
    """NEXT-3: op (a) with an NVFP4 output: out_fp4 uint8 [M, D/2] (two e2m1
    per byte), out_sf uint8 scale factors (see nvfp4_sf_bytes), global_scale
    fp32[1] on the device."""
    M, D = x.shape
    st = load().frt_residual_rmsnorm_nvfp4(
        _ptr(x), _ptr(residual_in), _ptr(residual_out), _ptr(weight), _ptr(out_fp4), _ptr(out_sf),
        _ptr(global_scale), M, D, float(eps), DTYPE[x.dtype], SF_LAYOUT[sf_layout], _stream(stream))
    _check("frt_residual_rmsnorm_nvfp4", st)


def frt_gate_act_nvfp4(gate_up, out_fp4, out_sf, global_scale, act="gelu_tanh", sf_layout="rows", stream=None):
    """NEXT-3: op (c) with an NVFP4 output: out_fp4 uint8 [M, I/2]."""
    M, two_i = gate_up.shape
    st = load().frt_gate_act_nvfp4(_ptr(gate_up), _ptr(out_fp4), _ptr(out_sf), _ptr(global_scale), M, two_i // 2,
                                   ACT[act], DTYPE[gate_up.dtype], SF_LAYOUT[sf_layout], _stream(stream))
    _check("frt_gate_act_nvfp4", st)


def frt_residual_layernorm_fp8(x, residual_in, residual_out, weight, bias, out_fp8, static_scale=None,
                              block_scales=None, eps=1e-6, quant="static", stream=None):
    """NEXT-4: op (a) with LayerNorm (weight / bias [D] or None) + FP8."""
    M, D = x.shape
    st = load().frt_residual_layernorm_fp8(
        _ptr(x), _ptr(residual_in), _ptr(residual_out), _ptr(weight), _ptr(bias), _ptr(out_fp8), _ptr(static_scale),
        _ptr(block_scales), M, D, float(eps), DTYPE[x.dtype], QUANT[quant], _stream(stream))
    _check("frt_residual_layernorm_fp8", st)


def frt_residual_layernorm_nvfp4(x, residual_in, residual_out, weight, bias, out_fp4, out_sf, global_scale, eps=1e-6,
                                 sf_layout="rows", stream=None):
    """NEXT-4: op (a) with LayerNorm + NVFP4 (the ViT add_layer_norm producer)."""
    M, D = x.shape
    st = load().frt_residual_layernorm_nvfp4(
        _ptr(x), _ptr(residual_in), _ptr(residual_out), _ptr(weight), _ptr(bias), _ptr(out_fp4), _ptr(out_sf),
        _ptr(global_scale), M, D, float(eps), DTYPE[x.dtype], SF_LAYOUT[sf_layout], _stream(stream))
    _check("frt_residual_layernorm_nvfp4", st)


def frt_qkv_layernorm_rope_kvcache(qkv, q_w, q_b, k_w, k_b, cos_tab, sin_tab, positions, q_out, k_cache, v_cache,
                                   Hq, Hkv, hd, status=None, eps=1e-6, stream=None):
    """NEXT-4: op (b) with per-head LayerNorm on Q and K (affine rows
    [Hq, hd] / [Hkv, hd], each optional)."""
    M = qkv.shape[0]
    st = load().frt_qkv_layernorm_rope_kvcache(
        _ptr(qkv), _ptr(q_w), _ptr(q_b), _ptr(k_w), _ptr(k_b), _ptr(cos_tab), _ptr(sin_tab), _ptr(positions),
        _ptr(q_out), _ptr(k_cache), _ptr(v_cache), _ptr(status), M, Hq, Hkv, hd, cos_tab.shape[0], k_cache.shape[0],
        float(eps), DTYPE[qkv.dtype], _stream(stream))
    _check("frt_qkv_layernorm_rope_kvcache", st)


# field order of frt_chain_layer (include/frt.h)
CHAIN_LAYER_FIELDS = ("x_attn", "x_ffn", "w_attn", "w_ffn", "qkv", "q_norm_w", "k_norm_w", "gate_up", "k_cache",
                      "v_cache", "q_out", "q8_attn", "q8_ffn", "act8", "bs_attn", "bs_ffn", "bs_act")


def chain_layer_table(layers, device):
    """Device array of frt_chain_layer structs (17 pointers each) for a list of
    objects carrying the CHAIN_LAYER_FIELDS tensors (or None)."""
    import ctypes as c
    host = (c.c_uint64 * (len(CHAIN_LAYER_FIELDS) * len(layers)))()
    for i, L in enumerate(layers):
        for j, name in enumerate(CHAIN_LAYER_FIELDS):
            t = getattr(L, name)
            host[i * len(CHAIN_LAYER_FIELDS) + j] = 0 if t is None else t.data_ptr()
    buf = torch.frombuffer(bytearray(bytes(host)), dtype=torch.uint8)
    return buf.to(device)


def frt_chain_persistent(table, n_layers, steps, residual, cos_tab, sin_tab, positions, scales, status, Hq, Hkv,
                         hd, I, capacity, eps=1e-6, quant="static", act="gelu_tanh", stream=None):
    """NEXT-4: steps x layers x (norm, QKV, norm, gate) as one kernel launch;
    table from chain_layer_table.  status (int32[1]) gets bit 0 for a row
    whose position is out of range and bit 2 when a layer record holds a
    pointer below its field's alignment (then nothing is written)."""
    M, D = residual.shape
    st = load().frt_chain_persistent(
        _ptr(table), n_layers, steps, _ptr(residual), _ptr(cos_tab), _ptr(sin_tab), _ptr(positions), _ptr(scales),
        _ptr(status), M, D, Hq, Hkv, hd, I, cos_tab.shape[0], capacity, float(eps), DTYPE[residual.dtype],
        QUANT[quant], ACT[act], _stream(stream))
    _check("frt_chain_persistent", st)


Q_LAYOUT = {"token": 0, "head": 1}
KV_FORMAT = {"16": 0, "e4m3": 1}


def frt_qkv_norm_rope_prepq_kvcache(qkv, q_norm_w, k_norm_w, cos_tab, sin_tab, positions, q_out, k_cache, v_cache,
                                    Hq, Hkv, hd, q_scale=1.0, q_layout="token", kv="16", kv_scales=None,
                                    status=None, eps=1e-6, stream=None):
    """NEXT-2: op (b) + Q softmax-scale pre-multiply / head-major Q layout
    (q_out [Hq, M, hd]) + optional e4m3 KV cache (uint8 caches; kv_scales
    fp32[2] = (k_scale, v_scale) on the device)."""
    M = qkv.shape[0]
    max_pos = cos_tab.shape[0]
    capacity = k_cache.shape[0]
    st = load().frt_qkv_norm_rope_prepq_kvcache(
        _ptr(qkv), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(cos_tab), _ptr(sin_tab), _ptr(positions), _ptr(q_out),
        _ptr(k_cache), _ptr(v_cache), _ptr(status), M, Hq, Hkv, hd, max_pos, capacity, float(eps), float(q_scale),
        Q_LAYOUT[q_layout], KV_FORMAT[kv], _ptr(kv_scales), DTYPE[qkv.dtype], _stream(stream))
    _check("frt_qkv_norm_rope_prepq_kvcache", st)


def frt_gate_act_fp8(gate_up, out_fp8, static_scale=None, block_scales=None, act="gelu_tanh", quant="static",
                     stream=None):
    """Op (c): act(g) * u on interleaved [M, 2I] gate/up + FP8 e4m3 -> [M, I]."""
    M, two_i = gate_up.shape
    st = load().frt_gate_act_fp8(_ptr(gate_up), _ptr(out_fp8), _ptr(static_scale), _ptr(block_scales), M,
                                 two_i // 2, ACT[act], DTYPE[gate_up.dtype], QUANT[quant], _stream(stream))
    _check("frt_gate_act_fp8", st)


def frt_gate_residual_adarms_fp8(x, gate, residual_in, residual_out, scale, shift, out_fp8, static_scale=None,
                                 block_scales=None, rows_per_cond=None, eps=1e-6, quant="static", stream=None):
    """NEXT-1: h = residual + gate * x (rounded once), y = RMSNorm(h) * (1 + scale)
    + shift, FP8 e4m3.  gate / scale / shift: [ceil(M / rows_per_cond), D] or
    None; rows_per_cond defaults to M (one condition for all rows)."""
    M, D = x.shape
    rpc = M if rows_per_cond is None else int(rows_per_cond)
    st = load().frt_gate_residual_adarms_fp8(
        _ptr(x), _ptr(gate), _ptr(residual_in), _ptr(residual_out), _ptr(scale), _ptr(shift), _ptr(out_fp8),
        _ptr(static_scale), _ptr(block_scales), M, D, max(rpc, 1), float(eps), DTYPE[x.dtype], QUANT[quant],
        _stream(stream))
    _check("frt_gate_residual_adarms_fp8", st)


def frt_set_pdl(enable: bool):
    """Programmatic dependent launch on/off for every later launch (process-wide)."""
    load().frt_set_pdl(1 if enable else 0)


def frt_get_pdl() -> bool:
    return bool(load().frt_get_pdl())


FRT_DEFAULT_WAIT_POLLS = 1 << 22


def frt_set_wait_polls(polls: int):
    """Bound on the polls of the QKV ops' bulk-copy barrier wait (process-wide;
    FRT_DEFAULT_WAIT_POLLS restores the default; 0 gives up at once)."""
    _check("frt_set_wait_polls", load().frt_set_wait_polls(int(polls)))


def frt_get_wait_polls() -> int:
    return int(load().frt_get_wait_polls())


def frt_noop(grid=1, block=32, stream=None):
    """Empty kernel: the launch floor."""
    _check("frt_noop", load().frt_noop(int(grid), int(block), _stream(stream)))


def frt_copy_rows(src, dst, stream=None):
    """Dependent-copy probe: each row of src ([rows, n] contiguous, n * itemsize
    a multiple of 16 bytes) copied to dst (may be src)."""
    rows = src.shape[0]
    row_bytes = src[0].numel() * src.element_size() if rows else 16
    _check("frt_copy_rows", load().frt_copy_rows(_ptr(src), _ptr(dst), rows, row_bytes, _stream(stream)))
