"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/frt.h declares, and rejects bad arguments on the host before any CUDA
call (fake, never-dereferenced pointers)."""
import ctypes
import os
import re

import pytest

import memory_bound_non_b200 as frt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
A = 0x100000          # a 256-byte aligned fake device address (never dereferenced)
INV, UNSUP, OK = frt.FRT_ERR_INVALID_ARG, frt.FRT_ERR_UNSUPPORTED, frt.FRT_OK


def declared_functions():
    src = open(os.path.join(ROOT, "include", "frt.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(frt_[a-z0-9_]+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_symbol():
    L = frt.load()
    names = declared_functions()
    assert set(names) == set(frt.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_debug_library_exports_every_declared_symbol():
    """libfrt_debug.so (the bounds-checked build) exports frt.h's entry points
    and the one include/frt_debug.h adds, which rejects a NULL count on the
    host."""
    src = open(os.path.join(ROOT, "include", "frt_debug.h")).read()
    extra = sorted(set(re.findall(r"\b(frt_[a-z0-9_]+)\s*\(", re.sub(r"/\*.*?\*/", "", src, flags=re.S))))
    assert extra == ["frt_debug_bounds_violations"]
    D = frt.load_debug()
    for n in declared_functions() + extra:
        assert hasattr(D, n), n
    assert not hasattr(frt.load(), "frt_debug_bounds_violations")
    assert D.frt_debug_bounds_violations(None) == INV


def test_status_strings():
    for s in (OK, INV, UNSUP, frt.FRT_ERR_CUDA, 99):
        assert isinstance(frt.status_string(s), str) and frt.status_string(s)


def a_call(M=4, D=256, x=A, r=A, ro=A, w=None, q=A, ss=A, bs=None, dt=1, qm=0):
    return frt.load().frt_residual_rmsnorm_fp8(x, r, ro, w, q, ss, bs, M, D, 1e-6, dt, qm, None)


@pytest.mark.parametrize("kw,want", [
    (dict(M=-1), INV), (dict(D=0), INV), (dict(D=12), INV), (dict(x=None), INV), (dict(ro=None), INV),
    (dict(q=None), INV), (dict(x=A + 8), INV), (dict(r=A + 4), INV), (dict(q=A + 4), INV),
    (dict(w=A + 2), INV), (dict(ss=None), INV), (dict(qm=1, bs=None), INV), (dict(dt=2), INV),
    (dict(qm=5), INV), (dict(D=32776), UNSUP), (dict(M=0), OK), (dict(M=0, qm=1, bs=A), OK),
    (dict(M=0, x=None, ro=None, q=None, ss=None), OK), (dict(M=0, D=12), INV), (dict(M=0, dt=4), INV),
])
def test_residual_rmsnorm_host_validation(kw, want):
    assert a_call(**kw) == want


def b_call(M=4, Hq=8, Hkv=2, hd=128, qkv=A, cos=A, sin=A, pos=A, qo=A, kc=A, vc=A, qw=None, kw=None,
           status=None, max_pos=64, cap=64, dt=1):
    return frt.load().frt_qkv_norm_rope_kvcache(qkv, qw, kw, cos, sin, pos, qo, kc, vc, status, M, Hq, Hkv, hd,
                                                max_pos, cap, 1e-6, dt, None)


@pytest.mark.parametrize("kw,want", [
    (dict(M=-3), INV), (dict(Hq=0), INV), (dict(Hkv=0), INV), (dict(Hq=6, Hkv=4), INV), (dict(hd=7), INV),
    (dict(hd=0), INV), (dict(hd=264), UNSUP),
    (dict(max_pos=0), INV), (dict(cap=0), INV), (dict(qkv=None), INV), (dict(cos=None), INV),
    (dict(pos=None), INV), (dict(kc=None), INV), (dict(qkv=A + 8), INV), (dict(hd=72, qkv=A + 8, M=0), OK),
    (dict(hd=72, qkv=A + 4), INV), (dict(cos=A + 8), INV), (dict(pos=A + 2), INV), (dict(status=A + 1), INV),
    (dict(qw=A + 8), INV), (dict(dt=9), INV), (dict(M=0), OK), (dict(M=0, qkv=None, kc=None), OK),
    (dict(M=0, hd=264), UNSUP), (dict(M=0, Hq=6, Hkv=4), INV),
    # any even hd (element-wise kernel): 2-byte 16-bit pointers, 4-byte tables
    (dict(hd=66, qkv=A + 1), INV), (dict(hd=66, kc=A + 3), INV), (dict(hd=100, cos=A + 2), INV),
    (dict(hd=66, qw=A + 1), INV), (dict(M=0, hd=66), OK), (dict(M=0, hd=2), OK),
])
def test_qkv_host_validation(kw, want):
    assert b_call(**kw) == want


def c_call(M=4, I=256, gu=A, q=A, ss=A, bs=None, act=0, dt=1, qm=0):
    return frt.load().frt_gate_act_fp8(gu, q, ss, bs, M, I, act, dt, qm, None)


@pytest.mark.parametrize("kw,want", [
    (dict(M=-1), INV), (dict(I=0), INV), (dict(I=6), INV), (dict(act=3), INV), (dict(act=-1), INV),
    (dict(gu=None), INV), (dict(gu=A + 8), INV), (dict(q=A + 2), INV), (dict(ss=None), INV),
    (dict(qm=1, bs=None), INV), (dict(qm=1, bs=A + 2), INV), (dict(dt=3), INV), (dict(M=0), OK),
    (dict(M=0, I=4, qm=1, bs=A), OK), (dict(M=0, gu=None, q=None, ss=None), OK), (dict(M=0, I=6), INV),
])
def test_gate_act_host_validation(kw, want):
    assert c_call(**kw) == want


def test_noop_host_validation():
    L = frt.load()
    assert L.frt_noop(0, 32, None) == INV
    assert L.frt_noop(1, 0, None) == INV
    assert L.frt_noop(1, 1025, None) == INV


def test_binding_rejects_host_tensors():
    import torch
    x = torch.zeros(2, 8, dtype=torch.bfloat16)
    with pytest.raises(frt.FrtError):
        frt.frt_residual_rmsnorm_fp8(x, x, x, None, torch.zeros(2, 8, dtype=torch.uint8),
                                     static_scale=torch.ones(1))


def test_pdl_switch():
    prev = frt.frt_get_pdl()
    try:
        frt.frt_set_pdl(False)
        assert frt.frt_get_pdl() is False
        frt.frt_set_pdl(True)
        assert frt.frt_get_pdl() is True
    finally:
        frt.frt_set_pdl(prev)


@pytest.mark.parametrize("args,want", [((A, A, -1, 32), INV), ((A, A, 2, 0), INV), ((A, A, 2, 24), INV),
                                       ((A + 8, A, 2, 32), INV), ((None, A, 2, 32), INV), ((None, None, 0, 32), OK)])
def test_copy_rows_host_validation(args, want):
    assert frt.load().frt_copy_rows(*args, None) == want


def test_wait_polls_setting():
    prev = frt.frt_get_wait_polls()
    assert prev == frt.FRT_DEFAULT_WAIT_POLLS
    try:
        frt.frt_set_wait_polls(0)
        assert frt.frt_get_wait_polls() == 0
        assert frt.load().frt_set_wait_polls(-1) == INV
        assert frt.frt_get_wait_polls() == 0
    finally:
        frt.frt_set_wait_polls(prev)
    assert frt.frt_get_wait_polls() == frt.FRT_DEFAULT_WAIT_POLLS


def ada_call(M=4, D=256, x=A, g=A, r=A, ro=A, sc=A, sh=A, q=A, ss=A, bs=None, rpc=4, dt=1, qm=0):
    return frt.load().frt_gate_residual_adarms_fp8(x, g, r, ro, sc, sh, q, ss, bs, M, D, rpc, 1e-6, dt, qm, None)


@pytest.mark.parametrize("kw,want", [
    (dict(M=-1), INV), (dict(D=12), INV), (dict(rpc=0), INV), (dict(x=None), INV), (dict(g=A + 8), INV),
    (dict(sc=A + 4), INV), (dict(sh=A + 2), INV), (dict(q=A + 4), INV), (dict(ss=None), INV),
    (dict(qm=1), INV), (dict(D=32776), UNSUP), (dict(M=0), OK), (dict(g=None, sc=None, sh=None), None),
])
def test_gate_residual_adarms_host_validation(kw, want):
    if want is None:   # NULL gate / scale / shift are valid: validation passes (no launch here at M = 0)
        assert ada_call(M=0, **kw) == OK
    else:
        assert ada_call(**kw) == want


def b8_call(M=4, Hq=8, Hkv=2, hd=128, kc=A, vc=A, qs=0.125, layout=1, kv=1, scales=A, dt=1):
    return frt.load().frt_qkv_norm_rope_prepq_kvcache(A, None, None, A, A, A, A, kc, vc, None, M, Hq, Hkv, hd, 64,
                                                      64, 1e-6, qs, layout, kv, scales, dt, None)


@pytest.mark.parametrize("kw,want", [
    (dict(layout=2), INV), (dict(layout=-1), INV), (dict(kv=2), INV), (dict(qs=float("inf")), INV),
    (dict(qs=float("nan")), INV), (dict(scales=None), INV), (dict(scales=A + 2), INV), (dict(kc=A + 4), INV),
    (dict(hd=72, vc=A + 2), INV), (dict(kc=None), INV), (dict(hd=264), UNSUP), (dict(M=-1), INV),
    (dict(M=0), OK), (dict(M=0, scales=None), OK), (dict(M=0, layout=3), INV), (dict(M=0, kv=0, scales=None), OK),
    (dict(hd=66, scales=A + 2), INV), (dict(hd=66, scales=None), INV), (dict(M=0, hd=66), OK),
])
def test_qkv_prepq_host_validation(kw, want):
    assert b8_call(**kw) == want


def a4_call(M=4, D=256, x=A, r=A, ro=A, w=None, q=A, sf=A, gs=A, dt=1, lay=0):
    return frt.load().frt_residual_rmsnorm_nvfp4(x, r, ro, w, q, sf, gs, M, D, 1e-6, dt, lay, None)


def c4_call(M=4, I=256, gu=A, q=A, sf=A, gs=A, act=0, dt=1, lay=0):
    return frt.load().frt_gate_act_nvfp4(gu, q, sf, gs, M, I, act, dt, lay, None)


@pytest.mark.parametrize("kw,want", [
    (dict(D=8), INV), (dict(D=24), INV), (dict(lay=2), INV), (dict(gs=None), INV), (dict(gs=A + 2), INV),
    (dict(sf=None), INV), (dict(q=A + 2), INV), (dict(x=A + 8), INV), (dict(D=32784), UNSUP), (dict(M=0), OK),
    (dict(M=0, lay=5), INV), (dict(M=-1), INV), (dict(dt=3), INV),
])
def test_residual_rmsnorm_nvfp4_host_validation(kw, want):
    assert a4_call(**kw) == want


@pytest.mark.parametrize("kw,want", [
    (dict(I=8), INV), (dict(I=20), INV), (dict(lay=-1), INV), (dict(gs=None), INV), (dict(sf=None), INV),
    (dict(q=A + 1), INV), (dict(gu=A + 4), INV), (dict(act=7), INV), (dict(M=0), OK), (dict(M=0, I=20), INV),
])
def test_gate_act_nvfp4_host_validation(kw, want):
    assert c4_call(**kw) == want


def ln_call(M=4, D=256, x=A, r=A, ro=A, w=None, b=None, q=A, ss=A, bs=None, dt=1, qm=0):
    return frt.load().frt_residual_layernorm_fp8(x, r, ro, w, b, q, ss, bs, M, D, 1e-6, dt, qm, None)


@pytest.mark.parametrize("kw,want", [
    (dict(D=12), INV), (dict(b=A + 4), INV), (dict(w=A + 2), INV), (dict(ss=None), INV), (dict(qm=1), INV),
    (dict(q=A + 4), INV), (dict(D=32776), UNSUP), (dict(M=0), OK), (dict(M=0, ss=None, q=None), OK),
])
def test_residual_layernorm_host_validation(kw, want):
    assert ln_call(**kw) == want


def qln_call(M=4, Hq=8, Hkv=2, hd=128, qkv=A, qw=None, qb=None, kw=None, kb=None, dt=1):
    return frt.load().frt_qkv_layernorm_rope_kvcache(qkv, qw, qb, kw, kb, A, A, A, A, A, A, None, M, Hq, Hkv, hd, 64,
                                                     64, 1e-6, dt, None)


@pytest.mark.parametrize("kw,want", [
    (dict(Hq=6, Hkv=4), INV), (dict(hd=264), UNSUP), (dict(qb=A + 8), INV), (dict(kw=A + 2), INV),
    (dict(qkv=A + 8), INV), (dict(qkv=None), INV), (dict(M=0), OK), (dict(M=0, qkv=None), OK), (dict(dt=4), INV),
    (dict(hd=66, qkv=A + 1), INV), (dict(hd=66, qb=A + 1), INV), (dict(M=0, hd=66), OK),
])
def test_qkv_layernorm_host_validation(kw, want):
    assert qln_call(**kw) == want


def chain_call(M=4, D=1024, Hq=8, Hkv=1, hd=128, I=4096, layers=A, n=2, steps=3, res=A, qm=0, act=0, dt=1):
    return frt.load().frt_chain_persistent(layers, n, steps, res, A, A, A, A, None, M, D, Hq, Hkv, hd, I, 64, 64,
                                           1e-6, dt, qm, act, None)


@pytest.mark.parametrize("kw,want", [
    (dict(hd=72), UNSUP), (dict(hd=264), UNSUP), (dict(hd=32), UNSUP), (dict(D=8200), UNSUP), (dict(I=4100), UNSUP),
    (dict(D=12), INV),
    (dict(Hq=6, Hkv=4), INV), (dict(act=5), INV), (dict(qm=3), INV), (dict(layers=None), INV),
    (dict(res=A + 8), INV), (dict(M=0), OK), (dict(steps=0), OK), (dict(n=0, layers=None), OK), (dict(M=-1), INV),
])
def test_chain_persistent_host_validation(kw, want):
    assert chain_call(**kw) == want
