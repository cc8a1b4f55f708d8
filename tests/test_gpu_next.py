"""GPU parity for the NEXT ops through the C ABI against the fp64 oracle.

NEXT-1, gated residual + AdaRMSNorm modulation + FP8 ("FlashRT kernel
fusion", §三, gate_res_adarms_fp8_static): the Pi0.5 decoder shape, every
mode (16-bit type, quantisation, gate present or not, modulation present or
not), condition-row groups, edge widths, in-place and guarded out-of-place
outputs, sums that land on a 16-bit rounding midpoint in fp32, and the
full-size large-M workload on sampled rows."""
import numpy as np
import pytest
import torch

import memory_bound_non_b200 as frt
import oracle
import parity as P
from memory_bound_non_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 256


def guarded(shape, dtype, fill):
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    raw = torch.full((n + GUARD,), fill, dtype=torch.uint8, device=DEV)
    return raw, raw[:n].view(dtype).view(shape)


def assert_guard(raw, n_bytes, fill):
    assert (raw[n_bytes:].cpu().numpy() == fill).all(), "write past the end of an output"


def ada_inputs(M, D, dt, seed, rpc, gated=True, modulated=True, device="cpu"):
    """x ~ N(0, 1), residual ~ N(0, 4), gate ~ N(0, 0.25), scale / shift ~
    N(0, 0.04), the last three one row per condition (ceil(M / rpc) rows)."""
    g = W.generator(seed, device)
    nc = (M + rpc - 1) // rpc
    x = W.normal16((M, D), dt, g)
    r = W.normal16((M, D), dt, g, scale=2.0)
    gate = W.normal16((nc, D), dt, g, scale=0.5) if gated else None
    sc = W.normal16((nc, D), dt, g, scale=0.2) if modulated else None
    sh = W.normal16((nc, D), dt, g, scale=0.2) if modulated else None
    return x, r, gate, sc, sh


def host_bits(t):
    return None if t is None else W.bits16(t.cpu())


def calibrate(x, r, gate, sc, sh, dt, rpc):
    o = oracle.gate_residual_adarms_fp8(x, gate, r, sc, sh, 1e-6, dt, "block128", rpc, want_y=True)
    return P.f32(np.abs(o["y"]).max() / 448.0)


def run_gpu(x, r, gate, sc, sh, quant, scale, rpc, inplace=True):
    M, D = x.shape
    dev = [None if t is None else t.to(DEV) for t in (x, r, gate, sc, sh)]
    xd, rd, gd, scd, shd = dev
    rd = rd.clone()
    if inplace:
        ro_raw, ro = None, rd
    else:
        ro_raw, ro = guarded((M, D), rd.dtype, 0x5A)
    q_raw, q = guarded((M, D), torch.uint8, 0xA5)
    nb = (D + 127) // 128
    bs_raw = bs = ss = None
    if quant == "block128":
        bs_raw, bs = guarded((M, nb), torch.float32, 0xFF)
    else:
        ss = torch.tensor([scale], dtype=torch.float32, device=DEV)
    frt.frt_gate_residual_adarms_fp8(xd, gd, rd, ro, scd, shd, q, static_scale=ss, block_scales=bs,
                                     rows_per_cond=rpc, eps=1e-6, quant=quant)
    torch.cuda.synchronize()
    assert_guard(q_raw, M * D, 0xA5)
    if bs_raw is not None:
        assert_guard(bs_raw, M * nb * 4, 0xFF)
    if ro_raw is not None:
        assert_guard(ro_raw, M * D * 2, 0x5A)
    return ro, q, bs


def check(M, D, dt, quant, rpc, gated=True, modulated=True, seed=11, inplace=True):
    x, r, gate, sc, sh = ada_inputs(M, D, dt, seed, rpc, gated, modulated)
    hx, hr, hg, hsc, hsh = (host_bits(t) for t in (x, r, gate, sc, sh))
    scale = calibrate(hx, hr, hg, hsc, hsh, dt, rpc) if quant == "static" else None
    ro, q, bs = run_gpu(x, r, gate, sc, sh, quant, scale, rpc, inplace=inplace)
    o = oracle.gate_residual_adarms_fp8(hx, hg, hr, hsc, hsh, 1e-6, dt, quant, rpc, static_scale=scale)
    np.testing.assert_array_equal(W.bits16(ro.cpu()), o["residual_out"])
    P.assert_fp8_codes(q.cpu().numpy(), o["out_fp8"], what="adarms codes")
    if quant == "block128":
        P.assert_scales_close(bs.cpu().numpy(), o["block_scales"])


@pytest.mark.parametrize("quant", ["static", "block128"])
def test_adarms_pi05_decoder_shape(quant):
    # Pi0.5 action expert: 10 action tokens, width 1024, one condition (the flow time step)
    check(10, 1024, "bf16", quant, rpc=10)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("quant", ["static", "block128"])
@pytest.mark.parametrize("gated,modulated", [(True, True), (True, False), (False, True), (False, False)])
def test_adarms_modes_out_of_place(dt, quant, gated, modulated):
    check(33, 1280, dt, quant, rpc=11, gated=gated, modulated=modulated, inplace=False)


@pytest.mark.parametrize("M,D,quant,rpc", [
    (1, 8, "static", 1), (3, 136, "block128", 2), (5, 1032, "block128", 1), (7, 2056, "static", 3),
    (4, 8192, "block128", 4), (3, 16384, "static", 1), (2, 16392, "block128", 1), (2, 32768, "block128", 2),
])
def test_adarms_edge_widths(M, D, quant, rpc):
    check(M, D, "bf16", quant, rpc=rpc, seed=M * 7 + D)


def test_adarms_fp16_wide_and_in_place():
    check(6, 4096, "f16", "block128", rpc=1, seed=21, inplace=True)


def _midpoint_triples(dt, n, rng):
    """r, g, x bit patterns where |r| is far below |g x| half of the time, so
    that r's bits fall below the fp32 ulp of the sum and, when g x sits on a
    16-bit midpoint, the sign of r alone decides the rounding."""
    sgn = lambda: rng.integers(0, 2, n) << 15
    coin = lambda: rng.integers(0, 2, n) == 1
    if dt == "bf16":
        r = np.where(coin(), rng.integers(0x3000, 0x3800, n), rng.integers(0x3800, 0x4800, n)) | sgn()
        g = rng.integers(0x3C00, 0x3F80, n)
        x = rng.integers(0x3F80, 0x4100, n) | sgn()
    else:
        r = np.where(coin(), rng.integers(0x0001, 0x0040, n), rng.integers(0x0400, 0x5000, n)) | sgn()
        g = np.where(coin(), rng.choice([0x3E00, 0x3D00, 0x3F00, 0x3A00, 0x3500], n), rng.integers(0x3000, 0x3C00, n))
        x = rng.integers(0x3C00, 0x4800, n) | sgn()
    return tuple(a.astype(np.uint16) for a in (r, g, x))


@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_adarms_sums_on_a_16bit_midpoint(dt):
    """Rows holding triples whose plain fp32 sum r + g x lies on a 16-bit
    rounding midpoint while the exact sum does not (rounding the fp32 sum again
    would give the wrong h): h must still be the oracle's, bit for bit."""
    rng = np.random.default_rng(7)
    D = 1024
    r, g, x = _midpoint_triples(dt, 1 << 18, rng)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float16
    tr, tg, tx = (torch.from_numpy(a.view(np.int16)).view(tdt) for a in (r, g, x))
    naive = W.bits16((tr.float() + tg.float() * tx.float()).to(tdt))
    o = oracle.gate_residual_adarms_fp8(x.reshape(-1, D), g.reshape(-1, D), r.reshape(-1, D), None, None, 1e-6,
                                        dt, "block128", 1)
    hard = naive.reshape(-1, D) != o["residual_out"]
    assert hard.sum() > 20, "the inputs do not exercise the midpoint case"
    rows = np.flatnonzero(hard.any(axis=1))[:64]
    xs, gs, rs = (torch.from_numpy(a.reshape(-1, D)[rows].copy().view(np.int16)).view(tdt) for a in (x, g, r))
    ro, q, bs = run_gpu(xs, rs, gs, None, None, "block128", None, 1)
    np.testing.assert_array_equal(W.bits16(ro.cpu()), o["residual_out"][rows])
    om = oracle.gate_residual_adarms_fp8(W.bits16(xs), W.bits16(gs), W.bits16(rs), None, None, 1e-6, dt,
                                         "block128", 1)
    P.assert_fp8_codes(q.cpu().numpy(), om["out_fp8"], what="midpoint rows codes")


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("gated", [True, False])
def test_adarms_subnormal_and_signed_zero_sums(dt, gated):
    """Subnormal residuals and products, exact cancellations (+0) and -0 + -0
    (-0): h is still the oracle's value bit for bit."""
    rng = np.random.default_rng(9)
    M, D = 4, 1024
    n = M * D
    sub_hi = 0x0080 if dt == "bf16" else 0x0400            # exponent field zero
    one = 0x3F80 if dt == "bf16" else 0x3C00
    sgn = lambda: (rng.integers(0, 2, n) << 15).astype(np.uint16)
    r = (rng.integers(1, sub_hi, n).astype(np.uint16) | sgn())
    x = (rng.integers(1, sub_hi, n).astype(np.uint16) | sgn())
    lo_g, hi_g = (0x3E80, 0x4000) if dt == "bf16" else (0x3400, 0x4000)   # gate in [0.25, 2)
    g = rng.integers(lo_g, hi_g, n).astype(np.uint16)
    k = np.arange(n)
    cancel, negzero = k % 16 == 3, k % 16 == 7
    g[cancel] = one
    x[cancel] = r[cancel] ^ 0x8000                          # 1 * (-r) + r = +0
    r[negzero] = 0x8000
    x[negzero] = 0x8000                                     # g * (-0) + (-0) = -0
    gate = g.reshape(M, D) if gated else None
    if not gated:
        x[cancel] = r[cancel] ^ 0x8000
    tdt = torch.bfloat16 if dt == "bf16" else torch.float16
    to_t = lambda a: torch.from_numpy(a.reshape(M, D).copy().view(np.int16)).view(tdt)
    o = oracle.gate_residual_adarms_fp8(x.reshape(M, D), None if gate is None else gate.reshape(M, D),
                                        r.reshape(M, D), None, None, 1e-6, dt, "block128", 1)
    want = o["residual_out"]
    assert (want.ravel()[cancel] == 0x0000).all() and (want.ravel()[negzero] == 0x8000).all()
    assert ((want & 0x7FFF) < sub_hi).sum() > n // 4, "few subnormal results"
    ro, q, bs = run_gpu(to_t(x), to_t(r), None if gate is None else to_t(g), None, None, "block128", None, 1)
    np.testing.assert_array_equal(W.bits16(ro.cpu()), want)
    P.assert_fp8_codes(q.cpu().numpy(), o["out_fp8"], what="subnormal rows codes")


def test_adarms_without_gate_or_modulation_equals_op_a():
    """No gate, no modulation: the op is op (a) with `_noweight`, bit for bit."""
    x, r, _, _, _ = ada_inputs(64, 2048, "bf16", 31, 64, gated=False, modulated=False)
    xd, rd = x.to(DEV), r.to(DEV)
    r1, r2 = rd.clone(), rd.clone()
    q1 = torch.empty((64, 2048), dtype=torch.uint8, device=DEV)
    q2 = torch.empty_like(q1)
    ss = torch.tensor([0.01], dtype=torch.float32, device=DEV)
    frt.frt_gate_residual_adarms_fp8(xd, None, r1, r1, None, None, q1, static_scale=ss)
    frt.frt_residual_rmsnorm_fp8(xd, r2, r2, None, q2, static_scale=ss)
    torch.cuda.synchronize()
    assert torch.equal(r1, r2)
    assert torch.equal(q1, q2)


@pytest.mark.parametrize("M", [16384, 65536])
def test_adarms_large_m_sampled(M):
    """Full-size launch (D = 4096, one condition per 1024 rows), sampled rows
    against the oracle (each sampled row with its own condition row)."""
    D, rpc, dt = 4096, 1024, "bf16"
    x, r, gate, sc, sh = ada_inputs(M, D, dt, 41, rpc, device=DEV)
    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([rng.choice(M, 256, replace=False), [0, M - 1]]))
    ti = torch.as_tensor(rows, device=DEV)
    ci = torch.as_tensor(rows // rpc, device=DEV)
    hx, hr = W.bits16(x[ti].cpu()), W.bits16(r[ti].cpu())
    hg, hsc, hsh = (W.bits16(t[ci].cpu()) for t in (gate, sc, sh))
    scale = calibrate(hx, hr, hg, hsc, hsh, dt, 1)
    q = torch.empty((M, D), dtype=torch.uint8, device=DEV)
    ss = torch.tensor([scale], dtype=torch.float32, device=DEV)
    frt.frt_gate_residual_adarms_fp8(x, gate, r, r, sc, sh, q, static_scale=ss, rows_per_cond=rpc)
    torch.cuda.synchronize()
    o = oracle.gate_residual_adarms_fp8(hx, hg, hr, hsc, hsh, 1e-6, dt, "static", 1, static_scale=scale)
    np.testing.assert_array_equal(W.bits16(r[ti].cpu()), o["residual_out"])
    P.assert_fp8_codes(q[ti].cpu().numpy(), o["out_fp8"], what="large-M adarms codes")


def test_adarms_deterministic():
    x, r, gate, sc, sh = ada_inputs(40, 3072, "bf16", 51, 8, device=DEV)
    outs = []
    for _ in range(2):
        rr = r.clone()
        q = torch.empty((40, 3072), dtype=torch.uint8, device=DEV)
        bs = torch.empty((40, 24), dtype=torch.float32, device=DEV)
        frt.frt_gate_residual_adarms_fp8(x, gate, rr, rr, sc, sh, q, block_scales=bs, rows_per_cond=8,
                                         quant="block128")
        outs.append((rr, q, bs))
    torch.cuda.synchronize()
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


# ================================================================== NEXT-2 ===
# Op (b) with the attention's Q preparation (softmax scale, head-major Q) and an
# optional e4m3 KV cache: Q staging within the 16-bit tolerance, K codes within
# one step on <= 0.1 %, V codes exact (a correctly rounded quotient of exact
# 16-bit values), untouched cache slots bit for bit, on the register kernel
# (small batches) and the bulk-copy kernel (M >= 592).

def softmax_scale(hd):
    return float(np.float32(1.0 / np.sqrt(hd)))


def run_prepq_gpu(wl, inp, q_layout, kv, q_scale, kv_scales=(0.02, 0.015), positions=None):
    L = inp.layers[0]
    pos = (inp.positions if positions is None else positions).to(DEV)
    shape = (wl.Hq, wl.M, wl.hd) if q_layout == "head" else (wl.M, wl.Hq, wl.hd)
    q_raw, q_out = guarded(shape, L.qkv.dtype, 0x3C)
    if kv == "e4m3":
        kc = torch.full((wl.capacity, wl.Hkv, wl.hd), 0x7E, dtype=torch.uint8, device=DEV)
        vc = torch.full_like(kc, 0x7E)
        sc = torch.tensor(kv_scales, dtype=torch.float32, device=DEV)
    else:
        kc, vc = L.k_cache.to(DEV).clone(), L.v_cache.to(DEV).clone()
        sc = None
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    dev = lambda t: None if t is None else t.to(DEV)
    frt.frt_qkv_norm_rope_prepq_kvcache(dev(L.qkv), dev(L.q_norm_w), dev(L.k_norm_w), inp.cos.to(DEV),
                                        inp.sin.to(DEV), pos, q_out, kc, vc, wl.Hq, wl.Hkv, wl.hd, q_scale=q_scale,
                                        q_layout=q_layout, kv=kv, kv_scales=sc, status=status, eps=wl.eps)
    torch.cuda.synchronize()
    assert_guard(q_raw, q_out.numel() * 2, 0x3C)
    return q_out, kc, vc, int(status.item())


@pytest.mark.parametrize("q_layout", ["token", "head"])
def test_prepq_bulk_copy_wait_give_up(q_layout):
    """Levels 1-2 of the bulk-copy kernel with its barrier wait forced to give
    up (0 polls): status bit 1 and no output written (Q keeps its fill, the
    e4m3 caches their 0x7E sentinel)."""
    wl = W.get("large_m_M4096", M=640, capacity=2048)
    inp = W.make_inputs(wl, n_layers=1, with_caches=False)
    frt.frt_set_wait_polls(0)
    try:
        q_out, kc, vc, status = run_prepq_gpu(wl, inp, q_layout, "e4m3", softmax_scale(wl.hd))
    finally:
        frt.frt_set_wait_polls(frt.FRT_DEFAULT_WAIT_POLLS)
    assert status == 2
    assert (P.np16(q_out) == 0x3C3C).all()
    assert bool((kc == 0x7E).all()) and bool((vc == 0x7E).all())


def oracle_prepq(wl, inp, q_layout, kv, q_scale, kv_scales=(0.02, 0.015), rows=None, positions=None):
    L = inp.layers[0]
    pos_t = inp.positions if positions is None else positions
    pos = (pos_t.cpu() if rows is None else pos_t.cpu()[torch.as_tensor(rows)]).numpy()
    qkv = W.bits16(L.qkv.cpu() if rows is None else L.qkv[torch.as_tensor(rows, device=L.qkv.device)].cpu())
    hb = lambda t: None if t is None else W.bits16(t.cpu())
    cap, slots, kinit, vinit = wl.capacity, None, None, None
    if rows is not None:
        cap, slots = len(rows), np.arange(len(rows))
    elif kv == "16":
        vinit = W.bits16(L.v_cache)
    return oracle.qkv_norm_rope_prepq_kvcache(
        qkv, hb(L.q_norm_w), hb(L.k_norm_w), inp.cos.cpu().numpy(), inp.sin.cpu().numpy(), pos, wl.Hq, wl.Hkv,
        wl.hd, cap, wl.eps, wl.dt, q_scale=q_scale, q_layout=q_layout, kv=kv, k_scale=kv_scales[0],
        v_scale=kv_scales[1], v_cache=vinit, slots=slots)


def check_prepq(wl, inp, q_layout, kv, q_scale):
    q_out, kc, vc, status = run_prepq_gpu(wl, inp, q_layout, kv, q_scale)
    o = oracle_prepq(wl, inp, q_layout, kv, q_scale)
    assert status == o["status"] == 0
    P.assert_16bit_close(P.decode16(q_out), o["q_out"], what="Q staging", dt=wl.dt)
    pos = np.unique(inp.positions.cpu().numpy())
    untouched = np.setdiff1d(np.arange(wl.capacity), pos)
    if kv == "e4m3":
        P.assert_fp8_codes(kc.cpu().numpy()[pos], o["k_cache"][pos], what="K cache codes")
        P.assert_fp8_codes(vc.cpu().numpy()[pos], o["v_cache"][pos], max_frac=0.0, what="V cache codes")
        assert (kc.cpu().numpy()[untouched] == 0x7E).all() and (vc.cpu().numpy()[untouched] == 0x7E).all()
    else:
        P.assert_16bit_close(P.decode16(kc)[pos], o["k_cache"][pos], what="K cache", dt=wl.dt)
        np.testing.assert_array_equal(P.np16(vc)[pos], o["v_cache"][pos])
        np.testing.assert_array_equal(P.np16(kc)[untouched], W.bits16(inp.layers[0].k_cache)[untouched])


PREPQ_CASES = [("tiny", {}), ("pi05", {}), ("vla_denoise", {}), ("qwen3_prefill_S512", {}), ("vit", {"M": 40}),
               ("tiny", {"M": 3, "hd": 24, "Hq": 4, "Hkv": 4}), ("tiny", {"M": 2, "hd": 256, "dt": "bf16"}),
               ("large_m_M4096", {"M": 640, "capacity": 2048}),
               ("large_m_M4096", {"M": 700, "hd": 72, "Hq": 16, "Hkv": 16, "capacity": 2048}),
               ("tiny", {"M": 5, "hd": 66}), ("vit", {"M": 9, "hd": 100, "qk_norm": True})]


@pytest.mark.parametrize("name,ov", PREPQ_CASES, ids=["%s%s" % (n, "".join("-%s%s" % kv for kv in o.items()))
                                                       for n, o in PREPQ_CASES])
@pytest.mark.parametrize("q_layout,kv", [("token", "e4m3"), ("head", "16"), ("head", "e4m3")])
def test_prepq_parity(name, ov, q_layout, kv):
    wl = W.get(name, **ov)
    check_prepq(wl, W.make_inputs(wl, n_layers=1, with_caches=True), q_layout, kv, softmax_scale(wl.hd))


@pytest.mark.parametrize("M", [16, 600])
def test_prepq_defaults_equal_op_b_bitwise(M):
    """Scale 1, token-major, 16-bit caches: the same bits as op (b), on the
    register kernel and on the bulk-copy kernel."""
    wl = W.get("large_m_M4096", M=M, capacity=1024)
    inp = W.make_inputs(wl, n_layers=1, with_caches=True)
    q1, k1, v1, _ = run_prepq_gpu(wl, inp, "token", "16", 1.0)
    L = inp.layers[0]
    kc, vc = L.k_cache.to(DEV).clone(), L.v_cache.to(DEV).clone()
    q2 = torch.empty_like(q1)
    frt.frt_qkv_norm_rope_kvcache(L.qkv.to(DEV), L.q_norm_w.to(DEV), L.k_norm_w.to(DEV), inp.cos.to(DEV),
                                  inp.sin.to(DEV), inp.positions.to(DEV), q2, kc, vc, wl.Hq, wl.Hkv, wl.hd,
                                  eps=wl.eps)
    torch.cuda.synchronize()
    assert torch.equal(q1, q2) and torch.equal(k1, kc) and torch.equal(v1, vc)


def test_prepq_bad_positions():
    for M in (6, 640):
        wl = W.get("large_m_M4096", M=M, capacity=2048)
        inp = W.make_inputs(wl, n_layers=1, with_caches=True)
        pos = inp.positions.clone()
        bad = torch.tensor([1, M - 2])
        pos[bad] = torch.tensor([-3, 2048], dtype=torch.int32)
        q_out, kc, vc, status = run_prepq_gpu(wl, inp, "head", "e4m3", 0.125, positions=pos)
        o = oracle_prepq(wl, inp, "head", "e4m3", 0.125, positions=pos)
        assert status == 1 and o["status"] == 1
        good = np.setdiff1d(np.arange(M), bad.numpy())
        P.assert_16bit_close(P.decode16(q_out)[:, good], o["q_out"][:, good], what="Q staging", dt=wl.dt)
        assert (P.np16(q_out)[:, bad.numpy()] == 0x3C3C).all()
        np.testing.assert_array_equal(vc.cpu().numpy(), o["v_cache"])


@pytest.mark.parametrize("M", [16384, 65536])
def test_prepq_large_m_sampled(M):
    wl = W.get("large_m_M%d" % M)
    inp = W.make_inputs(wl, n_layers=1, with_caches=False, device=DEV)
    q_out, kc, vc, status = run_prepq_gpu(wl, inp, "head", "e4m3", softmax_scale(wl.hd))
    assert status == 0
    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([rng.choice(M, 256, replace=False), [0, M - 1]]))
    o = oracle_prepq(wl, inp, "head", "e4m3", softmax_scale(wl.hd), rows=rows)
    ti = torch.as_tensor(rows, device=DEV)
    P.assert_16bit_close(P.decode16(q_out[:, ti]), o["q_out"], what="Q staging", dt=wl.dt)
    slots = inp.positions[ti].long()
    P.assert_fp8_codes(kc[slots].cpu().numpy(), o["k_cache"], what="K cache codes")
    P.assert_fp8_codes(vc[slots].cpu().numpy(), o["v_cache"], max_frac=0.0, what="V cache codes")
    mask = torch.ones(wl.capacity, dtype=torch.bool, device=DEV)
    mask[inp.positions.long()] = False
    assert bool((kc[mask] == 0x7E).all()) and bool((vc[mask] == 0x7E).all())


# ================================================================== NEXT-3 ===
# NVFP4 outputs of ops (a) and (c): e2m1 codes in 16-element blocks with e4m3
# scale factors and a global fp32 scale, scale factors row-major or in the
# 128x4-swizzled layout of block-scaled GEMMs.

def unswizzle(swz, rows, cols):
    """Row-major [rows, cols] view of a 128x4-swizzled scale-factor array,
    gathered through the oracle's offsets."""
    idx = np.array([[oracle.sf_swizzle_offset(r, c, cols) for c in range(cols)] for r in range(rows)])
    return np.asarray(swz)[idx]


def check_nvfp4(q, sf, o_codes, o_sf, sf_layout, what):
    """GPU NVFP4 output against the oracle (parity.assert_nvfp4); the
    swizzled layout is read back through the oracle's offsets.  Prints the
    mismatch counts."""
    rows, nsf = o_sf.shape
    got_sf = sf.cpu().numpy()
    if sf_layout == "rows":
        got_sf = got_sf.reshape(rows, nsf)
    else:
        pad = oracle.sf_swizzle(np.ones((rows, nsf), dtype=np.uint8)) == 0
        assert (got_sf[pad] == 0).all(), what + ": a padding byte of the swizzled layout was written"
        got_sf = unswizzle(got_sf, rows, nsf)
    n_sf, n = P.assert_nvfp4(q.cpu().numpy(), got_sf, o_codes, o_sf, what=what)
    print("%s: %d of %d scale factors, %d of %d codes one step off" % (what, n_sf, o_sf.size, n,
                                                                       2 * np.asarray(o_codes).size))
    return n_sf, n


def global_scale_for(vals):
    """gs so the largest block scale lands near the top of e4m3: amax / (6 * 448)."""
    return float(np.float32(np.abs(vals).max() / (6.0 * 448.0)))


def run_a_nvfp4(x, r, w, gs, sf_layout="rows", inplace=True):
    M, D = x.shape
    xd, rd = x.to(DEV), r.to(DEV).clone()
    ro = rd if inplace else torch.empty_like(rd)
    q_raw, q = guarded((M, D // 2), torch.uint8, 0xA5)
    nsf = frt.nvfp4_sf_bytes(M, D, sf_layout)
    sf_raw, sf = guarded((nsf,), torch.uint8, 0)
    gsd = torch.tensor([gs], dtype=torch.float32, device=DEV)
    frt.frt_residual_rmsnorm_nvfp4(xd, rd, ro, None if w is None else w.to(DEV), q, sf, gsd, sf_layout=sf_layout)
    torch.cuda.synchronize()
    assert_guard(q_raw, M * D // 2, 0xA5)
    assert_guard(sf_raw, nsf, 0)
    return ro, q, sf


A4_CASES = [("pi05", {}), ("vla_denoise", {}), ("vit", {}), ("tiny", {"M": 3, "D": 16}),
            ("tiny", {"M": 5, "D": 1040}), ("large_m_M4096", {"M": 300}), ("vit", {"M": 2, "D": 32768}),
            ("tiny", {"M": 130, "D": 2048, "dt": "bf16"})]


@pytest.mark.parametrize("name,ov", A4_CASES, ids=["%s%s" % (n, "".join("-%s%s" % kv for kv in o.items()))
                                                   for n, o in A4_CASES])
@pytest.mark.parametrize("sf_layout", ["rows", "swizzled"])
def test_residual_rmsnorm_nvfp4_parity(name, ov, sf_layout):
    wl = W.get(name, **ov)
    inp = W.make_inputs(wl, n_layers=1, with_caches=False)
    L = inp.layers[0]
    x, r = W.bits16(L.x_attn), W.bits16(inp.residual)
    w = None if L.w_attn is None else W.bits16(L.w_attn)
    y = oracle.residual_rmsnorm_fp8(x, r, w, wl.eps, wl.dt, "block128", want_y=True)["y"]
    gs = global_scale_for(y)
    ro, q, sf = run_a_nvfp4(L.x_attn, inp.residual, L.w_attn, gs, sf_layout)
    o = oracle.residual_rmsnorm_nvfp4(x, r, w, wl.eps, wl.dt, gs)
    np.testing.assert_array_equal(W.bits16(ro.cpu()), o["residual_out"])
    check_nvfp4(q, sf, o["out_fp4"], o["sf"], sf_layout, "op a nvfp4")


@pytest.mark.parametrize("gs", [1e-6, 1e4])
def test_residual_rmsnorm_nvfp4_scale_saturation_and_underflow(gs):
    """A tiny global scale saturates every block scale at 448 (codes saturate
    at 6); a huge one rounds small blocks' scales to 0 (all-zero codes)."""
    wl = W.get("vla_denoise", M=9)
    inp = W.make_inputs(wl, n_layers=1, with_caches=False)
    L = inp.layers[0]
    x, r, w = W.bits16(L.x_attn), W.bits16(inp.residual), W.bits16(L.w_attn)
    ro, q, sf = run_a_nvfp4(L.x_attn, inp.residual, L.w_attn, gs)
    o = oracle.residual_rmsnorm_nvfp4(x, r, w, wl.eps, wl.dt, gs)
    check_nvfp4(q, sf, o["out_fp4"], o["sf"], "rows", "op a nvfp4")
    assert (o["sf"] == 0x7E).all() if gs < 1 else (o["sf"] == 0).all()


def run_c_nvfp4(gu, gs, act, sf_layout="rows"):
    M, two_i = gu.shape
    I = two_i // 2
    q_raw, q = guarded((M, I // 2), torch.uint8, 0xA5)
    nsf = frt.nvfp4_sf_bytes(M, I, sf_layout)
    sf_raw, sf = guarded((nsf,), torch.uint8, 0)
    gsd = torch.tensor([gs], dtype=torch.float32, device=DEV)
    frt.frt_gate_act_nvfp4(gu.to(DEV), q, sf, gsd, act=act, sf_layout=sf_layout)
    torch.cuda.synchronize()
    assert_guard(q_raw, M * I // 2, 0xA5)
    assert_guard(sf_raw, nsf, 0)
    return q, sf


C4_CASES = [("pi05", {}), ("vla_denoise", {}), ("vit", {}), ("tiny", {"M": 1, "I": 16}),
            ("tiny", {"M": 3, "I": 48, "act": "relu2"}), ("large_m_M4096", {"M": 160})]


@pytest.mark.parametrize("name,ov", C4_CASES, ids=["%s%s" % (n, "".join("-%s%s" % kv for kv in o.items()))
                                                   for n, o in C4_CASES])
@pytest.mark.parametrize("sf_layout", ["rows", "swizzled"])
def test_gate_act_nvfp4_parity(name, ov, sf_layout):
    wl = W.get(name, **ov)
    gu = W.make_inputs(wl, n_layers=1, with_caches=False).layers[0].gate_up
    hb = W.bits16(gu)
    a = oracle.gate_act_fp8(hb, wl.act, wl.dt, "block128", want_a=True)["a"]
    gs = global_scale_for(a)
    q, sf = run_c_nvfp4(gu, gs, wl.act, sf_layout)
    o = oracle.gate_act_nvfp4(hb, wl.act, wl.dt, gs)
    check_nvfp4(q, sf, o["out_fp4"], o["sf"], sf_layout, "op c nvfp4")


def test_nvfp4_large_m_sampled():
    """Full-size launches (65536 x 4096 norm, 16384 x 16384 gate), sampled rows
    against the oracle."""
    M, D = 65536, 4096
    wl = W.get("large_m_M65536")
    inp = W.make_inputs(wl, n_layers=1, with_caches=False, device=DEV)
    L = inp.layers[0]
    rows = np.unique(np.concatenate([np.random.default_rng(3).choice(M, 192, replace=False), [0, M - 1]]))
    ti = torch.as_tensor(rows, device=DEV)
    x, r, w = W.bits16(L.x_attn[ti].cpu()), W.bits16(inp.residual[ti].cpu()), W.bits16(L.w_attn.cpu())
    gs = global_scale_for(oracle.residual_rmsnorm_fp8(x, r, w, wl.eps, wl.dt, "block128", want_y=True)["y"])
    q = torch.empty((M, D // 2), dtype=torch.uint8, device=DEV)
    sf = torch.empty((M * D // 16,), dtype=torch.uint8, device=DEV)
    rr = inp.residual.clone()
    frt.frt_residual_rmsnorm_nvfp4(L.x_attn, rr, rr, L.w_attn, q, sf,
                                   torch.tensor([gs], dtype=torch.float32, device=DEV))
    torch.cuda.synchronize()
    o = oracle.residual_rmsnorm_nvfp4(x, r, w, wl.eps, wl.dt, gs)
    np.testing.assert_array_equal(W.bits16(rr[ti].cpu()), o["residual_out"])
    check_nvfp4(q[ti], sf.view(M, D // 16)[ti], o["out_fp4"], o["sf"], "rows", "large-M op a nvfp4")
    # op c on the first 16384 rows of the large-M gate/up buffer
    Mc, I = 16384, wl.I
    gu = L.gate_up[:Mc]
    rows = rows[rows < Mc]
    tc = torch.as_tensor(rows, device=DEV)
    hb = W.bits16(gu[tc].cpu())
    gs = global_scale_for(oracle.gate_act_fp8(hb, wl.act, wl.dt, "block128", want_a=True)["a"])
    q = torch.empty((Mc, I // 2), dtype=torch.uint8, device=DEV)
    sf = torch.empty((Mc * I // 16,), dtype=torch.uint8, device=DEV)
    frt.frt_gate_act_nvfp4(gu, q, sf, torch.tensor([gs], dtype=torch.float32, device=DEV), act=wl.act)
    torch.cuda.synchronize()
    o = oracle.gate_act_nvfp4(hb, wl.act, wl.dt, gs)
    check_nvfp4(q[tc], sf.view(Mc, I // 16)[tc], o["out_fp4"], o["sf"], "rows", "large-M op c nvfp4")


# ================================================================== NEXT-4 ===
# LayerNorm variants: residual add + LayerNorm producers (FP8 and NVFP4) and the
# per-head LayerNorm(Q/K) + RoPE kernel.

def ln_inputs(M, D, dt, seed, weighted=True, biased=True):
    g = W.generator(seed)
    x = W.normal16((M, D), dt, g)
    r = W.normal16((M, D), dt, g, scale=2.0)
    w = W.norm_weight(D, dt, g) if weighted else None
    b = W.normal16((D,), dt, g, scale=0.2) if biased else None
    return x, r, w, b


LN_CASES = [(10, 1024, "bf16", "static", True, True), (41, 2048, "bf16", "block128", True, False),
            (7, 1040, "f16", "block128", False, True), (1176, 1152, "bf16", "static", True, True),
            (3, 16, "f16", "nvfp4", True, True), (33, 1280, "bf16", "nvfp4", False, False),
            (5, 8192, "bf16", "nvfp4", True, True), (2, 32768, "bf16", "block128", True, True)]


@pytest.mark.parametrize("M,D,dt,quant,weighted,biased", LN_CASES)
def test_residual_layernorm_parity(M, D, dt, quant, weighted, biased):
    x, r, w, b = ln_inputs(M, D, dt, M + D, weighted, biased)
    hx, hr = W.bits16(x), W.bits16(r)
    hw, hb = (None if t is None else W.bits16(t) for t in (w, b))
    y = oracle.residual_layernorm(hx, hr, hw, hb, 1e-6, dt, "block128", want_y=True)["y"]
    xd, rd = x.to(DEV), r.to(DEV).clone()
    wd, bd = (None if t is None else t.to(DEV) for t in (w, b))
    if quant == "nvfp4":
        gs = global_scale_for(y)
        q = torch.empty((M, D // 2), dtype=torch.uint8, device=DEV)
        sf = torch.empty((M * D // 16,), dtype=torch.uint8, device=DEV)
        frt.frt_residual_layernorm_nvfp4(xd, rd, rd, wd, bd, q, sf, torch.tensor([gs], device=DEV))
        torch.cuda.synchronize()
        o = oracle.residual_layernorm(hx, hr, hw, hb, 1e-6, dt, "nvfp4", global_scale=gs)
        check_nvfp4(q, sf, o["out"], o["sf"], "rows", "LN nvfp4")
    else:
        q_raw, q = guarded((M, D), torch.uint8, 0xA5)
        ss = bs = None
        scale = None
        if quant == "static":
            scale = P.f32(np.abs(y).max() / 448.0)
            ss = torch.tensor([scale], dtype=torch.float32, device=DEV)
        else:
            bs = torch.full((M, (D + 127) // 128), float("nan"), dtype=torch.float32, device=DEV)
        frt.frt_residual_layernorm_fp8(xd, rd, rd, wd, bd, q, static_scale=ss, block_scales=bs, quant=quant)
        torch.cuda.synchronize()
        assert_guard(q_raw, M * D, 0xA5)
        o = oracle.residual_layernorm(hx, hr, hw, hb, 1e-6, dt, quant, static_scale=scale)
        P.assert_fp8_codes(q.cpu().numpy(), o["out"], what="LN codes")
        if quant == "block128":
            P.assert_scales_close(bs.cpu().numpy(), o["block_scales"])
    np.testing.assert_array_equal(W.bits16(rd.cpu()), o["residual_out"])


def test_residual_layernorm_large_m_sampled():
    M, D, dt = 65536, 4096, "bf16"
    g = W.generator(71, DEV)
    x, r = W.normal16((M, D), dt, g), W.normal16((M, D), dt, g, scale=2.0)
    w, b = W.norm_weight(D, dt, g), W.normal16((D,), dt, g, scale=0.2)
    rows = np.unique(np.concatenate([np.random.default_rng(71).choice(M, 192, replace=False), [0, M - 1]]))
    ti = torch.as_tensor(rows, device=DEV)
    hx, hr, hw, hb = W.bits16(x[ti].cpu()), W.bits16(r[ti].cpu()), W.bits16(w.cpu()), W.bits16(b.cpu())
    y = oracle.residual_layernorm(hx, hr, hw, hb, 1e-6, dt, "block128", want_y=True)["y"]
    scale = P.f32(np.abs(y).max() / 448.0)
    q = torch.empty((M, D), dtype=torch.uint8, device=DEV)
    frt.frt_residual_layernorm_fp8(x, r, r, w, b, q, static_scale=torch.tensor([scale], device=DEV))
    torch.cuda.synchronize()
    o = oracle.residual_layernorm(hx, hr, hw, hb, 1e-6, dt, "static", static_scale=scale)
    np.testing.assert_array_equal(W.bits16(r[ti].cpu()), o["residual_out"])
    P.assert_fp8_codes(q[ti].cpu().numpy(), o["out"], what="large-M LN codes")


def test_qkv_layernorm_bulk_copy_wait_give_up():
    """The LayerNorm level of the bulk-copy kernel with its wait forced to
    give up: status bit 1, nothing written."""
    M, Hq, Hkv, hd, dt = 700, 32, 8, 128, "bf16"
    g = W.generator(5)
    qkv = W.normal16((M, (Hq + 2 * Hkv) * hd), dt, g)
    cos, sin = W.rope_tables(1024, hd, 1e4)
    pos = torch.randperm(1024, generator=g)[:M].to(torch.int32)
    kc = torch.full((1024, Hkv, hd), 0x7E7E, dtype=torch.int16).view(W.DTYPES[dt]).to(DEV)
    vc = kc.clone()
    q_raw, q_out = guarded((M, Hq, hd), qkv.dtype, 0x3C)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    frt.frt_set_wait_polls(0)
    try:
        frt.frt_qkv_layernorm_rope_kvcache(qkv.to(DEV), None, None, None, None, cos.to(DEV), sin.to(DEV),
                                           pos.to(DEV), q_out, kc, vc, Hq, Hkv, hd, status=status)
        torch.cuda.synchronize()
    finally:
        frt.frt_set_wait_polls(frt.FRT_DEFAULT_WAIT_POLLS)
    assert int(status.item()) == 2
    assert (P.np16(q_out) == 0x3C3C).all()
    assert (P.np16(kc) == 0x7E7E).all() and (P.np16(vc) == 0x7E7E).all()


QLN_CASES = [dict(M=10, Hq=8, Hkv=1, hd=256, dt="bf16"), dict(M=41, Hq=16, Hkv=8, hd=128, dt="bf16"),
             dict(M=6, Hq=32, Hkv=32, hd=128, dt="bf16"),          # Chameleon-like: 96 heads over two CTAs
             dict(M=7, Hq=16, Hkv=16, hd=72, dt="f16"), dict(M=700, Hq=32, Hkv=8, hd=128, dt="bf16"),
             dict(M=5, Hq=4, Hkv=2, hd=66, dt="bf16"), dict(M=9, Hq=8, Hkv=8, hd=100, dt="f16")]


@pytest.mark.parametrize("c", QLN_CASES, ids=lambda c: "M%d-H%d-%d-hd%d-%s" % (c["M"], c["Hq"], c["Hkv"], c["hd"],
                                                                             c["dt"]))
@pytest.mark.parametrize("affine", ["both", "q_only", "none"])
def test_qkv_layernorm_parity(c, affine):
    M, Hq, Hkv, hd, dt = c["M"], c["Hq"], c["Hkv"], c["hd"], c["dt"]
    g = W.generator(M * 7 + hd)
    H = Hq + 2 * Hkv
    qkv = W.normal16((M, H * hd), dt, g, scale=1.5)
    qw = W.normal16((Hq, hd), dt, g) if affine != "none" else None
    qb = W.normal16((Hq, hd), dt, g, scale=0.1) if affine != "none" else None
    kw = W.normal16((Hkv, hd), dt, g) if affine == "both" else None
    kb = W.normal16((Hkv, hd), dt, g, scale=0.1) if affine == "both" else None
    cap = max(64, 2 * M)
    cos, sin = W.rope_tables(cap, hd, 1e4)
    pos = torch.randperm(cap, generator=g)[:M].to(torch.int32)
    kc = torch.full((cap, Hkv, hd), 0x7E7E, dtype=torch.int16).view(W.DTYPES[dt])
    vc = kc.clone()
    q_raw, q_out = guarded((M, Hq, hd), qkv.dtype, 0x3C)
    dev = lambda t: None if t is None else t.to(DEV)
    kcd, vcd = kc.to(DEV), vc.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    frt.frt_qkv_layernorm_rope_kvcache(dev(qkv), dev(qw), dev(qb), dev(kw), dev(kb), dev(cos), dev(sin), dev(pos),
                                       q_out, kcd, vcd, Hq, Hkv, hd, status=status)
    torch.cuda.synchronize()
    assert_guard(q_raw, q_out.numel() * 2, 0x3C)
    hb = lambda t: None if t is None else W.bits16(t)
    o = oracle.qkv_layernorm_rope_kvcache(W.bits16(qkv), hb(qw), hb(qb), hb(kw), hb(kb), cos.numpy(), sin.numpy(),
                                          pos.numpy(), Hq, Hkv, hd, cap, 1e-6, dt, v_cache=W.bits16(vc))
    assert int(status.item()) == o["status"] == 0
    P.assert_16bit_close(P.decode16(q_out), o["q_out"], what="LN Q", dt=dt)
    p = pos.long().numpy()
    P.assert_16bit_close(P.decode16(kcd)[p], o["k_cache"][p], what="LN K", dt=dt)
    np.testing.assert_array_equal(P.np16(vcd), o["v_cache"])
    untouched = np.setdiff1d(np.arange(cap), p)
    assert (P.np16(kcd)[untouched] == 0x7E7E).all()
