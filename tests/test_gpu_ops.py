"""GPU parity: each fused op through the C ABI against the fp64 oracle, on the
seeded workloads (tiny, Pi0.5-like, Qwen3 prefill, VLA denoise, ViT, large-M)
and on edge shapes (single row, partial 128-blocks, odd head dims, the
largest supported widths).  Full-size large-M cases run the whole op on the
GPU and compare sampled rows with the oracle."""
import numpy as np
import pytest
import torch

import memory_bound_non_b200 as frt
import oracle
import parity as P
from memory_bound_non_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 256  # guard-band bytes after every output


def guarded(shape, dtype, fill):
    """Output tensor followed by a guard band filled with `fill` bytes."""
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    raw = torch.full((n + GUARD,), fill, dtype=torch.uint8, device=DEV)
    return raw, raw[:n].view(dtype).view(shape)


def assert_guard(raw, n_bytes, fill):
    tail = raw[n_bytes:].cpu().numpy()
    assert (tail == fill).all(), "write past the end of an output"


def sample_rows(M, k, seed=0):
    if M <= k:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    rows = rng.choice(M, size=k, replace=False)
    return np.unique(np.concatenate([rows, [0, M - 1]]))


# ================================================================ op (a) ===
A_CASES = [
    ("tiny", {}), ("pi05", {}), ("vla_denoise", {}), ("vit", {}), ("vit", {"quant": "block128"}),
    ("qwen3_prefill_S128", {}), ("qwen3_prefill_S192", {}), ("qwen3_prefill_S512", {}),
    ("qwen3_prefill_S1024", {}), ("large_m_M4096", {}),
    # edge shapes: one row, a single chunk, partial 128-blocks, every K variant
    ("tiny", {"M": 1, "D": 8}), ("tiny", {"M": 3, "D": 136, "quant": "block128"}),
    ("pi05", {"M": 5, "D": 1032, "quant": "block128"}), ("tiny", {"M": 2, "D": 8192, "dt": "bf16"}),
    ("vit", {"M": 3, "D": 16384, "quant": "block128"}), ("vit", {"M": 2, "D": 32768, "quant": "block128"}),
    ("pi05", {"M": 7, "D": 2056}), ("tiny", {"M": 9, "D": 4104, "quant": "block128", "weighted": False}),
    # small batches run one chunk per thread up to D = 4096 (512 threads a row)
    ("large_m_M4096", {"M": 100}), ("large_m_M4096", {"M": 591, "quant": "block128"}),
]


def run_a_gpu(wl, inp, scale, inplace=True):
    L = inp.layers[0]
    x = L.x_attn.to(DEV)
    r = inp.residual.to(DEV).clone()
    w = None if L.w_attn is None else L.w_attn.to(DEV)
    if inplace:
        r_out_raw, r_out = None, r
    else:
        r_out_raw, r_out = guarded((wl.M, wl.D), r.dtype, 0x5A)
    q_raw, q = guarded((wl.M, wl.D), torch.uint8, 0xA5)
    nb = (wl.D + 127) // 128
    bs_raw = bs = ss = None
    if wl.quant == "block128":
        bs_raw, bs = guarded((wl.M, nb), torch.float32, 0xFF)  # NaN fill: every scale must be written
    else:
        ss = torch.tensor([scale], dtype=torch.float32, device=DEV)
    frt.frt_residual_rmsnorm_fp8(x, r, r_out, w, q, static_scale=ss, block_scales=bs, eps=wl.eps,
                                 quant=wl.quant)
    torch.cuda.synchronize()
    assert_guard(q_raw, wl.M * wl.D, 0xA5)
    if bs_raw is not None:
        assert_guard(bs_raw, wl.M * nb * 4, 0xFF)
    if r_out_raw is not None:
        assert_guard(r_out_raw, wl.M * wl.D * 2, 0x5A)
    return r_out, q, bs


def take(t, rows):
    """Rows of a tensor (any device) as a host copy; rows=None: all."""
    if rows is None:
        return t.cpu()
    return t[torch.as_tensor(rows, device=t.device, dtype=torch.long)].cpu()


def check_a(wl, inp, rows=None, inplace=True):
    L = inp.layers[0]
    x, r = W.bits16(take(L.x_attn, rows)), W.bits16(take(inp.residual, rows))
    w = None if L.w_attn is None else W.bits16(L.w_attn)
    scale = P.calibrate_a(x, r, w, wl.eps, wl.dt)[0] if wl.quant == "static" else None
    r_out, q, bs = run_a_gpu(wl, inp, scale, inplace=inplace)
    o = oracle.residual_rmsnorm_fp8(x, r, w, wl.eps, wl.dt, wl.quant, static_scale=scale)
    np.testing.assert_array_equal(W.bits16(take(r_out, rows)), o["residual_out"])
    P.assert_fp8_codes(take(q, rows).numpy(), o["out_fp8"], what="op a codes")
    if wl.quant == "block128":
        P.assert_scales_close(take(bs, rows).numpy(), o["block_scales"])


@pytest.mark.parametrize("name,ov", A_CASES, ids=["%s%s" % (n, "".join("-%s%s" % kv for kv in o.items()))
                                                   for n, o in A_CASES])
def test_residual_rmsnorm_parity(name, ov):
    wl = W.get(name, **ov)
    check_a(wl, W.make_inputs(wl, n_layers=1, with_caches=False))


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("quant", ["static", "block128"])
@pytest.mark.parametrize("weighted", [True, False])
def test_residual_rmsnorm_modes_out_of_place(dt, quant, weighted):
    wl = W.get("vla_denoise", dt=dt, quant=quant, weighted=weighted, M=33, D=1280)
    check_a(wl, W.make_inputs(wl, n_layers=1, with_caches=False), inplace=False)


@pytest.mark.parametrize("M", [16384, 65536])
def test_residual_rmsnorm_large_m_sampled(M):
    wl = W.get("large_m_M%d" % M)
    check_a(wl, W.make_inputs(wl, n_layers=1, with_caches=False, device=DEV), rows=sample_rows(M, 384))


def test_residual_rmsnorm_saturates_and_is_deterministic():
    wl = W.get("qwen3_prefill_S512", quant="static")
    inp = W.make_inputs(wl, n_layers=1, with_caches=False)
    L = inp.layers[0]
    x, r, w = W.bits16(L.x_attn), W.bits16(inp.residual), W.bits16(L.w_attn)
    s = P.calibrate_a(x, r, w, wl.eps, wl.dt)[0] / 8  # a scale 8x too small: many saturate
    _, q1, _ = run_a_gpu(wl, inp, s)
    _, q2, _ = run_a_gpu(wl, inp, s)
    assert torch.equal(q1, q2)
    o = oracle.residual_rmsnorm_fp8(x, r, w, wl.eps, wl.dt, "static", static_scale=s)
    sat = (o["out_fp8"] & 0x7F) == 0x7E
    assert sat.mean() > 0.001
    P.assert_fp8_codes(q1.cpu().numpy(), o["out_fp8"])


@pytest.mark.parametrize("s", [2.0 ** -110, 2.0 ** -99, 2.0 ** 99, 2.0 ** 110])
def test_residual_rmsnorm_static_scale_far_from_one(s):
    """A static scale whose ratio to rstd leaves (or nears the edge of) the
    range where the kernel folds 1/s into its fp32-pair product: the codes
    still follow e4m3(y / s) (all saturated for the tiny scales, all +-0 or
    subnormal for the huge ones)."""
    wl = W.get("tiny", quant="static")
    inp = W.make_inputs(wl, n_layers=1, with_caches=False)
    L = inp.layers[0]
    x, r = W.bits16(L.x_attn), W.bits16(inp.residual)
    w = None if L.w_attn is None else W.bits16(L.w_attn)
    _, q, _ = run_a_gpu(wl, inp, s)
    o = oracle.residual_rmsnorm_fp8(x, r, w, wl.eps, wl.dt, "static", static_scale=s)
    P.assert_fp8_codes(q.cpu().numpy(), o["out_fp8"], what="op a codes, scale %g" % s)


# ================================================================ op (b) ===
B_CASES = [
    ("tiny", {}), ("pi05", {}), ("vla_denoise", {}), ("vit", {}), ("qwen3_prefill_S128", {}),
    ("qwen3_prefill_S192", {}), ("qwen3_prefill_S512", {}), ("qwen3_prefill_S1024", {}), ("large_m_M4096", {}),
    # head dims: P=8 / P=4 lanes, group sizes 1..32
    ("tiny", {"M": 3, "hd": 8}), ("tiny", {"M": 3, "hd": 16}), ("tiny", {"M": 3, "hd": 24, "Hq": 4, "Hkv": 4}),
    ("tiny", {"M": 5, "hd": 40, "Hq": 6, "Hkv": 3}), ("tiny", {"M": 4, "hd": 64}),
    ("vit", {"M": 7, "qk_norm": True}), ("tiny", {"M": 2, "hd": 248, "Hq": 2, "Hkv": 1}),
    ("tiny", {"M": 2, "hd": 256, "dt": "bf16"}), ("tiny", {"M": 1}),
    # hd % 8 != 0: the element-wise kernel (odd hd / 2 for 66 and 2)
    ("tiny", {"M": 5, "hd": 66}), ("vit", {"M": 9, "hd": 100, "qk_norm": True}),
    ("tiny", {"M": 4, "hd": 2, "Hq": 4, "Hkv": 2}), ("tiny", {"M": 3, "hd": 250, "Hq": 2, "Hkv": 1, "dt": "bf16"}),
    ("large_m_M4096", {"M": 700, "hd": 100, "Hq": 20, "Hkv": 4, "capacity": 2048}),
]


def b_inputs(wl):
    return W.make_inputs(wl, n_layers=1, with_caches=True)


def run_b_gpu(wl, inp, positions=None):
    L = inp.layers[0]
    pos = (inp.positions if positions is None else positions).to(DEV)
    kc, vc = L.k_cache.to(DEV).clone(), L.v_cache.to(DEV).clone()
    q_raw, q_out = guarded((wl.M, wl.Hq, wl.hd), L.qkv.dtype, 0x3C)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    frt.frt_qkv_norm_rope_kvcache(L.qkv.to(DEV), None if L.q_norm_w is None else L.q_norm_w.to(DEV),
                                  None if L.k_norm_w is None else L.k_norm_w.to(DEV), inp.cos.to(DEV),
                                  inp.sin.to(DEV), pos, q_out, kc, vc, wl.Hq, wl.Hkv, wl.hd, status=status,
                                  eps=wl.eps)
    torch.cuda.synchronize()
    assert_guard(q_raw, q_out.numel() * 2, 0x3C)
    return q_out, kc, vc, int(status.item())


def oracle_b(wl, inp, rows=None, positions=None):
    L = inp.layers[0]
    pos = take(inp.positions if positions is None else positions, rows).numpy()
    qkv = W.bits16(take(L.qkv, rows))
    slots = None
    cap = wl.capacity
    vinit = None
    if rows is not None:  # compact cache for the sampled rows
        slots = np.arange(len(rows))
        cap = len(rows)
    else:
        vinit = W.bits16(L.v_cache)
    return oracle.qkv_norm_rope_kvcache(
        qkv, None if L.q_norm_w is None else W.bits16(L.q_norm_w),
        None if L.k_norm_w is None else W.bits16(L.k_norm_w), inp.cos.cpu().numpy(), inp.sin.cpu().numpy(),
        pos, wl.Hq, wl.Hkv, wl.hd, cap, wl.eps, wl.dt, slots=slots, v_cache=vinit)


def check_b_full(wl, inp):
    q_out, kc, vc, status = run_b_gpu(wl, inp)
    o = oracle_b(wl, inp)
    assert status == o["status"] == 0
    P.assert_16bit_close(P.decode16(q_out), o["q_out"], what="Q staging", dt=wl.dt)
    written = ~np.isnan(o["k_cache"]).all(axis=(1, 2))
    k0, v0 = W.bits16(inp.layers[0].k_cache), W.bits16(inp.layers[0].v_cache)
    kg, vg = P.np16(kc), P.np16(vc)
    P.assert_16bit_close(P.decode16(kc)[written], o["k_cache"][written], what="K cache", dt=wl.dt)
    np.testing.assert_array_equal(vg[written], o["v_cache"][written])
    np.testing.assert_array_equal(kg[~written], k0[~written])   # untouched slots keep their bits
    np.testing.assert_array_equal(vg[~written], v0[~written])
    assert written.sum() == len(np.unique(inp.positions.numpy()))


@pytest.mark.parametrize("name,ov", B_CASES, ids=["%s%s" % (n, "".join("-%s%s" % kv for kv in o.items()))
                                                   for n, o in B_CASES])
def test_qkv_norm_rope_kvcache_parity(name, ov):
    wl = W.get(name, **ov)
    check_b_full(wl, b_inputs(wl))


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("qn,kn", [(True, False), (False, True)])
def test_qkv_one_sided_norm(dt, qn, kn):
    wl = W.get("tiny", dt=dt, M=6, Hq=4, Hkv=2, hd=128, qk_norm=True)
    inp = b_inputs(wl)
    L = inp.layers[0]
    if not qn:
        L.q_norm_w = None
    if not kn:
        L.k_norm_w = None
    check_b_full(wl, inp)


@pytest.mark.parametrize("M", [16384, 65536])
def test_qkv_large_m_sampled(M):
    wl = W.get("large_m_M%d" % M)
    inp = W.make_inputs(wl, n_layers=1, with_caches=True, device=DEV)
    q_out, kc, vc, status = run_b_gpu(wl, inp)
    assert status == 0
    rows = sample_rows(M, 256)
    o = oracle_b(wl, inp, rows=rows)
    pos = take(inp.positions, rows).numpy()
    P.assert_16bit_close(P.decode16(q_out[torch.from_numpy(rows).to(DEV)]), o["q_out"], what="Q staging", dt=wl.dt)
    P.assert_16bit_close(P.decode16(kc[torch.from_numpy(pos).long().to(DEV)]), o["k_cache"], what="K cache", dt=wl.dt)
    np.testing.assert_array_equal(P.np16(vc[torch.from_numpy(pos).long().to(DEV)]), o["v_cache"])
    # every slot outside the written set still holds the sentinel
    mask = torch.ones(wl.capacity, dtype=torch.bool, device=DEV)
    mask[inp.positions.long().to(DEV)] = False
    sent = torch.tensor(0x7E7E, dtype=torch.int16, device=DEV)
    assert bool((kc[mask].view(torch.int16) == sent).all()) and bool((vc[mask].view(torch.int16) == sent).all())
    assert int((~mask).sum()) == M


def test_qkv_bad_positions_set_status_and_skip_rows():
    wl = W.get("tiny", M=6, capacity=32)
    inp = b_inputs(wl)
    pos = torch.tensor([3, 32, 0, -1, 31, 1 << 30], dtype=torch.int32)
    q_out, kc, vc, status = run_b_gpu(wl, inp, positions=pos)
    o = oracle_b(wl, inp, positions=pos)
    assert status == 1 and o["status"] == 1
    good = np.array([0, 2, 4])
    P.assert_16bit_close(P.decode16(q_out)[good], o["q_out"][good], what="Q staging", dt=wl.dt)
    # skipped rows leave their Q staging rows as they were (guard fill 0x3C3C)
    assert (P.np16(q_out)[[1, 3, 5]] == 0x3C3C).all()
    written = ~np.isnan(o["k_cache"]).all(axis=(1, 2))
    assert sorted(np.flatnonzero(written).tolist()) == [0, 3, 31]
    np.testing.assert_array_equal(P.np16(kc)[~written], W.bits16(inp.layers[0].k_cache)[~written])
    np.testing.assert_array_equal(P.np16(vc)[written], o["v_cache"][written])


# --------------------------------------------- large batches (bulk-copy path)
@pytest.mark.parametrize("ov", [
    {"M": 600, "dt": "f16"},                                   # smallest batch on the bulk-copy path
    {"M": 700, "hd": 256, "Hq": 8, "Hkv": 2, "capacity": 1024},  # 16 lanes per head, 4 KB+ rows
    {"M": 640, "hd": 64, "Hq": 12, "Hkv": 4, "capacity": 1024},
    {"M": 1200, "hd": 72, "Hq": 16, "Hkv": 16, "qk_norm": True, "capacity": 2048},  # P = 4
])
def test_qkv_bulk_copy_path_parity(ov):
    wl = W.get("large_m_M4096", **ov)
    check_b_full(wl, b_inputs(wl))


def test_qkv_bulk_copy_path_bad_positions():
    wl = W.get("large_m_M4096", M=640, capacity=2048)
    inp = b_inputs(wl)
    pos = inp.positions.clone()
    bad = torch.tensor([3, 100, 639])
    pos[bad] = torch.tensor([-5, 2048, 1 << 29], dtype=torch.int32)
    q_out, kc, vc, status = run_b_gpu(wl, inp, positions=pos)
    o = oracle_b(wl, inp, positions=pos)
    assert status == 1 and o["status"] == 1
    good = np.setdiff1d(np.arange(wl.M), bad.numpy())
    P.assert_16bit_close(P.decode16(q_out)[good], o["q_out"][good], what="Q staging", dt=wl.dt)
    assert (P.np16(q_out)[bad.numpy()] == 0x3C3C).all()          # skipped rows untouched
    written = ~np.isnan(o["k_cache"]).all(axis=(1, 2))
    assert written.sum() == wl.M - 3
    np.testing.assert_array_equal(P.np16(kc)[~written], W.bits16(inp.layers[0].k_cache)[~written])
    np.testing.assert_array_equal(P.np16(vc), o["v_cache"])


def test_qkv_bulk_copy_wait_give_up_sets_bit1_and_writes_nothing():
    """The bulk-copy kernel's bounded barrier wait, forced to give up (a bound
    of 0 polls): every token sets status bit 1 and writes none of its
    outputs (Q staging keeps its fill, both caches their contents); the
    kernel drains its copies before exiting, and the next call with the
    default bound is correct."""
    wl = W.get("large_m_M4096", M=640, capacity=2048)
    inp = b_inputs(wl)
    L = inp.layers[0]
    frt.frt_set_wait_polls(0)
    try:
        q_out, kc, vc, status = run_b_gpu(wl, inp)
    finally:
        frt.frt_set_wait_polls(frt.FRT_DEFAULT_WAIT_POLLS)
    assert status == 2
    assert (P.np16(q_out) == 0x3C3C).all()
    np.testing.assert_array_equal(P.np16(kc), W.bits16(L.k_cache))
    np.testing.assert_array_equal(P.np16(vc), W.bits16(L.v_cache))
    check_b_full(wl, inp)


@pytest.mark.parametrize("qn,kn", [(True, False), (False, True), (False, False)])
def test_qkv_bulk_copy_path_one_sided_norm(qn, kn):
    wl = W.get("large_m_M4096", M=600)
    inp = b_inputs(wl)
    L = inp.layers[0]
    L.q_norm_w = L.q_norm_w if qn else None
    L.k_norm_w = L.k_norm_w if kn else None
    check_b_full(wl, inp)


def test_qkv_large_batch_with_8_byte_aligned_rows_uses_the_register_kernel():
    # hd = 72 needs only 8-byte alignment; views offset by 8 bytes rule out the
    # bulk-copy path, so the register kernel runs the large batch
    wl = W.get("vit", M=800, qk_norm=True)
    inp = b_inputs(wl)
    L = inp.layers[0]
    o = oracle_b(wl, inp)

    def off8(t):
        raw = torch.empty(t.numel() + 4, dtype=t.dtype, device=DEV)
        v = raw[4:].view(t.shape)                                   # +8 bytes
        v.copy_(t.to(DEV))
        return v
    qkv = off8(L.qkv)
    kc, vc = off8(L.k_cache), off8(L.v_cache)
    q_out = off8(torch.zeros((wl.M, wl.Hq, wl.hd), dtype=L.qkv.dtype))
    frt.frt_qkv_norm_rope_kvcache(qkv, off8(L.q_norm_w), off8(L.k_norm_w), inp.cos.to(DEV), inp.sin.to(DEV),
                                  inp.positions.to(DEV), q_out, kc, vc, wl.Hq, wl.Hkv, wl.hd, eps=wl.eps)
    torch.cuda.synchronize()
    assert qkv.data_ptr() % 16 == 8
    P.assert_16bit_close(P.decode16(q_out), o["q_out"], what="Q staging", dt=wl.dt)
    written = ~np.isnan(o["k_cache"]).all(axis=(1, 2))
    P.assert_16bit_close(P.decode16(kc)[written], o["k_cache"][written], what="K cache", dt=wl.dt)
    np.testing.assert_array_equal(P.np16(vc), o["v_cache"])


# ================================================================ op (c) ===
C_CASES = [
    ("tiny", {}), ("pi05", {}), ("vla_denoise", {}), ("vit", {}), ("vit", {"quant": "block128"}),
    ("qwen3_prefill_S128", {}), ("qwen3_prefill_S192", {}), ("qwen3_prefill_S512", {}),
    ("qwen3_prefill_S1024", {}), ("large_m_M4096", {}),
    ("tiny", {"M": 1, "I": 4}), ("tiny", {"M": 3, "I": 132, "quant": "block128"}),
    ("vit", {"M": 5, "I": 4304, "quant": "block128", "dt": "f16"}), ("pi05", {"M": 2, "I": 20, "act": "silu"}),
    ("tiny", {"M": 37, "I": 1000, "quant": "block128", "act": "relu2"}),
]


def run_c_gpu(wl, gu, scale):
    q_raw, q = guarded((wl.M, wl.I), torch.uint8, 0xA5)
    nb = (wl.I + 127) // 128
    bs_raw = bs = ss = None
    if wl.quant == "block128":
        bs_raw, bs = guarded((wl.M, nb), torch.float32, 0xFF)
    else:
        ss = torch.tensor([scale], dtype=torch.float32, device=DEV)
    frt.frt_gate_act_fp8(gu.to(DEV), q, static_scale=ss, block_scales=bs, act=wl.act, quant=wl.quant)
    torch.cuda.synchronize()
    assert_guard(q_raw, wl.M * wl.I, 0xA5)
    if bs_raw is not None:
        assert_guard(bs_raw, wl.M * nb * 4, 0xFF)
    return q, bs


def check_c(wl, gu_in, rows=None):
    gu = W.bits16(take(gu_in, rows))
    scale = P.calibrate_c(gu, wl.act, wl.dt) if wl.quant == "static" else None
    q, bs = run_c_gpu(wl, gu_in, scale)
    o = oracle.gate_act_fp8(gu, wl.act, wl.dt, wl.quant, static_scale=scale)
    P.assert_fp8_codes(take(q, rows).numpy(), o["out_fp8"], what="op c codes")
    if wl.quant == "block128":
        P.assert_scales_close(take(bs, rows).numpy(), o["block_scales"])


@pytest.mark.parametrize("name,ov", C_CASES, ids=["%s%s" % (n, "".join("-%s%s" % kv for kv in o.items()))
                                                   for n, o in C_CASES])
def test_gate_act_parity(name, ov):
    wl = W.get(name, **ov)
    check_c(wl, W.make_inputs(wl, n_layers=1, with_caches=False).layers[0].gate_up)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("act", ["gelu_tanh", "silu", "relu2"])
@pytest.mark.parametrize("quant", ["static", "block128"])
def test_gate_act_modes(dt, act, quant):
    wl = W.get("vit", dt=dt, act=act, quant=quant, M=19, I=1156)
    g = W.generator(31)
    gu = W.normal16((wl.M, 2 * wl.I), dt, g, scale=3.0)   # wide range: both tails of each activation
    check_c(wl, gu)


@pytest.mark.parametrize("M", [16384, 65536])
def test_gate_act_large_m_sampled(M):
    wl = W.get("large_m_M%d" % M)
    gu = W.make_inputs(wl, n_layers=1, with_caches=False, device=DEV).layers[0].gate_up
    check_c(wl, gu, rows=sample_rows(M, 128))


def test_gate_act_deterministic_and_saturating():
    wl = W.get("qwen3_prefill_S512")
    gu = W.make_inputs(wl, n_layers=1, with_caches=False).layers[0].gate_up
    q1, b1 = run_c_gpu(wl, gu, None)
    q2, b2 = run_c_gpu(wl, gu, None)
    assert torch.equal(q1, q2) and torch.equal(b1, b2)
    wl_s = W.get("qwen3_prefill_S512", quant="static")
    s = P.calibrate_c(W.bits16(gu), wl_s.act, wl_s.dt) / 16
    q, _ = run_c_gpu(wl_s, gu, s)
    o = oracle.gate_act_fp8(W.bits16(gu), wl_s.act, wl_s.dt, "static", static_scale=s)
    assert ((o["out_fp8"] & 0x7F) == 0x7E).mean() > 0.001
    P.assert_fp8_codes(q.cpu().numpy(), o["out_fp8"])


# ================================================================= misc ===
def test_empty_batch_launches_nothing():
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device=DEV)
    q = torch.zeros((0, 64), dtype=torch.uint8, device=DEV)
    frt.frt_residual_rmsnorm_fp8(x, x, x, None, q, static_scale=torch.ones(1, device=DEV))
    frt.frt_gate_act_fp8(torch.zeros((0, 64), dtype=torch.bfloat16, device=DEV), torch.zeros((0, 32),
                         dtype=torch.uint8, device=DEV), static_scale=torch.ones(1, device=DEV))
    torch.cuda.synchronize()


def test_noop_runs():
    frt.frt_noop(148, 128)
    torch.cuda.synchronize()
