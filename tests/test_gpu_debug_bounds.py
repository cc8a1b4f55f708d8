"""The bounds-checked build (libfrt_debug.so, include/frt_debug.h) as a
stand-in for an address sanitizer: every op family runs through it on small
shapes, every global access must fall inside the extents its call implies
(zero violations), and its outputs must be bit-identical to the product
library's on the same inputs."""
import numpy as np
import pytest
import torch

import memory_bound_non_b200 as frt
from memory_bound_non_b200 import workloads as W
from memory_bound_non_b200.chain import LayerChain

pytestmark = pytest.mark.gpu
DEV = "cuda"


def both_builds(fn):
    """fn() -> list of device tensors; run it on the product library and on
    the bounds-checked one, require no violation and equal bits."""
    ref = [t.clone() for t in fn()]
    torch.cuda.synchronize()
    with frt.using_library(frt.load_debug()):
        frt.bounds_violations()          # start from zero
        got = [t.clone() for t in fn()]
        n = frt.bounds_violations()
    assert n == 0, "%d out-of-range accesses" % n
    for a, b in zip(ref, got):
        np.testing.assert_array_equal(a.view(torch.uint8).cpu().numpy(), b.view(torch.uint8).cpu().numpy())


def chain_outputs(ch):
    outs = [ch.residual, ch.status]
    for L in ch.layers:
        outs += [L.q8_attn, L.q8_ffn, L.act8, L.q_out, L.k_cache, L.v_cache]
        outs += [t for t in (L.bs_attn, L.bs_ffn, L.bs_act) if t is not None]
    return outs


@pytest.mark.parametrize("name,ov", [("tiny", {"layers": 2, "steps": 2}), ("pi05", {"layers": 2, "steps": 1}),
                                     ("vla_denoise", {"layers": 1, "steps": 1}),
                                     ("qwen3_prefill_S128", {"layers": 1, "steps": 1}),
                                     ("vit", {"M": 40, "layers": 1, "steps": 1}),
                                     ("large_m_M4096", {"M": 600, "layers": 1, "steps": 1, "capacity": 2048}),
                                     # clusters of 2 (one worker CTA) and of 1 (one CTA does every op),
                                     # every position in range (a skipped row leaves q_out as allocated)
                                     ("pi05", {"M": 74, "layers": 2, "steps": 1, "capacity": 2048}),
                                     ("pi05", {"M": 80, "layers": 2, "steps": 1, "capacity": 2048})])
@pytest.mark.parametrize("persistent", [False, True])
def test_chain_in_bounds(name, ov, persistent):
    wl = W.get(name, **ov)
    if persistent and (wl.hd % 16 != 0 or wl.M > 80):
        pytest.skip("outside the persistent chain's shapes")
    inp = W.make_inputs(wl)

    def run():
        ch = LayerChain(wl, inp)
        ch.calibrate_static_scales()
        ch.run_persistent() if persistent else ch.run()
        torch.cuda.synchronize()
        return chain_outputs(ch)
    both_builds(run)


def test_next_ops_in_bounds():
    g = W.generator(7, DEV)
    M, D, I = 130, 1040, 4304
    x, r = W.normal16((M, D), "bf16", g), W.normal16((M, D), "bf16", g)
    w, b = W.norm_weight(D, "bf16", g), W.normal16((D,), "bf16", g, scale=0.1)
    gate, sc, sh = (W.normal16((3, D), "bf16", g, scale=0.3) for _ in range(3))
    gu = W.normal16((M, 2 * 4352), "bf16", g)
    gsd = torch.tensor([0.002], device=DEV)
    ss = torch.tensor([0.02], device=DEV)

    def run():
        rr = r.clone()
        out = []
        q = torch.empty((M, D), dtype=torch.uint8, device=DEV)
        bs = torch.empty((M, (D + 127) // 128), dtype=torch.float32, device=DEV)
        frt.frt_gate_residual_adarms_fp8(x, gate, rr, rr, sc, sh, q, block_scales=bs, rows_per_cond=50,
                                         quant="block128")
        out += [rr.clone(), q.clone(), bs.clone()]
        for layout in ("rows", "swizzled"):
            q4 = torch.empty((M, D // 2), dtype=torch.uint8, device=DEV)
            sf = torch.zeros((frt.nvfp4_sf_bytes(M, D, layout),), dtype=torch.uint8, device=DEV)
            frt.frt_residual_rmsnorm_nvfp4(x, rr, rr, w, q4, sf, gsd, sf_layout=layout)
            out += [rr.clone(), q4, sf]
            qc = torch.empty((M, 4352 // 2), dtype=torch.uint8, device=DEV)
            sfc = torch.zeros((frt.nvfp4_sf_bytes(M, 4352, layout),), dtype=torch.uint8, device=DEV)
            frt.frt_gate_act_nvfp4(gu, qc, sfc, gsd, act="silu", sf_layout=layout)
            out += [qc, sfc]
        q8 = torch.empty((M, D), dtype=torch.uint8, device=DEV)
        frt.frt_residual_layernorm_fp8(x, rr, rr, w, b, q8, static_scale=ss)
        out += [rr.clone(), q8]
        a8 = torch.empty((M, I), dtype=torch.uint8, device=DEV)
        bsi = torch.empty((M, (I + 127) // 128), dtype=torch.float32, device=DEV)
        frt.frt_gate_act_fp8(gu[:, :2 * I].contiguous(), a8, block_scales=bsi, act="gelu_tanh", quant="block128")
        out += [a8, bsi]
        torch.cuda.synchronize()
        return out
    both_builds(run)


@pytest.mark.parametrize("M,Hq,Hkv,hd", [(7, 8, 2, 128), (650, 32, 8, 128), (9, 16, 16, 72), (5, 8, 2, 66),
                                         (6, 4, 4, 100)])
def test_qkv_forms_in_bounds(M, Hq, Hkv, hd):
    g = W.generator(M + hd, DEV)
    cap = 2 * M + 3
    qkv = W.normal16((M, (Hq + 2 * Hkv) * hd), "bf16", g)
    qw, kw = W.norm_weight(hd, "bf16", g), W.norm_weight(hd, "bf16", g)
    lw, lb = W.normal16((Hq, hd), "bf16", g), W.normal16((Hq, hd), "bf16", g, scale=0.1)
    cos, sin = W.rope_tables(cap, hd, 1e4)
    cos, sin = cos.to(DEV), sin.to(DEV)
    pos = torch.randperm(cap, generator=torch.Generator().manual_seed(M))[:M].to(torch.int32).to(DEV)
    kvs = torch.tensor([0.02, 0.015], device=DEV)

    def run():
        out = []
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        qo = torch.zeros((M, Hq, hd), dtype=torch.bfloat16, device=DEV)
        kc = torch.zeros((cap, Hkv, hd), dtype=torch.bfloat16, device=DEV)
        vc = torch.zeros_like(kc)
        frt.frt_qkv_norm_rope_kvcache(qkv, qw, kw, cos, sin, pos, qo, kc, vc, Hq, Hkv, hd, status=st)
        out += [qo.clone(), kc.clone(), vc.clone()]
        frt.frt_qkv_layernorm_rope_kvcache(qkv, lw, lb, None, None, cos, sin, pos, qo, kc, vc, Hq, Hkv, hd,
                                           status=st)
        out += [qo.clone(), kc.clone(), vc.clone()]
        qh = torch.zeros((Hq, M, hd), dtype=torch.bfloat16, device=DEV)
        k8 = torch.zeros((cap, Hkv, hd), dtype=torch.uint8, device=DEV)
        v8 = torch.zeros_like(k8)
        frt.frt_qkv_norm_rope_prepq_kvcache(qkv, qw, kw, cos, sin, pos, qh, k8, v8, Hq, Hkv, hd, q_scale=0.125,
                                            q_layout="head", kv="e4m3", kv_scales=kvs, status=st)
        out += [qh, k8, v8, st]
        torch.cuda.synchronize()
        return out
    both_builds(run)
