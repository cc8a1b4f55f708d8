"""GPU parity of the graphed layer chain: layers x steps invocations of
a -> b -> a -> c captured in one CUDA graph, against the oracle replaying the
same sequence (residual carried in place from one invocation to the next)."""
import numpy as np
import pytest
import torch

import memory_bound_non_b200 as frt
import parity as P
from memory_bound_non_b200 import workloads as W
from memory_bound_non_b200.chain import LayerChain

pytestmark = pytest.mark.gpu


def compare_chain(wl, inp, chain, r_ref, outs):
    np.testing.assert_array_equal(P.np16(chain.residual), r_ref)
    assert int(chain.status.item()) == 0
    for l, (L, o) in enumerate(zip(chain.layers, outs)):
        P.assert_fp8_codes(L.q8_attn.cpu().numpy(), o["a1"]["out_fp8"], what="layer %d attn fp8" % l)
        P.assert_fp8_codes(L.q8_ffn.cpu().numpy(), o["a2"]["out_fp8"], what="layer %d ffn fp8" % l)
        P.assert_fp8_codes(L.act8.cpu().numpy(), o["c"]["out_fp8"], what="layer %d act fp8" % l)
        if wl.quant == "block128":
            P.assert_scales_close(L.bs_attn.cpu().numpy(), o["a1"]["block_scales"])
            P.assert_scales_close(L.bs_act.cpu().numpy(), o["c"]["block_scales"])
        P.assert_16bit_close(P.decode16(L.q_out), o["b"]["q_out"], what="layer %d Q" % l, dt=wl.dt)
        written = ~np.isnan(o["b"]["k_cache"]).all(axis=(1, 2))
        P.assert_16bit_close(P.decode16(L.k_cache)[written], o["b"]["k_cache"][written], what="layer %d K" % l, dt=wl.dt)
        np.testing.assert_array_equal(P.np16(L.v_cache), o["b"]["v_cache"])
        k0 = W.bits16(inp.layers[l].k_cache)
        np.testing.assert_array_equal(P.np16(L.k_cache)[~written], k0[~written])


@pytest.mark.parametrize("name,steps", [("pi05", 10), ("vla_denoise", 10), ("tiny", 3),
                                        ("qwen3_prefill_S128", 2)])
def test_graphed_chain_matches_oracle(name, steps):
    wl = W.get(name, steps=steps, layers=max(W.get(name).layers, 2))
    inp = W.make_inputs(wl)
    scales = P.chain_scales(wl, inp)
    chain = LayerChain(wl, inp, scales=scales)
    chain.capture()
    chain.reset()
    chain.replay()
    torch.cuda.synchronize()
    r_ref, outs = P.oracle_chain(wl, inp, scales, steps)
    compare_chain(wl, inp, chain, r_ref, outs)


def test_graph_replay_equals_stream_launches_and_is_bitwise_repeatable():
    wl = W.get("pi05", steps=3)
    inp = W.make_inputs(wl)
    chain = LayerChain(wl, inp, scales=P.chain_scales(wl, inp))
    chain.reset()
    chain.run()
    torch.cuda.synchronize()
    eager = [t.clone() for L in chain.layers for t in (L.q8_attn, L.q8_ffn, L.act8, L.q_out, L.k_cache)]
    r_eager = chain.residual.clone()
    chain.capture()
    for _ in range(5):  # five replays from the same start: bit-identical
        chain.reset()
        chain.replay()
        torch.cuda.synchronize()
        assert torch.equal(chain.residual, r_eager)
        got = [t for L in chain.layers for t in (L.q8_attn, L.q8_ffn, L.act8, L.q_out, L.k_cache)]
        assert all(torch.equal(a, b) for a, b in zip(eager, got))


def test_calibrated_static_scales_match_oracle_calibration():
    wl = W.get("pi05")
    inp = W.make_inputs(wl, n_layers=1)
    chain = LayerChain(wl, inp)
    got = chain.calibrate_static_scales().cpu().numpy()
    want = np.array(P.chain_scales(wl, inp))
    np.testing.assert_allclose(got, want, rtol=1e-6)


def test_pdl_on_and_off_give_identical_results():
    wl = W.get("vla_denoise", steps=2, layers=4)
    inp = W.make_inputs(wl)
    scales = P.chain_scales(wl, inp)
    results = []
    prev = frt.frt_get_pdl()
    try:
        for pdl in (False, True):
            frt.frt_set_pdl(pdl)
            chain = LayerChain(wl, inp, scales=scales)
            chain.capture()
            chain.reset()
            chain.replay()
            chain.run()  # and the same chain launched stream by stream
            torch.cuda.synchronize()
            results.append([chain.residual.clone()] + [t.clone() for L in chain.layers
                                                         for t in (L.q8_attn, L.q8_ffn, L.act8, L.q_out, L.k_cache)])
    finally:
        frt.frt_set_pdl(prev)
    assert all(torch.equal(a, b) for a, b in zip(*results))


# ------------------------------------------------- NEXT-4: persistent chain ---
@pytest.mark.parametrize("name,steps", [("pi05", 10), ("vla_denoise", 10), ("tiny", 3),
                                        ("qwen3_prefill_S128", 2)])
def test_persistent_chain_matches_oracle(name, steps):
    wl = W.get(name, steps=steps, layers=max(W.get(name).layers, 2))
    inp = W.make_inputs(wl)
    scales = P.chain_scales(wl, inp)
    chain = LayerChain(wl, inp, scales=scales)
    chain.reset()
    chain.run_persistent()
    torch.cuda.synchronize()
    r_ref, outs = P.oracle_chain(wl, inp, scales, steps)
    compare_chain(wl, inp, chain, r_ref, outs)


@pytest.mark.parametrize("name,ov", [("pi05", {}), ("vla_denoise", {}), ("tiny", {}),
                                     # clusters of 2 (one worker CTA) and of 1 (one CTA does every op); a
                                     # cache deep enough that every row's position is in range (a skipped
                                     # row leaves q_out as allocated, which is not an output)
                                     ("pi05", {"M": 74, "layers": 4, "capacity": 2048}),
                                     ("pi05", {"M": 80, "layers": 4, "capacity": 2048})])
def test_persistent_chain_equals_graphed_chain_bitwise(name, ov):
    """One launch for steps x layers x 4 ops gives the same bits as the
    graph of per-op launches."""
    wl = W.get(name, steps=3, **ov)
    inp = W.make_inputs(wl)
    chain = LayerChain(wl, inp, scales=P.chain_scales(wl, inp))
    chain.capture()
    chain.reset()
    chain.replay()
    torch.cuda.synchronize()
    ref = [t.clone() for L in chain.layers for t in (L.q8_attn, L.q8_ffn, L.act8, L.q_out, L.k_cache, L.v_cache)]
    r_ref = chain.residual.clone()
    for L in chain.layers:               # clear the outputs so stale values cannot pass
        for t in (L.q8_attn, L.q8_ffn, L.act8, L.q_out):
            t.zero_()
    chain.reset()
    chain.capture_persistent()
    chain.reset()
    chain.graph_persistent.replay()
    torch.cuda.synchronize()
    bits = lambda t: t.view(torch.uint8)   # bit patterns: the fp16 cache sentinel 0x7E7E is a NaN
    assert int(chain.status.item()) == 0
    assert torch.equal(bits(chain.residual), bits(r_ref))
    got = [t for L in chain.layers for t in (L.q8_attn, L.q8_ffn, L.act8, L.q_out, L.k_cache, L.v_cache)]
    assert all(torch.equal(bits(a), bits(b)) for a, b in zip(ref, got))


@pytest.mark.parametrize("field,offset", [("x_attn", 2), ("q8_attn", 4), ("act8", 2), ("k_cache", 8)])
def test_persistent_chain_misaligned_table_pointer_sets_bit2_and_writes_nothing(field, offset):
    """A layer record whose pointer sits below its field's alignment (16 bytes
    for the staged inputs and the caches, 8 for the norm codes, 4 for the
    activation codes) is caught in the kernel before anything is read through
    the table: status bit 2, and every output keeps its contents."""
    wl = W.get("pi05", layers=3, steps=1)
    inp = W.make_inputs(wl)
    chain = LayerChain(wl, inp, scales=P.chain_scales(wl, inp))
    chain.reset()
    L = chain.layers[1]
    t = getattr(L, field)
    nbytes = t.numel() * t.element_size()
    raw = torch.zeros(nbytes + 16, dtype=torch.uint8, device=t.device)
    raw[offset:offset + nbytes].copy_(t.reshape(-1).view(torch.uint8))
    setattr(L, field, raw[offset:offset + nbytes].view(t.dtype).view(t.shape))
    assert getattr(L, field).data_ptr() % 16 == offset
    before = [x.clone() for x in [chain.residual] + [getattr(Y, n) for Y in chain.layers
                                                     for n in ("q8_attn", "q8_ffn", "act8", "q_out", "k_cache",
                                                               "v_cache")]]
    chain.run_persistent()
    torch.cuda.synchronize()
    assert int(chain.status.item()) == 4
    after = [chain.residual] + [getattr(Y, n) for Y in chain.layers
                                for n in ("q8_attn", "q8_ffn", "act8", "q_out", "k_cache", "v_cache")]
    bits = lambda x: x.view(torch.uint8)
    assert all(torch.equal(bits(a), bits(b)) for a, b in zip(before, after))
