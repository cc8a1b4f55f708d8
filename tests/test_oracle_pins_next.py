"""Pins for the oracle of the NEXT ops (CPU only).

NEXT-1, gated residual + AdaRMSNorm modulation + FP8 ("FlashRT kernel
fusion", §三, gate_res_adarms_fp8_static): reduction to op (a) when the gate is
one and the modulation zero, a zero gate, a closed form on constant rows, the
condition-row mapping, and the brute-force rational restatement on 4 x 8."""
import math

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
