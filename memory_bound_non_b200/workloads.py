"""Seeded synthetic workloads for the fused layer ops.

This module only draws inputs: shapes, seeds, value distributions, position
sets and the precomputed RoPE cos/sin table that a caller hands to the op.  It
holds none of the ops' arithmetic, so the CUDA path and the CPU oracle can
both consume exactly the same host buffers.

Every tensor is drawn from a seeded ``torch.Generator``: on the host
(``device="cpu"``, the default, used for every case the oracle checks in
full) or, for the multi-GB large-M workloads, on the GPU (``device="cuda"``;
the same recipe and seed, a different stream of numbers), with host copies
taken for the oracle.  The shapes follow the workloads of the source pages:
  * a Pi0.5-like action decoder (M=10 tokens; 18 layers x 10 flow steps),
  * a Qwen3-style text prefill (S = 128..1024, q/k norm, block-128 FP8),
  * a VLA denoise step (M=41, 32 layers x 10 steps) and its ViT (M=1176,
    head_dim 72),
  * a large-M bandwidth sweep (M up to 65536, squared-ReLU FFN),
as described in "FlashRT kernel fusion" (§一-§三), "FlashRT port of
Hy-Embodied-0.5-VLA" (01 WORKLOAD, 05 CASE), "sm89 prefill FFN megakernel"
(Phase 0) and "Falcon-Perception inference optimisation" (third technique).
"""
from dataclasses import dataclass, field, replace
import math
from typing import Optional, Tuple

import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}

# Bound on the float32 temporary used while drawing one tensor.
_CHUNK_ELEMS = 1 << 26


@dataclass(frozen=True)
class Workload:
    name: str
    M: int                      # token rows
    D: int                      # hidden size
    dt: str                     # "f16" | "bf16"
    weighted: bool              # RMSNorm weight present (else `_noweight`)
    quant: str                  # "static" | "block128"
    Hq: int
    Hkv: int
    hd: int
    qk_norm: bool
    theta: float
    positions: str              # "range" | "unique_random"
    pos_start: int              # first position for "range"
    capacity: int               # KV-cache slots (== RoPE table rows)
    prefill: int                # cache slots [0, prefill) hold earlier tokens
    I: int                      # FFN intermediate size
    act: str                    # "gelu_tanh" | "silu" | "relu2"
    seed: int
    outlier_frac: float = 0.0   # fraction of channels scaled by outlier_mult
    outlier_mult: float = 50.0
    layers: int = 1
    steps: int = 1
    eps: float = 1e-6

    @property
    def qkv_width(self) -> int:
        return (self.Hq + 2 * self.Hkv) * self.hd

    @property
    def max_pos(self) -> int:
        return self.capacity


WORKLOADS = {
    # tiny chain, seed 0 (fp16, weighted, static FP8, qk-norm, GeGLU-tanh)
    "tiny": Workload("tiny", M=10, D=1024, dt="f16", weighted=True, quant="static", Hq=8, Hkv=1, hd=128,
                     qk_norm=True, theta=1e4, positions="range", pos_start=0, capacity=64, prefill=0,
                     I=4096, act="gelu_tanh", seed=0),
    # Pi0.5-like action decoder: 18 layers x 10 flow steps in one graph
    "pi05": Workload("pi05", M=10, D=1024, dt="bf16", weighted=False, quant="static", Hq=8, Hkv=1, hd=256,
                     qk_norm=False, theta=1e4, positions="range", pos_start=968, capacity=1024, prefill=968,
                     I=4096, act="gelu_tanh", seed=1, layers=18, steps=10),
    # VLA denoise: M=41 action tokens after a 181-token prefix, 32 layers x 10 steps
    "vla_denoise": Workload("vla_denoise", M=41, D=2048, dt="bf16", weighted=True, quant="static", Hq=16,
                            Hkv=8, hd=128, qk_norm=True, theta=1e4, positions="range", pos_start=181,
                            capacity=256, prefill=181, I=8192, act="silu", seed=3, layers=32, steps=10),
    # ViT: 6 frames x 196 patches, head_dim 72 unpadded, GeGLU-tanh inter 4304
    "vit": Workload("vit", M=1176, D=1152, dt="bf16", weighted=True, quant="static", Hq=16, Hkv=16, hd=72,
                    qk_norm=False, theta=1e4, positions="range", pos_start=0, capacity=1176, prefill=0,
                    I=4304, act="gelu_tanh", seed=3),
}
for _S in (128, 192, 512, 1024):
    WORKLOADS["qwen3_prefill_S%d" % _S] = Workload(
        "qwen3_prefill_S%d" % _S, M=_S, D=2048, dt="bf16", weighted=True, quant="block128", Hq=16, Hkv=8,
        hd=128, qk_norm=True, theta=1e6, positions="range", pos_start=0, capacity=1024, prefill=0, I=6144,
        act="silu", seed=2, outlier_frac=0.01)
for _M in (4096, 16384, 65536):
    WORKLOADS["large_m_M%d" % _M] = Workload(
        "large_m_M%d" % _M, M=_M, D=4096, dt="bf16", weighted=True, quant="static", Hq=32, Hkv=8, hd=128,
        qk_norm=True, theta=1e4, positions="unique_random", pos_start=0, capacity=131072, prefill=0,
        I=16384, act="relu2", seed=4)


def get(name: str, **overrides) -> Workload:
    wl = WORKLOADS[name]
    return replace(wl, **overrides) if overrides else wl


# ------------------------------------------------------------ primitives --
def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device)
    g.manual_seed(int(seed))
    return g


def normal16(shape: Tuple[int, ...], dt: str, g: torch.Generator, scale: float = 1.0,
             col_mult: Optional[torch.Tensor] = None) -> torch.Tensor:
    """N(0, scale^2) drawn in float32 then rounded to the 16-bit type.

    col_mult (float32 [shape[-1]]) multiplies columns before the rounding (used
    for the outlier channels)."""
    out = torch.empty(shape, dtype=DTYPES[dt], device=g.device)
    flat = out.view(-1, shape[-1]) if len(shape) > 1 else out.view(1, -1)
    rows = flat.shape[0]
    step = max(1, _CHUNK_ELEMS // max(1, flat.shape[1]))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        t = torch.randn((r1 - r0, flat.shape[1]), generator=g, dtype=torch.float32, device=g.device)
        if scale != 1.0:
            t.mul_(scale)
        if col_mult is not None:
            t.mul_(col_mult)
        flat[r0:r1].copy_(t)
    return out


def norm_weight(n: int, dt: str, g: torch.Generator) -> torch.Tensor:
    """A norm weight ~ 1 + 0.1 N(0, 1) (any +1 of the model already included)."""
    t = torch.randn((n,), generator=g, dtype=torch.float32, device=g.device).mul_(0.1).add_(1.0)
    return t.to(DTYPES[dt])


def outlier_multipliers(n: int, frac: float, mult: float, g: torch.Generator) -> Optional[torch.Tensor]:
    """float32 [n]: 1 everywhere except a seeded ceil(frac*n) channels at mult."""
    if frac <= 0.0:
        return None
    k = max(1, math.ceil(frac * n))
    idx = torch.randperm(n, generator=g, device=g.device)[:k]
    m = torch.ones(n, dtype=torch.float32, device=g.device)
    m[idx] = mult
    return m


def rope_tables(max_pos: int, hd: int, theta: float) -> Tuple[torch.Tensor, torch.Tensor]:
    """The precomputed RoPE table the caller passes in: angle(p, j) =
    p * theta^(-2j/hd), j < hd/2, evaluated in float64 and stored as float32
    [max_pos, hd/2] cos and sin tables."""
    half = hd // 2
    j = torch.arange(half, dtype=torch.float64)
    inv_freq = torch.pow(torch.tensor(float(theta), dtype=torch.float64), -2.0 * j / hd)
    p = torch.arange(max_pos, dtype=torch.float64)
    ang = torch.outer(p, inv_freq)
    return torch.cos(ang).to(torch.float32).contiguous(), torch.sin(ang).to(torch.float32).contiguous()


def positions(wl: Workload, g: torch.Generator) -> torch.Tensor:
    if wl.positions == "range":
        return torch.arange(wl.pos_start, wl.pos_start + wl.M, dtype=torch.int32, device=g.device)
    # unique slots sampled without replacement from the whole cache
    return torch.randperm(wl.capacity, generator=g, device=g.device)[: wl.M].to(torch.int32)


# ---------------------------------------------------------------- inputs --
@dataclass
class LayerInputs:
    """Host tensors for one layer invocation of the chain a -> b -> a -> c."""
    x_attn: torch.Tensor          # [M, D] stand-in attention-output (O-proj) rows
    x_ffn: torch.Tensor           # [M, D] stand-in FFN down-proj rows
    w_attn: Optional[torch.Tensor]  # [D] or None (`_noweight`)
    w_ffn: Optional[torch.Tensor]
    qkv: torch.Tensor             # [M, (Hq+2Hkv)*hd] stand-in QKV GEMM output
    q_norm_w: Optional[torch.Tensor]
    k_norm_w: Optional[torch.Tensor]
    gate_up: torch.Tensor         # [M, 2I] stand-in gate/up GEMM output, interleaved
    k_cache: torch.Tensor         # [capacity, Hkv, hd] initial cache contents
    v_cache: torch.Tensor


@dataclass
class Inputs:
    wl: Workload
    residual: torch.Tensor        # [M, D] initial residual stream
    positions: torch.Tensor       # int32 [M]
    cos: torch.Tensor             # float32 [max_pos, hd/2]
    sin: torch.Tensor
    layers: list = field(default_factory=list)


def make_inputs(wl: Workload, n_layers: Optional[int] = None, with_caches: bool = True,
                device="cpu") -> Inputs:
    """All inputs for ``n_layers`` (default wl.layers) distinct layers, drawn
    on ``device``."""
    g = generator(wl.seed, device)
    L = wl.layers if n_layers is None else n_layers
    col_d = outlier_multipliers(wl.D, wl.outlier_frac, wl.outlier_mult, g)
    col_i = outlier_multipliers(wl.I, wl.outlier_frac, wl.outlier_mult, g)
    col_gu = None if col_i is None else col_i.repeat_interleave(2)  # scale g and u of a channel
    residual = normal16((wl.M, wl.D), wl.dt, g, col_mult=col_d)
    pos = positions(wl, g)
    cos, sin = (t.to(g.device) for t in rope_tables(wl.max_pos, wl.hd, wl.theta))
    inp = Inputs(wl=wl, residual=residual, positions=pos, cos=cos, sin=sin)
    for _ in range(L):
        x_attn = normal16((wl.M, wl.D), wl.dt, g, col_mult=col_d)
        x_ffn = normal16((wl.M, wl.D), wl.dt, g, col_mult=col_d)
        w_attn = norm_weight(wl.D, wl.dt, g) if wl.weighted else None
        w_ffn = norm_weight(wl.D, wl.dt, g) if wl.weighted else None
        qkv = normal16((wl.M, wl.qkv_width), wl.dt, g)
        qw = norm_weight(wl.hd, wl.dt, g) if wl.qk_norm else None
        kw = norm_weight(wl.hd, wl.dt, g) if wl.qk_norm else None
        gate_up = normal16((wl.M, 2 * wl.I), wl.dt, g, col_mult=col_gu)
        if with_caches:
            kc = torch.empty((wl.capacity, wl.Hkv, wl.hd), dtype=DTYPES[wl.dt], device=g.device)
            vc = torch.empty((wl.capacity, wl.Hkv, wl.hd), dtype=DTYPES[wl.dt], device=g.device)
            if wl.prefill > 0:  # earlier tokens already in the cache
                kc[: wl.prefill] = normal16((wl.prefill, wl.Hkv, wl.hd), wl.dt, g)
                vc[: wl.prefill] = normal16((wl.prefill, wl.Hkv, wl.hd), wl.dt, g)
            # untouched slots carry a sentinel bit pattern (0x7E7E: finite in both types)
            kc[wl.prefill:].view(torch.int16).fill_(0x7E7E)
            vc[wl.prefill:].view(torch.int16).fill_(0x7E7E)
        else:
            kc = vc = None
        inp.layers.append(LayerInputs(x_attn, x_ffn, w_attn, w_ffn, qkv, qw, kw, gate_up, kc, vc))
    return inp


def bits16(t: torch.Tensor):
    """uint16 numpy bits of a 16-bit tensor, copied to the host (for the oracle)."""
    import numpy as np
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
