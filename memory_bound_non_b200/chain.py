"""Graphed layer chain: the fused ops of every layer x step in one CUDA graph.

Per layer invocation the chain runs the non-GEMM nodes of a transformer layer
("FlashRT kernel fusion", §二 table, steps 1, 3, 7 and 8-10):

    a  frt_residual_rmsnorm_fp8   attention-input norm (residual updated in place)
    b  frt_qkv_norm_rope_kvcache  QKV post-processing + KV-cache write
    a  frt_residual_rmsnorm_fp8   FFN-input norm (residual updated in place)
    c  frt_gate_act_fp8           gated activation + FP8

The GEMM outputs that feed these ops (attention output, QKV, down-proj, gate/up)
are fixed per-layer input buffers; the residual stream carries from one
invocation to the next.  ``layers x steps`` invocations (e.g. 18 x 10 for a
Pi0.5-like decoder, "FlashRT kernel fusion" §三) are captured once into a CUDA
graph and replayed with no host work in between, the way the decode loop of
"Falcon-Perception inference optimisation" (second technique) is replayed.

PyTorch only allocates the device buffers and owns the stream and the graph
object; every node of the graph is a libfrt kernel.
"""
from dataclasses import dataclass
from typing import List, Optional

import torch

from . import (chain_layer_table, frt_chain_persistent, frt_gate_act_fp8, frt_qkv_norm_rope_kvcache,
               frt_residual_rmsnorm_fp8)
from .workloads import Inputs, Workload


@dataclass
class DeviceLayer:
    x_attn: torch.Tensor
    x_ffn: torch.Tensor
    w_attn: Optional[torch.Tensor]
    w_ffn: Optional[torch.Tensor]
    qkv: torch.Tensor
    q_norm_w: Optional[torch.Tensor]
    k_norm_w: Optional[torch.Tensor]
    gate_up: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    q8_attn: torch.Tensor
    q8_ffn: torch.Tensor
    q_out: torch.Tensor
    act8: torch.Tensor
    bs_attn: Optional[torch.Tensor]
    bs_ffn: Optional[torch.Tensor]
    bs_act: Optional[torch.Tensor]


def _dev(t, device):
    return None if t is None else t.to(device, non_blocking=False).contiguous()


class LayerChain:
    """Device-resident buffers for ``layers`` layers and the chain over them."""

    def __init__(self, wl: Workload, inp: Inputs, scales=None, device="cuda"):
        self.wl = wl
        self.device = torch.device(device)
        self.residual0 = _dev(inp.residual, self.device)
        self.residual = self.residual0.clone()
        self.positions = _dev(inp.positions, self.device)
        self.cos = _dev(inp.cos, self.device)
        self.sin = _dev(inp.sin, self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        # static per-tensor scales for the three FP8 sites (attn norm, ffn norm, act)
        self.scales = torch.ones(3, dtype=torch.float32, device=self.device)
        if scales is not None:
            self.scales.copy_(torch.as_tensor(scales, dtype=torch.float32))
        block = wl.quant == "block128"
        nbd, nbi = (wl.D + 127) // 128, (wl.I + 127) // 128
        u8 = dict(dtype=torch.uint8, device=self.device)
        f32 = dict(dtype=torch.float32, device=self.device)
        self.layers: List[DeviceLayer] = []
        for L in inp.layers:
            self.layers.append(DeviceLayer(
                x_attn=_dev(L.x_attn, self.device), x_ffn=_dev(L.x_ffn, self.device),
                w_attn=_dev(L.w_attn, self.device), w_ffn=_dev(L.w_ffn, self.device),
                qkv=_dev(L.qkv, self.device), q_norm_w=_dev(L.q_norm_w, self.device),
                k_norm_w=_dev(L.k_norm_w, self.device), gate_up=_dev(L.gate_up, self.device),
                k_cache=_dev(L.k_cache, self.device), v_cache=_dev(L.v_cache, self.device),
                q8_attn=torch.empty((wl.M, wl.D), **u8), q8_ffn=torch.empty((wl.M, wl.D), **u8),
                q_out=torch.empty((wl.M, wl.Hq, wl.hd), dtype=L.qkv.dtype, device=self.device),
                act8=torch.empty((wl.M, wl.I), **u8),
                bs_attn=torch.empty((wl.M, nbd), **f32) if block else None,
                bs_ffn=torch.empty((wl.M, nbd), **f32) if block else None,
                bs_act=torch.empty((wl.M, nbi), **f32) if block else None))
        self.graph = None

    # ------------------------------------------------------------ ops --
    def attn_norm(self, l, stream=None):
        wl, L = self.wl, self.layers[l]
        frt_residual_rmsnorm_fp8(L.x_attn, self.residual, self.residual, L.w_attn, L.q8_attn,
                                 static_scale=self.scales[0:1], block_scales=L.bs_attn, eps=wl.eps,
                                 quant=wl.quant, stream=stream)

    def qkv(self, l, stream=None):
        wl, L = self.wl, self.layers[l]
        frt_qkv_norm_rope_kvcache(L.qkv, L.q_norm_w, L.k_norm_w, self.cos, self.sin, self.positions, L.q_out,
                                  L.k_cache, L.v_cache, wl.Hq, wl.Hkv, wl.hd, status=self.status, eps=wl.eps,
                                  stream=stream)

    def ffn_norm(self, l, stream=None):
        wl, L = self.wl, self.layers[l]
        frt_residual_rmsnorm_fp8(L.x_ffn, self.residual, self.residual, L.w_ffn, L.q8_ffn,
                                 static_scale=self.scales[1:2], block_scales=L.bs_ffn, eps=wl.eps,
                                 quant=wl.quant, stream=stream)

    def gate(self, l, stream=None):
        wl, L = self.wl, self.layers[l]
        frt_gate_act_fp8(L.gate_up, L.act8, static_scale=self.scales[2:3], block_scales=L.bs_act, act=wl.act,
                         quant=wl.quant, stream=stream)

    def layer(self, l, stream=None):
        self.attn_norm(l, stream)
        self.qkv(l, stream)
        self.ffn_norm(l, stream)
        self.gate(l, stream)

    def run(self, steps=None, stream=None):
        """Launch the whole chain in stream order (no graph)."""
        for _ in range(self.wl.steps if steps is None else steps):
            for l in range(len(self.layers)):
                self.layer(l, stream)

    def run_persistent(self, steps=None, stream=None):
        """The same chain as one persistent kernel launch (one CTA per row runs
        the row's steps x layers x 4 ops; see frt_chain_persistent)."""
        wl = self.wl
        if getattr(self, "_table", None) is None:
            self._table = chain_layer_table(self.layers, self.device)
        frt_chain_persistent(self._table, len(self.layers), wl.steps if steps is None else steps, self.residual,
                             self.cos, self.sin, self.positions, self.scales, self.status, wl.Hq, wl.Hkv, wl.hd, wl.I,
                             self.layers[0].k_cache.shape[0], eps=wl.eps, quant=wl.quant, act=wl.act, stream=stream)

    def capture_persistent(self, steps=None):
        """One-node CUDA graph of the persistent chain (warmed up once first)."""
        self.run_persistent(steps=1)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run_persistent(steps=steps)
        self.graph_persistent = g
        return g

    @property
    def launches_per_chain(self) -> int:
        return 4 * len(self.layers) * self.wl.steps

    # ---------------------------------------------------------- graph --
    def capture(self, steps=None):
        """Capture steps x layers invocations into one CUDA graph.  The chain is
        launched once eagerly first (module load / warm-up), so the residual and
        the outputs should be reset by the caller before relying on them."""
        s = torch.cuda.Stream(device=self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self.run(steps=1)
        torch.cuda.current_stream(self.device).wait_stream(s)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run(steps=steps)
        self.graph = g
        return g

    def replay(self):
        self.graph.replay()

    def reset(self):
        """Restore the initial residual and clear the status word."""
        self.residual.copy_(self.residual0)
        self.status.zero_()

    # ---------------------------------------------------- calibration --
    def calibrate_static_scales(self):
        """Static scale = amax / 448 of each FP8 site's output on the first
        invocation, measured with the block-128 mode of the same kernels (the
        largest block scale is the tensor's amax / 448).  Leaves the residual
        at its initial value."""
        wl, L = self.wl, self.layers[0]
        nbd, nbi = (wl.D + 127) // 128, (wl.I + 127) // 128
        r = self.residual0.clone()
        q8 = torch.empty((wl.M, wl.D), dtype=torch.uint8, device=self.device)
        bs = torch.empty((wl.M, nbd), dtype=torch.float32, device=self.device)
        frt_residual_rmsnorm_fp8(L.x_attn, r, r, L.w_attn, q8, block_scales=bs, eps=wl.eps, quant="block128")
        s_attn = bs.max()
        frt_residual_rmsnorm_fp8(L.x_ffn, r, r, L.w_ffn, q8, block_scales=bs, eps=wl.eps, quant="block128")
        s_ffn = bs.max()
        a8 = torch.empty((wl.M, wl.I), dtype=torch.uint8, device=self.device)
        bsi = torch.empty((wl.M, nbi), dtype=torch.float32, device=self.device)
        frt_gate_act_fp8(L.gate_up, a8, block_scales=bsi, act=wl.act, quant="block128")
        s_act = bsi.max()
        self.scales.copy_(torch.stack([s_attn, s_ffn, s_act]))
        return self.scales
