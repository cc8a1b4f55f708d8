#!/usr/bin/env python
"""Benchmark of the fused non-GEMM layer chain on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload large_m_M65536] [--no-chain] [--no-e2e] [--no-cpu]

One step = one pass of the whole hot path over one batch: the four fused-op
launches of a layer (attention-input residual+RMSNorm+FP8, QKV
norm+RoPE+KV-cache write, FFN-input residual+RMSNorm+FP8, gated activation +
FP8) on the large-M workload (M=65536 tokens, D=4096, 32/8 heads of 128,
squared-ReLU FFN with I=16384, 131072-slot KV cache): about 10.8 GB of
algorithmic HBM traffic per step, far larger than L2.  `value` is the
achieved HBM bandwidth of the step (algorithmic bytes / device time, summed
over ranks / max over ranks).

Also reported on the same JSON line:
  per_op        each op's CUDA-event time inside the timed steps, GB/s and
                fraction of the measured HBM copy peak and of 8 TB/s;
  roofline      the dominant kernel (gated activation) against the HBM peak;
  chain         microseconds per graphed layer chain: the Pi0.5-like decoder
                (18 layers x 10 steps = 720 nodes) and the VLA denoise loop
                (32 x 10 = 1280 nodes), each one CUDA graph, L2 flushed
                between replays; per-node cost against the launch floor;
                and the same chain as one persistent kernel ("persistent");
  launch_floor  an empty kernel per stream launch and per graph node;
  small_m       per-op microseconds at M <= 41 against the launch floor;
  next_ops      the widened ops timed alone (gated residual + AdaRMSNorm +
                FP8 at 65536 x 4096 and at the Pi0.5 action-expert shape);
  e2e           the same step through the public API with pinned host
                buffers: host->device copy of the step's inputs, the four ops,
                device->host copy of the step's outputs;
  clocks        nvidia-smi SM clock and throttle reasons sampled while timing;
  parity        the step's four ops on the GPU for the CPU leg's row sample
                against the oracle outputs of the same rows (residual and V
                bit-exact, Q/K within the 16-bit tolerance, FP8 codes at most
                one step off on at most 0.1 %);
  cpu_baseline  the CPU oracle (single thread) on a bounded row sample;
                cpu_baseline_all_cores the same oracle in one spawned process
                per host core, each on its own row block.

Multi-GPU (torchrun): each rank runs its own row shard (weak scaling, no
collective on the data path); timing is max over ranks.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "achieved HBM GB/s (% of roofline) per fused op; µs per graphed layer chain"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 512 << 20


# ---------------------------------------------------------------- helpers --
def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=500)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="large_m_M65536")
    p.add_argument("--no-chain", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-parity", action="store_true",
                   help="skip comparing the GPU step on the CPU leg's row sample with the oracle outputs")
    p.add_argument("--e2e-steps", type=int, default=5)
    p.add_argument("--chain-reps", type=int, default=30)
    p.add_argument("--json-out", default=None)
    p.add_argument("--next-only", action="store_true",
                   help="time only the widened ops (gated residual + AdaRMSNorm + FP8) and print their JSON")
    p.add_argument("--next-m", type=int, default=65536, help="rows of the large widened-op case")
    p.add_argument("--next-reps", type=int, default=50)
    p.add_argument("--table", action="store_true",
                   help="per-op GPU and CPU-oracle microseconds on every named workload (one JSON object per row)")
    p.add_argument("--persistent-chain", default=None, metavar="WORKLOAD",
                   help="only run the named chain (e.g. pi05) as one persistent kernel, --chain-reps times")
    return p.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class Dist:
    """Process-group plumbing of a multi-rank run (one process per GPU): a
    barrier and a max over ranks.  Single-process runs need no group."""

    def __init__(self, world, backend="nccl", device=None, timeout_s=120):
        self.world = world
        self.pg = None
        self.device = device
        if world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
            if backend == "nccl" and device is not None:
                kw["device_id"] = device
            dist.init_process_group(backend, **kw)
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max_over_ranks(self, x):
        if self.pg is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device if self.device is not None else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.barrier()
            self.pg.destroy_process_group()
            self.pg = None


def rank_workload(wl, rank):
    """Each rank draws its own row shard: same shapes, seed offset by rank
    (weak scaling: per-rank work is fixed as ranks are added)."""
    import dataclasses
    return dataclasses.replace(wl, seed=wl.seed + 1000 * rank, layers=1, steps=1)


def job_throughput(bytes_per_rank, world, ms_per_step_max):
    """Whole-job GB/s: bytes all ranks moved / the slowest rank's time."""
    return bytes_per_rank * world / (ms_per_step_max * 1e-3) / 1e9


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def op_bytes(wl):
    """Algorithmic HBM bytes of one call of each op (what it must move).
    a: x, residual in, residual out (2 B each), FP8 out (1 B), + weight,
       + scales; b: qkv read + Q/K/V written (2 B each), the token's cos and
       sin rows (4 B x hd/2 x 2), its position, + q/k norm weights;
    c: gate/up read (2 x 2 B per output), FP8 out (1 B), + scales."""
    M, D, I, hd = wl.M, wl.D, wl.I, wl.hd
    nbd, nbi = (D + 127) // 128, (I + 127) // 128
    width = (wl.Hq + 2 * wl.Hkv) * hd
    a = M * D * 7 + (2 * D if wl.weighted else 0) + (4 * M * nbd if wl.quant == "block128" else 4)
    b = M * width * 4 + M * hd * 4 + 4 * M + (4 * hd if wl.qk_norm else 0)
    c = M * I * 5 + (4 * M * nbi if wl.quant == "block128" else 4)
    return {"attn_norm": a, "qkv": b, "ffn_norm": a, "gate": c}


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampling in the background."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device=0):
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            pass
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                if self.uuid and self.uuid not in parts[0] and parts[0] not in self.uuid:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        busy = [r for r in rows if (num(r[4]) or 0) >= 50] or rows
        sm = [num(r[1]) for r in busy if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][2]),
                "reasons": reasons, "samples": len(rows), "samples_busy": len(busy),
                "power_w_max": max((num(r[3]) or 0) for r in rows)}


# Sources a traffic record depends on: the kernel's own file and the shared
# device and host headers.
SHARED_SOURCES = ("frt_device.cuh", "frt_host.h")
KERNEL_SOURCE = {"attn_norm": "residual_rmsnorm_fp8.cu", "ffn_norm": "residual_rmsnorm_fp8.cu",
                 "qkv": "qkv_norm_rope_kvcache.cu", "gate": "gate_act_fp8.cu",
                 "gate_residual_adarms": "gate_residual_adarms_fp8.cu", "qkv_prepq": "qkv_norm_rope_kvcache.cu",
                 "residual_rmsnorm_nvfp4": "residual_rmsnorm_fp8.cu", "gate_act_nvfp4": "gate_act_fp8.cu",
                 "residual_layernorm": "residual_rmsnorm_fp8.cu", "qkv_layernorm": "qkv_norm_rope_kvcache.cu"}


def source_hashes():
    """sha256 of each CUDA source file: ties a recorded ncu traffic figure to
    the kernel it was measured on."""
    import glob
    import hashlib
    out = {}
    csrc = os.path.join(ROOT, "memory_bound_non_b200", "csrc")
    for path in sorted(glob.glob(os.path.join(csrc, "*"))):
        if path.endswith((".cu", ".cuh", ".h")):
            with open(path, "rb") as f:
                out[os.path.basename(path)] = hashlib.sha256(f.read()).hexdigest()
    return out


def _traffic_sources(workload, op):
    """The source files behind one traffic record: `op` names the kernel for
    the step's ops, the workload key does for the widened ops."""
    kernel = KERNEL_SOURCE.get(op)
    for prefix in ("gate_residual_adarms", "qkv_prepq", "residual_rmsnorm_nvfp4", "gate_act_nvfp4",
                   "residual_layernorm", "qkv_layernorm"):
        if workload.startswith(prefix):
            kernel = KERNEL_SOURCE[prefix]
    return (kernel,) + SHARED_SOURCES if kernel else None


def measured_traffic(workload, op):
    """DRAM bytes per launch (read + write) of `op` on `workload` from the
    committed ncu record, or None when its kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    files = _traffic_sources(workload, op)
    recorded = rec.get("source_sha256", {})
    now = source_hashes()
    if files is None or any(recorded.get(f) is None or recorded.get(f) != now.get(f) for f in files):
        return None
    v = rec.get("per_launch_bytes", {}).get(workload, {}).get(op)
    return int(v) if v is not None else None


def flush_l2(buf):
    buf.zero_()


def time_graph(graph, reps, flush_buf, stream):
    """Median and mean device time of one replay, L2 flushed before each."""
    times = []
    for _ in range(reps):
        flush_l2(flush_buf)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    return statistics.median(times), times


# ------------------------------------------------------------- GPU legs --
def launch_floor(reps=2000):
    """Empty-kernel floor, with the library's current PDL setting."""
    import memory_bound_non_b200 as frt
    s = torch.cuda.current_stream()
    for _ in range(50):
        frt.frt_noop(1, 32)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        frt.frt_noop(1, 32)
    e1.record(s)
    e1.synchronize()
    per_launch = e0.elapsed_time(e1) * 1e3 / reps
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(s)
    with torch.cuda.stream(side):
        frt.frt_noop(1, 32)
    s.wait_stream(side)
    with torch.cuda.graph(g):
        for _ in range(1000):
            frt.frt_noop(1, 32)
    g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(20):
        e0.record(s)
        g.replay()
        e1.record(s)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3 / 1000)
    del g
    return {"stream_launch_us": per_launch, "graph_node_us": statistics.median(ts),
            "kernel": "frt_noop <<<1, 32>>>"}


def small_m_ops(floor, reps=400):
    """Per-op us at M <= 41: back-to-back stream launches and graph nodes,
    against the empty-kernel floor and against the dependent-copy floor (a
    graph of in-place row copies of the residual, [M, D] 16-bit: one
    dependent load and store per node, what any op whose input is its
    predecessor's output pays at least)."""
    import memory_bound_non_b200 as frt
    from memory_bound_non_b200 import workloads as W
    from memory_bound_non_b200.chain import LayerChain
    out = {}
    s = torch.cuda.current_stream()
    for name in ("tiny", "pi05", "vla_denoise"):
        wl = W.get(name, layers=1, steps=1)
        ch = LayerChain(wl, W.make_inputs(wl, n_layers=1))
        ch.calibrate_static_scales()
        res = {}
        buf = ch.residual.clone()
        for op in ("dep_copy", "attn_norm", "qkv", "gate"):
            fn = (lambda _l: frt.frt_copy_rows(buf, buf)) if op == "dep_copy" else getattr(ch, op)
            for _ in range(20):
                fn(0)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(reps):
                fn(0)
            e1.record(s)
            e1.synchronize()
            stream_us = e0.elapsed_time(e1) * 1e3 / reps
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(200):
                    fn(0)
            g.replay()
            torch.cuda.synchronize()
            ts = []
            for _ in range(10):
                e0.record(s)
                g.replay()
                e1.record(s)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3 / 200)
            del g
            node_us = statistics.median(ts)
            res[op] = {"stream_us": round(stream_us, 3), "graph_node_us": round(node_us, 3),
                       "x_stream_floor": round(stream_us / floor["stream_launch_us"], 3),
                       "x_graph_floor": round(node_us / floor["graph_node_us"], 3)}
            if op != "dep_copy":
                res[op]["x_dep_copy_floor"] = round(node_us / res["dep_copy"]["graph_node_us"], 3)
        out[name] = res
    return out


def next_ops_leg(peak, floor, reps=50, big_m=65536):
    """The widened ops, timed alone: NEXT-1 (gated residual + AdaRMSNorm + FP8)
    at big_m x 4096 bf16 with one condition row per 1024 rows (inputs larger
    than L2 at the default 65536), static and block-128 scales, and at the
    Pi0.5 action-expert shape (10 x 1024) as a graph node."""
    import memory_bound_non_b200 as frt
    from memory_bound_non_b200 import workloads as W
    out = {}
    s = torch.cuda.current_stream()
    for M, D, rpc, quant in ((big_m, 4096, 1024, "static"), (big_m, 4096, 1024, "block128"),
                             (10, 1024, 10, "static")):
        g = W.generator(61, "cuda")
        nc = (M + rpc - 1) // rpc
        x = W.normal16((M, D), "bf16", g)
        r = W.normal16((M, D), "bf16", g, scale=2.0)
        gate = W.normal16((nc, D), "bf16", g, scale=0.5)
        sc = W.normal16((nc, D), "bf16", g, scale=0.2)
        sh = W.normal16((nc, D), "bf16", g, scale=0.2)
        q = torch.empty((M, D), dtype=torch.uint8, device="cuda")
        ss = torch.tensor([0.02], dtype=torch.float32, device="cuda")
        bs = torch.empty((M, (D + 127) // 128), dtype=torch.float32, device="cuda")

        def op():
            if quant == "static":
                frt.frt_gate_residual_adarms_fp8(x, gate, r, r, sc, sh, q, static_scale=ss, rows_per_cond=rpc)
            else:
                frt.frt_gate_residual_adarms_fp8(x, gate, r, r, sc, sh, q, block_scales=bs, rows_per_cond=rpc,
                                                 quant="block128")
        nbytes = M * D * 7 + nc * D * 6 + (bs.numel() * 4 if quant == "block128" else 0)
        for _ in range(5):
            op()
        torch.cuda.synchronize()
        key = "gate_residual_adarms_M%d_D%d_%s" % (M, D, quant)
        if M > 1024:
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps)]
            for i in range(reps):
                ev[2 * i].record(s)
                op()
                ev[2 * i + 1].record(s)
            torch.cuda.synchronize()
            ts = [ev[2 * i].elapsed_time(ev[2 * i + 1]) * 1e3 for i in range(reps)]
            us = sum(ts) / len(ts)
            gbs = nbytes / (us * 1e-6) / 1e9
            out[key] = {"us_mean": round(us, 2), "us_median": round(statistics.median(ts), 2), "bytes": nbytes,
                        "GBps": round(gbs, 1), "frac_of_measured": round(gbs / peak, 4),
                        "frac_of_8TBps": round(gbs / NOMINAL_HBM_GBS, 4),
                        "l2": "inputs larger than L2" if nbytes > (252 << 20) else "fits in L2",
                        "traffic": measured_traffic(key, "gate_residual_adarms")}
        else:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                for _ in range(200):
                    op()
            gr.replay()
            torch.cuda.synchronize()
            ts = []
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for _ in range(10):
                e0.record(s)
                gr.replay()
                e1.record(s)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3 / 200)
            del gr
            node = statistics.median(ts)
            out[key] = {"graph_node_us": round(node, 3), "x_graph_floor": round(node / floor["graph_node_us"], 3)}
        del x, r, gate, sc, sh, q, bs
    # NEXT-2: the QKV op with the Q epilogue (softmax scale, head-major Q) and
    # an e4m3 KV cache, on the large-M QKV shape (32 q / 8 kv heads of 128).
    wl = W.get("large_m_M65536", M=big_m)
    g = W.generator(62, "cuda")
    H, hd = wl.Hq + 2 * wl.Hkv, wl.hd
    qkv = W.normal16((big_m, H * hd), "bf16", g)
    qw, kw = W.norm_weight(hd, "bf16", g), W.norm_weight(hd, "bf16", g)
    cos, sin = W.rope_tables(wl.capacity, hd, wl.theta)
    cos, sin = cos.cuda(), sin.cuda()
    pos = W.positions(wl, g)
    q_out = torch.empty((wl.Hq, big_m, hd), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((wl.capacity, wl.Hkv, hd), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    kvs = torch.tensor([0.02, 0.015], dtype=torch.float32, device="cuda")
    qs = float(1.0 / np.sqrt(hd))

    def qop():
        frt.frt_qkv_norm_rope_prepq_kvcache(qkv, qw, kw, cos, sin, pos, q_out, kc, vc, wl.Hq, wl.Hkv, hd,
                                            q_scale=qs, q_layout="head", kv="e4m3", kv_scales=kvs, eps=wl.eps)
    nbytes = big_m * (H * hd * 2 + wl.Hq * hd * 2 + 2 * wl.Hkv * hd + hd * 4 + 4) + 2 * hd * 2
    for _ in range(5):
        qop()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps)]
    for i in range(reps):
        ev[2 * i].record(s)
        qop()
        ev[2 * i + 1].record(s)
    torch.cuda.synchronize()
    ts = [ev[2 * i].elapsed_time(ev[2 * i + 1]) * 1e3 for i in range(reps)]
    us = sum(ts) / len(ts)
    gbs = nbytes / (us * 1e-6) / 1e9
    key = "qkv_prepq_e4m3_M%d" % big_m
    out[key] = {"us_mean": round(us, 2), "us_median": round(statistics.median(ts), 2), "bytes": nbytes,
                "GBps": round(gbs, 1), "frac_of_measured": round(gbs / peak, 4),
                "frac_of_8TBps": round(gbs / NOMINAL_HBM_GBS, 4), "q_layout": "head-major", "kv": "e4m3",
                "traffic": measured_traffic(key, "qkv_prepq")}
    del qkv, q_out, kc, vc
    # NEXT-3: the NVFP4 producers on the large-M shapes (norm 65536 x 4096,
    # gated activation 65536 x 16384 squared ReLU), row-major scale factors.
    g = W.generator(63, "cuda")
    D, I = wl.D, wl.I
    x = W.normal16((big_m, D), "bf16", g)
    r = W.normal16((big_m, D), "bf16", g)
    w = W.norm_weight(D, "bf16", g)
    q = torch.empty((big_m, D // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((big_m * D // 16,), dtype=torch.uint8, device="cuda")
    gsd = torch.tensor([0.0015], dtype=torch.float32, device="cuda")
    cases = [("residual_rmsnorm_nvfp4_M%d_D%d" % (big_m, D), big_m * D * 6.5 + big_m * D // 16 + 2 * D,
              lambda: frt.frt_residual_rmsnorm_nvfp4(x, r, r, w, q, sf, gsd))]
    gu = W.normal16((big_m, 2 * I), "bf16", g)
    qc = torch.empty((big_m, I // 2), dtype=torch.uint8, device="cuda")
    sfc = torch.empty((big_m * I // 16,), dtype=torch.uint8, device="cuda")
    cases.append(("gate_act_nvfp4_relu2_M%d_I%d" % (big_m, I), big_m * I * 4.5 + big_m * I // 16,
                  lambda: frt.frt_gate_act_nvfp4(gu, qc, sfc, gsd, act="relu2")))
    for key, nbytes, fn in cases:
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps)]
        for i in range(reps):
            ev[2 * i].record(s)
            fn()
            ev[2 * i + 1].record(s)
        torch.cuda.synchronize()
        ts = [ev[2 * i].elapsed_time(ev[2 * i + 1]) * 1e3 for i in range(reps)]
        us = sum(ts) / len(ts)
        gbs = nbytes / (us * 1e-6) / 1e9
        out[key] = {"us_mean": round(us, 2), "us_median": round(statistics.median(ts), 2), "bytes": int(nbytes),
                    "GBps": round(gbs, 1), "frac_of_measured": round(gbs / peak, 4),
                    "frac_of_8TBps": round(gbs / NOMINAL_HBM_GBS, 4), "sf_layout": "rows",
                    "traffic": measured_traffic(key, "nvfp4")}
    del q, sf, gu, qc, sfc
    # NEXT-4: the LayerNorm producer (weight + bias, static FP8) on the norm
    # shape, and the per-head LayerNorm(Q/K) + RoPE op on the QKV shape.
    bvec = W.normal16((D,), "bf16", g, scale=0.2)
    q8 = torch.empty((big_m, D), dtype=torch.uint8, device="cuda")
    ss8 = torch.tensor([0.02], dtype=torch.float32, device="cuda")
    H, hd = wl.Hq + 2 * wl.Hkv, wl.hd
    qkv = W.normal16((big_m, H * hd), "bf16", g)
    qlw, qlb = W.normal16((wl.Hq, hd), "bf16", g), W.normal16((wl.Hq, hd), "bf16", g, scale=0.1)
    klw, klb = W.normal16((wl.Hkv, hd), "bf16", g), W.normal16((wl.Hkv, hd), "bf16", g, scale=0.1)
    cos, sin = W.rope_tables(wl.capacity, hd, wl.theta)
    cos, sin = cos.cuda(), sin.cuda()
    pos = W.positions(wl, g)
    q_out = torch.empty((big_m, wl.Hq, hd), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((wl.capacity, wl.Hkv, hd), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    cases = [("residual_layernorm_fp8_M%d_D%d" % (big_m, D), big_m * D * 7 + 4 * D,
              lambda: frt.frt_residual_layernorm_fp8(x, r, r, w, bvec, q8, static_scale=ss8)),
             ("qkv_layernorm_rope_M%d" % big_m, big_m * (H * hd * 4 + hd * 4 + 4) + 4 * (wl.Hq + wl.Hkv) * hd,
              lambda: frt.frt_qkv_layernorm_rope_kvcache(qkv, qlw, qlb, klw, klb, cos, sin, pos, q_out, kc, vc,
                                                         wl.Hq, wl.Hkv, hd))]
    for key, nbytes, fn in cases:
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps)]
        for i in range(reps):
            ev[2 * i].record(s)
            fn()
            ev[2 * i + 1].record(s)
        torch.cuda.synchronize()
        ts = [ev[2 * i].elapsed_time(ev[2 * i + 1]) * 1e3 for i in range(reps)]
        us = sum(ts) / len(ts)
        gbs = nbytes / (us * 1e-6) / 1e9
        out[key] = {"us_mean": round(us, 2), "us_median": round(statistics.median(ts), 2), "bytes": int(nbytes),
                    "GBps": round(gbs, 1), "frac_of_measured": round(gbs / peak, 4),
                    "frac_of_8TBps": round(gbs / NOMINAL_HBM_GBS, 4), "traffic": measured_traffic(key, "layernorm")}
    del x, r, q8, qkv, q_out, kc, vc
    return out


def chain_leg(reps, floor):
    from memory_bound_non_b200 import workloads as W
    from memory_bound_non_b200.chain import LayerChain
    out = {}
    s = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    for name in ("pi05", "vla_denoise"):
        wl = W.get(name)
        ch = LayerChain(wl, W.make_inputs(wl))
        ch.calibrate_static_scales()
        ch.capture()
        for _ in range(3):
            ch.replay()
        torch.cuda.synchronize()
        med, ts = time_graph(ch.graph, reps, flush, s)
        # back-to-back replays (warm L2), for reference
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(reps):
            ch.replay()
        e1.record(s)
        e1.synchronize()
        warm = e0.elapsed_time(e1) * 1e3 / reps
        nodes = ch.launches_per_chain
        b = op_bytes(wl)
        chain_bytes = sum(b.values()) * wl.layers * wl.steps
        out[name] = {"layers": wl.layers, "steps": wl.steps, "nodes": nodes, "us_per_chain": round(med, 2),
                     "us_per_chain_warm_l2": round(warm, 2), "us_per_layer": round(med / (wl.layers * wl.steps), 3),
                     "us_per_node": round(med / nodes, 3),
                     "x_graph_node_floor": round(med / nodes / floor["graph_node_us"], 3),
                     "hbm_bytes_per_chain": chain_bytes,
                     "hbm_us_at_8TBps": round(chain_bytes / NOMINAL_HBM_GBS / 1e3, 2),
                     "l2": "flushed before each replay (512 MiB write)"}
        # the same chain as one persistent kernel (one launch per chain)
        gp = ch.capture_persistent()
        for _ in range(3):
            gp.replay()
        torch.cuda.synchronize()
        pmed, _ = time_graph(gp, reps, flush, s)
        out[name]["persistent"] = {"us_per_chain": round(pmed, 2), "launches": 1,
                                   "us_per_op": round(pmed / nodes, 3),
                                   "x_graph_node_floor": round(pmed / nodes / floor["graph_node_us"], 3),
                                   "speedup_vs_graph": round(med / pmed, 2),
                                   "l2": "flushed before each replay (512 MiB write)"}
        del ch, gp
    return out


# ------------------------------------------------------------ large-M step --
class Step:
    """Device buffers of one layer at the bench workload, and its four ops."""

    def __init__(self, wl, rank):
        from memory_bound_non_b200 import workloads as W
        from memory_bound_non_b200.chain import LayerChain
        wl_r = rank_workload(wl, rank)
        self.wl = wl_r
        t0 = time.time()
        self.host = W.make_inputs(wl_r, n_layers=1, device="cuda")  # seeded device generator
        self.gen_s = time.time() - t0
        self.chain = LayerChain(wl_r, self.host)
        self.chain.calibrate_static_scales()
        self.ops = [("attn_norm", self.chain.attn_norm), ("qkv", self.chain.qkv),
                    ("ffn_norm", self.chain.ffn_norm), ("gate", self.chain.gate)]

    def run(self):
        for _, fn in self.ops:
            fn(0)


def timed_step_leg(step, K, W_, barrier):
    s = torch.cuda.current_stream()
    for _ in range(W_):
        step.run()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    nops = len(step.ops)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nops + 1)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s)
    for k in range(K):
        ev[k][0].record(s)
        for i, (_, fn) in enumerate(step.ops):
            fn(0)
            ev[k][i + 1].record(s)
    end.record(s)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    total_ms = start.elapsed_time(end)
    per_op = {}
    for i, (name, _) in enumerate(step.ops):
        per_op[name] = [ev[k][i].elapsed_time(ev[k][i + 1]) * 1e3 for k in range(K)]
    return total_ms, per_op


def run_rows(ch, r0, r1, stream):
    """The step's four ops on token rows [r0, r1) (every op is row-independent)."""
    import memory_bound_non_b200 as frt
    wl, L = ch.wl, ch.layers[0]
    frt.frt_residual_rmsnorm_fp8(L.x_attn[r0:r1], ch.residual[r0:r1], ch.residual[r0:r1], L.w_attn,
                                 L.q8_attn[r0:r1], static_scale=ch.scales[0:1], eps=wl.eps, quant=wl.quant,
                                 stream=stream)
    frt.frt_qkv_norm_rope_kvcache(L.qkv[r0:r1], L.q_norm_w, L.k_norm_w, ch.cos, ch.sin, ch.positions[r0:r1],
                                  L.q_out[r0:r1], L.k_cache, L.v_cache, wl.Hq, wl.Hkv, wl.hd, status=ch.status,
                                  eps=wl.eps, stream=stream)
    frt.frt_residual_rmsnorm_fp8(L.x_ffn[r0:r1], ch.residual[r0:r1], ch.residual[r0:r1], L.w_ffn,
                                 L.q8_ffn[r0:r1], static_scale=ch.scales[1:2], eps=wl.eps, quant=wl.quant,
                                 stream=stream)
    frt.frt_gate_act_fp8(L.gate_up[r0:r1], L.act8[r0:r1], static_scale=ch.scales[2:3], act=wl.act,
                         quant=wl.quant, stream=stream)


def e2e_leg(step, K, W_, chunks=8):
    """Public-API step with host buffers: the step's inputs are copied from
    pinned host memory and its outputs copied back inside the timed region.
    Rows are cut into `chunks` pieces pipelined over three streams (copy in,
    compute, copy out), so the transfers overlap each other and the kernels."""
    ch = step.chain
    L, H = ch.layers[0], step.host
    hl = H.layers[0]
    ins = [(hl.x_attn, L.x_attn), (H.residual, ch.residual), (hl.qkv, L.qkv), (H.positions, ch.positions),
           (hl.x_ffn, L.x_ffn), (hl.gate_up, L.gate_up)]
    ins = [(torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t), d) for t, d in ins]
    outs = [(d, torch.empty(d.shape, dtype=d.dtype, pin_memory=True))
            for d in (L.q8_attn, L.q_out, ch.residual, L.q8_ffn, L.act8)]
    h2d = sum(h.numel() * h.element_size() for h, _ in ins)
    d2h = sum(h.numel() * h.element_size() for _, h in outs)
    M = ch.wl.M
    bounds = [(M * i // chunks, M * (i + 1) // chunks) for i in range(chunks)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()

    def one():
        for s in (s_in, s_comp, s_out):
            s.wait_stream(main)
        done = []
        for r0, r1 in bounds:
            with torch.cuda.stream(s_in):
                for h, d in ins:
                    d[r0:r1].copy_(h[r0:r1], non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            s_comp.wait_event(e_in)
            run_rows(ch, r0, r1, s_comp)
            e_c = torch.cuda.Event()
            e_c.record(s_comp)
            s_out.wait_event(e_c)
            with torch.cuda.stream(s_out):
                for d, h in outs:
                    h[r0:r1].copy_(d[r0:r1], non_blocking=True)
        for s in (s_in, s_comp, s_out):
            main.wait_stream(s)

    for _ in range(W_):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for _ in range(K):
        one()
    e1.record(main)
    e1.synchronize()
    return e0.elapsed_time(e1) / K, h2d, d2h


# -------------------------------------------------------------- CPU legs --
def oracle_sample(wl, host, rows, keep=None):
    """Run the oracle on the first `rows` rows of every op of the step.
    Returns seconds; with `keep` (a dict) the outputs are stored in it."""
    import oracle
    from memory_bound_non_b200 import workloads as W
    hl = host.layers[0]
    x_a, x_f = W.bits16(hl.x_attn[:rows]), W.bits16(hl.x_ffn[:rows])
    r = W.bits16(host.residual[:rows])
    wa = None if hl.w_attn is None else W.bits16(hl.w_attn)
    wf = None if hl.w_ffn is None else W.bits16(hl.w_ffn)
    qkv = W.bits16(hl.qkv[:rows])
    qw = None if hl.q_norm_w is None else W.bits16(hl.q_norm_w)
    kw = None if hl.k_norm_w is None else W.bits16(hl.k_norm_w)
    gu = W.bits16(hl.gate_up[:rows])
    pos = host.positions[:rows].cpu().numpy()
    cos, sin = host.cos.cpu().numpy(), host.sin.cpu().numpy()
    t0 = time.perf_counter()
    o = oracle.residual_rmsnorm_fp8(x_a, r, wa, wl.eps, wl.dt, wl.quant, static_scale=0.01)
    ob = oracle.qkv_norm_rope_kvcache(qkv, qw, kw, cos, sin, pos, wl.Hq, wl.Hkv, wl.hd, rows, wl.eps, wl.dt,
                                      slots=np.arange(rows))
    of = oracle.residual_rmsnorm_fp8(x_f, o["residual_out"], wf, wl.eps, wl.dt, wl.quant, static_scale=0.01)
    oc = oracle.gate_act_fp8(gu, wl.act, wl.dt, wl.quant, static_scale=0.01)
    secs = time.perf_counter() - t0
    if keep is not None:
        keep.update(a=o, b=ob, f=of, c=oc)
    return secs


def _code_steps(got, want):
    """FP8 e4m3 codes: how many differ, and the largest difference in steps
    (codes of one sign are ordered like their magnitudes)."""
    g, w = got.astype(np.int32).ravel(), want.astype(np.int32).ravel()
    same_sign = (g & 0x80) == (w & 0x80)
    steps = np.where(same_sign, np.abs((g & 0x7F) - (w & 0x7F)), (g & 0x7F) + (w & 0x7F))
    return int((g != w).sum()), int(steps.max()) if steps.size else 0


def _rel_16bit_ok(got16, want64, dt):
    """16-bit outputs against fp64 values: |g - o| <= 2e-3 max(|o|, 2^-6) +
    half an ulp of the 16-bit type."""
    g = got16.astype(np.float64)
    ulp = 2.0 ** (-7 if dt == "bf16" else -10)
    tol = 2e-3 * np.maximum(np.abs(want64), 2.0 ** -6) + 0.5 * ulp * np.abs(want64)
    return bool(np.all(np.abs(g - want64) <= tol + 1e-30))


def step_parity(wl, host, rows, keep):
    """The step's four ops on the GPU for the first `rows` rows of the bench's
    inputs (the same kernels, static scale 0.01 as the CPU leg), compared with
    the oracle outputs the CPU leg kept for the same rows."""
    import memory_bound_non_b200 as frt
    from memory_bound_non_b200 import workloads as W
    dev = torch.device("cuda")
    hl = host.layers[0]
    D, I, hd = wl.D, wl.I, wl.hd
    s = torch.tensor([0.01], dtype=torch.float32, device=dev)
    x_a, x_f = hl.x_attn[:rows].to(dev), hl.x_ffn[:rows].to(dev)
    r = host.residual[:rows].to(dev).clone()
    wa = None if hl.w_attn is None else hl.w_attn.to(dev)
    wf = None if hl.w_ffn is None else hl.w_ffn.to(dev)
    qa = torch.empty((rows, D), dtype=torch.uint8, device=dev)
    qf = torch.empty_like(qa)
    frt.frt_residual_rmsnorm_fp8(x_a, r, r, wa, qa, static_scale=s, eps=wl.eps, quant="static")
    r_a = r.clone()
    frt.frt_residual_rmsnorm_fp8(x_f, r, r, wf, qf, static_scale=s, eps=wl.eps, quant="static")
    # op b with the RoPE position as the slot: the rows' caches are read back
    # at their positions (the oracle wrote slot i for row i)
    pos = host.positions[:rows].to(dev)
    cap = int(host.positions[:rows].max()) + 1
    q_out = torch.empty((rows, wl.Hq, hd), dtype=x_a.dtype, device=dev)
    kc = torch.zeros((cap, wl.Hkv, hd), dtype=x_a.dtype, device=dev)
    vc = torch.zeros_like(kc)
    qw = None if hl.q_norm_w is None else hl.q_norm_w.to(dev)
    kw = None if hl.k_norm_w is None else hl.k_norm_w.to(dev)
    frt.frt_qkv_norm_rope_kvcache(hl.qkv[:rows].to(dev), qw, kw, host.cos.to(dev), host.sin.to(dev), pos, q_out,
                                  kc, vc, wl.Hq, wl.Hkv, hd, eps=wl.eps)
    qc = torch.empty((rows, I), dtype=torch.uint8, device=dev)
    frt.frt_gate_act_fp8(hl.gate_up[:rows].to(dev), qc, static_scale=s, act=wl.act, quant="static")
    torch.cuda.synchronize()
    p = pos.long()
    out = {"rows": rows}
    out["residual_bit_exact"] = bool(np.array_equal(W.bits16(r_a.cpu()), keep["a"]["residual_out"])
                                     and np.array_equal(W.bits16(r.cpu()), keep["f"]["residual_out"]))
    na, sa = _code_steps(qa.cpu().numpy(), keep["a"]["out_fp8"])
    nf, sf = _code_steps(qf.cpu().numpy(), keep["f"]["out_fp8"])
    nc, sc = _code_steps(qc.cpu().numpy(), keep["c"]["out_fp8"])
    out["fp8_codes_differing"] = {"attn_norm": na, "ffn_norm": nf, "gate": nc}
    out["fp8_max_step"] = max(sa, sf, sc)
    q_ok = _rel_16bit_ok(q_out.float().cpu().numpy(), keep["b"]["q_out"], wl.dt)
    k_ok = _rel_16bit_ok(kc[p].float().cpu().numpy(), keep["b"]["k_cache"][:rows], wl.dt)
    v_ok = bool(np.array_equal(W.bits16(vc[p].cpu()).reshape(rows, -1),
                               W.bits16(hl.qkv[:rows])[:, (wl.Hq + wl.Hkv) * hd:]))
    out["qkv_within_tolerance"] = bool(q_ok and k_ok)
    out["v_bit_exact"] = v_ok
    n_codes = rows * (2 * D + I)
    out["ok"] = bool(out["residual_bit_exact"] and q_ok and k_ok and v_ok and out["fp8_max_step"] <= 1
                     and (na + nf + nc) <= 0.001 * n_codes)
    return out


def cpu_baseline(wl, host, budget_s=12.0, keep=None):
    import dataclasses
    rows = 16
    secs = oracle_sample(wl, host, rows)
    rows = int(max(16, min(wl.M, rows * budget_s / max(secs, 1e-6))))
    secs = oracle_sample(wl, host, rows, keep=keep)
    b = sum(op_bytes(dataclasses.replace(wl, M=rows)).values())
    return {"value": round(b / secs / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "first %d of %d token rows of every op of the step (%.1f s, single thread)"
                      % (rows, wl.M, secs)}, rows / secs, rows


def _oracle_worker(task):
    """One process of the all-cores oracle leg: its own seeded inputs for a
    row block, then the oracle on them; returns seconds."""
    import dataclasses
    from memory_bound_non_b200 import workloads as W
    wl, rows = task
    small = dataclasses.replace(wl, M=rows)
    host = W.make_inputs(small, n_layers=1)
    return oracle_sample(small, host, rows)


def cpu_baseline_all_cores(wl, rows_per_s, budget_s=4.0, max_cores=32, max_rows=1024):
    """The same oracle, as it stands, in one process per host core (spawned,
    never forked from this CUDA process), each on its own block of rows;
    throughput = all rows' bytes / the slowest process's time."""
    import dataclasses
    import multiprocessing as mp
    cores = max(1, min(os.cpu_count() or 1, max_cores))
    rows = int(max(16, min(max_rows, rows_per_s * budget_s)))  # bounds each process's host memory
    with mp.get_context("spawn").Pool(cores) as pool:
        secs = pool.map(_oracle_worker, [(wl, rows)] * cores)
    b = cores * sum(op_bytes(dataclasses.replace(wl, M=rows)).values())
    return {"value": round(b / max(secs) / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": "%d processes x %d token rows of every op of the step (slowest %.1f s)"
                      % (cores, rows, max(secs))}


# ------------------------------------------------------- per-op table --
TABLE_WORKLOADS = ("tiny", "pi05", "qwen3_prefill_S128", "qwen3_prefill_S192", "qwen3_prefill_S512",
                   "qwen3_prefill_S1024", "vla_denoise", "vit", "large_m_M4096", "large_m_M16384", "large_m_M65536")


def _oracle_op(wl, host, op, rows):
    """Seconds the oracle takes for one op on the first `rows` rows."""
    import oracle
    from memory_bound_non_b200 import workloads as W
    hl = host.layers[0]
    if op in ("attn_norm", "ffn_norm"):
        x = W.bits16((hl.x_attn if op == "attn_norm" else hl.x_ffn)[:rows])
        r = W.bits16(host.residual[:rows])
        w = hl.w_attn if op == "attn_norm" else hl.w_ffn
        w = None if w is None else W.bits16(w)
        t0 = time.perf_counter()
        oracle.residual_rmsnorm_fp8(x, r, w, wl.eps, wl.dt, wl.quant, static_scale=0.01)
    elif op == "qkv":
        qkv = W.bits16(hl.qkv[:rows])
        qw = None if hl.q_norm_w is None else W.bits16(hl.q_norm_w)
        kw = None if hl.k_norm_w is None else W.bits16(hl.k_norm_w)
        pos = host.positions[:rows].cpu().numpy()
        cos, sin = host.cos.cpu().numpy(), host.sin.cpu().numpy()
        t0 = time.perf_counter()
        oracle.qkv_norm_rope_kvcache(qkv, qw, kw, cos, sin, pos, wl.Hq, wl.Hkv, wl.hd, rows, wl.eps, wl.dt,
                                     slots=np.arange(rows))
    else:
        gu = W.bits16(hl.gate_up[:rows])
        t0 = time.perf_counter()
        oracle.gate_act_fp8(gu, wl.act, wl.dt, wl.quant, static_scale=0.01)
    return time.perf_counter() - t0


def _oracle_op_worker(task):
    """One process of the all-cores column: its own seeded rows (torch on one
    thread, so the processes do not oversubscribe the cores), one op; a first
    untimed call on one row loads the oracle library, then the best of three
    timed runs (the processes start their runs at slightly different times)."""
    import dataclasses
    from memory_bound_non_b200 import workloads as W
    torch.set_num_threads(1)
    wl, op, rows = task
    small = dataclasses.replace(wl, M=rows)
    host = W.make_inputs(small, n_layers=1)
    _oracle_op(small, host, op, 1)
    return min(_oracle_op(small, host, op, rows) for _ in range(3))


def baseline_table(peak, reps=20, max_cores=32, sample_s=1.0):
    """Per op and workload: GPU microseconds (CUDA events around each launch,
    L2 flushed before it; at M <= 41 also per graph node), GB/s and roofline
    fractions, and the CPU oracle's microseconds for the whole batch on one
    host thread (timed on a row sample, scaled to all rows) and on all host
    cores (one spawned process per core, each on its share of the rows)."""
    import dataclasses
    import multiprocessing as mp
    from memory_bound_non_b200 import workloads as W
    from memory_bound_non_b200.chain import LayerChain
    cores = max(1, min(os.cpu_count() or 1, max_cores))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream()
    rows_out = []
    pool = mp.get_context("spawn").Pool(cores)
    try:
        for name in TABLE_WORKLOADS:
            wl = W.get(name, layers=1, steps=1)
            big = wl.M >= 4096
            inp = W.make_inputs(wl, n_layers=1, device="cuda" if big else "cpu")
            ch = LayerChain(wl, inp)
            ch.calibrate_static_scales()
            nbytes = op_bytes(wl)
            for op in ("attn_norm", "qkv", "ffn_norm", "gate"):
                fn = getattr(ch, op)
                for _ in range(3):
                    fn(0)
                ts = []
                for _ in range(reps):
                    flush_l2(flush)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(s)
                    fn(0)
                    e1.record(s)
                    e1.synchronize()
                    ts.append(e0.elapsed_time(e1) * 1e3)
                us = statistics.median(ts)
                gbs = nbytes[op] / (us * 1e-6) / 1e9
                row = {"workload": name, "op": op, "M": wl.M, "bytes": nbytes[op], "gpu_us": round(us, 2),
                       "GBps": round(gbs, 1), "frac_of_8TBps": round(gbs / NOMINAL_HBM_GBS, 4),
                       "frac_of_measured": round(gbs / peak, 4)}
                if wl.M <= 41:
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        for _ in range(100):
                            fn(0)
                    g.replay()
                    torch.cuda.synchronize()
                    gt = []
                    for _ in range(5):
                        e0.record(s)
                        g.replay()
                        e1.record(s)
                        e1.synchronize()
                        gt.append(e0.elapsed_time(e1) * 1e3 / 100)
                    del g
                    row["gpu_us_graph_node"] = round(statistics.median(gt), 3)
                # CPU oracle: one thread on a sample of rows, scaled to M
                host = inp if not big else None
                n = min(wl.M, 16)
                if big:
                    sub = dataclasses.replace(wl, M=n)
                    host = W.make_inputs(sub, n_layers=1)
                _oracle_op(wl if not big else sub, host, op, 1)  # loads the oracle library
                t1 = _oracle_op(wl if not big else sub, host, op, n)
                n2 = int(max(n, min(wl.M, n * sample_s / max(t1, 1e-6))))
                if n2 > n:
                    if big:
                        sub = dataclasses.replace(wl, M=n2)
                        host = W.make_inputs(sub, n_layers=1)
                    t1 = _oracle_op(wl if not big else sub, host, op, n2)
                    n = n2
                else:
                    t1 = min(t1, _oracle_op(wl if not big else sub, host, op, n))
                row["cpu_1thread_us"] = round(t1 / n * wl.M * 1e6, 1)
                row["cpu_1thread_sample_rows"] = n
                per = max(1, -(-wl.M // cores))
                per_run = min(per, max(1, int(n * 2 / 3)))  # bounded: each process times about 2 s in all
                secs = pool.map(_oracle_op_worker, [(wl, op, per_run)] * min(cores, wl.M))
                row["cpu_all_cores_us"] = round(max(secs) / per_run * per * 1e6, 1)
                row["cpu_all_cores_rows_per_process"] = per_run
                rows_out.append(row)
                print(json.dumps(row), flush=True)
            del ch, inp
            torch.cuda.empty_cache()
    finally:
        pool.close()
        pool.join()
    return {"cores": cores, "cpu": _cpu_model(), "rows": rows_out}


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def reference_arm(args):
    """The oracle, as it stands, timed on host cores on the same workload."""
    import dataclasses
    from memory_bound_non_b200 import workloads as W
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    wl = W.get(args.workload)
    # inputs for a row sample only (the oracle runs on the first rows)
    probe_rows = 16
    host = W.make_inputs(dataclasses.replace(wl, M=4096), n_layers=1)
    t = oracle_sample(wl, host, probe_rows) / probe_rows
    budget = 150.0
    rows = int(max(1, min(4096, budget / max(1, args.steps + args.warmup) / max(t, 1e-9))))
    for _ in range(args.warmup):
        oracle_sample(wl, host, rows)
    secs = 0.0
    for _ in range(args.steps):
        secs += oracle_sample(wl, host, rows)
    per_step = secs / args.steps
    b = sum(op_bytes(dataclasses.replace(wl, M=rows)).values())
    val = b / per_step / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "io_dtypes": {"in": wl.dt, "out": "e4m3", "residual": wl.dt,
                          "arithmetic": "fp64 (FP8 decisions on fp32 quotients)"},
            "data": "synthetic (seeded torch.Generator('cpu'))",
            "config": {"workload": wl.name, "M": wl.M, "D": wl.D, "Hq": wl.Hq, "Hkv": wl.Hkv, "hd": wl.hd,
                       "I": wl.I, "act": wl.act, "quant": wl.quant, "sample_rows_per_step": rows},
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": "first %d token rows of every op per step" % rows},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main --
def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return reference_arm(args)
    import memory_bound_non_b200 as frt
    from memory_bound_non_b200 import workloads as W
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    frt.load()
    dist = Dist(world, "nccl", torch.device("cuda", local))
    barrier, max_over_ranks = dist.barrier, dist.max_over_ranks

    wl = W.get(args.workload)
    peak, peak_kind = measured_peak()
    if args.persistent_chain:
        if rank == 0:
            from memory_bound_non_b200.chain import LayerChain
            cw = W.get(args.persistent_chain)
            ch = LayerChain(cw, W.make_inputs(cw))
            ch.calibrate_static_scales()
            st = torch.cuda.current_stream()
            ts = []
            for _ in range(args.chain_reps):
                ch.reset()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(st)
                ch.run_persistent()
                e1.record(st)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3)
            print(json.dumps({"persistent_chain": cw.name, "launches": len(ts),
                              "us_median": round(statistics.median(ts), 2)}), flush=True)
        dist.close()
        return 0
    if args.table:
        if rank == 0:
            t = baseline_table(peak)
            t.update(peak=peak, peak_kind=peak_kind)
            s = json.dumps(t)
            print(s, flush=True)
            if args.json_out:
                with open(args.json_out, "w") as f:
                    f.write(s + "\n")
        dist.close()
        return 0
    if args.next_only:
        if rank == 0:
            floor = launch_floor()
            s = json.dumps({"next_ops": next_ops_leg(peak, floor, args.next_reps, args.next_m),
                            "launch_floor": floor, "peak": peak, "peak_kind": peak_kind})
            print(s, flush=True)
            if args.json_out:
                with open(args.json_out, "w") as f:
                    f.write(s + "\n")
        dist.close()
        return 0
    step = Step(wl, rank)
    bytes_op = op_bytes(step.wl)
    step_bytes = sum(bytes_op.values())

    clocks = ClockSampler(local)
    clocks.start()
    total_ms, per_op_us = timed_step_leg(step, args.steps, args.warmup, barrier)
    clk = clocks.stop()
    total_ms = max_over_ranks(total_ms)
    ms_per_step = total_ms / args.steps
    value = job_throughput(step_bytes, world, ms_per_step)

    per_op = {}
    for name, ts in per_op_us.items():
        mean_us = sum(ts) / len(ts)
        gbs = bytes_op[name] / (mean_us * 1e-6) / 1e9
        q = statistics.quantiles(ts, n=10) if len(ts) >= 2 else [mean_us] * 9
        per_op[name] = {"us_mean": round(mean_us, 2), "us_median": round(statistics.median(ts), 2),
                        "us_p10": round(q[0], 2), "us_p90": round(q[8], 2), "bytes": bytes_op[name], "GBps": round(gbs, 1), "frac_of_measured": round(gbs / peak, 4),
                        "frac_of_8TBps": round(gbs / NOMINAL_HBM_GBS, 4)}
    dom = max(per_op, key=lambda k: per_op[k]["us_mean"])
    traffic = measured_traffic(wl.name, dom)
    roofline = {"bound": "hbm", "kernel": {"gate": "frt_gate_act_fp8", "qkv": "frt_qkv_norm_rope_kvcache",
                                          "attn_norm": "frt_residual_rmsnorm_fp8",
                                          "ffn_norm": "frt_residual_rmsnorm_fp8"}[dom],
                "achieved": per_op[dom]["GBps"], "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                "frac": round(per_op[dom]["GBps"] / peak, 4), "traffic": traffic,
                "algorithmic_bytes_per_launch": bytes_op[dom]}

    extra = {}
    if rank == 0 and not args.no_chain:
        pdl0 = frt.frt_get_pdl()
        for pdl in (True, False):
            frt.frt_set_pdl(pdl)
            tag = "" if pdl else "_no_pdl"
            floor = launch_floor()
            extra["launch_floor" + tag] = {k: (round(v, 3) if isinstance(v, float) else v) for k, v in floor.items()}
            extra["chain" + tag] = chain_leg(args.chain_reps, floor)
            extra["small_m" + tag] = small_m_ops(floor)
            if pdl:
                extra["next_ops"] = next_ops_leg(peak, floor, args.next_reps, args.next_m)
        frt.frt_set_pdl(pdl0)
    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h = e2e_leg(step, args.e2e_steps, 1)
        e2e_ms = max_over_ranks(e2e_ms)
        e2e = {"value": round(job_throughput(step_bytes, world, e2e_ms), 2), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3)}
    cpu = cpu_all = parity = None
    if rank == 0 and world == 1 and not args.no_cpu:
        want_parity = not args.no_parity
        keep = {} if want_parity else None
        cpu, rows_per_s, rows = cpu_baseline(step.wl, step.host, keep=keep)
        cpu_all = cpu_baseline_all_cores(step.wl, rows_per_s)
        if want_parity and step.wl.quant != "static":
            parity = {"ok": None, "skipped": "the CPU leg's sample uses a static scale"}
        elif want_parity:
            try:
                parity = step_parity(step.wl, step.host, rows, keep)
            except Exception as exc:  # reported, never fatal to the timing line
                parity = {"ok": False, "error": "%s: %s" % (type(exc).__name__, exc)}

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "io_dtypes": {"in": wl.dt, "out": "e4m3", "residual": wl.dt,
                              "arithmetic": "fp32, fp64 row sums of squares"},
                "data": "synthetic: seeded torch.Generator('cpu'), N(0,1) activations, 1+0.1N norm weights",
                "config": {"workload": wl.name, "M": wl.M, "D": wl.D, "Hq": wl.Hq, "Hkv": wl.Hkv, "hd": wl.hd,
                           "I": wl.I, "act": wl.act, "quant": wl.quant, "io": "bf16 in, e4m3 out",
                           "capacity": wl.capacity, "bytes_per_step_per_gpu": step_bytes,
                           "l2": "inputs larger than L2 (%.1f GB per step)" % (step_bytes / 1e9),
                           "parallelism": "row shards, no collective" if world > 1 else "single GPU"},
                "roofline": roofline, "per_op": per_op, "gpu_launches": 4 * args.steps, "clocks": clk,
                "e2e": e2e, "cpu_baseline": cpu, "cpu_baseline_all_cores": cpu_all, "parity": parity,
                "input_gen_s": round(step.gen_s, 1)}
        line.update(extra)
        s = json.dumps(line)
        print(s, flush=True)
        if args.json_out:
            with open(args.json_out, "w") as f:
                f.write(s + "\n")
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
