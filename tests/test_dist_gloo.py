"""Multi-rank host logic of the bench on CPU: two gloo ranks on 127.0.0.1.

The data path shards by rows with no collective; what the ranks share is the
barrier and the max-over-ranks timing that turns per-rank times into one
whole-job number.  Also: every rank draws its own shard of the workload.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
from memory_bound_non_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    d = bench.Dist(world, backend="gloo", timeout_s=60)
    d.barrier()
    local_ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
    worst = d.max_over_ranks(local_ms)
    wl = bench.rank_workload(W.get("tiny"), rank)
    inp = W.make_inputs(wl, n_layers=1, with_caches=False)
    out[rank] = (worst, float(inp.residual.float().sum()), tuple(inp.residual.shape))
    d.close()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_shard_inputs():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][2] == out[1][2]            # same shapes on every rank
    assert out[0][1] != out[1][1]            # different rows on every rank
    # whole-job throughput: both ranks' bytes over the slowest rank's time
    assert bench.job_throughput(1e9, world, 15.0) == pytest.approx(2e9 / 15e-3 / 1e9)


def test_single_rank_needs_no_group():
    d = bench.Dist(1)
    d.barrier()
    assert d.max_over_ranks(3.5) == 3.5
    d.close()


def test_reference_arm_prints_only_on_rank_zero(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""


def test_op_bytes_are_the_algorithmic_bytes():
    wl = W.get("large_m_M65536")
    b = bench.op_bytes(wl)
    # a: x, r_in, r_out (2 B) + fp8 (1 B) per element, weight, static scale
    assert b["attn_norm"] == 65536 * 4096 * 7 + 2 * 4096 + 4
    # b: QKV read + Q/K/V written (2 B each), cos+sin rows, position, two norm weights
    assert b["qkv"] == 65536 * 6144 * 4 + 65536 * 128 * 4 + 4 * 65536 + 4 * 128
    # c: gate/up read (4 B per output) + fp8 out, static scale
    assert b["gate"] == 65536 * 16384 * 5 + 4


def test_all_cores_oracle_leg_counts_every_process_rows():
    """The all-cores CPU leg: spawned processes, each on its own row block;
    the reported throughput counts every process's rows over the slowest
    process's time, and the rows per process are bounded."""
    wl = W.get("tiny")
    out = bench.cpu_baseline_all_cores(wl, rows_per_s=1e6, budget_s=1.0, max_cores=2, max_rows=32)
    assert out["kind"] == "oracle" and out["unit"] == "GB/s"
    assert out["cores"] == min(2, os.cpu_count() or 1)
    assert "%d processes x 32 token rows" % out["cores"] in out["sample"]
    assert out["value"] > 0


def test_parity_helpers_count_code_steps_and_16bit_tolerance():
    """The bench's parity summary: FP8 codes compared by count and by steps
    (one sign's codes are ordered like their magnitudes; across signs the
    steps go through zero), 16-bit outputs against fp64 values."""
    import numpy as np
    want = np.array([0x00, 0x38, 0x38, 0xB8, 0x7E], dtype=np.uint8)
    got = np.array([0x00, 0x39, 0x38, 0x38, 0x7E], dtype=np.uint8)
    n, steps = bench._code_steps(got, want)
    assert n == 2 and steps == 2 * 0x38
    n, steps = bench._code_steps(want, want)
    assert n == 0 and steps == 0
    o = np.array([1.0, -3.0, 1e-3])
    assert bench._rel_16bit_ok(o.astype(np.float32), o, "bf16")
    assert not bench._rel_16bit_ok((o * 1.02).astype(np.float32), o, "bf16")


def test_traffic_records_follow_their_own_kernel_source(tmp_path, monkeypatch):
    """A DRAM-traffic record is used only while its kernel's source file and
    the shared headers keep the sha256 recorded with it: editing another
    kernel's file leaves it valid, editing its own voids it."""
    import json
    import bench
    now = bench.source_hashes()
    rec = {"source_sha256": dict(now),
           "per_launch_bytes": {"large_m_M65536": {"gate": 123, "attn_norm": 456},
                                "qkv_prepq_e4m3_M65536": {"qkv_prepq": 789}}}
    root = tmp_path
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    monkeypatch.setattr(bench, "source_hashes", lambda: now)

    def write(r):
        (root / "profiles" / "traffic.json").write_text(json.dumps(r))
    write(rec)
    assert bench.measured_traffic("large_m_M65536", "gate") == 123
    assert bench.measured_traffic("qkv_prepq_e4m3_M65536", "qkv_prepq") == 789
    assert bench.measured_traffic("large_m_M65536", "qkv") is None          # no record
    changed = dict(rec, source_sha256=dict(now, **{"residual_rmsnorm_fp8.cu": "0" * 64}))
    write(changed)
    assert bench.measured_traffic("large_m_M65536", "attn_norm") is None    # its own file changed
    assert bench.measured_traffic("large_m_M65536", "gate") == 123         # another kernel's file
    shared = dict(rec, source_sha256=dict(now, **{"frt_device.cuh": "0" * 64}))
    write(shared)
    assert bench.measured_traffic("large_m_M65536", "gate") is None        # a shared header changed
