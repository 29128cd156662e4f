"""Multi-rank host logic of the benchmark, on CPU with gloo (world size 2):
the whole-job numbers take the slowest rank's time and every rank's scored
tokens; the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms, loss_ms, scored = bench.reduce_over_ranks(10.0 + rank * 5.0, 1.0 + rank, 100.0 * (rank + 1),
                                                      torch.device("cpu"))
        out[rank] = (ms, loss_ms, scored)
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo_two_ranks():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for r in (0, 1):
        assert res[r] == (15.0, 2.0, 300.0)


def test_reduce_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(3.0, 1.5, 42.0, torch.device("cpu")) == (3.0, 1.5, 42.0)


def _run_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
               OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "abs_b2_l64_v1024", "--steps", "3", "--warmup", "3",
                           "--gpus", str(world)], capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_on_rank0_only():
    r1 = _run_reference(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_reference(0, 2)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["n_gpus"] == 2


def test_reference_arm_on_typed_decisions():
    """The reference arm on the typed-decision workload (label slots
    scaled down): the decision oracle over every slot, one line."""
    env = dict(os.environ, RANK="0", LOCAL_RANK="0", WORLD_SIZE="1", OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "dec_s128_k26_v126464", "--slots", "8", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["config"]["label_slots"] == 8
    assert line["config"]["workload"] == "dec_s8_k26_v126464" and line["cpu_baseline"]["kind"] == "oracle"


def test_cpu_baseline_all_cores_and_one_thread():
    """The CPU baseline: the oracle on a bounded sample for about its time
    budget, then again on one thread in a child process."""
    sys.path.insert(0, ROOT)
    import bench
    import dlm_inputs as di
    r = bench.cpu_baseline(di.WORKLOADS["abs_b2_l64_v1024"], budget_s=0.5, single_thread_s=0.3)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1
    assert "steps" in r["sample"] and r["unit"] == bench.UNIT
    one = r["single_thread"]
    assert one["cores"] == 1 and one["value"] > 0, one


def test_cpu_baseline_fused_head_workloads(monkeypatch):
    """The fused-head oracle as a CPU baseline, on small versions of both
    fused-head workloads; and the skip when its host memory would not fit."""
    sys.path.insert(0, ROOT)
    import bench
    import dlm_inputs as di
    small = {"lin_t16384_d4096_v126464": dict(n_tokens_packed=300, d_model=64, vocab=2048, ids_high=2000,
                                              mask_id=2047),
             "lin_unif_b4_p512_c1024_d4096_v262144": dict(n_units=2, seq_len=64, prefix=16, d_model=64,
                                                          vocab=2048, ids_high=2047)}
    for key, kw in small.items():
        spec = di.WORKLOADS[key].scaled(**kw)
        r = bench.cpu_baseline(spec, budget_s=0.5, single_thread_s=0.3)
        assert r["value"] > 0 and "dH and dW" in r["sample"], r
        assert r["single_thread"]["value"] > 0 and r["single_thread"]["cores"] == 1, r
    import psutil

    class _Mem:
        available = 1 << 30
    monkeypatch.setattr(psutil, "virtual_memory", lambda: _Mem())
    r = bench.cpu_baseline(di.WORKLOADS["lin_unif_b4_p512_c1024_d4096_v262144"], single_thread_s=0)
    assert r["value"] is None and "host memory" in r["skipped"]
