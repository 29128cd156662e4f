"""The benchmark's per-workload legs on scaled-down workloads, on the GPU:
every record carries a measured end-to-end figure (inputs from pinned host
memory, the loss read back), a roofline with the kernel's launch time,
clocks, and a positive throughput -- for the logits, fused-head and
typed-decision legs -- so a broken leg cannot hide behind an error string in
the JSON line."""
import argparse
import os
import sys

import pytest
import torch

import dlm_inputs as di

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _args(**kw):
    a = dict(gpus=1, steps=8, warmup=3, impl="ours", workload="", no_cpu_baseline=True, no_e2e=False,
             e2e_steps=3, keep_unscored=False, align="aligned", objective="plain")
    a.update(kw)
    return argparse.Namespace(**a)


def _check(rec):
    assert "error" not in rec, rec.get("error")
    assert rec["value"] > 0 and rec["ms_per_step"] > 0
    e = rec["e2e"]
    assert e is not None and "error" not in e, e
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] == 4
    r = rec["roofline"]
    assert r["achieved"] > 0 and r["launch_ms"] > 0 and 0 < r["frac"] < 2
    assert rec["clocks"] is not None and rec["gpu_launches"] > 0


@pytest.mark.parametrize("key,scale", [
    ("abs_b1_l4096_v126464", dict(seq_len=512)),
    ("unif_b4_p512_c1024_v262144", dict(n_units=1, seq_len=128, prefix=64)),
])
def test_logits_leg(key, scale):
    import bench
    rec = bench.run_logits(_args(), di.WORKLOADS[key].scaled(**scale), torch.device("cuda", 0), 0, 1,
                           headline=False)
    _check(rec)


@pytest.mark.parametrize("key,scale", [
    ("lin_t16384_d4096_v126464", dict(n_tokens_packed=1024, d_model=512, vocab=20000, ids_high=19000,
                                      mask_id=19999)),
    ("lin_unif_b4_p512_c1024_d4096_v262144", dict(n_units=2, seq_len=128, prefix=64, d_model=256,
                                                  vocab=16384, ids_high=16383)),
])
def test_fused_head_leg_measures_end_to_end(key, scale):
    import bench
    rec = bench.run_linear(_args(), di.WORKLOADS[key].scaled(**scale), torch.device("cuda", 0), 0, 1,
                           headline=False)
    _check(rec)
    assert rec["roofline"]["bound"] == "tensor"


def test_decision_leg():
    import bench
    rec = bench.run_decision(_args(steps=16), di.WORKLOADS["dec_s128_k26_v126464"].scaled(n_units=24),
                             torch.device("cuda", 0), 0, 1, headline=False)
    _check(rec)
    assert rec["steps"] % 8 == 0
