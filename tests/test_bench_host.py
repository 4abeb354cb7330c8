"""Host-side arithmetic of bench.py (no GPU): the algorithmic bytes and flops
the roofline divides by, the roofline's binding resource, the workload
descriptions, and the guard that drops a recorded DRAM traffic figure once
the kernels' sources change."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_algorithmic_work_of_the_headline_batch():
    wl = bench.workload("dsv3_64k", 1)
    a = bench.algorithmic(wl)
    T = 64 * 65536
    # the latent cache read once: [c (512) ; k_rope (64)] bf16 per token
    assert a["absorb_bytes"] == 2 * T * 576 == 4_831_838_208
    # per (head, key): 2 flop per multiply-add over the 576 score dims and the
    # 512 value dims; plus the new token's q~ and up-projection GEMMs
    keys = T
    assert a["absorb_flops"] == 128 * keys * 2 * (2 * 512 + 64) + 64 * 128 * 2 * 512 * (128 + 128)
    # the expanded cache: K (192) and V (128) per group and token
    assert a["gqa_bytes"] == 2 * T * 16 * (192 + 128)
    assert a["gqa_flops"] == 128 * keys * 2 * (192 + 128)
    # the shared-RoPE K pool stores the 64 RoPE dims once per token
    assert a["gqa_shared_bytes"] == 2 * T * (16 * (128 + 128) + 64)
    # one new token per sequence: its latent row, then its K/V rows of every group
    assert a["append_bytes"] == 2 * 64 * 576
    assert a["expand_new_bytes"] == 2 * 64 * 576 + 2 * 64 * 16 * 320


def test_causal_keys_with_several_new_tokens():
    # query i of s_q sees L - s_q + i + 1 keys (bottom-right causal alignment)
    wl = bench.workload("llama3_8b", 2)
    a = bench.algorithmic(wl)
    L, B = 8192, 32
    keys = B * ((L - 1) + L)
    assert a["gqa_flops"] == 32 * keys * 2 * (192 + 128)


def test_roofline_binding_resource():
    # 1 GB at 1000 GB/s = 1 ms; 1 TFLOP at 1000 TFLOP/s = 1 ms
    t, b = bench.roof_time(2e9, 1e12, 1000.0, 1000.0)
    assert b == "hbm" and t == pytest.approx(2e-3)
    t, b = bench.roof_time(1e9, 3e12, 1000.0, 1000.0)
    assert b == "tensor" and t == pytest.approx(3e-3)
    # the headline: balanced, the HBM side a little larger at the measured peaks
    wl = bench.workload("dsv3_64k", 1)
    a = bench.algorithmic(wl)
    t, b = bench.roof_time(a["absorb_bytes"], a["absorb_flops"], 6559.0, 1656.2)
    assert b == "hbm" and 0.70e-3 < t < 0.75e-3


def test_configs_name_the_workload_and_the_parallelism():
    c = bench.bench_config(bench.workload("dsv3_64k", 1))
    assert c["workload"] == "dsv3_gqla B64 L65536 s_q1"
    assert (c["batch"], c["seq_len"], c["n_h"], c["G"], c["r"], c["dtype"]) == (64, 65536, 128, 16, 512, "bf16")
    assert "no flush" in c["l2"] and c["parallelism"].startswith("replicas x1")
    t = bench.bench_config(bench.workload("dsv3_64k", 1), world=8, tp=True)
    assert t["parallelism"].startswith("tp8 over groups")


def test_recorded_traffic_is_dropped_when_a_source_changes(tmp_path, monkeypatch):
    # a copy of the tree's csrc and profiles under a temporary root
    csrc = tmp_path / "latent_kv_cache_flash_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"gqla_decode_absorb @ w": {"files": ["k.cu"], "bytes_per_launch": 123,
                                      "source_sha": bench.kernel_sha(["k.cu"])}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("gqla_decode_absorb", "w") == 123
    assert bench.recorded_traffic("gqla_decode_absorb", "other workload") is None
    (csrc / "k.cu").write_text("kernel v2\n")
    assert bench.recorded_traffic("gqla_decode_absorb", "w") is None


def test_committed_traffic_record_matches_the_sources():
    # the committed record of the headline call is valid for the tree as it is
    v = bench.recorded_traffic("gqla_decode_absorb", "dsv3_gqla B64 L65536 s_q1")
    assert v is not None and 5.0e9 < v < 5.8e9
