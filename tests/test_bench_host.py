"""Host logic of the benchmark, without a GPU: the round's algorithmic cost
model, the scaling of the committed DRAM-traffic capture to a full-size launch,
and the peak figures it reports against."""

import json
import os

import pytest

import bench

FULL = bench.WORKLOADS["full"]["cfg"]


def test_step_cost_matches_the_stage_by_stage_totals():
    """With every expert touched in every layer, the full-size round is
    1.97 TFLOP and 50.27 GB, summed stage by stage from the model's shapes:
    experts 45.68 GB, attention projections 1.43, attention at context 1024
    0.17, LM head 1.48, expected embedding and self-conditioning 1.49, router
    0.02."""
    flops, nbytes = bench.step_cost(FULL, 1, 1024, [128] * FULL["n_layers"])
    assert flops == pytest.approx(1.97e12, rel=5e-3)
    assert nbytes == pytest.approx(50.27e9, rel=5e-3)


def test_step_cost_counts_each_distinct_expert_once():
    """The FLOPs follow the tokens (every token runs k experts), the bytes the
    experts the router touches: one more distinct expert in one layer adds
    its gate, up and down weights (3 x d_ff x d_model bf16) and nothing else."""
    L = FULL["n_layers"]
    f1, b1 = bench.step_cost(FULL, 1, 1024, [12] * L)
    f2, b2 = bench.step_cost(FULL, 1, 1024, [12] * (L - 1) + [13])
    assert f1 == f2
    assert b2 - b1 == 3 * FULL["d_ff"] * FULL["d_model"] * 2


def test_step_cost_grows_with_batch_and_context():
    L = FULL["n_layers"]
    f1, b1 = bench.step_cost(FULL, 1, 1024, [16] * L)
    f2, b2 = bench.step_cost(FULL, 2, 1024, [16] * L)
    # the weights are read once whatever the batch; only the K/V bytes double
    kv1 = L * 2.0 * 1 * FULL["n_kv_heads"] * (1024 + 256) * FULL["head_dim"] * 2
    assert b2 - b1 == pytest.approx(kv1)
    assert f2 > 1.99 * f1
    f3, b3 = bench.step_cost(FULL, 1, 2048, [16] * L)
    assert b3 > b1 and f3 > f1


def test_ncu_traffic_scales_the_capture_by_distinct_experts(monkeypatch):
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")))
    key, e = next(iter(rec.items()))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: e["source_hash"])
    measured = e["read_bytes"] + e["write_bytes"]
    # at the capture's own expert count the capture itself comes back
    assert bench.ncu_traffic(key, e["distinct_experts"]) == pytest.approx(measured)
    # linear in the distinct experts, through the expert-independent bytes
    half = bench.ncu_traffic(key, e["distinct_experts"] / 2)
    assert half == pytest.approx(e["fixed_bytes"] + (measured - e["fixed_bytes"]) / 2)
    assert bench.ncu_traffic("no such kernel", 10.0) is None
    assert bench.ncu_traffic(key, 0.0) is None


def test_ncu_traffic_is_null_once_the_kernel_sources_change(monkeypatch):
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")))
    key = next(iter(rec))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.ncu_traffic(key, 18.3) is None


def test_traffic_record_names_a_kernel_source_hash_of_the_right_form():
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")))
    for key, e in rec.items():
        assert len(e["source_hash"]) == 16 and int(e["source_hash"], 16) >= 0
        assert e["read_bytes"] > e["fixed_bytes"] > 0 and e["distinct_experts"] > 0
        assert "--clock-control none" in e["command"] and "bench.py" in e["command"]


def test_peaks_fall_back_to_the_stated_figures_without_the_measured_file(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback"
    assert (p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"]) == (6650.0, 1590.0, 1400.0)
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}))
    p = bench.load_peaks()
    assert p["source"] == "measured" and p["bf16_tflops_sustained"] == 1600.0


def test_oracle_timing_of_the_tiny_loop_on_all_cores_and_one_thread():
    """The oracle baselines of the smaller configurations: the tiny model's
    whole 4-round loop, timed on the cores it is given and on one thread, and
    on the plain C++ oracle."""
    out = bench.oracle_other_configs(2, full_width=False)
    assert [e["cores"] for e in out] == [2, 1, 1]
    assert "C++" in out[2]["kind"]
    for e in out:
        assert e["kind"].startswith("oracle") and e["unit"] == bench.UNIT and e["value"] > 0
        assert "4-round loop" in e["workload"]
