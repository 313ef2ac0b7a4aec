"""Host-side bookkeeping of bench.py (CPU only): algorithmic bytes and FLOPs per
token, the L2 rotation of small workloads and the whole-job throughput."""

import math

import pytest

import bench
import workloads as synth


def test_bytes_per_token_is_x_plus_y():
    w = synth.CYCLIC_WORKLOADS["c8_t131072_160x160_bf16"]
    assert bench.bytes_per_token(w) == (160 + 160) * 8 * 2          # 5120 B
    w = synth.CYCLIC_WORKLOADS["c4_t64_16x16_f32"]
    assert bench.bytes_per_token(w) == (16 + 16) * 4 * 4
    w = synth.D8_WORKLOADS["d8_t131072_c1280_gelu_bf16"]
    assert bench.bytes_per_token(w) == 2 * 1280 * 2


def test_flops_per_token_counts_the_real_products_of_the_half_spectrum():
    # C_8: bins 0 and 4 real (one product each), bins 1..3 complex (four each)
    w = synth.CYCLIC_WORKLOADS["c8_t131072_160x160_bf16"]
    assert bench.flops_per_token(w) == 2 * 14 * 160 * 160
    # C_16: 2 real + 7 complex bins = 30 real products
    w = synth.CYCLIC_WORKLOADS["c16_t65536_96x384_bf16"]
    assert bench.flops_per_token(w) == 2 * 30 * 96 * 384
    # D8: 3 C^2 / 16 multiplies per token
    w = synth.D8_WORKLOADS["d8_t131072_c1280_gelu_bf16"]
    assert bench.flops_per_token(w) == 2 * 3 * 1280 * 1280 // 16


def test_workloads_larger_than_l2_do_not_rotate():
    for name in ("c8_t131072_160x160_bf16", "c16_t65536_96x384_bf16", "c8_t131072_160x640_bf16"):
        w = synth.CYCLIC_WORKLOADS[name]
        step = bench.bytes_per_token(w) * w.T
        assert bench.rotation_sets(step) == 1
        assert "larger than L2" in bench.l2_note(w, 1)


def test_small_workloads_rotate_past_l2():
    w = synth.CYCLIC_WORKLOADS["c8_t8192_64x64_bf16"]
    step = bench.bytes_per_token(w) * w.T
    R = bench.rotation_sets(step)
    assert R > 1 and R * step >= 3 * bench.L2_BYTES and (R - 1) * step < 3 * bench.L2_BYTES
    assert "rotate over" in bench.l2_note(w, R) and "still fit" not in bench.l2_note(w, R)
    # a toy workload cannot leave L2 within 64 sets: labelled as such
    w = synth.CYCLIC_WORKLOADS["c4_t64_16x16_f32"]
    R = bench.rotation_sets(bench.bytes_per_token(w) * w.T)
    assert R == 64 and "still fit in L2" in bench.l2_note(w, R)


def test_job_throughput_counts_every_ranks_tokens():
    assert bench.job_tokens_per_s(1000, 4, 10, 2.0) == pytest.approx(1000 * 4 * 10 / 2e-3)
    assert math.isclose(bench.job_tokens_per_s(131072, 1, 1, 0.1755), 131072 / 0.1755e-3)


def test_mlp_pass_counts_both_layers_and_the_hidden_round_trip():
    w = synth.D8_WORKLOADS["d8_t131072_c1280_gelu_bf16"]
    C = 1280
    # z in (C), hidden out and back in (4C each), y out (C), bf16
    assert bench.bytes_per_token(w, "mlp") == (C + 4 * C + 4 * C + C) * 2
    # expand C -> 4C and contract 4C -> C: 3 C_in C_out / 16 products each
    assert bench.flops_per_token(w, "mlp") == 2 * (3 * C * 4 * C // 16 + 3 * 4 * C * C // 16)
    # the other passes keep the layer's own counts
    assert bench.bytes_per_token(w, "forward") == bench.bytes_per_token(w)


@pytest.mark.parametrize("name,which,fn", [
    ("c8_t131072_160x160_bf16", "forward", "cyclic_forward"),
    ("c8_t131072_160x160_bf16", "backward_data", "cyclic_backward_data"),
    ("c8_t131072_160x160_bf16", "weight_grad", "cyclic_weight_grad"),
    ("d8_t131072_c1280_gelu_bf16", "forward", "d8_forward"),
    ("d8_t131072_c1280_gelu_bf16", "mlp", "d8_mlp_block"),
])
def test_cpu_baseline_times_the_oracle_of_the_timed_pass(monkeypatch, name, which, fn):
    import oracle
    w = bench.workload(name)
    called = []
    real = getattr(oracle, fn)
    monkeypatch.setattr(oracle, fn, lambda *a, **k: called.append(a[0].shape[0]) or real(*a, **k))
    bench.oracle_rows_fn(w, which)(3)
    assert called == [3]


def test_recorded_traffic_holds_only_for_the_profiled_sources(monkeypatch, tmp_path):
    """roofline.traffic comes from profiles/traffic.json only while the sources a
    pass runs hash to what was profiled; any other hash gives null."""
    import json
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({
        "tcgen05:w": {"source_hash": "aaaa", "dram_bytes_per_launch": 123.0},
        "tcgen05:w:weight_grad": {"source_hash": "bbbb", "dram_bytes_per_launch": 456.0}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda weight_grad=False: "bbbb" if weight_grad else "aaaa")
    assert bench.recorded_traffic("tcgen05:w") == 123.0
    assert bench.recorded_traffic("tcgen05:w:weight_grad") == 456.0
    assert bench.recorded_traffic("tcgen05:other") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda weight_grad=False: "cccc")
    assert bench.recorded_traffic("tcgen05:w") is None
    assert bench.recorded_traffic("tcgen05:w:weight_grad") is None
