"""The benchmark's host side without a GPU: option parsing, the launch counts it
claims, and the reference arm (the oracle on the host cores) for the default
step, the MSE-optimised scales and the outlier statistics, each printing one
JSON line with the keys the measurement contract asks for."""
import json

import pytest

import bench


def test_parse_new_options():
    a = bench.parse_args([])
    assert a.search is None and a.outlier_stats is None
    a = bench.parse_args(["--scale-search", "2,1", "--outlier-stats", "0.999"])
    assert a.search == (2, 1) and a.outlier_stats == 0.999


def test_bytes_per_element_cover_every_stage():
    b = bench.bytes_per_element(16)
    for stage in ("amax", "quantize", "quantize_search", "quantize_mse", "quantize_mse_dequantize", "dequantize",
                  "block_mse", "outlier_stats"):
        assert b[stage] > 0
    assert b["quantize_mse_dequantize"] == 2.0 + 0.5 + 1 / 16 + 4 / 16 + 2.0


@pytest.mark.parametrize("extra", [[], ["--scale-search", "2,1"],
                                   ["--workload", "rotated_activations_8192x5120", "--rot", "0",
                                    "--outlier-stats", "0.999"]])
def test_reference_arm_line(extra, capsys, monkeypatch):
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"] + extra)) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    if "--scale-search" in extra:
        assert "MSE search" in line["config"]["block_scales"]
    if "--outlier-stats" in extra:
        assert "P99.9" in line["config"]["outlier_stats"]


def test_cpu_baseline_single_core_and_all_cores():
    args = bench.parse_args(["--cpu-seconds", "0.3"])
    cb = bench.cpu_baseline("nvfp4_qwen25_7b_mlp", args)
    assert cb["cores"] == 1 and cb["kind"] == "oracle" and cb["value"] > 0
    ac = cb["all_cores"]
    assert "unavailable" not in ac, ac
    assert ac["value"] > 0 and 1 <= ac["cores"] <= bench.MAX_ORACLE_PROCS
