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


class _FakeStream:
    cuda_stream = 0


class _FakeLib:
    """Stands in for libfp4q.so's entry points: records the calls a step makes."""

    def __init__(self):
        self.log = []

    def __getattr__(self, name):
        def fn(*args):
            self.log.append((name, args[0]))
            return 0
        return fn


class _FakeFq:
    def __init__(self):
        self.L = _FakeLib()
        import microscaling_fp4_quantization_block_b200 as m
        self.Fp4qTensor = m.Fp4qTensor

    def lib(self):
        return self.L

    @staticmethod
    def fp4q_quantize_batch_workspace_size(count):
        return 64 * count

    @staticmethod
    def fp4q_block_mse_workspace_size(rows, cols, block):
        return 64


def test_weight_pass_schedule():
    """Variant by variant, layer by layer; in each layer group the amax passes of
    the NVFP4 variants come before the quantizer passes, and every call of
    every item runs exactly once per step."""
    import torch
    xs = [(f"L{l}.{t}", torch.zeros((2, 64), dtype=torch.bfloat16)) for l in range(3) for t in "abc"]
    items, groups = bench.weight_pass_items(xs, 3)
    assert len(items) == 4 * 9 and len(groups) == 4 * 3
    assert [bench.item_tag(lbl) for lbl, *_ in items[::9]] == [v[0] for v in bench.WEIGHT_PASS_VARIANTS]
    fq = _FakeFq()
    pipe = bench.Pipeline(fq, items, "cpu", _FakeStream(), groups=groups)
    fq.L.log.clear()
    pipe.step(_FakeStream())
    names = [n for n, _ in fq.L.log]
    n_nv = sum(1 for v in bench.WEIGHT_PASS_VARIANTS if v[4] == 1)
    # one batched amax call per NVFP4 layer group, then one batched quantizer call on the same tensors
    assert names.count("fp4q_tensor_amax_batched") == 3 * n_nv
    assert names.count("fp4q_tensor_amax_accumulate") == 0
    assert names.count("fp4q_quantize_mse_dequantize_batched") == 12
    assert names.count("fp4q_quantize_mse_dequantize") == 0
    assert pipe.launches_per_step == 12 + 3 * n_nv
    steps = [(bench.stage_kind(st), idx) for st, _, _, idx in pipe.step_calls]
    nv_first = next(j for j, (kind, _) in enumerate(steps) if kind == "amax")
    grp = steps[nv_first:nv_first + 2]
    assert [k for k, _ in grp] == ["amax", "quantize_mse_dequantize"]
    assert grp[0][1] == grp[1][1]
    args = pipe.step_calls[nv_first][2]
    assert args[0] == 3 and args[6] == 1                       # three tensors, accumulating into zeroed slots
    assert list(args[3]) == [items[i][1].shape[1] for i in grp[0][1]]
    assert list(args[5]) == [pipe.bufs[i]["gscale"].data_ptr() for i in grp[0][1]]
    qargs = pipe.step_calls[nv_first + 1][2]
    assert qargs[0] == 3 and qargs[2:6] == (1, 16, items[grp[0][1][0]][4], bench.FROM_AMAX)
    assert [qargs[1][j].gscale for j in range(3)] == [pipe.bufs[i]["gscale"].data_ptr() for i in grp[0][1]]
    assert [qargs[1][j].terms for j in range(3)] == [pipe.bufs[i]["terms"].data_ptr() for i in grp[0][1]]
    mx = next(st for st in pipe.step_calls if st[0].endswith("mxfp4_rot0"))
    assert mx[2][2:6] == (0, 32, 0, bench.NONE) and mx[2][1][0].gscale is None
    # the per-tensor form: three amax calls, then three quantizer calls on the same tensors
    fq2 = _FakeFq()
    pipe2 = bench.Pipeline(fq2, items, "cpu", _FakeStream(), groups=groups, batch_amax=False, batch_quantize=False)
    fq2.L.log.clear()
    pipe2.step(_FakeStream())
    names2 = [n for n, _ in fq2.L.log]
    assert names2.count("fp4q_tensor_amax_accumulate") == 9 * n_nv
    assert names2.count("fp4q_quantize_mse_dequantize") == 36
    assert pipe2.launches_per_step == 36 + 9 * n_nv
    order = [(bench.stage_kind(pipe2.calls[i][k][0]), i) for i, k in pipe2.order]
    nv_first = next(j for j, (kind, _) in enumerate(order) if kind == "amax")
    grp = order[nv_first:nv_first + 6]
    assert [k for k, _ in grp] == ["amax"] * 3 + ["quantize_mse_dequantize"] * 3
    assert [i for _, i in grp[:3]] == [i for _, i in grp[3:]]
    # one dequantized-output buffer per input tensor, shared by the variants
    assert len({b["deq"].data_ptr() for b in pipe.bufs}) == 9
    # stage names carry the variant
    assert {bench.item_tag(lbl) for lbl, *_ in items} == {st.split("@")[1] for st, *_ in pipe.step_calls}


def test_weight_pass_and_sweep_defaults():
    a = bench.parse_args([])
    assert a.workload == "qwen25_14b_weight_pass" and a.steps >= 3 and a.warmup >= 3
    assert a.layers is None and not a.no_batch_quantize and not a.no_batch_amax and not a.no_graph
    a = bench.parse_args(["--layers", "2", "--no-batch-quantize"])
    assert a.layers == 2 and a.no_batch_quantize
    a = bench.parse_args(["--workload", "block_size_sweep_4096", "--steps", "7"])
    assert a.steps == 7 and a.warmup == bench.WORKLOAD_DEFAULTS["block_size_sweep_4096"]["warmup"]


def test_reference_arm_sweep(capsys, monkeypatch):
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0",
                                                 "--workload", "block_size_sweep_4096"])) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"]["workload"] == "block_size_sweep_4096"


def test_ncu_traffic_follows_the_kernel_sources(monkeypatch):
    """The roofline's measured traffic is read from the committed counters only
    while the kernel sources they were taken on are unchanged; otherwise, and
    for a kernel without counters, the line carries null."""
    import os
    with open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as f:
        table = json.load(f)
    wl = "qwen25_14b_weight_pass"
    for kernel, e in table[wl].items():
        assert e["csrc_files"] and 1.9 < e["dram_bytes_per_element"] < 5.0, kernel
        v = bench.ncu_traffic(kernel, wl)
        if e["csrc_sha"] == bench.csrc_hash(e["csrc_files"]):
            assert v == e["dram_bytes_per_element"], kernel
        else:
            assert v is None, kernel
    assert bench.ncu_traffic("no_such_kernel@x", wl) is None
    assert bench.ncu_traffic("amax@nvfp4_rot0", "no_such_workload") is None
    monkeypatch.setattr(bench, "csrc_hash", lambda files=None: "0" * 16)
    assert all(bench.ncu_traffic(k, wl) is None for k in table[wl])
