"""The JSON line bench.py prints: every key its consumers read, with sane values.

The reference arm (the fp64 oracle on a bounded sample) runs on CPU; the GPU arm is run on
the tiny workload (marked gpu).
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
COMMON = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
          "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e"}


def _run(args, timeout):
    env = dict(os.environ, PYTHONPATH=ROOT)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         env=env, capture_output=True, text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "0",
              "--reference-budget-s", "4"], timeout=600)
    assert COMMON <= set(d)
    assert d["impl"] == "reference"
    assert d["warmup"] >= 3 and d["steps"] == 2
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


@pytest.mark.parametrize("workload,unit", [("qk_prologue", "GB/s"), ("na3d_decoder", "TFLOP/s")])
def test_reference_arm_line_other_workloads(workload, unit):
    d = _run(["--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "0",
              "--reference-budget-s", "2"], timeout=600)
    assert COMMON <= set(d) and d["impl"] == "reference" and d["dtype"] == "f64"
    assert d["unit"] == unit and d["value"] > 0 and d["config"]["workload"] == workload
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


@pytest.mark.gpu
def test_gpu_arm_line():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d = _run(["--workload", "tiny", "--steps", "3", "--warmup", "3", "--cpu-seconds", "2"],
             timeout=900)
    assert COMMON <= set(d) and "impl" not in d
    assert d["n_gpus"] == 1 and d["scaling"] == "weak" and d["dtype"] == "bf16"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    r = d["roofline"]
    assert r["bound"] in ("tensor", "hbm") and r["achieved"] > 0 and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    # four calls per step in three launches: audio self-attention and a2v share one grouped
    # launch (no key-range parts at these sizes)
    assert d["launch_items"] == [["video_self"], ["audio_self", "a2v"], ["v2a"]]
    assert d["gpu_launches"] == 3 * d["steps"]
    assert set(d["per_call"]) == {"video_self", "audio_self", "v2a", "a2v"}
    for name in ("audio_self", "a2v"):
        g = d["per_call"][name]["group"]
        assert g["members"] == ["audio_self", "a2v"] and g["us_median"] > 0
    for name, pc in d["per_call"].items():  # the timed outputs against the oracle
        par = pc["parity"]
        assert par["finite"] and par["max_abs"] <= 2e-2 and par["rel_l2"] <= 5e-3, (name, par)
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] > 0


@pytest.mark.gpu
@pytest.mark.parametrize("workload,unit", [("na3d_decoder", "TFLOP/s"), ("qk_prologue", "GB/s")])
def test_gpu_arm_line_other_workloads(workload, unit):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d = _run(["--workload", workload, "--steps", "3", "--warmup", "3", "--cpu-seconds", "1"],
             timeout=900)
    assert COMMON <= set(d) and "impl" not in d
    assert d["unit"] == unit and d["value"] > 0 and d["config"]["workload"] == workload
    r = d["roofline"]
    assert r["achieved"] > 0 and r["peak"] > 0 and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == d["steps"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] > 0


@pytest.mark.gpu
def test_gpu_arm_per_config_table():
    # the headline workload also times every other config and next-row workload on its own,
    # each with parity against the oracle on sampled rows
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d = _run(["--steps", "3", "--warmup", "3", "--per-config-steps", "2", "--cpu-seconds", "1"],
             timeout=1500)
    assert d["config"]["workload"] == "block768"
    pc = d["per_config"]
    assert set(pc) == {"tiny", "video15360_b1", "audio_stream", "longclip", "text_xattn",
                       "qk_prologue", "na3d_decoder"}
    pars = [c["parity"] for cfg in pc.values() if "calls" in cfg for c in cfg["calls"].values()]
    pars += [pc["qk_prologue"]["parity"], pc["na3d_decoder"]["parity"]]
    pars += [c["parity"] for c in d["per_call"].values()]
    for par in pars:
        assert par["finite"] and par["max_abs"] <= 2e-2 and par["rel_l2"] <= 5e-3, par
    for cfg in pc.values():
        for c in cfg.get("calls", {"_": cfg}).values():
            assert c["us_p10"] <= c["us_median"] <= c["us_p90"]
    assert pc["na3d_decoder"]["density"] > 0 and pc["qk_prologue"]["frac_hbm"] > 0


@pytest.mark.gpu
def test_gpu_arm_context_parallel_line():
    # context-parallel mode on one GPU: a one-rank NCCL group, the long clip's video self and
    # v2a through the partial + merge path, with parity against the oracle on sampled rows
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d = _run(["--cp", "--steps", "2", "--warmup", "3", "--cpu-seconds", "1"], timeout=1500)
    assert COMMON <= set(d) and d["scaling"] == "strong" and d["n_gpus"] == 1
    assert d["config"]["workload"] == "cp_longclip" and d["value"] > 0
    for name, par in d["parity"].items():
        assert par["finite"] and par["max_abs"] <= 2e-2 and par["rel_l2"] <= 5e-3, (name, par)
    assert d["gpu_launches"] == 4 * d["steps"]  # one shard: partial + merge, v2a: partial + merge


def test_launch_items_group_the_one_tile_head_dim_64_calls():
    import bench
    from joint_audio_video_flash_b200 import workloads
    _, calls = workloads.configs()["block768"]
    assert bench.launch_items(calls) == [[0], [1, 3], [2]]
    assert bench.launch_items(calls, grouped=False) == [[0], [1], [2], [3]]
    # the long clip's audio side has 252 valid keys (two tiles): nothing to group
    _, calls = workloads.configs()["longclip"]
    assert bench.launch_items(calls) == [[0], [1], [2], [3]]
    assert bench.item_launches([1, 3], [1, 1, 4, 1]) == 1
    assert bench.item_launches([2], [1, 1, 4, 1]) == 2      # key split + merge
    assert bench.item_launches(list(range(6)), [1] * 6) == 2  # four calls per launch


def test_group_share_splits_the_grouped_launch():
    import bench
    # interleaved loop: group 80-82 µs; without audio self (index 1) 77-78; without a2v (3) 12-13
    mu = {("group", 0): [80.0, 82.0, 81.0],
          ("alone", 1): [10.0, 10.0, 11.0], ("alone", 3): [70.0, 71.0, 70.0],
          ("without", 1): [77.0, 78.0, 77.0], ("without", 3): [12.0, 12.0, 13.0]}
    item = [1, 3]
    assert bench.group_base(item, mu) == 3                     # a2v: the longer own launch
    audio = bench.group_share(item, 1, mu, [item])
    a2v = bench.group_share(item, 3, mu, [item])
    assert audio == [3.0, 4.0, 4.0]                            # what audio self adds
    assert a2v == [77.0, 78.0, 77.0]                           # the rest of the group
    assert [x + y for x, y in zip(audio, a2v)] == mu[("group", 0)]
