"""bench.py's reference arm on CPU: one JSON line with the keys the benchmark contract names,
printed by rank 0 only (the other ranks exit 0 without work). The arm times the CPU oracle,
so this runs without a GPU; the GPU arm's line is checked by the GPU runs themselves."""
import json
import os
import subprocess
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]
CMD = [sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--workload", "tiny",
       "--steps", "2", "--warmup", "1", "--cpu-seconds", "1"]


def run(env_extra):
    env = dict(os.environ)
    env.update(env_extra)
    env.pop("CUDA_VISIBLE_DEVICES", None)
    r = subprocess.run(CMD, capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    lines = run({"RANK": "0", "WORLD_SIZE": "1", "LOCAL_RANK": "0"})
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["metric"] == "MoE-layer forward tokens/s" and d["unit"] == "tokens/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["vs_baseline"] is None
    assert "tiny" in d["config"]["workload"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["unit"] == d["unit"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_no_work():
    assert run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_roofline_fractions_follow_the_sampled_clock():
    """The tensor peak regime is read from the median sampled SM clock (burst at >= 0.9 of
    the maximum, sustained below), and the line carries the burst and clock-scaled fractions
    too, so each can be recomputed from the JSON line and the measured peaks."""
    sys.path.insert(0, str(ROOT))
    import bench

    peaks = {"hbm_gbs": 6520.2, "bf16_tflops": 1656.8, "bf16_tflops_sustained": 1388.7}
    # a short run at the maximum clock, a few power-cap samples: burst
    hot = {"sm_mhz": 1942.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    d = bench.tensor_fracs(1333.0, peaks, hot)
    assert d["regime"] == "burst" and d["peak"] == 1656.8
    assert abs(d["frac"] - 1333.0 / 1656.8) < 1e-12 and d["frac"] == d["frac_burst"]
    assert abs(d["frac_clock_scaled"] - 1333.0 / (1656.8 * 1942.0 / 1965.0)) < 1e-12
    # a long run settled under the cap: sustained
    capped = {"sm_mhz": 1340.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    d = bench.tensor_fracs(1100.0, peaks, capped)
    assert d["regime"] == "sustained" and d["peak"] == 1388.7
    assert abs(d["frac_burst"] - 1100.0 / 1656.8) < 1e-12
    # no clock record: burst, no clock-scaled figure
    d = bench.tensor_fracs(1000.0, peaks, None)
    assert d["regime"] == "burst" and "frac_clock_scaled" not in d
    # e4m3: twice the bf16 figures
    d = bench.tensor_fracs(2000.0, peaks, hot, fp8=True)
    assert d["peak"] == 2 * 1656.8


def test_layer0_roofline_bound_and_bytes():
    """Separate launches: layer0's useful FLOPs 4TkHF (SwiGLU) and its algorithmic bytes; the
    persistent launch: both GEMMs' FLOPs 6TkHF and the compulsory bytes."""
    sys.path.insert(0, str(ROOT))
    import bench
    from mixture_experts_layer_forward_b200 import synth

    cfg = synth.CONFIGS["mixtral"]
    peaks = {"hbm_gbs": 6520.2, "bf16_tflops": 1656.8, "bf16_tflops_sustained": 1388.7}
    r = bench.layer0_roofline(cfg, 2.9, 8, peaks, "measured", None, False, "k")
    T, k, H, F = cfg.T, cfg.k, cfg.H, cfg.F
    assert r["algorithmic_flops_per_launch"] == 4 * T * k * H * F
    assert r["algorithmic_bytes_per_launch"] == 2 * (8 * H * 2 * F + T * H) + 2 * T * k * F
    assert r["bound"] == "tensor"
    r = bench.layer0_roofline(cfg, 4.6, 8, peaks, "measured", None, False, "k", fused=True)
    assert r["algorithmic_flops_per_launch"] == 6 * T * k * H * F
    assert r["algorithmic_bytes_per_launch"] == 2 * (8 * H * 3 * F + T * k * H) + 2 * T * H
    decode = synth.CONFIGS["skew_decode"]
    r = bench.layer0_roofline(decode, 0.46, 49, peaks, "measured", None, False, "k")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    # the whole layer in one launch: + the router's FLOPs and its reads of x and W_g
    E = cfg.E
    r = bench.layer0_roofline(cfg, 4.75, 8, peaks, "measured", None, False,
                              "moe_fused_layer_kernel<0, true>", fused=True, whole=True)
    assert r["algorithmic_flops_per_launch"] == 6 * T * k * H * F + 2 * T * H * E
    assert r["algorithmic_bytes_per_launch"] == (2 * (8 * H * 3 * F + T * k * H) + 2 * T * H +
                                                 2 * T * H + 2 * H * E)
    assert abs(r["achieved"] - r["algorithmic_flops_per_launch"] / 4.75e-3 / 1e12) < 1e-6


def test_traffic_is_read_only_for_unchanged_sources():
    """roofline.traffic comes from profiles/traffic.json only while the kernel's sources hash
    to the value recorded with the counters; the committed entries match the tree."""
    sys.path.insert(0, str(ROOT))
    import bench

    d = json.loads((ROOT / "profiles" / "traffic.json").read_text())
    for kernel, per in d.items():
        for name, ent in per.items():
            assert bench.traffic_for(kernel, name) == ent["bytes_per_launch"], (kernel, name)
    assert bench.traffic_for("moe_fused_layer_kernel<0, true>", "mixtral") > 0
    assert bench.traffic_for("no_such_kernel", "mixtral") is None


def test_profile_commands_parse_with_the_current_bench():
    """Every bench.py command quoted in profiles/ must still run: its flags parse with
    bench.py's own parser, its workload exists, and any other script it names is committed."""
    import re

    sys.path.insert(0, str(ROOT))
    import bench
    from mixture_experts_layer_forward_b200 import synth

    def expand(cmd):
        """Each `for W in a b c; do ... done` loop, unrolled over its values."""
        loop = re.search(r"for (\w+) in ([^;]+); do(.*?)done", cmd, re.S)
        if not loop:
            return [cmd]
        var, values, body = loop.group(1), loop.group(2).split(), loop.group(3)
        return [c for v in values
                for c in expand(cmd[:loop.start()] + body.replace("$" + var, v) + cmd[loop.end():])]

    def bench_commands():
        for md in sorted((ROOT / "profiles").glob("*.md")):
            for block in re.findall(r"```\n(.*?)```", md.read_text(), re.S):
                for cmd in expand(block.replace("\\\n", " ")):
                    for m in re.finditer(r"python (\S+\.py)([^\n&|>]*)", cmd):
                        yield md.name, m.group(1), m.group(2).split()

    checked = 0
    for name, script, args in bench_commands():
        assert (ROOT / script).is_file(), f"{name}: {script} is not in the tree"
        if script != "bench.py":
            continue
        old = sys.argv
        sys.argv = ["bench.py", *args]
        try:
            parsed = bench.parse_args()
        finally:
            sys.argv = old
        assert parsed.workload in synth.CONFIGS, f"{name}: {parsed.workload}"
        checked += 1
    assert checked >= 10
