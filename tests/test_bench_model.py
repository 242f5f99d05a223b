"""The roofline denominators bench.py reports: algorithmic bytes and flops of a
draft block, checked against the arithmetic of the Qwen3 shapes written out by
hand (V = 151936, H = 1024, r = 256, block 16; d = E = 4096 for 8B, 2560 for 4B); and the
reference arm's JSON line (the oracle timed on the host cores)."""
import importlib.util
import json
import os
import sys

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv, sys.argv = sys.argv, ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_loop_bytes_qwen3_8b():
    b = _bench()
    cfg = synth.CONFIGS["qwen3_8b_b1"]
    # per step, read once: W2 151936x256 + W1 256x(4096+1024) + W_ih 3072x4096 + W_hh 3072x1024, bf16
    per_step = (151936 * 256 + 256 * 5120 + 3072 * 4096 + 3072 * 1024) * 2
    assert per_step == 111_869_952
    # per request per step: the fp32 base-logit row, h_i and the fed embedding (bf16)
    per_req = 151936 * 4 + 4096 * 2 + 4096 * 2
    assert per_req == 624_128
    assert b.loop_bytes(cfg, 1) == 16 * (per_step + per_req) == 1_799_905_280
    assert b.loop_bytes(synth.sweep_config(256), 256) == 16 * (per_step + 256 * per_req)


def test_loop_bytes_qwen3_4b():
    b = _bench()
    cfg = synth.CONFIGS["qwen3_4b_b1"]
    per_step = (151936 * 256 + 256 * (2560 + 1024) + 3072 * 2560 + 3072 * 1024) * 2
    per_req = 151936 * 4 + 2560 * 2 + 2560 * 2
    assert b.loop_bytes(cfg, 1) == 16 * (per_step + per_req)
    assert abs(b.loop_bytes(cfg, 1) / 1e9 - 1.636) < 0.001


def test_lm_head_bytes_and_flops():
    b = _bench()
    cfg = synth.CONFIGS["qwen3_8b_b1"]
    assert b.lm_head_bytes(cfg, 1) == 151936 * 4096 * 2 + 16 * 4096 * 2 + 16 * 151936 * 4
    assert abs(b.lm_head_bytes(cfg, 1) / 1e9 - 1.255) < 0.001
    assert b.lm_head_flops(cfg, 32) == 2 * 16 * 32 * 151936 * 4096
    assert abs(b.lm_head_flops(cfg, 1) / 1e9 - 19.9) < 0.05


def _run_bench(args, env_extra=None):
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE")}
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the oracle on the host cores and prints
    one JSON line with the same metric, unit and workload as the GPU arm."""
    bench = _bench()
    r = _run_bench(["--impl", "reference", "--steps", "2", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1 and line["value"] > 0
    assert line["config"]["workload"] == bench.WORKLOAD.format(B=1)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["vs_baseline"] is None


def test_reference_arm_other_ranks_exit_without_work():
    r = _run_bench(["--impl", "reference", "--steps", "2", "--warmup", "3"],
                   {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and r.stdout.strip() == ""
