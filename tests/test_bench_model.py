"""The roofline denominators bench.py reports: algorithmic bytes and flops of a
draft block, checked against the arithmetic of the Qwen3 shapes written out by
hand (V = 151936, H = 1024, r = 256, block 16; d = E = 4096 for 8B, 2560 for 4B)."""
import importlib.util
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
