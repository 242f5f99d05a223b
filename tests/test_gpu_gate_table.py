"""GPU checks of the token->gate table variant: the table against its fp64
definition G[t] = W_ih E[t] + b_ih, and draft blocks through the batched loop
that gathers table rows instead of multiplying W_ih, against the oracle (which
always multiplies W_ih: the two agree up to fp32 summation order)."""
import numpy as np
import pytest
import torch

import draft_model_b200 as dm
import oracle
import synth
from _harness import aligned_workspace, check_against_oracle, device_weights, run_gpu

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _small(**kw):
    base = dict(name="small", B=9, K=7, d=200, V=5000, H=64, r=32, E=136, dtype="bf16", tied=False, seed=5)
    base.update(kw)
    return synth.Config(**base)


def _table(dw):
    t = torch.empty((dw.V, 3 * dw.H), dtype=torch.float32, device="cuda")
    assert dm.domino_gate_table_bytes(dw) == t.numel() * 4
    ws = aligned_workspace(1024)
    dm.domino_build_gate_table(dw, t, workspace=ws)
    assert dm.domino_poll(ws) == 0
    return t


def _reference_rows(w, tokens):
    m = oracle.Model.from_storage(w)
    x = m.embed_rows(np.asarray(tokens))
    g = x @ m.w_ih.T
    return g + (m.b_ih if m.b_ih is not None else 0.0)


@cuda
@pytest.mark.parametrize("cfg", [_small(), _small(dtype="f32", V=3001, seed=6), _small(d=136, E=136, tied=True)],
                         ids=["bf16", "f32", "tied"])
def test_gate_table_matches_definition(cfg):
    w = synth.make_weights(cfg)
    dw = device_weights(w)
    t = _table(dw).cpu().numpy().astype(np.float64)
    ref = _reference_rows(w, np.arange(cfg.V))
    assert np.abs(t - ref).max() < 1e-4


@cuda
def test_gate_table_full_size_sampled_rows():
    cfg = synth.CONFIGS["qwen3_8b_b1"]
    w = synth.make_weights(cfg)
    dw = device_weights(w)
    t = _table(dw)
    rows = np.random.default_rng(0).integers(0, cfg.V, size=64)
    got = t[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    assert np.abs(got - _reference_rows(w, rows)).max() < 1e-4


@cuda
@pytest.mark.parametrize("cfg", [_small(), _small(B=17, K=5, mode="gumbel", temperature=1.0, seed=8),
                                 _small(B=1, K=16, seed=10), _small(B=3, K=8, mode="gumbel", temperature=0.8, seed=11),
                                 synth.CONFIGS["tiny_f32"]],
                         ids=["greedy_b9", "gumbel_b17", "persistent_b1", "persistent_gumbel_b3", "tiny_f32"])
def test_block_with_gate_table(cfg):
    w = synth.make_weights(cfg)
    m = oracle.Model.from_storage(w)
    dw = device_weights(w)
    n0 = dm.domino_launches_per_block(dw, cfg.B, cfg.K)
    dw.set_gate_table(_table(dw))
    # the batched loop drops the first position's gate GEMM; the persistent loop's count is unchanged
    assert dm.domino_launches_per_block(dw, cfg.B, cfg.K) == (n0 - 1 if cfg.B >= 4 and cfg.dtype == "bf16" else n0)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    gpu = run_gpu(dw, cfg, hidden, anchor)
    assert gpu["status"] == 0
    _, stats = check_against_oracle(m, cfg, hidden, anchor, gpu)
    assert stats["agree"] > 0.5


@cuda
def test_block_with_gate_table_full_size_b1():
    cfg = synth.CONFIGS["qwen3_8b_b1"]
    w = synth.make_weights(cfg)
    m = oracle.Model.from_storage(w)
    dw = device_weights(w)
    dw.set_gate_table(_table(dw))
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    gpu = run_gpu(dw, cfg, hidden, anchor)
    assert gpu["status"] == 0
    check_against_oracle(m, cfg, hidden, anchor, gpu)


@cuda
def test_block_with_gate_table_full_size_b32_sampled():
    cfg = synth.CONFIGS["qwen3_8b_b32_gumbel"]
    w = synth.make_weights(cfg)
    m = oracle.Model.from_storage(w)
    dw = device_weights(w)
    dw.set_gate_table(_table(dw))
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    gpu = run_gpu(dw, cfg, hidden, anchor)
    assert gpu["status"] == 0
    check_against_oracle(m, cfg, hidden, anchor, gpu, rows=[0, 13, 31])
