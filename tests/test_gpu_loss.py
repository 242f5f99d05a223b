"""GPU parity of the training forward (teacher forcing + base-anchored curriculum
loss) through the C ABI, against oracle/training.py.

Tolerances: on given fp32 logits the kernels are compared with fp64
cross-entropy of the same values (log-sum-exp in fp32 chunks merged in fp64:
1e-4 absolute per position).  End to end, each cross-entropy moves by at most
twice the logits' max-abs error (|d lse| <= max |dL|, plus the label's logit),
so the bound is 2 x the block's logit tolerance (2e-2 bf16, 1e-4 fp32).
"""
import numpy as np
import pytest
import torch

import draft_model_b200 as dm
import oracle
import synth
from _harness import TOL, aligned_workspace, device_weights, to_dev

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _loss_on(final, base, labels, lam, gamma):
    B, K, V = final.shape
    ws = aligned_workspace(dm.domino_curriculum_loss_workspace_bytes(B, K, V))
    loss = torch.zeros(4, dtype=torch.float32, device="cuda")
    ce = torch.zeros((B, K, 2), dtype=torch.float32, device="cuda")
    dm.domino_curriculum_loss(final, base, labels, lam=lam, gamma=gamma, loss_out=loss, ce_out=ce, workspace=ws)
    status = dm.domino_poll(ws)
    return float(loss[0].item()), ce.cpu().numpy().astype(np.float64), status


@cuda
@pytest.mark.parametrize("B,K,V,lam,gamma", [(3, 5, 5000, 0.3, 0.8), (1, 16, 151936, 1.0, 0.9),
                                             (2, 16, 151936, 0.0, 1.0), (17, 3, 777, 0.5, 0.5), (1, 1, 7, 0.5, 1.0)])
def test_curriculum_loss_kernel_on_given_logits(B, K, V, lam, gamma):
    rng = np.random.default_rng(B * 1000 + K)
    final = rng.normal(0.0, 4.0, size=(B, K, V)).astype(np.float32)
    base = rng.normal(0.0, 4.0, size=(B, K, V)).astype(np.float32)
    labels = rng.integers(0, V, size=(B, K)).astype(np.int32)
    loss, ce, status = _loss_on(torch.from_numpy(final).cuda(), torch.from_numpy(base).cuda(),
                                torch.from_numpy(labels).cuda(), lam, gamma)
    assert status == 0
    ref, cf, cb = oracle.curriculum_loss(final.astype(np.float64), base.astype(np.float64), labels, lam, gamma)
    assert np.abs(ce[..., 0] - cf).max() < 1e-4
    assert np.abs(ce[..., 1] - cb).max() < 1e-4
    assert abs(loss - ref) <= 1e-4 * max(1.0, abs(ref))


@cuda
def test_curriculum_loss_extreme_rows():
    # one dominant logit (CE ~ 0 or ~ 80), a uniform row (CE = log V), large offsets
    V = 4096
    final = np.zeros((1, 3, V), dtype=np.float32)
    final[0, 0, 17] = 80.0
    final[0, 2] = 1000.0
    base = final.copy()
    labels = np.array([[17, 5, 4095]], dtype=np.int32)
    loss, ce, status = _loss_on(torch.from_numpy(final).cuda(), torch.from_numpy(base).cuda(),
                                torch.from_numpy(labels).cuda(), 0.5, 1.0)
    assert status == 0
    np.testing.assert_allclose(ce[0, :, 0], [0.0, np.log(V), np.log(V)], atol=1e-4)
    final[0, 0, 17] = 0.0
    final[0, 0, 18] = 80.0
    _, ce2, _ = _loss_on(torch.from_numpy(final).cuda(), torch.from_numpy(base).cuda(),
                         torch.from_numpy(labels).cuda(), 0.5, 1.0)
    assert abs(ce2[0, 0, 0] - 80.0) < 1e-3


@cuda
def test_bad_label_is_flagged():
    final = torch.zeros((1, 2, 100), device="cuda")
    labels = torch.tensor([[3, 100]], dtype=torch.int32, device="cuda")
    _, _, status = _loss_on(final, final, labels, 0.5, 1.0)
    assert status == 6   # DOMINO_ERR_BAD_TOKEN


def _draft_loss(dw, hidden, anchor, labels, lam, gamma, dtype):
    B, K = labels.shape
    ws = aligned_workspace(dm.domino_draft_loss_workspace_bytes(dw, B, K))
    loss = torch.zeros(4, dtype=torch.float32, device="cuda")
    ce = torch.zeros((B, K, 2), dtype=torch.float32, device="cuda")
    dm.domino_draft_loss(dw, to_dev(hidden, dtype), torch.from_numpy(anchor).cuda(), torch.from_numpy(labels).cuda(),
                         lam=lam, gamma=gamma, loss_out=loss, ce_out=ce, workspace=ws)
    return float(loss[0].item()), ce.cpu().numpy().astype(np.float64), dm.domino_poll(ws)


def _small(**kw):
    base = dict(name="small", B=3, K=5, d=200, V=5000, H=64, r=32, E=136, dtype="bf16", tied=False, seed=1)
    base.update(kw)
    return synth.Config(**base)


@cuda
@pytest.mark.parametrize("cfg,lam,gamma", [
    (synth.CONFIGS["tiny_f32"], 0.4, 0.9),
    (_small(), 0.3, 0.8),                         # persistent loop (B < 4)
    (_small(B=9, K=7, seed=5), 1.0, 0.7),         # tensor-core loop
    (_small(B=5, K=6, dtype="f32", seed=9), 0.0, 1.0),
], ids=["tiny_f32", "bf16_b3", "bf16_b9_tc", "f32_b5"])
def test_draft_loss_matches_oracle(cfg, lam, gamma):
    w = synth.make_weights(cfg)
    m = oracle.Model.from_storage(w)
    dw = device_weights(w)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    labels = np.random.default_rng(cfg.seed + 100).integers(0, cfg.V, size=(cfg.B, cfg.K)).astype(np.int32)
    loss, ce, status = _draft_loss(dw, hidden, anchor, labels, lam, gamma, cfg.dtype)
    assert status == 0
    ref, cf, cb, _ = oracle.train_forward(m, hidden, anchor, labels, lam, gamma)
    bound = 2 * TOL[cfg.dtype]
    assert np.abs(ce[..., 0] - cf).max() <= bound
    assert np.abs(ce[..., 1] - cb).max() <= bound
    assert abs(loss - ref) <= bound


@cuda
def test_draft_loss_full_size_b1():
    cfg = synth.CONFIGS["qwen3_8b_b1"]
    w = synth.make_weights(cfg)
    m = oracle.Model.from_storage(w)
    dw = device_weights(w)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    labels = np.random.default_rng(7).integers(0, cfg.V, size=(cfg.B, cfg.K)).astype(np.int32)
    loss, ce, status = _draft_loss(dw, hidden, anchor, labels, 0.5, 0.9, cfg.dtype)
    assert status == 0
    ref, cf, cb, _ = oracle.train_forward(m, hidden, anchor, labels, 0.5, 0.9)
    bound = 2 * TOL[cfg.dtype]
    assert np.abs(ce[..., 0] - cf).max() <= bound
    assert np.abs(ce[..., 1] - cb).max() <= bound
    assert abs(loss - ref) <= bound
