"""Pins of the training-loss oracle (oracle/training.py) against closed forms, an
independent library implementation and the limits of its curriculum mix.
CPU only."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import Model, cross_entropy_rows, curriculum_loss, draft_block, position_weights, train_forward


def test_ce_of_uniform_rows_is_log_v():
    for V in (2, 7, 151936):
        x = np.full((3, V), 2.5)
        np.testing.assert_allclose(cross_entropy_rows(x, np.array([0, V // 2, V - 1])), math.log(V), rtol=0,
                                   atol=1e-12)


def test_ce_two_way_closed_form():
    a, b = 1.25, -3.0
    x = np.array([[a, b], [a, b]])
    ce = cross_entropy_rows(x, np.array([0, 1]))
    np.testing.assert_allclose(ce, [math.log1p(math.exp(b - a)), math.log1p(math.exp(a - b))], rtol=1e-13)


def test_ce_matches_torch_cross_entropy():
    rng = np.random.default_rng(0)
    x = rng.normal(0.0, 20.0, size=(5, 7, 300))
    y = rng.integers(0, 300, size=(5, 7))
    ref = torch.nn.functional.cross_entropy(torch.from_numpy(x).reshape(-1, 300), torch.from_numpy(y).reshape(-1),
                                            reduction="none").numpy().reshape(5, 7)
    np.testing.assert_allclose(cross_entropy_rows(x, y), ref, rtol=1e-12, atol=1e-12)


def test_ce_shift_invariance():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(4, 50))
    y = rng.integers(0, 50, size=4)
    np.testing.assert_allclose(cross_entropy_rows(x + 123.0, y), cross_entropy_rows(x, y), atol=1e-11)


def test_position_weights():
    np.testing.assert_array_equal(position_weights(5, 1.0), np.ones(5))
    np.testing.assert_allclose(position_weights(4, 0.5), [1.0, 0.5, 0.25, 0.125])


def test_curriculum_mix_and_weights_by_hand():
    rng = np.random.default_rng(2)
    B, K, V = 2, 3, 11
    fin, base = rng.normal(size=(B, K, V)), rng.normal(size=(B, K, V))
    y = rng.integers(0, V, size=(B, K))
    cf, cb = cross_entropy_rows(fin, y), cross_entropy_rows(base, y)
    w = np.array([1.0, 0.8, 0.64])
    lf = sum(w[i] * cf[b, i] for b in range(B) for i in range(K)) / (B * w.sum())
    lb = sum(w[i] * cb[b, i] for b in range(B) for i in range(K)) / (B * w.sum())
    for lam in (0.0, 0.3, 1.0):
        loss, _, _ = curriculum_loss(fin, base, y, lam, 0.8)
        assert loss == pytest.approx((1 - lam) * lf + lam * lb, rel=1e-14)
    # gamma = 1: plain mean over batch and positions
    loss, _, _ = curriculum_loss(fin, base, y, 0.0, 1.0)
    assert loss == pytest.approx(cf.mean(), rel=1e-14)


def _tiny():
    cfg = synth.CONFIGS["tiny_f32"]
    w = synth.make_weights(cfg)
    return cfg, w, Model.from_storage(w)


def test_train_forward_is_the_teacher_forced_block():
    cfg, w, m = _tiny()
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    labels = np.random.default_rng(3).integers(0, cfg.V, size=(cfg.B, cfg.K)).astype(np.int32)
    loss, cf, cb, res = train_forward(m, hidden, anchor, labels, 0.25, 0.9)
    ref = draft_block(m, hidden, anchor, forced=labels)
    np.testing.assert_array_equal(res.logits, ref.logits)
    np.testing.assert_allclose(cf, cross_entropy_rows(ref.logits, labels), rtol=1e-15)
    np.testing.assert_allclose(cb, cross_entropy_rows(ref.base, labels), rtol=1e-15)


def test_zero_correction_makes_the_mix_irrelevant():
    cfg, w, _ = _tiny()
    w.w2 = np.zeros_like(w.w2)
    m = Model.from_storage(w)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    labels = np.random.default_rng(4).integers(0, cfg.V, size=(cfg.B, cfg.K)).astype(np.int32)
    l0, cf, cb, _ = train_forward(m, hidden, anchor, labels, 0.0, 0.7)
    l1, _, _, _ = train_forward(m, hidden, anchor, labels, 1.0, 0.7)
    np.testing.assert_allclose(cf, cb, atol=1e-12)
    assert l0 == pytest.approx(l1, rel=1e-12)


def test_labels_feed_the_gru_causally():
    cfg, w, m = _tiny()
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    labels = np.random.default_rng(5).integers(0, cfg.V, size=(cfg.B, cfg.K)).astype(np.int32)
    _, cf, _, res = train_forward(m, hidden, anchor, labels, 0.5, 0.9)
    j = 1
    other = labels.copy()
    other[:, j] = (other[:, j] + 7) % cfg.V
    _, cf2, _, res2 = train_forward(m, hidden, anchor, other, 0.5, 0.9)
    # logits up to and including position j do not depend on label j; later ones do
    np.testing.assert_array_equal(res.logits[:, :j + 1], res2.logits[:, :j + 1])
    assert np.abs(res.logits[:, j + 1:] - res2.logits[:, j + 1:]).max() > 0
    np.testing.assert_array_equal(cf[:, :j], cf2[:, :j])
