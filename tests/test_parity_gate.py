"""The parity gate rejects what it must (CPU only).

``check_against_oracle`` is the comparison every GPU parity test applies. Here
it gets outputs made on the CPU, in the form the device path returns them
(int32 tokens, fp32 logits, int32 tau). The oracle's own block must pass. The
same block with one planted error must fail. The planted errors are a pick
changed where the oracle's margin exceeds 0.05, one logit moved past the
tolerance, a tau off by one, and a teacher-forced pick that is not the best.
Small deviations inside the stated tolerances must still pass.  The same holds
for the stochastic-verification protocol: a tau off by one, a poor or
out-of-range emitted token fail it.
"""
import numpy as np
import pytest

import oracle
import synth
from _harness import MARGIN, SCORE_TIE, TOL, check_against_oracle, check_verify_sample, emission_scores_of


def _setup(dtype, mode):
    cfg = synth.Config(name="gate", B=3, K=6, d=48, V=300, H=16, r=8, E=32, dtype=dtype, tied=False, mode=mode,
                       seed=4, target_p=0.3)
    w = synth.make_weights(cfg)
    model = oracle.Model.from_storage(w)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    ref = oracle.draft_block(model, hidden, anchor, mode=cfg.mode, temperature=cfg.temperature, seed=cfg.seed)
    target = synth.make_targets(cfg, ref.tokens)
    gpu = {"tokens": ref.tokens.astype(np.int32), "logits": ref.logits.astype(np.float32),
           "tau": oracle.verify(ref.tokens, target).astype(np.int32)}
    return cfg, model, hidden, anchor, target, ref, gpu


def _wide_margin_position(ref):
    """A (request, position) whose top-1 / top-2 pick margin exceeds the gate's."""
    b, p = np.argwhere(ref.top1 - ref.top2 > 2 * MARGIN)[0]
    return int(b), int(p)


@pytest.mark.parametrize("dtype,mode", [("f32", "greedy"), ("bf16", "greedy"), ("bf16", "gumbel")])
def test_the_oracles_own_block_passes(dtype, mode):
    cfg, model, hidden, anchor, target, ref, gpu = _setup(dtype, mode)
    check_against_oracle(model, cfg, hidden, anchor, gpu, target=target)


@pytest.mark.parametrize("mode", ["greedy", "gumbel"])
def test_a_pick_off_beyond_the_margin_fails(mode):
    cfg, model, hidden, anchor, target, ref, gpu = _setup("bf16", mode)
    b, p = _wide_margin_position(ref)
    gpu["tokens"] = gpu["tokens"].copy()
    gpu["tokens"][b, p] = (gpu["tokens"][b, p] + 1) % cfg.V
    gpu["logits"] = None        # the pick alone must be caught
    with pytest.raises(AssertionError, match="picks off"):
        check_against_oracle(model, cfg, hidden, anchor, gpu)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_logits_past_the_tolerance_fail_and_inside_it_pass(dtype):
    cfg, model, hidden, anchor, target, ref, gpu = _setup(dtype, "greedy")
    tol = TOL[dtype]
    inside = gpu["logits"].copy()
    inside[1, 2, 7] += np.float32(0.5 * tol)
    check_against_oracle(model, cfg, hidden, anchor, dict(gpu, logits=inside))
    past = gpu["logits"].copy()
    past[1, 2, 7] += np.float32(1.5 * tol)
    with pytest.raises(AssertionError, match="final logits"):
        check_against_oracle(model, cfg, hidden, anchor, dict(gpu, logits=past))


def test_tau_off_by_one_fails():
    cfg, model, hidden, anchor, target, ref, gpu = _setup("bf16", "greedy")
    tau = gpu["tau"].copy()
    tau[0] = tau[0] + 1 if tau[0] < cfg.K else tau[0] - 1
    with pytest.raises(AssertionError):
        check_against_oracle(model, cfg, hidden, anchor, dict(gpu, tau=tau), target=target)


def test_teacher_forced_pick_that_is_not_the_best_fails():
    cfg, model, hidden, anchor, target, ref, gpu = _setup("bf16", "greedy")
    forced = np.random.default_rng(9).integers(0, cfg.V, size=(cfg.B, cfg.K)).astype(np.int32)
    tf = oracle.draft_block(model, hidden, anchor, forced=forced)
    good = {"tokens": tf.tokens.astype(np.int32), "logits": tf.logits.astype(np.float32), "tau": None}
    check_against_oracle(model, cfg, hidden, anchor, good, forced=forced)
    b, p = _wide_margin_position(tf)
    bad = dict(good, tokens=good["tokens"].copy(), logits=None)
    bad["tokens"][b, p] = (bad["tokens"][b, p] + 1) % cfg.V
    with pytest.raises(AssertionError, match="picks off"):
        check_against_oracle(model, cfg, hidden, anchor, bad, forced=forced)


# ---------------------------------------------------------------- stochastic verification

def _verify_case():
    rng = np.random.default_rng(31)
    B, K, V = 12, 4, 200
    dl = rng.normal(0.0, 2.0, size=(B, K, V)).astype(np.float32)
    tl = np.concatenate([dl + rng.normal(0.0, 0.8, size=(B, K, V)), rng.normal(0.0, 2.0, size=(B, 1, V))],
                        axis=1).astype(np.float32)
    draft = rng.integers(0, V, size=(B, K)).astype(np.int32)
    ref = oracle.verify_sample(dl.astype(np.float64), tl.astype(np.float64), draft, 1.0, 17)
    return dl, tl, draft, ref


def test_verify_gate_passes_the_oracles_own_result():
    dl, tl, draft, ref = _verify_case()
    stats = check_verify_sample(dl, tl, draft, 1.0, 17, ref.tau, ref.token)
    assert stats["compared"] + stats["ties"] == len(ref.tau) and stats["compared"] >= len(ref.tau) - 1


def test_verify_gate_rejects_a_wrong_tau_or_token():
    dl, tl, draft, ref = _verify_case()
    K, V = dl.shape[1], dl.shape[2]
    b = int(np.flatnonzero(ref.tau < K)[0])
    tau = ref.tau.copy()
    tau[b] += 1
    with pytest.raises(AssertionError):
        check_verify_sample(dl, tl, draft, 1.0, 17, tau, ref.token)
    score = emission_scores_of(dl, tl, b, int(ref.tau[b]), 1.0, 17)
    tok = ref.token.copy()
    tok[b] = int(np.argmin(np.where(np.isfinite(score), score, np.inf)))   # a valid but poor draw
    assert score[tok[b]] < score.max() - SCORE_TIE
    with pytest.raises(AssertionError):
        check_verify_sample(dl, tl, draft, 1.0, 17, ref.tau, tok)
    tok[b] = V                                                           # out of range
    with pytest.raises(AssertionError):
        check_verify_sample(dl, tl, draft, 1.0, 17, ref.tau, tok)
