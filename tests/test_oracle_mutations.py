"""The oracle's pins catch plausible mistakes (CPU only).

Each case below plants one slip in a copy of the oracle, the kind that can
hide in a restatement of the method: a swapped gate or operand, a dropped term,
a wrong sign, an index off by one, a shared random stream. The three pin
suites then run against that copy in a subprocess, and at least one pin must
fail. An unmutated copy must pass. If a planted slip survives, the pins do not
fix that part of the oracle.

The copies live in a temporary directory and the real oracle is never
modified. Every mutation must match its source text exactly as often as it
declares, so an edit to the oracle that moves the text breaks this test loudly
rather than silently planting nothing.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ("test_oracle_pins.py", "test_oracle_training_pins.py", "test_oracle_sampling_pins.py")

# (name, oracle file, text, replacement, occurrences)
MUTATIONS = [
    # GRU cell (PyTorch gate order r, z, n; b_hn inside r * (.))
    ("gru_r_z_swapped", "domino_ref.py",
     "    r = sigmoid(gi[:, 0:H] + gh[:, 0:H])\n    z = sigmoid(gi[:, H:2 * H] + gh[:, H:2 * H])",
     "    r = sigmoid(gi[:, H:2 * H] + gh[:, H:2 * H])\n    z = sigmoid(gi[:, 0:H] + gh[:, 0:H])", 1),
    ("gru_update_sides_swapped", "domino_ref.py",
     "return (1.0 - z) * n + z * s", "return z * n + (1.0 - z) * s", 1),
    ("gru_reset_gate_dropped", "domino_ref.py",
     "+ r * gh[:, 2 * H:3 * H])", "+ gh[:, 2 * H:3 * H])", 1),
    ("gru_b_hn_outside_reset", "domino_ref.py",
     "+ r * gh[:, 2 * H:3 * H])",
     "+ r * (gh[:, 2 * H:3 * H] - b_hh[2 * H:3 * H]) + b_hh[2 * H:3 * H])", 1),
    ("sigmoid_sign", "domino_ref.py", "1.0 / (1.0 + np.exp(-x))", "1.0 / (1.0 + np.exp(x))", 1),
    ("silu_is_sigmoid", "domino_ref.py", "return x * sigmoid(x)", "return sigmoid(x)", 1),
    ("widen_bf16_shift", "domino_ref.py", "<< np.uint32(16)", "<< np.uint32(15)", 1),
    ("gru_biases_dropped", "domino_ref.py",
     "return np.zeros(H3) if a is None else np.asarray(a, np.float32).astype(np.float64)",
     "return np.zeros(H3)", 1),
    ("embedding_read_from_lm_head", "domino_ref.py",
     "widen_f64(self.embed[np.asarray(tokens, dtype=np.int64)], self.dtype)",
     "widen_f64(self.w_lm[np.asarray(tokens, dtype=np.int64)], self.dtype)", 1),
    # the correction loop
    ("concat_state_first", "domino_ref.py",
     "np.concatenate([hidden64[:, p, :], s], axis=1)", "np.concatenate([s, hidden64[:, p, :]], axis=1)", 1),
    ("bottleneck_activation_dropped", "domino_ref.py", "u = silu(cat @ model.w1.T)", "u = cat @ model.w1.T", 1),
    ("residual_base_dropped", "domino_ref.py", "L = base[:, p, :] + u @ model.w2.T", "L = u @ model.w2.T", 1),
    ("state_used_before_its_update", "domino_ref.py",
     "        s = gru_cell(x, s, model.w_ih, model.w_hh, model.b_ih, model.b_hh)   # S_{i-1}\n"
     "        cat = np.concatenate([hidden64[:, p, :], s], axis=1)",
     "        s_next = gru_cell(x, s, model.w_ih, model.w_hh, model.b_ih, model.b_hh)\n"
     "        cat = np.concatenate([hidden64[:, p, :], s], axis=1)\n"
     "        s = s_next", 1),
    ("anchor_not_fed", "domino_ref.py",
     "prev = np.asarray(anchor, dtype=np.int64).copy()", "prev = np.zeros_like(np.asarray(anchor, dtype=np.int64))", 1),
    ("feeds_base_argmax", "domino_ref.py",
     "if forced is not None else pick.astype(np.int64)",
     "if forced is not None else np.argmax(base[:, p, :], axis=1).astype(np.int64)", 1),
    ("forced_tokens_ignored", "domino_ref.py",
     "prev = np.asarray(forced, dtype=np.int64)[:, p] if forced is not None else pick.astype(np.int64)",
     "prev = pick.astype(np.int64)", 1),
    ("margin_sides_swapped", "domino_ref.py",
     "        top2[:, p] = srt[:, 0]\n        top1[:, p] = srt[:, 1]",
     "        top2[:, p] = srt[:, 1]\n        top1[:, p] = srt[:, 0]", 1),
    ("forced_gap_sign", "domino_ref.py",
     "gap[:, p] = top1[:, p] - score[np.arange(B), fed]", "gap[:, p] = score[np.arange(B), fed] - top1[:, p]", 1),
    ("lm_head_rows_position_major", "domino_ref.py",
     "hk = hidden64.reshape(B * K, d)", "hk = hidden64.transpose(1, 0, 2).reshape(B * K, d)", 1),
    ("gumbel_temperature_multiplies", "domino_ref.py", "score = L / temperature + g", "score = L * temperature + g", 1),
    ("gumbel_noise_shared_by_requests", "domino_ref.py",
     "gumbel_noise(seed, int(rid[b]), p + 1, V)", "gumbel_noise(seed, 0, p + 1, V)", 1),
    ("tau_counts_every_match", "domino_ref.py",
     "        n = 0\n        while n < K and draft[b, n] == target[b, n]:\n            n += 1\n        tau[b] = n",
     "        tau[b] = int((draft[b] == target[b]).sum())", 1),
    # Philox4x32-10 and the uniform / Gumbel maps
    ("philox_multipliers_swapped", "philox.py",
     "        p0 = PHILOX_M0 * x0\n        p1 = PHILOX_M1 * x2",
     "        p0 = PHILOX_M1 * x0\n        p1 = PHILOX_M0 * x2", 1),
    ("philox_vectorised_key_schedule", "philox.py",
     "k1 = (k1 + np.uint64(PHILOX_W1)) & m", "k1 = (k1 + np.uint64(PHILOX_W0)) & m", 1),
    ("philox_nine_rounds", "philox.py", "for _ in range(10):", "for _ in range(9):", 2),
    ("uniform_can_be_zero", "philox.py", "* 2.0 + 1.0) * 2.0 ** -24", "* 2.0) * 2.0 ** -24", 1),
    ("gumbel_sign", "philox.py", "return -np.log(-np.log(u))", "return np.log(-np.log(u))", 1),
    # training forward and curriculum loss
    ("ce_sign", "training.py", "return lse - picked", "return picked - lse", 1),
    ("ce_row_max_dropped", "training.py",
     "lse = m + np.log(np.exp(x - m[..., None]).sum(axis=-1))", "lse = np.log(np.exp(x - m[..., None]).sum(axis=-1))", 1),
    ("weights_start_at_gamma", "training.py",
     "np.arange(K, dtype=np.float64)", "np.arange(1, K + 1, dtype=np.float64)", 1),
    ("base_loss_on_final_logits", "training.py",
     "ce_base = cross_entropy_rows(base_logits, labels)", "ce_base = cross_entropy_rows(final_logits, labels)", 1),
    ("weights_normalised_by_k", "training.py", "/ (B * w.sum()))", "/ (B * K))", 2),
    ("mix_swapped", "training.py",
     "(1.0 - lam) * l_final + lam * l_base", "lam * l_final + (1.0 - lam) * l_base", 1),
    ("batch_mean_dropped", "training.py", "/ (B * w.sum()))", "/ w.sum())", 2),
    ("training_runs_free", "training.py", "forced=labels", "forced=None", 1),
    # stochastic verification
    ("ratio_inverted", "sampling.py",
     "ratio[b, i] = q[b, i, t] / p[b, i, t]", "ratio[b, i] = p[b, i, t] / q[b, i, t]", 1),
    ("residual_sign", "sampling.py",
     "np.maximum(q_row - np.asarray(p_row, dtype=np.float64), 0.0)",
     "np.maximum(np.asarray(p_row, dtype=np.float64) - q_row, 0.0)", 1),
    ("resample_from_target_not_residual", "sampling.py",
     "resid = np.maximum(q_row - np.asarray(p_row, dtype=np.float64), 0.0)", "resid = q_row", 1),
    ("empty_residual_fallback_dropped", "sampling.py", "if (resid > 0.0).any():", "if True:", 1),
    ("bonus_from_last_draft_position", "sampling.py",
     "emission_scores(None, q[b, K], seed, b, K)", "emission_scores(None, q[b, K - 1], seed, b, K)", 1),
    ("no_stop_at_first_rejection", "sampling.py",
     "                pos = i\n                break", "                pos = i", 1),
    ("softmax_temperature_multiplies", "sampling.py",
     "np.float64) / float(temperature)", "np.float64) * float(temperature)", 1),
    ("accept_and_resample_share_a_stream", "sampling.py", "STREAM_ACCEPT = 2", "STREAM_ACCEPT = 1", 1),
    ("one_uniform_for_every_position", "sampling.py",
     "uni[b, i] = accept_uniform(seed, b, i)", "uni[b, i] = accept_uniform(seed, b, 0)", 1),
]


# Runs the statistical pins (seconds each) after the rest, so that most planted
# slips stop the copy's suite early; the order changes no outcome.
_ORDER_PLUGIN = """
SLOW = ("exact_law", "follows_the_target_law", "residual_draw", "acceptance_length_law", "acceptance_rate",
        "draws_from_the_target")


def pytest_collection_modifyitems(items):
    items.sort(key=lambda item: any(k in item.name for k in SLOW))
"""


def _base_copy(dst: str) -> None:
    """The oracle, the input generators and the pin suites, laid out like the repository."""
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__", "*.so", "*.o"))
    shutil.copytree(os.path.join(ROOT, "synth"), os.path.join(dst, "synth"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    tests = os.path.join(dst, "tests")
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(tests, "golden"))
    for f in ("conftest.py",) + PIN_FILES:
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(tests, f))
    with open(os.path.join(dst, "_pin_order.py"), "w") as f:
        f.write(_ORDER_PLUGIN)


def _plant(dst: str, fname: str, old: str, new: str, occurrences: int) -> None:
    path = os.path.join(dst, "oracle", fname)
    with open(path) as f:
        src = f.read()
    assert src.count(old) == occurrences, f"{fname}: expected {occurrences} match(es) of {old!r}"
    with open(path, "w") as f:
        f.write(src.replace(old, new))


def _run_pins(dst: str) -> subprocess.CompletedProcess:
    env = {k: v for k, v in os.environ.items() if k != "PYTHONPATH"}
    env.update(OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-p", "_pin_order",
                           *(os.path.join("tests", f) for f in PIN_FILES)],
                          cwd=dst, env=env, capture_output=True, text=True, timeout=900)


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    base = str(tmp_path_factory.mktemp("oracle_copies"))
    jobs = {}
    for name, fname, old, new, occ in [("unmutated", None, None, None, 0)] + MUTATIONS:
        dst = os.path.join(base, name)
        _base_copy(dst)
        if fname is not None:
            _plant(dst, fname, old, new, occ)
        jobs[name] = dst
    with ThreadPoolExecutor(max_workers=max(2, os.cpu_count() or 2)) as ex:
        done = dict(zip(jobs, ex.map(_run_pins, jobs.values())))
    return done


def test_unmutated_copy_passes(outcomes):
    r = outcomes["unmutated"]
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", [m[0] for m in MUTATIONS])
def test_planted_slip_fails_a_pin(outcomes, name):
    r = outcomes[name]
    # exit status 1: tests ran and at least one failed (not a collection or usage error)
    assert r.returncode == 1, f"{name} survived the pins (exit {r.returncode}):\n" + r.stdout[-2000:]
    assert " failed" in r.stdout
