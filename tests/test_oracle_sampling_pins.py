"""Pins of the stochastic-verification oracle (oracle/sampling.py): the exact
output law of speculative sampling, its acceptance probability, and its limits.
CPU only."""
import numpy as np
import pytest
from scipy import stats

from oracle import accept_uniform, resample_noise, softmax_rows, verify_sample


def _first_emitted(res, draft):
    """First token the block emits: t_1 if accepted, else the residual sample."""
    return np.where(res.tau > 0, draft[:, 0], res.token)


def test_first_emitted_token_follows_the_target_law():
    # Leviathan et al. / Chen et al.: with t_1 ~ p_1 the first emitted token is distributed as q_1
    V, K, T = 5, 2, 1.0
    rng = np.random.default_rng(0)
    dl = rng.normal(0.0, 1.5, size=(1, K, V))
    tl = rng.normal(0.0, 1.5, size=(1, K + 1, V))
    p, q = softmax_rows(dl, T)[0, 0], softmax_rows(tl, T)[0, 0]
    n = 20000
    counts = np.zeros(V)
    for trial in range(n):
        draft = np.array([[rng.choice(V, p=p), rng.choice(V, p=softmax_rows(dl, T)[0, 1])]])
        res = verify_sample(dl, tl, draft, T, seed=trial)
        counts[_first_emitted(res, draft)[0]] += 1
    chi2 = stats.chisquare(counts, q * n)
    assert chi2.pvalue > 1e-3, (counts / n, q)
    # and not the draft law
    assert stats.chisquare(counts, p * n).pvalue < 1e-6


def test_acceptance_rate_is_min_one_ratio():
    V, T = 6, 0.7
    rng = np.random.default_rng(1)
    dl = rng.normal(size=(1, 1, V))
    tl = rng.normal(size=(1, 2, V))
    p, q = softmax_rows(dl, T)[0, 0], softmax_rows(tl, T)[0, 0]
    t = int(np.argmax(p / q))          # a token the target under-weights: acceptance < 1
    a = min(1.0, q[t] / p[t])
    assert a < 1.0
    n = 4000
    acc = sum(int(verify_sample(dl, tl, np.array([[t]]), T, seed=s).tau[0]) for s in range(n))
    assert stats.binomtest(acc, n, a).pvalue > 1e-3


def test_equal_distributions_accept_everything_and_draw_the_bonus():
    rng = np.random.default_rng(2)
    B, K, V = 3, 4, 50
    dl = rng.normal(size=(B, K, V))
    tl = np.concatenate([dl, rng.normal(size=(B, 1, V))], axis=1)
    draft = rng.integers(0, V, size=(B, K))
    res = verify_sample(dl, tl, draft, 1.0, seed=7)
    np.testing.assert_array_equal(res.tau, K)
    for b in range(B):
        q = softmax_rows(tl[b, K], 1.0)
        assert res.token[b] == np.argmax(np.log(q) + resample_noise(7, b, K, V))


def test_zero_target_mass_rejects_and_never_resamples_the_token():
    rng = np.random.default_rng(3)
    V = 40
    dl = rng.normal(size=(1, 2, V))
    tl = rng.normal(size=(1, 3, V))
    t = 11
    tl[0, 0, t] = -1e4                 # q_1(t) == 0 in fp64
    for s in range(200):
        res = verify_sample(dl, tl, np.array([[t, 3]]), 1.0, seed=s)
        assert res.tau[0] == 0 and res.token[0] != t


def test_uniforms_and_noise_streams():
    u = [accept_uniform(5, b, i) for b in range(3) for i in range(4)]
    assert len(set(u)) == len(u) and all(0.0 < x < 1.0 for x in u)
    g1, g2 = resample_noise(5, 0, 0, 64), resample_noise(5, 0, 1, 64)
    assert not np.allclose(g1, g2)
    assert abs(np.mean(resample_noise(9, 2, 3, 200000)) - np.euler_gamma) < 0.01


def test_deterministic_and_tau_range():
    rng = np.random.default_rng(4)
    B, K, V = 4, 6, 30
    dl, tl = rng.normal(size=(B, K, V)), rng.normal(size=(B, K + 1, V))
    draft = rng.integers(0, V, size=(B, K))
    r1, r2 = verify_sample(dl, tl, draft, 1.0, 11), verify_sample(dl, tl, draft, 1.0, 11)
    np.testing.assert_array_equal(r1.tau, r2.tau)
    np.testing.assert_array_equal(r1.token, r2.token)
    assert ((r1.tau >= 0) & (r1.tau <= K)).all()
