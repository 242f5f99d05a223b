"""Pins of the stochastic-verification oracle (oracle/sampling.py): the exact
output law of speculative sampling, its acceptance probability, the law of the
acceptance length and of the residual draw, and its limits.
CPU only."""
import numpy as np
import pytest
from scipy import special, stats

from oracle import accept_uniform, emission_scores, resample_noise, softmax_rows, verify_sample


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


@pytest.mark.parametrize("T", [0.5, 1.0, 2.5])
def test_softmax_rows_matches_scipy_at_temperature(T):
    x = np.random.default_rng(5).normal(0.0, 3.0, size=(4, 7, 33))
    np.testing.assert_allclose(softmax_rows(x, T), special.softmax(x / T, axis=-1), rtol=1e-13, atol=0)


def test_softmax_rows_temperature_limits():
    x = np.array([[0.3, 1.9, -0.4, 1.2]])
    cold = softmax_rows(x, 1e-3)                     # T -> 0: one-hot at the argmax
    np.testing.assert_allclose(cold, [[0.0, 1.0, 0.0, 0.0]], atol=1e-12)
    hot = softmax_rows(x, 1e6)                       # T -> inf: uniform
    np.testing.assert_allclose(hot, 0.25, atol=1e-6)


def test_acceptance_length_law_is_the_product_of_acceptances():
    # with independent uniforms, P(tau >= k) = prod_{i <= k} a_i, a_i = min(1, q_i(t_i) / p_i(t_i))
    K, T = 3, 1.0
    want = np.array([0.7, 0.5, 0.6])                  # acceptance of token 0 at each position
    pd = np.array([[0.5, 0.2, 0.2, 0.1]] * K)
    qd = np.stack([[0.5 * x, 0.2, 0.3, 0.5 - 0.5 * x] for x in want])
    dl, tl = np.log(pd)[None], np.log(np.concatenate([qd, [[0.25] * 4]]))[None]
    p, q = softmax_rows(dl, T)[0], softmax_rows(tl, T)[0]
    draft = np.zeros((1, K), dtype=np.int64)
    a = np.array([min(1.0, q[i, 0] / p[i, 0]) for i in range(K)])
    np.testing.assert_allclose(a, want, rtol=1e-12)
    at_least = np.concatenate([[1.0], np.cumprod(a)])            # P(tau >= k), k = 0..K
    law = at_least - np.concatenate([at_least[1:], [0.0]])       # P(tau == k)
    n = 6000
    counts = np.bincount([int(verify_sample(dl, tl, draft, T, seed=s).tau[0]) for s in range(n)], minlength=K + 1)
    assert stats.chisquare(counts, law * n).pvalue > 1e-3, (counts / n, law)


def test_residual_draw_follows_the_normalised_residual():
    # given a rejection at position 1, the emitted token is distributed as norm(max(0, q_1 - p_1))
    V, T = 4, 1.0
    dl = np.log(np.array([[[0.10, 0.60, 0.15, 0.15]]]))
    tl = np.log(np.array([[[0.30, 0.10, 0.30, 0.30], [0.25, 0.25, 0.25, 0.25]]]))
    p, q = softmax_rows(dl, T)[0, 0], softmax_rows(tl, T)[0, 0]
    resid = np.maximum(q - p, 0.0)
    resid /= resid.sum()
    draft = np.array([[1]])                           # a = q(1) / p(1) = 1/6
    tokens = []
    for s in range(12000):
        res = verify_sample(dl, tl, draft, T, seed=s)
        if res.tau[0] == 0:
            tokens.append(int(res.token[0]))
    counts = np.bincount(tokens, minlength=V)
    assert counts[1] == 0                             # the rejected token has no residual mass
    keep = resid > 0
    assert stats.chisquare(counts[keep], resid[keep] * len(tokens)).pvalue > 1e-3, (counts / len(tokens), resid)


def test_empty_residual_draws_from_the_target():
    # p and q agree in fp64 except at the drafted token, whose probability (~1e-20) is
    # below fp64 resolution: the acceptance ratio is e^-1, yet max(0, q - p) is zero
    # everywhere.  The emitted token after such a rejection is drawn from q.
    T = 1.0
    dl = np.array([[[0.0, 1.0, 2.0, 0.5, -45.0]]])
    tl = np.concatenate([dl, [[[0.3, 0.1, 0.2, 0.4, 0.0]]]], axis=1)
    tl[0, 0, 4] = -46.0
    p, q = softmax_rows(dl, T)[0, 0], softmax_rows(tl, T)[0, 0]
    assert not (np.maximum(q - p, 0.0) > 0).any()
    np.testing.assert_allclose(q[4] / p[4], np.exp(-1.0), rtol=1e-12)
    draft = np.array([[4]])
    tokens = []
    for s in range(6000):
        res = verify_sample(dl, tl, draft, T, seed=s)
        if res.tau[0] == 0:
            tokens.append(int(res.token[0]))
            assert res.token[0] == np.argmax(np.log(q) + resample_noise(s, 0, 0, 5))
    assert abs(len(tokens) / 6000 - (1 - np.exp(-1.0))) < 0.03
    counts = np.bincount(tokens, minlength=5)
    keep = q > 1e-6
    assert counts[~keep].sum() == 0
    assert stats.chisquare(counts[keep], q[keep] / q[keep].sum() * len(tokens)).pvalue > 1e-3, (counts, q)


def test_emission_scores_cases():
    q = np.array([0.1, 0.2, 0.3, 0.4])
    p = np.array([0.4, 0.1, 0.3, 0.2])
    g = resample_noise(3, 1, 2, 4)
    with np.errstate(divide="ignore"):
        np.testing.assert_array_equal(emission_scores(p, q, 3, 1, 2), np.log([0.0, 0.1, 0.0, 0.2]) + g)
        np.testing.assert_array_equal(emission_scores(None, q, 3, 1, 2), np.log(q) + g)
        np.testing.assert_array_equal(emission_scores(q, q, 3, 1, 2), np.log(q) + g)   # empty residual
