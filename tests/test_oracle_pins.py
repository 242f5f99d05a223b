"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a swapped gate) fails at least one:

* Philox            -> published known-answer vectors (tests/golden)
* GRU step          -> torch.nn.GRUCell in fp64, and a hand-computed closed form
* SiLU              -> closed form / torch.nn.functional.silu
* LM head           -> brute-force triple loop
* correction        -> W2 = 0 and W1 = 0 reduce every pick to argmax of the base logits
* [h ; S] order     -> zeroing either column block removes exactly that dependence
* state indexing    -> position 1 already sees GRU(e(anchor), 0) (hand-computed),
                       with each request's own anchor embedding as that input
* loop              -> teacher forcing on the free-running picks changes nothing;
                       causality; brute-force greedy fixed point
* pick margins      -> top1 / top2 / forced_gap by sorting each position's scores
* Gumbel-max        -> chi-square against the exact law prod_i softmax(L_i / T)[t_i];
                       noise moments (Euler-Mascheroni mean, pi^2/6 variance)
* tau               -> brute force over every mismatch position
* shapes            -> the pages' "56M" head parameter count
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy import stats

import synth
from oracle import (Model, draft_block, gru_cell, gumbel_noise, lm_head, philox4x32_10, philox4x32_10_np,
                    silu, uniform_from_word, verify, widen_f64)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_cfg(**kw):
    base = dict(name="small", B=2, K=4, d=24, V=40, H=8, r=6, E=16, dtype="f32", tied=False, seed=3)
    base.update(kw)
    return synth.Config(**base)


def model_of(cfg, **override):
    w = synth.make_weights(cfg)
    for k, v in override.items():
        setattr(w, k, v)
    return w, Model.from_storage(w)


# ---------------------------------------------------------------- Philox / Gumbel

def _kat_rows():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            v = [int(x, 16) for x in line.split()]
            rows.append((v[0:4], v[4:6], v[6:10]))
    return rows


def test_philox_known_answers():
    rows = _kat_rows()
    assert len(rows) == 3
    for ctr, key, out in rows:
        assert list(philox4x32_10(ctr, key)) == out
        vec = philox4x32_10_np(*[np.array([c], dtype=np.uint32) for c in ctr], key[0], key[1])
        assert [int(x[0]) for x in vec] == out


def test_philox_vectorised_matches_scalar():
    rng = np.random.default_rng(7)
    c = rng.integers(0, 2 ** 32, size=(4, 64), dtype=np.uint64)
    k = rng.integers(0, 2 ** 32, size=2, dtype=np.uint64)
    vec = philox4x32_10_np(c[0], c[1], c[2], c[3], int(k[0]), int(k[1]))
    for n in range(64):
        assert tuple(int(x[n]) for x in vec) == philox4x32_10(tuple(int(c[i, n]) for i in range(4)), tuple(int(x) for x in k))


def test_uniform_mapping_bounds_and_uniformity():
    assert uniform_from_word(0) == 2.0 ** -24
    assert uniform_from_word(0xFFFFFFFF) == 1.0 - 2.0 ** -24
    n = 1 << 18
    w = philox4x32_10_np(np.arange(n // 4, dtype=np.uint64), np.zeros(n // 4, np.uint64),
                         np.zeros(n // 4, np.uint64), np.zeros(n // 4, np.uint64), 12345, 0)
    u = uniform_from_word(np.stack(w, 1).reshape(-1))
    assert np.all((u > 0) & (u < 1))
    counts, _ = np.histogram(u, bins=64, range=(0, 1))
    assert stats.chisquare(counts).pvalue > 1e-4


def test_gumbel_noise_moments():
    g = gumbel_noise(seed=99, b=0, i=1, V=1 << 20)
    assert abs(g.mean() - 0.5772156649) < 0.01
    assert abs(g.var() - math.pi ** 2 / 6) < 0.02


def test_gumbel_noise_streams_differ():
    a = gumbel_noise(1, 0, 1, 64)
    assert not np.array_equal(a, gumbel_noise(1, 1, 1, 64))   # request
    assert not np.array_equal(a, gumbel_noise(1, 0, 2, 64))   # position
    assert not np.array_equal(a, gumbel_noise(2, 0, 1, 64))   # seed
    assert not np.array_equal(a, gumbel_noise(1 << 32 | 1, 0, 1, 64))  # high key word
    np.testing.assert_array_equal(a, gumbel_noise(1, 0, 1, 64))


@pytest.mark.parametrize("temperature", [1.0, 0.5])
def test_gumbel_max_follows_exact_law(temperature):
    """Empirical sequence frequencies vs prod_i softmax(L_i(t_<i) / T)[t_i]."""
    cfg = small_cfg(B=1, K=2, V=4, d=8, H=4, r=3, E=8)
    w, m = model_of(cfg)
    hidden = synth.make_hidden(cfg)
    anchor = synth.make_anchor(cfg)
    V, K = cfg.V, cfg.K
    # exact law by teacher forcing every prefix
    probs = {}
    for t1 in range(V):
        forced = np.array([[t1, 0]], dtype=np.int32)
        r = draft_block(m, hidden, anchor, mode="greedy", forced=forced)
        p1 = np.exp(r.logits[0, 0] / temperature)
        p1 /= p1.sum()
        p2 = np.exp(r.logits[0, 1] / temperature)
        p2 /= p2.sum()
        for t2 in range(V):
            probs[(t1, t2)] = p1[t1] * p2[t2]
    # many independent draws: requests b use independent Philox streams
    nrep = 20000
    hb = np.repeat(hidden, nrep, axis=0)
    ab = np.repeat(anchor, nrep, axis=0)
    counts = np.zeros(V ** K)
    for seed in range(3):
        r = draft_block(m, hb, ab, mode="gumbel", temperature=temperature, seed=seed, want_logits=False)
        idx = r.tokens[:, 0] * V + r.tokens[:, 1]
        counts += np.bincount(idx, minlength=V ** K)
    expected = np.array([probs[(a, b)] for a in range(V) for b in range(V)]) * counts.sum()
    keep = expected > 5
    chi = ((counts[keep] - expected[keep]) ** 2 / expected[keep]).sum()
    pval = stats.chi2.sf(chi, keep.sum() - 1)
    assert pval > 1e-4, (chi, pval)


# ---------------------------------------------------------------- GRU / SiLU / LM head

def test_gru_cell_matches_torch_grucell():
    rng = np.random.default_rng(0)
    B, E, H = 3, 7, 5
    cell = torch.nn.GRUCell(E, H, dtype=torch.float64)
    x = rng.standard_normal((B, E))
    s = rng.standard_normal((B, H))
    with torch.no_grad():
        want = cell(torch.from_numpy(x), torch.from_numpy(s)).numpy()
    got = gru_cell(x, s, cell.weight_ih.detach().numpy(), cell.weight_hh.detach().numpy(),
                   cell.bias_ih.detach().numpy(), cell.bias_hh.detach().numpy())
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


def test_gru_cell_hand_computed():
    """All weights zero: gates are functions of the biases alone."""
    H = 2
    b_ih = np.array([0.3, -0.2, 0.5, 0.1, 0.7, -0.4])   # r, z, n blocks of length 2
    b_hh = np.array([0.1, 0.4, -0.6, 0.2, 0.9, 0.3])
    s = np.array([[0.25, -0.5]])
    out = gru_cell(np.zeros((1, 3)), s, np.zeros((3 * H, 3)), np.zeros((3 * H, H)), b_ih, b_hh)
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))  # noqa: E731
    for k in range(H):
        r = sig(b_ih[k] + b_hh[k])
        z = sig(b_ih[H + k] + b_hh[H + k])
        n = math.tanh(b_ih[2 * H + k] + r * b_hh[2 * H + k])   # b_hn sits inside r * (.)
        assert abs(out[0, k] - ((1 - z) * n + z * s[0, k])) < 1e-15


def test_silu_closed_form():
    x = np.linspace(-20, 20, 4001)
    np.testing.assert_allclose(silu(x), x / (1.0 + np.exp(-x)), rtol=1e-15, atol=1e-300)
    np.testing.assert_allclose(silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(), rtol=1e-14, atol=1e-300)


def test_widen_bf16_matches_torch():
    rng = np.random.default_rng(1)
    vals = rng.standard_normal(1000).astype(np.float32) * 10
    bits = synth.f32_to_bf16_bits(vals)
    want = torch.from_numpy(vals).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(widen_f64(bits, "bf16"), want)


def test_lm_head_bruteforce():
    rng = np.random.default_rng(2)
    B, K, d, V = 2, 3, 5, 7
    h = rng.standard_normal((B, K, d))
    w = rng.standard_normal((V, d)).astype(np.float32)
    got = lm_head(h, w, "f32", chunk=3)
    for b in range(B):
        for i in range(K):
            for v in range(V):
                acc = 0.0
                for k in range(d):
                    acc += float(w[v, k]) * h[b, i, k]
                assert abs(got[b, i, v] - acc) < 1e-12


# ---------------------------------------------------------------- loop invariants

@pytest.mark.parametrize("which", ["w2", "w1"])
def test_zero_correction_gives_base_argmax(which):
    cfg = small_cfg()
    w = synth.make_weights(cfg)
    setattr(w, which, np.zeros_like(getattr(w, which)))
    m = Model.from_storage(w)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    r = draft_block(m, hidden, anchor)
    np.testing.assert_array_equal(r.tokens, np.argmax(r.base, axis=2))
    if which == "w2":
        np.testing.assert_array_equal(r.logits, r.base)


def test_correction_is_active():
    cfg = small_cfg()
    w, m = model_of(cfg)
    r = draft_block(m, synth.make_hidden(cfg), synth.make_anchor(cfg))
    assert np.abs(r.logits - r.base).max() > 1e-3


def test_teacher_forcing_on_own_picks_is_identity():
    cfg = small_cfg(B=3, K=6)
    w, m = model_of(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    free = draft_block(m, hidden, anchor)
    tf = draft_block(m, hidden, anchor, forced=free.tokens)
    np.testing.assert_array_equal(tf.tokens, free.tokens)
    np.testing.assert_array_equal(tf.logits, free.logits)
    np.testing.assert_array_equal(tf.forced_gap, np.zeros_like(tf.forced_gap))


def test_causality():
    cfg = small_cfg(B=1, K=5)
    w, m = model_of(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    free = draft_block(m, hidden, anchor)
    for j in range(cfg.K - 1):
        forced = free.tokens.copy()
        forced[0, j] = (forced[0, j] + 1) % cfg.V
        r = draft_block(m, hidden, anchor, forced=forced)
        np.testing.assert_array_equal(r.logits[:, :j + 1], free.logits[:, :j + 1])
        assert np.abs(r.logits[:, j + 1] - free.logits[:, j + 1]).max() > 1e-6


def test_concat_order_hidden_first():
    """[h_i ; S_{i-1}]: the first d columns of W1 see h, the last H see S."""
    cfg = small_cfg(B=1, K=3)
    w = synth.make_weights(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    base = np.zeros((1, cfg.K, cfg.V))           # hold base logits fixed
    other = hidden.copy()
    other[:, :, :] = synth.make_hidden(cfg.replace(seed=11))
    # W1 acting on S only: correction independent of h
    w_s = synth.make_weights(cfg)
    w_s.w1 = w.w1.copy()
    w_s.w1[:, :cfg.d] = 0
    m = Model.from_storage(w_s)
    a = draft_block(m, hidden, anchor, base=base)
    b = draft_block(m, other, anchor, base=base)
    np.testing.assert_array_equal(a.logits, b.logits)
    # W1 acting on h only: correction independent of the GRU (anchor / tokens)
    w_h = synth.make_weights(cfg)
    w_h.w1 = w.w1.copy()
    w_h.w1[:, cfg.d:] = 0
    m = Model.from_storage(w_h)
    a = draft_block(m, hidden, anchor, base=base)
    b = draft_block(m, hidden, (anchor + 1) % cfg.V, base=base)
    np.testing.assert_array_equal(a.logits, b.logits)
    c = draft_block(m, other, anchor, base=base)
    assert np.abs(a.logits - c.logits).max() > 1e-6


def test_first_position_sees_anchor_step_hand_computed():
    """Position 1 uses S after one GRU step on e(anchor) from the zero state."""
    H, r, V, d, E = 2, 2, 3, 2, 2
    b_ih = np.array([0.3, -0.2, 0.5, 0.1, 0.7, -0.4], dtype=np.float32)
    b_hh = np.array([0.1, 0.4, -0.6, 0.2, 0.9, 0.3], dtype=np.float32)
    w = synth.Weights(
        dtype="f32",
        w_lm=np.zeros((V, d), np.float32), embed=np.zeros((V, E), np.float32),
        w_ih=np.zeros((3 * H, E), np.float32), w_hh=np.zeros((3 * H, H), np.float32),
        b_ih=b_ih, b_hh=b_hh,
        w1=np.array([[0, 0, 1, 0], [0, 0, 0, 1]], np.float32),   # u = silu(S) on the S block
        w2=np.array([[1, 0], [0, 1], [1, 1]], np.float32))
    m = Model.from_storage(w)
    res = draft_block(m, np.zeros((1, 1, d), np.float32), np.array([0]))
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))  # noqa: E731
    s1 = []
    for k in range(H):
        rr = sig(float(b_ih[k]) + float(b_hh[k]))
        z = sig(float(b_ih[H + k]) + float(b_hh[H + k]))
        n = math.tanh(float(b_ih[2 * H + k]) + rr * float(b_hh[2 * H + k]))
        s1.append((1 - z) * n)
    u = [x * sig(x) for x in s1]
    want = [u[0], u[1], u[0] + u[1]]
    np.testing.assert_allclose(res.logits[0, 0], want, rtol=0, atol=1e-15)


def test_first_position_reads_each_requests_anchor_embedding_hand_computed():
    """The GRU's first input is E[anchor] of that request (H = E = d = r = 1).

    Only W_ih, the embedding and W2 are nonzero, so S_1 = (1 - z) n with
    r = sigmoid(W_ir x), z = sigmoid(W_iz x), n = tanh(W_in x), x = E[anchor],
    and L_1 = W2 SiLU(S_1).  Anchor 0 has a zero embedding, so feeding any
    token but the anchor changes the logits.
    """
    V = 3
    emb = np.array([[0.0], [0.5], [-1.5]], np.float32)
    w_ih = np.array([[0.4], [-0.3], [0.8]], np.float32)
    w = synth.Weights(
        dtype="f32", w_lm=np.zeros((V, 1), np.float32), embed=emb, w_ih=w_ih,
        w_hh=np.zeros((3, 1), np.float32), b_ih=None, b_hh=None,
        w1=np.array([[0.0, 1.0]], np.float32), w2=np.array([[1.0], [2.0], [-1.0]], np.float32))
    res = draft_block(Model.from_storage(w), np.zeros((2, 1, 1), np.float32), np.array([2, 1]))
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))  # noqa: E731
    for b, anchor in enumerate((2, 1)):
        x = float(emb[anchor, 0])
        z = sig(float(w_ih[1, 0]) * x)
        s1 = (1.0 - z) * math.tanh(float(w_ih[2, 0]) * x)
        u = s1 * sig(s1)
        np.testing.assert_allclose(res.logits[b, 0], [u, 2.0 * u, -u], rtol=0, atol=1e-15)


def test_bruteforce_greedy_fixed_point():
    cfg = small_cfg(B=1, K=3, V=5, d=6, H=3, r=2, E=4, seed=5)
    w, m = model_of(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    free = draft_block(m, hidden, anchor)
    fixed = []
    for a in range(cfg.V):
        for b in range(cfg.V):
            for c in range(cfg.V):
                seq = np.array([[a, b, c]], dtype=np.int32)
                r = draft_block(m, hidden, anchor, forced=seq)
                if all(int(np.argmax(r.logits[0, p])) == seq[0, p] for p in range(cfg.K)):
                    fixed.append(seq[0].tolist())
    assert fixed == [free.tokens[0].tolist()]


# ---------------------------------------------------------------- tau / shapes / configs

@pytest.mark.parametrize("mode", ["greedy", "gumbel"])
def test_pick_margins_bruteforce(mode):
    """top1 / top2 are the two largest pick scores and forced_gap = top1 - score(fed) >= 0.

    The parity protocol accepts a GPU pick within a margin of the best, so these
    fields are checked by sorting each position's scores directly.
    """
    cfg = small_cfg(B=3, K=5, V=40)
    w, m = model_of(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    fed = np.random.default_rng(8).integers(0, cfg.V, size=(cfg.B, cfg.K))
    T, seed = 0.8, 21
    res = draft_block(m, hidden, anchor, forced=fed, mode=mode, temperature=T, seed=seed)
    for b in range(cfg.B):
        for p in range(cfg.K):
            score = [float(x) for x in res.logits[b, p]]
            if mode == "gumbel":
                g = gumbel_noise(seed, b, p + 1, cfg.V)
                score = [score[j] / T + float(g[j]) for j in range(cfg.V)]
            order = sorted(range(cfg.V), key=lambda j: (-score[j], j))
            assert res.tokens[b, p] == order[0]
            assert res.top1[b, p] == score[order[0]] and res.top2[b, p] == score[order[1]]
            assert res.forced_gap[b, p] == score[order[0]] - score[int(fed[b, p])]
            assert res.forced_gap[b, p] >= 0.0


def test_tau_bruteforce():
    rng = np.random.default_rng(4)
    for K in range(1, 17):
        for mis in range(K + 1):           # mis == K: full agreement
            d = rng.integers(0, 100, size=(1, K)).astype(np.int32)
            t = d.copy()
            if mis < K:
                t[0, mis] = (t[0, mis] + 1 + rng.integers(0, 50)) % 1000 + 1000
                t[0, mis + 1:] = rng.integers(0, 100, size=K - mis - 1)
            assert verify(d, t)[0] == mis


def test_head_parameter_count_matches_pages():
    vals = {}
    with open(os.path.join(GOLDEN, "head_params.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v = line.split()
            vals[k] = int(v)
    cfg = synth.CONFIGS["qwen3_8b_b1"]
    assert (cfg.d, cfg.H, cfg.r, cfg.V, cfg.E) == (vals["d"], vals["H"], vals["r"], vals["V"], vals["E"])
    n = cfg.head_params
    assert n == 55_934_976
    assert round(n / 1e6) == vals["stated_millions"]


def test_tiny_config_expected_tau():
    cfg = synth.CONFIGS["tiny_f32"]
    w, m = model_of(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    r = draft_block(m, hidden, anchor)
    target = synth.make_targets(cfg, r.tokens)
    assert verify(r.tokens, target)[0] == 3
    # logits have the intended scale (W_lm x 4 -> std ~ 4)
    assert 2.5 < r.base.std() < 5.5
