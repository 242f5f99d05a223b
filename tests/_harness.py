"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the CUDA path through the C ABI, and apply the comparison protocol against
the fp64 oracle.

Comparison protocol (the divergence-safe gate):
  (i)   run the oracle teacher-forced along the GPU's own picks;
  (ii)  at every position the GPU pick must be the oracle's best pick, or its
        oracle score must be within MARGIN = 0.05 of the best (a near-tie);
        this makes picks bit-exact wherever the oracle's top-1/top-2 margin
        exceeds 0.05;
  (iii) final logits within max-abs 2e-2 (bf16 storage) or 1e-4 (fp32);
  (iv)  tau exact given the GPU draft.
"""
from __future__ import annotations

import numpy as np
import torch

import draft_model_b200 as dm
import oracle
import synth
from draft_model_b200.tensors import aligned_workspace, device_weights, to_dev, workspace_for  # noqa: F401

MARGIN = 0.05
TOL = {"bf16": 2e-2, "f32": 1e-4}


def run_gpu(dw, cfg: synth.Config, hidden: np.ndarray, anchor: np.ndarray, *, forced=None, target=None,
            want_logits=True, ws=None):
    B, K = hidden.shape[0], hidden.shape[1]
    dev = "cuda"
    h = to_dev(hidden, cfg.dtype)
    a = torch.from_numpy(np.asarray(anchor, np.int32)).to(dev)
    f = None if forced is None else torch.from_numpy(np.asarray(forced, np.int32)).to(dev)
    t = None if target is None else torch.from_numpy(np.asarray(target, np.int32)).to(dev)
    draft = torch.empty((B, K), dtype=torch.int32, device=dev)
    logits = torch.empty((B, K, cfg.V), dtype=torch.float32, device=dev) if want_logits else None
    tau = torch.empty((B,), dtype=torch.int32, device=dev) if target is not None else None
    ws = workspace_for(dw, B, K) if ws is None else ws
    dm.domino_draft_block(dw, h, a, mode=0 if cfg.mode == "greedy" else 1, temperature=cfg.temperature,
                          seed=cfg.seed, forced=f, target=t, draft_out=draft, logits_out=logits, tau_out=tau,
                          workspace=ws)
    st = dm.domino_poll(ws)
    torch.cuda.synchronize()
    return {
        "status": st,
        "tokens": draft.cpu().numpy(),
        "logits": None if logits is None else logits.cpu().numpy(),
        "tau": None if tau is None else tau.cpu().numpy(),
    }


def check_against_oracle(model: oracle.Model, cfg: synth.Config, hidden, anchor, gpu, *, target=None,
                         rows=None, forced=None):
    """Apply the comparison protocol; ``rows`` selects a sample of requests."""
    rows = np.arange(hidden.shape[0]) if rows is None else np.asarray(rows)
    feed = gpu["tokens"][rows] if forced is None else np.asarray(forced)[rows]
    ref = oracle.draft_block(model, hidden[rows], anchor[rows], mode=cfg.mode, temperature=cfg.temperature,
                             seed=cfg.seed, forced=feed, want_logits=gpu["logits"] is not None, request_ids=rows)
    g_tok = gpu["tokens"][rows]
    if forced is None:
        gap = ref.forced_gap
    else:   # picks are still reported under forcing: compare each against the best
        scores_gap = []
        for bi in range(len(rows)):
            scores_gap.append([0.0 if g_tok[bi, p] == ref.tokens[bi, p] else np.inf for p in range(cfg.K)])
        gap = np.asarray(scores_gap)
        near = (ref.top1 - ref.top2) <= MARGIN
        gap = np.where(near & np.isinf(gap), 0.0, gap)
    bad = gap > MARGIN
    assert not bad.any(), f"picks off beyond the {MARGIN} margin at {np.argwhere(bad)[:5].tolist()}"
    stats = {"agree": float((g_tok == ref.tokens).mean())}
    if gpu["logits"] is not None:
        err = np.abs(gpu["logits"][rows].astype(np.float64) - ref.logits).max()
        stats["logit_err"] = float(err)
        assert err <= TOL[cfg.dtype], f"final logits max-abs error {err} > {TOL[cfg.dtype]}"
    if target is not None and gpu["tau"] is not None:
        want = oracle.verify(g_tok, np.asarray(target)[rows])
        np.testing.assert_array_equal(gpu["tau"][rows], want)
    return ref, stats


# ---------------------------------------------------------------- stochastic verification

ACCEPT_TIE = 1e-5
SCORE_TIE = 1e-3


def emission_scores_of(dl, tl, b, pos, T, seed):
    """The oracle's Gumbel-max scores of request b's emitted token after pos accepted drafts."""
    K = dl.shape[1]
    q = oracle.softmax_rows(tl[b, pos].astype(np.float64), T)
    p = oracle.softmax_rows(dl[b, pos].astype(np.float64), T) if pos < K else None
    return oracle.emission_scores(p, q, seed, b, pos)


def check_verify_sample(dl, tl, draft, T, seed, tau, tok):
    """Comparison protocol of stochastic verification.

    Floating point decides integers here (accept or reject; the Gumbel-max
    draw).  A request whose acceptance test at any examined position lies within
    ACCEPT_TIE of its threshold (|u - min(1, q/p)|) is a precision tie and only
    checked for validity.  Otherwise tau must match the oracle exactly, and the
    emitted token must score within SCORE_TIE of the oracle's best draw (it is
    the oracle's own pick wherever the oracle's top-2 margin exceeds that).
    """
    ref = oracle.verify_sample(dl.astype(np.float64), tl.astype(np.float64), draft, T, seed)
    B, K, V = dl.shape
    stats = {"compared": 0, "ties": 0, "rejected": 0}
    for b in range(B):
        assert 0 <= tau[b] <= K and 0 <= tok[b] < V
        examined = min(int(ref.tau[b]) + 1, K)
        margin = np.abs(ref.uniform[b, :examined] - np.minimum(1.0, ref.ratio[b, :examined]))
        if (margin < ACCEPT_TIE).any():
            stats["ties"] += 1
            continue
        assert tau[b] == ref.tau[b], (b, tau[b], ref.tau[b])
        score = emission_scores_of(dl, tl, b, int(ref.tau[b]), T, seed)
        assert np.isfinite(score[tok[b]]), (b, tok[b])
        assert score[tok[b]] >= score.max() - SCORE_TIE, (b, tok[b], int(np.argmax(score)))
        stats["compared"] += 1
        stats["rejected"] += int(ref.tau[b] < K)
    return stats
