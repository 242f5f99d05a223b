"""fp64 CPU oracle of Domino's training forward (teacher forcing + base-anchored loss).

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference legs may use it; the CUDA path never does.

What it computes, from the Domino study notes (gsyq.cn), §二.2 配套专属训练方案:

1. Teacher-forced causal encoding (§二.2(1) Teacher-Forced): during training the
   GRU reads the ground-truth continuation instead of the drafter's own picks.
   Here the labels y[b, i] (the true token at block position i+1) are both the
   target of position i+1 and the GRU input after it, i.e. the draft block run
   with ``forced = labels``.
2. Base-anchored curriculum loss (§二.2(2)): the base logits and the corrected
   final logits are supervised jointly,
       L = (1 - lambda_t) L_final + lambda_t L_base,
   with lambda_t annealed linearly from 1 to 0 over training (an input here),
   and every position's loss carrying an exponentially decaying weight that
   favours the front of the block.

Readings where the notes are silent:
- the per-position loss is the cross-entropy -log softmax(L)[y] of the logits
  without temperature;
- the decay weight of block position i+1 (i = 0..K-1) is w_i = gamma**i with
  gamma in (0, 1] an input (the decay constant is not given);
- L_final and L_base are weighted means over positions and plain means over
  the batch: sum_{b,i} w_i CE[b, i] / (B sum_i w_i).
"""
from __future__ import annotations

import numpy as np

from .domino_ref import Model, draft_block


def cross_entropy_rows(logits: np.ndarray, labels: np.ndarray) -> np.ndarray:
    """-log softmax(logits[..., :])[label] for every row, in fp64.

    logits [..., V], labels [...] int.  log-sum-exp is taken around the row
    maximum so that it is exact for any finite logits.
    """
    x = np.asarray(logits, dtype=np.float64)
    y = np.asarray(labels, dtype=np.int64)
    m = x.max(axis=-1)
    lse = m + np.log(np.exp(x - m[..., None]).sum(axis=-1))
    picked = np.take_along_axis(x, y[..., None], axis=-1)[..., 0]
    return lse - picked


def position_weights(K: int, gamma: float) -> np.ndarray:
    """Exponentially decaying weight of block positions 1..K: gamma**(position - 1)."""
    return np.power(float(gamma), np.arange(K, dtype=np.float64))


def curriculum_loss(final_logits: np.ndarray, base_logits: np.ndarray, labels: np.ndarray, lam: float,
                    gamma: float):
    """(loss, ce_final [B, K], ce_base [B, K]) of the base-anchored curriculum loss."""
    ce_final = cross_entropy_rows(final_logits, labels)
    ce_base = cross_entropy_rows(base_logits, labels)
    B, K = ce_final.shape
    w = position_weights(K, gamma)
    l_final = float((ce_final * w).sum() / (B * w.sum()))
    l_base = float((ce_base * w).sum() / (B * w.sum()))
    return (1.0 - lam) * l_final + lam * l_base, ce_final, ce_base


def train_forward(model: Model, hidden: np.ndarray, anchor: np.ndarray, labels: np.ndarray, lam: float,
                  gamma: float, base: np.ndarray | None = None):
    """Teacher-forced forward of one block per request and its curriculum loss.

    Returns (loss, ce_final, ce_base, result) where result is the teacher-forced
    draft block (final logits L_i, base logits, picks).
    """
    res = draft_block(model, hidden, anchor, forced=labels, want_logits=True, base=base)
    loss, ce_final, ce_base = curriculum_loss(res.logits, res.base, labels, lam, gamma)
    return loss, ce_final, ce_base, res
