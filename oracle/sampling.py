"""fp64 CPU oracle of stochastic verification at T > 0 (speculative sampling).

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference legs may use it; the CUDA path never does.

The pages report Domino's acceptance at temperature 1 (Domino study notes,
gsyq.cn, §三.2(1)) but give no verification mechanism for T > 0.  Reading taken
here: the standard lossless speculative-sampling rule applied to the block's
draft distributions p_i = softmax(L_i / T) (L_i the final logits the drafted
tokens were sampled from) and the target model's q_i = softmax(Lq_i / T):

    for i = 1..K:
        accept t_i with probability min(1, q_i(t_i) / p_i(t_i));
        at the first rejection emit a token from norm(max(0, q_i - p_i)) and stop;
    if all K are accepted emit a bonus token from q_{K+1}.

tau counts the accepted draft tokens (0..K); the emitted token follows them.
Random numbers use the same Philox4x32-10 as the draft's Gumbel picks (key =
seed), on streams the draft never uses (counter word 3):
  - acceptance uniform of request b, position i (1-based): counter
    (0, i - 1, b, 2), word 0, u = (2 (w >> 9) + 1) 2^-24;
  - resampling noise over the vocabulary at position i (i = K + 1 for the
    bonus): Gumbel g[j] = -log(-log u) from counter (j >> 2, i - 1, b, 1),
    word j & 3; the residual sample is argmax_j (log r[j] + g[j]) (Gumbel-max,
    log 0 = -inf), the bonus argmax_j (log q[j] + g[j]).

A degenerate case the rule leaves open: a rejection whose residual
max(0, q_i - p_i) is zero everywhere in working precision.  This happens when
p_i and q_i agree to that precision except at the drafted token, whose
probability lies below it.  Reading taken here: the token is then drawn from
q_i with the same noise, which keeps the law of the emitted token equal to q_i.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .philox import _MASK32, philox4x32_10_np, uniform_from_word

STREAM_RESAMPLE = 1
STREAM_ACCEPT = 2


def _words(seed: int, b: int, pos0: int, stream: int, nblocks: int) -> np.ndarray:
    blocks = np.arange(nblocks, dtype=np.uint64)
    w = philox4x32_10_np(blocks, np.full_like(blocks, pos0), np.full_like(blocks, b),
                         np.full_like(blocks, stream), seed & _MASK32, (seed >> 32) & _MASK32)
    return np.stack(w, axis=1).reshape(-1)


def accept_uniform(seed: int, b: int, pos0: int) -> float:
    """Acceptance uniform of request b at 0-based position pos0."""
    return float(uniform_from_word(_words(seed, b, pos0, STREAM_ACCEPT, 1)[:1])[0])


def resample_noise(seed: int, b: int, pos0: int, V: int) -> np.ndarray:
    """Gumbel noise over the vocabulary for the residual / bonus sample at 0-based position pos0."""
    u = uniform_from_word(_words(seed, b, pos0, STREAM_RESAMPLE, (V + 3) // 4)[:V])
    return -np.log(-np.log(u))


def emission_scores(p_row, q_row, seed: int, b: int, pos0: int) -> np.ndarray:
    """Gumbel-max scores of the token emitted after the accepted prefix of request b.

    p_row is None for the bonus draw (pos0 = K): scores log q + g.  Otherwise
    the residual draw at the rejected 0-based position pos0: log max(0, q - p) + g,
    or log q + g when the residual is zero everywhere.
    """
    q_row = np.asarray(q_row, dtype=np.float64)
    noise = resample_noise(seed, b, pos0, q_row.shape[-1])
    with np.errstate(divide="ignore"):
        if p_row is not None:
            resid = np.maximum(q_row - np.asarray(p_row, dtype=np.float64), 0.0)
            if (resid > 0.0).any():
                return np.log(resid) + noise
        return np.log(q_row) + noise


def softmax_rows(logits: np.ndarray, temperature: float) -> np.ndarray:
    x = np.asarray(logits, dtype=np.float64) / float(temperature)
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return e / e.sum(axis=-1, keepdims=True)


@dataclasses.dataclass
class VerifyResult:
    tau: np.ndarray          # [B] accepted draft tokens
    token: np.ndarray        # [B] the emitted (residual or bonus) token
    ratio: np.ndarray        # [B, K] q_i(t_i) / p_i(t_i)
    uniform: np.ndarray      # [B, K] acceptance uniforms
    score_top2: np.ndarray   # [B, 2] best and second-best score of the emitted token's draw


def verify_sample(draft_logits: np.ndarray, target_logits: np.ndarray, draft: np.ndarray, temperature: float,
                  seed: int) -> VerifyResult:
    """Speculative sampling over one block per request.

    draft_logits [B, K, V] (the logits the draft tokens were drawn from, before
    temperature), target_logits [B, K + 1, V], draft [B, K].
    """
    B, K, V = draft_logits.shape
    p = softmax_rows(draft_logits, temperature)
    q = softmax_rows(target_logits, temperature)
    tau = np.zeros(B, dtype=np.int32)
    token = np.zeros(B, dtype=np.int32)
    ratio = np.zeros((B, K))
    uni = np.zeros((B, K))
    top2 = np.zeros((B, 2))
    for b in range(B):
        pos = K
        for i in range(K):
            t = int(draft[b, i])
            ratio[b, i] = q[b, i, t] / p[b, i, t]
            uni[b, i] = accept_uniform(seed, b, i)
            if not uni[b, i] < min(1.0, ratio[b, i]):
                pos = i
                break
        if pos < K:
            score = emission_scores(p[b, pos], q[b, pos], seed, b, pos)
        else:
            score = emission_scores(None, q[b, K], seed, b, K)
        tau[b] = pos
        token[b] = int(np.argmax(score))
        srt = np.sort(score)[-2:]
        top2[b] = [srt[1], srt[0]]
    return VerifyResult(tau, token, ratio, uni, top2)
