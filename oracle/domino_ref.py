"""Plain fp64 CPU oracle of the Domino draft block.

TEST INFRASTRUCTURE: this is the oracle that the CUDA path is checked against.
Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
legs may import it; the product path never does.  It shares no code with the
CUDA path: it reads storage-form tensors (bf16 bit patterns or fp32) produced by
``synth`` and widens them exactly to fp64 itself.

What it computes, in the pages' order and notation:

1. Base logits.  The parallel backbone's hidden state h_i of every block
   position goes once through the frozen target LM head:
   L_i^base = W_lm h_i  (Domino study notes, gsyq.cn, §二.1(1) 并行草稿主干;
   yhxrc.cn article, §三 第一个阶段).
2. Causal encoder.  A GRU (hidden 1024 in the pages) reads the embeddings of the
   tokens already fixed in the block one by one; at position i its state
   S_{i-1} summarises the tokens before i (study notes §二.1(2) item 1;
   yhxrc.cn §四 因果編碼器).  Reading taken here: the state starts at zero and
   the first input is the anchor token x_t, so position i sees the GRU after it
   consumed (anchor, t_1, ..., t_{i-1}).  Gates follow PyTorch's GRU (r, z, n
   order, b_hn inside r * (.)).
3. Low-rank correction.  [h_i ; S_{i-1}] (hidden state first) -> W1 -> rank-256
   bottleneck -> SiLU -> W2 -> vocabulary gives Delta L_i (study notes §二.1(2)
   item 2; yhxrc.cn §四 低秩修正頭).  No biases are stated, none are used.
4. Logit residual.  L_i = L_i^base + Delta L_i (study notes §二.1(2) item 3).
5. Pick.  Greedy at T=0: t_i = argmax_j L_i[j], lowest index on ties.  At T>0
   (the pages report T=1 runs, study notes §三.2(1), but give no mechanism):
   Gumbel-max, t_i = argmax_j (L_i[j] / T + g[b, i, j]) with Philox noise
   (see ``oracle.philox``).  t_i is fed back as the next GRU input, or, in the
   teacher-forced mode (study notes §二.2(1) Teacher-Forced), a given token is
   fed instead while the pick is still reported.
6. Verification.  The acceptance length tau is the number of leading draft
   tokens that equal the target's (study notes §一.1 接受长度τ; digest page
   "大三本科生一作…" §4 简单批量验证).
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .philox import gumbel_noise


# ---------------------------------------------------------------- storage -> fp64

def widen_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of storage-form values to fp64.

    bf16 values are stored as their uint16 bit pattern: the value is the fp32
    number whose top 16 bits are those bits and whose low 16 bits are zero.
    """
    if dtype == "bf16":
        bits = np.asarray(a, dtype=np.uint16)
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    raise ValueError(f"unknown storage dtype {dtype!r}")


# ---------------------------------------------------------------- elementary ops

def sigmoid(x: np.ndarray) -> np.ndarray:
    """Logistic function 1 / (1 + e^-x)."""
    return 1.0 / (1.0 + np.exp(-x))


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x) (the bottleneck activation, yhxrc.cn §四)."""
    return x * sigmoid(x)


def gru_cell(x, s, w_ih, w_hh, b_ih, b_hh):
    """One GRU step on a batch: x [B, E], s [B, H] -> new state [B, H].

    r = sigmoid(W_ir x + b_ir + W_hr s + b_hr)
    z = sigmoid(W_iz x + b_iz + W_hz s + b_hz)
    n = tanh(W_in x + b_in + r * (W_hn s + b_hn))
    s' = (1 - z) * n + z * s
    with the gate rows of W_ih / W_hh / b_ih / b_hh stacked in the order r, z, n.
    """
    H = s.shape[-1]
    gi = x @ w_ih.T + b_ih
    gh = s @ w_hh.T + b_hh
    r = sigmoid(gi[:, 0:H] + gh[:, 0:H])
    z = sigmoid(gi[:, H:2 * H] + gh[:, H:2 * H])
    n = np.tanh(gi[:, 2 * H:3 * H] + r * gh[:, 2 * H:3 * H])
    return (1.0 - z) * n + z * s


def lm_head(hidden64: np.ndarray, w_lm: np.ndarray, dtype: str, chunk: int = 16384) -> np.ndarray:
    """Base logits L^base[b, i, v] = sum_k W_lm[v, k] h[b, i, k] in fp64.

    hidden64: [B, K, d] fp64; w_lm in storage form [V, d].  W_lm is widened in
    row chunks so the 8B-shaped table never exists whole in fp64.
    """
    B, K, d = hidden64.shape
    V = w_lm.shape[0]
    out = np.empty((B, K, V), dtype=np.float64)
    hk = hidden64.reshape(B * K, d)
    for v0 in range(0, V, chunk):
        w = widen_f64(w_lm[v0:v0 + chunk], dtype)
        out.reshape(B * K, V)[:, v0:v0 + w.shape[0]] = hk @ w.T
    return out


def verify(draft: np.ndarray, target: np.ndarray) -> np.ndarray:
    """Acceptance length: number of leading positions where draft == target."""
    draft = np.asarray(draft)
    target = np.asarray(target)
    B, K = draft.shape
    tau = np.zeros(B, dtype=np.int32)
    for b in range(B):
        n = 0
        while n < K and draft[b, n] == target[b, n]:
            n += 1
        tau[b] = n
    return tau


# ---------------------------------------------------------------- the block

@dataclasses.dataclass
class Model:
    """fp64 view of a weight set (W_lm and the embedding stay in storage form)."""
    dtype: str
    w_lm: np.ndarray      # storage [V, d]
    embed: np.ndarray     # storage [V, E]
    w_ih: np.ndarray      # fp64 [3H, E]
    w_hh: np.ndarray      # fp64 [3H, H]
    b_ih: np.ndarray      # fp64 [3H]
    b_hh: np.ndarray      # fp64 [3H]
    w1: np.ndarray        # fp64 [r, d + H]
    w2: np.ndarray        # fp64 [V, r]

    @classmethod
    def from_storage(cls, w) -> "Model":
        dt = w.dtype
        H3 = w.w_ih.shape[0]

        def bias(a):  # GRU biases are fp32 in storage; absent means zero
            return np.zeros(H3) if a is None else np.asarray(a, np.float32).astype(np.float64)

        return cls(dt, w.w_lm, w.embed, widen_f64(w.w_ih, dt), widen_f64(w.w_hh, dt),
                   bias(w.b_ih), bias(w.b_hh), widen_f64(w.w1, dt), widen_f64(w.w2, dt))

    @property
    def V(self) -> int:
        return self.w2.shape[0]

    @property
    def H(self) -> int:
        return self.w_hh.shape[1]

    def embed_rows(self, tokens: np.ndarray) -> np.ndarray:
        """Embedding lookup x = E[t] for a batch of tokens, widened to fp64."""
        return widen_f64(self.embed[np.asarray(tokens, dtype=np.int64)], self.dtype)


@dataclasses.dataclass
class Result:
    tokens: np.ndarray        # [B, K] int32 picks t_1..t_K
    logits: np.ndarray | None  # [B, K, V] fp64 final logits L_i (before temperature / noise)
    base: np.ndarray          # [B, K, V] fp64 base logits
    top1: np.ndarray          # [B, K] best pick score
    top2: np.ndarray          # [B, K] second-best pick score
    forced_gap: np.ndarray | None  # [B, K] best score minus the score of the fed token
    tau: np.ndarray | None    # [B] acceptance length (if a target was given)


def positions(model: Model, hidden64: np.ndarray, anchor: np.ndarray, base: np.ndarray, *,
              mode: str = "greedy", temperature: float = 1.0, seed: int = 0,
              forced: np.ndarray | None = None, request_ids: np.ndarray | None = None):
    """The sequential correction loop, one block position per iteration.

    Yields (p, L, score, pick) for p = 0..K-1 (block position i = p + 1): the
    final logits L_i [B, V], the pick scores and the picks.
    """
    B, K, d = hidden64.shape
    V, H = model.V, model.H
    rid = np.arange(B) if request_ids is None else np.asarray(request_ids, dtype=np.int64)
    s = np.zeros((B, H))
    prev = np.asarray(anchor, dtype=np.int64).copy()
    for p in range(K):                      # block position i = p + 1
        x = model.embed_rows(prev)          # embedding of the token fed at this step
        s = gru_cell(x, s, model.w_ih, model.w_hh, model.b_ih, model.b_hh)   # S_{i-1}
        cat = np.concatenate([hidden64[:, p, :], s], axis=1)                 # [h_i ; S_{i-1}]
        u = silu(cat @ model.w1.T)                                           # rank-r bottleneck
        L = base[:, p, :] + u @ model.w2.T                                   # L_i = L_i^base + dL_i
        if mode == "greedy":
            score = L
        else:
            g = np.stack([gumbel_noise(seed, int(rid[b]), p + 1, V) for b in range(B)])
            score = L / temperature + g
        pick = np.argmax(score, axis=1)      # first index among equal maxima
        yield p, L, score, pick
        prev = np.asarray(forced, dtype=np.int64)[:, p] if forced is not None else pick.astype(np.int64)


def draft_block(model: Model, hidden: np.ndarray, anchor: np.ndarray, *,
                mode: str = "greedy", temperature: float = 1.0, seed: int = 0,
                forced: np.ndarray | None = None, target: np.ndarray | None = None,
                want_logits: bool = True, base: np.ndarray | None = None,
                request_ids: np.ndarray | None = None) -> Result:
    """Run one draft block for every request.

    hidden: storage-form [B, K, d]; anchor: [B] int.  ``forced`` [B, K] feeds
    forced[b, i] to the GRU after position i instead of the pick (the last
    column is never fed).  ``base`` may pass precomputed fp64 base logits.
    ``request_ids`` [B] names each row's request index in the Gumbel stream
    (default 0..B-1), so a sample of a larger batch draws the same noise.
    """
    if mode not in ("greedy", "gumbel"):
        raise ValueError(mode)
    if mode == "gumbel" and not temperature > 0:
        raise ValueError("Gumbel picks need T > 0")
    h64 = widen_f64(hidden, model.dtype)
    B, K, d = h64.shape
    V = model.V
    if base is None:
        base = lm_head(h64, model.w_lm, model.dtype)

    tokens = np.zeros((B, K), dtype=np.int32)
    top1 = np.zeros((B, K))
    top2 = np.zeros((B, K))
    gap = np.zeros((B, K)) if forced is not None else None
    logits = np.zeros((B, K, V)) if want_logits else None
    for p, L, score, pick in positions(model, h64, anchor, base, mode=mode, temperature=temperature, seed=seed,
                                       forced=forced, request_ids=request_ids):
        if logits is not None:
            logits[:, p, :] = L
        tokens[:, p] = pick
        srt = np.partition(score, V - 2, axis=1)[:, V - 2:]
        top2[:, p] = srt[:, 0]
        top1[:, p] = srt[:, 1]
        if forced is not None:
            fed = np.asarray(forced, dtype=np.int64)[:, p]
            gap[:, p] = top1[:, p] - score[np.arange(B), fed]
    tau = verify(tokens, target) if target is not None else None
    return Result(tokens, logits, base, top1, top2, gap, tau)
