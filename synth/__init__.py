"""Seeded synthetic inputs for the Domino draft-block hot path.

This module only draws random numbers and rounds them to the storage type.  It
holds none of the method's arithmetic (no projection, no GRU, no correction, no
pick, no verification), so both the fp64 oracle and the CUDA path may consume
its tensors without sharing any computation.

Shapes follow the Qwen3 targets named by the pages (Domino study notes,
gsyq.cn, §三.1 实验基础配置: Qwen3-4B / Qwen3-8B, block size 16).  The pages'
evaluation datasets (GSM8K, MATH-500, AIME25, HumanEval, MBPP, LiveCodeBench,
MT-Bench, Alpaca) are not available; seeded Gaussian hidden states and uniform
anchor tokens stand in for them.  No dataset item is reproduced.

Recipe (one generator per tensor, ``numpy.random.default_rng([seed, tensor_id,
chunk])``, standard normal in fp32, scaled, then rounded to bf16 with
round-to-nearest-even):

* W_lm ~ N(0, 1/d) x 4 (logit std ~ 4), embedding E ~ N(0, 1/d) (or E is W_lm
  when tied), W_ih ~ N(0, 1/E), W_hh ~ N(0, 1/H), W1 ~ N(0, 1/(d+H)),
  W2 ~ N(0, 1/r); GRU biases b_ih, b_hh ~ N(0, 1/H) kept in fp32;
* backbone hidden states ~ N(0, 1); anchor tokens uniform in [0, V);
* synthetic target tokens agree with a given draft on a Geometric(p) prefix
  (support {0, 1, ...}, capped at K), then differ.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# tensor ids: fixed so every tensor has its own independent stream
TID_W_LM, TID_EMBED, TID_W_IH, TID_W_HH, TID_B_IH, TID_B_HH = 1, 2, 3, 4, 5, 6
TID_W1, TID_W2, TID_HIDDEN, TID_ANCHOR, TID_TARGET = 7, 8, 9, 10, 11

_CHUNK = 1 << 22  # elements per independent generator chunk (threaded fill)


@dataclasses.dataclass(frozen=True)
class Config:
    """One synthetic workload: shapes, dtype, pick mode and target recipe."""
    name: str
    B: int
    K: int
    d: int
    V: int
    H: int
    r: int
    E: int
    dtype: str            # "bf16" or "f32": storage type of weights and hidden states
    tied: bool            # embedding table is the (scaled) W_lm tensor itself
    mode: str = "greedy"  # "greedy" or "gumbel"
    temperature: float = 1.0
    seed: int = 0         # config seed for all tensors and the Gumbel stream
    target_p: float = 0.1  # geometric parameter of the synthetic acceptance prefix
    target_prefix: int | None = None  # fixed prefix length (overrides target_p)

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)

    @property
    def head_params(self) -> int:
        """Domino-head parameters: W1, W2 and the GRU weight matrices."""
        return self.r * (self.d + self.H) + self.V * self.r + 3 * self.H * (self.E + self.H)


QWEN3_8B = dict(d=4096, V=151936, H=1024, r=256, E=4096, dtype="bf16", tied=False)
QWEN3_4B = dict(d=2560, V=151936, H=1024, r=256, E=2560, dtype="bf16", tied=True)

CONFIGS = {
    "tiny_f32": Config("tiny_f32", B=1, K=4, d=64, V=512, H=32, r=16, E=64, dtype="f32",
                       tied=False, mode="greedy", seed=0, target_prefix=3),
    "qwen3_4b_b1": Config("qwen3_4b_b1", B=1, K=16, mode="greedy", target_p=0.15, **QWEN3_4B),
    "qwen3_8b_b1": Config("qwen3_8b_b1", B=1, K=16, mode="greedy", target_p=0.10, **QWEN3_8B),
    "qwen3_8b_b32_gumbel": Config("qwen3_8b_b32_gumbel", B=32, K=16, mode="gumbel",
                                  temperature=1.0, target_p=0.20, **QWEN3_8B),
}
SWEEP_BATCHES = (1, 2, 8, 32, 128, 256)


def sweep_config(B: int) -> Config:
    """Qwen3-8B batch-sweep member: greedy, block 16, same weights for every B."""
    return Config(f"qwen3_8b_sweep_b{B}", B=B, K=16, mode="greedy", target_p=0.10, **QWEN3_8B)


# ---------------------------------------------------------------- primitives

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even) and return the raw uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits to fp32 (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(seed: int, tid: int, n: int, scale: float, out_dtype: str) -> np.ndarray:
    """n scaled standard normals, chunked so chunks can be drawn on threads.

    Returns uint16 bf16 bits when out_dtype == "bf16", else float32.
    """
    out = np.empty(n, dtype=np.uint16 if out_dtype == "bf16" else np.float32)
    nch = max(1, (n + _CHUNK - 1) // _CHUNK)

    def fill(c: int) -> None:
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        a = np.random.default_rng([seed, tid, c]).standard_normal(hi - lo, dtype=np.float32)
        a *= np.float32(scale)
        out[lo:hi] = f32_to_bf16_bits(a) if out_dtype == "bf16" else a

    if nch == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(8) as ex:
            list(ex.map(fill, range(nch)))
    return out


# ---------------------------------------------------------------- tensors

@dataclasses.dataclass
class Weights:
    """Domino-head weights in storage form.

    bf16 tensors are held as uint16 bit patterns, f32 tensors as float32.
    ``embed`` is the same array object as ``w_lm`` when the table is tied.
    """
    dtype: str
    w_lm: np.ndarray   # [V, d]
    embed: np.ndarray  # [V, E]
    w_ih: np.ndarray   # [3H, E], gate rows r, z, n
    w_hh: np.ndarray   # [3H, H]
    b_ih: np.ndarray   # [3H] float32
    b_hh: np.ndarray   # [3H] float32
    w1: np.ndarray     # [r, d + H]
    w2: np.ndarray     # [V, r]


def make_weights(cfg: Config) -> Weights:
    """Draw the weight set of a config (depends on shapes, dtype and seed only)."""
    s, dt = cfg.seed, cfg.dtype
    V, d, H, r, E = cfg.V, cfg.d, cfg.H, cfg.r, cfg.E
    w_lm = _normal(s, TID_W_LM, V * d, 4.0 / np.sqrt(d), dt).reshape(V, d)
    if cfg.tied:
        if E != d:
            raise ValueError("a tied embedding table needs E == d")
        embed = w_lm
    else:
        embed = _normal(s, TID_EMBED, V * E, 1.0 / np.sqrt(d), dt).reshape(V, E)
    w_ih = _normal(s, TID_W_IH, 3 * H * E, 1.0 / np.sqrt(E), dt).reshape(3 * H, E)
    w_hh = _normal(s, TID_W_HH, 3 * H * H, 1.0 / np.sqrt(H), dt).reshape(3 * H, H)
    b_ih = _normal(s, TID_B_IH, 3 * H, 1.0 / np.sqrt(H), "f32")
    b_hh = _normal(s, TID_B_HH, 3 * H, 1.0 / np.sqrt(H), "f32")
    w1 = _normal(s, TID_W1, r * (d + H), 1.0 / np.sqrt(d + H), dt).reshape(r, d + H)
    w2 = _normal(s, TID_W2, V * r, 1.0 / np.sqrt(r), dt).reshape(V, r)
    return Weights(dt, w_lm, embed, w_ih, w_hh, b_ih, b_hh, w1, w2)


def make_hidden(cfg: Config, B: int | None = None, first: int = 0) -> np.ndarray:
    """Backbone hidden states [B, K, d] ~ N(0, 1) in storage form.

    Request b is drawn from its own stream, so any slice of requests (the first B
    of the batch sweep, one replica's share) matches the same rows of a larger
    draw.  ``first`` is the global index of the first request returned.
    """
    B = cfg.B if B is None else B
    rows = [_normal(cfg.seed, TID_HIDDEN * 1000003 + first + b, cfg.K * cfg.d, 1.0, cfg.dtype) for b in range(B)]
    return np.stack(rows).reshape(B, cfg.K, cfg.d)


def make_anchor(cfg: Config, B: int | None = None, first: int = 0) -> np.ndarray:
    """Anchor (last confirmed) tokens [B] uniform in [0, V), int32."""
    B = cfg.B if B is None else B
    out = np.empty(B, dtype=np.int32)
    for b in range(B):
        out[b] = np.random.default_rng([cfg.seed, TID_ANCHOR, first + b]).integers(0, cfg.V)
    return out


def make_targets(cfg: Config, draft: np.ndarray) -> np.ndarray:
    """Synthetic target tokens that agree with ``draft`` on a random prefix.

    Prefix length n ~ Geometric(p) on {0, 1, ...}, capped at K (or the config's
    fixed prefix).  Position n (if < K) gets a uniform token different from the
    draft's; later positions are uniform.
    """
    draft = np.asarray(draft, dtype=np.int32)
    B, K = draft.shape
    out = np.empty_like(draft)
    for b in range(B):
        rng = np.random.default_rng([cfg.seed, TID_TARGET, b])
        if cfg.target_prefix is not None:
            n = min(cfg.target_prefix, K)
        else:
            n = min(int(rng.geometric(cfg.target_p)) - 1, K)
        out[b, :n] = draft[b, :n]
        for i in range(n, K):
            t = int(rng.integers(0, cfg.V))
            if i == n:
                while t == int(draft[b, i]):
                    t = int(rng.integers(0, cfg.V))
            out[b, i] = t
    return out


def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage form -> float32 values (exact)."""
    return bf16_bits_to_f32(a) if dtype == "bf16" else np.asarray(a, dtype=np.float32)
