"""fp64 CPU oracle of the Domino draft block.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference legs may import this package.  The product path
(``draft_model_b200``) never imports, calls or links it, and shares no code
with it; the two meet only at the seeded inputs from ``synth``.

Pins (tests/test_oracle_pins.py): Philox against its published known-answer
vectors; the GRU step against torch.nn.GRUCell and a hand-computed closed form;
SiLU against its closed form; the LM head against a brute-force triple loop;
zero-correction invariants; teacher-forcing and causality invariants; a
brute-force greedy fixed point; the exact Gumbel-max law; tau by brute force;
the head's parameter count against the pages' "56M"; the training loss's
cross-entropy against torch's and closed forms (uniform rows, two-way rows),
its curriculum mix and position weights against their limits; stochastic
verification against the exact output law of speculative sampling (chi-square),
its acceptance rate, and its p == q and q(t) == 0 limits.
"""
from .domino_ref import Model, Result, draft_block, gru_cell, lm_head, positions, sigmoid, silu, verify, widen_f64
from .philox import gumbel_noise, philox4x32_10, philox4x32_10_np, uniform_from_word
from .sampling import VerifyResult, accept_uniform, emission_scores, resample_noise, softmax_rows, verify_sample
from .training import cross_entropy_rows, curriculum_loss, position_weights, train_forward

__all__ = ["Model", "Result", "draft_block", "gru_cell", "lm_head", "positions", "sigmoid", "silu", "verify",
           "widen_f64", "gumbel_noise", "philox4x32_10", "philox4x32_10_np", "uniform_from_word",
           "cross_entropy_rows", "curriculum_loss", "position_weights", "train_forward",
           "VerifyResult", "accept_uniform", "resample_noise", "softmax_rows", "verify_sample"]
