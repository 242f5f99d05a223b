"""B200-native Domino draft-block hot path.

The compute lives in ``libdomino.so`` (CUDA C++ for sm_100a, C ABI declared in
include/domino.h).  This package is a thin ctypes binding with the same entry
point names: it only marshals torch tensors (device memory) and CUDA streams to
plain pointers.  There is no CPU fallback: every call raises if the library is
missing or returns an error.
"""
from ._binding import (DominoError, DominoWeights, STATUS, domino_build_gate_table, domino_correct_loop,
                       domino_correct_loop_noalloc, domino_gate_table_bytes,
                       domino_curriculum_loss, domino_curriculum_loss_workspace_bytes, domino_draft_block,
                       domino_draft_block_events, domino_draft_block_host, domino_draft_loss,
                       domino_draft_loss_workspace_bytes, domino_launches_per_block, domino_lm_head, domino_poll,
                       domino_selftest_wait_timeout, domino_set_wait_budget_ns, domino_status_str, domino_verify,
                       domino_verify_sample, domino_verify_sample_workspace_bytes, domino_workspace_bytes, domino_workspace_bytes_host, domino_workspace_init, library_path,
                       load_library)

GREEDY = 0
GUMBEL = 1
BF16 = 0
F32 = 1

__all__ = [
    "DominoError", "DominoWeights", "STATUS", "GREEDY", "GUMBEL", "BF16", "F32", "domino_build_gate_table",
    "domino_gate_table_bytes",
    "domino_correct_loop", "domino_correct_loop_noalloc", "domino_curriculum_loss",
    "domino_curriculum_loss_workspace_bytes", "domino_draft_block", "domino_draft_block_events",
    "domino_draft_block_host", "domino_draft_loss", "domino_draft_loss_workspace_bytes", "domino_launches_per_block",
    "domino_lm_head", "domino_poll", "domino_selftest_wait_timeout", "domino_set_wait_budget_ns", "domino_status_str",
    "domino_verify", "domino_verify_sample", "domino_verify_sample_workspace_bytes", "domino_workspace_bytes", "domino_workspace_bytes_host", "domino_workspace_init",
    "library_path", "load_library",
]
