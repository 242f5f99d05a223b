"""Marshalling helpers: storage-form host arrays to device tensors, and workspaces.

Weights and hidden states are held on the host in storage form: bf16 values as
their uint16 bit patterns, fp32 values as float32.  These helpers move them to
the device as torch tensors of the matching dtype, and allocate the 256-byte
aligned workspaces the C ABI expects, with the control block zeroed.  None of
the method's arithmetic happens here.
"""
from __future__ import annotations

import numpy as np
import torch

from ._binding import DominoWeights, domino_workspace_bytes, domino_workspace_bytes_host, domino_workspace_init


def to_dev(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Storage-form numpy array -> contiguous device tensor (bf16 bits -> torch.bfloat16)."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    elif dtype == "f32":
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device)


def device_weights(w, device="cuda") -> DominoWeights:
    """A storage-form weight set on the device.

    ``w`` has the attributes dtype ("bf16" or "f32"), w_lm [V, d], embed [V, E]
    (the same object as w_lm when the table is tied), w_ih [3H, E], w_hh [3H, H],
    b_ih and b_hh ([3H] float32 or None), w1 [r, d + H] and w2 [V, r].
    """
    dt = w.dtype
    w_lm = to_dev(w.w_lm, dt, device)
    embed = w_lm if w.embed is w.w_lm else to_dev(w.embed, dt, device)
    b_ih = None if w.b_ih is None else torch.from_numpy(w.b_ih).to(device)
    b_hh = None if w.b_hh is None else torch.from_numpy(w.b_hh).to(device)
    return DominoWeights(w_lm, embed, to_dev(w.w_ih, dt, device), to_dev(w.w_hh, dt, device), b_ih, b_hh,
                         to_dev(w.w1, dt, device), to_dev(w.w2, dt, device))


def aligned_workspace(n: int, device="cuda") -> torch.Tensor:
    """n bytes of 256-byte aligned device memory with a zeroed control block."""
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    domino_workspace_init(ws)
    return ws


def workspace_for(dw: DominoWeights, B: int, K: int, host: bool = False, device="cuda") -> torch.Tensor:
    """The workspace of one draft block of B requests (``host``: the host-buffer entry point's)."""
    n = domino_workspace_bytes_host(dw, B, K) if host else domino_workspace_bytes(dw, B, K)
    return aligned_workspace(n, device)
