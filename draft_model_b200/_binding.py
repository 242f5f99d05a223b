"""ctypes binding of libdomino.so: argument marshalling only."""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdomino.so")
_lib = None

STATUS = {
    0: "DOMINO_OK", 1: "DOMINO_ERR_INVALID_ARG", 2: "DOMINO_ERR_UNSUPPORTED", 3: "DOMINO_ERR_LAUNCH",
    4: "DOMINO_ERR_CUDA", 5: "DOMINO_ERR_TIMEOUT", 6: "DOMINO_ERR_BAD_TOKEN", 7: "DOMINO_ERR_WORKSPACE",
}


class DominoError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class _CWeights(ctypes.Structure):
    _fields_ = [
        ("vocab", ctypes.c_int32), ("d_model", ctypes.c_int32), ("embed_dim", ctypes.c_int32),
        ("gru_hidden", ctypes.c_int32), ("rank", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("w_lm", ctypes.c_void_p), ("embed", ctypes.c_void_p), ("w_ih", ctypes.c_void_p),
        ("w_hh", ctypes.c_void_p), ("b_ih", ctypes.c_void_p), ("b_hh", ctypes.c_void_p),
        ("w1", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("gate_table", ctypes.c_void_p),
    ]


def library_path() -> str:
    return _LIB_PATH


def load_library() -> ctypes.CDLL:
    """Load libdomino.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing; build it with `python -m draft_model_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I32, U64, F, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_float, ctypes.c_size_t
    W = ctypes.POINTER(_CWeights)
    sig = {
        "domino_workspace_bytes": (SZ, [W, I32, I32]),
        "domino_workspace_bytes_host": (SZ, [W, I32, I32]),
        "domino_launches_per_block": (I32, [W, I32, I32]),
        "domino_curriculum_loss_workspace_bytes": (SZ, [I32, I32, I32]),
        "domino_curriculum_loss": (I32, [P, P, P, I32, I32, I32, F, F, P, P, P, SZ, P]),
        "domino_draft_loss_workspace_bytes": (SZ, [W, I32, I32]),
        "domino_draft_loss": (I32, [W, P, P, P, I32, I32, F, F, P, P, P, SZ, P]),
        "domino_verify_sample_workspace_bytes": (SZ, [I32, I32, I32]),
        "domino_gate_table_bytes": (SZ, [W]),
        "domino_build_gate_table": (I32, [W, P, P, SZ, P]),
        "domino_verify_sample": (I32, [P, P, P, I32, I32, I32, F, U64, P, P, P, SZ, P]),
        "domino_workspace_init": (I32, [P, SZ, P]),
        "domino_draft_block": (I32, [W, P, P, I32, I32, I32, F, U64, P, P, P, P, P, P, SZ, P]),
        "domino_draft_block_events": (I32, [W, P, P, I32, I32, I32, F, U64, P, P, P, P, P, P, SZ, P,
                                             ctypes.POINTER(ctypes.c_void_p)]),
        "domino_lm_head": (I32, [W, P, I32, I32, P, P, SZ, P]),
        "domino_correct_loop": (I32, [W, P, P, P, I32, I32, I32, F, U64, P, P, P, P, P, P, SZ, P]),
        "domino_correct_loop_noalloc": (I32, [W, P, P, P, I32, I32, I32, F, U64, P, P, P, P, P, P]),
        "domino_verify": (I32, [P, P, I32, I32, P, P]),
        "domino_draft_block_host": (I32, [W, P, P, I32, I32, I32, F, U64, P, P, P, P, P, SZ, P]),
        "domino_poll": (I32, [P, P]),
        "domino_set_wait_budget_ns": (None, [U64]),
        "domino_selftest_wait_timeout": (I32, [P, SZ, U64, P]),
        "domino_status_str": (ctypes.c_char_p, [I32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


# ---------------------------------------------------------------- marshalling helpers

def _ptr(t) -> int | None:
    """Device pointer: a contiguous CUDA tensor, None, or a raw integer address."""
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_cuda:
            raise ValueError("expected a CUDA tensor (device memory), got a tensor on " + str(t.device))
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return t.data_ptr()
    return int(t)


def _hptr(t) -> int | None:
    """Host pointer: a contiguous CPU tensor (pinned memory makes the copies asynchronous),
    None, or a raw integer address."""
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if t.is_cuda:
            raise ValueError("expected a host (CPU) tensor, got a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return t.data_ptr()
    return int(t)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str) -> None:
    if status != 0:
        raise DominoError(status, where)


class DominoWeights:
    """Keeps the weight tensors alive and exposes the C struct.

    Tensors: w_lm [V, d], embed [V, E] (may be w_lm), w_ih [3H, E], w_hh [3H, H],
    b_ih / b_hh [3H] float32 or None, w1 [r, d + H], w2 [V, r]; all bfloat16 or all
    float32 (biases always float32), contiguous, on the device.
    """

    def __init__(self, w_lm, embed, w_ih, w_hh, b_ih, b_hh, w1, w2):
        dt = w_lm.dtype
        if dt not in (torch.bfloat16, torch.float32):
            raise ValueError("weights must be bfloat16 or float32")
        for t in (embed, w_ih, w_hh, w1, w2):
            if t.dtype != dt:
                raise ValueError("all weight matrices must share one dtype")
        self.tensors = (w_lm, embed, w_ih, w_hh, b_ih, b_hh, w1, w2)
        V, d = w_lm.shape
        E = embed.shape[1]
        H = w_hh.shape[1]
        r = w1.shape[0]
        self.V, self.d, self.E, self.H, self.r = V, d, E, H, r
        self.dtype = dt
        self.c = _CWeights(V, d, E, H, r, 0 if dt == torch.bfloat16 else 1,
                           _ptr(w_lm), _ptr(embed), _ptr(w_ih), _ptr(w_hh), _ptr(b_ih), _ptr(b_hh),
                           _ptr(w1), _ptr(w2))

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def set_gate_table(self, table) -> None:
        """Use a [V, 3H] float32 token->gate table (domino_build_gate_table), or None."""
        self.gate_table = table
        self.c.gate_table = _ptr(table)


# ---------------------------------------------------------------- entry points (same names as the C ABI)

def domino_workspace_bytes(w: DominoWeights, B: int, K: int) -> int:
    return int(load_library().domino_workspace_bytes(w.ref, B, K))


def domino_workspace_bytes_host(w: DominoWeights, B: int, K: int) -> int:
    return int(load_library().domino_workspace_bytes_host(w.ref, B, K))


def domino_launches_per_block(w: DominoWeights, B: int, K: int) -> int:
    return int(load_library().domino_launches_per_block(w.ref, B, K))


def domino_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check(load_library().domino_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                                _stream(stream)), "domino_workspace_init")


def _ws(workspace):
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def domino_draft_block(w: DominoWeights, hidden, anchor, *, mode=0, temperature=1.0, seed=0, forced=None,
                       target=None, draft_out, logits_out=None, tau_out=None, workspace, stream=None) -> None:
    B, K = draft_out.shape
    wp, wn = _ws(workspace)
    _check(load_library().domino_draft_block(w.ref, _ptr(hidden), _ptr(anchor), B, K, mode, temperature, seed,
                                             _ptr(forced), _ptr(target), _ptr(draft_out), _ptr(logits_out),
                                             _ptr(tau_out), wp, wn, _stream(stream)), "domino_draft_block")


def domino_draft_block_events(w: DominoWeights, hidden, anchor, *, mode=0, temperature=1.0, seed=0, forced=None,
                              target=None, draft_out, logits_out=None, tau_out=None, workspace, stream=None,
                              events) -> None:
    """domino_draft_block recording three torch.cuda.Event objects around its stages."""
    B, K = draft_out.shape
    wp, wn = _ws(workspace)
    arr = (ctypes.c_void_p * 3)(*[None if e is None else e.cuda_event for e in events])
    _check(load_library().domino_draft_block_events(w.ref, _ptr(hidden), _ptr(anchor), B, K, mode, temperature, seed,
                                                    _ptr(forced), _ptr(target), _ptr(draft_out), _ptr(logits_out),
                                                    _ptr(tau_out), wp, wn, _stream(stream), arr),
           "domino_draft_block_events")


def domino_lm_head(w: DominoWeights, hidden, base_out, *, workspace, stream=None) -> None:
    B, K = hidden.shape[0], hidden.shape[1]
    wp, wn = _ws(workspace)
    _check(load_library().domino_lm_head(w.ref, _ptr(hidden), B, K, _ptr(base_out), wp, wn, _stream(stream)),
           "domino_lm_head")


def domino_correct_loop(w: DominoWeights, hidden, base, anchor, *, mode=0, temperature=1.0, seed=0, forced=None,
                        target=None, draft_out, logits_out=None, tau_out=None, workspace, stream=None) -> None:
    B, K = draft_out.shape
    wp, wn = _ws(workspace)
    _check(load_library().domino_correct_loop(w.ref, _ptr(hidden), _ptr(base), _ptr(anchor), B, K, mode,
                                              temperature, seed, _ptr(forced), _ptr(target), _ptr(draft_out),
                                              _ptr(logits_out), _ptr(tau_out), wp, wn, _stream(stream)),
           "domino_correct_loop")


def domino_correct_loop_noalloc(w: DominoWeights, hidden, base, anchor, *, mode=0, temperature=1.0, seed=0,
                                forced=None, target=None, draft_out, logits_out=None, tau_out=None,
                                stream=None) -> None:
    """Stage 2 without a workspace (scratch in a fixed array inside the library); waits for its work."""
    B, K = draft_out.shape
    _check(load_library().domino_correct_loop_noalloc(w.ref, _ptr(hidden), _ptr(base), _ptr(anchor), B, K, mode,
                                                      temperature, seed, _ptr(forced), _ptr(target),
                                                      _ptr(draft_out), _ptr(logits_out), _ptr(tau_out),
                                                      _stream(stream)), "domino_correct_loop_noalloc")


def domino_curriculum_loss_workspace_bytes(B: int, K: int, V: int) -> int:
    return int(load_library().domino_curriculum_loss_workspace_bytes(B, K, V))


def domino_curriculum_loss(final_logits, base_logits, labels, *, lam: float, gamma: float, loss_out, ce_out=None,
                           workspace, stream=None) -> None:
    """Base-anchored curriculum loss of [B, K, V] fp32 logits against [B, K] labels."""
    B, K, V = final_logits.shape
    wp, wn = _ws(workspace)
    _check(load_library().domino_curriculum_loss(_ptr(final_logits), _ptr(base_logits), _ptr(labels), B, K, V, lam,
                                                 gamma, _ptr(ce_out), _ptr(loss_out), wp, wn, _stream(stream)),
           "domino_curriculum_loss")


def domino_draft_loss_workspace_bytes(w: DominoWeights, B: int, K: int) -> int:
    return int(load_library().domino_draft_loss_workspace_bytes(w.ref, B, K))


def domino_draft_loss(w: DominoWeights, hidden, anchor, labels, *, lam: float, gamma: float, loss_out, ce_out=None,
                      workspace, stream=None) -> None:
    """Teacher-forced training forward (GRU fed the labels) and its curriculum loss."""
    B, K = labels.shape
    wp, wn = _ws(workspace)
    _check(load_library().domino_draft_loss(w.ref, _ptr(hidden), _ptr(anchor), _ptr(labels), B, K, lam, gamma,
                                            _ptr(ce_out), _ptr(loss_out), wp, wn, _stream(stream)),
           "domino_draft_loss")


def domino_verify_sample_workspace_bytes(B: int, K: int, V: int) -> int:
    return int(load_library().domino_verify_sample_workspace_bytes(B, K, V))


def domino_verify_sample(draft_logits, target_logits, draft, *, temperature: float, seed: int, tau_out, token_out,
                         workspace, stream=None) -> None:
    """Speculative sampling of a block: accepted draft tokens and the emitted token per request."""
    B, K, V = draft_logits.shape
    wp, wn = _ws(workspace)
    _check(load_library().domino_verify_sample(_ptr(draft_logits), _ptr(target_logits), _ptr(draft), B, K, V,
                                               temperature, seed, _ptr(tau_out), _ptr(token_out), wp, wn,
                                               _stream(stream)), "domino_verify_sample")


def domino_gate_table_bytes(w: DominoWeights) -> int:
    return int(load_library().domino_gate_table_bytes(w.ref))


def domino_build_gate_table(w: DominoWeights, table_out, *, workspace, stream=None) -> None:
    """G[t] = W_ih E[t] + b_ih for every token into a [V, 3H] float32 tensor."""
    wp, wn = _ws(workspace)
    _check(load_library().domino_build_gate_table(w.ref, _ptr(table_out), wp, wn, _stream(stream)),
           "domino_build_gate_table")


def domino_verify(draft, target, tau_out, stream=None) -> None:
    B, K = draft.shape
    _check(load_library().domino_verify(_ptr(draft), _ptr(target), B, K, _ptr(tau_out), _stream(stream)),
           "domino_verify")


def domino_draft_block_host(w: DominoWeights, hidden_host, anchor_host, *, mode=0, temperature=1.0, seed=0,
                            forced_host=None, target_host=None, draft_out_host, tau_out_host=None, workspace,
                            stream=None) -> None:
    """Host-buffer variant: host tensors in and out (pinned memory recommended)."""
    B, K = draft_out_host.shape
    wp, wn = _ws(workspace)
    _check(load_library().domino_draft_block_host(w.ref, _hptr(hidden_host), _hptr(anchor_host), B, K, mode,
                                                  temperature, seed, _hptr(forced_host), _hptr(target_host),
                                                  _hptr(draft_out_host), _hptr(tau_out_host), wp, wn,
                                                  _stream(stream)), "domino_draft_block_host")


def domino_poll(workspace, stream=None) -> int:
    """Synchronise and return the device-side status (0 = OK) without raising."""
    return int(load_library().domino_poll(_ptr(workspace), _stream(stream)))


def domino_set_wait_budget_ns(ns: int) -> None:
    load_library().domino_set_wait_budget_ns(int(ns))


def domino_selftest_wait_timeout(workspace, budget_ns: int, stream=None) -> int:
    wp, wn = _ws(workspace)
    return int(load_library().domino_selftest_wait_timeout(wp, wn, int(budget_ns), _stream(stream)))


def domino_status_str(status: int) -> str:
    return load_library().domino_status_str(int(status)).decode()
