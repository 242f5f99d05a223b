"""C-ABI checks that need no GPU: the library builds and loads, it exports every
entry point include/domino.h declares, and host-side validation rejects bad
arguments synchronously (before any CUDA call)."""
import ctypes
import os
import re
import shutil
import subprocess

import pytest

import draft_model_b200 as dm
from draft_model_b200 import build as dbuild
from draft_model_b200._binding import _CWeights

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "domino.h")


@pytest.fixture(scope="module")
def lib():
    dbuild.build()
    return dm.load_library()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"DOMINO_API\s+[\w\s\*]+?\b(domino_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("domino_draft_block", "domino_lm_head", "domino_correct_loop", "domino_verify", "domino_poll",
                 "domino_status_str", "domino_workspace_bytes"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(dm.library_path())
    for name in declared_functions():
        assert hasattr(raw, name), f"{name} declared in domino.h but not exported"


def test_status_strings(lib):
    for code, name in dm.STATUS.items():
        assert dm.domino_status_str(code) == name
    assert dm.domino_status_str(99) == "DOMINO_ERR_UNKNOWN"


def _cw(V=151936, d=4096, E=4096, H=1024, r=256, dtype=0, ptr=0x10000):
    p = ctypes.c_void_p(ptr)
    return _CWeights(V, d, E, H, r, dtype, p, p, p, p, None, None, p, p)


def test_workspace_bytes(lib):
    w = _cw()
    n = lib.domino_workspace_bytes(ctypes.byref(w), 1, 16)
    # control block + base logits (B*K*V fp32) + GRU state + u + argmax keys, 256-aligned pieces
    assert n >= 16 * 151936 * 4 + 256
    assert n % 256 == 0
    assert lib.domino_workspace_bytes(ctypes.byref(w), 2, 16) > n
    assert lib.domino_workspace_bytes_host(ctypes.byref(w), 1, 16) > n
    assert lib.domino_workspace_bytes(ctypes.byref(w), 0, 16) == 0
    assert lib.domino_workspace_bytes(ctypes.byref(w), 1, 33) == 0
    bad = _cw(d=4095)
    assert lib.domino_workspace_bytes(ctypes.byref(bad), 1, 16) == 0


def test_launches_per_block(lib):
    w = _cw()
    # persistent loop: LM head + one launch per group of up to 8 requests
    assert lib.domino_launches_per_block(ctypes.byref(w), 1, 16) == 2
    assert lib.domino_launches_per_block(ctypes.byref(w), 2, 16) == 2
    # tensor-core loop: LM head + anchor gather + per step 5 kernels and one W2 GEMM per 128 requests
    assert lib.domino_launches_per_block(ctypes.byref(w), 8, 16) == 2 + 16 * 6
    assert lib.domino_launches_per_block(ctypes.byref(w), 256, 16) == 2 + 16 * 7
    # fp32 weights always take the persistent loop
    wf = _cw(dtype=1)
    assert lib.domino_launches_per_block(ctypes.byref(wf), 17, 4) == 1 + 3
    assert lib.domino_launches_per_block(ctypes.byref(w), 0, 16) == -1
    assert lib.domino_launches_per_block(ctypes.byref(w), 1, 33) == -1


def _block(lib, w, *, B=1, K=16, mode=0, T=1.0, hidden=0x20000, anchor=0x30000, draft=0x40000, target=None,
           tau=None, ws=0x100000, wsn=1 << 40):
    return lib.domino_draft_block(ctypes.byref(w), hidden, anchor, B, K, mode, T, 0, None, target, draft, None, tau,
                                  ws, wsn, None)


def test_validation_is_synchronous_and_host_side(lib):
    w = _cw()
    INVALID, UNSUP, WS = 1, 2, 7
    assert _block(lib, w, B=0) == INVALID
    assert _block(lib, w, K=0) == INVALID
    assert _block(lib, w, K=33) == INVALID
    assert _block(lib, w, mode=2) == INVALID
    assert _block(lib, w, mode=1, T=0.0) == INVALID
    assert _block(lib, w, mode=1, T=float("nan")) == INVALID
    assert _block(lib, w, hidden=None) == INVALID
    assert _block(lib, w, hidden=0x20001) == INVALID          # misaligned
    assert _block(lib, w, draft=None) == INVALID
    assert _block(lib, w, target=0x50000, tau=None) == INVALID  # tau needed with a target
    assert _block(lib, _cw(r=264)) == UNSUP                     # rank above the bf16 limit
    assert _block(lib, _cw(dtype=1, r=136)) == UNSUP            # rank above the f32 limit
    assert _block(lib, _cw(dtype=3)) == INVALID
    assert _block(lib, w, ws=None) == WS
    assert _block(lib, w, ws=0x100010) == WS                    # workspace not 256-aligned
    assert _block(lib, w, wsn=1024) == WS                       # workspace too small
    nullw = _cw(ptr=0)
    assert _block(lib, nullw) == INVALID


def test_verify_and_init_validation(lib):
    assert lib.domino_verify(0x1000, 0x2000, 1, 33, 0x3000, None) == 1
    assert lib.domino_verify(None, 0x2000, 1, 4, 0x3000, None) == 1
    assert lib.domino_verify(0x1000, 0x2000, 0, 4, 0x3000, None) == 1
    assert lib.domino_workspace_init(0x1001, 4096, None) == 7
    assert lib.domino_workspace_init(0x1000, 16, None) == 7


def test_product_path_fails_loudly_without_library(tmp_path, monkeypatch):
    from draft_model_b200 import _binding
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _binding.load_library()


def test_loss_validation_is_host_side(lib):
    INVALID = 1
    p = 0x100000
    n = lib.domino_curriculum_loss_workspace_bytes(2, 4, 1000)
    assert n > 0 and lib.domino_curriculum_loss_workspace_bytes(0, 4, 1000) == 0
    call = lambda lam, gamma, B=2, K=4: lib.domino_curriculum_loss(p, p, p, B, K, 1000, lam, gamma, None, p, p, n, None)
    assert call(-0.1, 1.0) == INVALID
    assert call(1.5, 1.0) == INVALID
    assert call(0.5, 0.0) == INVALID
    assert call(0.5, float("inf")) == INVALID
    assert call(0.5, 1.0, K=33) == INVALID
    assert lib.domino_curriculum_loss(p, p, None, 2, 4, 1000, 0.5, 1.0, None, p, p, n, None) == INVALID
    w = _cw()
    assert lib.domino_draft_loss_workspace_bytes(ctypes.byref(w), 1, 16) > lib.domino_workspace_bytes(ctypes.byref(w), 1, 16)
    assert lib.domino_draft_loss(ctypes.byref(w), p, p, None, 1, 16, 0.5, 1.0, None, p, p, 1 << 40, None) == INVALID


def test_verify_sample_validation_is_host_side(lib):
    INVALID = 1
    p = 0x100000
    n = lib.domino_verify_sample_workspace_bytes(2, 4, 1000)
    assert n > 0 and lib.domino_verify_sample_workspace_bytes(2, 33, 1000) == 0
    call = lambda T, B=2, K=4, draft=p: lib.domino_verify_sample(p, p, draft, B, K, 1000, T, 0, p, p, p, n, None)
    assert call(0.0) == INVALID
    assert call(float("nan")) == INVALID
    assert call(1.0, K=0) == INVALID
    assert call(1.0, B=2000, K=32) == INVALID
    assert call(1.0, draft=None) == INVALID


def test_gate_table_abi(lib):
    w = _cw(V=1000, H=64)
    assert lib.domino_gate_table_bytes(ctypes.byref(w)) == 1000 * 3 * 64 * 4
    assert lib.domino_gate_table_bytes(ctypes.byref(_cw(d=4095))) == 0
    # NULL or misaligned table: rejected before any CUDA call
    assert lib.domino_build_gate_table(ctypes.byref(w), None, 0x100000, 1024, None) == 1
    assert lib.domino_build_gate_table(ctypes.byref(w), 0x100004, 0x100000, 1024, None) == 1
    # a table changes the batched loop's launch count by one (no gate GEMM at the first position)
    n0 = lib.domino_launches_per_block(ctypes.byref(w), 8, 16)
    w.gate_table = 0x200000
    assert lib.domino_launches_per_block(ctypes.byref(w), 8, 16) == n0 - 1


def test_stage_entry_points_validate_on_the_host(lib):
    INVALID, UNSUP, WS = 1, 2, 7
    w = _cw()
    p, ws, big = 0x100000, 0x200000, 1 << 40
    # stage 1
    assert lib.domino_lm_head(ctypes.byref(w), p, 0, 16, p, ws, big, None) == INVALID
    assert lib.domino_lm_head(ctypes.byref(w), None, 1, 16, p, ws, big, None) == INVALID
    assert lib.domino_lm_head(ctypes.byref(w), p, 1, 16, 0x100008, ws, big, None) == INVALID   # misaligned out
    assert lib.domino_lm_head(ctypes.byref(w), p, 1, 16, p, None, big, None) == WS
    # stage 2 with given base logits
    loop = lambda B=1, K=16, base=p, ws_=ws: lib.domino_correct_loop(ctypes.byref(w), p, base, p, B, K, 0, 1.0, 0,
                                                                     None, None, p, None, None, ws_, big, None)
    assert loop(K=33) == INVALID
    assert loop(base=None) == INVALID
    assert loop(ws_=0x200010) == WS
    # host-buffer entry point
    assert lib.domino_draft_block_host(ctypes.byref(w), None, p, 1, 16, 0, 1.0, 0, None, None, p, None, ws, big,
                                       None) == INVALID
    assert lib.domino_draft_block_host(ctypes.byref(w), p, p, 1, 16, 0, 1.0, 0, None, p, p, None, ws, big,
                                       None) == INVALID                     # target without tau
    # allocation-free loop: its fixed scratch limits are checked before any device work
    noalloc = lambda B=1, K=16, ww=w: lib.domino_correct_loop_noalloc(ctypes.byref(ww), p, p, p, B, K, 0, 1.0, 0,
                                                                      None, None, p, None, None, None)
    assert noalloc(B=9) == UNSUP
    assert noalloc(ww=_cw(H=8192)) == UNSUP
    assert noalloc(K=0) == INVALID


def test_binding_rejects_host_tensors_for_device_arguments():
    """A CPU tensor where the C ABI takes device memory raises in the binding,
    before any call into the library (a host pointer must never reach a kernel)."""
    import torch
    from draft_model_b200 import _binding
    d = torch.zeros((2, 4), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dm.domino_verify(d, d, torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        dm.domino_workspace_init(torch.zeros(1024, dtype=torch.uint8))
    # host-buffer arguments take CPU tensors, raw addresses pass through unchanged
    assert _binding._hptr(d) == d.data_ptr()
    assert _binding._ptr(None) is None and _binding._ptr(4096) == 4096
    with pytest.raises(ValueError, match="contiguous"):
        _binding._hptr(torch.zeros((4, 4), dtype=torch.int32).t())


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "domino.h"
int main(void) {
  domino_weights w;
  memset(&w, 0, sizeof w);
  if (strcmp(domino_status_str(DOMINO_ERR_INVALID_ARG), "DOMINO_ERR_INVALID_ARG") != 0) return 1;
  if (domino_launches_per_block(&w, 1, 16) != -1) return 2;         /* no weights: rejected */
  if (domino_workspace_bytes(&w, 1, 16) != 0) return 3;
  if (domino_verify(NULL, NULL, 1, 16, NULL, NULL) != DOMINO_ERR_INVALID_ARG) return 4;
  puts("ok");
  return 0;
}
"""


@pytest.mark.skipif(not shutil.which("gcc"), reason="needs gcc")
def test_plain_c99_client_compiles_links_and_calls_the_library(lib, tmp_path):
    """The boundary is a C ABI: a strict C99 program includes the header, links
    libdomino.so and calls host-side entry points (no GPU needed for these)."""
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    libdir = os.path.dirname(dm.library_path())
    exe = tmp_path / "client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.dirname(HEADER),
                    str(src), "-L", libdir, "-ldomino", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)
