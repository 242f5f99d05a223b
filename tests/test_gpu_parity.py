"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small cases span several tiles and ragged tails (vocabulary not a multiple of
the 128-row UMMA tile or the 32-row W2 chunk, d not a multiple of the 64-wide
k-block, batches that split into several request groups); the full-size
Qwen3-shaped configs run in the launch configuration bench.py times, with the
oracle on every request (B=1) or on a sample of requests (B=32, B=256).
"""
import numpy as np
import pytest
import torch

import draft_model_b200 as dm
import oracle
import synth
from _harness import TOL, check_against_oracle, device_weights, run_gpu, to_dev, workspace_for

pytestmark = pytest.mark.gpu

cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def small(**kw):
    base = dict(name="small", B=3, K=5, d=200, V=5000, H=64, r=32, E=136, dtype="bf16", tied=False, seed=1)
    base.update(kw)
    return synth.Config(**base)


_cache = {}


def setup(cfg):
    key = (cfg.d, cfg.V, cfg.H, cfg.r, cfg.E, cfg.dtype, cfg.tied, cfg.seed)
    if key not in _cache:
        w = synth.make_weights(cfg)
        _cache.clear()
        _cache[key] = (w, oracle.Model.from_storage(w), device_weights(w))
    return _cache[key]


# ---------------------------------------------------------------- stage 1

@cuda
@pytest.mark.parametrize("B,K,d,V", [(1, 16, 256, 1000), (3, 5, 200, 5000), (20, 16, 136, 777), (1, 4, 64, 128),
                                     (2, 16, 4096, 3000),
                                     # more 128-row tiles than SMs, ragged: stream-K splits tiles across CTAs
                                     (1, 16, 512, 30000), (1, 16, 1032, 20011), (3, 16, 256, 40000),
                                     # 256 block positions per tile: vocabulary tiles run in pairs
                                     # (odd tile count -> a half-empty last pair), with stream-K
                                     (16, 16, 512, 40000), (20, 16, 264, 20011)])
def test_lm_head_bf16_tcgen05(B, K, d, V):
    cfg = small(B=B, K=K, d=d, V=V)
    w, m, dw = setup(cfg)
    hidden = synth.make_hidden(cfg)
    ws = workspace_for(dw, B, K)
    out = torch.empty((B, K, V), dtype=torch.float32, device="cuda")
    dm.domino_lm_head(dw, to_dev(hidden, "bf16"), out, workspace=ws)
    assert dm.domino_poll(ws) == 0
    ref = oracle.lm_head(oracle.widen_f64(hidden, "bf16"), w.w_lm, "bf16")
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref).max()
    assert err < 2e-3, err


@cuda
@pytest.mark.parametrize("B,K,d,V", [(1, 4, 64, 512), (3, 5, 200, 5000)])
def test_lm_head_f32(B, K, d, V):
    cfg = small(B=B, K=K, d=d, V=V, dtype="f32")
    w, m, dw = setup(cfg)
    hidden = synth.make_hidden(cfg)
    ws = workspace_for(dw, B, K)
    out = torch.empty((B, K, V), dtype=torch.float32, device="cuda")
    dm.domino_lm_head(dw, to_dev(hidden, "f32"), out, workspace=ws)
    ref = oracle.lm_head(oracle.widen_f64(hidden, "f32"), w.w_lm, "f32")
    assert np.abs(out.cpu().numpy() - ref).max() < 1e-4


# ---------------------------------------------------------------- stage 3

@cuda
@pytest.mark.parametrize("K", [1, 5, 16, 32])
def test_verify_kernel_bit_exact(K):
    rng = np.random.default_rng(K)
    B = 1000
    draft = rng.integers(0, 4, size=(B, K)).astype(np.int32)
    target = np.where(rng.random((B, K)) < 0.9, draft, rng.integers(0, 4, size=(B, K))).astype(np.int32)
    d, t = torch.from_numpy(draft).cuda(), torch.from_numpy(target).cuda()
    tau = torch.empty(B, dtype=torch.int32, device="cuda")
    dm.domino_verify(d, t, tau)
    np.testing.assert_array_equal(tau.cpu().numpy(), oracle.verify(draft, target))


# ---------------------------------------------------------------- whole block, small shapes

@cuda
def test_tiny_f32_config():
    cfg = synth.CONFIGS["tiny_f32"]
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    free = oracle.draft_block(m, hidden, anchor)
    target = synth.make_targets(cfg, free.tokens)
    gpu = run_gpu(dw, cfg, hidden, anchor, target=target)
    assert gpu["status"] == 0
    np.testing.assert_array_equal(gpu["tokens"], free.tokens)
    assert np.abs(gpu["logits"] - free.logits).max() <= TOL["f32"]
    assert gpu["tau"][0] == 3
    check_against_oracle(m, cfg, hidden, anchor, gpu, target=target)


@cuda
@pytest.mark.parametrize("cfg", [
    small(B=1, K=16, mode="gumbel", temperature=1.0, seed=4),
    small(B=9, K=7, seed=5),
    small(B=5, K=6, dtype="f32", seed=9),
], ids=["persistent_gumbel_b1", "tensor_core_b9", "f32_b5"])
def test_repeated_blocks_are_bit_identical(cfg):
    """No float atomics and fixed reduction orders: two runs of the same block give
    the same picks and bit-identical final logits (a barrier race would not)."""
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    first = run_gpu(dw, cfg, hidden, anchor)
    second = run_gpu(dw, cfg, hidden, anchor)
    assert first["status"] == 0 and second["status"] == 0
    np.testing.assert_array_equal(first["tokens"], second["tokens"])
    np.testing.assert_array_equal(first["logits"].view(np.uint32), second["logits"].view(np.uint32))


@cuda
@pytest.mark.parametrize("cfg", [
    small(),
    small(B=1, K=16, mode="gumbel", temperature=1.0, seed=4),
    small(B=9, K=7, mode="gumbel", temperature=0.7, seed=5),
    small(B=2, K=16, d=136, E=136, tied=True, seed=6),
    small(B=17, K=3, seed=7),
    small(B=4, K=32, V=4100, H=96, r=256, seed=8),
    small(B=5, K=6, dtype="f32", V=3001 // 8 * 8 + 5, seed=9),
], ids=["ragged", "gumbel_b1", "gumbel_b9", "tied", "b17_groups", "k32_r256", "f32_ragged"])
def test_block_small(cfg):
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    draft0 = run_gpu(dw, cfg, hidden, anchor, want_logits=False)["tokens"]
    target = synth.make_targets(cfg.replace(target_p=0.3), draft0)
    gpu = run_gpu(dw, cfg, hidden, anchor, target=target)
    assert gpu["status"] == 0
    np.testing.assert_array_equal(gpu["tokens"], draft0)   # deterministic across calls
    _, stats = check_against_oracle(m, cfg, hidden, anchor, gpu, target=target)
    assert stats["agree"] > 0.5


@cuda
def test_teacher_forced_block():
    cfg = small(B=3, K=8, seed=11)
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    rng = np.random.default_rng(3)
    forced = rng.integers(0, cfg.V, size=(cfg.B, cfg.K)).astype(np.int32)
    gpu = run_gpu(dw, cfg, hidden, anchor, forced=forced)
    assert gpu["status"] == 0
    check_against_oracle(m, cfg, hidden, anchor, gpu, forced=forced)
    # forcing the free-running picks reproduces them
    free = run_gpu(dw, cfg, hidden, anchor)
    again = run_gpu(dw, cfg, hidden, anchor, forced=free["tokens"])
    np.testing.assert_array_equal(again["tokens"], free["tokens"])
    np.testing.assert_array_equal(again["logits"], free["logits"])


@cuda
def test_zero_correction_gives_base_argmax():
    cfg = small(B=2, K=6, seed=12)
    w = synth.make_weights(cfg)
    w.w2 = np.zeros_like(w.w2)
    dw = device_weights(w)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    gpu = run_gpu(dw, cfg, hidden, anchor)
    base = oracle.lm_head(oracle.widen_f64(hidden, "bf16"), w.w_lm, "bf16")
    srt = np.sort(base, axis=2)
    clear = (srt[:, :, -1] - srt[:, :, -2]) > 1e-3
    np.testing.assert_array_equal(gpu["tokens"][clear], np.argmax(base, axis=2)[clear])


# ---------------------------------------------------------------- device-side error reporting

@cuda
def test_bad_token_is_clamped_and_flagged():
    cfg = small(B=2, K=4, seed=13)
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    bad = anchor.copy()
    bad[1] = cfg.V + 5
    gpu = run_gpu(dw, cfg, hidden, bad)
    assert gpu["status"] == 6   # DOMINO_ERR_BAD_TOKEN
    clamped = bad.copy()
    clamped[1] = cfg.V - 1
    ok = run_gpu(dw, cfg, hidden, clamped)
    assert ok["status"] == 0
    np.testing.assert_array_equal(gpu["tokens"], ok["tokens"])


@cuda
def test_bounded_wait_times_out_and_gpu_stays_usable():
    cfg = small(B=1, K=4, seed=14)
    w, m, dw = setup(cfg)
    ws = workspace_for(dw, 1, 4)
    assert dm.domino_selftest_wait_timeout(ws, 2_000_000) == 5   # DOMINO_ERR_TIMEOUT, 2 ms budget
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    gpu = run_gpu(dw, cfg, hidden, anchor, ws=ws)
    assert gpu["status"] == 0
    check_against_oracle(m, cfg, hidden, anchor, gpu)


# ---------------------------------------------------------------- full-size Qwen3-shaped configs

@cuda
@pytest.mark.parametrize("name", ["qwen3_8b_b1", "qwen3_4b_b1"])
def test_full_size_b1(name):
    cfg = synth.CONFIGS[name]
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    draft0 = run_gpu(dw, cfg, hidden, anchor, want_logits=False)["tokens"]
    target = synth.make_targets(cfg, draft0)
    gpu = run_gpu(dw, cfg, hidden, anchor, target=target)
    assert gpu["status"] == 0
    np.testing.assert_array_equal(gpu["tokens"], draft0)
    check_against_oracle(m, cfg, hidden, anchor, gpu, target=target)


@cuda
def test_full_size_b32_gumbel_sampled():
    cfg = synth.CONFIGS["qwen3_8b_b32_gumbel"]
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    draft0 = run_gpu(dw, cfg, hidden, anchor, want_logits=False)["tokens"]
    target = synth.make_targets(cfg, draft0)
    gpu = run_gpu(dw, cfg, hidden, anchor, target=target)
    assert gpu["status"] == 0
    check_against_oracle(m, cfg, hidden, anchor, gpu, target=target, rows=[0, 9, 31])


@cuda
@pytest.mark.parametrize("B", [2, 8])
def test_full_size_sweep_small_batches(B):
    cfg = synth.sweep_config(B)
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    gpu = run_gpu(dw, cfg, hidden, anchor, want_logits=False)
    assert gpu["status"] == 0
    check_against_oracle(m, cfg, hidden, anchor, gpu, rows=[0, B - 1])


@cuda
def test_full_size_sweep_b256_sampled():
    cfg = synth.sweep_config(256)
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    gpu = run_gpu(dw, cfg, hidden, anchor, want_logits=False)
    assert gpu["status"] == 0
    check_against_oracle(m, cfg, hidden, anchor, gpu, rows=[0, 100, 255])


# ---------------------------------------------------------------- degenerate cases

@cuda
@pytest.mark.parametrize("cfg", [small(B=1, K=1, seed=21), small(B=6, K=1, seed=22),
                                 small(B=5, K=1, mode="gumbel", temperature=1.0, seed=23)],
                         ids=["persistent", "tensor_core", "gumbel_tc"])
def test_single_position_block(cfg):
    w, m, dw = setup(cfg)
    hidden, anchor = synth.make_hidden(cfg), synth.make_anchor(cfg)
    target = np.zeros((cfg.B, 1), dtype=np.int32)
    gpu = run_gpu(dw, cfg, hidden, anchor, target=target)
    assert gpu["status"] == 0
    check_against_oracle(m, cfg, hidden, anchor, gpu, target=target)


@cuda
@pytest.mark.parametrize("B", [2, 6], ids=["persistent", "tensor_core"])
def test_exact_ties_pick_the_lowest_index(B):
    # W2 = 0 (L_i = L_base) and a dominant W_lm row copied to several tokens: their
    # base logits are bit-identical maxima, and the pick must be the lowest of them
    cfg = small(B=B, K=4, seed=24)
    w = synth.make_weights(cfg)
    w.w2 = np.zeros_like(w.w2)
    hidden = synth.make_hidden(cfg)
    h0 = oracle.widen_f64(hidden, "bf16")[0, 0]
    row = synth.f32_to_bf16_bits((np.sign(h0) * 0.5).astype(np.float32))
    tied = [4097, 137, 2500, 4999]
    w.w_lm = w.w_lm.copy()
    for t in tied:
        w.w_lm[t] = row
    dw = device_weights(w)
    hidden[:, :, :] = hidden[0, 0]          # every position sees the same hidden state
    anchor = synth.make_anchor(cfg)
    gpu = run_gpu(dw, cfg, hidden, anchor)
    assert gpu["status"] == 0
    np.testing.assert_array_equal(gpu["tokens"], min(tied))
