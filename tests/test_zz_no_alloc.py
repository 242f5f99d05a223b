"""The allocation-free stage-2 entry point, through the C ABI, against the
workspace entry point on the same inputs, on two calls in a row.

Callers that cannot hand the library device memory (engines that own every
device allocation, plugins inside them, deployments that must not allocate
after start-up) use domino_correct_loop_noalloc, whose scratch is a fixed
array inside the library.  This file is collected last so that a run stopping
at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import draft_model_b200 as dm
import synth
from _harness import TOL, device_weights, to_dev, workspace_for

pytestmark = pytest.mark.gpu


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("mode", ["greedy", "gumbel"])
def test_noalloc_matches_workspace_entry_point(mode):
    cfg = synth.Config("noalloc", B=5, K=9, d=200, V=5000, H=64, r=32, E=136, dtype="bf16", tied=False,
                       mode=mode, temperature=0.8, seed=21)
    w = synth.make_weights(cfg)
    dw = device_weights(w)
    hidden_np, anchor_np = synth.make_hidden(cfg), synth.make_anchor(cfg)
    hidden, anchor = to_dev(hidden_np, "bf16"), torch.from_numpy(anchor_np).cuda()
    B, K, V = cfg.B, cfg.K, cfg.V
    target = torch.from_numpy(np.random.default_rng(1).integers(0, V, (B, K)).astype(np.int32)).cuda()
    ws = workspace_for(dw, B, K)
    base = torch.empty((B, K, V), dtype=torch.float32, device="cuda")
    dm.domino_lm_head(dw, hidden, base, workspace=ws)
    m = 0 if mode == "greedy" else 1

    def run(noalloc):
        draft = torch.full((B, K), -1, dtype=torch.int32, device="cuda")
        logits = torch.full((B, K, V), float("nan"), dtype=torch.float32, device="cuda")
        tau = torch.full((B,), -1, dtype=torch.int32, device="cuda")
        kw = dict(mode=m, temperature=cfg.temperature, seed=cfg.seed, target=target, draft_out=draft,
                  logits_out=logits, tau_out=tau)
        if noalloc:
            dm.domino_correct_loop_noalloc(dw, hidden, base, anchor, **kw)
        else:
            dm.domino_correct_loop(dw, hidden, base, anchor, workspace=ws, **kw)
            assert dm.domino_poll(ws) == 0
        torch.cuda.synchronize()
        return draft.cpu().numpy(), logits.cpu().numpy(), tau.cpu().numpy()

    ref = run(False)
    for _ in range(2):                  # two calls in a row share the library's scratch
        got = run(True)
        np.testing.assert_array_equal(got[0], ref[0])
        assert np.abs(got[1].astype(np.float64) - ref[1]).max() <= TOL["bf16"]
        np.testing.assert_array_equal(got[2], ref[2])


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_noalloc_rejects_sizes_beyond_its_scratch():
    cfg = synth.Config("noalloc_big", B=9, K=4, d=64, V=512, H=32, r=16, E=64, dtype="bf16", tied=False)
    dw = device_weights(synth.make_weights(cfg))
    hidden = to_dev(synth.make_hidden(cfg), "bf16")
    anchor = torch.from_numpy(synth.make_anchor(cfg)).cuda()
    base = torch.zeros((cfg.B, cfg.K, cfg.V), dtype=torch.float32, device="cuda")
    draft = torch.empty((cfg.B, cfg.K), dtype=torch.int32, device="cuda")
    with pytest.raises(dm.DominoError) as err:
        dm.domino_correct_loop_noalloc(dw, hidden, base, anchor, draft_out=draft)
    assert err.value.status == 2    # DOMINO_ERR_UNSUPPORTED: B > 8
