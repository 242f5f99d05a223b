"""GPU parity of stochastic verification (speculative sampling) through the C ABI
against oracle/sampling.py, with the comparison protocol of
_harness.check_verify_sample (precision ties on the acceptance test are checked
for validity only; otherwise tau exact and the emitted token within 1e-3 of the
oracle's best draw).
"""
import numpy as np
import pytest
import torch

import draft_model_b200 as dm
import oracle
from _harness import aligned_workspace, check_verify_sample

pytestmark = pytest.mark.gpu
cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

def _gpu(dl, tl, draft, T, seed):
    B, K, V = dl.shape
    ws = aligned_workspace(dm.domino_verify_sample_workspace_bytes(B, K, V))
    tau = torch.zeros(B, dtype=torch.int32, device="cuda")
    tok = torch.zeros(B, dtype=torch.int32, device="cuda")
    dm.domino_verify_sample(torch.from_numpy(dl).cuda(), torch.from_numpy(tl).cuda(), torch.from_numpy(draft).cuda(),
                            temperature=T, seed=seed, tau_out=tau, token_out=tok, workspace=ws)
    return tau.cpu().numpy(), tok.cpu().numpy(), dm.domino_poll(ws)


def _check(dl, tl, draft, T, seed):
    tau, tok, status = _gpu(dl, tl, draft, T, seed)
    assert status == 0
    return check_verify_sample(dl, tl, draft, T, seed, tau, tok)


def _inputs(B, K, V, noise, seed):
    rng = np.random.default_rng(seed)
    dl = rng.normal(0.0, 2.0, size=(B, K, V)).astype(np.float32)
    tl = np.concatenate([dl + rng.normal(0.0, noise, size=(B, K, V)), rng.normal(0.0, 2.0, size=(B, 1, V))],
                        axis=1).astype(np.float32)
    # drafted tokens: Gumbel-max samples of the draft distributions (any valid tokens would do)
    g = -np.log(-np.log(rng.random(size=(B, K, V))))
    draft = np.argmax(dl / 1.0 + g, axis=2).astype(np.int32)
    return dl, tl, draft


@cuda
@pytest.mark.parametrize("B,K,V,noise,T,seed", [(6, 6, 5000, 0.5, 1.0, 1), (9, 16, 4100, 1.0, 1.0, 2),
                                                (3, 4, 777, 0.3, 0.7, 3), (2, 16, 151936, 0.5, 1.0, 4),
                                                (1, 1, 13, 2.0, 1.0, 5)])
def test_verify_sample_matches_oracle(B, K, V, noise, T, seed):
    dl, tl, draft = _inputs(B, K, V, noise, seed)
    stats = _check(dl, tl, draft, T, seed)
    assert stats["compared"] >= B - 1


@cuda
def test_verify_sample_mixes_accepts_and_rejects():
    dl, tl, draft = _inputs(64, 3, 3000, 0.5, 6)
    stats = _check(dl, tl, draft, 1.0, 6)
    assert stats["compared"] >= 60
    assert 5 <= stats["rejected"] <= stats["compared"] - 5


@cuda
def test_equal_distributions_accept_all():
    rng = np.random.default_rng(7)
    B, K, V = 4, 5, 2000
    dl = rng.normal(size=(B, K, V)).astype(np.float32)
    tl = np.concatenate([dl, rng.normal(size=(B, 1, V)).astype(np.float32)], axis=1)
    draft = rng.integers(0, V, size=(B, K)).astype(np.int32)
    tau, tok, status = _gpu(dl, tl, draft, 1.0, 9)
    assert status == 0
    np.testing.assert_array_equal(tau, K)
    _check(dl, tl, draft, 1.0, 9)


@cuda
def test_bad_draft_token_is_flagged():
    dl = np.zeros((1, 2, 100), dtype=np.float32)
    tl = np.zeros((1, 3, 100), dtype=np.float32)
    _, _, status = _gpu(dl, tl, np.array([[5, 100]], dtype=np.int32), 1.0, 0)
    assert status == 6   # DOMINO_ERR_BAD_TOKEN


@cuda
def test_empty_residual_draws_from_the_target():
    # draft and target rows equal except the drafted token, whose probability
    # (~e^-60) lies below fp32 and fp64 resolution: rejections (ratio e^-1) leave a
    # residual with no positive entry on either side, and the token comes from q
    rng = np.random.default_rng(12)
    B, K, V = 48, 2, 3000
    dl = rng.normal(0.0, 2.0, size=(B, K, V)).astype(np.float32)
    draft = rng.integers(0, V, size=(B, K)).astype(np.int32)
    dl[np.arange(B), 0, draft[:, 0]] = -60.0
    tl = np.concatenate([dl, rng.normal(0.0, 2.0, size=(B, 1, V)).astype(np.float32)], axis=1)
    tl[np.arange(B), 0, draft[:, 0]] = -61.0
    stats = _check(dl, tl, draft, 1.0, 13)
    assert stats["rejected"] >= 15
    ref = oracle.verify_sample(dl.astype(np.float64), tl.astype(np.float64), draft, 1.0, 13)
    tau, tok, _ = _gpu(dl, tl, draft, 1.0, 13)
    assert ((tok >= 0) & (tok < V)).all()
    for b in np.flatnonzero(ref.tau == 0):
        q = oracle.softmax_rows(tl[b, 0].astype(np.float64), 1.0)
        p = oracle.softmax_rows(dl[b, 0].astype(np.float64), 1.0)
        assert not (np.maximum(q - p, 0.0) > 0).any()
