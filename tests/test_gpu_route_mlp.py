"""GPU parity of mobi_route_mlp (threshold routing with a two-layer MLP scorer)
against the CPU oracle.

Bar: k_t equals the oracle's count wherever every residual slice's fp64 score
lies outside the kernel's derived fp32 error band around the threshold
(parity.mlp_score_bound); where a slice is inside the band, k_t lies between
the surely-active and the possibly-active counts. perm and offsets are exact
(the oracle's stable bucketing of the GPU's k_t). At the full T=2048 size the
band is computed on a sample of 256 tokens; the other tokens may differ from
the oracle only where its margin is below ten times the largest sampled band.
"""
import math

import numpy as np
import pytest
import torch

from parity import check_route_mlp, mlp_score_bound
from token_adaptive_mixed_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def mobi():
    import token_adaptive_mixed_b200 as m
    from token_adaptive_mixed_b200 import build
    build.build()
    assert torch.cuda.is_available()
    m.lib()
    return m


def thr_of(tau, delta):
    return tau * math.log(delta / (1.0 - delta))


def run(mobi, R, tau, delta, null_bias=False):
    W1 = torch.from_numpy(R.W1).to(DEV)
    W2 = torch.from_numpy(np.ascontiguousarray(R.W2)).to(DEV)
    b1 = None if null_bias else torch.from_numpy(R.b1).to(DEV)
    b2 = None if null_bias else torch.from_numpy(R.b2).to(DEV)
    k_t, perm, off = mobi.mobi_route_mlp(R.X.to(DEV), W1, b1, W2, b2, tau, delta)
    mobi.mobi_sync_check()
    return k_t.cpu().numpy(), perm.cpu().numpy(), off.cpu().numpy()


def check(mobi, oracle, R, tau, delta, tag, null_bias=False):
    b1 = np.zeros_like(R.b1) if null_bias else R.b1
    b2 = np.zeros_like(R.b2) if null_bias else R.b2
    k_gpu, perm, off = run(mobi, R, tau, delta, null_bias)
    k_ref, _, scores = oracle.route_mlp(R.X, R.W1, b1, R.W2, b2, tau, delta)
    thr = thr_of(tau, delta)
    bound = mlp_score_bound(R.X.float().numpy(), R.W1, b1, R.W2, b2, thr)
    check_route_mlp(k_gpu, scores, bound, thr, tag)
    perm_ref, off_ref = oracle.bucket(k_gpu, R.S)
    assert np.array_equal(perm, perm_ref), tag
    assert np.array_equal(off, off_ref), tag
    return k_gpu, k_ref


@pytest.mark.parametrize("T,K,H", [(1, 128, 1), (5, 1024, 7), (16, 4096, 128), (37, 512, 100), (300, 1024, 32),
                                   (129, 256, 33), (700, 1024, 128), (513, 512, 200)])
def test_route_mlp_parity(mobi, oracle, T, K, H):
    R = wl.mlp_router("mlp", T, K, H, seed=900 + T + H)
    k_gpu, k_ref = check(mobi, oracle, R, 1.0, 0.5, f"mlp T={T} K={K} H={H}")
    assert k_gpu.min() >= 1 and k_gpu.max() <= 3


@pytest.mark.parametrize("tau,delta", [(0.5, 0.3), (2.0, 0.8), (1.0, 0.999), (0.25, 1e-3)])
def test_route_mlp_tau_delta(mobi, oracle, tau, delta):
    R = wl.mlp_router("mlp_td", 200, 1024, 64, seed=950)
    check(mobi, oracle, R, tau, delta, f"mlp tau={tau} delta={delta}")


@pytest.mark.parametrize("S", [1, 2, 3])
def test_route_mlp_slices(mobi, oracle, S):
    R = wl.mlp_router("mlp_s", 64, 512, 48, seed=960 + S, S=S)
    if S == 1:  # no residual slice: every token keeps the base slice only
        X = R.X.to(DEV)
        W1 = torch.from_numpy(R.W1).to(DEV)
        W2 = torch.empty((48, 0), dtype=torch.float32, device=DEV)
        k_t, perm, off = mobi.mobi_route_mlp(X, W1, None, W2, None, 1.0, 0.5)
        mobi.mobi_sync_check()
        assert np.all(k_t.cpu().numpy() == 1)
        assert np.array_equal(perm.cpu().numpy(), np.arange(64))
        assert np.array_equal(off.cpu().numpy(), [0, 64])
        return
    check(mobi, oracle, R, 1.0, 0.5, f"mlp S={S}")


def test_route_mlp_null_biases(mobi, oracle):
    R = wl.mlp_router("mlp_nb", 48, 1024, 64, seed=970)
    check(mobi, oracle, R, 1.0, 0.5, "mlp null biases", null_bias=True)


def test_route_mlp_skewed_offsets(mobi, oracle):
    """Positive score offsets move tokens to more slices: the same tokens with
    offsets (1.5, 0.5) never take fewer slices than with none, and few keep one."""
    kw = dict(token_scaled_frac=0.02, token_scale=8.0)
    R = wl.mlp_router("mlp_sk", 500, 2048, 128, seed=980, b2=(1.5, 0.5), **kw)
    R0 = wl.mlp_router("mlp_sk0", 500, 2048, 128, seed=980, **kw)
    k_gpu, _ = check(mobi, oracle, R, 1.0, 0.5, "mlp skewed")
    k0, _ = check(mobi, oracle, R0, 1.0, 0.5, "mlp unskewed")
    assert np.all(k_gpu >= k0)
    cnt = np.bincount(k_gpu, minlength=4)
    assert cnt[1] < cnt[3] < cnt[2]


def test_route_mlp_empty(mobi):
    X = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    W1 = torch.zeros((256, 16), dtype=torch.float32, device=DEV)
    W2 = torch.zeros((16, 2), dtype=torch.float32, device=DEV)
    k_t, perm, off = mobi.mobi_route_mlp(X, W1, None, W2, None, 1.0, 0.5)
    mobi.mobi_sync_check()
    assert k_t.numel() == 0 and perm.numel() == 0
    assert np.array_equal(off.cpu().numpy(), [0, 0, 0, 0])


def test_route_mlp_monotone_in_delta_and_deterministic(mobi):
    """The same scores meet a higher threshold: k_t never grows with delta, and
    a repeated call gives the same k_t bit for bit."""
    R = wl.mlp_router("mlp_mono", 333, 1024, 128, seed=990)
    prev = None
    for delta in (0.05, 0.2, 0.5, 0.8, 0.95):
        k, _, _ = run(mobi, R, 1.0, delta)
        k2, _, _ = run(mobi, R, 1.0, delta)
        assert np.array_equal(k, k2)
        if prev is not None:
            assert np.all(k <= prev)
        prev = k
    assert prev.min() >= 1


@pytest.mark.slow
def test_route_mlp_full_size(mobi, oracle):
    """T=2048, K=4096, H=128, S=3: band on 256 sampled tokens (the last token
    among them), a margin-based property on the rest."""
    R = wl.mlp_route_prefill()
    tau, delta = 1.0, 0.5
    thr = thr_of(tau, delta)
    k_gpu, perm, off = run(mobi, R, tau, delta)
    k_ref, margin, scores = oracle.route_mlp(R.X, R.W1, R.b1, R.W2, R.b2, tau, delta)
    rows = np.sort(np.append(np.random.default_rng(5).choice(R.T - 1, 255, replace=False), R.T - 1))
    bound = mlp_score_bound(R.X[torch.from_numpy(rows)].float().numpy(), R.W1, R.b1, R.W2, R.b2, thr)
    check_route_mlp(k_gpu[rows], scores[rows], bound, thr, "mlp full size")
    diff = np.nonzero(k_gpu != k_ref)[0]
    assert np.all(margin[diff] < 10 * bound.max()), diff[:10]
    perm_ref, off_ref = oracle.bucket(k_gpu, 3)
    assert np.array_equal(perm, perm_ref) and np.array_equal(off, off_ref)
