"""Failure detection without a GPU fault: the bounded device waits.

A tiny wait limit makes a kernel's first mbarrier wait run out, as a flag
that is never set would (below 64 the decode kernel's warps first wait on a
barrier that nothing completes, so its timeout path runs on every call). The
kernel must record MOBI_ERR_TIMEOUT, drain its copies (and, in the prefill
kernel, its MMAs and tensor memory) and return, leaving the context usable:
the next call with the default limit must be correct again. Covered for the
prefill kernel and the decode kernel (both fragment classes).
"""
import numpy as np
import pytest
import torch

from parity import check_gemm
from token_adaptive_mixed_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_timeout_is_reported_and_context_survives(oracle):
    import token_adaptive_mixed_b200 as mobi
    N, K, T = 256, 512, 300
    L = wl.layer("to", N, K, T, seed=9)
    codes, sz, _ = oracle.pack(L.W, S=3)
    k = np.random.default_rng(0).integers(1, 4, T).astype(np.int32)
    perm = np.argsort(k, kind="stable").astype(np.int32)
    off = np.concatenate([[0], np.cumsum(np.bincount(k, minlength=4)[1:])]).astype(np.int32)
    args = [L.X.to(DEV), torch.from_numpy(k).to(DEV), torch.from_numpy(perm).to(DEV), torch.from_numpy(off).to(DEV),
            torch.from_numpy(codes.view(np.int32)).to(DEV), torch.from_numpy(sz.view(np.int32)).to(DEV), N]
    mobi.mobi_sync_check()
    mobi.mobi_debug_set_wait_limit(1)
    try:
        mobi.mobi_gemm_path(*args, path=2)
        with pytest.raises(mobi.MobiError) as ei:
            mobi.mobi_sync_check()
        assert ei.value.status == 6  # MOBI_ERR_TIMEOUT
    finally:
        mobi.mobi_debug_set_wait_limit(0)
    mobi.mobi_sync_check()  # error word cleared, context healthy
    Y = mobi.mobi_gemm_path(*args, path=2)
    mobi.mobi_sync_check()
    check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k, codes, sz, N), "after timeout")


@pytest.mark.parametrize("T", [4, 16])
def test_decode_timeout_is_reported_and_context_survives(oracle, T):
    import token_adaptive_mixed_b200 as mobi
    # A large layer, so every CTA has work when the limit runs out; four K
    # chunks, so the chunk-reduction kernel runs behind the decode kernel.
    N, K = 28672, 4096
    L = wl.layer("tod", N, K, T, seed=19 + T)
    codes, sz, _ = oracle.pack(L.W, S=3)
    k = np.random.default_rng(T).integers(1, 4, T).astype(np.int32)
    perm = np.argsort(k, kind="stable").astype(np.int32)
    off = np.concatenate([[0], np.cumsum(np.bincount(k, minlength=4)[1:])]).astype(np.int32)
    args = [L.X.to(DEV), torch.from_numpy(k).to(DEV), torch.from_numpy(perm).to(DEV), torch.from_numpy(off).to(DEV),
            torch.from_numpy(codes.view(np.int32)).to(DEV), torch.from_numpy(sz.view(np.int32)).to(DEV), N]
    mobi.mobi_sync_check()
    mobi.mobi_debug_set_wait_limit(1)
    try:
        mobi.mobi_gemm_path(*args, path=1)
        with pytest.raises(mobi.MobiError) as ei:
            mobi.mobi_sync_check()
        assert ei.value.status == 6  # MOBI_ERR_TIMEOUT
        assert "wait site" in mobi.mobi_last_error()
    finally:
        mobi.mobi_debug_set_wait_limit(0)
    mobi.mobi_sync_check()  # error word cleared, context healthy
    Y = mobi.mobi_gemm_path(*args, path=1)
    mobi.mobi_sync_check()
    check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k, codes, sz, N), f"decode after timeout, T={T}")
