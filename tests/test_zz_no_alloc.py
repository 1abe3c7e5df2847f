"""The decode GEMM entry point that allocates nothing (mobi_gemm_decode_noalloc).

It serves callers that cannot hand the library a workspace (for example an
engine plugin that must not allocate while it enqueues work, or a host whose
device memory belongs to another runtime): its scratch is a fixed 8 MiB array
of static device memory. This test calls it through the C ABI twice in a row
(the array keeps the first call's contents) and checks both outputs against
mobi_gemm, the entry point that takes a workspace, and against the CPU oracle,
within the GEMM tolerance of the other tests; it also checks that a shape
needing more scratch than the array holds is refused before anything runs. It
passes alone in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity import check_gemm
from token_adaptive_mixed_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def mobi():
    import token_adaptive_mixed_b200 as m
    from token_adaptive_mixed_b200 import build
    build.build()
    m.lib()
    return m


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("N,K,T", [(4096, 4096, 16), (11008, 4096, 5), (512, 11008, 1)])
def test_noalloc_matches_workspace_entry_point(mobi, oracle, N, K, T):
    L = wl.layer("na", N, K, T, seed=N + K + T, outlier_frac_cols=0.005)
    W = torch.from_numpy(L.W).to(DEV)
    codes, sz = mobi.mobi_pack(W, S=3)
    X = L.X.to(DEV)
    k_t, perm, off = mobi.mobi_route(X, torch.from_numpy(L.Wr).to(DEV))
    y_ws = mobi.mobi_gemm(X, k_t, perm, off, codes, sz, N)
    mobi.mobi_sync_check()
    ref = y_ws.cpu().numpy().astype(np.float64)
    k = k_t.cpu().numpy()
    y_oracle = oracle.gemm(L.X, k, codes.cpu().numpy().view(np.uint32), sz.cpu().numpy().view(np.uint32), N)
    check_gemm(ref, y_oracle, f"workspace entry point, N={N} K={K} T={T}")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        Y = torch.full((T, N), float("nan"), dtype=torch.float32, device=DEV)
        st = mobi.lib().mobi_gemm_decode_noalloc(_p(X), T, K, _p(k_t), _p(codes), _p(sz), N, 128, 3, _p(Y), stream)
        assert st == 0, mobi.mobi_last_error()
        mobi.mobi_sync_check()
        y = Y.cpu().numpy()
        check_gemm(y, ref, f"no-alloc call {call + 1} vs mobi_gemm, N={N} K={K} T={T}")
        check_gemm(y, y_oracle, f"no-alloc call {call + 1} vs the oracle, N={N} K={K} T={T}")


def test_noalloc_refuses_oversized_scratch(mobi):
    """28672 x 8192 needs ~14 MiB of decode scratch: refused, nothing launched."""
    N, K, T = 28672, 8192, 4
    small = torch.zeros(1024, dtype=torch.int32, device=DEV)  # never read: the size check comes first
    Y = torch.zeros(16, dtype=torch.float32, device=DEV)
    st = mobi.lib().mobi_gemm_decode_noalloc(_p(small), T, K, _p(small), _p(small), _p(small), N, 128, 3, _p(Y),
                                             None)
    assert st == 4  # MOBI_ERR_WORKSPACE
    assert "static array" in mobi.mobi_last_error()
    mobi.mobi_sync_check()
