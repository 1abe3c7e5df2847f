"""GPU parity of mobi_linear (routing + mixed-bit GEMM in one call) against the
CPU oracle, and against the two separate calls it fuses.

Bars as in the other GEMM tests: routing decisions equal except inside the
oracle's 1e-5 near-tie band, perm/offsets exact given the GPU's k_t, outputs
within max |y - y_ref| <= 1e-2 (|y_ref| + 1e-3) and relative Frobenius <= 2e-3.
The fused call runs the same kernels as mobi_route + mobi_gemm, so its output
must equal theirs bit for bit.
"""
import numpy as np
import pytest
import torch

from parity import check_gemm, check_route
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


def packed(mobi, L, S=3):
    codes, sz = mobi.mobi_pack(torch.from_numpy(np.ascontiguousarray(L.W)).to(DEV), S=S)
    return codes, sz


def check_linear(mobi, oracle, L, codes, sz, tag):
    Wr = torch.from_numpy(L.Wr).to(DEV)
    b = None if L.bias is None else torch.from_numpy(L.bias).to(DEV)
    Y, k_t, perm, off = mobi.mobi_linear(L.X.to(DEV), Wr, b, codes, sz, L.N)
    mobi.mobi_sync_check()
    k_gpu = k_t.cpu().numpy()
    k_ref, gap, _ = oracle.route(L.X, L.Wr, L.bias)
    check_route(k_gpu, k_ref, gap, tag)
    perm_ref, off_ref = oracle.bucket(k_gpu, L.Wr.shape[1])
    assert np.array_equal(perm.cpu().numpy(), perm_ref), tag
    assert np.array_equal(off.cpu().numpy(), off_ref), tag
    c = codes.cpu().numpy().view(np.uint32)
    s = sz.cpu().numpy().view(np.uint32)
    check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k_gpu, c, s, L.N), tag)
    return Y


@pytest.mark.parametrize("N,K,T,mix", [(256, 512, 1, None), (256, 512, 16, (0.2, 0.3, 0.5)),
                                       (80, 2176, 9, (0.5, 0.3, 0.2)), (48, 1152, 13, None),
                                       (4096, 4096, 4, (0.3, 0.3, 0.4))])
def test_linear_decode(mobi, oracle, N, K, T, mix):
    L = wl.layer("lin", N, K, T, seed=500 + N + T, mix=mix, outlier_frac_cols=0.005)
    codes, sz = packed(mobi, L)
    check_linear(mobi, oracle, L, codes, sz, f"linear N={N} K={K} T={T}")


@pytest.mark.parametrize("T", [40, 300])
def test_linear_prefill(mobi, oracle, T):
    L = wl.layer("linp", 256, 1024, T, seed=600 + T, mix=(0.4, 0.3, 0.3))
    codes, sz = packed(mobi, L)
    check_linear(mobi, oracle, L, codes, sz, f"linear prefill T={T}")


@pytest.mark.parametrize("T", [1, 8, 16])
def test_linear_equals_route_then_gemm(mobi, T):
    """The early start of the fused call changes nothing in the result."""
    L = wl.layer("leq", 1024, 4096, T, seed=700 + T, mix=(0.3, 0.3, 0.4))
    codes, sz = packed(mobi, L)
    X = L.X.to(DEV)
    Wr = torch.from_numpy(L.Wr).to(DEV)
    b = torch.from_numpy(L.bias).to(DEV)
    k_t, perm, off = mobi.mobi_route(X, Wr, b)
    Y_sep = mobi.mobi_gemm(X, k_t, perm, off, codes, sz, L.N)
    Y_lin, k_lin, perm_lin, off_lin = mobi.mobi_linear(X, Wr, b, codes, sz, L.N)
    mobi.mobi_sync_check()
    assert torch.equal(k_t, k_lin) and torch.equal(perm, perm_lin) and torch.equal(off, off_lin)
    assert torch.equal(Y_sep, Y_lin)


def test_linear_chain_of_layers(mobi, oracle):
    """Many calls back to back on one stream (each kernel a programmatic
    dependent of the one before), different shapes and token counts."""
    layers = [wl.layer("ch", N, K, T, seed=800 + i, mix=(0.3, 0.3, 0.4))
              for i, (N, K, T) in enumerate([(256, 512, 4), (512, 2048, 16), (256, 1024, 1), (1024, 4096, 9),
                                             (256, 512, 40), (512, 2048, 2)])]
    packs = [packed(mobi, L) for L in layers]
    outs = []
    for _ in range(3):
        outs = []
        for L, (codes, sz) in zip(layers, packs):
            b = torch.from_numpy(L.bias).to(DEV)
            outs.append(mobi.mobi_linear(L.X.to(DEV), torch.from_numpy(L.Wr).to(DEV), b, codes, sz, L.N))
    mobi.mobi_sync_check()
    for L, (codes, sz), (Y, k_t, _, _) in zip(layers, packs, outs):
        k_gpu = k_t.cpu().numpy()
        c = codes.cpu().numpy().view(np.uint32)
        s = sz.cpu().numpy().view(np.uint32)
        check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k_gpu, c, s, L.N), f"chain N={L.N} T={L.T}")
