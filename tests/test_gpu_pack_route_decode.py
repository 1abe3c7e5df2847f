"""GPU parity: mobi_pack, mobi_route and the decode GEMM against the CPU oracle.

Bars: packed codes and scale/zero words bit-exact; routing decisions equal
except where the oracle's fp64 top-two logit gap is below 1e-5 (counted);
perm/offsets exact given the GPU's k_t; GEMM outputs within
max |y - y_ref| <= 1e-2 (|y_ref| + 1e-3) and relative Frobenius <= 2e-3.
"""
import numpy as np
import pytest
import torch

from parity import check_gemm, check_route, guarded_output
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


def gpu_pack(mobi, W_np, S=3):
    W = torch.from_numpy(np.ascontiguousarray(W_np)).to(DEV)
    codes, sz = mobi.mobi_pack(W, S=S)
    mobi.mobi_sync_check()
    return codes.cpu().numpy().view(np.uint32), sz.cpu().numpy().view(np.uint32)


def to_dev_u32(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)


# ---- pack --------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,seed", [(256, 512, 0), (16, 128, 1), (48, 384, 2), (32, 640, 3), (64, 1152, 4),
                                      (16, 11008, 5)])
def test_pack_bit_exact(mobi, oracle, N, K, seed):
    W = wl.draw_weights(np.random.default_rng(seed), N, K, 0.02, max(1, K // 200))
    codes_ref, sz_ref, _ = oracle.pack(W, S=3)
    codes, sz = gpu_pack(mobi, W)
    assert np.array_equal(sz, sz_ref)
    assert np.array_equal(codes, codes_ref)


def test_pack_closed_form_groups(mobi, oracle):
    """Rows built from the hand-derived groups of the oracle pins (ties to even,
    clamps, the 2^-14 floor, all-negative and constant groups)."""
    pats = [[-1.5 / 16, -0.5 / 16, 0.5 / 16, 1.5 / 16], [-4 / 64, -3 / 64, -2 / 64, -1 / 64], [1.0],
            [-2 ** -5, 0.0, 2 ** -5, 2 ** -4], [0.0], [-0.0, 0.0]]
    rows = []
    for i in range(16):
        p = pats[i % len(pats)]
        rows.append(np.array([p[j % len(p)] for j in range(256)], np.float16))
    W = np.stack(rows)
    codes_ref, sz_ref, _ = oracle.pack(W, S=3)
    codes, sz = gpu_pack(mobi, W)
    assert np.array_equal(sz, sz_ref) and np.array_equal(codes, codes_ref)


def test_pack_slices_1_and_2(mobi, oracle):
    W = wl.draw_weights(np.random.default_rng(9), 32, 256, 0.02, 2)
    for S in (1, 2):
        codes_ref, sz_ref, _ = oracle.pack(W, S=S)
        codes, sz = gpu_pack(mobi, W, S=S)
        assert np.array_equal(codes, codes_ref) and np.array_equal(sz, sz_ref)


# ---- route -------------------------------------------------------------------------

@pytest.mark.parametrize("T,K,mix", [(16, 512, None), (1, 4096, None), (3, 11008, None), (17, 256, None),
                                     (16, 128, None), (16, 11008, (0.5, 0.3, 0.2)), (9, 4096, (0.1, 0.1, 0.8)),
                                     (100, 1024, (0.2, 0.3, 0.5)), (2048, 4096, (1 / 3, 1 / 3, 1 / 3)),
                                     (1500, 2048, (0.7, 0.2, 0.1))])
def test_route_and_bucket(mobi, oracle, T, K, mix):
    L = wl.layer("r", 16, K, T, seed=100 + T, mix=mix)
    k_ref, gap, _ = oracle.route(L.X, L.Wr, L.bias)
    X = L.X.to(DEV)
    Wr = torch.from_numpy(L.Wr).to(DEV)
    b = None if L.bias is None else torch.from_numpy(L.bias).to(DEV)
    k_t, perm, off = mobi.mobi_route(X, Wr, b)
    mobi.mobi_sync_check()
    k_gpu = k_t.cpu().numpy()
    check_route(k_gpu, k_ref, gap, f"T={T}")
    perm_ref, off_ref = oracle.bucket(k_gpu)
    assert np.array_equal(perm.cpu().numpy(), perm_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)


@pytest.mark.parametrize("S", [1, 2])
@pytest.mark.parametrize("T", [1, 13])
def test_route_small_fewer_slices(mobi, oracle, T, S):
    """Up to 16 tokens (one cluster launch) with one or two slices."""
    L = wl.layer("r", 16, 1024, T, seed=300 + T + S)
    Wr = np.ascontiguousarray(L.Wr[:, :S])
    k_ref, gap, _ = oracle.route(L.X, Wr, None)
    k_t, perm, off = mobi.mobi_route(L.X.to(DEV), torch.from_numpy(Wr).to(DEV))
    mobi.mobi_sync_check()
    k_gpu = k_t.cpu().numpy()
    check_route(k_gpu, k_ref, gap, f"T={T} S={S}")
    perm_ref, off_ref = oracle.bucket(k_gpu, S)
    assert np.array_equal(perm.cpu().numpy(), perm_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)


def test_route_empty(mobi):
    X = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    Wr = torch.zeros((256, 3), dtype=torch.float32, device=DEV)
    k_t, perm, off = mobi.mobi_route(X, Wr)
    mobi.mobi_sync_check()
    assert off.cpu().tolist() == [0, 0, 0, 0]


def test_route_ties_lowest_index(mobi):
    T, K = 8, 128
    X = torch.ones((T, K), dtype=torch.bfloat16, device=DEV)
    Wr = torch.zeros((K, 3), dtype=torch.float32, device=DEV)
    k_t, _, _ = mobi.mobi_route(X, Wr, torch.tensor([0.0, 1.0, 1.0], device=DEV))
    assert k_t.cpu().tolist() == [2] * T


# ---- decode GEMM ---------------------------------------------------------------------

def run_gemm(mobi, L, codes, sz, k, path=0, X=None):
    """The GEMM on the GPU with canary words around Y (checked: nothing written
    outside the output)."""
    X = (L.X if X is None else X).to(DEV)
    k_t = torch.from_numpy(k.astype(np.int32)).to(DEV)
    perm = torch.from_numpy(np.argsort(k, kind="stable").astype(np.int32)).to(DEV)
    off = torch.from_numpy(np.concatenate([[0], np.cumsum(np.bincount(k, minlength=4)[1:])]).astype(np.int32)).to(DEV)
    Y, guards = guarded_output(X.shape[0], L.N)
    mobi.mobi_gemm_path(X, k_t, perm, off, to_dev_u32(codes), to_dev_u32(sz), L.N, path=path, Y=Y)
    mobi.mobi_sync_check()
    guards(f"N={L.N} K={L.K} T={X.shape[0]}")
    return Y.cpu().numpy()


@pytest.mark.parametrize("T", [1, 4, 16])
def test_decode_tiny(mobi, oracle, T):
    L = wl.tiny(T)
    codes, sz, _ = oracle.pack(L.W, S=3)
    k, _, _ = oracle.route(L.X, L.Wr)
    Y = run_gemm(mobi, L, codes, sz, k)
    check_gemm(Y, oracle.gemm(L.X, k, codes, sz, L.N), f"tiny T={T}")


@pytest.mark.parametrize("N,K", [(48, 384), (16, 1152), (80, 2176), (4096, 4096)])
@pytest.mark.parametrize("T", [1, 5, 9, 16])
def test_decode_shapes(mobi, oracle, N, K, T):
    """Several row blocks (64 rows), column chunks (1024) with ragged tails, and
    both token widths (<= 8 and <= 16)."""
    L = wl.layer("d", N, K, T, seed=N + K + T, outlier_frac_cols=0.005)
    codes, sz, _ = oracle.pack(L.W, S=3)
    rng = np.random.default_rng(T)
    k = rng.integers(1, 4, T).astype(np.int32)
    Y = run_gemm(mobi, L, codes, sz, k)
    check_gemm(Y, oracle.gemm(L.X, k, codes, sz, L.N), f"N={N} K={K} T={T}")


@pytest.mark.parametrize("kval", [1, 2, 3])
def test_decode_uniform_k(mobi, oracle, kval):
    """Every token the same k: the kernel streams exactly k slices."""
    L = wl.layer("u", 128, 1024, 8, seed=7)
    codes, sz, _ = oracle.pack(L.W, S=3)
    k = np.full(8, kval, np.int32)
    Y = run_gemm(mobi, L, codes, sz, k)
    check_gemm(Y, oracle.gemm(L.X, k, codes, sz, L.N), f"k={kval}")


@pytest.mark.slow
@pytest.mark.parametrize("N,K", wl.DECODE_SHAPES)
def test_decode_llama_shapes_full(mobi, oracle, N, K):
    """The decode workload at full size: pack on the GPU (checked bit-exact on
    sampled rows) and the GEMM for T = 16 against the oracle on all outputs."""
    L = wl.decode(N, K, 16)
    W = torch.from_numpy(L.W).to(DEV)
    codes_t, sz_t = mobi.mobi_pack(W, S=3)
    mobi.mobi_sync_check()
    codes = codes_t.cpu().numpy().view(np.uint32)
    sz = sz_t.cpu().numpy().view(np.uint32)
    rows = np.random.default_rng(0).choice(N, 64, replace=False)
    c_ref, s_ref, _ = oracle.pack(L.W[rows], S=3)
    assert np.array_equal(codes[:, rows], c_ref)
    assert np.array_equal(sz[:, :, rows], s_ref)
    k, gap, _ = oracle.route(L.X, L.Wr)
    X = L.X.to(DEV)
    k_t, perm, off = mobi.mobi_route(X, torch.from_numpy(L.Wr).to(DEV))
    check_route(k_t.cpu().numpy(), k, gap)
    Y = mobi.mobi_gemm(X, k_t, perm, off, codes_t, sz_t, N)
    mobi.mobi_sync_check()
    check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k, codes, sz, N), f"decode {N}x{K}")


def test_decode_activation_range(mobi, oracle):
    """The decode kernel takes |x| < 2^31 (it scales x by up to 2^96 in bf16).
    One x = 2^31 is reported by mobi_sync_check as MOBI_ERR_INVALID_ARG; the
    largest bf16 below 2^31 is accepted (within the bars and the fp32
    cancellation bound of the folded zero point); the prefill kernel (any T)
    has no such limit; the context stays usable."""
    L = wl.tiny(4)
    codes, sz, _ = oracle.pack(L.W, S=3)
    k = np.array([3, 1, 2, 3], np.int32)
    big = L.X.clone()
    big[1, 5] = 2.0 ** 31
    with pytest.raises(mobi.MobiError) as ei:
        run_gemm(mobi, L, codes, sz, k, path=1, X=big)
    assert ei.value.status == 1 and "2^31" in mobi.mobi_last_error()
    check_gemm(run_gemm(mobi, L, codes, sz, k, path=2, X=big), oracle.gemm(big, k, codes, sz, L.N), "prefill, x=2^31")
    edge = L.X.clone()
    edge[1, 5] = 2.0 ** 31 - 2.0 ** 23  # bf16 0x4EFF, the largest bf16 below 2^31
    assert float(edge[1, 5]) == 2.0 ** 31 - 2.0 ** 23
    # Accepted and finite; the zero point is folded as sum x q - z sum x in fp32,
    # so the absolute error grows with |x|: per (slice, group) both terms are at
    # most 3 sum|x| and the fp32 sums (tensor core, then one fma each) round at
    # most ~32 times by u = 2^-24, i.e. |err| <= 2^-18 sum_s sum_g scale * 3 sum_g |x|
    # on top of the element bar. The relative Frobenius bar holds as usual.
    y = run_gemm(mobi, L, codes, sz, k, path=1, X=edge)
    y_ref = oracle.gemm(edge, k, codes, sz, L.N)
    assert np.isfinite(y).all()
    xs = np.abs(edge.float().numpy().astype(np.float64)).reshape(edge.shape[0], -1, 128).sum(2)  # [T][K/128]
    scale = (sz & 0xFFFF).astype(np.uint16).view(np.float16).astype(np.float64)  # [S][K/128][N]
    allow = np.stack([2.0 ** -18 * 3 * np.einsum("sgn,g->n", scale[:k[t]], xs[t]) for t in range(len(k))])
    assert np.all(np.abs(y - y_ref) <= 1e-2 * (np.abs(y_ref) + 1e-3) + allow)
    assert np.linalg.norm(y - y_ref) <= 2e-3 * np.linalg.norm(y_ref)
    check_gemm(run_gemm(mobi, L, codes, sz, k, path=1), oracle.gemm(L.X, k, codes, sz, L.N), "decode after the error")
