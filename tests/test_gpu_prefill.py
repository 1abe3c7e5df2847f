"""GPU parity of the tcgen05 prefill GEMM against the CPU oracle.

Sizes span several weight tiles (128 rows) and token tiles (192 tokens) with
ragged tails, every mix of slice counts, tokens unsorted (the routing order is
applied inside), and the full prefill workloads: every token of the 2048-token
one; for the 4096-token skewed one every x8-scaled token and whole 192-token
tiles of every bucket. The bar is
max |y - y_ref| <= 1e-2 (|y_ref| + 1e-3) element-wise and a relative
Frobenius error <= 2e-3.
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
    m.lib()
    return m


def u32(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)


def bucket_host(k):
    perm = np.argsort(k, kind="stable").astype(np.int32)
    off = np.concatenate([[0], np.cumsum(np.bincount(k, minlength=4)[1:])]).astype(np.int32)
    return perm, off


def gemm(mobi, X, k, codes, sz, N, path):
    """The GEMM on the GPU with canary words around Y (checked: nothing written
    outside the output, ragged token and row tails included)."""
    perm, off = bucket_host(k)
    Y, guards = guarded_output(X.shape[0], N)
    mobi.mobi_gemm_path(X.to(DEV), torch.from_numpy(k).to(DEV), torch.from_numpy(perm).to(DEV),
                        torch.from_numpy(off).to(DEV), u32(codes), u32(sz), N, path=path, Y=Y)
    mobi.mobi_sync_check()
    guards(f"N={N} T={X.shape[0]} path={path}")
    return Y.cpu().numpy()


@pytest.mark.parametrize("N,K,T", [(128, 128, 17), (256, 384, 100), (272, 1152, 191), (128, 256, 192),
                                   (384, 640, 193), (144, 2048, 500), (512, 512, 1000)])
def test_prefill_shapes(mobi, oracle, N, K, T):
    L = wl.layer("p", N, K, T, seed=N * 7 + K + T, outlier_frac_cols=0.005)
    codes, sz, _ = oracle.pack(L.W, S=3)
    k = np.random.default_rng(T).integers(1, 4, T).astype(np.int32)
    Y = gemm(mobi, L.X, k, codes, sz, N, path=2)
    check_gemm(Y, oracle.gemm(L.X, k, codes, sz, N), f"prefill N={N} K={K} T={T}")


@pytest.mark.parametrize("N,K,T", [(1664, 256, 2304), (2048, 128, 4000)])
def test_prefill_persistent_multi_tile(mobi, oracle, N, K, T):
    """More tiles (128 rows x 192 tokens) than SMs, so CTAs walk several tiles
    and the pipeline state carries across tile boundaries; sampled tokens from
    every bucket and every token tile against the oracle (all N)."""
    L = wl.layer("mt", N, K, T, seed=T + 3, outlier_frac_cols=0.005)
    codes, sz, _ = oracle.pack(L.W, S=3)
    k = np.random.default_rng(T).integers(1, 4, T).astype(np.int32)
    Y = gemm(mobi, L.X, k, codes, sz, N, path=2)
    perm = np.argsort(k, kind="stable")
    toks = np.unique(np.concatenate([perm[::97], perm[191::192], perm[:3], perm[-3:]])).astype(np.int32)
    check_gemm(Y[toks], oracle.gemm(L.X, k, codes, sz, N, tokens=toks), f"multi-tile N={N} K={K} T={T}")


@pytest.mark.parametrize("mix", [(1, 0, 0), (0, 0, 1), (0, 1, 0), (0.7, 0.2, 0.1), (0.1, 0.1, 0.8)])
def test_prefill_bucket_mixes(mobi, oracle, mix):
    """Empty buckets, single-bucket batches and skewed mixes."""
    N, K, T = 256, 512, 400
    L = wl.layer("m", N, K, T, seed=55, outlier_frac_cols=0.01)
    codes, sz, _ = oracle.pack(L.W, S=3)
    rng = np.random.default_rng(3)
    k = (rng.choice(3, T, p=np.array(mix) / sum(mix)) + 1).astype(np.int32)
    Y = gemm(mobi, L.X, k, codes, sz, N, path=2)
    check_gemm(Y, oracle.gemm(L.X, k, codes, sz, N), f"mix {mix}")


@pytest.mark.parametrize("T", [1, 7, 16])
def test_prefill_matches_decode_small_T(mobi, oracle, T):
    """Both kernels on the same small batch: each within the bar of the oracle."""
    L = wl.tiny(T)
    codes, sz, _ = oracle.pack(L.W, S=3)
    k, _, _ = oracle.route(L.X, L.Wr)
    ref = oracle.gemm(L.X, k, codes, sz, L.N)
    check_gemm(gemm(mobi, L.X, k, codes, sz, L.N, path=2), ref, "prefill")
    check_gemm(gemm(mobi, L.X, k, codes, sz, L.N, path=1), ref, "decode")


def test_prefill_one_slice(mobi, oracle):
    """S = 1 packing: a plain 2-bit RTN GEMM."""
    N, K, T = 128, 256, 64
    L = wl.layer("s1", N, K, T, seed=8)
    codes, sz, _ = oracle.pack(L.W, S=1)
    k = np.ones(T, np.int32)
    perm, off = np.arange(T, dtype=np.int32), np.array([0, T], np.int32)
    Y = mobi.mobi_gemm_path(L.X.to(DEV), torch.from_numpy(k).to(DEV), torch.from_numpy(perm).to(DEV),
                            torch.from_numpy(off).to(DEV), u32(codes), u32(sz), N, path=2, S=1)
    mobi.mobi_sync_check()
    check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k, codes, sz, N, S=1), "S=1")


def _full_workload(mobi, oracle, L, pick_tokens):
    """Pack, route and GEMM the whole workload on the GPU (as the benchmark's
    prefill does); then pack bit-exact on sampled rows, routing on every token,
    and every output row n < N of the tokens pick_tokens(k) selects against the
    oracle."""
    W = torch.from_numpy(L.W).to(DEV)
    codes_t, sz_t = mobi.mobi_pack(W, S=3)
    X = L.X.to(DEV)
    b = None if L.bias is None else torch.from_numpy(L.bias).to(DEV)
    k_t, perm, off = mobi.mobi_route(X, torch.from_numpy(L.Wr).to(DEV), b)
    Y = mobi.mobi_gemm(X, k_t, perm, off, codes_t, sz_t, L.N)
    mobi.mobi_sync_check()
    codes = codes_t.cpu().numpy().view(np.uint32)
    sz = sz_t.cpu().numpy().view(np.uint32)
    rows = np.random.default_rng(1).choice(L.N, 48, replace=False)
    c_ref, s_ref, _ = oracle.pack(L.W[rows], S=3)
    assert np.array_equal(codes[:, rows], c_ref) and np.array_equal(sz[:, :, rows], s_ref)
    k_ref, gap, _ = oracle.route(L.X, L.Wr, L.bias)
    k_gpu = k_t.cpu().numpy()
    check_route(k_gpu, k_ref, gap)
    assert np.array_equal(perm.cpu().numpy(), np.argsort(k_gpu, kind="stable"))
    toks = np.asarray(sorted(set(int(t) for t in pick_tokens(k_gpu))), np.int32)
    ref = oracle.gemm(L.X, k_gpu, codes, sz, L.N, tokens=toks)
    check_gemm(Y.cpu().numpy()[toks], ref, L.name)
    return toks


def bucket_tiles(k, tile=192, per_bucket=2):
    """Tokens of whole 192-token tiles in bucket order (the prefill kernel's token
    tiles): the first and last tile, and `per_bucket` tiles lying wholly inside
    each slice-count bucket (the first ones of the bucket and the last)."""
    perm = np.argsort(k, kind="stable")
    T = len(k)
    starts = {0, (T - 1) // tile * tile}
    for j in (1, 2, 3):
        idx = np.nonzero(k[perm] == j)[0]
        if idx.size == 0:
            continue
        lo = (idx[0] + tile - 1) // tile * tile        # first tile starting inside the bucket
        hi = (idx[-1] + 1) // tile * tile - tile        # last tile ending inside it
        inside = list(range(lo, hi + 1, tile)) if hi >= lo else [idx[0] // tile * tile]
        starts.update(inside[:per_bucket - 1] + inside[-1:])
    return np.concatenate([perm[s:s + tile] for s in sorted(starts)])


@pytest.mark.slow
def test_prefill_workload_full_size(mobi, oracle):
    """T=2048, N=11008, K=4096, thirds: every token and every output row against the oracle."""
    L = wl.prefill()
    toks = _full_workload(mobi, oracle, L, lambda k: range(len(k)))
    assert len(toks) == L.T


@pytest.mark.slow
def test_skewed_prefill_workload_full_size(mobi, oracle):
    """T=4096, N=28672, K=8192, 70/20/10 with 2% of tokens x8: every x8 token,
    two whole 192-token tiles inside each bucket plus the first and last tile of
    the bucket order, all output rows, against the oracle."""
    L = wl.skewed_prefill()
    assert len(L.scaled_tokens) == 82

    def pick(k):
        return np.concatenate([L.scaled_tokens, bucket_tiles(k)])
    toks = _full_workload(mobi, oracle, L, pick)
    assert set(L.scaled_tokens.tolist()) <= set(toks.tolist())
