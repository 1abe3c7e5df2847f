"""Generic slicing on the GPU: b-bit slices (b = 1, 2) over G-wide groups
(G = 128, 256, 512) and up to four slices, against the CPU oracle.

Pack: codes bit-exact (1-bit codes at 32 per word); the scale/zero words
bit-exact after repeating each G-wide group's word over its G/128 sub-groups
(the layout the GEMM kernels read). GEMMs (decode and prefill kernels reading
1-bit codes in their own layout), routing and bucketing: the bars of the other
parity tests, with the oracle computing at the native group width.
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


def expand_sz(sz, G):
    """Oracle sz [S][K/G][N] -> the GPU layout [S][K/128][N]."""
    return np.repeat(sz, G // 128, axis=1)


@pytest.mark.parametrize("bits,G,S,N,K", [(1, 128, 4, 256, 1024), (1, 256, 4, 80, 2304), (2, 256, 3, 128, 4096),
                                          (2, 512, 2, 48, 1024), (1, 512, 3, 64, 11264), (2, 128, 4, 32, 384)])
def test_pack_generic_bit_exact(mobi, oracle, bits, G, S, N, K):
    L = wl.layer("gp", N, K, 1, seed=2000 + bits + G + S, outlier_frac_cols=0.01)
    codes, sz = mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), S=S, G=G, bits=bits)
    torch.cuda.synchronize()
    c_ref, s_ref, q_ref = oracle.pack_bits(L.W, G=G, S=S, bits=bits)
    assert codes.numel() * 4 == mobi.mobi_codes_bytes(N, K, S, bits=bits) == S * N * K * bits // 8
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), c_ref)
    assert np.array_equal(sz.cpu().numpy().view(np.uint32), expand_sz(s_ref, G))
    assert q_ref.max() <= (1 << bits) - 1


def _layer_s(name, N, K, T, S, seed, mix=None):
    return wl.layer(name, N, K, T, seed=seed, outlier_frac_cols=0.005, S=S,
                    mix=mix if mix is not None else tuple([1.0 / S] * S))


@pytest.mark.parametrize("T", [1, 4, 16, 300])
@pytest.mark.parametrize("bits,G", [(1, 128), (1, 256)])
def test_four_slice_linear(mobi, oracle, T, bits, G):
    """Four b-bit slices (1..4 bits for b = 1) through route + GEMM (decode for
    T <= 16, tcgen05 prefill for T = 300)."""
    N, K, S = 512, 2048, 4
    L = _layer_s("l4", N, K, T, S, seed=2100 + T + bits + G)
    codes, sz = mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), S=S, G=G, bits=bits)
    Wr = torch.from_numpy(L.Wr).to(DEV)
    b = torch.from_numpy(L.bias).to(DEV)
    Y, k_t, perm, off = mobi.mobi_linear(L.X.to(DEV), Wr, b, codes, sz, N, bits=bits)
    mobi.mobi_sync_check()
    tag = f"S=4 b={bits} G={G} T={T}"
    k_gpu = k_t.cpu().numpy()
    k_ref, gap, _ = oracle.route(L.X, L.Wr, L.bias)
    check_route(k_gpu, k_ref, gap, tag)
    perm_ref, off_ref = oracle.bucket(k_gpu, S)
    assert np.array_equal(perm.cpu().numpy(), perm_ref) and np.array_equal(off.cpu().numpy(), off_ref)
    c_ref, s_ref, _ = oracle.pack_bits(L.W, G=G, S=S, bits=bits)
    check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k_gpu, c_ref, s_ref, N, G=G, S=S, bits=bits), tag)
    if T > 1:
        assert len(set(k_gpu.tolist())) > 1, "the mix should use several precisions"


@pytest.mark.parametrize("T", [1, 5, 8, 9, 16, 17, 130])
@pytest.mark.parametrize("S", [1, 3])
def test_one_bit_gemm_both_kernels(mobi, oracle, T, S):
    """1-bit slices through both kernels with an explicit path: K = 1152 ends in
    a ragged 1024-column chunk (decode) and N = 208 in a partial 128-row tile
    (prefill); k_t drawn over 1..S."""
    N, K = 208, 1152
    L = wl.layer("b1", N, K, T, seed=2400 + T + 10 * S, outlier_frac_cols=0.01)
    codes, sz = mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), S=S, bits=1)
    c_ref, s_ref, _ = oracle.pack_bits(L.W, G=128, S=S, bits=1)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), c_ref)
    k = np.random.default_rng(T + S).integers(1, S + 1, T).astype(np.int32)
    perm_np, off_np = oracle.bucket(k, S)
    ref = oracle.gemm(L.X, k, c_ref, s_ref, N, S=S, bits=1)
    paths = [1, 2] if T <= 16 else [2]
    for path in paths:
        Y = mobi.mobi_gemm_path(L.X.to(DEV), torch.from_numpy(k).to(DEV), torch.from_numpy(perm_np).to(DEV),
                                torch.from_numpy(off_np).to(DEV), codes, sz, N, path=path, bits=1)
        mobi.mobi_sync_check()
        check_gemm(Y.cpu().numpy(), ref, f"1-bit S={S} T={T} path={path}")


def test_one_bit_grouped_decode(mobi, oracle):
    """A grouped decode step of 4-slice 1-bit layers (both fragment classes):
    the grouped results equal single calls bit for bit and meet the oracle."""
    S = 4
    specs = [(256, 1024, 3), (512, 2048, 16), (128, 512, 8), (4096, 4096, 4)]
    probs, layers = [], []
    for i, (N, K, T) in enumerate(specs):
        L = _layer_s("g1", N, K, T, S, seed=2250 + i)
        codes, sz = mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), S=S, bits=1)
        layers.append(L)
        probs.append({"X": L.X.to(DEV), "Wr": torch.from_numpy(L.Wr).to(DEV), "bias": torch.from_numpy(L.bias).to(DEV),
                      "codes": codes, "sz": sz, "N": N})
    outs = mobi.mobi_linear_grouped(probs, S=S, bits=1)
    mobi.mobi_sync_check()
    for pr, L, (Y, k_t, perm, off) in zip(probs, layers, outs):
        Ys, ks, _, _ = mobi.mobi_linear(pr["X"], pr["Wr"], pr["bias"], pr["codes"], pr["sz"], pr["N"], bits=1)
        mobi.mobi_sync_check()
        assert torch.equal(Y, Ys) and torch.equal(k_t, ks)
        c_ref, s_ref, _ = oracle.pack_bits(L.W, G=128, S=S, bits=1)
        check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k_t.cpu().numpy(), c_ref, s_ref, pr["N"], S=S, bits=1),
                   f"grouped 1-bit N={pr['N']} T={L.T}")


def test_four_slice_grouped_and_checkpoint(mobi, oracle, tmp_path):
    """Grouped decode step and a checkpoint of 4-slice (2-bit) layers: the
    grouped results equal single calls, and a checkpoint loaded at 2 slices
    serves tokens routed to at most 2 slices exactly like the full pack."""
    S = 4
    specs = [(256, 1024, 3), (512, 2048, 16), (128, 512, 8)]
    probs, layers = [], []
    for i, (N, K, T) in enumerate(specs):
        L = _layer_s("g4", N, K, T, S, seed=2200 + i)
        codes, sz = mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), S=S, bits=2)
        layers.append(L)
        probs.append({"X": L.X.to(DEV), "Wr": torch.from_numpy(L.Wr).to(DEV), "bias": torch.from_numpy(L.bias).to(DEV),
                      "codes": codes, "sz": sz, "N": N})
    outs = mobi.mobi_linear_grouped(probs, S=S)
    mobi.mobi_sync_check()
    for pr, (Y, k_t, perm, off) in zip(probs, outs):
        Ys, ks, _, _ = mobi.mobi_linear(pr["X"], pr["Wr"], pr["bias"], pr["codes"], pr["sz"], pr["N"])
        assert torch.equal(Y, Ys) and torch.equal(k_t, ks)
    path = tmp_path / "four.mobi"
    mobi.mobi_ckpt_save(path, [(f"p{i}", pr["codes"], pr["sz"]) for i, pr in enumerate(probs)])
    with mobi.MobiCheckpoint(path) as ck:
        for i, (pr, L) in enumerate(zip(probs, layers)):
            c2, z2 = ck.load(f"p{i}", 2, device=DEV)
            assert torch.equal(c2, pr["codes"][:2]) and torch.equal(z2, pr["sz"][:2])
            k_np = np.random.default_rng(i).integers(1, 3, L.T).astype(np.int32)
            perm_np, off2 = oracle.bucket(k_np, 2)
            _, off4 = oracle.bucket(k_np, 4)
            k_t = torch.from_numpy(k_np).to(DEV)
            perm = torch.from_numpy(perm_np).to(DEV)
            Y2 = mobi.mobi_gemm(pr["X"], k_t, perm, torch.from_numpy(off2).to(DEV), c2, z2, pr["N"])
            Y4 = mobi.mobi_gemm(pr["X"], k_t, perm, torch.from_numpy(off4).to(DEV), pr["codes"], pr["sz"], pr["N"])
            mobi.mobi_sync_check()
            assert torch.equal(Y2, Y4)


def test_four_slice_threshold_routing(mobi, oracle):
    """Threshold routing with three residual slices (S = 4)."""
    from parity import check_route_mlp, mlp_score_bound
    R = wl.mlp_router("mlp4", 200, 1024, 64, seed=2300, S=4)
    W1 = torch.from_numpy(R.W1).to(DEV)
    W2 = torch.from_numpy(np.ascontiguousarray(R.W2)).to(DEV)
    k_t, perm, off = mobi.mobi_route_mlp(R.X.to(DEV), W1, torch.from_numpy(R.b1).to(DEV), W2,
                                         torch.from_numpy(R.b2).to(DEV), 1.0, 0.5)
    mobi.mobi_sync_check()
    k_gpu = k_t.cpu().numpy()
    k_ref, _, scores = oracle.route_mlp(R.X, R.W1, R.b1, R.W2, R.b2, 1.0, 0.5)
    check_route_mlp(k_gpu, scores, mlp_score_bound(R.X.float().numpy(), R.W1, R.b1, R.W2, R.b2, 0.0), 0.0,
                    "mlp S=4")
    perm_ref, off_ref = oracle.bucket(k_gpu, 4)
    assert np.array_equal(perm.cpu().numpy(), perm_ref) and np.array_equal(off.cpu().numpy(), off_ref)
    assert k_gpu.max() == 4 and len(set(k_gpu.tolist())) >= 3


# ---- slices of mixed widths in one layer ---------------------------------------

MIXED = (2, 1, 1, 2)  # 2, 3, 4 and 6 bits per weight


@pytest.mark.parametrize("widths,N,K", [(MIXED, 256, 1024), ((1, 2), 80, 1152), ((2, 1, 2), 208, 4096)])
def test_pack_slices_bit_exact(mobi, oracle, widths, N, K):
    L = wl.layer("ps", N, K, 1, seed=2500 + N + len(widths), outlier_frac_cols=0.01)
    codes, sz = mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), widths=widths)
    torch.cuda.synchronize()
    c_ref, s_ref, _ = oracle.pack_slices(L.W, widths)
    assert codes.numel() * 4 == mobi.mobi_codes_bytes(N, K, widths=widths) == c_ref.size * 4
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), c_ref)
    assert np.array_equal(sz.cpu().numpy().view(np.uint32), s_ref)


@pytest.mark.parametrize("T", [1, 6, 16, 130])
@pytest.mark.parametrize("widths", [MIXED, (1, 2)])
def test_mixed_gemm_both_kernels(mobi, oracle, T, widths):
    """Mixed widths through both kernels with an explicit path: K = 1152 ends
    in a ragged 1024-column chunk, N = 208 in a partial 128-row tile; k_t over
    1..S, so every slice width is read."""
    S = len(widths)
    N, K = 208, 1152
    L = wl.layer("mx", N, K, T, seed=2600 + T + 10 * S, outlier_frac_cols=0.01)
    codes, sz = mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), widths=widths)
    c_ref, s_ref, _ = oracle.pack_slices(L.W, widths)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), c_ref)
    k = np.random.default_rng(T + S).integers(1, S + 1, T).astype(np.int32)
    perm_np, off_np = oracle.bucket(k, S)
    ref = oracle.gemm(L.X, k, c_ref, s_ref, N, S=S, widths=widths)
    for path in ([1, 2] if T <= 16 else [2]):
        Y = mobi.mobi_gemm_path(L.X.to(DEV), torch.from_numpy(k).to(DEV), torch.from_numpy(perm_np).to(DEV),
                                torch.from_numpy(off_np).to(DEV), codes, sz, N, path=path, widths=widths)
        mobi.mobi_sync_check()
        check_gemm(Y.cpu().numpy(), ref, f"widths={widths} T={T} path={path}")


def test_mixed_linear_and_grouped(mobi, oracle):
    """Route + GEMM with widths (2, 1, 1, 2) (2, 3, 4, 6 bits): single calls and
    one grouped call over both fragment classes; grouped results equal single
    calls bit for bit and meet the oracle."""
    S = 4
    specs = [(512, 2048, 4), (256, 1024, 16), (4096, 4096, 8)]
    probs, layers = [], []
    for i, (N, K, T) in enumerate(specs):
        L = _layer_s("lm", N, K, T, S, seed=2700 + i)
        codes, sz = mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), widths=MIXED)
        layers.append(L)
        probs.append({"X": L.X.to(DEV), "Wr": torch.from_numpy(L.Wr).to(DEV), "bias": torch.from_numpy(L.bias).to(DEV),
                      "codes": codes, "sz": sz, "N": N})
    outs = mobi.mobi_linear_grouped(probs, S=S, widths=MIXED)
    mobi.mobi_sync_check()
    for pr, L, (Y, k_t, perm, off) in zip(probs, layers, outs):
        Ys, ks, _, _ = mobi.mobi_linear(pr["X"], pr["Wr"], pr["bias"], pr["codes"], pr["sz"], pr["N"], widths=MIXED)
        mobi.mobi_sync_check()
        assert torch.equal(Y, Ys) and torch.equal(k_t, ks)
        c_ref, s_ref, _ = oracle.pack_slices(L.W, MIXED)
        k_gpu = k_t.cpu().numpy()
        k_ref, gap, _ = oracle.route(L.X, L.Wr, L.bias)
        check_route(k_gpu, k_ref, gap, f"mixed N={pr['N']}")
        check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k_gpu, c_ref, s_ref, pr["N"], S=S, widths=MIXED),
                   f"mixed linear N={pr['N']} T={L.T}")
    # the GEMM half alone, k_t given
    gp = [{"X": pr["X"], "k_t": o[1], "codes": pr["codes"], "sz": pr["sz"], "N": pr["N"]} for pr, o in zip(probs, outs)]
    Yg = mobi.mobi_gemm_grouped(gp, S=S, widths=MIXED)
    mobi.mobi_sync_check()
    for y, o in zip(Yg, outs):
        assert torch.equal(y, o[0])
