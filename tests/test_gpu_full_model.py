"""Full-model workload: the 7 linear projections x 32 layers of a Llama-2-7B-
shaped stack (6.5e9 fp16 parameters drawn on the device), packed by mobi_pack,
then batch-8 decode through every projection with mobi_linear (random router
per projection), and again with one mobi_linear_grouped call per layer.

Every projection is packed and run; for one projection of each kind, spread
over the layers, 64 sampled rows are checked against the oracle: packed codes
and scale/zero words bit-exact, routing decisions equal outside the 1e-5
near-tie band, outputs within max |y - y_ref| <= 1e-2 (|y_ref| + 1e-3) and
relative Frobenius <= 2e-3. All other outputs must be finite.
"""
import numpy as np
import pytest
import torch

from parity import check_gemm, check_route
from token_adaptive_mixed_b200 import workloads as wl

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DEV = "cuda:0"
LAYERS = 32
SAMPLED = {(0, 0), (5, 1), (10, 2), (15, 3), (20, 4), (25, 5), (31, 6)}


@pytest.fixture(scope="module")
def mobi():
    import token_adaptive_mixed_b200 as m
    from token_adaptive_mixed_b200 import build
    build.build()
    assert torch.cuda.is_available()
    m.lib()
    return m


def test_full_model_pack_and_decode(mobi, oracle):
    nproj = len(wl.LLAMA7B_PROJECTIONS)
    params = 0
    for layer in range(LAYERS):
        for p in range(nproj):
            L = wl.full_model_projection(layer, p, T=8, device=DEV)
            params += L.N * L.K
            codes, sz = mobi.mobi_pack(L.W, S=3)
            Wr = torch.from_numpy(L.Wr).to(DEV)
            Y, k_t, _, _ = mobi.mobi_linear(L.X.to(DEV), Wr, None, codes, sz, L.N)
            mobi.mobi_sync_check()
            assert torch.isfinite(Y).all(), L.name
            if (layer, p) not in SAMPLED:
                continue
            rows = np.sort(np.random.default_rng(layer * 7 + p).choice(L.N, 64, replace=False))
            W_rows = L.W[torch.from_numpy(rows).to(DEV)].cpu().numpy()
            c_ref, s_ref, _ = oracle.pack(W_rows, S=3)
            c_gpu = codes.cpu().numpy().view(np.uint32)[:, rows]
            s_gpu = sz.cpu().numpy().view(np.uint32)[:, :, rows]
            assert np.array_equal(c_gpu, c_ref), L.name
            assert np.array_equal(s_gpu, s_ref), L.name
            k_gpu = k_t.cpu().numpy()
            k_ref, gap, _ = oracle.route(L.X, L.Wr)
            check_route(k_gpu, k_ref, gap, L.name)
            y_ref = oracle.gemm(L.X, k_gpu, c_ref, s_ref, len(rows))
            check_gemm(Y.cpu().numpy()[:, rows], y_ref, L.name)
    assert params == 32 * (4 * 4096 * 4096 + 3 * 11008 * 4096)  # 6.48e9


def test_full_model_grouped_decode(mobi, oracle):
    """The same stack through mobi_linear_grouped, one call per layer with its
    seven projections (as the benchmark's full-model step runs it): every
    output and routing decision equal, bit for bit, to one mobi_linear call per
    projection, and 64 sampled rows of every one of the 224 projections against
    the oracle (packed words bit-exact, routing, outputs within the bars)."""
    nproj = len(wl.LLAMA7B_PROJECTIONS)
    checked = 0
    for layer in range(LAYERS):
        Ls = [wl.full_model_projection(layer, p, T=8, device=DEV) for p in range(nproj)]
        packed = [mobi.mobi_pack(L.W, S=3) for L in Ls]
        probs = [{"X": L.X.to(DEV), "Wr": torch.from_numpy(L.Wr).to(DEV), "bias": None, "codes": c, "sz": z,
                  "N": L.N} for L, (c, z) in zip(Ls, packed)]
        outs = mobi.mobi_linear_grouped(probs)
        mobi.mobi_sync_check()
        for L, pr, (Yg, kg, _, _) in zip(Ls, probs, outs):
            Y1, k1, _, _ = mobi.mobi_linear(pr["X"], pr["Wr"], None, pr["codes"], pr["sz"], L.N)
            mobi.mobi_sync_check()
            assert torch.equal(kg, k1), L.name
            assert torch.equal(Yg, Y1), L.name  # same kernels, same per-block order: bit-identical
            assert torch.isfinite(Yg).all(), L.name
            rows = np.sort(np.random.default_rng(layer * 7 + len(L.name)).choice(L.N, 64, replace=False))
            W_rows = L.W[torch.from_numpy(rows).to(DEV)].cpu().numpy()
            c_ref, s_ref, _ = oracle.pack(W_rows, S=3)
            assert np.array_equal(pr["codes"].cpu().numpy().view(np.uint32)[:, rows], c_ref), L.name
            assert np.array_equal(pr["sz"].cpu().numpy().view(np.uint32)[:, :, rows], s_ref), L.name
            k_gpu = kg.cpu().numpy()
            k_ref, gap, _ = oracle.route(L.X, L.Wr)
            check_route(k_gpu, k_ref, gap, L.name)
            check_gemm(Yg.cpu().numpy()[:, rows], oracle.gemm(L.X, k_gpu, c_ref, s_ref, len(rows)), L.name)
            checked += 1
        del packed, probs, outs
    assert checked == LAYERS * nproj
