"""Full-model workload: the 7 linear projections x 32 layers of a Llama-2-7B-
shaped stack (6.5e9 fp16 parameters drawn on the device), packed by mobi_pack,
then batch-8 decode through every projection with mobi_linear (random router
per projection).

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
