"""The decode workload in the launch configuration the benchmark times: the
nine Llama-7B-shaped problems ((N,K) in {(4096,4096), (11008,4096),
(4096,11008)} x T in {1,4,16}), each with its own packed copy, as one
mobi_linear_grouped call (one routing launch, a decode launch per fragment
class, one chunk reduction).

Every output is checked against the oracle (routing exact outside the 1e-5
near-tie band, GEMM bars of the other tests), and the grouped results must
equal one mobi_linear call per problem bit for bit.
"""
import numpy as np
import pytest
import torch

from parity import check_gemm, check_route
from token_adaptive_mixed_b200 import workloads as wl

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DEV = "cuda:0"


@pytest.fixture(scope="module")
def mobi():
    import token_adaptive_mixed_b200 as m
    from token_adaptive_mixed_b200 import build
    build.build()
    assert torch.cuda.is_available()
    m.lib()
    return m


def test_headline_decode_step(mobi, oracle):
    layers, probs, packs_ref = [], [], []
    for (N, K) in wl.DECODE_SHAPES:
        W_np = wl.decode(N, K, 1).W
        W = torch.from_numpy(W_np).to(DEV)
        c_ref, s_ref, _ = oracle.pack(W_np, S=3)
        for T in wl.DECODE_TOKENS:
            L = wl.decode(N, K, T)
            codes, sz = mobi.mobi_pack(W, S=3)
            layers.append(L)
            packs_ref.append((c_ref, s_ref))
            probs.append({"X": L.X.to(DEV), "Wr": torch.from_numpy(L.Wr).to(DEV), "bias": None, "codes": codes,
                          "sz": sz, "N": N})
        del W
    outs = mobi.mobi_linear_grouped(probs)
    mobi.mobi_sync_check()
    for L, pr, (c_ref, s_ref), (Y, k_t, perm, off) in zip(layers, probs, packs_ref, outs):
        tag = f"headline {L.N}x{L.K} T={L.T}"
        assert np.array_equal(pr["codes"].cpu().numpy().view(np.uint32), c_ref), tag
        assert np.array_equal(pr["sz"].cpu().numpy().view(np.uint32), s_ref), tag
        k_gpu = k_t.cpu().numpy()
        k_ref, gap, _ = oracle.route(L.X, L.Wr)
        check_route(k_gpu, k_ref, gap, tag)
        perm_ref, off_ref = oracle.bucket(k_gpu, 3)
        assert np.array_equal(perm.cpu().numpy(), perm_ref) and np.array_equal(off.cpu().numpy(), off_ref), tag
        check_gemm(Y.cpu().numpy(), oracle.gemm(L.X, k_gpu, c_ref, s_ref, L.N), tag)
        Ys, ks, _, _ = mobi.mobi_linear(pr["X"], pr["Wr"], None, pr["codes"], pr["sz"], pr["N"])
        mobi.mobi_sync_check()
        assert torch.equal(Y, Ys) and torch.equal(k_t, ks), tag
