"""GPU parity of mobi_linear_grouped (up to 8 decode-sized mobi_linear problems
in one step) against the CPU oracle, and against one mobi_linear call per
problem.

Each 32-row block of a problem is summed the same way whichever CTA takes it,
and chunk partials are added in chunk order, so the grouped outputs must equal
the separate calls' bit for bit. Oracle bars as in the other GEMM tests.
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


def make_problems(mobi, specs, seed0):
    layers, probs = [], []
    for i, (N, K, T) in enumerate(specs):
        L = wl.layer("grp", N, K, T, seed=seed0 + i, mix=(0.3, 0.3, 0.4), outlier_frac_cols=0.005)
        codes, sz = mobi.mobi_pack(torch.from_numpy(np.ascontiguousarray(L.W)).to(DEV), S=3)
        layers.append(L)
        probs.append({"X": L.X.to(DEV), "Wr": torch.from_numpy(L.Wr).to(DEV),
                      "bias": torch.from_numpy(L.bias).to(DEV), "codes": codes, "sz": sz, "N": N})
    return layers, probs


def check_against_separate(mobi, probs, outs):
    for pr, (Y, k_t, perm, off) in zip(probs, outs):
        Ys, ks, ps, os_ = mobi.mobi_linear(pr["X"], pr["Wr"], pr["bias"], pr["codes"], pr["sz"], pr["N"])
        mobi.mobi_sync_check()
        assert torch.equal(k_t, ks) and torch.equal(perm, ps) and torch.equal(off, os_)
        assert torch.equal(Y, Ys)


def check_against_oracle(oracle, layers, probs, outs, rows_cap=None):
    for L, pr, (Y, k_t, perm, off) in zip(layers, probs, outs):
        tag = f"grouped N={L.N} K={L.K} T={L.T}"
        k_gpu = k_t.cpu().numpy()
        k_ref, gap, _ = oracle.route(L.X, L.Wr, L.bias)
        check_route(k_gpu, k_ref, gap, tag)
        perm_ref, off_ref = oracle.bucket(k_gpu, 3)
        assert np.array_equal(perm.cpu().numpy(), perm_ref), tag
        assert np.array_equal(off.cpu().numpy(), off_ref), tag
        rows = np.arange(L.N)
        if rows_cap is not None and L.N > rows_cap:
            rows = np.sort(np.random.default_rng(L.N + L.T).choice(L.N, rows_cap, replace=False))
        c = pr["codes"].cpu().numpy().view(np.uint32)[:, rows]
        s = pr["sz"].cpu().numpy().view(np.uint32)[:, :, rows]
        check_gemm(Y.cpu().numpy()[:, rows], oracle.gemm(L.X, k_gpu, c, s, len(rows)), tag)


@pytest.mark.parametrize("specs", [
    [(256, 512, 1), (512, 2048, 4), (256, 1024, 9), (1024, 4096, 16)],          # both fragment classes
    [(48, 1152, 13), (80, 2176, 2), (256, 512, 16), (512, 1024, 8), (128, 4096, 5), (64, 128, 3),
     (96, 2304, 11), (256, 3072, 7)],                                            # eight problems, ragged
    [(1024, 4096, 1)],                                                           # a group of one
])
def test_grouped_small(mobi, oracle, specs):
    layers, probs = make_problems(mobi, specs, seed0=1200 + len(specs))
    outs = mobi.mobi_linear_grouped(probs)
    mobi.mobi_sync_check()
    check_against_oracle(oracle, layers, probs, outs)
    check_against_separate(mobi, probs, outs)


def test_grouped_llama_layer(mobi, oracle):
    """The seven projections of a Llama-2-7B layer at batch 8 in one step;
    64 sampled rows of each checked against the oracle."""
    specs = [(N, K, 8) for _, N, K in wl.LLAMA7B_PROJECTIONS]
    layers, probs = make_problems(mobi, specs, seed0=1300)
    outs = mobi.mobi_linear_grouped(probs)
    mobi.mobi_sync_check()
    check_against_oracle(oracle, layers, probs, outs, rows_cap=64)
    check_against_separate(mobi, probs, outs)


def test_grouped_with_empty_problem(mobi, oracle):
    layers, probs = make_problems(mobi, [(256, 1024, 4), (512, 2048, 16)], seed0=1400)
    empty = {"X": torch.empty((0, 1024), dtype=torch.bfloat16, device=DEV), "Wr": probs[0]["Wr"],
             "codes": probs[0]["codes"], "sz": probs[0]["sz"], "N": 256}
    outs = mobi.mobi_linear_grouped([probs[0], empty, probs[1]])
    mobi.mobi_sync_check()
    assert np.array_equal(outs[1][3].cpu().numpy(), [0, 0, 0, 0])
    check_against_oracle(oracle, layers, probs, [outs[0], outs[2]])


def test_grouped_repeated_in_a_graph(mobi, oracle):
    """Captured once in a CUDA graph and replayed: the problem table is a kernel
    parameter, so replays need no host work and give the same results."""
    layers, probs = make_problems(mobi, [(512, 2048, 4), (1024, 4096, 12), (256, 1024, 1)], seed0=1500)
    outs = mobi.mobi_linear_grouped(probs)
    probs = [dict(p, Y=o[0], k_t=o[1], perm=o[2], offsets=o[3]) for p, o in zip(probs, outs)]
    ws = torch.empty(max(mobi.mobi_linear_grouped_workspace_bytes(probs), 16), dtype=torch.uint8, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        mobi.mobi_linear_grouped(probs, ws=ws)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        mobi.mobi_linear_grouped(probs, ws=ws)
    for o in outs:
        o[0].zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    mobi.mobi_sync_check()
    check_against_oracle(oracle, layers, probs, outs)
    del graph


def test_gemm_grouped_equals_gemm_calls(mobi):
    """mobi_gemm_grouped (k_t given) equals one mobi_gemm call per problem bit for bit."""
    layers, probs = make_problems(mobi, [(256, 512, 2), (1024, 4096, 16), (512, 11008, 7), (64, 1024, 12)],
                                  seed0=1800)
    gprobs = []
    for pr in probs:
        k_t, perm, off = mobi.mobi_route(pr["X"], pr["Wr"], pr["bias"])
        gprobs.append({"X": pr["X"], "k_t": k_t, "perm": perm, "off": off, "codes": pr["codes"], "sz": pr["sz"],
                       "N": pr["N"]})
    Ys = mobi.mobi_gemm_grouped(gprobs)
    mobi.mobi_sync_check()
    for g, Y in zip(gprobs, Ys):
        Y1 = mobi.mobi_gemm(g["X"], g["k_t"], g["perm"], g["off"], g["codes"], g["sz"], g["N"])
        mobi.mobi_sync_check()
        assert torch.equal(Y, Y1)
