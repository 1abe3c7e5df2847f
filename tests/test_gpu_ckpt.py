"""Checkpoints on the GPU: packed layers saved from device memory and loaded
back at every slice count, and GEMMs run on a checkpoint loaded at k slices.

A layer loaded at k slices is a packed array with S = k. For tokens that use
at most k slices the GEMM on it must equal, bit for bit, the GEMM on the full
three-slice pack (the kernels read the same slices in the same order), and
both must meet the oracle bars.
"""
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
    assert torch.cuda.is_available()
    m.lib()
    return m


def test_device_round_trip(mobi, tmp_path):
    layers = [wl.layer(f"l{i}", N, K, 1, seed=1600 + i) for i, (N, K) in enumerate([(256, 512), (1024, 4096),
                                                                                      (512, 11008)])]
    packs = [mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), S=3) for L in layers]
    path = tmp_path / "dev.mobi"
    mobi.mobi_ckpt_save(path, [(f"proj{i}", c, z) for i, (c, z) in enumerate(packs)])
    with mobi.MobiCheckpoint(path) as ck:
        for i, (c, z) in enumerate(packs):
            for k in (1, 2, 3):
                cd, zd = ck.load(f"proj{i}", k, device=DEV)
                assert torch.equal(cd, c[:k]) and torch.equal(zd, z[:k])
            ch, zh = ck.load(f"proj{i}", 2)  # to host memory
            assert torch.equal(ch, c[:2].cpu()) and torch.equal(zh, z[:2].cpu())


@pytest.mark.parametrize("T", [4, 64])
def test_gemm_from_partial_load(mobi, oracle, tmp_path, T):
    N, K = 1024, 2048
    L = wl.layer("ck", N, K, T, seed=1700 + T)
    codes, sz = mobi.mobi_pack(torch.from_numpy(L.W).to(DEV), S=3)
    path = tmp_path / "layer.mobi"
    mobi.mobi_ckpt_save(path, [("layer", codes, sz)])
    X = L.X.to(DEV)
    rng = np.random.default_rng(T)
    with mobi.MobiCheckpoint(path) as ck:
        for k in (1, 2):
            ck_codes, ck_sz = ck.load("layer", k, device=DEV)
            k_np = rng.integers(1, k + 1, T).astype(np.int32)  # every token within the loaded precision
            perm_np, off_k = oracle.bucket(k_np, k)
            _, off_3 = oracle.bucket(k_np, 3)
            k_t = torch.from_numpy(k_np).to(DEV)
            perm = torch.from_numpy(perm_np).to(DEV)
            Y_k = mobi.mobi_gemm(X, k_t, perm, torch.from_numpy(off_k).to(DEV), ck_codes, ck_sz, N)
            Y_3 = mobi.mobi_gemm(X, k_t, perm, torch.from_numpy(off_3).to(DEV), codes, sz, N)
            mobi.mobi_sync_check()
            assert torch.equal(Y_k, Y_3), f"k={k} T={T}"
            c = ck_codes.cpu().numpy().view(np.uint32)
            s = ck_sz.cpu().numpy().view(np.uint32)
            check_gemm(Y_k.cpu().numpy(), oracle.gemm(L.X, k_np, c, s, N, S=k), f"checkpoint k={k} T={T}")
