"""The C ABI loads and exports every function include/mobi.h declares; host-side
validation returns the documented status before anything reaches CUDA.

These tests run without a GPU: the calls below fail validation (bad shape,
null or misaligned pointer, short workspace) and return before any CUDA call.
"""
import ctypes
import os
import re

import pytest

import token_adaptive_mixed_b200 as mobi
from token_adaptive_mixed_b200 import build as mobi_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    mobi_build.build()
    return mobi.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mobi.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mobi_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert sorted(mobi.EXPORTED_SYMBOLS) == names


def test_status_strings_and_sizes(L):
    assert mobi.mobi_status_string(0) == "MOBI_OK"
    assert mobi.mobi_status_string(6) == "MOBI_ERR_TIMEOUT"
    assert mobi.mobi_status_string(7) == "MOBI_ERR_IO"
    assert [mobi.mobi_status_string(i) for i in range(8)] == mobi.STATUS_NAMES
    assert mobi.mobi_codes_bytes(4096, 4096, 4) == 4 * 4096 * 256 * 4  # four slices (generic slicing)
    assert mobi.mobi_codes_bytes(4096, 4096, 5) == 0
    assert mobi.mobi_version() >= 100
    assert mobi.mobi_codes_bytes(4096, 4096, 3) == 3 * 4096 * 256 * 4
    assert mobi.mobi_sz_bytes(4096, 4096, 3, 128) == 3 * 4096 * 32 * 4
    assert mobi.mobi_codes_bytes(16, 100, 3) == 0  # K % 32 != 0
    assert mobi.mobi_codes_bytes(4096, 4096, 4, bits=1) == 4 * 4096 * 128 * 4  # 1-bit codes: 32 per word
    assert L.mobi_codes_bytes_bits(4096, 4096, 3, 3) == 0
    assert mobi.mobi_codes_bytes(4096, 4096, widths=(2, 1, 1, 2)) == 4096 * 4096 * 6 // 8  # 2+1+1+2 bits
    assert mobi.mobi_codes_bytes(4096, 4096, widths=(2, 3)) == 0
    assert mobi.mobi_gemm_workspace_bytes(16, 4096, 4096, 3) > 0


FAKE = 1 << 20  # a 16-byte-aligned non-null address; never dereferenced: validation fails first


def test_pack_validation(L):
    p = ctypes.c_void_p
    assert L.mobi_pack(p(FAKE), 16, 100, 128, 3, p(FAKE), p(FAKE), None) == 2   # K % 128
    assert L.mobi_pack(p(FAKE), 24, 128, 128, 3, p(FAKE), p(FAKE), None) == 2   # N % 16
    assert L.mobi_pack(p(FAKE), 16, 128, 64, 3, p(FAKE), p(FAKE), None) == 2    # G != 128
    assert L.mobi_pack(p(FAKE), 16, 128, 128, 5, p(FAKE), p(FAKE), None) == 1   # S > 4
    assert L.mobi_pack(None, 16, 128, 128, 3, p(FAKE), p(FAKE), None) == 1      # null W
    assert L.mobi_pack(p(FAKE + 2), 16, 128, 128, 3, p(FAKE), p(FAKE), None) == 3  # misaligned
    assert L.mobi_pack(p(FAKE), 0, 128, 128, 3, p(FAKE), p(FAKE), None) == 0    # empty: no-op


def test_route_validation(L):
    p = ctypes.c_void_p
    args = lambda X=p(FAKE), T=16, K=256, S=3, ws=None, wsb=0: (X, T, K, p(FAKE), None, S, p(FAKE), p(FAKE),
                                                                 p(FAKE), ws, wsb, None)
    assert L.mobi_route(*args(K=100)) == 2
    assert L.mobi_route(*args(S=0)) == 1
    assert L.mobi_route(*args(X=None)) == 1
    assert L.mobi_route(*args(X=p(FAKE + 8))) == 3
    T, K = 32, 4096  # two token tiles: K is split, which needs a workspace
    assert mobi.mobi_route_workspace_bytes(T, K, 3) > 0
    assert L.mobi_route(*args(T=T, K=K)) == 4
    assert mobi.mobi_route_workspace_bytes(16, K, 3) == 0  # up to 16 tokens: one cluster launch, no workspace


def test_gemm_validation(L):
    p = ctypes.c_void_p

    def call(T=16, K=256, N=64, S=3, G=128, ws=p(FAKE), wsb=1 << 30, path=0, X=p(FAKE), Y=p(FAKE)):
        return L.mobi_gemm_path(X, T, K, p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), N, G, S, Y, ws, wsb,
                                None, path)
    assert call(K=200) == 2
    assert call(N=24) == 2
    assert call(G=32) == 2
    assert call(S=0) == 1
    assert call(path=7) == 1
    assert call(T=17, path=1) == 2        # decode kernel takes at most 16 tokens
    assert call(X=None) == 1
    assert call(Y=p(FAKE + 4)) == 3
    assert call(wsb=16) == 4
    assert call(T=0) == 0                 # nothing to do

    def call_bits(bits, T=16, K=256, N=64, S=3, G=128):
        return L.mobi_gemm_bits(p(FAKE), T, K, p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), N, G, S, bits, p(FAKE),
                                p(FAKE), 1 << 30, None, 0)
    assert call_bits(0) == 1 and call_bits(3) == 1   # code width 1 or 2
    assert call_bits(1, K=200) == 2
    assert call_bits(1, T=0) == 0
    prob = mobi.GemmProblem(p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), 4, 64, 256)
    assert L.mobi_gemm_grouped_bits(ctypes.byref(prob), 1, 128, 3, 4, p(FAKE), 1 << 30, None) == 1

    def call_slices(widths, T=16, K=256, N=64, S=None):
        w = mobi._int_array(widths)
        S = len(widths) if S is None else S
        return L.mobi_gemm_slices(p(FAKE), T, K, p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), N, 128, S, w,
                                  p(FAKE), p(FAKE), 1 << 30, None, 0)
    assert call_slices((2, 0, 1)) == 1 and call_slices((2, 3)) == 1 and call_slices((2, 1), S=5) == 1
    assert call_slices((2, 1), K=200) == 2
    assert call_slices((2, 1, 1, 2), T=0) == 0
    assert L.mobi_gemm_slices(p(FAKE), 16, 256, p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), 64, 128, 2, None,
                              p(FAKE), p(FAKE), 1 << 30, None, 0) == 1  # widths missing
    assert L.mobi_pack_slices(p(FAKE), 16, 256, 128, 2, mobi._int_array((2, 4)), p(FAKE), p(FAKE), None) == 1


def test_linear_validation(L):
    p = ctypes.c_void_p

    def call(T=16, K=256, N=64, S=3, G=128, ws=p(FAKE), wsb=1 << 30, X=p(FAKE), Y=p(FAKE), codes=p(FAKE)):
        return L.mobi_linear(X, T, K, p(FAKE), None, codes, p(FAKE), N, G, S, p(FAKE), p(FAKE), p(FAKE), Y, ws,
                             wsb, None)
    assert call(K=200) == 2
    assert call(N=24) == 2
    assert call(G=64) == 2
    assert call(S=5) == 1
    assert call(X=None) == 1
    assert call(codes=None) == 1
    assert call(Y=p(FAKE + 4)) == 3
    assert call(wsb=16) == 4
    T, N, K = 16, 4096, 4096
    assert mobi.mobi_linear_workspace_bytes(T, N, K, 3) >= mobi.mobi_gemm_workspace_bytes(T, N, K, 3)
    assert mobi.mobi_linear_workspace_bytes(64, N, K, 3) >= (mobi.mobi_route_workspace_bytes(64, K, 3)
                                                             + mobi.mobi_gemm_workspace_bytes(64, N, K, 3))


def test_workspace_sizes_edge_cases(L):
    assert mobi.mobi_route_workspace_bytes(0, 256, 3) == 0
    assert mobi.mobi_route_workspace_bytes(2048, 4096, 3) == 0   # many token tiles: no split
    assert mobi.mobi_gemm_workspace_bytes(0, 0, 0, 3) >= 0


def test_route_mlp_validation(L):
    """Every rejection happens on the host, before a launch (no GPU needed)."""
    p = ctypes.c_void_p

    def call(T=16, K=256, H=128, S=3, tau=1.0, delta=0.5, X=p(FAKE), W1=p(FAKE), W2=p(FAKE), ws=p(FAKE),
             wsb=1 << 30, perm=p(FAKE)):
        return L.mobi_route_mlp(X, T, K, W1, None, H, W2, None, S, tau, delta, p(FAKE), perm, p(FAKE), ws, wsb,
                                None)
    assert call(tau=0.0) == 1
    assert call(tau=-1.0) == 1
    assert call(tau=float("inf")) == 1
    assert call(tau=float("nan")) == 1
    assert call(delta=0.0) == 1
    assert call(delta=1.0) == 1
    assert call(delta=float("nan")) == 1
    assert call(S=0) == 1 and call(S=5) == 1
    assert call(H=0) == 1
    assert call(T=-1) == 1
    assert call(K=200) == 2
    assert call(H=65537) == 2
    assert call(X=None) == 1 and call(perm=None) == 1
    assert call(W1=None) == 1 and call(W2=None) == 1
    assert call(X=p(FAKE + 8)) == 3
    assert call(ws=p(FAKE + 8)) == 3
    assert call(W1=p(FAKE + 2)) == 3
    assert call(wsb=16) == 4
    assert call(ws=None, wsb=0) == 4
    for T, K, H in ((16, 4096, 128), (3, 128, 7), (2048, 4096, 128), (1, 128, 65536)):
        b = mobi.mobi_route_mlp_workspace_bytes(T, K, H)
        assert b >= T * H * 4 and b % 256 == 0, (T, K, H, b)
        assert b <= max(K // 64, 1) * T * H * 4 + 255  # at most one split per 64 rows of K
    assert mobi.mobi_route_mlp_workspace_bytes(0, 4096, 128) == 0
    assert mobi.mobi_route_mlp_workspace_bytes(16, 4096, 0) == 0


def test_linear_grouped_validation(L):
    P = mobi.LinearProblem

    def prob(T=8, N=4096, K=4096, X=FAKE, Y=FAKE, codes=FAKE):
        return P(X, FAKE, None, codes, FAKE, Y, FAKE, FAKE, FAKE, T, N, K)

    def call(probs, S=3, G=128, ws=FAKE, wsb=1 << 30):
        arr = (P * max(len(probs), 1))(*probs)
        return L.mobi_linear_grouped(arr if probs else None, len(probs), G, S, ws, wsb, None)
    assert call([]) == 1
    assert call([prob()] * 17) == 1                 # more than MOBI_MAX_GROUP
    assert call([prob(), prob(T=17)]) == 2          # decode-sized problems only
    assert call([prob(), prob(K=200)]) == 2
    assert call([prob(), prob(N=24)]) == 2
    assert call([prob()], G=64) == 2
    assert call([prob()], S=5) == 1
    assert call([prob(), prob(X=None)]) == 1
    assert call([prob(), prob(codes=None)]) == 1
    assert call([prob(), prob(Y=FAKE + 4)]) == 3
    assert call([prob()], ws=FAKE + 8) == 3
    assert call([prob()], wsb=16) == 4
    arr = (P * 2)(prob(T=4, N=4096, K=4096), prob(T=16, N=11008, K=4096))
    need = L.mobi_linear_grouped_workspace_bytes(arr, 2, 3)
    per = [L.mobi_linear_grouped_workspace_bytes((P * 1)(arr[i]), 1, 3) for i in range(2)]
    assert need == sum(per) and all(b % 256 == 0 and b > 0 for b in per)
    assert L.mobi_linear_grouped_workspace_bytes(arr, 2, 5) == 0


def test_gemm_grouped_validation(L):
    P = mobi.GemmProblem

    def prob(T=8, N=4096, K=4096, X=FAKE, Y=FAKE, k_t=FAKE):
        return P(X, k_t, FAKE, FAKE, Y, T, N, K)

    def call(probs, S=3, G=128, ws=FAKE, wsb=1 << 30):
        arr = (P * max(len(probs), 1))(*probs)
        return L.mobi_gemm_grouped(arr if probs else None, len(probs), G, S, ws, wsb, None)
    assert call([]) == 1
    assert call([prob()] * 17) == 1
    assert call([prob(T=17)]) == 2
    assert call([prob(K=200)]) == 2
    assert call([prob(k_t=None)]) == 1
    assert call([prob(Y=FAKE + 4)]) == 3
    assert call([prob(k_t=FAKE + 2)]) == 3
    assert call([prob()], wsb=16) == 4
    arr = (P * 2)(prob(T=4), prob(T=16, N=11008))
    assert L.mobi_gemm_grouped_workspace_bytes(arr, 2, 3) == sum(
        L.mobi_gemm_grouped_workspace_bytes((P * 1)(arr[i]), 1, 3) for i in range(2))


def test_pack_bits_validation(L):
    p = ctypes.c_void_p

    def call(N=16, K=512, G=256, S=4, bits=1, W=p(FAKE), codes=p(FAKE)):
        return L.mobi_pack_bits(W, N, K, G, S, bits, codes, p(FAKE), None)
    assert call(bits=0) == 1 and call(bits=3) == 1
    assert call(S=5) == 1 and call(S=0) == 1
    assert call(G=64) == 2 and call(G=384) == 2
    assert call(K=384, G=256) == 2          # K % G
    assert call(N=24) == 2
    assert call(W=None) == 1 and call(codes=None) == 1
    assert call(W=p(FAKE + 2)) == 3
    assert call(N=0) == 0                   # empty: no-op
