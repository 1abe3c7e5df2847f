"""Property tests on random shapes (CPU): invariants of the oracle's packer
that hold for every slicing, and checkpoint round trips of random layer sets.

Packer (the recursion R_1 = W, W_s = Q(R_s), R_{s+1} = R_s - W_s with Q the
b-bit asymmetric min-max RTN): codes lie in [0, 2^b - 1], zeros are integers
in that range, every stored scale is a normal fp16 >= 2^-14, the residual
never grows element by element, and a group whose values already sit on one
slice's grid is reproduced exactly by that slice.
"""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import token_adaptive_mixed_b200 as mobi
from token_adaptive_mixed_b200 import build as mobi_build

F16 = np.float16


@st.composite
def slicing(draw):
    bits = draw(st.sampled_from([1, 2]))
    G = draw(st.sampled_from([128, 256]))
    K = G * draw(st.integers(1, 3))
    N = draw(st.integers(1, 24))
    S = draw(st.integers(1, 4))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    scale = draw(st.sampled_from([1e-3, 0.02, 1.0, 40.0]))
    return bits, G, K, N, S, seed, scale


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(slicing())
def test_packer_invariants(oracle, case):
    bits, G, K, N, S, seed, scale = case
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * scale).astype(F16)
    codes, sz, q = oracle.pack_bits(W, G=G, S=S, bits=bits)
    L = (1 << bits) - 1
    assert q.max() <= L
    sc = (sz & 0xFFFF).astype(np.uint16).view(F16).astype(np.float64)
    zr = (sz >> 16).astype(np.uint16).view(F16).astype(np.float64)
    assert np.all(sc >= 2.0 ** -14) and np.all(np.isfinite(sc))
    assert np.all((zr == np.round(zr)) & (zr >= 0) & (zr <= L))
    # the documented word layout holds the unpacked codes
    assert np.array_equal(oracle.unpack(codes, N, K, S, bits=bits), q)
    Wd = W.astype(np.float64)
    prev = np.abs(Wd)
    for k in range(1, S + 1):
        err = np.abs(Wd - oracle.reconstruct(codes, sz, N, K, k=k, G=G, S=S, bits=bits))
        assert np.all(err <= prev + 1e-6 * np.abs(Wd) + 1e-12)
        prev = err


@settings(max_examples=25, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(st.integers(0, 2 ** 31 - 1), st.sampled_from([1, 2]), st.integers(0, 3))
def test_on_grid_group_is_exact(oracle, seed, bits, zshift):
    """Values z' + c * s for codes c in [0, L] (min and max present) are one
    slice's grid: slice 1 reproduces them exactly and leaves a zero residual."""
    L = (1 << bits) - 1
    rng = np.random.default_rng(seed)
    step = float(F16(2.0 ** rng.integers(-6, 3)))
    z = min(zshift, L)
    c = rng.integers(0, L + 1, 128)
    c[0], c[1] = 0, L
    W = ((c - z) * step).astype(F16).reshape(1, 128)
    codes, sz, q = oracle.pack_bits(W, G=128, S=2, bits=bits)
    assert np.array_equal(q[0, 0], c)
    W1 = oracle.reconstruct(codes, sz, 1, 128, k=1, G=128, S=2, bits=bits)
    assert np.array_equal(W1, W.astype(np.float64))


@pytest.fixture(scope="module")
def L():
    mobi_build.build()
    return mobi.lib()


@settings(max_examples=20, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(st.lists(st.tuples(st.integers(1, 6), st.integers(1, 4), st.integers(1, 4)), min_size=1, max_size=5),
       st.integers(0, 2 ** 31 - 1))
def test_checkpoint_round_trip(L, tmp_path_factory, layers, seed):
    rng = np.random.default_rng(seed)
    tensors, arrays = [], {}
    for i, (n16, kblocks, S) in enumerate(layers):
        N, K = 16 * n16, 128 * kblocks
        codes = rng.integers(0, 2 ** 32, (S, N, K // 16), dtype=np.uint64).astype(np.uint32).view(np.int32)
        sz = rng.integers(0, 2 ** 32, (S, K // 128, N), dtype=np.uint64).astype(np.uint32).view(np.int32)
        name = f"layer{i}.proj"
        tensors.append((name, codes, sz))
        arrays[name] = (codes, sz, S)
    path = tmp_path_factory.mktemp("ck") / "m.mobi"
    mobi.mobi_ckpt_save(path, tensors)
    with mobi.MobiCheckpoint(path) as ck:
        assert ck.names() == [t[0] for t in tensors]
        for name, (codes, sz, S) in arrays.items():
            k = int(rng.integers(1, S + 1))
            c, z = ck.load(name, k)
            assert np.array_equal(c.numpy(), codes[:k]) and np.array_equal(z.numpy(), sz[:k])
