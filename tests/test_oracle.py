"""Pins of the CPU oracle against things other than itself.

The MoBiQuant explainer pages print no worked numeric example, so each oracle
function is pinned by (a) groups whose quantisation is derived by hand below
(closed forms), (b) library routines for special cases (torch's fake-quantise
and MinMax observer for one round of asymmetric min-max RTN, numpy fp64 matmul
and argmax, numpy stable argsort), (c) invariants of the recursion of
[ja] §2.1 / [en] §2.A (R_{s+1} = R_s - Q(R_s): the residual never grows, a
rounding error stays within half a step) and (d) brute force on tiny shapes.
"""
import numpy as np
import pytest
import torch

from token_adaptive_mixed_b200 import workloads as wl

F16 = np.float16


def f16_bits(x: float) -> int:
    return int(np.array([x], F16).view(np.uint16)[0])


def group_row(pattern, G=128):
    """One fp16 row of G weights repeating `pattern`."""
    vals = np.array([pattern[i % len(pattern)] for i in range(G)], np.float64)
    W = vals.astype(F16)
    assert np.all(W.astype(np.float64) == vals), "pattern must be fp16-exact"
    return W.reshape(1, G)


# ---- (a) closed-form groups --------------------------------------------------

def test_exact_grid_group(oracle):
    """Values {-1,0,1,2} * 2^-5: range 3*2^-5, so the step is exactly 2^-5 and
    zero = rint(1) = 1; codes are 0,1,2,3 repeated and slice 1 is exact. The
    residual is 0, so slices 2 and 3 see a degenerate group: step floored to
    2^-14 (fp16 0x0400), zero 0, all codes 0."""
    s = 2.0 ** -5
    W = group_row([-s, 0.0, s, 2 * s])
    codes, sz, q = oracle.pack(W, S=3)
    assert np.all(codes[0] == 0xE4E4E4E4)        # fields 0,1,2,3 -> 0b11100100 per byte
    assert np.all(sz[0] == (f16_bits(s) | (f16_bits(1.0) << 16)))
    assert np.all(codes[1:] == 0)
    assert np.all(sz[1:] == 0x0400)              # scale 2^-14, zero +0
    W1 = oracle.reconstruct(codes, sz, 1, 128, k=1)
    assert np.array_equal(W1, W.astype(np.float64))


def test_rounding_ties_and_clamps(oracle):
    """Values {-1.5,-0.5,0.5,1.5}/16, derived by hand:
    slice 1: step 1/16 (0x2C00), zero rint(1.5)=2 (ties to even), R/step rounds
      to {-2,-0,0,2} -> codes {0,2,2,3} (4 clamps to 3) -> byte 0xE8;
      residual {1,-1,1,1}/32.
    slice 2: (2/32)/3 = 1/48 rounds in fp16 to 1365/65536 (0x2555); zero
      rint(2048/1365)=2; R/step = +-1.50037 -> +-2 -> codes {3,0,3,3} -> 0xF3;
      residual {683,682,683,683}/65536.
    slice 3: range 1/65536 -> step floored to 2^-14; zero rint(-170.5) = -170
      clamps to 0; R/step = 170.75 / 170.5 -> codes all 3 (clamped) -> 0xFF."""
    W = group_row([-1.5 / 16, -0.5 / 16, 0.5 / 16, 1.5 / 16])
    codes, sz, q = oracle.pack(W, S=3)
    assert np.all(codes[0] == 0xE8E8E8E8)
    assert np.all(sz[0] == (0x2C00 | (f16_bits(2.0) << 16)))
    assert np.all(codes[1] == 0xF3F3F3F3)
    assert np.all(sz[1] == (0x2555 | (f16_bits(2.0) << 16)))
    assert np.all(codes[2] == 0xFFFFFFFF)
    assert np.all(sz[2] == 0x0400)
    W2 = oracle.reconstruct(codes, sz, 1, 128, k=2)
    resid = W.astype(np.float64) - W2
    expect = np.array([683, 682, 683, 683] * 32, np.float64) / 65536
    assert np.array_equal(resid.ravel(), expect)
    W3 = oracle.reconstruct(codes, sz, 1, 128, k=3)
    expect3 = np.array([671, 670, 671, 671] * 32, np.float64) / 65536
    assert np.array_equal((W.astype(np.float64) - W3).ravel(), expect3)


def test_all_negative_group(oracle):
    """Values {-4,-3,-2,-1}/64: step 1/64 (0x2400), zero rint(4) = 4 -> clamps
    to 3 (0x4200); codes {0,0,1,2} (byte 0x90); residual {-1,0,0,0}/64.
    slice 2: step fp16(1/192) = 1365/262144, zero rint(3.0007) = 3, codes
    {0,3,3,3} (byte 0xFC); residual {-1,0,0,0}/262144.
    slice 3: step 2^-14, zero rint(1/16) = 0, codes all 0."""
    W = group_row([-4 / 64, -3 / 64, -2 / 64, -1 / 64])
    codes, sz, _ = oracle.pack(W, S=3)
    assert np.all(codes[0] == 0x90909090)
    assert np.all(sz[0] == (0x2400 | (0x4200 << 16)))
    assert np.all(codes[1] == 0xFCFCFCFC)
    assert np.all(sz[1] == (f16_bits(1365 / 262144) | (0x4200 << 16)))
    assert f16_bits(1365 / 262144) == 0x1D55
    assert np.all(codes[2] == 0)
    assert np.all(sz[2] == 0x0400)
    W3 = oracle.reconstruct(codes, sz, 1, 128, k=3)
    expect = np.array([-1, 0, 0, 0] * 32, np.float64) / 262144
    assert np.array_equal((W.astype(np.float64) - W3).ravel(), expect)


def test_constant_positive_group(oracle):
    """A constant group c = 1: range 0 -> step 2^-14, zero clamps to 0, every
    code clamps to 3, so each slice removes exactly 3 * 2^-14."""
    W = group_row([1.0])
    codes, sz, _ = oracle.pack(W, S=3)
    assert np.all(codes == 0xFFFFFFFF)
    assert np.all(sz == 0x0400)
    for k in (1, 2, 3):
        Wk = oracle.reconstruct(codes, sz, 1, 128, k=k)
        assert np.all(Wk == 3 * k * 2.0 ** -14)


def test_packed_word_bit_order(oracle):
    """Code of k = 16w + i sits in bits [2i+1:2i] of word w: a row whose slice-1
    codes are 3 only at k = 5 and k = 16+15 gives words 0x00000C00 and 0xC0000000."""
    s = 2.0 ** -4
    vals = np.zeros(128)
    vals[:] = 0.0
    vals[5] = 3 * s
    vals[31] = 3 * s
    # min 0, max 3s -> step s, zero 0: codes are 3 at k=5, 31 and 0 elsewhere.
    W = vals.astype(F16).reshape(1, 128)
    codes, sz, q = oracle.pack(W, S=1)
    assert codes[0, 0, 0] == 0x00000C00
    assert codes[0, 0, 1] == 0xC0000000
    assert np.all(codes[0, 0, 2:] == 0)
    assert np.array_equal(oracle.unpack(codes, 1, 128, 1), q)


# ---- (b) library special cases -----------------------------------------------

def _random_W(N, K, seed, outliers=4):
    return wl.draw_weights(np.random.default_rng(seed), N, K, 0.02, outliers)


def test_slice1_matches_torch_fake_quantize(oracle):
    """Slice 1 is one round of asymmetric RTN: given the oracle's per-group
    scale and zero, torch.fake_quantize_per_channel_affine (round half to even,
    clamp to [0,3]) must give the oracle's dequantised slice bit for bit."""
    N, K = 64, 512
    W = _random_W(N, K, 11)
    codes, sz, q = oracle.pack(W, S=1)
    scale = (sz[0].T & 0xFFFF).astype(np.uint16).view(F16).astype(np.float32).ravel()
    zero = (sz[0].T >> 16).astype(np.uint16).view(F16).astype(np.float32).ravel().astype(np.int32)
    x = torch.from_numpy(W.astype(np.float32).reshape(N * K // 128, 128))
    fq = torch.fake_quantize_per_channel_affine(x, torch.from_numpy(scale), torch.from_numpy(zero), 0, 0, 3)
    W1 = oracle.reconstruct(codes, sz, N, K, k=1, S=1)
    assert np.array_equal(fq.numpy().astype(np.float64).reshape(N, K), W1)


def test_scale_matches_torch_minmax_observer(oracle):
    """For a group holding both signs, torch's MinMax observer (quint8 with
    quant range [0,3]) computes the step (max - min)/3 in fp32; rounded to fp16
    it is the oracle's stored slice-1 scale."""
    from torch.ao.quantization.observer import MinMaxObserver
    N, K = 8, 256
    W = _random_W(N, K, 12)
    codes, sz, _ = oracle.pack(W, S=1)
    for n in range(N):
        for g in range(K // 128):
            grp = torch.from_numpy(W[n, g * 128:(g + 1) * 128].astype(np.float32))
            assert grp.min() < 0 < grp.max()
            obs = MinMaxObserver(dtype=torch.quint8, quant_min=0, quant_max=3)
            obs(grp)
            sc, _ = obs.calculate_qparams()
            assert f16_bits(float(sc.to(torch.float16))) == int(sz[0, g, n] & 0xFFFF)


# ---- (c) invariants ------------------------------------------------------------

def test_residual_never_grows(oracle):
    """0 is always on the grid (integer zero in [0,3]) and clamping moves toward
    it, so |W - W^(k+1)| <= |W - W^(k)| element by element (up to the fp32
    rounding of the residual), and the Frobenius error falls with k."""
    N, K = 128, 1024
    W = _random_W(N, K, 13, outliers=8)
    codes, sz, _ = oracle.pack(W, S=3)
    Wd = W.astype(np.float64)
    errs = [np.abs(Wd)]
    fro = [np.linalg.norm(Wd)]
    for k in (1, 2, 3):
        e = np.abs(Wd - oracle.reconstruct(codes, sz, N, K, k=k))
        errs.append(e)
        fro.append(np.linalg.norm(e))
    for a, b in zip(errs[:-1], errs[1:]):
        assert np.all(b <= a + 1e-6 * np.abs(Wd) + 1e-9)
    assert fro[1] < fro[0] and fro[2] < fro[1] and fro[3] < fro[2]
    rel = [f / fro[0] for f in fro[1:]]
    assert rel[2] < 0.2 * rel[0]


def test_half_step_bound(oracle):
    """Where a group holds both signs and no code clamps, slice s leaves each
    element within half a step (plus the gap left when the fp16 step times 3
    falls short of the range)."""
    N, K = 64, 512
    W = _random_W(N, K, 14)
    codes, sz, q = oracle.pack(W, S=1)
    Wd = W.astype(np.float64).reshape(N, K // 128, 128)
    W1 = oracle.reconstruct(codes, sz, N, K, k=1, S=1).reshape(N, K // 128, 128)
    step = (sz[0].T & 0xFFFF).astype(np.uint16).view(F16).astype(np.float64)
    rng_ = Wd.max(-1) - Wd.min(-1)
    slack = np.maximum(rng_ - 3 * step, 0.0)
    err = np.abs(Wd - W1).max(-1)
    assert np.all(err <= step / 2 * (1 + 1e-6) + slack)


# ---- (d) routing, bucketing and GEMM -------------------------------------------

def test_route_brute_force(oracle):
    L = wl.layer("t", 16, 256, 64, seed=21)
    k, gap, logits = oracle.route(L.X, L.Wr)
    ref = L.X.to(torch.float64).numpy() @ L.Wr.astype(np.float64)
    assert np.allclose(logits, ref, rtol=0, atol=1e-12)
    assert np.array_equal(k, np.argmax(ref, axis=1) + 1)


def test_route_ties_and_dominant_column(oracle):
    T, K = 8, 128
    X = wl.to_bf16(np.ones((T, K), np.float32))
    Wr = np.zeros((K, 3), np.float32)
    k, gap, _ = oracle.route(X, Wr)                       # all logits equal: lowest index
    assert np.all(k == 1) and np.all(gap == 0)
    k, _, _ = oracle.route(X, Wr, np.array([0, 1, 1], np.float32))   # tie between 2 and 3
    assert np.all(k == 2)
    Wr[:, 2] = 1.0                                        # column 3 dominates a positive x
    k, gap, _ = oracle.route(X, Wr)
    assert np.all(k == 3) and np.allclose(gap, K)


def test_bucket_is_stable_sort(oracle):
    rng = np.random.default_rng(5)
    for T in (0, 1, 7, 1000):
        k = rng.integers(1, 4, T).astype(np.int32)
        perm, off = oracle.bucket(k)
        assert np.array_equal(perm, np.argsort(k, kind="stable"))
        assert off[0] == 0 and off[3] == T
        for j in range(3):
            assert np.all(k[perm[off[j]:off[j + 1]]] == j + 1)


def test_gemm_brute_force(oracle):
    """Y = x_t . W^(k_t)^T: against numpy fp64 matmul of the per-k reconstructions."""
    N, K, T = 48, 384, 24
    W = _random_W(N, K, 31)
    rng = np.random.default_rng(32)
    X = wl.draw_activations(rng, T, K)
    k = rng.integers(1, 4, T).astype(np.int32)
    codes, sz, _ = oracle.pack(W, S=3)
    Y = oracle.gemm(X, k, codes, sz, N)
    Xd = X.to(torch.float64).numpy()
    for t in range(T):
        Wk = oracle.reconstruct(codes, sz, N, K, k=int(k[t]))
        ref = Wk @ Xd[t]
        assert np.allclose(Y[t], ref, rtol=1e-13, atol=1e-13)
    sub = np.array([3, 0, 17], np.int32)
    Ys = oracle.gemm(X, k, codes, sz, N, tokens=sub)
    assert np.array_equal(Ys, Y[sub])


def test_gemm_one_hot(oracle):
    """x = e_j picks column j of W^(k_t): checks the orientation of the product."""
    N, K = 32, 256
    W = _random_W(N, K, 41)
    codes, sz, _ = oracle.pack(W, S=3)
    cols = [0, 1, 127, 128, 255]
    X = np.zeros((len(cols), K), np.float32)
    for i, j in enumerate(cols):
        X[i, j] = 1.0
    k = np.array([1, 2, 3, 2, 1], np.int32)
    Y = oracle.gemm(wl.to_bf16(X), k, codes, sz, N)
    for i, j in enumerate(cols):
        assert np.array_equal(Y[i], oracle.reconstruct(codes, sz, N, K, k=int(k[i]))[:, j])


def test_tiny_workload_fractions_and_error(oracle):
    """The tiny workload: relative reconstruction error falls with each slice
    and the 2-slice error is well under the 1-slice one."""
    L = wl.tiny()
    codes, sz, _ = oracle.pack(L.W, S=3)
    Wd = L.W.astype(np.float64)
    rel = [np.linalg.norm(Wd - oracle.reconstruct(codes, sz, L.N, L.K, k=k)) / np.linalg.norm(Wd)
           for k in (1, 2, 3)]
    assert rel[0] > rel[1] > rel[2]
    assert rel[2] < 0.15


def test_golden_tiny_fixture(oracle):
    """The oracle reproduces its committed outputs on the tiny workload."""
    import os
    g = np.load(os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.npz"))
    L = wl.tiny()
    codes, sz, _ = oracle.pack(L.W, S=3)
    k, gap, _ = oracle.route(L.X, L.Wr, L.bias)
    perm, off = oracle.bucket(k)
    assert np.array_equal(codes, g["codes"]) and np.array_equal(sz, g["sz"])
    assert np.array_equal(k, g["k_t"]) and np.array_equal(perm, g["perm"]) and np.array_equal(off, g["offsets"])
    assert np.array_equal(oracle.gemm(L.X, k, codes, sz, L.N), g["Y"])


@pytest.mark.slow
def test_workload_mixes(oracle):
    """The bias solver gives the stated slice-count mixes on the prefill workloads."""
    L = wl.prefill()
    k, _, _ = oracle.route(L.X, L.Wr, L.bias)
    frac = np.bincount(k, minlength=4)[1:] / L.T
    assert np.all(np.abs(frac - 1 / 3) < 0.05), frac
    L = wl.skewed_prefill()
    k, _, _ = oracle.route(L.X, L.Wr, L.bias)
    frac = np.bincount(k, minlength=4)[1:] / L.T
    assert np.all(np.abs(frac - np.array([0.7, 0.2, 0.1])) < 0.04), frac


# ---- threshold routing with an MLP scorer ([ja] §2.2, [en] §2.B) ---------------------

def _mlp_case(T=6, K=256, H=32, S=3, seed=11):
    rng = np.random.default_rng(seed)
    X = wl.to_bf16(rng.standard_normal((T, K), dtype=np.float32))
    W1 = (rng.standard_normal((K, H)) / np.sqrt(K)).astype(np.float32)
    b1 = (rng.standard_normal(H) * 0.1).astype(np.float32)
    W2 = (rng.standard_normal((H, S - 1)) / np.sqrt(H)).astype(np.float32)
    b2 = (rng.standard_normal(S - 1) * 0.1).astype(np.float32)
    return X, W1, b1, W2, b2


def test_route_mlp_scores_match_torch(oracle):
    """Library pin: torch's fp64 linear layers with ReLU give the same scores."""
    X, W1, b1, W2, b2 = _mlp_case()
    _, _, scores = oracle.route_mlp(X, W1, b1, W2, b2, tau=1.0, delta=0.5)
    x = X.to(torch.float64)
    h = torch.nn.functional.relu(torch.nn.functional.linear(x, torch.from_numpy(W1).double().T,
                                                            torch.from_numpy(b1).double()))
    s = torch.nn.functional.linear(h, torch.from_numpy(W2).double().T, torch.from_numpy(b2).double())
    assert np.allclose(scores, s.numpy(), rtol=1e-12, atol=1e-12)


def test_route_mlp_constant_score_closed_form(oracle):
    """W2 = 0: the score is b2 for every token, so sigmoid(b2 / tau) > delta
    decides every token alike (closed form)."""
    X, W1, b1, _, _ = _mlp_case(T=5, S=3)
    W2 = np.zeros((W1.shape[1], 2), np.float32)
    # sigmoid(0.5) = 0.6225 and sigmoid(-0.5) = 0.3775
    k, _, _ = oracle.route_mlp(X, W1, b1, W2, np.array([0.5, -0.5], np.float32), tau=1.0, delta=0.5)
    assert k.tolist() == [2] * 5                 # first residual slice on, second off
    k, _, _ = oracle.route_mlp(X, W1, b1, W2, np.array([0.5, 0.5], np.float32), tau=1.0, delta=0.6)
    assert k.tolist() == [3] * 5                 # 0.6225 > 0.6 for both
    k, _, _ = oracle.route_mlp(X, W1, b1, W2, np.array([0.5, 0.5], np.float32), tau=1.0, delta=0.7)
    assert k.tolist() == [1] * 5                 # 0.6225 < 0.7
    k, _, _ = oracle.route_mlp(X, W1, b1, W2, np.array([0.5, 0.5], np.float32), tau=4.0, delta=0.55)
    assert k.tolist() == [1] * 5                 # sigmoid(0.5 / 4) = 0.5312 < 0.55: temperature matters

def test_route_mlp_delta_half_is_sign(oracle):
    """delta = 0.5: sigmoid(s / tau) > 1/2 exactly when s > 0, for any tau > 0."""
    X, W1, b1, W2, b2 = _mlp_case(T=40, S=3, seed=12)
    for tau in (0.3, 1.0, 7.0):
        k, _, scores = oracle.route_mlp(X, W1, b1, W2, b2, tau=tau, delta=0.5)
        assert np.array_equal(k, 1 + (scores > 0).sum(axis=1))


def test_route_mlp_monotone_in_delta(oracle):
    """[en] §2.B: raising delta activates fewer slices, never more."""
    X, W1, b1, W2, b2 = _mlp_case(T=64, S=3, seed=13)
    prev = None
    for delta in (0.05, 0.2, 0.4, 0.5, 0.6, 0.8, 0.95):
        k, _, _ = oracle.route_mlp(X, W1, b1, W2, b2, tau=0.5, delta=delta)
        if prev is not None:
            assert np.all(k <= prev)
        prev = k
    assert prev.min() >= 1


def test_route_mlp_brute_force_tiny(oracle):
    """Pure-Python loops on a tiny case."""
    import math
    X, W1, b1, W2, b2 = _mlp_case(T=3, K=8, H=3, S=3, seed=14)
    x = X.float().numpy().astype(np.float64)
    tau, delta = 0.7, 0.45
    k, _, _ = oracle.route_mlp(X, W1, b1, W2, b2, tau=tau, delta=delta)
    for t in range(3):
        h = [max(0.0, sum(x[t, kk] * float(W1[kk, i]) for kk in range(8)) + float(b1[i])) for i in range(3)]
        active = 0
        for j in range(2):
            sj = sum(h[i] * float(W2[i, j]) for i in range(3)) + float(b2[j])
            active += 1.0 / (1.0 + math.exp(-sj / tau)) > delta
        assert k[t] == 1 + active


def test_route_mlp_one_slice_and_bad_args(oracle):
    X, W1, b1, _, _ = _mlp_case(T=4, S=3)
    k, margin, _ = oracle.route_mlp(X, W1, b1, np.zeros((W1.shape[1], 0), np.float32), np.zeros(0, np.float32),
                                    tau=1.0, delta=0.5)
    assert k.tolist() == [1] * 4 and np.all(np.isinf(margin))
    with pytest.raises(ValueError):
        oracle.route_mlp(X, W1, b1, np.zeros((W1.shape[1], 2), np.float32), np.zeros(2, np.float32),
                         tau=0.0, delta=0.5)


# ---- generic slicings: b-bit slices over G-wide groups ------------------------

def test_pack_bits_two_is_the_method_packer(oracle):
    """The generic packer with 2-bit slices and G = 128 is the method's packer."""
    W = _random_W(32, 512, 21)
    c0, s0, q0 = oracle.pack(W, S=3)
    c1, s1, q1 = oracle.pack_bits(W, G=128, S=3, bits=2)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1) and np.array_equal(q0, q1)


@pytest.mark.parametrize("bits,G", [(1, 128), (1, 256), (2, 256), (2, 512), (1, 64)])
def test_generic_slice1_matches_torch_fake_quantize(oracle, bits, G):
    """Slice 1 of b-bit slicing over G-wide groups is one round of asymmetric
    min-max RTN with 2^b - 1 steps: torch's fake quantiser (quant range
    [0, 2^b - 1], round half to even) with the oracle's scale and zero gives the
    oracle's dequantised slice bit for bit."""
    N, K = 32, 1024
    W = _random_W(N, K, 22 + bits + G)
    codes, sz, q = oracle.pack_bits(W, G=G, S=1, bits=bits)
    assert q.max() <= (1 << bits) - 1
    scale = (sz[0].T & 0xFFFF).astype(np.uint16).view(F16).astype(np.float32).ravel()
    zero = (sz[0].T >> 16).astype(np.uint16).view(F16).astype(np.float32).ravel().astype(np.int32)
    x = torch.from_numpy(W.astype(np.float32).reshape(N * K // G, G))
    fq = torch.fake_quantize_per_channel_affine(x, torch.from_numpy(scale), torch.from_numpy(zero), 0, 0,
                                                (1 << bits) - 1)
    W1 = oracle.reconstruct(codes, sz, N, K, k=1, G=G, S=1, bits=bits)
    assert np.array_equal(fq.numpy().astype(np.float64).reshape(N, K), W1)


@pytest.mark.parametrize("bits", [1, 2])
def test_generic_scale_matches_torch_minmax_observer(oracle, bits):
    """torch's MinMax observer with quant range [0, 2^b - 1] computes the step
    (max - min) / (2^b - 1) in fp32; rounded to fp16 it is the stored scale, here
    over 256-wide groups."""
    from torch.ao.quantization.observer import MinMaxObserver
    N, K, G = 4, 512, 256
    W = _random_W(N, K, 30 + bits)
    codes, sz, _ = oracle.pack_bits(W, G=G, S=1, bits=bits)
    for n in range(N):
        for g in range(K // G):
            grp = torch.from_numpy(W[n, g * G:(g + 1) * G].astype(np.float32))
            obs = MinMaxObserver(dtype=torch.quint8, quant_min=0, quant_max=(1 << bits) - 1)
            obs(grp)
            sc, _ = obs.calculate_qparams()
            assert f16_bits(float(sc.to(torch.float16))) == int(sz[0, g, n] & 0xFFFF)


def test_one_bit_hand_group(oracle):
    """Derived by hand: a 128-group of -1 and 2 (alternating). Slice 1: step
    (2 - (-1)) / 1 = 3, zero rint(1/3) = 0, codes 0 for -1 and 1 for 2 (2/3 rounds
    to 1), residual -1 everywhere. Slice 2: a constant group, step floored at
    2^-14, zero clamped to 1, codes rint(-2^14) + 1 -> clamped to 0, so each
    residual moves by one step: -1 + 2^-14."""
    W = group_row([-1.0, 2.0])
    codes, sz, q = oracle.pack_bits(W, G=128, S=2, bits=1)
    assert int(sz[0, 0, 0]) == f16_bits(3.0) | (f16_bits(0.0) << 16)
    assert np.array_equal(q[0, 0], np.tile([0, 1], 64))
    # 1 bit per weight: 4 words per 128-group; word 0 holds k = 0..15 on the
    # even bits and k = 16..31 on the odd bits, and every odd k is 1.
    assert codes.shape == (2, 1, 4)
    assert int(codes[0, 0, 0]) == 0xCCCCCCCC
    assert int(sz[1, 0, 0]) == 0x0400 | (f16_bits(1.0) << 16)  # 2^-14, zero 1
    assert np.all(q[1, 0] == 0)
    W2 = oracle.reconstruct(codes, sz, 1, 128, k=2, G=128, S=2, bits=1)
    assert np.all(W2[0] == np.tile([0.0 - 2.0 ** -14, 3.0 - 2.0 ** -14], 64))


@pytest.mark.parametrize("bits,G", [(1, 128), (1, 256), (2, 256)])
def test_generic_residual_never_grows(oracle, bits, G):
    """0 is on the grid for any b (integer zero in [0, 2^b - 1]) and clamping
    moves toward it, so the residual never grows element by element and the
    Frobenius error falls with every slice (four 1-bit slices: 1 to 4 bits)."""
    N, K, S = 64, 1024, 4
    W = _random_W(N, K, 40 + bits + G, outliers=4)
    codes, sz, _ = oracle.pack_bits(W, G=G, S=S, bits=bits)
    Wd = W.astype(np.float64)
    prev, fro = np.abs(Wd), [np.linalg.norm(Wd)]
    for k in range(1, S + 1):
        e = np.abs(Wd - oracle.reconstruct(codes, sz, N, K, k=k, G=G, S=S, bits=bits))
        assert np.all(e <= prev + 1e-6 * np.abs(Wd) + 1e-9)
        prev = e
        fro.append(np.linalg.norm(e))
    assert all(b < a for a, b in zip(fro[:-1], fro[1:]))


def test_one_bit_words_hand_derived(oracle):
    """Derived by hand from the documented 1-bit layout: a 0/1 row quantises to
    itself in one 1-bit slice (step 1, zero 0), so ones at k = 0, 15, 16, 31,
    32 and 127 give word 0 = bits 0, 30, 1, 31 = 0xC0000003, word 1 = bit 0,
    word 2 = 0 and word 3 = bit 31 (k = 96 + 31)."""
    row = np.zeros(128, np.float32)
    row[[0, 15, 16, 31, 32, 127]] = 1.0
    W = row.astype(np.float16)[None, :]
    codes, sz, q = oracle.pack_bits(W, G=128, S=1, bits=1)
    assert int(sz[0, 0, 0]) == f16_bits(1.0)  # scale 1, zero 0
    assert [int(w) for w in codes[0, 0]] == [0xC0000003, 0x00000001, 0x00000000, 0x80000000]
    assert np.array_equal(oracle.unpack(codes, 1, 128, 1, bits=1)[0, 0], row.astype(np.uint8))


@pytest.mark.parametrize("S", [1, 4])
def test_one_bit_gemm_equals_two_bit_storage(oracle, S):
    """The same 1-bit codes stored in the 2-bit word layout (pinned above by
    hand words) give the same reconstruction and GEMM, bit for bit: the 1-bit
    reader only changes where a code is read from."""
    N, K, T = 24, 512, 5
    W = _random_W(N, K, 60 + S, outliers=3)
    codes1, sz, q = oracle.pack_bits(W, G=128, S=S, bits=1)
    assert codes1.shape == (S, N, K // 32)
    assert np.array_equal(oracle.unpack(codes1, N, K, S, bits=1), q)
    codes2 = np.zeros((S, N, K // 16), np.uint32)  # 2-bit layout: q(16w + i) in bits [2i+1 : 2i]
    for i in range(16):
        codes2 |= q[:, :, i::16].astype(np.uint32) << np.uint32(2 * i)
    for k in range(1, S + 1):
        assert np.array_equal(oracle.reconstruct(codes1, sz, N, K, k=k, S=S, bits=1),
                              oracle.reconstruct(codes2, sz, N, K, k=k, S=S, bits=2))
    rng = np.random.default_rng(S)
    X = torch.from_numpy(rng.standard_normal((T, K), dtype=np.float32)).to(torch.bfloat16)
    k_t = rng.integers(1, S + 1, T).astype(np.int32)
    assert np.array_equal(oracle.gemm(X, k_t, codes1, sz, N, S=S, bits=1), oracle.gemm(X, k_t, codes2, sz, N, S=S))


def test_pack_bits_rejects_bad_arguments(oracle):
    W = _random_W(4, 256, 50)
    for kw in ({"bits": 0}, {"bits": 3}, {"G": 96}):
        with pytest.raises(ValueError):
            oracle.pack_bits(W, **{"G": 128, "S": 2, "bits": 2, **kw})


# ---- slices of mixed widths in one layer ---------------------------------------

def test_mixed_uniform_widths_are_pack_bits(oracle):
    """One width for every slice is the uniform packer, bit for bit."""
    W = _random_W(32, 512, 70, outliers=2)
    for b in (1, 2):
        c1, s1, q1 = oracle.pack_bits(W, G=128, S=3, bits=b)
        c2, s2, q2 = oracle.pack_slices(W, (b, b, b), G=128)
        assert np.array_equal(c1.ravel(), c2) and np.array_equal(s1, s2) and np.array_equal(q1, q2)


def test_mixed_each_round_quantises_its_residual(oracle):
    """Widths (2, 1, 1, 2): round s is one asymmetric min-max RTN of the fp32
    residual left by rounds < s with 2^w_s - 1 steps. The residual is rebuilt
    here in fp32 from the oracle's own earlier codes, scales and zeros, then
    torch's fake quantiser (range [0, 2^w_s - 1], the oracle's scale and zero)
    and MinMax observer (its step, rounded to fp16) must give round s's
    dequantised slice and stored scale."""
    from torch.ao.quantization.observer import MinMaxObserver
    N, K, G, widths = 16, 512, 128, (2, 1, 1, 2)
    W = _random_W(N, K, 71, outliers=3)
    codes, sz, q = oracle.pack_slices(W, widths, G=G)
    R = W.astype(np.float32)
    for s, b in enumerate(widths):
        L = (1 << b) - 1
        scale = (sz[s].T & 0xFFFF).astype(np.uint16).view(F16).astype(np.float32)  # [N, K/G]
        zero = (sz[s].T >> 16).astype(np.uint16).view(F16).astype(np.float32)
        x = torch.from_numpy(R.reshape(N * K // G, G).copy())
        fq = torch.fake_quantize_per_channel_affine(x, torch.from_numpy(scale.ravel()),
                                                    torch.from_numpy(zero.ravel().astype(np.int32)), 0, 0, L)
        deq = (q[s].astype(np.float32) - np.repeat(zero, G, axis=1)) * np.repeat(scale, G, axis=1)
        assert np.array_equal(fq.numpy().reshape(N, K), deq), f"round {s}"
        for n in range(0, N, 5):
            for g in range(K // G):
                obs = MinMaxObserver(dtype=torch.quint8, quant_min=0, quant_max=L)
                obs(torch.from_numpy(R[n, g * G:(g + 1) * G].copy()))
                sc, _ = obs.calculate_qparams()
                assert f16_bits(float(sc.to(torch.float16))) == int(sz[s, g, n] & 0xFFFF)
        R = (R - deq).astype(np.float32)


def test_mixed_layout_is_slice_major(oracle):
    """Slice 0 of widths (2, 1, 1, 2) is the first N*K/16 words and equals a
    one-slice 2-bit pack; every slice unpacks to the codes of its round, and
    the layer's code words total N*K*(2+1+1+2)/32."""
    N, K, widths = 24, 1024, (2, 1, 1, 2)
    W = _random_W(N, K, 72)
    codes, sz, q = oracle.pack_slices(W, widths)
    assert codes.shape == (N * K * 6 // 32,)
    c0, s0, _ = oracle.pack_bits(W, G=128, S=1, bits=2)
    assert np.array_equal(codes[:N * K // 16], c0.ravel()) and np.array_equal(sz[:1], s0)
    assert np.array_equal(oracle.unpack(codes, N, K, 4, widths=widths), q)


def test_mixed_gemm_equals_two_bit_storage(oracle):
    """The same codes in the (hand-pinned) uniform 2-bit layout give the same
    reconstruction and GEMM bit for bit, and the error falls with every slice
    (2, 3, 4 and 6 bits)."""
    N, K, T, widths = 24, 512, 6, (2, 1, 1, 2)
    W = _random_W(N, K, 73, outliers=2)
    codes, sz, q = oracle.pack_slices(W, widths)
    codes2 = np.zeros((4, N, K // 16), np.uint32)
    for i in range(16):
        codes2 |= q[:, :, i::16].astype(np.uint32) << np.uint32(2 * i)
    Wd = W.astype(np.float64)
    fro = []
    for k in range(1, 5):
        Wk = oracle.reconstruct(codes, sz, N, K, k=k, S=4, widths=widths)
        assert np.array_equal(Wk, oracle.reconstruct(codes2, sz, N, K, k=k, S=4, bits=2))
        fro.append(np.linalg.norm(Wd - Wk))
    assert all(b < a for a, b in zip(fro[:-1], fro[1:]))
    rng = np.random.default_rng(9)
    X = torch.from_numpy(rng.standard_normal((T, K), dtype=np.float32)).to(torch.bfloat16)
    k_t = rng.integers(1, 5, T).astype(np.int32)
    assert np.array_equal(oracle.gemm(X, k_t, codes, sz, N, S=4, widths=widths),
                          oracle.gemm(X, k_t, codes2, sz, N, S=4, bits=2))
