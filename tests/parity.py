"""Shared checks of the parity tests (tolerances of the acceptance bar)."""
import numpy as np

# GEMM: max |y - y_ref| <= 1e-2 (|y_ref| + 1e-3) element-wise and a relative
# Frobenius error <= 2e-3 against the oracle's fp64 result.
ELEM_RTOL = 1e-2
ELEM_FLOOR = 1e-3
FRO_TOL = 2e-3
# Routing: decisions must agree except where the oracle's top-two fp64 logit
# gap is below this band (counted and reported).
TIE_BAND = 1e-5


def check_gemm(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = "") -> dict:
    y_gpu = np.asarray(y_gpu, np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = ELEM_RTOL * (np.abs(y_ref) + ELEM_FLOOR)
    bad = int(np.count_nonzero(err > bound))
    fro = float(np.linalg.norm(y_gpu - y_ref) / max(np.linalg.norm(y_ref), 1e-300))
    stats = {"max_abs_err": float(err.max(initial=0.0)), "violations": bad, "rel_fro": fro,
             "worst_ratio": float((err / bound).max(initial=0.0))}
    assert bad == 0, f"{what}: {bad} elements outside the bound; {stats}"
    assert fro <= FRO_TOL, f"{what}: relative Frobenius error {fro}"
    return stats


CANARY_BITS = 0x7FC0DEAD  # a quiet-NaN pattern no kernel writes


def guarded_output(T: int, N: int, device: str = "cuda:0", pad: int = 64):
    """Y [T, N] fp32 inside a buffer with `pad` canary words on each side (pad a
    multiple of 4 keeps Y 16-byte aligned). Returns (Y, check) where check()
    asserts every canary word is unchanged: nothing was written outside Y."""
    import torch
    buf = torch.full((pad + T * N + pad,), CANARY_BITS, dtype=torch.int32, device=device)
    Y = buf[pad:pad + T * N].view(torch.float32).view(T, N)

    def check(what: str = ""):
        b = buf.cpu().numpy().view(np.uint32)
        head, tail = b[:pad], b[pad + T * N:]
        assert np.all(head == CANARY_BITS) and np.all(tail == CANARY_BITS), \
            f"{what}: writes outside Y (head {np.count_nonzero(head != CANARY_BITS)}, tail {np.count_nonzero(tail != CANARY_BITS)})"
    return Y, check


def check_route(k_gpu: np.ndarray, k_ref: np.ndarray, gap_ref: np.ndarray, what: str = "") -> int:
    diff = np.nonzero(np.asarray(k_gpu) != np.asarray(k_ref))[0]
    near = gap_ref[diff] < TIE_BAND
    assert np.all(near), f"{what}: routing differs at tokens {diff[~near][:10]} with gaps {gap_ref[diff][~near][:10]}"
    return int(diff.size)


# Threshold routing with an MLP scorer: first-order error bound of the
# kernel's fp32 arithmetic, per token and slice. The hidden sums run over k in
# index order within each contiguous split of K (splits of at least 32 rows),
# one rounding per fused multiply-add, each at most u times the running sum;
# the splits are then added in order. With P_ik the exact partial sums from
# k = 0 and M_i = max_k |P_ik|, a running sum inside a split is at most
# |P_ik| + M_i and a running sum of splits at most M_i, so
#   |dh_i| <= u (sum_k |P_ik| + (K + K/32) M_i + |P_iK + b1_i|)
# (ReLU does not enlarge it). The score adds this through |W2|, plus at most
# `depth` roundings of the second sum (per-thread sums over a strided share
# of H, a 5-level warp tree, the warps in order, the bias), each at most
# u (sum_i |h_i W2_ij| + |b2_j|). Twice that (for second-order terms) plus
# 1e-12 (1 + |thr|) for the oracle's sigmoid form of the test is the band
# outside which decisions must agree.
U32 = 2.0 ** -24


def mlp_score_bound(X: np.ndarray, W1: np.ndarray, b1: np.ndarray, W2: np.ndarray, b2: np.ndarray,
                    thr: float, tokens_per_block: int = 8) -> np.ndarray:
    X = np.asarray(X, np.float64)
    W1 = np.asarray(W1, np.float64)
    b1 = np.asarray(b1, np.float64)
    W2 = np.abs(np.asarray(W2, np.float64))
    b2 = np.abs(np.asarray(b2, np.float64))
    T, K = X.shape
    H = W1.shape[1]
    e_h = np.empty((T, H))
    h_abs = np.empty((T, H))
    for t0 in range(0, T, tokens_per_block):
        P = np.cumsum(X[t0:t0 + tokens_per_block, :, None] * W1[None], axis=1)  # [tb, K, H]
        absP = np.abs(P)
        final = P[:, -1, :] + b1
        e_h[t0:t0 + tokens_per_block] = U32 * (absP.sum(axis=1) + (K + K / 32) * absP.max(axis=1) + np.abs(final))
        h_abs[t0:t0 + tokens_per_block] = np.maximum(final, 0.0)
    depth = -(-H // 32) + 11
    bound = e_h @ W2 + U32 * depth * (h_abs @ W2 + b2)
    return 2.0 * bound + 1e-12 * (1.0 + abs(thr))


def check_route_mlp(k_gpu: np.ndarray, scores_ref: np.ndarray, bound: np.ndarray, thr: float,
                    what: str = "", max_undecided: float = 0.05) -> int:
    """k_t must lie between the counts of surely-active and possibly-active slices;
    returns the number of tokens with an undecided slice (at most max_undecided of T, or 2)."""
    d = scores_ref - thr
    k_lo = 1 + np.count_nonzero(d > bound, axis=1)
    k_hi = 1 + np.count_nonzero(d >= -bound, axis=1)
    k_gpu = np.asarray(k_gpu)
    bad = np.nonzero((k_gpu < k_lo) | (k_gpu > k_hi))[0]
    assert bad.size == 0, f"{what}: k_t outside the decided range at tokens {bad[:10]}: gpu {k_gpu[bad[:10]]}, " \
                          f"range [{k_lo[bad[:10]]}, {k_hi[bad[:10]]}]"
    undecided = int(np.count_nonzero(k_lo != k_hi))
    assert undecided <= max(2, max_undecided * len(k_gpu)), f"{what}: {undecided} undecided tokens"
    return undecided
