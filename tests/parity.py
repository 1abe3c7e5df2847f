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


def check_route(k_gpu: np.ndarray, k_ref: np.ndarray, gap_ref: np.ndarray, what: str = "") -> int:
    diff = np.nonzero(np.asarray(k_gpu) != np.asarray(k_ref))[0]
    near = gap_ref[diff] < TIE_BAND
    assert np.all(near), f"{what}: routing differs at tokens {diff[~near][:10]} with gaps {gap_ref[diff][~near][:10]}"
    return int(diff.size)
