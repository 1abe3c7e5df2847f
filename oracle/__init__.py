"""CPU oracle of the MoBiQuant token-routed mixed-bit linear layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the product package.

The arithmetic lives in ``mobi_oracle.c`` (plain C, fp32 quantiser, fp64
routing and GEMM); this module compiles it with gcc on first use and wraps it
with numpy arrays. See the C file's header for the sources it follows
(the MoBiQuant explainer pages, §2.1/§2.A MoBiSlice and §2.2/§2.B MoBiRoute)
and for the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mobi_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

# -ffp-contract=off: no fused multiply-add, so every fp32 operation of the
# quantiser rounds exactly once, as IEEE arithmetic written out.
CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/liboracle.so`` (if stale) and return its path."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            p = ctypes.c_void_p
            i64 = ctypes.c_int64
            ci = ctypes.c_int
            lib.oracle_pack.argtypes = [p, i64, i64, ci, ci, p, p, p, ci]
            lib.oracle_pack.restype = ci
            lib.oracle_unpack.argtypes = [p, i64, i64, ci, p]
            lib.oracle_unpack.restype = None
            lib.oracle_reconstruct.argtypes = [p, p, i64, i64, ci, ci, ci, p]
            lib.oracle_reconstruct.restype = None
            lib.oracle_route.argtypes = [p, i64, i64, p, p, ci, p, p, p, ci]
            lib.oracle_route.restype = None
            lib.oracle_pack_bits.argtypes = [p, i64, i64, ci, ci, ci, p, p, p, ci]
            lib.oracle_pack_bits.restype = ci
            lib.oracle_route_mlp.argtypes = [p, i64, i64, p, p, i64, p, p, ci, ctypes.c_double, ctypes.c_double,
                                             p, p, p, ci]
            lib.oracle_route_mlp.restype = ci
            lib.oracle_bucket.argtypes = [p, i64, ci, p, p]
            lib.oracle_bucket.restype = ci
            lib.oracle_gemm.argtypes = [p, i64, i64, p, p, p, i64, ci, ci, p, i64, p, ci]
            lib.oracle_gemm.restype = None
            lib.oracle_gemm_bits.argtypes = [p, i64, i64, p, p, p, i64, ci, ci, ci, p, i64, p, ci]
            lib.oracle_gemm_bits.restype = None
            lib.oracle_unpack_bits.argtypes = [p, i64, i64, ci, ci, p]
            lib.oracle_unpack_bits.restype = None
            lib.oracle_reconstruct_bits.argtypes = [p, p, i64, i64, ci, ci, ci, ci, p]
            lib.oracle_reconstruct_bits.restype = None
            lib.oracle_pack_slices.argtypes = [p, i64, i64, ci, ci, p, p, p, p, ci]
            lib.oracle_pack_slices.restype = ci
            lib.oracle_unpack_slices.argtypes = [p, i64, i64, ci, p, p]
            lib.oracle_unpack_slices.restype = None
            lib.oracle_reconstruct_slices.argtypes = [p, p, i64, i64, ci, ci, p, ci, p]
            lib.oracle_reconstruct_slices.restype = None
            lib.oracle_gemm_slices.argtypes = [p, i64, i64, p, p, p, i64, ci, ci, p, p, i64, p, ci]
            lib.oracle_gemm_slices.restype = None
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = ci
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """fp16 / bf16 arrays (numpy, or CPU torch tensors) travel as their uint16 bit patterns."""
    if hasattr(a, "element_size") and hasattr(a, "view"):  # a torch tensor
        import torch
        a = a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    return a.view(np.uint16) if a.dtype != np.uint16 else a


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def pack(W_f16: np.ndarray, G: int = 128, S: int = 3, nthreads: int = 0):
    """MoBiSlice packing. Returns (codes uint32 [S,N,K/16], sz uint32 [S,K/G,N], q uint8 [S,N,K])."""
    lib = _load()
    W = _u16(W_f16)
    N, K = W.shape
    codes = np.zeros((S, N, K // 16), np.uint32)
    sz = np.zeros((S, K // G, N), np.uint32)
    q = np.zeros((S, N, K), np.uint8)
    rc = lib.oracle_pack(_ptr(W), N, K, G, S, _ptr(codes), _ptr(sz), _ptr(q), nthreads)
    if rc != 0:
        raise ValueError("oracle_pack: unsupported arguments")
    return codes, sz, q


def pack_bits(W_f16: np.ndarray, G: int = 128, S: int = 3, bits: int = 2, nthreads: int = 0):
    """MoBiSlice packing with `bits`-bit slices (1 or 2) over G-wide groups.
    Returns (codes uint32 [S,N,K*bits/32], sz uint32 [S,K/G,N], q uint8 [S,N,K]):
    2-bit codes 16 per word, 1-bit codes 32 per word (documented layouts)."""
    lib = _load()
    W = _u16(W_f16)
    N, K = W.shape
    codes = np.zeros((S, N, K * bits // 32), np.uint32)
    sz = np.zeros((S, K // G, N), np.uint32)
    q = np.zeros((S, N, K), np.uint8)
    rc = lib.oracle_pack_bits(_ptr(W), N, K, G, S, bits, _ptr(codes), _ptr(sz), _ptr(q), nthreads)
    if rc != 0:
        raise ValueError("oracle_pack_bits: unsupported arguments")
    return codes, sz, q


def _widths(S: int, widths) -> np.ndarray:
    w = np.ascontiguousarray(widths, np.int32).reshape(-1)
    if w.shape[0] != S:
        raise ValueError("one width per slice")
    return w


def codes_words(N: int, K: int, widths) -> int:
    """32-bit words of the codes of slices of the given widths, stored one after another."""
    return sum(N * K * int(b) // 32 for b in widths)


def pack_slices(W_f16: np.ndarray, widths, G: int = 128, nthreads: int = 0):
    """MoBiSlice packing with slice s of widths[s]-bit codes (1 or 2), G-wide groups.
    Returns (codes uint32 flat [sum_s N*K*w_s/32], sz uint32 [S,K/G,N], q uint8 [S,N,K])."""
    lib = _load()
    W = _u16(W_f16)
    N, K = W.shape
    S = len(widths)
    w = _widths(S, widths)
    codes = np.zeros(codes_words(N, K, w), np.uint32)
    sz = np.zeros((S, K // G, N), np.uint32)
    q = np.zeros((S, N, K), np.uint8)
    if lib.oracle_pack_slices(_ptr(W), N, K, G, S, _ptr(w), _ptr(codes), _ptr(sz), _ptr(q), nthreads) != 0:
        raise ValueError("oracle_pack_slices: unsupported arguments")
    return codes, sz, q


def unpack(codes: np.ndarray, N: int, K: int, S: int, bits: int = 2, widths=None) -> np.ndarray:
    """Packed words -> codes uint8 [S,N,K] by the documented layout of `bits`-bit codes
    (or of slices of the given widths)."""
    lib = _load()
    codes = np.ascontiguousarray(codes, np.uint32)
    q = np.zeros((S, N, K), np.uint8)
    if widths is not None:
        lib.oracle_unpack_slices(_ptr(codes), N, K, S, _ptr(_widths(S, widths)), _ptr(q))
    else:
        lib.oracle_unpack_bits(_ptr(codes), N, K, S, bits, _ptr(q))
    return q


def reconstruct(codes: np.ndarray, sz: np.ndarray, N: int, K: int, k: int, G: int = 128, S: int = 3,
                bits: int = 2, widths=None) -> np.ndarray:
    """W^(k) = sum of the first k dequantised slices, fp64 [N,K]."""
    lib = _load()
    out = np.zeros((N, K), np.float64)
    c = _ptr(np.ascontiguousarray(codes, np.uint32))
    z = _ptr(np.ascontiguousarray(sz, np.uint32))
    if widths is not None:
        lib.oracle_reconstruct_slices(c, z, N, K, G, S, _ptr(_widths(S, widths)), k, _ptr(out))
    else:
        lib.oracle_reconstruct_bits(c, z, N, K, G, S, bits, k, _ptr(out))
    return out


def route(X_bf16: np.ndarray, Wr: np.ndarray, bias: np.ndarray | None = None, nthreads: int = 0):
    """Returns (k_t int32 [T], gap fp64 [T], logits fp64 [T,S])."""
    lib = _load()
    X = _u16(X_bf16)
    T, K = X.shape
    Wr = np.ascontiguousarray(Wr, np.float32)
    S = Wr.shape[1]
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    k = np.zeros(T, np.int32)
    gap = np.zeros(T, np.float64)
    logits = np.zeros((T, S), np.float64)
    lib.oracle_route(_ptr(X), T, K, _ptr(Wr), _ptr(b), S, _ptr(k), _ptr(gap), _ptr(logits), nthreads)
    return k, gap, logits


def route_mlp(X_bf16: np.ndarray, W1: np.ndarray, b1: np.ndarray, W2: np.ndarray, b2: np.ndarray, tau: float,
              delta: float, nthreads: int = 0):
    """Threshold routing with a 2-layer MLP scorer (S = W2.shape[1] + 1).
    Returns (k_t int32 [T], margin fp64 [T], scores fp64 [T, S-1])."""
    lib = _load()
    X = _u16(X_bf16)
    T, K = X.shape
    W1 = np.ascontiguousarray(W1, np.float32)
    H = W1.shape[1]
    b1 = np.ascontiguousarray(b1, np.float32)
    W2 = np.ascontiguousarray(W2, np.float32).reshape(H, -1)
    b2 = np.ascontiguousarray(b2, np.float32).reshape(-1)
    S = W2.shape[1] + 1
    k = np.zeros(T, np.int32)
    margin = np.zeros(T, np.float64)
    scores = np.zeros((T, max(S - 1, 1)), np.float64)
    if lib.oracle_route_mlp(_ptr(X), T, K, _ptr(W1), _ptr(b1), H, _ptr(W2), _ptr(b2), S, float(tau), float(delta),
                            _ptr(k), _ptr(margin), _ptr(scores), nthreads) != 0:
        raise ValueError("oracle_route_mlp: tau must be > 0 and delta in (0, 1)")
    return k, margin, scores[:, : S - 1]


def bucket(k_t: np.ndarray, S: int = 3):
    """Returns (perm int32 [T], offsets int32 [S+1])."""
    lib = _load()
    k_t = np.ascontiguousarray(k_t, np.int32)
    T = k_t.shape[0]
    perm = np.zeros(T, np.int32)
    offsets = np.zeros(S + 1, np.int32)
    if lib.oracle_bucket(_ptr(k_t), T, S, _ptr(perm), _ptr(offsets)) != 0:
        raise ValueError("oracle_bucket: k_t outside 1..S")
    return perm, offsets


def gemm(X_bf16: np.ndarray, k_t: np.ndarray, codes: np.ndarray, sz: np.ndarray, N: int,
         G: int = 128, S: int = 3, tokens: np.ndarray | None = None, nthreads: int = 0, bits: int = 2,
         widths=None) -> np.ndarray:
    """Y fp64 [len(tokens) or T, N] = x_t . W^(k_t)^T for the listed tokens (`bits`-bit codes,
    or slices of the given widths)."""
    lib = _load()
    X = _u16(X_bf16)
    T, K = X.shape
    k_t = np.ascontiguousarray(k_t, np.int32)
    tok = None if tokens is None else np.ascontiguousarray(tokens, np.int32)
    n_tok = T if tok is None else tok.shape[0]
    Y = np.zeros((n_tok, N), np.float64)
    c = _ptr(np.ascontiguousarray(codes, np.uint32))
    z = _ptr(np.ascontiguousarray(sz, np.uint32))
    if widths is not None:
        lib.oracle_gemm_slices(_ptr(X), T, K, _ptr(k_t), c, z, N, G, S, _ptr(_widths(S, widths)), _ptr(tok), n_tok,
                               _ptr(Y), nthreads)
    else:
        lib.oracle_gemm_bits(_ptr(X), T, K, _ptr(k_t), c, z, N, G, S, bits, _ptr(tok), n_tok, _ptr(Y), nthreads)
    return Y
