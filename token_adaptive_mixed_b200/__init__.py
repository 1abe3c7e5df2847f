"""token_adaptive_mixed_b200 — the MoBiQuant token-routed mixed-bit linear layer on B200.

A thin ctypes binding over ``libmobi.so`` (the C ABI declared in
``include/mobi.h``). Every function here only marshals torch tensors into
pointers, sizes and the current CUDA stream; all arithmetic runs in the
library's sm_100a kernels. There is no CPU fallback: if the library is missing
or a tensor is not on a CUDA device, the call raises (the checkpoint calls,
which move bytes between a file and memory, also take host tensors).

Entry points (same names as the C ABI; `bits=` selects the *_bits form and
`widths=` the *_slices form of a call):
  mobi_pack(W, S, G, bits, widths)  MoBiSlice packing   -> (codes, sz)
  mobi_route(X, Wr, bias)           MoBiRoute routing   -> (k_t, perm, offsets)
  mobi_route_mlp(X, W1, b1, W2, b2, tau, delta)  threshold routing, MLP scorer -> (k_t, perm, offsets)
  mobi_gemm(X, k_t, perm, offsets, codes, sz, N)         -> Y  (fp32)
  mobi_gemm_path(..., path)         the same with a forced kernel
  mobi_linear(X, Wr, bias, codes, sz, N)  route + GEMM in one call -> (Y, k_t, perm, offsets)
  mobi_linear_grouped(problems)     up to 16 decode-sized mobi_linear problems in one step
  mobi_gemm_grouped(problems)       the GEMM half of it (k_t given)
  mobi_ckpt_save / MobiCheckpoint   many-in-one checkpoint of packed layers (load any slice count)
  mobi_sync_check()                 sync + device-side error word
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MobiError", "lib", "mobi_version", "mobi_status_string", "mobi_codes_bytes", "mobi_sz_bytes",
    "mobi_route_workspace_bytes", "mobi_gemm_workspace_bytes", "mobi_pack", "mobi_route", "mobi_gemm", "mobi_last_error",
    "mobi_gemm_path", "mobi_sync_check", "mobi_debug_set_wait_limit", "mobi_gemm_decode_noalloc", "mobi_linear",
    "mobi_linear_workspace_bytes", "mobi_route_mlp", "mobi_route_mlp_workspace_bytes", "mobi_linear_grouped",
    "mobi_linear_grouped_workspace_bytes", "mobi_gemm_grouped", "mobi_gemm_grouped_workspace_bytes", "MAX_GROUP",
    "mobi_ckpt_save", "MobiCheckpoint", "mobi_crc32c",
    "PATH_AUTO",
    "PATH_DECODE",
    "PATH_PREFILL", "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MOBI_LIB", os.path.join(_HERE, "libmobi.so"))

PATH_AUTO, PATH_DECODE, PATH_PREFILL = 0, 1, 2
MAX_GROUP = 16  # MOBI_MAX_GROUP


class CkptTensor(ctypes.Structure):
    """mobi_ckpt_tensor (include/mobi.h)."""
    _fields_ = [("name", ctypes.c_char_p), ("codes", ctypes.c_void_p), ("sz", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("G", ctypes.c_int), ("S", ctypes.c_int)]


class GemmProblem(ctypes.Structure):
    """mobi_gemm_problem (include/mobi.h)."""
    _fields_ = [("X", ctypes.c_void_p), ("k_t", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("sz", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("T", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64)]


class LinearProblem(ctypes.Structure):
    """mobi_linear_problem (include/mobi.h): pointers and sizes of one problem."""
    _fields_ = [("X", ctypes.c_void_p), ("Wr", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("codes", ctypes.c_void_p), ("sz", ctypes.c_void_p), ("Y", ctypes.c_void_p),
                ("k_t", ctypes.c_void_p), ("perm", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("T", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]
STATUS_NAMES = ["MOBI_OK", "MOBI_ERR_INVALID_ARG", "MOBI_ERR_UNSUPPORTED_SHAPE", "MOBI_ERR_MISALIGNED",
                "MOBI_ERR_WORKSPACE", "MOBI_ERR_CUDA", "MOBI_ERR_TIMEOUT", "MOBI_ERR_IO"]

# Every symbol include/mobi.h declares.
EXPORTED_SYMBOLS = (
    "mobi_status_string", "mobi_last_error", "mobi_version", "mobi_codes_bytes", "mobi_sz_bytes", "mobi_route_workspace_bytes",
    "mobi_gemm_workspace_bytes", "mobi_pack", "mobi_route", "mobi_gemm", "mobi_gemm_path", "mobi_sync_check",
    "mobi_debug_set_wait_limit", "mobi_gemm_decode_noalloc", "mobi_linear", "mobi_linear_workspace_bytes",
    "mobi_route_mlp", "mobi_route_mlp_workspace_bytes", "mobi_linear_grouped", "mobi_linear_grouped_workspace_bytes",
    "mobi_gemm_grouped", "mobi_gemm_grouped_workspace_bytes",
    "mobi_ckpt_save", "mobi_ckpt_open", "mobi_ckpt_count", "mobi_ckpt_find", "mobi_ckpt_info", "mobi_ckpt_load",
    "mobi_ckpt_bytes_read", "mobi_ckpt_close", "mobi_crc32c", "mobi_pack_bits", "mobi_codes_bytes_bits",
    "mobi_gemm_bits", "mobi_gemm_grouped_bits", "mobi_linear_bits", "mobi_linear_grouped_bits",
    "mobi_codes_bytes_slices", "mobi_pack_slices", "mobi_gemm_slices", "mobi_linear_slices",
    "mobi_gemm_grouped_slices", "mobi_linear_grouped_slices",
)


class MobiError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else f"status {status}"
        super().__init__(f"{fn}: {name}" + (f" [{detail}]" if detail else ""))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmobi.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmobi.so not found at {LIB_PATH}; build it with "
                              f"`python -m token_adaptive_mixed_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        p, i64, ci, sz_t = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.mobi_status_string.argtypes = [ci]
        L.mobi_status_string.restype = ctypes.c_char_p
        L.mobi_last_error.argtypes = []
        L.mobi_last_error.restype = ctypes.c_char_p
        L.mobi_version.argtypes = []
        L.mobi_version.restype = ci
        L.mobi_codes_bytes.argtypes = [i64, i64, ci]
        L.mobi_codes_bytes.restype = sz_t
        L.mobi_codes_bytes_bits.argtypes = [i64, i64, ci, ci]
        L.mobi_codes_bytes_bits.restype = sz_t
        L.mobi_codes_bytes_slices.argtypes = [i64, i64, ci, p]
        L.mobi_codes_bytes_slices.restype = sz_t
        L.mobi_pack_slices.argtypes = [p, i64, i64, ci, ci, p, p, p, p]
        L.mobi_pack_slices.restype = ci
        L.mobi_gemm_slices.argtypes = [p, i64, i64, p, p, p, p, p, i64, ci, ci, p, p, p, sz_t, p, ci]
        L.mobi_gemm_slices.restype = ci
        L.mobi_linear_slices.argtypes = [p, i64, i64, p, p, p, p, i64, ci, ci, p, p, p, p, p, p, sz_t, p]
        L.mobi_linear_slices.restype = ci
        L.mobi_gemm_grouped_slices.argtypes = [p, ci, ci, ci, p, p, sz_t, p]
        L.mobi_gemm_grouped_slices.restype = ci
        L.mobi_linear_grouped_slices.argtypes = [p, ci, ci, ci, p, p, sz_t, p]
        L.mobi_linear_grouped_slices.restype = ci
        L.mobi_sz_bytes.argtypes = [i64, i64, ci, ci]
        L.mobi_sz_bytes.restype = sz_t
        L.mobi_route_workspace_bytes.argtypes = [i64, i64, ci]
        L.mobi_route_workspace_bytes.restype = sz_t
        L.mobi_gemm_workspace_bytes.argtypes = [i64, i64, i64, ci]
        L.mobi_gemm_workspace_bytes.restype = sz_t
        L.mobi_pack.argtypes = [p, i64, i64, ci, ci, p, p, p]
        L.mobi_pack.restype = ci
        L.mobi_pack_bits.argtypes = [p, i64, i64, ci, ci, ci, p, p, p]
        L.mobi_pack_bits.restype = ci
        L.mobi_route.argtypes = [p, i64, i64, p, p, ci, p, p, p, p, sz_t, p]
        L.mobi_route.restype = ci
        L.mobi_gemm.argtypes = [p, i64, i64, p, p, p, p, p, i64, ci, ci, p, p, sz_t, p]
        L.mobi_gemm.restype = ci
        L.mobi_gemm_path.argtypes = [p, i64, i64, p, p, p, p, p, i64, ci, ci, p, p, sz_t, p, ci]
        L.mobi_gemm_path.restype = ci
        L.mobi_gemm_bits.argtypes = [p, i64, i64, p, p, p, p, p, i64, ci, ci, ci, p, p, sz_t, p, ci]
        L.mobi_gemm_bits.restype = ci
        L.mobi_gemm_decode_noalloc.argtypes = [p, i64, i64, p, p, p, i64, ci, ci, p, p]
        L.mobi_gemm_decode_noalloc.restype = ci
        L.mobi_linear_workspace_bytes.argtypes = [i64, i64, i64, ci]
        L.mobi_linear_workspace_bytes.restype = sz_t
        L.mobi_linear.argtypes = [p, i64, i64, p, p, p, p, i64, ci, ci, p, p, p, p, p, sz_t, p]
        L.mobi_linear.restype = ci
        L.mobi_linear_bits.argtypes = [p, i64, i64, p, p, p, p, i64, ci, ci, ci, p, p, p, p, p, sz_t, p]
        L.mobi_linear_bits.restype = ci
        L.mobi_route_mlp_workspace_bytes.argtypes = [i64, i64, i64]
        L.mobi_route_mlp_workspace_bytes.restype = sz_t
        L.mobi_route_mlp.argtypes = [p, i64, i64, p, p, i64, p, p, ci, ctypes.c_double, ctypes.c_double, p, p, p,
                                     p, sz_t, p]
        L.mobi_route_mlp.restype = ci
        L.mobi_linear_grouped_workspace_bytes.argtypes = [p, ci, ci]
        L.mobi_linear_grouped_workspace_bytes.restype = sz_t
        L.mobi_linear_grouped.argtypes = [p, ci, ci, ci, p, sz_t, p]
        L.mobi_linear_grouped.restype = ci
        L.mobi_linear_grouped_bits.argtypes = [p, ci, ci, ci, ci, p, sz_t, p]
        L.mobi_linear_grouped_bits.restype = ci
        L.mobi_gemm_grouped_workspace_bytes.argtypes = [p, ci, ci]
        L.mobi_gemm_grouped_workspace_bytes.restype = sz_t
        L.mobi_gemm_grouped.argtypes = [p, ci, ci, ci, p, sz_t, p]
        L.mobi_gemm_grouped.restype = ci
        L.mobi_gemm_grouped_bits.argtypes = [p, ci, ci, ci, ci, p, sz_t, p]
        L.mobi_gemm_grouped_bits.restype = ci
        L.mobi_ckpt_save.argtypes = [ctypes.c_char_p, p, ci, ci, p]
        L.mobi_ckpt_save.restype = ci
        L.mobi_ckpt_open.argtypes = [ctypes.c_char_p, ctypes.POINTER(p)]
        L.mobi_ckpt_open.restype = ci
        L.mobi_ckpt_count.argtypes = [p]
        L.mobi_ckpt_count.restype = ci
        L.mobi_ckpt_find.argtypes = [p, ctypes.c_char_p]
        L.mobi_ckpt_find.restype = ci
        L.mobi_ckpt_info.argtypes = [p, ci, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(i64),
                                     ctypes.POINTER(i64), ctypes.POINTER(ci), ctypes.POINTER(ci)]
        L.mobi_ckpt_info.restype = ci
        L.mobi_ckpt_load.argtypes = [p, ci, ci, p, p, ci, ci, p]
        L.mobi_ckpt_load.restype = ci
        L.mobi_ckpt_bytes_read.argtypes = [p]
        L.mobi_ckpt_bytes_read.restype = i64
        L.mobi_ckpt_close.argtypes = [p]
        L.mobi_ckpt_close.restype = None
        L.mobi_crc32c.argtypes = [ctypes.c_uint32, p, sz_t]
        L.mobi_crc32c.restype = ctypes.c_uint32
        L.mobi_sync_check.argtypes = [p]
        L.mobi_sync_check.restype = ci
        L.mobi_debug_set_wait_limit.argtypes = [i64]
        L.mobi_debug_set_wait_limit.restype = ci
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise MobiError(fn, status, lib().mobi_last_error().decode(errors="replace"))


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmobi takes CUDA tensors only (no CPU path)")
    if not t.is_contiguous():
        raise ValueError("libmobi takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def mobi_version() -> int:
    return lib().mobi_version()


def mobi_status_string(status: int) -> str:
    return lib().mobi_status_string(status).decode()


def mobi_last_error() -> str:
    return lib().mobi_last_error().decode(errors="replace")


def _int_array(vals):
    """A host int32 array for an `const int*` argument (kept alive by the caller)."""
    return (ctypes.c_int * len(vals))(*[int(v) for v in vals])


def mobi_codes_bytes(N: int, K: int, S: int = 3, bits: int = 2, widths=None) -> int:
    if widths is not None:
        return lib().mobi_codes_bytes_slices(N, K, len(widths), _int_array(widths))
    return lib().mobi_codes_bytes_bits(N, K, S, bits)


def mobi_sz_bytes(N: int, K: int, S: int = 3, G: int = 128) -> int:
    return lib().mobi_sz_bytes(N, K, S, G)


def mobi_route_workspace_bytes(T: int, K: int, S: int = 3) -> int:
    return lib().mobi_route_workspace_bytes(T, K, S)


def mobi_gemm_workspace_bytes(T: int, N: int, K: int, S: int = 3) -> int:
    return lib().mobi_gemm_workspace_bytes(T, N, K, S)


def _workspace(nbytes: int, device, ws: torch.Tensor | None) -> torch.Tensor:
    if ws is not None:
        return ws
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def mobi_pack(W: torch.Tensor, S: int = 3, G: int = 128, codes: torch.Tensor | None = None,
              sz: torch.Tensor | None = None, stream=None, bits: int = 2, widths=None):
    """MoBiSlice packing of fp16 W[N,K] -> (codes int32 [S,N,K*bits/32], sz int32 [S,K/128,N]).
    bits = 2 and G = 128 is the method's slicing (mobi_pack); other values go
    through mobi_pack_bits (bits 1 or 2, G 128/256/512, S up to 4; 1-bit codes
    at 32 per word)."""
    if W.dtype != torch.float16 or W.dim() != 2:
        raise ValueError("W must be a 2-D fp16 tensor")
    N, K = W.shape
    if widths is not None:  # one width per slice: codes are one flat array of every slice's words
        S = len(widths)
        wa = _int_array(widths)
        if codes is None:
            codes = torch.empty(max(mobi_codes_bytes(N, K, widths=widths) // 4, 1), dtype=torch.int32,
                                device=W.device)
        if sz is None:
            sz = torch.empty((S, K // 128, N), dtype=torch.int32, device=W.device)
        _check("mobi_pack_slices", lib().mobi_pack_slices(_ptr(W), N, K, G, S, wa, _ptr(codes), _ptr(sz),
                                                          _stream(stream)))
        return codes, sz
    if codes is None:
        codes = torch.empty((S, N, K * bits // 32), dtype=torch.int32, device=W.device)
    if sz is None:
        sz = torch.empty((S, K // 128, N), dtype=torch.int32, device=W.device)
    if bits == 2 and G == 128:
        _check("mobi_pack", lib().mobi_pack(_ptr(W), N, K, G, S, _ptr(codes), _ptr(sz), _stream(stream)))
    else:
        _check("mobi_pack_bits", lib().mobi_pack_bits(_ptr(W), N, K, G, S, bits, _ptr(codes), _ptr(sz),
                                                      _stream(stream)))
    return codes, sz


def mobi_route(X: torch.Tensor, Wr: torch.Tensor, bias: torch.Tensor | None = None, k_t=None, perm=None,
               offsets=None, ws: torch.Tensor | None = None, stream=None):
    """MoBiRoute: k_t = 1 + argmax(x.Wr + b) and the stable bucketing -> (k_t, perm, offsets)."""
    if X.dtype != torch.bfloat16 or Wr.dtype != torch.float32:
        raise ValueError("X must be bf16 and Wr fp32")
    T, K = X.shape
    S = Wr.shape[1]
    dev = X.device
    k_t = torch.empty(T, dtype=torch.int32, device=dev) if k_t is None else k_t
    perm = torch.empty(T, dtype=torch.int32, device=dev) if perm is None else perm
    offsets = torch.empty(S + 1, dtype=torch.int32, device=dev) if offsets is None else offsets
    need = mobi_route_workspace_bytes(T, K, S)
    ws = _workspace(need, dev, ws) if need > 0 else ws
    _check("mobi_route", lib().mobi_route(_ptr(X), T, K, _ptr(Wr), _ptr(bias), S, _ptr(k_t), _ptr(perm),
                                          _ptr(offsets), _ptr(ws), 0 if ws is None else ws.numel(),
                                          _stream(stream)))
    return k_t, perm, offsets


def mobi_route_mlp_workspace_bytes(T: int, K: int, H: int) -> int:
    return lib().mobi_route_mlp_workspace_bytes(T, K, H)


def mobi_route_mlp(X: torch.Tensor, W1: torch.Tensor, b1: torch.Tensor | None, W2: torch.Tensor,
                   b2: torch.Tensor | None, tau: float = 1.0, delta: float = 0.5, S: int | None = None, k_t=None,
                   perm=None, offsets=None, ws: torch.Tensor | None = None, stream=None):
    """Threshold routing with a two-layer MLP scorer: k_t = 1 + #{j : sigmoid(s_j / tau) > delta},
    s = ReLU(x.W1 + b1).W2 + b2, then the stable bucketing -> (k_t, perm, offsets).
    S defaults to W2.shape[1] + 1."""
    if X.dtype != torch.bfloat16 or W1.dtype != torch.float32 or W2.dtype != torch.float32:
        raise ValueError("X must be bf16, W1 and W2 fp32")
    T, K = X.shape
    H = W1.shape[1]
    S = W2.shape[1] + 1 if S is None else S
    dev = X.device
    k_t = torch.empty(T, dtype=torch.int32, device=dev) if k_t is None else k_t
    perm = torch.empty(T, dtype=torch.int32, device=dev) if perm is None else perm
    offsets = torch.empty(S + 1, dtype=torch.int32, device=dev) if offsets is None else offsets
    need = mobi_route_mlp_workspace_bytes(T, K, H) if S > 1 else 0
    ws = _workspace(need, dev, ws) if need > 0 else ws
    _check("mobi_route_mlp", lib().mobi_route_mlp(_ptr(X), T, K, _ptr(W1), _ptr(b1), H, _ptr(W2), _ptr(b2), S,
                                                  float(tau), float(delta), _ptr(k_t), _ptr(perm), _ptr(offsets),
                                                  _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return k_t, perm, offsets


def _problem_array(problems, S: int):
    """problems: sequence of dicts with X, Wr, codes, sz, N and optionally bias, Y, k_t, perm,
    offsets (allocated here when absent). Returns the ctypes array and the filled dicts."""
    arr = (LinearProblem * len(problems))()
    filled = []
    for i, pr in enumerate(problems):
        X = pr["X"]
        T, K = X.shape
        N = pr["N"]
        dev = X.device
        d = dict(pr)
        d.setdefault("bias", None)
        if d.get("Y") is None:
            d["Y"] = torch.empty((T, N), dtype=torch.float32, device=dev)
        if d.get("k_t") is None:
            d["k_t"] = torch.empty(T, dtype=torch.int32, device=dev)
        if d.get("perm") is None:
            d["perm"] = torch.empty(T, dtype=torch.int32, device=dev)
        if d.get("offsets") is None:
            d["offsets"] = torch.empty(S + 1, dtype=torch.int32, device=dev)
        arr[i] = LinearProblem(_ptr(X), _ptr(d["Wr"]), _ptr(d["bias"]), _ptr(d["codes"]), _ptr(d["sz"]),
                               _ptr(d["Y"]), _ptr(d["k_t"]), _ptr(d["perm"]), _ptr(d["offsets"]), T, N, K)
        filled.append(d)
    return arr, filled


def mobi_linear_grouped_workspace_bytes(problems, S: int = 3) -> int:
    arr, _ = _problem_array(problems, S)
    return lib().mobi_linear_grouped_workspace_bytes(arr, len(problems), S)


def mobi_linear_grouped(problems, S: int = 3, G: int = 128, ws: torch.Tensor | None = None, stream=None,
                        bits: int = 2, widths=None):
    """Up to MAX_GROUP independent decode-sized (T <= 16) mobi_linear problems in one step.
    Each problem is a dict with X, Wr, codes, sz, N (and optionally bias, Y, k_t, perm, offsets);
    `bits` is the code width of every slice. Returns [(Y, k_t, perm, offsets)] in problem order."""
    arr, filled = _problem_array(problems, S)
    if len(filled) == 0:
        raise ValueError("mobi_linear_grouped needs at least one problem")
    need = lib().mobi_linear_grouped_workspace_bytes(arr, len(filled), S)
    ws = _workspace(need, filled[0]["X"].device, ws) if need > 0 else ws
    if widths is not None:
        _check("mobi_linear_grouped", lib().mobi_linear_grouped_slices(arr, len(filled), G, len(widths),
                                                                       _int_array(widths), _ptr(ws),
                                                                       0 if ws is None else ws.numel(),
                                                                       _stream(stream)))
    else:
        _check("mobi_linear_grouped", lib().mobi_linear_grouped_bits(arr, len(filled), G, S, bits, _ptr(ws),
                                                                     0 if ws is None else ws.numel(),
                                                                     _stream(stream)))
    return [(d["Y"], d["k_t"], d["perm"], d["offsets"]) for d in filled]


def _gemm_problem_array(problems):
    arr = (GemmProblem * len(problems))()
    filled = []
    for i, pr in enumerate(problems):
        X = pr["X"]
        T, K = X.shape
        d = dict(pr)
        if d.get("Y") is None:
            d["Y"] = torch.empty((T, d["N"]), dtype=torch.float32, device=X.device)
        arr[i] = GemmProblem(_ptr(X), _ptr(d["k_t"]), _ptr(d["codes"]), _ptr(d["sz"]), _ptr(d["Y"]), T, d["N"], K)
        filled.append(d)
    return arr, filled


def mobi_gemm_grouped_workspace_bytes(problems, S: int = 3) -> int:
    arr, _ = _gemm_problem_array(problems)
    return lib().mobi_gemm_grouped_workspace_bytes(arr, len(problems), S)


def mobi_gemm_grouped(problems, S: int = 3, G: int = 128, ws: torch.Tensor | None = None, stream=None,
                      bits: int = 2, widths=None):
    """Up to MAX_GROUP decode-sized mobi_gemm problems (dicts with X, k_t, codes, sz, N and
    optionally Y) in one launch per fragment class; `bits` is the code width of every
    slice (mobi_gemm_grouped_bits). Returns [Y] in problem order."""
    arr, filled = _gemm_problem_array(problems)
    if len(filled) == 0:
        raise ValueError("mobi_gemm_grouped needs at least one problem")
    need = lib().mobi_gemm_grouped_workspace_bytes(arr, len(filled), S)
    ws = _workspace(need, filled[0]["X"].device, ws) if need > 0 else ws
    if widths is not None:
        _check("mobi_gemm_grouped", lib().mobi_gemm_grouped_slices(arr, len(filled), G, len(widths),
                                                                   _int_array(widths), _ptr(ws),
                                                                   0 if ws is None else ws.numel(), _stream(stream)))
    else:
        _check("mobi_gemm_grouped", lib().mobi_gemm_grouped_bits(arr, len(filled), G, S, bits, _ptr(ws),
                                                                 0 if ws is None else ws.numel(), _stream(stream)))
    return [d["Y"] for d in filled]


def _any_ptr(t):
    """(pointer, is_host) of a contiguous tensor or numpy array."""
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("checkpoint tensors must be contiguous")
        return ctypes.c_void_p(t.data_ptr()), not t.is_cuda
    import numpy as np
    a = np.ascontiguousarray(t)
    return ctypes.c_void_p(a.ctypes.data), True


def mobi_crc32c(data, crc: int = 0) -> int:
    """CRC-32C of a bytes-like object or a CPU tensor / numpy array."""
    if isinstance(data, (bytes, bytearray)):
        buf = (ctypes.c_char * len(data)).from_buffer_copy(bytes(data))
        return lib().mobi_crc32c(crc, ctypes.cast(buf, ctypes.c_void_p), len(data))
    ptr, host = _any_ptr(data)
    if not host:
        raise ValueError("mobi_crc32c takes host memory")
    nbytes = data.numel() * data.element_size() if isinstance(data, torch.Tensor) else data.nbytes
    return lib().mobi_crc32c(crc, ptr, nbytes)


def mobi_ckpt_save(path: str, tensors, G: int = 128, stream=None) -> None:
    """Write packed layers to one checkpoint. tensors: sequence of (name, codes, sz) with
    codes int32/uint32 [S, N, K/16] and sz [S, K/G, N], all on the device or all on the host."""
    arr = (CkptTensor * len(tensors))()
    keep = []
    host_flags = set()
    for i, (name, codes, sz) in enumerate(tensors):
        S, N, K16 = codes.shape
        cp, ch = _any_ptr(codes)
        zp, zh = _any_ptr(sz)
        host_flags.update((ch, zh))
        nb = name.encode()
        keep.append(nb)
        arr[i] = CkptTensor(nb, cp, zp, N, K16 * 16, G, S)
    if len(host_flags) != 1:
        raise ValueError("checkpoint tensors must be all on the host or all on the device")
    host = host_flags.pop()
    _check("mobi_ckpt_save", lib().mobi_ckpt_save(str(path).encode(), arr, len(tensors), int(host),
                                                  None if host else _stream(stream)))


class MobiCheckpoint:
    """A checkpoint opened for reading; load(name, slices) returns packed (codes, sz) with S = slices."""

    def __init__(self, path: str):
        h = ctypes.c_void_p()
        _check("mobi_ckpt_open", lib().mobi_ckpt_open(str(path).encode(), ctypes.byref(h)))
        self._h = h

    def close(self) -> None:
        if self._h:
            lib().mobi_ckpt_close(self._h)
            self._h = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __len__(self) -> int:
        return lib().mobi_ckpt_count(self._h)

    def names(self) -> list[str]:
        return [self.info(i)[0] for i in range(len(self))]

    def find(self, name: str) -> int:
        return lib().mobi_ckpt_find(self._h, name.encode())

    def info(self, index: int):
        """(name, N, K, G, S) of tensor `index`."""
        nm = ctypes.c_char_p()
        N, K = ctypes.c_int64(), ctypes.c_int64()
        G, S = ctypes.c_int(), ctypes.c_int()
        _check("mobi_ckpt_info", lib().mobi_ckpt_info(self._h, index, ctypes.byref(nm), ctypes.byref(N),
                                                      ctypes.byref(K), ctypes.byref(G), ctypes.byref(S)))
        return nm.value.decode(), N.value, K.value, G.value, S.value

    @property
    def bytes_read(self) -> int:
        return lib().mobi_ckpt_bytes_read(self._h)

    def load(self, name_or_index, slices: int | None = None, device=None, verify: bool = True, codes=None,
             sz=None, stream=None):
        idx = self.find(name_or_index) if isinstance(name_or_index, str) else int(name_or_index)
        if idx < 0:
            raise KeyError(name_or_index)
        _, N, K, G, S = self.info(idx)
        k = S if slices is None else slices
        dev = torch.device("cpu") if device is None else torch.device(device)
        if codes is None:
            codes = torch.empty((k, N, K // 16), dtype=torch.int32, device=dev)
        if sz is None:
            sz = torch.empty((k, K // G, N), dtype=torch.int32, device=dev)
        host = dev.type == "cpu"
        _check("mobi_ckpt_load", lib().mobi_ckpt_load(self._h, idx, k, ctypes.c_void_p(codes.data_ptr()),
                                                      ctypes.c_void_p(sz.data_ptr()), int(host), int(verify),
                                                      None if host else _stream(stream)))
        return codes, sz


def mobi_gemm_path(X: torch.Tensor, k_t: torch.Tensor, perm: torch.Tensor, offsets: torch.Tensor,
                   codes: torch.Tensor, sz: torch.Tensor, N: int, path: int = PATH_AUTO, S: int | None = None,
                   G: int = 128, Y: torch.Tensor | None = None, ws: torch.Tensor | None = None, stream=None,
                   bits: int = 2, widths=None):
    """Token-routed mixed-bit GEMM y_t = x_t . W^(k_t)^T (fp32) with an explicit kernel choice
    and the code width of the slices (mobi_gemm_bits)."""
    T, K = X.shape
    S = (len(widths) if widths is not None else codes.shape[0]) if S is None else S
    Y = torch.empty((T, N), dtype=torch.float32, device=X.device) if Y is None else Y
    ws = _workspace(mobi_gemm_workspace_bytes(T, N, K, S), X.device, ws)
    if widths is not None:
        _check("mobi_gemm", lib().mobi_gemm_slices(_ptr(X), T, K, _ptr(k_t), _ptr(perm), _ptr(offsets), _ptr(codes),
                                                   _ptr(sz), N, G, S, _int_array(widths), _ptr(Y), _ptr(ws),
                                                   ws.numel(), _stream(stream), path))
    else:
        _check("mobi_gemm", lib().mobi_gemm_bits(_ptr(X), T, K, _ptr(k_t), _ptr(perm), _ptr(offsets), _ptr(codes),
                                                 _ptr(sz), N, G, S, bits, _ptr(Y), _ptr(ws), ws.numel(),
                                                 _stream(stream), path))
    return Y


def mobi_gemm(X, k_t, perm, offsets, codes, sz, N, S=None, G=128, Y=None, ws=None, stream=None, bits=2,
              widths=None):
    """Token-routed mixed-bit GEMM (decode kernel for T <= 16, tcgen05 prefill kernel above)."""
    return mobi_gemm_path(X, k_t, perm, offsets, codes, sz, N, PATH_AUTO, S, G, Y, ws, stream, bits, widths)


def mobi_gemm_decode_noalloc(X, k_t, codes, sz, N, S=None, G=128, Y=None, stream=None):
    """Decode GEMM (T <= 16) whose scratch is the library's static device array (no workspace)."""
    T, K = X.shape
    S = codes.shape[0] if S is None else S
    Y = torch.empty((T, N), dtype=torch.float32, device=X.device) if Y is None else Y
    _check("mobi_gemm_decode_noalloc", lib().mobi_gemm_decode_noalloc(_ptr(X), T, K, _ptr(k_t), _ptr(codes),
                                                                      _ptr(sz), N, G, S, _ptr(Y), _stream(stream)))
    return Y


def mobi_linear_workspace_bytes(T: int, N: int, K: int, S: int = 3) -> int:
    return lib().mobi_linear_workspace_bytes(T, N, K, S)


def mobi_linear(X, Wr, bias, codes, sz, N, G=128, Y=None, k_t=None, perm=None, offsets=None, ws=None, stream=None,
                bits=2, widths=None):
    """Route + mixed-bit GEMM in one call (S = Wr.shape[1], slices of `bits`-bit codes)
    -> (Y fp32 [T,N], k_t, perm, offsets)."""
    if X.dtype != torch.bfloat16 or Wr.dtype != torch.float32:
        raise ValueError("X must be bf16 and Wr fp32")
    T, K = X.shape
    S = Wr.shape[1]
    dev = X.device
    Y = torch.empty((T, N), dtype=torch.float32, device=dev) if Y is None else Y
    k_t = torch.empty(T, dtype=torch.int32, device=dev) if k_t is None else k_t
    perm = torch.empty(T, dtype=torch.int32, device=dev) if perm is None else perm
    offsets = torch.empty(S + 1, dtype=torch.int32, device=dev) if offsets is None else offsets
    ws = _workspace(mobi_linear_workspace_bytes(T, N, K, S), dev, ws)
    if widths is not None:
        if len(widths) != S:
            raise ValueError("one width per slice (the router's column count)")
        _check("mobi_linear", lib().mobi_linear_slices(_ptr(X), T, K, _ptr(Wr), _ptr(bias), _ptr(codes), _ptr(sz),
                                                       N, G, S, _int_array(widths), _ptr(k_t), _ptr(perm),
                                                       _ptr(offsets), _ptr(Y), _ptr(ws), ws.numel(),
                                                       _stream(stream)))
    else:
        _check("mobi_linear", lib().mobi_linear_bits(_ptr(X), T, K, _ptr(Wr), _ptr(bias), _ptr(codes), _ptr(sz), N,
                                                     G, S, bits, _ptr(k_t), _ptr(perm), _ptr(offsets), _ptr(Y),
                                                     _ptr(ws), ws.numel(), _stream(stream)))
    return Y, k_t, perm, offsets


def mobi_sync_check(stream=None) -> None:
    """Synchronise the stream and raise MobiError if a kernel recorded a device-side error."""
    _check("mobi_sync_check", lib().mobi_sync_check(_stream(stream)))


def mobi_debug_set_wait_limit(limit: int) -> None:
    _check("mobi_debug_set_wait_limit", lib().mobi_debug_set_wait_limit(limit))
