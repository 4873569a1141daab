"""Python binding of libslim (include/slim.h). Argument marshalling only.

Every function has the name of the C entry point it calls. Device arrays are
torch CUDA tensors (PyTorch provides the memory and the stream); outputs that
are not supplied are allocated with torch.empty on the input's device. All the
arithmetic runs in the library's kernels. There is no fallback: if libslim.so
is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libslim.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "slim.h")

SLIM_X_F32, SLIM_X_BF16 = 0, 1
SLIM_OBJ_KL, SLIM_OBJ_MSE = 0, 1
OBJECTIVES = {"kl": SLIM_OBJ_KL, "mse": SLIM_OBJ_MSE}
SLIM_SBA_ADAPTIVE, SLIM_SBA_FULL = 0, 1
PRECISIONS = {"adaptive": SLIM_SBA_ADAPTIVE, "full": SLIM_SBA_FULL}
STATUS = {0: "SLIM_OK", 1: "SLIM_EINVAL", 2: "SLIM_ENOMEM", 3: "SLIM_ECUDA", 4: "SLIM_ETIMEOUT",
          5: "SLIM_ENOTPD", 6: "SLIM_ENODEV", 7: "SLIM_EINJECTED", 8: "SLIM_ERANGE"}


class SlimError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        self.device_detail = _lib().slim_last_status_detail()
        if self.device_detail:
            detail = (detail + " " if detail else "") + f"[device detail {self.device_detail}]"
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_lib().slim_status_string(status).decode()})"
                         + (f" {detail}" if detail else ""))


_L = None
i64, i32, dbl, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_size_t


class SlimDiag(ctypes.Structure):
    _fields_ = [("H", vp), ("h", vp), ("S", vp), ("order", vp), ("kl", vp), ("tau_idx", vp),
                ("p_star", ctypes.c_int32), ("stage_ms", ctypes.c_float * 8), ("sba_split", vp)]


class SlimOptions(ctypes.Structure):
    _fields_ = [("objective", ctypes.c_int), ("sba_precision", ctypes.c_int), ("gptq", ctypes.c_int),
                ("order", vp)]


_SIGS = {
    "slim_status_string": (ctypes.c_char_p, [i32]),
    "slim_last_cuda_error": (ctypes.c_char_p, []),
    "slim_last_status_detail": (i32, []),
    "slim_version": (ctypes.c_char_p, []),
    "slim_num_candidates": (i32, [i64, i32]),
    "slim_row_words": (i64, [i64, i32]),
    "slim_launch_count": (i64, []),
    "slim_peak_fp64": (i32, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double), vp]),
    "slim_hessian_workspace_bytes": (sz, [i64, i64, i32]),
    "slim_hessian": (i32, [vp, i32, i64, i64, vp, vp, sz, vp]),
    "slim_hinv_diag_workspace_bytes": (sz, [i64]),
    "slim_hinv_diag": (i32, [vp, i64, dbl, vp, vp, sz, vp]),
    "slim_salience_workspace_bytes": (sz, [i64, i64, i32]),
    "slim_salience": (i32, [vp, i64, i64, vp, i32, vp, vp, vp, sz, vp]),
    "slim_salience_noalloc": (i32, [vp, i64, i64, vp, i32, vp, vp, vp]),
    "slim_sba_workspace_bytes": (sz, [i64, i64, i64, i32, i32]),
    "slim_sba_search": (i32, [vp, i64, i64, vp, i32, i64, i32, i32, vp, vp, vp, vp, vp, sz, vp]),
    "slim_sba_search_ex": (i32, [vp, i64, i64, vp, i32, i64, i32, i32, vp, i32, i32, vp, vp, vp, vp, sz, vp]),
    "slim_sba_split_workspace_bytes": (sz, [i64, i64, i64, i32, i32]),
    "slim_sba_search_split": (i32, [vp, i64, i64, vp, i32, i64, i32, i32, vp, vp, vp, vp, i64, vp, sz, vp]),
    "slim_sqc": (i32, [vp, i64, i64, vp, vp, i32, i32, dbl, i32, vp, vp, vp, vp, vp]),
    "slim_gptq_workspace_bytes": (sz, [i64, i64]),
    "slim_gptq": (i32, [vp, i64, i64, vp, vp, i32, i32, dbl, i32, vp, vp, vp, vp, vp, sz, vp]),
    "slim_dequant_gemv_workspace_bytes": (sz, [i64, i64, i32, i32, i64]),
    "slim_dequant_gemv": (i32, [vp, vp, vp, vp, i64, i64, i32, i32, vp, i32, i64, vp, vp, sz, vp]),
    "slim_workspace_bytes": (sz, [i64, i64, i64, i32, i32, i32]),
    "slim_quantize_layer": (i32, [vp, i64, i64, vp, i32, i64, i32, i32, dbl, i32, vp, vp, vp, vp, vp, sz, vp]),
    "slim_quantize_layer_ex": (i32, [vp, i64, i64, vp, i32, i64, i32, i32, dbl, i32, vp, vp, vp, vp, vp, sz, vp,
                                     ctypes.POINTER(SlimDiag)]),
    "slim_quantize_layer_opts": (i32, [vp, i64, i64, vp, i32, i64, i32, i32, dbl, i32, vp, vp, vp, vp, vp, sz, vp,
                                       ctypes.POINTER(SlimOptions), ctypes.POINTER(SlimDiag)]),
    "slim_quantize_layer_host": (i32, [vp, i64, i64, vp, i32, i64, i32, i32, dbl, i32, vp, vp, vp, vp, vp]),
}


def header_functions() -> list:
    """Names of every function declared in include/slim.h."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(slim_[a-z0-9_]+)\s*\(", txt)))


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m post_weight_quantization_hessian_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _L = L
    return _L


def lib_path() -> str:
    _lib()
    return LIB_PATH


def _check(rc: int, where: str):
    if rc != 0:
        raise SlimError(rc, where, _lib().slim_last_cuda_error().decode())


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return t.data_ptr()
    return int(t)


def _xdtype(X: torch.Tensor) -> int:
    if X.dtype in (torch.bfloat16, torch.uint16, torch.int16):
        return SLIM_X_BF16
    if X.dtype == torch.float32:
        return SLIM_X_F32
    raise ValueError(f"X must be bf16 (or its uint16 bits) or float32, got {X.dtype}")


def _x_np_dtype(X: np.ndarray) -> int:
    if X.dtype == np.uint16:
        return SLIM_X_BF16
    if X.dtype == np.float32:
        return SLIM_X_F32
    raise ValueError("host X must be uint16 bf16 bits or float32")


# --------------------------------------------------------------------- host-only queries
def slim_num_candidates(n: int, group: int) -> int:
    return _lib().slim_num_candidates(n, group)


def slim_row_words(n: int, avg_bits: int) -> int:
    return _lib().slim_row_words(n, avg_bits)


def slim_workspace_bytes(m, n, N, xdtype, group, avg_bits) -> int:
    return _lib().slim_workspace_bytes(m, n, N, xdtype, group, avg_bits)


def slim_launch_count() -> int:
    return _lib().slim_launch_count()


def slim_version() -> str:
    return _lib().slim_version().decode()


def slim_peak_fp64(stream=None):
    """(fp64 tensor-core MMA, fp64 FMA) rates of the current device, TFLOP/s."""
    a, b = ctypes.c_double(), ctypes.c_double()
    _check(_lib().slim_peak_fp64(ctypes.byref(a), ctypes.byref(b), _stream(stream)), "slim_peak_fp64")
    return a.value, b.value


# --------------------------------------------------------------------- stages
def slim_hessian(X: torch.Tensor, H: Optional[torch.Tensor] = None, ws=None, stream=None) -> torch.Tensor:
    N, n = X.shape
    if H is None:
        H = torch.empty((n, n), dtype=torch.float64, device=X.device)
    wsb = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(_lib().slim_hessian(_ptr(X), _xdtype(X), N, n, _ptr(H), _ptr(ws), wsb, _stream(stream)), "slim_hessian")
    return H


def slim_hinv_diag(H: torch.Tensor, alpha: float = 0.01, h: Optional[torch.Tensor] = None, ws=None,
                   stream=None) -> torch.Tensor:
    n = H.shape[0]
    if h is None:
        h = torch.empty(n, dtype=torch.float64, device=H.device)
    wsb = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(_lib().slim_hinv_diag(_ptr(H), n, float(alpha), _ptr(h), _ptr(ws), wsb, _stream(stream)),
           "slim_hinv_diag")
    return h


def slim_salience(W: torch.Tensor, h: torch.Tensor, group: int, S=None, order=None, ws=None, stream=None):
    m, n = W.shape
    k = n // group
    if S is None:
        S = torch.empty(k, dtype=torch.float64, device=W.device)
    if order is None:
        order = torch.empty(k, dtype=torch.int32, device=W.device)
    wsb = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(_lib().slim_salience(_ptr(W), m, n, _ptr(h), group, _ptr(S), _ptr(order), _ptr(ws), wsb,
                                _stream(stream)), "slim_salience")
    return S, order


def slim_salience_noalloc(W: torch.Tensor, h: torch.Tensor, group: int, S=None, order=None, stream=None):
    """slim_salience without any device allocation by the library (fixed internal scratch)."""
    m, n = W.shape
    k = n // group
    if S is None:
        S = torch.empty(k, dtype=torch.float64, device=W.device)
    if order is None:
        order = torch.empty(k, dtype=torch.int32, device=W.device)
    _check(_lib().slim_salience_noalloc(_ptr(W), m, n, _ptr(h), group, _ptr(S), _ptr(order), _stream(stream)),
           "slim_salience_noalloc")
    return S, order


def slim_sba_search(W: torch.Tensor, X: torch.Tensor, group: int, avg_bits: int, order: torch.Tensor, ws=None,
                    stream=None):
    m, n = W.shape
    N = X.shape[0]
    k = n // group
    P = k // 2 + 1
    kl = torch.empty(P, dtype=torch.float64, device=W.device)
    p_star = torch.empty(1, dtype=torch.int32, device=W.device)
    bits = torch.empty(k, dtype=torch.uint8, device=W.device)
    wsb = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(_lib().slim_sba_search(_ptr(W), m, n, _ptr(X), _xdtype(X), N, group, avg_bits, _ptr(order), _ptr(kl),
                                  _ptr(p_star), _ptr(bits), _ptr(ws), wsb, _stream(stream)), "slim_sba_search")
    return kl, p_star, bits


def slim_sba_search_ex(W: torch.Tensor, X: torch.Tensor, group: int, avg_bits: int, order: torch.Tensor,
                       objective: str = "kl", precision: str = "adaptive", ws=None, stream=None):
    """slim_sba_search with the objective "kl" or "mse" and the operand precision "adaptive" or
    "full"; order is any permutation of the groups."""
    m, n = W.shape
    N = X.shape[0]
    k = n // group
    P = k // 2 + 1
    kl = torch.empty(P, dtype=torch.float64, device=W.device)
    p_star = torch.empty(1, dtype=torch.int32, device=W.device)
    bits = torch.empty(k, dtype=torch.uint8, device=W.device)
    wsb = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(_lib().slim_sba_search_ex(_ptr(W), m, n, _ptr(X), _xdtype(X), N, group, avg_bits, _ptr(order),
                                     OBJECTIVES[objective], PRECISIONS[precision], _ptr(kl), _ptr(p_star), _ptr(bits),
                                     _ptr(ws), wsb,
                                     _stream(stream)), "slim_sba_search_ex")
    return kl, p_star, bits


def slim_sba_search_split(W: torch.Tensor, X: torch.Tensor, group: int, avg_bits: int, order: torch.Tensor,
                          chunk_tokens: int, ws=None, stream=None):
    """slim_sba_search's outputs from the two-part schedule: phase A per chunk of
    chunk_tokens tokens (a multiple of 256), then the candidate steps."""
    m, n = W.shape
    N = X.shape[0]
    k = n // group
    P = k // 2 + 1
    kl = torch.empty(P, dtype=torch.float64, device=W.device)
    p_star = torch.empty(1, dtype=torch.int32, device=W.device)
    bits = torch.empty(k, dtype=torch.uint8, device=W.device)
    wsb = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(_lib().slim_sba_search_split(_ptr(W), m, n, _ptr(X), _xdtype(X), N, group, avg_bits, _ptr(order),
                                        _ptr(kl), _ptr(p_star), _ptr(bits), int(chunk_tokens), _ptr(ws), wsb,
                                        _stream(stream)), "slim_sba_search_split")
    return kl, p_star, bits


def slim_sqc(W: torch.Tensor, h: torch.Tensor, bits: torch.Tensor, group: int, avg_bits: int, lam: float,
             n_tau: int, stream=None):
    m, n = W.shape
    k = n // group
    codes = torch.empty((m, n * avg_bits // 32), dtype=torch.int32, device=W.device)
    scale = torch.empty((m, k), dtype=torch.float32, device=W.device)
    zero = torch.empty((m, k), dtype=torch.float32, device=W.device)
    tau = torch.empty((m, k), dtype=torch.uint8, device=W.device)
    _check(_lib().slim_sqc(_ptr(W), m, n, _ptr(h), _ptr(bits), group, avg_bits, float(lam), n_tau, _ptr(codes),
                           _ptr(scale), _ptr(zero), _ptr(tau), _stream(stream)), "slim_sqc")
    return codes, scale, zero, tau


def slim_gptq(W: torch.Tensor, H: torch.Tensor, bits: torch.Tensor, group: int, avg_bits: int, lam: float,
              n_tau: int, ws=None, stream=None):
    """SQC's quantizer inside the GPTQ column loop (error compensation along U)."""
    m, n = W.shape
    k = n // group
    codes = torch.empty((m, n * avg_bits // 32), dtype=torch.int32, device=W.device)
    scale = torch.empty((m, k), dtype=torch.float32, device=W.device)
    zero = torch.empty((m, k), dtype=torch.float32, device=W.device)
    tau = torch.empty((m, k), dtype=torch.uint8, device=W.device)
    wsb = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(_lib().slim_gptq(_ptr(W), m, n, _ptr(H), _ptr(bits), group, avg_bits, float(lam), n_tau, _ptr(codes),
                            _ptr(scale), _ptr(zero), _ptr(tau), _ptr(ws), wsb, _stream(stream)), "slim_gptq")
    return codes, scale, zero, tau


def slim_dequant_gemv(codes: torch.Tensor, bits: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor, group: int,
                      avg_bits: int, x: torch.Tensor, y: Optional[torch.Tensor] = None, ws=None, stream=None):
    """y = x W_hat^T for a packed layer; x is [batch, n] (batch <= 8), float32 or bf16."""
    m, k = scale.shape
    n = k * group
    if x.dim() == 1:
        x = x.view(1, -1)
    B = x.shape[0]
    if y is None:
        y = torch.empty((B, m), dtype=torch.float32, device=codes.device)
    wsb = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(_lib().slim_dequant_gemv(_ptr(codes), _ptr(bits), _ptr(scale), _ptr(zero), m, n, group, avg_bits, _ptr(x),
                                    _xdtype(x), B, _ptr(y), _ptr(ws), wsb, _stream(stream)), "slim_dequant_gemv")
    return y


# --------------------------------------------------------------------- whole layer
def _layer_outputs(W, group, avg_bits):
    m, n = W.shape
    k = n // group
    return (torch.empty((m, n * avg_bits // 32), dtype=torch.int32, device=W.device),
            torch.empty((m, k), dtype=torch.float32, device=W.device),
            torch.empty((m, k), dtype=torch.float32, device=W.device),
            torch.empty(k, dtype=torch.uint8, device=W.device))


def alloc_workspace(W: torch.Tensor, X: torch.Tensor, group: int, avg_bits: int) -> torch.Tensor:
    m, n = W.shape
    nb = slim_workspace_bytes(m, n, X.shape[0], _xdtype(X), group, avg_bits)
    if nb == 0:
        raise ValueError("invalid layer shape")
    return torch.empty(nb, dtype=torch.uint8, device=W.device)


def slim_quantize_layer(W: torch.Tensor, X: torch.Tensor, group: int, avg_bits: int, lam: float = 0.1,
                        n_tau: int = 50, ws: Optional[torch.Tensor] = None, out=None, stream=None):
    m, n = W.shape
    codes, scale, zero, bits = out if out is not None else _layer_outputs(W, group, avg_bits)
    wsb = ws.numel() if isinstance(ws, torch.Tensor) else 0
    _check(_lib().slim_quantize_layer(_ptr(W), m, n, _ptr(X), _xdtype(X), X.shape[0], group, avg_bits, float(lam),
                                      n_tau, _ptr(codes), _ptr(scale), _ptr(zero), _ptr(bits), _ptr(ws), wsb,
                                      _stream(stream)), "slim_quantize_layer")
    return codes, scale, zero, bits


def slim_quantize_layer_ex(W: torch.Tensor, X: torch.Tensor, group: int, avg_bits: int, lam: float = 0.1,
                           n_tau: int = 50, ws: Optional[torch.Tensor] = None, want_H: bool = True, stream=None,
                           bufs: Optional[dict] = None):
    return slim_quantize_layer_opts(W, X, group, avg_bits, lam, n_tau, ws=ws, want_H=want_H, stream=stream,
                                    bufs=bufs)


def layer_buffers(W: torch.Tensor, group: int, avg_bits: int, want_H: bool = True) -> dict:
    """Output and diagnostic tensors of slim_quantize_layer_ex / _opts for a layer shape, to
    pass as bufs= to repeated calls (the same device addresses every call)."""
    m, n = W.shape
    k = n // group
    P = k // 2 + 1
    dev = W.device
    codes, scale, zero, bits = _layer_outputs(W, group, avg_bits)
    return {"codes": codes, "scale": scale, "zero": zero, "bits": bits,
            "H": torch.empty((n, n), dtype=torch.float64, device=dev) if want_H else None,
            "h": torch.empty(n, dtype=torch.float64, device=dev),
            "S": torch.empty(k, dtype=torch.float64, device=dev),
            "order": torch.empty(k, dtype=torch.int32, device=dev),
            "kl": torch.empty(P, dtype=torch.float64, device=dev),
            "tau_idx": torch.empty((m, k), dtype=torch.uint8, device=dev),
            "sba_split": torch.empty((n + 63) // 64, dtype=torch.uint8, device=dev)}


def slim_quantize_layer_opts(W: torch.Tensor, X: torch.Tensor, group: int, avg_bits: int, lam: float = 0.1,
                             n_tau: int = 50, ws: Optional[torch.Tensor] = None, want_H: bool = True,
                             objective: str = "kl", order: Optional[torch.Tensor] = None,
                             precision: str = "adaptive", gptq: bool = False, stream=None,
                             bufs: Optional[dict] = None):
    """The whole path with every intermediate (slim_quantize_layer_ex when the options are the
    defaults, else slim_quantize_layer_opts): objective "kl" or "mse", and optionally a
    caller's group order (device int32 permutation) in place of the salience order."""
    m, n = W.shape
    b = bufs if bufs is not None else layer_buffers(W, group, avg_bits, want_H)
    codes, scale, zero, bits = b["codes"], b["scale"], b["zero"], b["bits"]
    d = {key: b[key] for key in ("H", "h", "S", "order", "kl", "tau_idx", "sba_split")}
    diag = SlimDiag(H=_ptr(d["H"]), h=_ptr(d["h"]), S=_ptr(d["S"]), order=_ptr(d["order"]), kl=_ptr(d["kl"]),
                    tau_idx=_ptr(d["tau_idx"]), sba_split=_ptr(d["sba_split"]))
    wsb = ws.numel() if isinstance(ws, torch.Tensor) else 0
    if objective == "kl" and order is None and precision == "adaptive" and not gptq:
        _check(_lib().slim_quantize_layer_ex(_ptr(W), m, n, _ptr(X), _xdtype(X), X.shape[0], group, avg_bits,
                                             float(lam), n_tau, _ptr(codes), _ptr(scale), _ptr(zero), _ptr(bits),
                                             _ptr(ws), wsb, _stream(stream), ctypes.byref(diag)),
               "slim_quantize_layer_ex")
    else:
        opt = SlimOptions(objective=OBJECTIVES[objective], sba_precision=PRECISIONS[precision], gptq=int(gptq),
                          order=_ptr(order))
        _check(_lib().slim_quantize_layer_opts(_ptr(W), m, n, _ptr(X), _xdtype(X), X.shape[0], group, avg_bits,
                                               float(lam), n_tau, _ptr(codes), _ptr(scale), _ptr(zero), _ptr(bits),
                                               _ptr(ws), wsb, _stream(stream), ctypes.byref(opt),
                                               ctypes.byref(diag)), "slim_quantize_layer_opts")
    d.update(codes=codes, scale=scale, zero=zero, bits=bits, p_star=int(diag.p_star),
             stage_ms=list(diag.stage_ms)[:6], kernel_ms=list(diag.stage_ms)[6:8])
    return d


def slim_quantize_layer_host(W: np.ndarray, X: np.ndarray, group: int, avg_bits: int, lam: float = 0.1,
                             n_tau: int = 50, out=None, stream=None):
    """HOST arrays in and out (numpy, or pinned torch CPU tensors via .numpy())."""
    m, n = W.shape
    k = n // group
    if out is None:
        out = (np.empty((m, n * avg_bits // 32), np.uint32), np.empty((m, k), np.float32),
               np.empty((m, k), np.float32), np.empty(k, np.uint8))
    codes, scale, zero, bits = out
    for a in (W, X, codes, scale, zero, bits):
        if not a.flags["C_CONTIGUOUS"]:
            raise ValueError("host arrays must be C-contiguous")
    _check(_lib().slim_quantize_layer_host(W.ctypes.data, m, n, X.ctypes.data, _x_np_dtype(X), X.shape[0], group,
                                           avg_bits, float(lam), n_tau, codes.ctypes.data, scale.ctypes.data,
                                           zero.ctypes.data, bits.ctypes.data, _stream(stream)),
           "slim_quantize_layer_host")
    return codes, scale, zero, bits
