"""Thin ctypes binding of libgq (include/gq.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does nothing but convert
torch tensors to pointers, check dtypes/shapes/devices, and raise on a non-OK status.  All
computation happens in the CUDA library; torch provides device memory and the stream.  The
library must be built (``python -m post_weight_quantization_22_b200.build``); importing this
module without it raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgq.so")

GQ_BF16, GQ_FP32 = 0, 1
ORDERS = {"natural": 0, "reverse": 1, "act": 2, "min_pivot": 3, "given": 4}  # gq_order
STATUS = {0: "ok", 1: "invalid argument", 2: "not positive definite", 3: "CUDA error",
          4: "unsupported", 5: "timeout", 6: "no fit", 7: "workspace"}


class GQError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: gq status {code} ({STATUS.get(code, '?')})")
        self.code = code


class _Cfg(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group_size", ctypes.c_int), ("reverse", ctypes.c_int),
                ("clip", ctypes.c_int), ("ladder", ctypes.c_float), ("ladder_max", ctypes.c_int),
                ("spacing", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libgq.so is not built ({LIB_PATH}); run "
                          "`python -m post_weight_quantization_22_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, SZ, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    lib.gq_version.restype = ctypes.c_char_p
    lib.gq_status_string.restype = ctypes.c_char_p
    lib.gq_status_string.argtypes = [I]
    lib.gq_hessian_accumulate.restype = I
    lib.gq_hessian_accumulate.argtypes = [P, P, I, I64, I64, I, P, SZ, P]
    lib.gq_hessian_workspace_size.restype = SZ
    lib.gq_hessian_workspace_size.argtypes = [I64, I64]
    lib.gq_prepare_workspace_size.restype = SZ
    lib.gq_prepare_workspace_size.argtypes = [I64]
    lib.gq_prepare_hinv.restype = I
    lib.gq_prepare_hinv.argtypes = [P, I64, ctypes.c_double, I, P, P, P, P, SZ, P]
    lib.gq_quantize_workspace_size.restype = SZ
    lib.gq_quantize_workspace_size.argtypes = [I64, I64, ctypes.POINTER(_Cfg)]
    lib.gq_quantize_layer.restype = I
    lib.gq_quantize_layer.argtypes = [P, I, I64, I64, P, P, P, ctypes.POINTER(_Cfg), P, P, P, P,
                                      P, SZ, P]
    lib.gq_prepare_hinv_ordered.restype = I
    lib.gq_prepare_hinv_ordered.argtypes = [P, I64, ctypes.c_double, I, P, P, P, P, P, SZ, P]
    lib.gq_quantize_layer_ordered.restype = I
    lib.gq_quantize_layer_ordered.argtypes = [P, I, I64, I64, P, P, P, ctypes.POINTER(_Cfg), P,
                                              P, P, P, P, P, SZ, P]
    lib.gq_prepare_hinv_static.restype = I
    lib.gq_prepare_hinv_static.argtypes = [P, I64, ctypes.c_double, I, P, P, P, P, P]
    lib.gq_huffman_workspace_size.restype = SZ
    lib.gq_huffman_workspace_size.argtypes = [I64]
    lib.gq_huffman_encode.restype = I
    lib.gq_huffman_encode.argtypes = [P, I64, P, I64, P, P, P, P, SZ, P]
    lib.gq_ssqr_workspace_size.restype = SZ
    lib.gq_ssqr_workspace_size.argtypes = [I64, I64]
    lib.gq_ssqr_quantize_layer.restype = I
    lib.gq_ssqr_quantize_layer.argtypes = [P, I, I64, I64, P, P, P, I, ctypes.c_double, I, I, P,
                                           P, P, P, P, P, P, I64, P, P, SZ, P]
    lib.gq_hptq_workspace_size.restype = SZ
    lib.gq_hptq_workspace_size.argtypes = [I64, I64]
    lib.gq_hptq_quantize_layer.restype = I
    lib.gq_hptq_quantize_layer.argtypes = [P, I, I64, I64, P, P, P, I, ctypes.c_double, I, I, P,
                                           P, P, P, P, P, SZ, P]
    lib.gq_zsic_spacing.restype = I
    lib.gq_zsic_spacing.argtypes = [P, I64, P, P]
    lib.gq_debug_wait_test.restype = I
    lib.gq_debug_wait_test.argtypes = [ctypes.c_uint32, I]
    lib.gq_workspace_status.restype = I
    lib.gq_workspace_status.argtypes = [P, ctypes.POINTER(ctypes.c_int), P]
    return lib


LIB = _load()
EXPORTED = ("gq_version", "gq_status_string", "gq_hessian_accumulate", "gq_hessian_workspace_size",
            "gq_prepare_workspace_size",
            "gq_prepare_hinv", "gq_quantize_workspace_size", "gq_quantize_layer",
            "gq_workspace_status", "gq_prepare_hinv_static", "gq_prepare_hinv_ordered",
            "gq_quantize_layer_ordered", "gq_zsic_spacing", "gq_huffman_workspace_size",
            "gq_huffman_encode", "gq_debug_wait_test", "gq_kernel_launches",
            "gq_ssqr_workspace_size", "gq_ssqr_quantize_layer", "gq_hptq_workspace_size",
            "gq_hptq_quantize_layer")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GQ_BF16
    if t.dtype == torch.float32:
        return GQ_FP32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _check(code: int, what: str):
    if code != 0:
        raise GQError(code, what)


def _need(t: torch.Tensor, dtype, shape, name):
    if not t.is_cuda or t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous cuda {dtype} {tuple(shape)}, got "
                         f"{t.device} {t.dtype} {tuple(t.shape)}")


def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned device byte buffer of at least nbytes (torch allocations are)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def gq_version() -> str:
    return LIB.gq_version().decode()


def gq_hessian_workspace_size(T: int, n: int) -> int:
    return int(LIB.gq_hessian_workspace_size(T, n))


def gq_hessian_accumulate(H: torch.Tensor, X: torch.Tensor, accumulate: bool = True, ws=None,
                          stream=None) -> torch.Tensor:
    """H (+)= 2 X^T X on the GPU (H fp64 n x n, X bf16/fp32 T x n, same device)."""
    T, n = X.shape
    _need(H, torch.float64, (n, n), "H")
    if not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous cuda tensor")
    ws = workspace(gq_hessian_workspace_size(T, n), X.device) if ws is None else ws
    _check(LIB.gq_hessian_accumulate(_ptr(H), _ptr(X), _dtype_code(X), T, n, int(bool(accumulate)),
                                     _ptr(ws), ws.numel(), _stream(stream)),
           "gq_hessian_accumulate")
    return H


def gq_prepare_workspace_size(n: int) -> int:
    return int(LIB.gq_prepare_workspace_size(n))


def gq_prepare_hinv(H: torch.Tensor, damp: float = 0.01, reverse: bool = False, U=None,
                    dead=None, delta=None, ws=None, stream=None):
    """U (fp32 n x n upper), dead mask (uint8 n), delta (fp64 [1]) from fp64 H."""
    n = H.shape[0]
    _need(H, torch.float64, (n, n), "H")
    dev = H.device
    U = torch.empty((n, n), dtype=torch.float32, device=dev) if U is None else U
    dead = torch.empty(n, dtype=torch.uint8, device=dev) if dead is None else dead
    delta = torch.empty(1, dtype=torch.float64, device=dev) if delta is None else delta
    need = gq_prepare_workspace_size(n)
    ws = workspace(need, dev) if ws is None else ws
    _need(U, torch.float32, (n, n), "U")
    _check(LIB.gq_prepare_hinv(_ptr(H), n, float(damp), int(bool(reverse)), _ptr(U), _ptr(dead),
                               _ptr(delta), _ptr(ws), ws.numel(), _stream(stream)),
           "gq_prepare_hinv")
    return U, dead, delta, ws


def gq_prepare_hinv_ordered(H: torch.Tensor, damp: float = 0.01, order: str = "act", perm=None,
                            U=None, dead=None, delta=None, ws=None, stream=None):
    """gq_prepare_hinv in a column order ("natural", "reverse", "act", "min_pivot", "given").
    Returns (perm int32 n, U, dead, delta, ws); for "given" pass perm, else it is written."""
    n = H.shape[0]
    _need(H, torch.float64, (n, n), "H")
    if order not in ORDERS:
        raise ValueError(f"unknown order {order!r}")
    dev = H.device
    if perm is None:
        if order == "given":
            raise ValueError("order 'given' needs perm")
        perm = torch.empty(n, dtype=torch.int32, device=dev)
    _need(perm, torch.int32, (n,), "perm")
    U = torch.empty((n, n), dtype=torch.float32, device=dev) if U is None else U
    dead = torch.empty(n, dtype=torch.uint8, device=dev) if dead is None else dead
    delta = torch.empty(1, dtype=torch.float64, device=dev) if delta is None else delta
    ws = workspace(gq_prepare_workspace_size(n), dev) if ws is None else ws
    _need(U, torch.float32, (n, n), "U")
    _check(LIB.gq_prepare_hinv_ordered(_ptr(H), n, float(damp), ORDERS[order], _ptr(perm),
                                       _ptr(U), _ptr(dead), _ptr(delta), _ptr(ws), ws.numel(),
                                       _stream(stream)),
           "gq_prepare_hinv_ordered")
    return perm, U, dead, delta, ws


def gq_prepare_hinv_static(H: torch.Tensor, damp: float = 0.01, reverse: bool = False, U=None,
                           dead=None, delta=None, status=None, stream=None):
    """gq_prepare_hinv on the library's built-in scratch (n <= 1024; no device allocation by
    the library).  Returns (U, dead, delta, status) with status a device int32 [1]."""
    n = H.shape[0]
    _need(H, torch.float64, (n, n), "H")
    dev = H.device
    U = torch.empty((n, n), dtype=torch.float32, device=dev) if U is None else U
    dead = torch.empty(n, dtype=torch.uint8, device=dev) if dead is None else dead
    delta = torch.empty(1, dtype=torch.float64, device=dev) if delta is None else delta
    status = torch.empty(1, dtype=torch.int32, device=dev) if status is None else status
    _need(U, torch.float32, (n, n), "U")
    _need(dead, torch.uint8, (n,), "dead")
    _need(delta, torch.float64, (1,), "delta")
    _need(status, torch.int32, (1,), "status")
    for t, name in ((U, "U"), (dead, "dead"), (delta, "delta"), (status, "status")):
        if t.device != dev:
            raise ValueError(f"{name}: on {t.device}, H is on {dev}")
    _check(LIB.gq_prepare_hinv_static(_ptr(H), n, float(damp), int(bool(reverse)), _ptr(U),
                                      _ptr(dead), _ptr(delta), _ptr(status), _stream(stream)),
           "gq_prepare_hinv_static")
    return U, dead, delta, status


@dataclass
class QuantCfg:
    bits: int = 4
    group_size: int = 0
    reverse: bool = False
    clip: bool | str = True  # True clamp, False clip-free ladder, "unbounded" lattice s Z
    ladder: float = 1.25
    ladder_max: int = 8
    spacing: str = "uniform"  # or "zsic": per-column steps, kappa_j = U_jj / geomean(U)

    def c(self) -> _Cfg:
        if self.spacing not in ("uniform", "zsic"):
            raise ValueError(f"unknown spacing {self.spacing!r}")
        clip = 2 if self.clip == "unbounded" else int(bool(self.clip))
        return _Cfg(int(self.bits), int(self.group_size), int(bool(self.reverse)), clip,
                    float(self.ladder), int(self.ladder_max), 1 if self.spacing == "zsic" else 0)


def gq_quantize_workspace_size(m: int, n: int, cfg: QuantCfg) -> int:
    c = cfg.c()
    return int(LIB.gq_quantize_workspace_size(m, n, ctypes.byref(c)))


def n_words(n: int, bits: int) -> int:
    return (n * bits + 31) // 32


def gq_quantize_layer(W: torch.Tensor, U: torch.Tensor, dead, delta, cfg: QuantCfg,
                      codes=None, scales=None, zeros=None, loss=None, ws=None, stream=None):
    """Run the column loop; returns (codes uint32 [m, words] as int32 view, scales, zeros, loss, ws)."""
    m, n = W.shape
    if not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous cuda tensor")
    dev = W.device
    _need(U, torch.float32, (n, n), "U")
    G = 1 if cfg.group_size == 0 else -(-n // cfg.group_size)
    ncols = n if cfg.clip == "unbounded" else n_words(n, cfg.bits)
    codes = torch.empty((m, ncols), dtype=torch.int32, device=dev) if codes is None else codes
    scales = torch.empty((m, G), dtype=torch.float32, device=dev) if scales is None else scales
    zeros = torch.empty((m, G), dtype=torch.uint8, device=dev) if zeros is None else zeros
    loss = torch.empty(3, dtype=torch.float64, device=dev) if loss is None else loss
    # a rejected configuration sizes to 0; the call itself then reports the precise status
    ws = workspace(gq_quantize_workspace_size(m, n, cfg), dev) if ws is None else ws
    c = cfg.c()
    _check(LIB.gq_quantize_layer(_ptr(W), _dtype_code(W), m, n, _ptr(U), _ptr(dead), _ptr(delta),
                                 ctypes.byref(c), _ptr(codes), _ptr(scales), _ptr(zeros),
                                 _ptr(loss), _ptr(ws), ws.numel(), _stream(stream)),
           "gq_quantize_layer")
    return codes, scales, zeros, loss, ws


def gq_quantize_layer_ordered(W: torch.Tensor, U: torch.Tensor, dead, delta, cfg: QuantCfg,
                              perm: torch.Tensor, codes=None, scales=None, zeros=None, loss=None,
                              ws=None, stream=None):
    """gq_quantize_layer with the columns in the order perm (from gq_prepare_hinv_ordered);
    codes stay indexed by original column, groups follow the processing order."""
    m, n = W.shape
    if not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous cuda tensor")
    dev = W.device
    _need(U, torch.float32, (n, n), "U")
    _need(perm, torch.int32, (n,), "perm")
    G = 1 if cfg.group_size == 0 else -(-n // cfg.group_size)
    ncols = n if cfg.clip == "unbounded" else n_words(n, cfg.bits)
    codes = torch.empty((m, ncols), dtype=torch.int32, device=dev) if codes is None else codes
    scales = torch.empty((m, G), dtype=torch.float32, device=dev) if scales is None else scales
    zeros = torch.empty((m, G), dtype=torch.uint8, device=dev) if zeros is None else zeros
    loss = torch.empty(3, dtype=torch.float64, device=dev) if loss is None else loss
    ws = workspace(gq_quantize_workspace_size(m, n, cfg), dev) if ws is None else ws
    c = cfg.c()
    _check(LIB.gq_quantize_layer_ordered(_ptr(W), _dtype_code(W), m, n, _ptr(U), _ptr(dead),
                                         _ptr(delta), ctypes.byref(c), _ptr(perm), _ptr(codes),
                                         _ptr(scales), _ptr(zeros), _ptr(loss), _ptr(ws),
                                         ws.numel(), _stream(stream)),
           "gq_quantize_layer_ordered")
    return codes, scales, zeros, loss, ws


def gq_ssqr_quantize_layer(W: torch.Tensor, U: torch.Tensor, dead, delta, bits: int,
                           density: float, steps: int = 20, max_doublings: int = 12,
                           capacity: int | None = None, ws=None, stream=None):
    """SSQR on the device: per-row scale search for a target outlier density, outliers kept
    in full precision.  Returns dict(codes (packed, outliers 0), scales [m], zeros [m],
    alpha [m] fp64, row_ptr [m+1] int64, col_idx, values (CSR of the outliers), loss, ws)."""
    m, n = W.shape
    if not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous cuda tensor")
    dev = W.device
    _need(U, torch.float32, (n, n), "U")
    if dead is not None:
        _need(dead, torch.uint8, (n,), "dead")
    if delta is not None:
        _need(delta, torch.float64, (1,), "delta")
    limit = int(density * n + 1e-9)
    cap = m * max(limit, 0) if capacity is None else int(capacity)
    codes = torch.empty((m, n_words(n, bits)), dtype=torch.int32, device=dev)
    scales = torch.empty(m, dtype=torch.float32, device=dev)
    zeros = torch.empty(m, dtype=torch.uint8, device=dev)
    alpha = torch.empty(m, dtype=torch.float64, device=dev)
    row_ptr = torch.empty(m + 1, dtype=torch.int64, device=dev)
    col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    values = torch.empty(max(cap, 1), dtype=torch.float32, device=dev)
    loss = torch.empty(3, dtype=torch.float64, device=dev)
    ws = workspace(int(LIB.gq_ssqr_workspace_size(m, n)), dev) if ws is None else ws
    _check(LIB.gq_ssqr_quantize_layer(_ptr(W), _dtype_code(W), m, n, _ptr(U), _ptr(dead),
                                      _ptr(delta), int(bits), float(density), int(steps),
                                      int(max_doublings), _ptr(codes), _ptr(scales),
                                      _ptr(zeros), _ptr(alpha), _ptr(row_ptr), _ptr(col_idx),
                                      _ptr(values), cap, _ptr(loss), _ptr(ws), ws.numel(),
                                      _stream(stream)),
           "gq_ssqr_quantize_layer")
    return dict(codes=codes, scales=scales, zeros=zeros, alpha=alpha, row_ptr=row_ptr,
                col_idx=col_idx, values=values, loss=loss, ws=ws)


def gq_hptq_quantize_layer(W: torch.Tensor, U: torch.Tensor, dead, delta, bits: int,
                           budget: float, steps: int = 12, max_doublings: int = 12, ws=None,
                           stream=None):
    """HPTQ rate control on the device: one lattice factor for the layer, the smallest whose
    Huffman-coded integers fit ``budget`` bits per weight.  Returns dict(codes int32 [m, n],
    scales [m], alpha [1] fp64, total_bits [1] int64, loss, ws)."""
    m, n = W.shape
    if not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous cuda tensor")
    dev = W.device
    _need(U, torch.float32, (n, n), "U")
    if dead is not None:
        _need(dead, torch.uint8, (n,), "dead")
    if delta is not None:
        _need(delta, torch.float64, (1,), "delta")
    codes = torch.empty((m, n), dtype=torch.int32, device=dev)
    scales = torch.empty(m, dtype=torch.float32, device=dev)
    alpha = torch.empty(1, dtype=torch.float64, device=dev)
    total = torch.empty(1, dtype=torch.int64, device=dev)
    loss = torch.empty(3, dtype=torch.float64, device=dev)
    ws = workspace(int(LIB.gq_hptq_workspace_size(m, n)), dev) if ws is None else ws
    _check(LIB.gq_hptq_quantize_layer(_ptr(W), _dtype_code(W), m, n, _ptr(U), _ptr(dead),
                                      _ptr(delta), int(bits), float(budget), int(steps),
                                      int(max_doublings), _ptr(codes), _ptr(scales),
                                      _ptr(alpha), _ptr(total), _ptr(loss), _ptr(ws),
                                      ws.numel(), _stream(stream)),
           "gq_hptq_quantize_layer")
    return dict(codes=codes, scales=scales, alpha=alpha, total_bits=total, loss=loss, ws=ws)


def gq_zsic_spacing(U: torch.Tensor, kappa=None, stream=None) -> torch.Tensor:
    """ZSIC column factors kappa_j = U_jj / geomean(U_kk) (fp64, processing order)."""
    n = U.shape[0]
    _need(U, torch.float32, (n, n), "U")
    kappa = torch.empty(n, dtype=torch.float64, device=U.device) if kappa is None else kappa
    _need(kappa, torch.float64, (n,), "kappa")
    _check(LIB.gq_zsic_spacing(_ptr(U), n, _ptr(kappa), _stream(stream)), "gq_zsic_spacing")
    return kappa


def gq_huffman_encode(codes: torch.Tensor, stream_words: int | None = None, ws=None,
                      stream=None, out=None, lengths=None, cw=None, info=None):
    """Canonical Huffman coding of int32 codes on the device.  Returns (stream uint64 words as
    an int64 tensor, lengths uint8[4096], codewords int64[4096], info int64[4]
    = [min value, symbols spanned, total bits, longest codeword], workspace); pass the
    returned buffers back in to reuse them."""
    if not codes.is_cuda or codes.dtype != torch.int32 or not codes.is_contiguous():
        raise ValueError("codes: expected a contiguous cuda int32 tensor")
    count = codes.numel()
    dev = codes.device
    words = (count if stream_words is None else int(stream_words)) if out is None else out.numel()
    out = torch.empty(max(words, 1), dtype=torch.int64, device=dev) if out is None else out
    lengths = torch.empty(4096, dtype=torch.uint8, device=dev) if lengths is None else lengths
    cw = torch.empty(4096, dtype=torch.int64, device=dev) if cw is None else cw
    info = torch.empty(4, dtype=torch.int64, device=dev) if info is None else info
    _need(out, torch.int64, (out.numel(),), "out")
    _need(lengths, torch.uint8, (4096,), "lengths")
    _need(cw, torch.int64, (4096,), "cw")
    _need(info, torch.int64, (4,), "info")
    ws = workspace(int(LIB.gq_huffman_workspace_size(count)), dev) if ws is None else ws
    _check(LIB.gq_huffman_encode(_ptr(codes), count, _ptr(out), out.numel(), _ptr(lengths),
                                 _ptr(cw), _ptr(info), _ptr(ws), ws.numel(), _stream(stream)),
           "gq_huffman_encode")
    return out, lengths, cw, info, ws


def gq_debug_wait_test(poll_limit: int = 0, withhold_arrival: bool = False) -> None:
    """Test setting of the bounded waits (see gq.h); gq_debug_wait_test() restores the
    defaults."""
    _check(LIB.gq_debug_wait_test(int(poll_limit), int(bool(withhold_arrival))),
           "gq_debug_wait_test")


def gq_workspace_status(ws: torch.Tensor, stream=None):
    """(status code, ladder rounds) recorded in a workspace by its last call; synchronizes."""
    r = ctypes.c_int(0)
    code = LIB.gq_workspace_status(_ptr(ws), ctypes.byref(r), _stream(stream))
    return int(code), int(r.value)
