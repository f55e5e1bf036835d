"""Thin Python binding of libsvg2 (include/svg2.h): argument marshalling only.

Every function here has the name of the C entry point it calls.  PyTorch supplies device memory
and the current CUDA stream; all of the method's steps run in the library's sm_100a kernels.
There is no fallback: if libsvg2.so is missing or a call fails, an exception is raised.
The library sees only pointers, so each wrapper checks its tensors' dtypes and element counts
against the sizes of the call (include/svg2.h) before it takes their pointers.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Dict, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
RELEASE_LIB_PATH = os.path.join(_PKG, "libsvg2.so")
# The debug build: the same ABI, and every data-derived index a kernel clamps or skips is also latched
# as SVG2_ERR_DEVICE_BOUNDS in the status word (built by build.build(debug=True)).
DEBUG_LIB_PATH = os.path.join(_PKG, "libsvg2_debug.so")
LIB_PATH = RELEASE_LIB_PATH

SVG2_BF16, SVG2_F32 = 0, 1
SVG2_INIT_GIVEN, SVG2_INIT_KMEANSPP = 0, 1
MAX_CLUSTERS = 1024
DEFAULT_SEED_TOKENS = 16384  # SVG2_DEFAULT_SEED_TOKENS

_EXPORTS = ("svg2_status_string", "svg2_workspace_size", "svg2_check_status", "svg2_kmeanspp", "svg2_kmeans", "svg2_select",
            "svg2_select_from_weights", "svg2_sort", "svg2_gather", "svg2_permute", "svg2_sparse_attn",
            "svg2_unpermute", "svg2_layer", "svg2_layer_host", "svg2_selftest_mma", "svg2_sparse_attn_noalloc",
            "svg2_dense_attn_workspace_size", "svg2_dense_attn", "svg2_driver_create", "svg2_driver_destroy",
            "svg2_driver_cache_bytes", "svg2_driver_bind_cache", "svg2_driver_reset", "svg2_driver_workspace_size",
            "svg2_driver_plan", "svg2_driver_layer", "svg2_set_wait_budget", "svg2_quantize_e4m3",
            "svg2_sparse_attn_fp8")

_lib = None


class Svg2Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


class SvgParams(ctypes.Structure):
    _fields_ = [("nQ", ctypes.c_int), ("nK", ctypes.c_int), ("iters", ctypes.c_int), ("init", ctypes.c_int),
                ("top_p", ctypes.c_float), ("scale", ctypes.c_float), ("seed_tokens", ctypes.c_int),
                ("fuse_unpermute", ctypes.c_int), ("attn_fp8", ctypes.c_int)]


class SvgDriverConfig(ctypes.Structure):
    _fields_ = [("num_steps", ctypes.c_int), ("num_layers", ctypes.c_int), ("dense_steps", ctypes.c_int),
                ("warm_iters", ctypes.c_int), ("layer", SvgParams)]


class SvgLayerOutputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "labels_q", "labels_k", "count_q", "count_k", "perm_q", "perm_k", "q_off", "k_off", "weights", "mask",
        "sel_count", "sel_idx", "stream_len")]


def lib() -> ctypes.CDLL:
    """Load libsvg2.so (built in-tree by sparse_attention_video_head_b200/build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python sparse_attention_video_head_b200/build.py`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.svg2_status_string.argtypes = [I]
        L.svg2_status_string.restype = ctypes.c_char_p
        L.svg2_workspace_size.argtypes = [I, I, I, I, I, I, ctypes.POINTER(S)]
        L.svg2_check_status.argtypes = [P, P, ctypes.POINTER(I), ctypes.POINTER(ctypes.c_uint32),
                                        ctypes.POINTER(ctypes.c_uint32)]
        L.svg2_set_wait_budget.argtypes = [P, ctypes.c_uint64, P]
        L.svg2_kmeanspp.argtypes = [P, I, I, I, I, I, I, P, I, P, P, S, P]
        L.svg2_kmeans.argtypes = [P, I, I, I, I, I, I, I, I, P, I, P, P, P, P, P, P, S, P]
        L.svg2_select.argtypes = [P, P, P, I, I, I, I, I, F, F, P, P, P, P, P, P, S, P]
        L.svg2_select_from_weights.argtypes = [P, P, I, I, I, I, F, P, P, P, P, P, S, P]
        L.svg2_sort.argtypes = [P, I, I, I, I, P, P, P, P, S, P]
        L.svg2_gather.argtypes = [P, I, P, I, I, I, I, P, P]
        L.svg2_permute.argtypes = [P, I, P, I, I, I, I, I, P, P, P, P, P, S, P]
        L.svg2_sparse_attn.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, S, P]
        L.svg2_unpermute.argtypes = [P, P, I, I, I, I, P, P]
        L.svg2_layer.argtypes = [P, P, P, I, I, I, I, I, ctypes.POINTER(SvgParams), P, P, P, P, P,
                                 ctypes.POINTER(SvgLayerOutputs), P, S, P]
        L.svg2_layer_host.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, ctypes.POINTER(SvgParams), P, P, P, P,
                                      I, P, S, P, P]
        L.svg2_selftest_mma.argtypes = [P, P, I, P, P, P, P, S, P]
        L.svg2_sparse_attn_noalloc.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, P]
        L.svg2_dense_attn_workspace_size.argtypes = [I, I, I, I, ctypes.POINTER(S)]
        L.svg2_dense_attn.argtypes = [P, P, P, I, I, I, I, F, P, P, S, P]
        L.svg2_quantize_e4m3.argtypes = [P, I, P, I, I, I, I, P, P, P]
        L.svg2_sparse_attn_fp8.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, S, P]
        L.svg2_driver_create.argtypes = [ctypes.POINTER(SvgDriverConfig), I, I, I, I, ctypes.POINTER(P)]
        L.svg2_driver_destroy.argtypes = [P]
        L.svg2_driver_cache_bytes.argtypes = [P, ctypes.POINTER(S)]
        L.svg2_driver_bind_cache.argtypes = [P, P, S]
        L.svg2_driver_reset.argtypes = [P]
        L.svg2_driver_workspace_size.argtypes = [P, ctypes.POINTER(S)]
        L.svg2_driver_plan.argtypes = [P, I, I, ctypes.POINTER(I)]
        L.svg2_driver_layer.argtypes = [P, I, I, P, P, P, P, P, P, P, S, P]
        for name in _EXPORTS:
            if name != "svg2_status_string":
                getattr(L, name).restype = I
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().svg2_status_string(int(code)).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise Svg2Error(rc, what)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libsvg2 takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libsvg2 takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _hp(t: torch.Tensor):
    """Host pointer of a contiguous CPU tensor (argument marshalling only)."""
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous host tensor")
    return ctypes.c_void_p(t.data_ptr())


_BF16, _F32, _F64, _I32, _U8 = (torch.bfloat16,), (torch.float32,), (torch.float64,), (torch.int32,), (torch.uint8,)
_DATA = (torch.bfloat16, torch.float32)
_E4M3 = (torch.uint8, torch.float8_e4m3fn)  # E4M3 codes, as raw bytes or as torch's own view of them


def _arg(t: Optional[torch.Tensor], name: str, dtypes, numel: int, optional: bool = False, host: bool = False):
    """Pointer of a tensor argument after checking it against the header's contract: its dtype and
    room for the `numel` elements the library reads or writes through it.  The library sees only a
    pointer, so a smaller buffer would be read or written past its end on the device; these checks
    run before the pointer is taken."""
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(x) for x in dtypes)}")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, the call uses {numel}")
    return _hp(t) if host else _p(t)


def _dims(t: torch.Tensor, name: str, ndim: int = 4):
    if t is None or t.dim() != ndim:
        raise ValueError(f"{name} must be a {ndim}-D tensor")
    return tuple(int(x) for x in t.shape)


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SVG2_BF16
    if t.dtype == torch.float32:
        return SVG2_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def svg2_workspace_size(B: int, H: int, N: int, d: int, nQ: int, nK: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().svg2_workspace_size(B, H, N, d, nQ, nK, ctypes.byref(out)), "svg2_workspace_size")
    return int(out.value)


def workspace(B: int, H: int, N: int, d: int, nQ: int, nK: int, device=None) -> torch.Tensor:
    """A workspace tensor for these sizes (device memory from torch; the status word starts at 0)."""
    return torch.zeros(svg2_workspace_size(B, H, N, d, nQ, nK), dtype=torch.uint8, device=device or "cuda")


def svg2_check_status(ws: torch.Tensor, stream=None):
    code = ctypes.c_int(0)
    where = ctypes.c_uint32(0)
    info = (ctypes.c_uint32 * 2)()
    _check(lib().svg2_check_status(_p(ws), _stream(stream), ctypes.byref(code), ctypes.byref(where), info),
           "svg2_check_status")
    return int(code.value), int(where.value), (int(info[0]), int(info[1]))


def use_debug_library(on: bool = True) -> None:
    """Make the following calls go to libsvg2_debug.so (on) or back to libsvg2.so (off)."""
    global LIB_PATH, _lib
    LIB_PATH = DEBUG_LIB_PATH if on else RELEASE_LIB_PATH
    _lib = None


def svg2_set_wait_budget(ws: torch.Tensor, cycles: int, stream=None):
    """Budget (SM clock cycles) of the bounded waits in the attention and assignment kernels for later
    calls with this workspace; 0 restores the default.  Diagnostics only."""
    if cycles < 0:
        raise ValueError("cycles must be >= 0")
    _check(lib().svg2_set_wait_budget(_arg(ws, "ws", _U8, 256), int(cycles), _stream(stream)),
           "svg2_set_wait_budget")


def raise_on_device_error(ws: torch.Tensor, stream=None):
    code, where, info = svg2_check_status(ws, stream)
    if code != 0:
        raise Svg2Error(code, f"device status (kernel tag {where}, info {info})")


def svg2_kmeanspp(X: torch.Tensor, k: int, u: torch.Tensor, centroids: torch.Tensor, ws: torch.Tensor,
                  seed_tokens: int = DEFAULT_SEED_TOKENS, stream=None):
    B, H, N, d = _dims(X, "X")
    BH = B * H
    _check(lib().svg2_kmeanspp(_arg(X, "X", _DATA, 0), _dtype(X), B, H, N, d, k, _arg(u, "u", _F64, BH * k),
                               int(seed_tokens), _arg(centroids, "centroids", _F32, BH * k * d), _p(ws),
                               _nbytes(ws), _stream(stream)), "svg2_kmeanspp")


def svg2_kmeans(X: torch.Tensor, k: int, iters: int, init: int, centroids: torch.Tensor, labels: torch.Tensor,
                counts: torch.Tensor, ws: torch.Tensor, u: Optional[torch.Tensor] = None,
                perm: Optional[torch.Tensor] = None, offsets: Optional[torch.Tensor] = None,
                seed_tokens: int = DEFAULT_SEED_TOKENS, stream=None):
    B, H, N, d = _dims(X, "X")
    BH = B * H
    u_ptr = _arg(u, "u", _F64, BH * k) if init == SVG2_INIT_KMEANSPP else _p(u)
    _check(lib().svg2_kmeans(_arg(X, "X", _DATA, 0), _dtype(X), B, H, N, d, k, iters, init, u_ptr, int(seed_tokens),
                             _arg(centroids, "centroids", _F32, BH * k * d), _arg(labels, "labels", _I32, BH * N),
                             _arg(counts, "counts", _I32, BH * k), _arg(perm, "perm", _I32, BH * N, optional=True),
                             _arg(offsets, "offsets", _I32, BH * (k + 1), optional=True), _p(ws), _nbytes(ws),
                             _stream(stream)), "svg2_kmeans")


def svg2_select(cq: torch.Tensor, ck: torch.Tensor, count_k: torch.Tensor, top_p: float, scale: float,
                mask: torch.Tensor, sel_count: torch.Tensor, sel_idx: torch.Tensor, ws: torch.Tensor,
                weights: Optional[torch.Tensor] = None, stream_len: Optional[torch.Tensor] = None, stream=None):
    B, H, nQ, d = _dims(cq, "cq")
    nK = _dims(ck, "ck")[2]
    BH = B * H
    _check(lib().svg2_select(_arg(cq, "cq", _F32, 0), _arg(ck, "ck", _F32, BH * nK * d),
                             _arg(count_k, "count_k", _I32, BH * nK), B, H, nQ, nK, d, float(top_p), float(scale),
                             _arg(weights, "weights", _F32, BH * nQ * nK, optional=True),
                             _arg(mask, "mask", _U8, BH * nQ * nK), _arg(sel_count, "sel_count", _I32, BH * nQ),
                             _arg(sel_idx, "sel_idx", _I32, BH * nQ * nK),
                             _arg(stream_len, "stream_len", _I32, BH * nQ, optional=True), _p(ws), _nbytes(ws),
                             _stream(stream)), "svg2_select")


def svg2_select_from_weights(weights: torch.Tensor, count_k: torch.Tensor, top_p: float, mask: torch.Tensor,
                             sel_count: torch.Tensor, sel_idx: torch.Tensor, ws: torch.Tensor,
                             stream_len: Optional[torch.Tensor] = None, stream=None):
    B, H, nQ, nK = _dims(weights, "weights")
    BH = B * H
    _check(lib().svg2_select_from_weights(_arg(weights, "weights", _F32, 0), _arg(count_k, "count_k", _I32, BH * nK),
                                          B, H, nQ, nK, float(top_p), _arg(mask, "mask", _U8, BH * nQ * nK),
                                          _arg(sel_count, "sel_count", _I32, BH * nQ),
                                          _arg(sel_idx, "sel_idx", _I32, BH * nQ * nK),
                                          _arg(stream_len, "stream_len", _I32, BH * nQ, optional=True), _p(ws),
                                          _nbytes(ws), _stream(stream)), "svg2_select_from_weights")


def svg2_sort(labels: torch.Tensor, k: int, perm: torch.Tensor, offsets: torch.Tensor, counts: Optional[torch.Tensor],
              ws: torch.Tensor, stream=None):
    B, H, N = _dims(labels, "labels", 3)
    BH = B * H
    _check(lib().svg2_sort(_arg(labels, "labels", _I32, 0), B, H, N, k, _arg(perm, "perm", _I32, BH * N),
                           _arg(offsets, "offsets", _I32, BH * (k + 1)),
                           _arg(counts, "counts", _I32, BH * k, optional=True), _p(ws), _nbytes(ws),
                           _stream(stream)), "svg2_sort")


def svg2_gather(X: torch.Tensor, perm: torch.Tensor, Xp: torch.Tensor, stream=None):
    B, H, N, d = _dims(X, "X")
    BH = B * H
    _check(lib().svg2_gather(_arg(X, "X", _DATA, 0), _dtype(X), _arg(perm, "perm", _I32, BH * N), B, H, N, d,
                             _arg(Xp, "Xp", _BF16, BH * N * d), _stream(stream)), "svg2_gather")


def svg2_permute(X: torch.Tensor, labels: torch.Tensor, k: int, Xp: torch.Tensor, perm: torch.Tensor,
                 offsets: torch.Tensor, counts: Optional[torch.Tensor], ws: torch.Tensor, stream=None):
    B, H, N, d = _dims(X, "X")
    BH = B * H
    _check(lib().svg2_permute(_arg(X, "X", _DATA, 0), _dtype(X), _arg(labels, "labels", _I32, BH * N), B, H, N, d, k,
                              _arg(Xp, "Xp", _BF16, BH * N * d), _arg(perm, "perm", _I32, BH * N),
                              _arg(offsets, "offsets", _I32, BH * (k + 1)),
                              _arg(counts, "counts", _I32, BH * k, optional=True), _p(ws), _nbytes(ws),
                              _stream(stream)), "svg2_permute")


def _attn_args(Qp, Kp, Vp, q_off, k_off, sel_count, sel_idx, O, perm_q):
    """Sizes and checked pointers (Qp, Kp, Vp, q_off, k_off, sel_count, sel_idx, O, perm_q) of an
    attention call; nQ and nK come from the offsets' last dimension."""
    B, H, N, d = _dims(Qp, "Qp")
    if q_off is None or k_off is None or q_off.dim() < 1 or k_off.dim() < 1:
        raise ValueError("q_off and k_off are required")
    BH = B * H
    nQ = int(q_off.shape[-1]) - 1
    nK = int(k_off.shape[-1]) - 1
    ptr = (_arg(Qp, "Qp", _BF16, 0), _arg(Kp, "Kp", _BF16, BH * N * d), _arg(Vp, "Vp", _BF16, BH * N * d),
           _arg(q_off, "q_off", _I32, BH * (nQ + 1)), _arg(k_off, "k_off", _I32, BH * (nK + 1)),
           _arg(sel_count, "sel_count", _I32, BH * nQ), _arg(sel_idx, "sel_idx", _I32, BH * nQ * nK),
           _arg(O, "O", _BF16, BH * N * d), _arg(perm_q, "perm_q", _I32, BH * N, optional=True))
    return B, H, N, d, nQ, nK, ptr


def svg2_sparse_attn(Qp: torch.Tensor, Kp: torch.Tensor, Vp: torch.Tensor, q_off: torch.Tensor, k_off: torch.Tensor,
                     sel_count: torch.Tensor, sel_idx: torch.Tensor, scale: float, O: torch.Tensor, ws: torch.Tensor,
                     perm_q: Optional[torch.Tensor] = None, stream=None):
    B, H, N, d, nQ, nK, ptr = _attn_args(Qp, Kp, Vp, q_off, k_off, sel_count, sel_idx, O, perm_q)
    _check(lib().svg2_sparse_attn(*ptr[:7], B, H, N, d, nQ, nK, float(scale), ptr[8], ptr[7], _p(ws), _nbytes(ws),
                                  _stream(stream)), "svg2_sparse_attn")


def svg2_quantize_e4m3(X: torch.Tensor, X8: torch.Tensor, scale: torch.Tensor,
                       perm: Optional[torch.Tensor] = None, stream=None):
    """Per-(b,h) E4M3 codes of X (rows gathered through perm when given) and their scales."""
    B, H, N, d = _dims(X, "X")
    BH = B * H
    _check(lib().svg2_quantize_e4m3(_arg(X, "X", _DATA, 0), _dtype(X), _arg(perm, "perm", _I32, BH * N, optional=True),
                                    B, H, N, d, _arg(X8, "X8", _E4M3, BH * N * d), _arg(scale, "scale", _F32, BH),
                                    _stream(stream)), "svg2_quantize_e4m3")


def svg2_sparse_attn_fp8(Qp8: torch.Tensor, Kp8: torch.Tensor, Vp8: torch.Tensor, scale_q: torch.Tensor,
                         scale_k: torch.Tensor, scale_v: torch.Tensor, q_off: torch.Tensor, k_off: torch.Tensor,
                         sel_count: torch.Tensor, sel_idx: torch.Tensor, scale: float, O: torch.Tensor,
                         ws: torch.Tensor, perm_q: Optional[torch.Tensor] = None, stream=None):
    """svg2_sparse_attn on E4M3 codes with per-(b,h) dequantisation scales (d = 128)."""
    B, H, N, d = _dims(Qp8, "Qp8")
    if q_off is None or k_off is None or q_off.dim() < 1 or k_off.dim() < 1:
        raise ValueError("q_off and k_off are required")
    BH, n = B * H, B * H * N * d
    nQ = int(q_off.shape[-1]) - 1
    nK = int(k_off.shape[-1]) - 1
    _check(lib().svg2_sparse_attn_fp8(
        _arg(Qp8, "Qp8", _E4M3, 0), _arg(Kp8, "Kp8", _E4M3, n), _arg(Vp8, "Vp8", _E4M3, n),
        _arg(scale_q, "scale_q", _F32, BH), _arg(scale_k, "scale_k", _F32, BH), _arg(scale_v, "scale_v", _F32, BH),
        _arg(q_off, "q_off", _I32, BH * (nQ + 1)), _arg(k_off, "k_off", _I32, BH * (nK + 1)),
        _arg(sel_count, "sel_count", _I32, BH * nQ), _arg(sel_idx, "sel_idx", _I32, BH * nQ * nK), B, H, N, d, nQ,
        nK, float(scale), _arg(perm_q, "perm_q", _I32, BH * N, optional=True), _arg(O, "O", _BF16, n), _p(ws),
        _nbytes(ws), _stream(stream)), "svg2_sparse_attn_fp8")


def svg2_dense_attn_workspace_size(B: int, H: int, N: int, d: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().svg2_dense_attn_workspace_size(B, H, N, d, ctypes.byref(out)), "svg2_dense_attn_workspace_size")
    return int(out.value)


def dense_workspace(B: int, H: int, N: int, d: int, device=None) -> torch.Tensor:
    """A workspace tensor for svg2_dense_attn (device memory from torch; the status word starts at 0)."""
    return torch.zeros(svg2_dense_attn_workspace_size(B, H, N, d), dtype=torch.uint8, device=device or "cuda")


def svg2_dense_attn(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, scale: float, O: torch.Tensor,
                    ws: torch.Tensor, stream=None):
    B, H, N, d = _dims(Q, "Q")
    n = B * H * N * d
    _check(lib().svg2_dense_attn(_arg(Q, "Q", _BF16, 0), _arg(K, "K", _BF16, n), _arg(V, "V", _BF16, n), B, H, N, d,
                                 float(scale), _arg(O, "O", _BF16, n), _p(ws), _nbytes(ws), _stream(stream)),
           "svg2_dense_attn")


def svg2_sparse_attn_noalloc(Qp: torch.Tensor, Kp: torch.Tensor, Vp: torch.Tensor, q_off: torch.Tensor,
                             k_off: torch.Tensor, sel_count: torch.Tensor, sel_idx: torch.Tensor, scale: float,
                             O: torch.Tensor, perm_q: Optional[torch.Tensor] = None,
                             device_status: Optional[torch.Tensor] = None, stream=None):
    """svg2_sparse_attn for callers that cannot allocate: scratch is the library's fixed array."""
    B, H, N, d, nQ, nK, ptr = _attn_args(Qp, Kp, Vp, q_off, k_off, sel_count, sel_idx, O, perm_q)
    if device_status is not None and _nbytes(device_status) < 16:
        raise ValueError("device_status: the status word takes 16 bytes")
    _check(lib().svg2_sparse_attn_noalloc(*ptr[:7], B, H, N, d, nQ, nK, float(scale), ptr[8], ptr[7],
                                          _p(device_status), _stream(stream)), "svg2_sparse_attn_noalloc")


def svg2_unpermute(Op: torch.Tensor, perm: torch.Tensor, O: torch.Tensor, stream=None):
    B, H, N, d = _dims(Op, "Op")
    _check(lib().svg2_unpermute(_arg(Op, "Op", _BF16, 0), _arg(perm, "perm", _I32, B * H * N), B, H, N, d,
                                _arg(O, "O", _BF16, B * H * N * d), _stream(stream)), "svg2_unpermute")


@dataclass
class LayerParams:
    nQ: int
    nK: int
    iters: int
    init: int = SVG2_INIT_KMEANSPP
    top_p: float = 0.9
    scale: float = 1.0 / 128 ** 0.5
    fuse_unpermute: int = 1
    seed_tokens: int = DEFAULT_SEED_TOKENS
    attn_fp8: int = 0

    def c(self) -> SvgParams:
        return SvgParams(self.nQ, self.nK, self.iters, self.init, self.top_p, self.scale, self.seed_tokens,
                         self.fuse_unpermute, self.attn_fp8)


def layer_output_buffers(B: int, H: int, N: int, nQ: int, nK: int, device="cuda") -> Dict[str, torch.Tensor]:
    """Device buffers for every intermediate result the layer can expose (see svg2_layer_outputs)."""
    i32 = dict(dtype=torch.int32, device=device)
    return {
        "labels_q": torch.empty(B, H, N, **i32), "labels_k": torch.empty(B, H, N, **i32),
        "count_q": torch.empty(B, H, nQ, **i32), "count_k": torch.empty(B, H, nK, **i32),
        "perm_q": torch.empty(B, H, N, **i32), "perm_k": torch.empty(B, H, N, **i32),
        "q_off": torch.empty(B, H, nQ + 1, **i32), "k_off": torch.empty(B, H, nK + 1, **i32),
        "weights": torch.empty(B, H, nQ, nK, dtype=torch.float32, device=device),
        "mask": torch.empty(B, H, nQ, nK, dtype=torch.uint8, device=device),
        "sel_count": torch.empty(B, H, nQ, **i32), "sel_idx": torch.empty(B, H, nQ, nK, **i32),
        "stream_len": torch.empty(B, H, nQ, **i32),
    }


# dtype and element count per (b, h) of each svg2_layer_outputs field
def _layer_out_sizes(N: int, nQ: int, nK: int):
    return {"labels_q": (_I32, N), "labels_k": (_I32, N), "count_q": (_I32, nQ), "count_k": (_I32, nK),
            "perm_q": (_I32, N), "perm_k": (_I32, N), "q_off": (_I32, nQ + 1), "k_off": (_I32, nK + 1),
            "weights": (_F32, nQ * nK), "mask": (_U8, nQ * nK), "sel_count": (_I32, nQ),
            "sel_idx": (_I32, nQ * nK), "stream_len": (_I32, nQ)}


def _layer_args(Q, K, V, params: "LayerParams", cq, ck, uq, uk, host: bool = False):
    """Sizes and checked pointers (Q, K, V, uq, uk, cq, ck) of a layer call; Q, K, V are host tensors
    when `host` is set (svg2_layer_host), everything else is on the device."""
    B, H, N, d = _dims(Q, "Q")
    BH = B * H
    n = BH * N * d
    cold = params.init == SVG2_INIT_KMEANSPP
    ptr = (_arg(Q, "Q", _DATA, 0, host=host), _arg(K, "K", (Q.dtype,), n, host=host),
           _arg(V, "V", (Q.dtype,), n, host=host),
           _arg(uq, "uq", _F64, BH * params.nQ) if cold else _p(uq),
           _arg(uk, "uk", _F64, BH * params.nK) if cold else _p(uk),
           _arg(cq, "cq", _F32, BH * params.nQ * d), _arg(ck, "ck", _F32, BH * params.nK * d))
    return B, H, N, d, ptr


def svg2_layer(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, params: LayerParams, cq: torch.Tensor,
               ck: torch.Tensor, O: torch.Tensor, ws: torch.Tensor, uq: Optional[torch.Tensor] = None,
               uk: Optional[torch.Tensor] = None, outs: Optional[Dict[str, torch.Tensor]] = None, stream=None):
    B, H, N, d, ptr = _layer_args(Q, K, V, params, cq, ck, uq, uk)
    prm = params.c()
    c_outs = None
    if outs is not None:
        sizes = _layer_out_sizes(N, params.nQ, params.nK)
        c_outs = SvgLayerOutputs(*[(_arg(outs[n], n, sizes[n][0], B * H * sizes[n][1]).value
                                    if outs.get(n) is not None else None) for n, _ in SvgLayerOutputs._fields_])
    _check(lib().svg2_layer(*ptr[:3], _dtype(Q), B, H, N, d, ctypes.byref(prm), *ptr[3:],
                            _arg(O, "O", _BF16, B * H * N * d), ctypes.byref(c_outs) if c_outs is not None else None,
                            _p(ws), _nbytes(ws), _stream(stream)), "svg2_layer")


def svg2_layer_host(Qh: torch.Tensor, Kh: torch.Tensor, Vh: torch.Tensor, Oh: torch.Tensor, Q: torch.Tensor,
                    K: torch.Tensor, V: torch.Tensor, O: torch.Tensor, params: LayerParams, cq: torch.Tensor,
                    ck: torch.Tensor, ws: torch.Tensor, uq: Optional[torch.Tensor] = None,
                    uk: Optional[torch.Tensor] = None, heads_per_group: int = 0, stream=None, copy_stream=None):
    """The layer with Q, K, V and O in (page-locked) host memory; Q, K, V, O here are the device
    staging buffers.  Copies run on copy_stream, overlapped with the compute of other head groups."""
    B, H, N, d, ptr = _layer_args(Qh, Kh, Vh, params, cq, ck, uq, uk, host=True)
    n = B * H * N * d
    prm = params.c()
    cs = ctypes.c_void_p(copy_stream.cuda_stream) if copy_stream is not None else None
    _check(lib().svg2_layer_host(*ptr[:3], _arg(Oh, "Oh", _BF16, n, host=True), _arg(Q, "Q", (Qh.dtype,), n),
                                 _arg(K, "K", (Qh.dtype,), n), _arg(V, "V", (Qh.dtype,), n), _arg(O, "O", _BF16, n),
                                 _dtype(Qh), B, H, N, d, ctypes.byref(prm), *ptr[3:], int(heads_per_group), _p(ws),
                                 _nbytes(ws), _stream(stream), cs), "svg2_layer_host")


SVG2_STEP_DENSE, SVG2_STEP_COLD, SVG2_STEP_WARM = 0, 1, 2


class Driver:
    """The denoising-loop driver (svg2_driver_*): dense attention for the first `dense_steps` steps,
    then per layer a cold k-means at its first sparse step and warm starts from its own cached
    centroids afterwards.  The cache and the workspace are torch device tensors owned here."""

    def __init__(self, B: int, H: int, N: int, d: int, num_steps: int, num_layers: int, dense_steps: int,
                 warm_iters: int, params: LayerParams, device="cuda", allocate: bool = True):
        self._h = ctypes.c_void_p(None)
        cfg = SvgDriverConfig(num_steps, num_layers, dense_steps, warm_iters, params.c())
        _check(lib().svg2_driver_create(ctypes.byref(cfg), B, H, N, d, ctypes.byref(self._h)), "svg2_driver_create")
        self.shape = (B, H, N, d)
        self.nQ, self.nK = params.nQ, params.nK
        self.cache = self.ws = None
        if allocate:
            self.cache = torch.zeros(self.cache_bytes() // 4, dtype=torch.float32, device=device)
            _check(lib().svg2_driver_bind_cache(self._h, _p(self.cache), self.cache.numel() * 4), "svg2_driver_bind_cache")
            self.ws = torch.zeros(self.workspace_bytes(), dtype=torch.uint8, device=device)

    def cache_bytes(self) -> int:
        out = ctypes.c_size_t(0)
        _check(lib().svg2_driver_cache_bytes(self._h, ctypes.byref(out)), "svg2_driver_cache_bytes")
        return int(out.value)

    def workspace_bytes(self) -> int:
        out = ctypes.c_size_t(0)
        _check(lib().svg2_driver_workspace_size(self._h, ctypes.byref(out)), "svg2_driver_workspace_size")
        return int(out.value)

    def plan(self, step: int, layer: int) -> int:
        kind = ctypes.c_int(-1)
        _check(lib().svg2_driver_plan(self._h, step, layer, ctypes.byref(kind)), "svg2_driver_plan")
        return int(kind.value)

    def reset(self):
        _check(lib().svg2_driver_reset(self._h), "svg2_driver_reset")

    def layer(self, step: int, layer: int, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, O: torch.Tensor,
              uq: Optional[torch.Tensor] = None, uk: Optional[torch.Tensor] = None, stream=None):
        if self.ws is None:
            raise ValueError("this driver was created without a workspace (allocate=False)")
        B, H, N, d = self.shape
        n = B * H * N * d
        _check(lib().svg2_driver_layer(self._h, step, layer, _arg(Q, "Q", _BF16, n), _arg(K, "K", _BF16, n),
                                       _arg(V, "V", _BF16, n), _arg(uq, "uq", _F64, B * H * self.nQ, optional=True),
                                       _arg(uk, "uk", _F64, B * H * self.nK, optional=True), _arg(O, "O", _BF16, n),
                                       _p(self.ws), _nbytes(self.ws), _stream(stream)), "svg2_driver_layer")

    def close(self):
        if self._h:
            lib().svg2_driver_destroy(self._h)
            self._h = ctypes.c_void_p(None)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def svg2_selftest_mma(A: torch.Tensor, Bm: torch.Tensor, V: torch.Tensor, ws: torch.Tensor, stream=None):
    n = _dims(Bm, "Bm", 2)[0]
    C = torch.empty(128, n, dtype=torch.float32, device=A.device)
    O = torch.empty(128, 128, dtype=torch.float32, device=A.device)
    _check(lib().svg2_selftest_mma(_arg(A, "A", _BF16, 128 * 128), _arg(Bm, "Bm", _BF16, n * 128), n,
                                   _arg(V, "V", _BF16, 128 * 128), _p(C), _p(O), _p(ws), _nbytes(ws), _stream(stream)),
           "svg2_selftest_mma")
    return C, O
