"""ctypes front end of the CPU oracle (oracle/svg2_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by bench.py's
cpu_baseline / reference leg.  The product path (the CUDA library and its Python binding) never
imports this module.

Per-head helpers compose the C functions in the order of the pages' Method section
("Sparse VideoGen2" wiki summary): k-means on Q and K, centroid scores, top-p, permutation,
sparse attention, inverse permutation.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svg2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-std=c11", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, f64, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_float
        L.svg2o_kmeanspp.argtypes = [P, i64, i32, i32, P, P, P]
        L.svg2o_kmeanspp.restype = i32
        L.svg2o_assign.argtypes = [P, i64, i32, P, i32, P, P, P]
        L.svg2o_update.argtypes = [P, i64, i32, P, i32, P, P]
        L.svg2o_lloyd.argtypes = [P, i64, i32, i32, i32, P, P, P]
        L.svg2o_select_weights.argtypes = [P, P, P, i32, i32, i32, f64, P]
        L.svg2o_topp.argtypes = [P, P, i32, i32, f32, P]
        L.svg2o_permute.argtypes = [P, i64, i32, P, P]
        L.svg2o_gather_rows.argtypes = [P, P, i64, i32, P]
        L.svg2o_unpermute.argtypes = [P, P, i64, i32, P]
        L.svg2o_sparse_attention_rows.argtypes = [P, P, P, i64, i32, P, P, i32, i32, P, f64, P, i64, P]
        L.svg2o_dense_attention_rows.argtypes = [P, P, P, i64, i32, f64, P, i64, P]
        L.svg2o_e4m3_value.argtypes = [ctypes.c_uint8]
        L.svg2o_e4m3_value.restype = f64
        L.svg2o_e4m3_round.argtypes = [f64]
        L.svg2o_e4m3_round.restype = ctypes.c_uint8
        L.svg2o_quantize_e4m3.argtypes = [P, i64, P, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def kmeanspp(X: np.ndarray, k: int, u: np.ndarray):
    X = _f32(X)
    N, d = X.shape
    u = np.ascontiguousarray(u, dtype=np.float64)
    seeds = np.zeros(k, np.int64)
    C = np.zeros((k, d), np.float64)
    rc = lib().svg2o_kmeanspp(_p(X), N, d, k, _p(u), _p(seeds), _p(C))
    if rc != 0:
        raise RuntimeError(f"svg2o_kmeanspp failed: {rc}")
    return seeds, C


def assign(X: np.ndarray, C: np.ndarray):
    X = _f32(X)
    C = np.ascontiguousarray(C, dtype=np.float64)
    N, d = X.shape
    labels = np.zeros(N, np.int32)
    d1 = np.zeros(N, np.float64)
    d2 = np.zeros(N, np.float64)
    lib().svg2o_assign(_p(X), N, d, _p(C), C.shape[0], _p(labels), _p(d1), _p(d2))
    return labels, d1, d2


def update(X: np.ndarray, labels: np.ndarray, C: np.ndarray):
    X = _f32(X)
    C = np.array(C, dtype=np.float64, copy=True, order="C")
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    counts = np.zeros(C.shape[0], np.int32)
    lib().svg2o_update(_p(X), X.shape[0], X.shape[1], _p(labels), C.shape[0], _p(C), _p(counts))
    return C, counts


def lloyd(X: np.ndarray, C0: np.ndarray, iters: int):
    X = _f32(X)
    C = np.array(C0, dtype=np.float64, copy=True, order="C")
    N, d = X.shape
    labels = np.zeros(N, np.int32)
    counts = np.zeros(C.shape[0], np.int32)
    lib().svg2o_lloyd(_p(X), N, d, C.shape[0], iters, _p(C), _p(labels), _p(counts))
    return C, labels, counts


def select_weights(cq: np.ndarray, ck: np.ndarray, count_k: np.ndarray, scale: float):
    cq, ck = _f32(cq), _f32(ck)
    count_k = np.ascontiguousarray(count_k, dtype=np.int32)
    nQ, d = cq.shape
    nK = ck.shape[0]
    w = np.zeros((nQ, nK), np.float32)
    lib().svg2o_select_weights(_p(cq), _p(ck), _p(count_k), nQ, nK, d, float(scale), _p(w))
    return w


def topp(w: np.ndarray, count_k: np.ndarray, p: float):
    w = _f32(w)
    count_k = np.ascontiguousarray(count_k, dtype=np.int32)
    nQ, nK = w.shape
    mask = np.zeros((nQ, nK), np.uint8)
    lib().svg2o_topp(_p(w), _p(count_k), nQ, nK, float(np.float32(p)), _p(mask))
    return mask


def permute(labels: np.ndarray, k: int):
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    perm = np.zeros(labels.size, np.int32)
    offsets = np.zeros(k + 1, np.int32)
    lib().svg2o_permute(_p(labels), labels.size, k, _p(perm), _p(offsets))
    return perm, offsets


def gather_rows(X: np.ndarray, perm: np.ndarray):
    X = _f32(X)
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    out = np.zeros_like(X)
    lib().svg2o_gather_rows(_p(X), _p(perm), X.shape[0], X.shape[1], _p(out))
    return out


def unpermute(Op: np.ndarray, perm: np.ndarray):
    Op = np.ascontiguousarray(Op, dtype=np.float64)
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    O = np.zeros_like(Op)
    lib().svg2o_unpermute(_p(Op), _p(perm), Op.shape[0], Op.shape[1], _p(O))
    return O


def sparse_attention_rows(Qp, Kp, Vp, q_off, k_off, mask, scale, rows=None):
    Qp, Kp, Vp = _f32(Qp), _f32(Kp), _f32(Vp)
    N, d = Qp.shape
    q_off = np.ascontiguousarray(q_off, dtype=np.int32)
    k_off = np.ascontiguousarray(k_off, dtype=np.int32)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    rows = np.arange(N, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, d), np.float64)
    lib().svg2o_sparse_attention_rows(_p(Qp), _p(Kp), _p(Vp), N, d, _p(q_off), _p(k_off),
                                      q_off.size - 1, k_off.size - 1, _p(mask), float(scale),
                                      _p(rows), rows.size, _p(out))
    return out


def dense_attention_rows(Q, K, V, scale, rows=None):
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    N, d = Q.shape
    rows = np.arange(N, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, d), np.float64)
    lib().svg2o_dense_attention_rows(_p(Q), _p(K), _p(V), N, d, float(scale), _p(rows), rows.size, _p(out))
    return out


def e4m3_value(codes) -> np.ndarray:
    """Values of E4M3 codes (svg2o_e4m3_value), float64, same shape."""
    c = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib().svg2o_e4m3_value(i) for i in range(256)], np.float64)
    return table[c]


def e4m3_round(x) -> np.ndarray:
    """E4M3 codes of values (svg2o_e4m3_round: nearest, ties to even, saturating), uint8."""
    a = np.asarray(x, dtype=np.float64)
    return np.array([lib().svg2o_e4m3_round(float(v)) for v in a.ravel()], np.uint8).reshape(a.shape)


def quantize_e4m3(X: np.ndarray):
    """Per-plane E4M3 quantisation (svg2o_quantize_e4m3) of X [..., n_plane]: the leading axes index
    planes, each quantised with its own scale.  Returns (codes uint8 like X, scale float32 [planes])."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    planes = X.reshape(X.shape[0], -1) if X.ndim > 1 else X.reshape(1, -1)
    codes = np.zeros(planes.shape, np.uint8)
    scale = np.zeros(planes.shape[0], np.float32)
    for b in range(planes.shape[0]):
        row = np.ascontiguousarray(planes[b])
        out = np.zeros(row.size, np.uint8)
        sc = np.zeros(1, np.float32)
        lib().svg2o_quantize_e4m3(_p(row), row.size, _p(out), _p(sc))
        codes[b] = out
        scale[b] = sc[0]
    return codes.reshape(X.shape), scale


def sparse_attention_fp8_rows(Q8, K8, V8, sq: float, sk: float, sv: float, q_off, k_off, mask, scale, rows=None):
    """The FP8 attention's definition for one (b,h): sparse_attention_rows over the dequantised
    values q = e4m3_value(Q8) * sq (likewise k, v).  The codes' values are exact in float32, and the
    plane scales are factored out of the sums: scores scale * sq * sk * (q8 . k8), output sv * (P v8)."""
    q = e4m3_value(Q8).astype(np.float32)
    k = e4m3_value(K8).astype(np.float32)
    v = e4m3_value(V8).astype(np.float32)
    out = sparse_attention_rows(q, k, v, q_off, k_off, mask, float(scale) * float(sq) * float(sk), rows)
    return out * float(sv)


def seed_candidates(N: int, seed_tokens: int) -> np.ndarray:
    """Token indices of the k-means++ candidates, ascending.

    0 or seed_tokens >= N: every token.  Otherwise S = seed_tokens candidates, one per stratum:
    stratum j covers tokens [floor(j N / S), floor((j + 1) N / S)) and its candidate sits at offset
    floor(r_j w_j / 2^32) inside it, w_j its width and r_j = (j * 2654435769) mod 2^32 (a
    multiplicative hash by the golden ratio), all in exact integer arithmetic.  The spacing thus
    varies from stratum to stratum, so the candidates cannot line up with the rows or columns of
    the video grid the tokens are flattened from (a fixed stride that divides the row length would
    see only some columns)."""
    if seed_tokens <= 0 or seed_tokens >= N:
        return np.arange(N, dtype=np.int64)
    S = np.uint64(seed_tokens)
    j = np.arange(seed_tokens, dtype=np.uint64)
    lo = (j * np.uint64(N)) // S
    hi = ((j + np.uint64(1)) * np.uint64(N)) // S
    r = (j * np.uint64(2654435769)) & np.uint64(0xFFFFFFFF)
    return (lo + ((r * (hi - lo)) >> np.uint64(32))).astype(np.int64)


def kmeans(X: np.ndarray, k: int, iters: int, u: Optional[np.ndarray] = None,
           C0: Optional[np.ndarray] = None, seed_tokens: int = 0):
    """k-means++ seeding on the candidate tokens X[seed_candidates(N, seed_tokens)] (or the given
    C0), then `iters` Lloyd iterations over all tokens."""
    if C0 is None:
        _, C0 = kmeanspp(np.ascontiguousarray(X[seed_candidates(X.shape[0], seed_tokens)]), k, u)
    return lloyd(X, C0, iters)


def layer_head(q, k, v, nQ, nK, iters, top_p, scale, uq=None, uk=None, cq0=None, ck0=None,
               rows=None, seed_tokens: int = 0) -> Dict[str, np.ndarray]:
    """The whole layer for one (batch, head), as the Method section orders it.

    `rows` (original token indices) restricts the attention to those output rows.
    """
    cq, lq, count_q = kmeans(q, nQ, iters, uq, cq0, seed_tokens)
    ck, lk, count_k = kmeans(k, nK, iters, uk, ck0, seed_tokens)
    w = select_weights(cq.astype(np.float32), ck.astype(np.float32), count_k, scale)
    mask = topp(w, count_k, top_p)
    perm_q, q_off = permute(lq, nQ)
    perm_k, k_off = permute(lk, nK)
    Qp, Kp, Vp = gather_rows(q, perm_q), gather_rows(k, perm_k), gather_rows(v, perm_k)
    out = {"cq": cq, "ck": ck, "labels_q": lq, "labels_k": lk, "count_q": count_q, "count_k": count_k,
           "weights": w, "mask": mask, "perm_q": perm_q, "perm_k": perm_k, "q_off": q_off, "k_off": k_off}
    if rows is None:
        Op = sparse_attention_rows(Qp, Kp, Vp, q_off, k_off, mask, scale)
        out["o"] = unpermute(Op, perm_q)
    else:
        inv = np.empty_like(perm_q)
        inv[perm_q] = np.arange(perm_q.size, dtype=np.int32)
        out["o_rows"] = sparse_attention_rows(Qp, Kp, Vp, q_off, k_off, mask, scale, inv[np.asarray(rows)])
    return out


def density(mask: np.ndarray, count_q: np.ndarray, count_k: np.ndarray) -> float:
    """Fraction of the dense score matrix that the selected cluster pairs cover."""
    cq = count_q.astype(np.float64)
    ck = count_k.astype(np.float64)
    n = cq.sum()
    return float((mask.astype(np.float64) * cq[:, None] * ck[None, :]).sum() / (n * n))
