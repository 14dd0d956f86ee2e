"""CPU oracle for Hierarchical Sparse Attention (HSA) -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. The product path (``ultra_long_context_b200``) never imports it, and the two share no
code.

The arithmetic lives in ``hsa_oracle.c`` (fp64 accumulation, written from the explainer page of
"Every Token Counts: Generalizing 16M Ultra-Long Context in Large Language Models", section
"How It Works (Technically)", Steps 1-4, and its per-token procedure "The algorithm, simplified").
This module only marshals numpy arrays into it. ``brute.py`` holds an independent dense numpy
formulation used to pin it on tiny inputs.
"""
import ctypes
import math

import numpy as np

from . import build as _build

_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        _int = ctypes.c_int
        lib.hsa_oracle_forward_rows.argtypes = [_f32p, _f32p, _f32p, _f32p, _f32p, _i64, _i64, _i64, _i64, _i64, _i64,
                                                _i64, ctypes.c_double, _int, _i64, _i64p, _f64p, _i32p, _f64p, _f64p,
                                                _f64p]
        lib.hsa_oracle_scores_rows.argtypes = [_f32p, _f32p, _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_double,
                                               _i64, _i64p, _f64p]
        lib.hsa_oracle_decode_select.argtypes = [_f32p, _f32p, _i64p, _i64, _i64, _i64, _i64, _i64, _i64, _i64,
                                                 ctypes.c_double, _i32p, _f64p, _f64p, _f64p, _f64p]
        lib.hsa_oracle_attend_gathered.argtypes = [_f32p, _f32p, _f32p, _f32p, _f32p, _i32p, _i64, _i64, _i64, _i64,
                                                   ctypes.c_double, _int, _f64p, _f64p]
        lib.hsa_oracle_backward.argtypes = [_f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _i32p, _i64, _i64, _i64, _i64,
                                            _i64, _i64, _i64, ctypes.c_double, _int, _f64p, _f64p, _f64p, _f64p,
                                            _f64p]
        for f in (lib.hsa_oracle_forward_rows, lib.hsa_oracle_scores_rows, lib.hsa_oracle_decode_select,
                  lib.hsa_oracle_attend_gathered, lib.hsa_oracle_backward):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f32(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a, a.ctypes.data_as(_f32p)


def _ptr(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"{name} failed with status {rc}")


def default_scale(D):
    return 1.0 / math.sqrt(D)


def _opt_f32(a, like):
    if a is None:
        return None, None
    a, p = _f32(a)
    assert a.shape == like.shape, "the retrieval query must have the shape of the attention query"
    return a, p


def _heads(H, K, L):
    Hkv = K.shape[1]
    assert Hkv >= 1 and H % Hkv == 0 and L.shape[1] == Hkv, "K, V, L need Hkv heads, H a multiple of Hkv"
    return Hkv


def forward(Q, K, V, L, chunk=64, topk=8, scale=None, rows=None, Qs=None, qk_norm=False):
    """HSA forward of rows of Q [B, H, T, D] against K, V [B, Hkv, T, D], L [B, Hkv, N, D] (float arrays
    holding bf16-exact values; query head h uses key head h // (H // Hkv)).

    Qs: separate retrieval queries shaped like Q (Step 2 scores Qs . L; Step 3 attends with Q), or
    None when Q does both. qk_norm: Step 3 attends with the L2-normalised query and keys.

    Returns a dict with out [R, D] (float64), sel_idx [R, topk] (int32, -1 padding), sel_w and sel_s
    [R, topk] (float64, 0 padding) and next_s [R] (score of the best unselected chunk, -inf if none),
    where R = B*H*T when ``rows`` is None (rows in (b, h, t) order) else len(rows) (flat row ids).
    """
    Q, qp = _f32(Q)
    K, kp = _f32(K)
    V, vp = _f32(V)
    L, lp = _f32(L)
    Qs, qsp = _opt_f32(Qs, Q)
    B, H, T, D = Q.shape
    Hkv = _heads(H, K, L)
    if scale is None:
        scale = default_scale(D)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R = rows.shape[0]
    else:
        R = B * H * T
    out = np.zeros((R, D), np.float64)
    sel_idx = np.zeros((R, topk), np.int32)
    sel_w = np.zeros((R, topk), np.float64)
    sel_s = np.zeros((R, topk), np.float64)
    next_s = np.zeros((R,), np.float64)
    rc = _load().hsa_oracle_forward_rows(qp, qsp, kp, vp, lp, B, H, Hkv, T, D, chunk, topk, scale, int(qk_norm), R,
                                         _ptr(rows, _i64p), _ptr(out, _f64p), _ptr(sel_idx, _i32p),
                                         _ptr(sel_w, _f64p), _ptr(sel_s, _f64p), _ptr(next_s, _f64p))
    _check(rc, "hsa_oracle_forward_rows")
    return dict(out=out, sel_idx=sel_idx, sel_w=sel_w, sel_s=sel_s, next_s=next_s)


def scores(Q, L, rows, chunk=64, scale=None):
    """All retrieval scores of the listed rows of Q [B, H, T, D] (the retrieval queries) against L
    [B, Hkv, N, D]: [R, N] float64, NaN where a chunk is not admissible."""
    Q, qp = _f32(Q)
    L, lp = _f32(L)
    B, H, T, D = Q.shape
    if scale is None:
        scale = default_scale(D)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    N = T // chunk
    out = np.zeros((rows.shape[0], N), np.float64)
    rc = _load().hsa_oracle_scores_rows(qp, lp, B, H, L.shape[1], T, D, chunk, scale, rows.shape[0],
                                        _ptr(rows, _i64p), _ptr(out, _f64p))
    _check(rc, "hsa_oracle_scores_rows")
    return out


def decode_select(q, Lc, cache_len, chunk=64, topk=16, scale=None, all_scores=False):
    """Decode retrieval: q [B, H, D] (retrieval queries), Lc [B, Hkv, Nmax, D], cache_len [B] -> selection
    dict [B, H, topk]. With all_scores, the dict also holds all_s [B, H, Nmax]: every retrieval score
    (NaN for chunks the token does not see)."""
    q, qp = _f32(q)
    Lc, lp = _f32(Lc)
    B, H, D = q.shape
    Nmax = Lc.shape[2]
    if scale is None:
        scale = default_scale(D)
    cl = np.ascontiguousarray(cache_len, dtype=np.int64)
    sel_idx = np.zeros((B, H, topk), np.int32)
    sel_s = np.zeros((B, H, topk), np.float64)
    sel_w = np.zeros((B, H, topk), np.float64)
    next_s = np.zeros((B, H), np.float64)
    all_s = np.zeros((B, H, Nmax), np.float64) if all_scores else None
    rc = _load().hsa_oracle_decode_select(qp, lp, _ptr(cl, _i64p), B, H, Lc.shape[1], D, Nmax, chunk, topk, scale,
                                          _ptr(sel_idx, _i32p), _ptr(sel_s, _f64p), _ptr(sel_w, _f64p),
                                          _ptr(next_s, _f64p), _ptr(all_s, _f64p))
    _check(rc, "hsa_oracle_decode_select")
    res = dict(sel_idx=sel_idx, sel_s=sel_s, sel_w=sel_w, next_s=next_s)
    if all_scores:
        res["all_s"] = all_s
    return res


def attend_gathered(q, Lg, Kg, Vg, nsel, scale=None, qs=None, qk_norm=False):
    """Steps 3-4 for R rows given their selected chunks gathered.

    q [R, D], Lg [R, topk, D], Kg / Vg [R, topk, chunk, D], nsel [R] -> (out [R, D], sel_w [R, topk]).
    qs [R, D]: separate retrieval queries (the fusion weights come from qs . Lg), or None.
    qk_norm: Step 3 attends with the L2-normalised query and keys.
    """
    q, qp = _f32(q)
    qs, qsp = _opt_f32(qs, q)
    Lg, lp = _f32(Lg)
    Kg, kp = _f32(Kg)
    Vg, vp = _f32(Vg)
    R, D = q.shape
    topk, chunk = Kg.shape[1], Kg.shape[2]
    if scale is None:
        scale = default_scale(D)
    ns = np.ascontiguousarray(nsel, dtype=np.int32)
    out = np.zeros((R, D), np.float64)
    sel_w = np.zeros((R, topk), np.float64)
    rc = _load().hsa_oracle_attend_gathered(qp, qsp, lp, kp, vp, _ptr(ns, _i32p), R, D, chunk, topk, scale,
                                            int(qk_norm), _ptr(out, _f64p), _ptr(sel_w, _f64p))
    _check(rc, "hsa_oracle_attend_gathered")
    return out, sel_w


def backward(Q, K, V, L, dO, sel_idx, chunk=64, scale=None, Qs=None, qk_norm=False):
    """Gradients of the HSA forward for a fixed selection sel_idx [B, H, T, topk] (-1 = empty).

    Shapes and options as in ``forward`` (K, V, L may have fewer heads than Q; qk_norm).

    Returns (dQ, dK, dV, dL) as float64 arrays shaped like Q, K, V, L; with separate retrieval queries
    Qs, (dQ, dK, dV, dL, dQs) where dQ is the attention query's gradient and dQs the retrieval query's.
    """
    Q, qp = _f32(Q)
    K, kp = _f32(K)
    V, vp = _f32(V)
    L, lp = _f32(L)
    dO, gp = _f32(dO)
    Qs, qsp = _opt_f32(Qs, Q)
    B, H, T, D = Q.shape
    Hkv = _heads(H, K, L)
    if scale is None:
        scale = default_scale(D)
    si = np.ascontiguousarray(sel_idx, dtype=np.int32)
    topk = si.shape[-1]
    dQ = np.zeros(Q.shape, np.float64)
    dK = np.zeros(K.shape, np.float64)
    dV = np.zeros(V.shape, np.float64)
    dL = np.zeros(L.shape, np.float64)
    dQs = np.zeros(Q.shape, np.float64) if Qs is not None else None
    rc = _load().hsa_oracle_backward(qp, qsp, kp, vp, lp, gp, _ptr(si, _i32p), B, H, Hkv, T, D, chunk, topk, scale,
                                     int(qk_norm), _ptr(dQ, _f64p), _ptr(dK, _f64p), _ptr(dV, _f64p), _ptr(dL, _f64p),
                                     _ptr(dQs, _f64p))
    _check(rc, "hsa_oracle_backward")
    return (dQ, dK, dV, dL) if Qs is None else (dQ, dK, dV, dL, dQs)
