"""CPU oracle for the CSA lightning-indexer top-k step -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.  The arithmetic lives in ``si_oracle.c`` (plain C,
fp64, full sort); this file only compiles it and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "si_oracle.c")
_LIB = os.path.join(_HERE, "libsi_oracle.so")
_lib = None

# Plain scalar code: no fast-math, no FMA contraction, so sums run in the
# written order with one rounding per operation.
CFLAGS = ["-O3", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle shared library (gcc) if missing or stale."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, src, "-lm"], check=True)
        os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """ctypes handle on the oracle library (builds the default one on demand)."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    L = ctypes.CDLL(path or build())
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    L.oracle_bf16_value.restype = ctypes.c_double
    L.oracle_bf16_value.argtypes = [ctypes.c_uint16]
    L.oracle_e4m3_value.restype = ctypes.c_double
    L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    L.oracle_visible_count.restype = i64
    L.oracle_visible_count.argtypes = [i64, i64, i64]
    L.oracle_topk_bf16.restype = ctypes.c_int
    L.oracle_topk_bf16.argtypes = [vp, vp, vp] + [i64] * 7 + [vp, i64, vp, vp, vp]
    L.oracle_topk_e4m3.restype = ctypes.c_int
    L.oracle_topk_e4m3.argtypes = [vp, vp, vp, vp, vp] + [i64] * 7 + [vp, i64, vp, vp, vp]
    L.oracle_e2m1_value.restype = ctypes.c_double
    L.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
    L.oracle_e8m0_value.restype = ctypes.c_double
    L.oracle_e8m0_value.argtypes = [ctypes.c_uint8]
    L.oracle_topk_mxfp4.restype = ctypes.c_int
    L.oracle_topk_mxfp4.argtypes = [vp, vp, vp, vp] + [i64] * 7 + [vp, i64, vp, vp, vp]
    L.oracle_mxfp4_decode.restype = ctypes.c_int
    L.oracle_mxfp4_decode.argtypes = [vp, vp, i64, i64, vp]
    L.oracle_pool_keys_bf16.restype = ctypes.c_int
    L.oracle_pool_keys_bf16.argtypes = [vp, i64, i64, i64, i64, vp]
    L.oracle_topk_two_stage_bf16.restype = ctypes.c_int
    L.oracle_topk_two_stage_bf16.argtypes = [vp, vp, vp] + [i64] * 9 + [vp, i64, vp, vp, vp]
    L.oracle_sparse_attention_bf16.restype = ctypes.c_int
    L.oracle_sparse_attention_bf16.argtypes = [vp, vp, vp] + [i64] * 7 + [ctypes.c_double, vp, vp]
    L.oracle_scores_bf16.restype = ctypes.c_int
    L.oracle_scores_bf16.argtypes = [vp, vp, vp] + [i64] * 6 + [i64, vp]
    if path is None:
        _lib = L
    return L


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def topk(q, kc, w, m: int, k: int, rows=None, q_scale=None, kc_scale=None, lib=None,
         kc_mx_scale=None):
    """Oracle top-k.

    q: [B,S,H,D] bf16 bits (uint16) or e4m3 codes (uint8, then q_scale
    [B,S,H] float32 and kc_scale [B,T] float32 are required); kc: [B,T,D];
    w: [B,S,H] float32.  With kc_mx_scale ([B,T,D/32] E8M0 bytes), q is
    bf16 and kc holds MXFP4 codes [B,T,D/2] (value d in the low nibble of
    byte d/2 when d is even, the high nibble when odd).
    rows: flat row ids b*S+t (default: all rows).
    Returns (idx int32 [n,k], score float32 [n,k], score64 float64 [n,k]).
    """
    L = lib or load()
    B, S, H, D = q.shape
    T = kc.shape[1]
    if rows is None:
        rows = np.arange(B * S, dtype=np.int64)
    rows = _c(np.asarray(rows, dtype=np.int64), np.int64)
    n = rows.shape[0]
    idx = np.empty((n, k), dtype=np.int32)
    sc = np.empty((n, k), dtype=np.float32)
    sc64 = np.empty((n, k), dtype=np.float64)
    w = _c(w, np.float32)
    if kc_mx_scale is not None:
        q, kc, ms = _c(q, np.uint16), _c(kc, np.uint8), _c(kc_mx_scale, np.uint8)
        assert kc.shape[2] * 2 == D and ms.shape == (B, T, D // 32), (kc.shape, ms.shape)
        rc = L.oracle_topk_mxfp4(q.ctypes.data, kc.ctypes.data, ms.ctypes.data, w.ctypes.data, B, S, T, H, D,
                                 m, k, rows.ctypes.data, n, idx.ctypes.data, sc.ctypes.data,
                                 sc64.ctypes.data)
    elif q.dtype == np.uint16:
        q, kc = _c(q, np.uint16), _c(kc, np.uint16)
        rc = L.oracle_topk_bf16(q.ctypes.data, kc.ctypes.data, w.ctypes.data, B, S, T, H, D, m, k,
                                rows.ctypes.data, n, idx.ctypes.data, sc.ctypes.data, sc64.ctypes.data)
    else:
        q, kc = _c(q, np.uint8), _c(kc, np.uint8)
        qs, ks = _c(q_scale, np.float32), _c(kc_scale, np.float32)
        rc = L.oracle_topk_e4m3(q.ctypes.data, qs.ctypes.data, kc.ctypes.data, ks.ctypes.data,
                                w.ctypes.data, B, S, T, H, D, m, k, rows.ctypes.data, n,
                                idx.ctypes.data, sc.ctypes.data, sc64.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle returned {rc}")
    return idx, sc, sc64


def pool_keys(kc, G: int = 8, lib=None) -> np.ndarray:
    """Pooled keys of the two-stage indexer: [B, T//G, D] float64 (bf16 values),
    the mean of each block of G keys rounded once to bf16."""
    L = lib or load()
    kc = _c(kc, np.uint16)
    B, T, D = kc.shape
    out = np.empty((B, T // G, D), dtype=np.float64)
    if T // G == 0:
        return out
    if L.oracle_pool_keys_bf16(kc.ctypes.data, B, T, D, G, out.ctypes.data) != 0:
        raise ValueError("oracle_pool_keys_bf16 failed")
    return out


def topk_two_stage(q, kc, w, m: int, k: int, G: int = 8, n_keep: int = 2048, rows=None, lib=None):
    """Two-stage oracle top-k (bf16 q [B,S,H,D], kc [B,T,D], w [B,S,H]): the
    best n_keep complete visible blocks of G keys by the score of their pooled
    key, then the top-k of their keys and the incomplete block's visible keys.
    Returns (idx int32 [n,k], score float32 [n,k], score64 float64 [n,k])."""
    L = lib or load()
    B, S, H, D = q.shape
    T = kc.shape[1]
    if rows is None:
        rows = np.arange(B * S, dtype=np.int64)
    rows = _c(np.asarray(rows, dtype=np.int64), np.int64)
    n = rows.shape[0]
    idx = np.empty((n, k), dtype=np.int32)
    sc = np.empty((n, k), dtype=np.float32)
    sc64 = np.empty((n, k), dtype=np.float64)
    q, kc, w = _c(q, np.uint16), _c(kc, np.uint16), _c(w, np.float32)
    rc = L.oracle_topk_two_stage_bf16(q.ctypes.data, kc.ctypes.data, w.ctypes.data, B, S, T, H, D, m, k, G,
                                      n_keep, rows.ctypes.data, n, idx.ctypes.data, sc.ctypes.data,
                                      sc64.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle returned {rc}")
    return idx, sc, sc64


def sparse_attention(q, kv, idx, dv: int, scale: float | None = None, lib=None):
    """Sparse attention over selected compressed entries: q [B,S,H,Dk] and
    kv [B,T,Dk] bf16 bits, idx [B,S,k] int32 (-1 = padding); every head
    attends over kv[idx] as keys (all Dk) and values (the first dv).
    scale defaults to 1/sqrt(Dk).  Returns (out float64 [B,S,H,dv], lse
    float64 [B,S,H])."""
    L = lib or load()
    q, kv, idx = _c(q, np.uint16), _c(kv, np.uint16), _c(idx, np.int32)
    B, S, H, Dk = q.shape
    T, k = kv.shape[1], idx.shape[2]
    scale = 1.0 / np.sqrt(Dk) if scale is None else float(scale)
    out = np.empty((B, S, H, dv), dtype=np.float64)
    lse = np.empty((B, S, H), dtype=np.float64)
    rc = L.oracle_sparse_attention_bf16(q.ctypes.data, kv.ctypes.data, idx.ctypes.data, B, S, T, H, Dk, dv, k,
                                        scale, out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle returned {rc}")
    return out, lse


def mxfp4_decode(codes, scales, lib=None) -> np.ndarray:
    """MXFP4 rows (codes [..., D/2] bytes, E8M0 scales [..., D/32]) as float64 [..., D]."""
    L = lib or load()
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    D = codes.shape[-1] * 2
    rows = int(np.prod(codes.shape[:-1]))
    assert scales.shape[-1] * 32 == D and int(np.prod(scales.shape[:-1])) == rows
    out = np.empty(codes.shape[:-1] + (D,), dtype=np.float64)
    if L.oracle_mxfp4_decode(codes.ctypes.data, scales.ctypes.data, rows, D, out.ctypes.data) != 0:
        raise ValueError("oracle_mxfp4_decode failed")
    return out


def scores(q, kc, w, m: int, row: int, lib=None) -> np.ndarray:
    """All T oracle scores (double) of one flat row; invisible keys are NaN."""
    L = lib or load()
    B, S, H, D = q.shape
    T = kc.shape[1]
    q, kc, w = _c(q, np.uint16), _c(kc, np.uint16), _c(w, np.float32)
    out = np.empty((T,), dtype=np.float64)
    rc = L.oracle_scores_bf16(q.ctypes.data, kc.ctypes.data, w.ctypes.data, B, S, T, H, D, m, row,
                              out.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle returned {rc}")
    return out


def visible_count(t: int, T: int, m: int, lib=None) -> int:
    return int((lib or load()).oracle_visible_count(t, T, m))
