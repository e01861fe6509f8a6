"""Python binding of the B200 CSA lightning-indexer top-k library.

Argument marshalling only: every step of the indexer runs in the CUDA kernels
of ``libstreaming_top.so`` (built by ``python streaming_top_b200/build.py``).
Tensors are torch CUDA tensors; torch provides device memory and streams.
There is no CPU fallback: without the built library this module fails to
import.

    q   [B, S, H_I, D] bf16 (or uint8 e4m3 codes + q_scale [B, S, H_I] fp32)
    kc  [B, T, D]      bf16 (or uint8 e4m3 codes + kc_scale [B, T] fp32)
    w   [B, S, H_I]    fp32
    ->  idx [B, S, k] int32 (-1 padded), score [B, S, k] fp32 (-inf padded)
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libstreaming_top.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python streaming_top_b200/build.py` "
                      "(the indexer has no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

SI_OK, SI_ERR_INVALID_ARGUMENT, SI_ERR_UNSUPPORTED, SI_ERR_OUT_OF_MEMORY, SI_ERR_CUDA, SI_ERR_TIMEOUT = range(6)
SI_DTYPE_BF16, SI_DTYPE_FP8_E4M3, SI_DTYPE_MXFP4_KEYS = 0, 1, 2

_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


class Options(ctypes.Structure):
    _fields_ = [("dtype", _i), ("q_scale", _vp), ("kc_scale", _vp), ("query_chunk", _i),
                ("key_tile", _i), ("workspace", _vp), ("workspace_bytes", _sz), ("unsorted", _i),
                ("kc_mx_scale", _vp)]


_ARGS = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp]
_lib.si_indexer_topk.restype = _i
_lib.si_indexer_topk.argtypes = _ARGS
_lib.si_indexer_topk_ex.restype = _i
_lib.si_indexer_topk_ex.argtypes = _ARGS + [ctypes.POINTER(Options)]
_lib.si_indexer_topk_rows.restype = _i
_lib.si_indexer_topk_rows.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                                      ctypes.POINTER(Options)]
_lib.si_sort_topk_rows.restype = _i
_lib.si_sort_topk_rows.argtypes = [_vp, _vp, ctypes.c_int64, _i, _vp]
_lib.si_indexer_materialize.restype = _i
_lib.si_indexer_materialize.argtypes = _ARGS + [ctypes.POINTER(Options)]
_lib.si_indexer_materialize_noalloc.restype = _i
_lib.si_indexer_materialize_noalloc.argtypes = _ARGS
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024  # SI_NOALLOC_SCRATCH_BYTES
_lib.si_indexer_workspace_size.restype = _sz
_lib.si_indexer_workspace_size.argtypes = [_i] * 8 + [ctypes.POINTER(Options)]
_lib.si_indexer_topk_two_stage.restype = _i
_lib.si_indexer_topk_two_stage.argtypes = [_vp, _vp, _vp] + [_i] * 9 + [_vp, _vp, _vp, ctypes.POINTER(Options)]
_lib.si_two_stage_workspace_size.restype = _sz
_lib.si_two_stage_workspace_size.argtypes = [_i] * 6
_lib.si_mxfp4_to_bf16.restype = _i
_lib.si_mxfp4_to_bf16.argtypes = [_vp, _vp, ctypes.c_int64, _i, _vp, _vp]
_lib.si_device_status.restype = _i
_lib.si_device_status.argtypes = [_vp]
_lib.si_status_string.restype = ctypes.c_char_p
_lib.si_status_string.argtypes = [_i]
_lib.si_last_error.restype = ctypes.c_char_p
_lib.si_last_error.argtypes = []
_lib.si_version.restype = _i
_lib.si_test_stream_timeout.restype = _i
_lib.si_test_stream_timeout.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, ctypes.c_ulonglong]


class SIError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.si_last_error().decode(errors="replace")
        super().__init__(f"{where}: {_lib.si_status_string(status).decode()}: {msg}")


def _check(st: int, where: str) -> None:
    if st != SI_OK:
        raise SIError(st, where)


def lib():
    """The ctypes handle on libstreaming_top.so."""
    return _lib


def version() -> int:
    return _lib.si_version()


def _stream_ptr(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _shapes(q, kc, w, mxfp4: bool = False):
    if q.dim() != 4 or kc.dim() != 3 or w.dim() != 3:
        raise ValueError("q [B,S,H,D], kc [B,T,D] (MXFP4: [B,T,D/2] codes), w [B,S,H] expected")
    B, S, H, D = q.shape
    kd = D // 2 if mxfp4 else D
    if kc.shape[0] != B or kc.shape[2] != kd or tuple(w.shape) != (B, S, H):
        raise ValueError(f"shape mismatch q{tuple(q.shape)} kc{tuple(kc.shape)} w{tuple(w.shape)}")
    for name, t in (("q", q), ("kc", kc), ("w", w)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if w.dtype != torch.float32:
        raise ValueError("w must be float32")
    return B, S, kc.shape[1], H, D


def _outputs(B, S, k, device, out_idx, out_score, with_score):
    if out_idx is None:
        out_idx = torch.empty((B, S, k), dtype=torch.int32, device=device)
    if out_score is None and with_score:
        out_score = torch.empty((B, S, k), dtype=torch.float32, device=device)
    return out_idx, out_score


def _options(q, kc, q_scale, kc_scale, query_chunk, key_tile, workspace=None, kc_mx_scale=None):
    o = Options()
    if kc_mx_scale is not None:
        B, _, _, D = q.shape
        shape = (B, kc.shape[1], D // 32)
        if q.dtype != torch.bfloat16 or kc.dtype != torch.uint8 or kc.shape[2] * 2 != D:
            raise ValueError("MXFP4 keys: q bfloat16 [B,S,H,D] and kc uint8 codes [B,T,D/2] expected")
        if (kc_mx_scale.dtype != torch.uint8 or tuple(kc_mx_scale.shape) != shape or not kc_mx_scale.is_cuda
                or not kc_mx_scale.is_contiguous()):
            raise ValueError(f"kc_mx_scale must be a contiguous uint8 CUDA tensor of shape {shape}")
        o.dtype = SI_DTYPE_MXFP4_KEYS
        o.kc_mx_scale = kc_mx_scale.data_ptr()
    elif kc.element_size() != q.element_size():
        raise ValueError(f"q ({q.dtype}) and kc ({kc.dtype}) must have the same element type")
    elif q.dtype == torch.bfloat16:
        o.dtype = SI_DTYPE_BF16
    elif q.dtype in (torch.uint8, torch.float8_e4m3fn):
        if q_scale is None or kc_scale is None:
            raise ValueError("fp8 inputs need q_scale and kc_scale")
        B, S, H, _ = q.shape
        for name, t, shape in (("q_scale", q_scale, (B, S, H)), ("kc_scale", kc_scale, (B, kc.shape[1]))):
            if (t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_cuda
                    or not t.is_contiguous()):
                raise ValueError(f"{name} must be a contiguous float32 CUDA tensor of shape {shape}")
        o.dtype = SI_DTYPE_FP8_E4M3
        o.q_scale = q_scale.data_ptr()
        o.kc_scale = kc_scale.data_ptr()
    else:
        raise ValueError(f"unsupported q dtype {q.dtype}")
    o.query_chunk = int(query_chunk)
    o.key_tile = int(key_tile)
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    return o


def indexer_topk(q, kc, w, m: int, k: int, *, q_scale=None, kc_scale=None, query_chunk: int = 0,
                 key_tile: int = 0, out_idx=None, out_score=None, with_score: bool = True,
                 unsorted: bool = False, stream=None, kc_mx_scale=None, workspace=None):
    """Streaming indexer top-k (``si_indexer_topk_ex``).  Returns (idx, score).
    With unsorted=True each row's results come in an unspecified order (valid
    entries first) and the row sort is skipped.  With kc_mx_scale (uint8
    [B,T,D/32] E8M0), kc holds MXFP4 codes [B,T,D/2] (uint8) and q is bf16."""
    B, S, T, H, D = _shapes(q, kc, w, kc_mx_scale is not None)
    out_idx, out_score = _outputs(B, S, k, q.device, out_idx, out_score, with_score)
    o = _options(q, kc, q_scale, kc_scale, query_chunk, key_tile, workspace, kc_mx_scale)
    o.unsorted = int(bool(unsorted))
    st = _lib.si_indexer_topk_ex(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, S, T, H, D, m, k,
                                 out_idx.data_ptr(), out_score.data_ptr() if out_score is not None else None,
                                 _stream_ptr(stream), ctypes.byref(o))
    _check(st, "si_indexer_topk_ex")
    return out_idx, out_score


def indexer_topk_rows(q, kc, w, m: int, k: int, row0: int, *, q_scale=None, kc_scale=None,
                      query_chunk: int = 0, key_tile: int = 0, out_idx=None, out_score=None,
                      with_score: bool = True, unsorted: bool = False, stream=None, kc_mx_scale=None,
                      workspace=None):
    """Streaming top-k for query rows row0 .. row0+R-1 (``si_indexer_topk_rows``):
    q [B, R, H_I, D] and w [B, R, H_I] hold those rows only, kc [B, T, D] all
    keys.  Returns (idx, score) of shape [B, R, k]."""
    B, R, T, H, D = _shapes(q, kc, w, kc_mx_scale is not None)
    out_idx, out_score = _outputs(B, R, k, q.device, out_idx, out_score, with_score)
    o = _options(q, kc, q_scale, kc_scale, query_chunk, key_tile, workspace, kc_mx_scale)
    o.unsorted = int(bool(unsorted))
    st = _lib.si_indexer_topk_rows(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, int(row0), R, T, H, D,
                                   m, k, out_idx.data_ptr(),
                                   out_score.data_ptr() if out_score is not None else None,
                                   _stream_ptr(stream), ctypes.byref(o))
    _check(st, "si_indexer_topk_rows")
    return out_idx, out_score


def indexer_topk_two_stage(q, kc, w, m: int, k: int, *, block: int = 8, n_keep: int = 2048,
                           query_chunk: int = 0, out_idx=None, out_score=None, workspace=None, stream=None):
    """Two-stage indexer top-k (``si_indexer_topk_two_stage``): the best
    n_keep blocks of `block` keys by the score of their pooled (mean) key,
    then the top-k of their keys and the incomplete block's visible keys.
    Returns (idx, score) [B, S, k], ordered as indexer_topk's."""
    B, S, T, H, D = _shapes(q, kc, w)
    out_idx, out_score = _outputs(B, S, k, q.device, out_idx, out_score, True)
    o = _options(q, kc, None, None, query_chunk, 0, workspace)
    st = _lib.si_indexer_topk_two_stage(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, S, T, H, D, m, k,
                                        int(block), int(n_keep), out_idx.data_ptr(), out_score.data_ptr(),
                                        _stream_ptr(stream), ctypes.byref(o))
    _check(st, "si_indexer_topk_two_stage")
    return out_idx, out_score


def two_stage_workspace_size(B, S, T, block=8, n_keep=2048, query_chunk=0) -> int:
    return int(_lib.si_two_stage_workspace_size(B, S, T, block, n_keep, query_chunk))


def mxfp4_to_bf16(codes, scales, out=None, stream=None):
    """Decode MXFP4 rows (``si_mxfp4_to_bf16``): codes uint8 [..., D/2], E8M0
    scales uint8 [..., D/32]; returns bf16 [..., D]."""
    if codes.dtype != torch.uint8 or scales.dtype != torch.uint8:
        raise ValueError("codes and scales must be uint8")
    D = codes.shape[-1] * 2
    if scales.shape[:-1] != codes.shape[:-1] or scales.shape[-1] * 32 != D:
        raise ValueError(f"scales {tuple(scales.shape)} do not match codes {tuple(codes.shape)}")
    for name, t in (("codes", codes), ("scales", scales)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if out is None:
        out = torch.empty(codes.shape[:-1] + (D,), dtype=torch.bfloat16, device=codes.device)
    rows = codes.numel() // (D // 2) if D else 0
    _check(_lib.si_mxfp4_to_bf16(codes.data_ptr(), scales.data_ptr(), rows, D, out.data_ptr(),
                                 _stream_ptr(stream)), "si_mxfp4_to_bf16")
    return out


def sort_topk_rows(idx, score, stream=None):
    """Sort every row of (idx [..., k] int32, score [..., k] fp32) in place by
    score descending, index ascending (``si_sort_topk_rows``)."""
    if idx.shape != score.shape or idx.dtype != torch.int32 or score.dtype != torch.float32:
        raise ValueError("idx int32 and score float32 of the same shape expected")
    for name, t in (("idx", idx), ("score", score)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    k = idx.shape[-1]
    rows = idx.numel() // k if k else 0
    _check(_lib.si_sort_topk_rows(idx.data_ptr(), score.data_ptr(), rows, k, _stream_ptr(stream)),
           "si_sort_topk_rows")
    return idx, score


def indexer_materialize(q, kc, w, m: int, k: int, *, out_idx=None, out_score=None,
                        with_score: bool = True, workspace=None, stream=None):
    """Materialize-path ground truth (``si_indexer_materialize``)."""
    B, S, T, H, D = _shapes(q, kc, w)
    out_idx, out_score = _outputs(B, S, k, q.device, out_idx, out_score, with_score)
    o = _options(q, kc, None, None, 0, 0, workspace)
    st = _lib.si_indexer_materialize(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, S, T, H, D, m, k,
                                     out_idx.data_ptr(),
                                     out_score.data_ptr() if out_score is not None else None,
                                     _stream_ptr(stream), ctypes.byref(o))
    _check(st, "si_indexer_materialize")
    return out_idx, out_score


def indexer_materialize_noalloc(q, kc, w, m: int, k: int, *, out_idx=None, out_score=None,
                                with_score: bool = True, stream=None):
    """Materialize path without device allocation (``si_indexer_materialize_noalloc``):
    its scratch is the library's fixed device array of NOALLOC_SCRATCH_BYTES.
    For callers that may not allocate device memory during the call; pass
    preallocated outputs to keep the call itself allocation-free."""
    B, S, T, H, D = _shapes(q, kc, w)
    out_idx, out_score = _outputs(B, S, k, q.device, out_idx, out_score, with_score)
    st = _lib.si_indexer_materialize_noalloc(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, S, T, H, D, m,
                                             k, out_idx.data_ptr(),
                                             out_score.data_ptr() if out_score is not None else None,
                                             _stream_ptr(stream))
    _check(st, "si_indexer_materialize_noalloc")
    return out_idx, out_score


def workspace_size(B, S, T, H, D, m, k, materialize: bool = False) -> int:
    return int(_lib.si_indexer_workspace_size(B, S, T, H, D, m, k, int(materialize), None))


def device_status(stream=None) -> int:
    """Synchronise the stream; return SI_OK or the status of a device-side failure."""
    return int(_lib.si_device_status(_stream_ptr(stream)))


def indexer_topk_host(q, kc, w, m: int, k: int, *, q_scale=None, kc_scale=None, device="cuda",
                      query_chunk: int = 0, key_tile: int = 0, bufs: dict | None = None,
                      sync: bool = True, row0: int | None = None, kc_mx_scale=None,
                      two_stage: dict | None = None):
    """End-to-end call on HOST tensors (pinned for best speed): copies the
    inputs to the device, runs the streaming top-k, copies (idx, score) back.
    `bufs` may hold reusable device buffers from a previous call.  With
    sync=False the copies back are only enqueued on the current stream.
    With `row0`, q and w hold only rows row0 .. row0+R-1 of the sequences
    (si_indexer_topk_rows).  With `two_stage` (keyword arguments of
    indexer_topk_two_stage: block, n_keep), the two-stage indexer runs."""
    bufs = {} if bufs is None else bufs
    stream = torch.cuda.current_stream(device)

    def dev(name, t):
        d = bufs.get(name)
        if d is None or d.shape != t.shape or d.dtype != t.dtype:
            d = torch.empty(t.shape, dtype=t.dtype, device=device)
            bufs[name] = d
        d.copy_(t, non_blocking=True)
        return d

    qd, kd, wd = dev("q", q), dev("kc", kc), dev("w", w)
    qs = dev("q_scale", q_scale) if q_scale is not None else None
    ks = dev("kc_scale", kc_scale) if kc_scale is not None else None
    kms = dev("kc_mx_scale", kc_mx_scale) if kc_mx_scale is not None else None
    B, S = q.shape[0], q.shape[1]
    oi = bufs.get("out_idx")
    os_ = bufs.get("out_score")
    if oi is None or oi.shape != (B, S, k):
        oi = bufs["out_idx"] = torch.empty((B, S, k), dtype=torch.int32, device=device)
        os_ = bufs["out_score"] = torch.empty((B, S, k), dtype=torch.float32, device=device)
    if two_stage is not None:
        indexer_topk_two_stage(qd, kd, wd, m, k, query_chunk=query_chunk, out_idx=oi, out_score=os_,
                               stream=stream, **two_stage)
    elif row0 is None:
        indexer_topk(qd, kd, wd, m, k, q_scale=qs, kc_scale=ks, query_chunk=query_chunk,
                     key_tile=key_tile, out_idx=oi, out_score=os_, stream=stream, kc_mx_scale=kms)
    else:
        indexer_topk_rows(qd, kd, wd, m, k, row0, q_scale=qs, kc_scale=ks, query_chunk=query_chunk,
                          key_tile=key_tile, out_idx=oi, out_score=os_, stream=stream, kc_mx_scale=kms)
    hi = bufs.get("h_idx")
    hs = bufs.get("h_score")
    if hi is None or hi.shape != oi.shape:
        hi = bufs["h_idx"] = torch.empty(oi.shape, dtype=oi.dtype, pin_memory=True)
        hs = bufs["h_score"] = torch.empty(os_.shape, dtype=os_.dtype, pin_memory=True)
    hi.copy_(oi, non_blocking=True)
    hs.copy_(os_, non_blocking=True)
    if sync:
        stream.synchronize()
    return hi, hs


def visible_pairs_before(t: int, T: int, m: int) -> int:
    """Visible (query, key) pairs of query rows 0 .. t-1 of one sequence:
    the sum over rows r < t of min(T, floor((r + 1) / m)) -- row r sees key s
    iff s*m + m - 1 <= r and s < T.  Closed form: with x = r + 1, floor(x/m)
    stays below T up to x = m*T - 1, and floor(x/m) summed over x = 1..N is
    m*a*(a-1)/2 + a*(b+1) for (a, b) = divmod(N, m)."""
    t = max(0, int(t))
    n = min(t, m * T - 1)
    a, b = divmod(n, m)
    return m * a * (a - 1) // 2 + a * (b + 1) + (t - n) * T


def row_shards(S: int, T: int, m: int, parts: int, align: int = 4) -> list[int]:
    """Boundaries 0 = r_0 <= r_1 <= ... <= r_parts = S splitting the query
    rows of a sequence into `parts` contiguous ranges of (nearly) equal
    visible pairs -- the work of each range -- for row-sharding one sequence
    over GPUs with si_indexer_topk_rows (the keys are replicated).  Inner
    boundaries are multiples of `align` (whole 4-query work units)."""
    if parts < 1 or S < 0:
        raise ValueError("parts >= 1 and S >= 0 required")
    total = visible_pairs_before(S, T, m)
    bounds = [0]
    for g in range(1, parts):
        target = total * g / parts
        lo, hi = 0, S  # smallest t with pairs_before(t) >= target
        while lo < hi:
            mid = (lo + hi) // 2
            if visible_pairs_before(mid, T, m) >= target:
                hi = mid
            else:
                lo = mid + 1
        r = min(S, max(bounds[-1], int(round(lo / align)) * align))
        bounds.append(r)
    bounds.append(S)
    return bounds


def test_stream_timeout(q, kc, w, m: int, k: int, out_idx, wait_limit_ns: int, stream=None) -> int:
    """Test hook: run the streaming kernel with one key tile withheld and a
    short bounded-wait limit; returns the launch status (the timeout itself is
    reported by device_status())."""
    B, S, T, H, D = _shapes(q, kc, w)
    return int(_lib.si_test_stream_timeout(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, S, T, m, k,
                                           out_idx.data_ptr(), _stream_ptr(stream), wait_limit_ns))
