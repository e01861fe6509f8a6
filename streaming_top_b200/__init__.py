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
                ("kc_mx_scale", _vp), ("device_status", _vp)]


_ARGS = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp]
_lib.si_indexer_topk.restype = _i
_lib.si_indexer_topk.argtypes = _ARGS
_lib.si_indexer_topk_ex.restype = _i
_lib.si_indexer_topk_ex.argtypes = _ARGS + [ctypes.POINTER(Options)]
_lib.si_indexer_topk_rows.restype = _i
_lib.si_indexer_topk_rows.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                                      ctypes.POINTER(Options)]
_lib.si_indexer_topk_host.restype = _i
_lib.si_indexer_topk_host.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                                      ctypes.POINTER(Options)]
_lib.si_indexer_topk_host_workspace_size.restype = _sz
_lib.si_indexer_topk_host_workspace_size.argtypes = [_i] * 7 + [ctypes.POINTER(Options)]
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
_lib.si_sparse_attention.restype = _i
_lib.si_sparse_attention.argtypes = [_vp, _vp, _vp] + [_i] * 7 + [ctypes.c_float, _vp, _vp, _vp,
                                                                    ctypes.POINTER(Options)]
_lib.si_mxfp4_to_bf16.restype = _i
_lib.si_mxfp4_to_bf16.argtypes = [_vp, _vp, ctypes.c_int64, _i, _vp, _vp]
_lib.si_device_status.restype = _i
_lib.si_device_status.argtypes = [_vp]
_lib.si_status_string.restype = ctypes.c_char_p
_lib.si_status_string.argtypes = [_i]
_lib.si_last_error.restype = ctypes.c_char_p
_lib.si_last_error.argtypes = []
_lib.si_version.restype = _i
_lib.si_version.argtypes = []
_lib.si_test_fail_allocations.restype = None
_lib.si_test_fail_allocations.argtypes = [_i]
_lib.si_test_stream_timeout.restype = _i
_lib.si_test_stream_timeout.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, ctypes.c_ulonglong, _vp]


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


def _shapes(q, kc, w, mxfp4: bool = False, host: bool = False):
    if q.dim() != 4 or kc.dim() != 3 or w.dim() != 3:
        raise ValueError("q [B,S,H,D], kc [B,T,D] (MXFP4: [B,T,D/2] codes), w [B,S,H] expected")
    B, S, H, D = q.shape
    kd = D // 2 if mxfp4 else D
    if kc.shape[0] != B or kc.shape[2] != kd or tuple(w.shape) != (B, S, H):
        raise ValueError(f"shape mismatch q{tuple(q.shape)} kc{tuple(kc.shape)} w{tuple(w.shape)}")
    for name, t in (("q", q), ("kc", kc), ("w", w)):
        if t.is_cuda == host or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {'host (CPU)' if host else 'CUDA'} tensor")
    if w.dtype != torch.float32:
        raise ValueError("w must be float32")
    return B, S, kc.shape[1], H, D


def _outputs(B, S, k, device, out_idx, out_score, with_score):
    if out_idx is None:
        out_idx = torch.empty((B, S, k), dtype=torch.int32, device=device)
    if out_score is None and with_score:
        out_score = torch.empty((B, S, k), dtype=torch.float32, device=device)
    return out_idx, out_score


def _options(q, kc, q_scale, kc_scale, query_chunk, key_tile, workspace=None, kc_mx_scale=None,
             device_status=None):
    o = Options()
    if device_status is not None:
        if (device_status.dtype != torch.int32 or device_status.numel() < 2 or not device_status.is_cuda
                or not device_status.is_contiguous()):
            raise ValueError("device_status must be a contiguous int32 CUDA tensor of >= 2 elements")
        o.device_status = device_status.data_ptr()
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
                 unsorted: bool = False, stream=None, kc_mx_scale=None, workspace=None, device_status=None):
    """Streaming indexer top-k (``si_indexer_topk_ex``).  Returns (idx, score).
    With unsorted=True each row's results come in an unspecified order (valid
    entries first) and the row sort is skipped.  With kc_mx_scale (uint8
    [B,T,D/32] E8M0), kc holds MXFP4 codes [B,T,D/2] (uint8) and q is bf16.
    device_status: optional zeroed int32 CUDA tensor (>= 2 elements), this
    call's own device error word."""
    B, S, T, H, D = _shapes(q, kc, w, kc_mx_scale is not None)
    out_idx, out_score = _outputs(B, S, k, q.device, out_idx, out_score, with_score)
    o = _options(q, kc, q_scale, kc_scale, query_chunk, key_tile, workspace, kc_mx_scale, device_status)
    o.unsorted = int(bool(unsorted))
    st = _lib.si_indexer_topk_ex(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, S, T, H, D, m, k,
                                 out_idx.data_ptr(), out_score.data_ptr() if out_score is not None else None,
                                 _stream_ptr(stream), ctypes.byref(o))
    _check(st, "si_indexer_topk_ex")
    return out_idx, out_score


def indexer_topk_rows(q, kc, w, m: int, k: int, row0: int, *, q_scale=None, kc_scale=None,
                      query_chunk: int = 0, key_tile: int = 0, out_idx=None, out_score=None,
                      with_score: bool = True, unsorted: bool = False, stream=None, kc_mx_scale=None,
                      workspace=None, device_status=None):
    """Streaming top-k for query rows row0 .. row0+R-1 (``si_indexer_topk_rows``):
    q [B, R, H_I, D] and w [B, R, H_I] hold those rows only, kc [B, T, D] all
    keys.  Returns (idx, score) of shape [B, R, k]."""
    B, R, T, H, D = _shapes(q, kc, w, kc_mx_scale is not None)
    out_idx, out_score = _outputs(B, R, k, q.device, out_idx, out_score, with_score)
    o = _options(q, kc, q_scale, kc_scale, query_chunk, key_tile, workspace, kc_mx_scale, device_status)
    o.unsorted = int(bool(unsorted))
    st = _lib.si_indexer_topk_rows(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, int(row0), R, T, H, D,
                                   m, k, out_idx.data_ptr(),
                                   out_score.data_ptr() if out_score is not None else None,
                                   _stream_ptr(stream), ctypes.byref(o))
    _check(st, "si_indexer_topk_rows")
    return out_idx, out_score


def indexer_topk_two_stage(q, kc, w, m: int, k: int, *, block: int = 8, n_keep: int = 2048,
                           query_chunk: int = 0, out_idx=None, out_score=None, workspace=None, stream=None,
                           device_status=None):
    """Two-stage indexer top-k (``si_indexer_topk_two_stage``): the best
    n_keep blocks of `block` keys by the score of their pooled (mean) key,
    then the top-k of their keys and the incomplete block's visible keys.
    Returns (idx, score) [B, S, k], ordered as indexer_topk's."""
    B, S, T, H, D = _shapes(q, kc, w)
    out_idx, out_score = _outputs(B, S, k, q.device, out_idx, out_score, True)
    o = _options(q, kc, None, None, query_chunk, 0, workspace, device_status=device_status)
    st = _lib.si_indexer_topk_two_stage(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, S, T, H, D, m, k,
                                        int(block), int(n_keep), out_idx.data_ptr(), out_score.data_ptr(),
                                        _stream_ptr(stream), ctypes.byref(o))
    _check(st, "si_indexer_topk_two_stage")
    return out_idx, out_score


def two_stage_workspace_size(B, S, T, block=8, n_keep=2048, query_chunk=0) -> int:
    return int(_lib.si_two_stage_workspace_size(B, S, T, block, n_keep, query_chunk))


def sparse_attention(q, kv, idx, *, scale: float = 0.0, out=None, lse=None, stream=None, device_status=None):
    """Sparse attention over the selected latents (``si_sparse_attention``):
    q [B,S,H,Dk] bf16, kv [B,T,Dk] bf16, idx [B,S,k] int32 (-1 padding).
    Returns (out [B,S,H,Dv=512] bf16, lse [B,S,H] fp32)."""
    if q.dim() != 4 or kv.dim() != 3 or idx.dim() != 3:
        raise ValueError("q [B,S,H,Dk], kv [B,T,Dk], idx [B,S,k] expected")
    B, S, H, Dk = q.shape
    T, k = kv.shape[1], idx.shape[2]
    Dv = 512
    if kv.shape[0] != B or kv.shape[2] != Dk or idx.shape[:2] != (B, S):
        raise ValueError(f"shape mismatch q{tuple(q.shape)} kv{tuple(kv.shape)} idx{tuple(idx.shape)}")
    for name, t, dt in (("q", q, torch.bfloat16), ("kv", kv, torch.bfloat16), ("idx", idx, torch.int32)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != dt:
            raise ValueError(f"{name} must be a contiguous {dt} CUDA tensor")
    if out is None:
        out = torch.empty((B, S, H, Dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, S, H), dtype=torch.float32, device=q.device)
    o = Options()
    if device_status is not None:
        o.device_status = device_status.data_ptr()
    _check(_lib.si_sparse_attention(q.data_ptr(), kv.data_ptr(), idx.data_ptr(), B, S, T, H, Dk, Dv, k,
                                    float(scale), out.data_ptr(), lse.data_ptr(), _stream_ptr(stream),
                                    ctypes.byref(o)), "si_sparse_attention")
    return out, lse


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


def workspace_size(B, S, T, H, D, m, k, materialize: bool = False, mxfp4: bool = False) -> int:
    """si_indexer_workspace_size: the materialize path's scratch, or the
    streaming path's (the decoded keys for MXFP4 keys, else 0)."""
    o = Options()
    o.dtype = SI_DTYPE_MXFP4_KEYS if mxfp4 else SI_DTYPE_BF16
    return int(_lib.si_indexer_workspace_size(B, S, T, H, D, m, k, int(materialize), ctypes.byref(o)))


def device_status(stream=None) -> int:
    """Synchronise the stream; return SI_OK or the status of a device-side failure."""
    return int(_lib.si_device_status(_stream_ptr(stream)))


def _host_options(q, kc, q_scale, kc_scale, kc_mx_scale, query_chunk, key_tile, unsorted, device_status):
    """si_options for the host-buffer entry point: the scales are host tensors."""
    o = Options()
    if kc_mx_scale is not None:
        if q.dtype != torch.bfloat16 or kc.dtype != torch.uint8 or kc_mx_scale.dtype != torch.uint8:
            raise ValueError("MXFP4 keys: q bfloat16, kc uint8 codes and kc_mx_scale uint8 expected")
        o.dtype = SI_DTYPE_MXFP4_KEYS
        o.kc_mx_scale = kc_mx_scale.data_ptr()
    elif q.dtype == torch.bfloat16 and kc.dtype == torch.bfloat16:
        o.dtype = SI_DTYPE_BF16
    elif q.dtype in (torch.uint8, torch.float8_e4m3fn) and kc.element_size() == 1:
        if q_scale is None or kc_scale is None:
            raise ValueError("fp8 inputs need q_scale and kc_scale")
        o.dtype = SI_DTYPE_FP8_E4M3
        o.q_scale = q_scale.data_ptr()
        o.kc_scale = kc_scale.data_ptr()
    else:
        raise ValueError(f"unsupported q / kc dtypes {q.dtype} / {kc.dtype}")
    for name, t in (("q", q), ("kc", kc), ("q_scale", q_scale), ("kc_scale", kc_scale),
                    ("kc_mx_scale", kc_mx_scale)):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous host (CPU) tensor")
    o.query_chunk = int(query_chunk)
    o.key_tile = int(key_tile)
    o.unsorted = int(bool(unsorted))
    if device_status is not None:
        o.device_status = device_status.data_ptr()
    return o


def indexer_topk_host(q, kc, w, m: int, k: int, *, q_scale=None, kc_scale=None, row0: int | None = None,
                      query_chunk: int = 0, key_tile: int = 0, out_idx=None, out_score=None,
                      with_score: bool = True, unsorted: bool = False, stream=None, kc_mx_scale=None,
                      device_status=None, device=None, workspace=None):
    """End to end on HOST tensors (``si_indexer_topk_host``): q [B, R, H_I, D],
    w [B, R, H_I], kc [B, T, D] (and the fp8 / MXFP4 scales) in host memory,
    page-locked for the copies to overlap the scoring.  The library copies the
    keys once and the query rows in chunks of `query_chunk` rows (0 = 4096)
    through two device slots, overlapping the copies with the scoring, and
    returns when (idx, score) [B, R, k] are in host memory.  With `row0` the
    rows are rows row0 .. row0+R-1 of the sequences (default 0: the whole
    sequence).  `device` selects the GPU (default: the current one);
    `workspace` (a CUDA uint8 tensor of indexer_topk_host_workspace_size()
    bytes) replaces the call's own device allocation."""
    B, R, T, H, D = _shapes(q, kc, w, kc_mx_scale is not None, host=True)
    pin = q.is_pinned()
    if out_idx is None:
        out_idx = torch.empty((B, R, k), dtype=torch.int32, pin_memory=pin)
    if out_score is None and with_score:
        out_score = torch.empty((B, R, k), dtype=torch.float32, pin_memory=pin)
    for name, t in (("out_idx", out_idx), ("out_score", out_score)):
        if t is not None and (t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, R, k)):
            raise ValueError(f"{name} must be a contiguous host tensor of shape {(B, R, k)}")
    o = _host_options(q, kc, q_scale, kc_scale, kc_mx_scale, query_chunk, key_tile, unsorted, device_status)
    if workspace is not None:
        if not workspace.is_cuda or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous CUDA tensor")
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        st = _lib.si_indexer_topk_host(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, int(row0 or 0), R, T, H, D,
                                       m, k, out_idx.data_ptr(),
                                       out_score.data_ptr() if out_score is not None else None,
                                       _stream_ptr(stream), ctypes.byref(o))
    _check(st, "si_indexer_topk_host")
    return out_idx, out_score


def indexer_topk_host_workspace_size(B, R, T, H, D, k, *, with_score=True, query_chunk=0, dtype=SI_DTYPE_BF16):
    o = Options()
    o.dtype = dtype
    o.query_chunk = int(query_chunk)
    return int(_lib.si_indexer_topk_host_workspace_size(B, R, T, H, D, k, int(with_score), ctypes.byref(o)))


def indexer_topk_two_stage_host(q, kc, w, m: int, k: int, *, device="cuda", query_chunk: int = 0,
                                bufs: dict | None = None, sync: bool = True, **two_stage):
    """The two-stage indexer end to end on HOST tensors: copies q, kc and w
    to the device, runs ``si_indexer_topk_two_stage`` and copies (idx, score)
    back.  `bufs` may hold reusable device buffers from a previous call; with
    sync=False the copies back are only enqueued on the current stream."""
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
    B, S = q.shape[0], q.shape[1]
    oi = bufs.get("out_idx")
    os_ = bufs.get("out_score")
    if oi is None or oi.shape != (B, S, k):
        oi = bufs["out_idx"] = torch.empty((B, S, k), dtype=torch.int32, device=device)
        os_ = bufs["out_score"] = torch.empty((B, S, k), dtype=torch.float32, device=device)
    ws = bufs.get("workspace")
    need = two_stage_workspace_size(B, S, kc.shape[1], two_stage.get("block", 8), two_stage.get("n_keep", 2048),
                                    query_chunk)
    if ws is None or ws.numel() < need:
        ws = bufs["workspace"] = torch.empty(need, dtype=torch.uint8, device=device)
    indexer_topk_two_stage(qd, kd, wd, m, k, query_chunk=query_chunk, out_idx=oi, out_score=os_,
                           stream=stream, workspace=ws, **two_stage)
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


def test_stream_timeout(q, kc, w, m: int, k: int, out_idx, wait_limit_ns: int, stream=None,
                        device_status=None) -> int:
    """Test hook: run the streaming kernel with one key tile withheld and a
    short bounded-wait limit; returns the launch status.  The timeout itself
    lands in device_status (a zeroed int32 CUDA tensor of >= 2 elements) when
    given, else in the record device_status() reads."""
    B, S, T, H, D = _shapes(q, kc, w)
    ds = None
    if device_status is not None:
        if device_status.dtype != torch.int32 or device_status.numel() < 2 or not device_status.is_cuda:
            raise ValueError("device_status must be an int32 CUDA tensor of >= 2 elements")
        ds = device_status.data_ptr()
    return int(_lib.si_test_stream_timeout(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, S, T, m, k,
                                           out_idx.data_ptr(), _stream_ptr(stream), wait_limit_ns, ds))


def test_fail_allocations(n: int) -> None:
    """Test hook: the library's next n scratch allocations fail as if the
    device were out of memory (``si_test_fail_allocations``)."""
    _lib.si_test_fail_allocations(int(n))
