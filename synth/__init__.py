"""Seeded synthetic inputs for the CSA lightning-indexer top-k step.

Shared by the CUDA path's tests and benchmark and by the CPU oracle's tests.
Nothing here computes an indexer score or a top-k: it only draws numbers
(counter-based SplitMix64, Box-Muller normals) and stores them as bf16,
fp8 e4m3 with per-row fp32 scales, or fp32.  The C source is ``synth.c``;
it is compiled on first use into ``libsynth.so`` beside it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

TENSOR_Q, TENSOR_KC, TENSOR_W = 1, 2, 3
TENSOR_QA, TENSOR_KV = 4, 5  # the sparse attention's queries and compressed latents


def build(force: bool = False) -> str:
    """Compile libsynth.so (gcc, -O2, pthreads) if missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-shared", "-fPIC", "-pthread",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.synth_draw.restype = ctypes.c_uint64
        L.synth_draw.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        L.synth_stream_key.restype = ctypes.c_uint64
        L.synth_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
        L.synth_normal.restype = ctypes.c_double
        L.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        L.synth_f32_to_bf16.restype = ctypes.c_uint16
        L.synth_f32_to_bf16.argtypes = [ctypes.c_float]
        L.synth_f32_to_e4m3.restype = ctypes.c_uint8
        L.synth_f32_to_e4m3.argtypes = [ctypes.c_float]
        L.synth_matrix.restype = ctypes.c_int
        L.synth_matrix.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                   ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_double,
                                   ctypes.c_int, ctypes.c_int]
        L.synth_matrix_range.restype = ctypes.c_int
        L.synth_matrix_range.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int,
                                         ctypes.c_double, ctypes.c_int, ctypes.c_int]
        L.synth_keys_planted.restype = ctypes.c_int
        L.synth_keys_planted.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_double,
                                         ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_void_p]
        L.synth_weights.restype = ctypes.c_int
        L.synth_weights.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32,
                                    ctypes.c_int, ctypes.c_double, ctypes.c_int]
        L.synth_sample_rows.restype = ctypes.c_int
        L.synth_sample_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_uint64]
        _lib = L
    return _lib


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def matrix(rows: int, D: int, seed: int, tensor_id: int, kind: str = "gauss", sigma: float = 1.0,
           fmt: str = "bf16", out: np.ndarray | None = None, scale_out: np.ndarray | None = None):
    """rows x D matrix. kind 'gauss' (N(0,1)*sigma) or 'int' ({-3..3}).

    fmt 'bf16' -> uint16 array of bf16 bit patterns; 'e4m3' -> (uint8 codes,
    float32 per-row scales)."""
    k = {"gauss": 0, "int": 1}[kind]
    if fmt == "bf16":
        o = out if out is not None else np.empty((rows, D), dtype=np.uint16)
        rc = lib().synth_matrix(_ptr(o), None, rows, D, seed, tensor_id, k, sigma, 0, _threads())
        assert rc == 0
        return o
    o = out if out is not None else np.empty((rows, D), dtype=np.uint8)
    s = scale_out if scale_out is not None else np.empty((rows,), dtype=np.float32)
    rc = lib().synth_matrix(_ptr(o), _ptr(s), rows, D, seed, tensor_id, k, sigma, 1, _threads())
    assert rc == 0
    return o, s


def matrix_range(row0: int, rows: int, D: int, seed: int, tensor_id: int, kind: str = "gauss",
                 sigma: float = 1.0, fmt: str = "bf16", out: np.ndarray | None = None,
                 scale_out: np.ndarray | None = None):
    """Rows [row0, row0+rows) of `matrix(...)` with the same arguments: the
    same values, generated alone (out / scale_out receive them from their
    first element on)."""
    k = {"gauss": 0, "int": 1}[kind]
    if fmt == "bf16":
        o = out if out is not None else np.empty((rows, D), dtype=np.uint16)
        assert o.dtype == np.uint16 and o.flags.c_contiguous and o.size >= rows * D
        rc = lib().synth_matrix_range(_ptr(o), None, row0, rows, D, seed, tensor_id, k, sigma, 0,
                                      _threads())
        assert rc == 0
        return o
    o = out if out is not None else np.empty((rows, D), dtype=np.uint8)
    s = scale_out if scale_out is not None else np.empty((rows,), dtype=np.float32)
    assert o.dtype == np.uint8 and o.flags.c_contiguous and o.size >= rows * D
    assert s.dtype == np.float32 and s.flags.c_contiguous and s.size >= rows
    rc = lib().synth_matrix_range(_ptr(o), _ptr(s), row0, rows, D, seed, tensor_id, k, sigma, 1,
                                  _threads())
    assert rc == 0
    return o, s


def keys_planted(B: int, T: int, D: int, seed: int, tensor_id: int, sigma: float, frac: float,
                 boost: float, fmt: str = "bf16", with_mask: bool = False):
    """[B*T, D] keys, N(0,1)*sigma with round(frac*T) rows per sequence boosted
    by `boost` times a per-sequence unit direction."""
    mask = np.empty((B * T,), dtype=np.uint8) if with_mask else None
    mptr = _ptr(mask) if with_mask else None
    if fmt == "bf16":
        o = np.empty((B * T, D), dtype=np.uint16)
        rc = lib().synth_keys_planted(_ptr(o), None, B, T, D, seed, tensor_id, sigma, frac, boost, 0,
                                      _threads(), mptr)
        assert rc == 0
        return (o, mask) if with_mask else o
    o = np.empty((B * T, D), dtype=np.uint8)
    s = np.empty((B * T,), dtype=np.float32)
    rc = lib().synth_keys_planted(_ptr(o), _ptr(s), B, T, D, seed, tensor_id, sigma, frac, boost, 1,
                                  _threads(), mptr)
    assert rc == 0
    return ((o, s), mask) if with_mask else (o, s)


def weights(n: int, seed: int, tensor_id: int, kind: str = "uniform", scale: float = 1.0,
            out: np.ndarray | None = None) -> np.ndarray:
    """n fp32 weights: 'uniform' U(0,1)*scale, or 'pow2' 2^-j with j in {0..6}."""
    o = out if out is not None else np.empty((n,), dtype=np.float32)
    rc = lib().synth_weights(_ptr(o), n, seed, tensor_id, {"uniform": 0, "pow2": 1}[kind], scale,
                             _threads())
    assert rc == 0
    return o


def sample_rows(count: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """`count` distinct integers drawn uniformly from [lo, hi), sorted."""
    o = np.empty((count,), dtype=np.int64)
    rc = lib().synth_sample_rows(_ptr(o), count, lo, hi, seed)
    assert rc == 0
    return o


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even) bit patterns, vectorised."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


# --------------------------------------------------------------------------
# The indexer workloads.  Shapes and value distributions are the tiny,
# integer-exact, sweep, V4-Flash and million-token cases of the lightning
# indexer at compression ratio m=4, H_I=64 heads, D=128.
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    m: int
    H: int
    D: int
    k: int
    seed: int
    kind: str            # "gauss" | "int" | "planted"
    sweep: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def T(self) -> int:
        return self.S // self.m

    def visible_pairs(self) -> int:
        """Number of causally visible (query, key) pairs for one sequence."""
        return self.B * visible_pairs(self.S, self.T, self.m)


def visible_pairs(S: int, T: int, m: int) -> int:
    """sum over t in [0, S) of min(T, floor((t+1)/m)), in closed form.

    With x = t+1: floor(x/m) < T for x <= m*T-1, and the sum of floor(x/m) for
    x = 1..N is m*q*(q-1)/2 + q*(r+1) with (q, r) = divmod(N, m)."""
    upto = min(S, m * T - 1)
    q, r = divmod(upto, m)
    return m * q * (q - 1) // 2 + q * (r + 1) + (S - upto) * T


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1024, 4, 64, 128, 64, 0, "gauss"),
    "integer": Workload("integer", 1, 8192, 4, 64, 128, 512, 1, "int"),
    "sweep": Workload("sweep", 1, 16384, 4, 64, 128, 512, 2, "gauss",
                      sweep={"query_chunk": [256, 512, 1024, 2048, 4096],
                             "key_tile": [64, 128, 256, 512, 1024],
                             "k": [64, 128, 256, 512, 1024]}),
    "v4flash": Workload("v4flash", 1, 65536, 4, 64, 128, 512, 3, "planted"),
    "million": Workload("million", 1, 1048576, 4, 64, 128, 512, 4, "planted"),
}

def quantize_mxfp4(x: np.ndarray):
    """OCP Microscaling FP4 of float rows [..., D] (D a multiple of 32): each
    block of 32 consecutive values gets the E8M0 scale 2^(floor(log2 amax) - 2)
    (2 is E2M1's largest exponent; an all-zero block gets 2^0), and each value
    / scale is rounded to nearest-even on the E2M1 grid, saturating at +-6.
    Returns (codes [..., D/2] uint8 -- value d in the low nibble of byte d/2
    when d is even, the high nibble when odd -- and scales [..., D/32] uint8)."""
    import ml_dtypes
    x = np.asarray(x, dtype=np.float32)
    D = x.shape[-1]
    assert D % 32 == 0
    blk = x.reshape(x.shape[:-1] + (D // 32, 32)).astype(np.float64)
    amax = np.abs(blk).max(axis=-1)
    e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2, 0).astype(np.int64)
    e = np.clip(e, -127, 127)
    scales = (e + 127).astype(np.uint8)
    v = np.clip(blk / np.ldexp(1.0, e)[..., None], -6.0, 6.0).astype(np.float32)
    codes = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    codes = codes.reshape(x.shape[:-1] + (D,))
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, scales


PLANTED_FRAC = 0.05
PLANTED_BOOST = 2.0


def make_inputs(wl: Workload, fmt: str = "bf16", S: int | None = None, B: int | None = None,
                seed: int | None = None, skip_q: bool = False):
    """Generate (q, kc, w[, q_scale, kc_scale]) host arrays for a workload.

    q: [B, S, H, D] (bf16 bits uint16, or e4m3 uint8 + q_scale [B, S, H])
    kc: [B, T, D]   (bf16 bits, or e4m3 + kc_scale [B, T])
    w: [B, S, H] float32
    `S`, `B` and `seed` override the workload's (for reduced-size cases).
    `skip_q` leaves q (and q_scale) out, for callers that make it piecewise
    with q_rows().
    fmt "mxfp4": q as for bf16; the bf16 keys quantised by quantize_mxfp4
    (kc: codes [B, T, D/2], kc_mx_scale: E8M0 [B, T, D/32]).
    """
    if fmt == "mxfp4":
        res = make_inputs(wl, "bf16", S=S, B=B, seed=seed, skip_q=skip_q)
        res["kc"], res["kc_mx_scale"] = quantize_mxfp4(bf16_bits_to_f32(res["kc"]))
        return res
    S = wl.S if S is None else S
    B = wl.B if B is None else B
    seed = wl.seed if seed is None else seed
    T = S // wl.m
    H, D = wl.H, wl.D
    sig = 1.0 / np.sqrt(D)
    kind = "int" if wl.kind == "int" else "gauss"
    qsig = 1.0 if kind == "int" else sig
    res = {}
    if skip_q:
        q = None
    elif fmt == "bf16":
        q = matrix(B * S * H, D, seed, TENSOR_Q, kind, qsig, "bf16").reshape(B, S, H, D)
    else:
        q8, qs = matrix(B * S * H, D, seed, TENSOR_Q, kind, qsig, "e4m3")
        q = q8.reshape(B, S, H, D)
        res["q_scale"] = qs.reshape(B, S, H)
    if wl.kind == "planted":
        kcr = keys_planted(B, T, D, seed, TENSOR_KC, sig, PLANTED_FRAC, PLANTED_BOOST, fmt)
    else:
        kcr = matrix(B * T, D, seed, TENSOR_KC, kind, qsig, fmt)
    if fmt == "bf16":
        kc = kcr.reshape(B, T, D)
    else:
        kc = kcr[0].reshape(B, T, D)
        res["kc_scale"] = kcr[1].reshape(B, T)
    if wl.kind == "int":
        w = weights(B * S * H, seed, TENSOR_W, "pow2").reshape(B, S, H)
    else:
        w = weights(B * S * H, seed, TENSOR_W, "uniform", 1.0 / np.sqrt(H)).reshape(B, S, H)
    res.update(kc=kc, w=w)
    if q is not None:
        res["q"] = q
    return res


def _q_kind(wl: Workload):
    kind = "int" if wl.kind == "int" else "gauss"
    return kind, (1.0 if kind == "int" else 1.0 / np.sqrt(wl.D))


def q_rows(wl: Workload, b: int, t0: int, n: int, fmt: str = "bf16", seed: int | None = None,
           S: int | None = None, out: np.ndarray | None = None, scale_out: np.ndarray | None = None):
    """q[b, t0:t0+n] of make_inputs(wl, fmt, S, seed=seed), generated alone:
    [n, H, D] bf16 bits, or (e4m3 codes, q_scale [n, H])."""
    S = wl.S if S is None else S
    seed = wl.seed if seed is None else seed
    fmt = "bf16" if fmt == "mxfp4" else fmt  # queries stay bf16 with MXFP4 keys
    kind, sig = _q_kind(wl)
    row0 = (b * S + t0) * wl.H
    res = matrix_range(row0, n * wl.H, wl.D, seed, TENSOR_Q, kind, sig, fmt, out=out, scale_out=scale_out)
    if fmt == "bf16":
        return res.reshape(n, wl.H, wl.D)
    return res[0].reshape(n, wl.H, wl.D), res[1].reshape(n, wl.H)


def make_inputs_rows(wl: Workload, rows, fmt: str = "bf16", seed: int | None = None):
    """make_inputs(wl, fmt, seed=seed) with q (and q_scale) generated only at
    the given flat query rows b*S+t; kc and w are complete.  The other q rows
    are left unwritten in a lazily allocated array, so a few rows of a
    million-token sequence cost a few MiB of host memory."""
    seed = wl.seed if seed is None else seed
    B, S, T, H, D = wl.B, wl.S, wl.T, wl.H, wl.D
    full = make_inputs(wl, fmt=fmt, S=S, B=B, seed=seed, skip_q=True)
    fmt = "bf16" if fmt == "mxfp4" else fmt  # queries stay bf16 with MXFP4 keys
    qdt = np.uint16 if fmt == "bf16" else np.uint8
    q = np.empty((B, S, H, D), dtype=qdt)
    qs = np.empty((B, S, H), dtype=np.float32) if fmt != "bf16" else None
    for r in np.asarray(rows, dtype=np.int64):
        b, t = divmod(int(r), S)
        if fmt == "bf16":
            q_rows(wl, b, t, 1, fmt, seed, out=q[b, t])
        else:
            q_rows(wl, b, t, 1, fmt, seed, out=q[b, t], scale_out=qs[b, t])
    full["q"] = q
    if qs is not None:
        full["q_scale"] = qs
    return full


def attention_inputs(B: int, S: int, T: int, seed: int, H: int = 64, Dk: int = 576, kind: str = "gauss"):
    """Inputs of the sparse attention over selected latents: q [B, S, H, Dk]
    and kv [B, T, Dk] as bf16 bits, N(0, 1) (so that with scale 1/sqrt(Dk) the
    logits have unit spread) or integers in {-3..3} (kind 'int')."""
    q = matrix(B * S * H, Dk, seed, TENSOR_QA, kind, 1.0).reshape(B, S, H, Dk)
    kv = matrix(B * T, Dk, seed, TENSOR_KV, kind, 1.0).reshape(B, T, Dk)
    return q, kv
