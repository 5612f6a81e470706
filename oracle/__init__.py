"""CPU oracle for single-query decode attention (ctypes shim over fd_oracle.c).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package. The CUDA
product path never imports it, and the two share no code.

What it computes ("Flash-Decoding for long-context inference", Dao, Haziza,
Massa, Sizov): section "Multi-head attention for decoding" defines the result,
softmax(scale * q K^T) V over the cached tokens of each row, plus the
log-sum-exp of the logits; section "A faster attention for decoding:
Flash-Decoding" gives the split / per-split log-sum-exp / rescaled reduction
steps that reach the same result. Inputs are bf16 bit patterns (numpy uint16);
outputs are float64. ``attention_quant`` reads a cache of 8-bit codes (OCP
E4M3 or int8) dequantised with one scale per key/value head.
"""
import ctypes

import numpy as np

from . import build as _build

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_f64p_or_null = ctypes.c_void_p
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")

KV_TYPES = {"e4m3": 1, "int8": 2}   # codes of fdo_attention_quant's kv_type


class Oracle:
    """Handle on one build of the oracle library."""

    def __init__(self, path: str | None = None):
        if path is None:
            path = _build.build()
        self.path = path
        lib = ctypes.CDLL(path)
        lib.fdo_attention.restype = ctypes.c_int
        lib.fdo_attention.argtypes = [ctypes.c_int] * 5 + [_u16p, _u16p, _u16p, _i32p,
                                                           ctypes.c_double, _f64p, _f64p, ctypes.c_int]
        lib.fdo_split_attention.restype = ctypes.c_int
        lib.fdo_split_attention.argtypes = ([ctypes.c_int] * 5 + [_u16p, _u16p, _u16p, _i32p, ctypes.c_double,
                                            ctypes.c_int, _i32p, _f64p, _f64p,
                                            _f64p_or_null, _f64p_or_null, ctypes.c_int])
        lib.fdo_attention_multi.restype = ctypes.c_int
        lib.fdo_attention_multi.argtypes = [ctypes.c_int] * 6 + [_u16p, _u16p, _u16p, _i32p, ctypes.c_double,
                                                                 _f64p, _f64p, ctypes.c_int]
        lib.fdo_attention_quant.restype = ctypes.c_int
        lib.fdo_attention_quant.argtypes = ([ctypes.c_int] * 7 + [_u16p, _u8p, _u8p, _f32p, _f32p, _i32p,
                                                                  ctypes.c_double, _f64p, _f64p, ctypes.c_int])
        lib.fdo_combine.restype = ctypes.c_int
        lib.fdo_combine.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p, _f64p, _f64p, _f64p]
        lib.fdo_mutant.restype = ctypes.c_int
        self.lib = lib
        self.mutant = lib.fdo_mutant()
        self.threads_used = 0

    @staticmethod
    def _shapes(q, k):
        B, Hq, D = q.shape
        B2, Hkv, Lmax, D2 = k.shape
        if B2 != B or D2 != D:
            raise ValueError("q and k shapes disagree")
        return B, Hq, Hkv, D, Lmax

    @staticmethod
    def _prep(q, k, v, seqlens):
        q = np.ascontiguousarray(q, dtype=np.uint16)
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
        if k.shape != v.shape:
            raise ValueError("k and v shapes disagree")
        return q, k, v, seqlens

    def attention(self, q, k, v, seqlens, scale, nthreads=0):
        """Plain attention. q [B,Hq,D], k/v [B,Hkv,Lmax,D] bf16 bits (uint16),
        seqlens [B]. Returns (out [B,Hq,D], lse [B,Hq]) as float64."""
        q, k, v, seqlens = self._prep(q, k, v, seqlens)
        B, Hq, Hkv, D, Lmax = self._shapes(q, k)
        out = np.zeros((B, Hq, D), np.float64)
        lse = np.zeros((B, Hq), np.float64)
        rc = self.lib.fdo_attention(B, Hq, Hkv, D, Lmax, q, k, v, seqlens, float(scale), out, lse, int(nthreads))
        if rc <= 0:
            raise RuntimeError(f"fdo_attention failed ({rc})")
        self.threads_used = rc
        return out, lse

    def attention_multi(self, q, k, v, seqlens, scale, nthreads=0):
        """Several queries per sequence, causal among the new tokens.
        q [B,q_len,Hq,D]; k/v [B,Hkv,Lmax,D]; query j of sequence b sees the
        first seqlens[b] - (q_len - 1 - j) tokens. Returns (out [B,q_len,Hq,D],
        lse [B,q_len,Hq]) as float64."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
        B, q_len, Hq, D = q.shape
        _, Hkv, Lmax, _ = k.shape
        out = np.zeros((B, q_len, Hq, D), np.float64)
        lse = np.zeros((B, q_len, Hq), np.float64)
        rc = self.lib.fdo_attention_multi(B, q_len, Hq, Hkv, D, Lmax, q, k, v, seqlens, float(scale), out, lse,
                                          int(nthreads))
        if rc <= 0:
            raise RuntimeError(f"fdo_attention_multi failed ({rc})")
        self.threads_used = rc
        return out, lse

    def attention_quant(self, q, k8, v8, k_scale, v_scale, seqlens, scale, kv_type, nthreads=0):
        """Attention over a quantised cache. q [B,Hq,D] or [B,q_len,Hq,D] bf16
        bits; k8/v8 [B,Hkv,Lmax,D] uint8 codes; k_scale/v_scale [Hkv] float32;
        kv_type "e4m3" or "int8". Returns (out, lse) shaped like q (without D
        for lse), float64."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        single = q.ndim == 3
        if single:
            q = q[:, None]
        k8 = np.ascontiguousarray(k8, dtype=np.uint8)
        v8 = np.ascontiguousarray(v8, dtype=np.uint8)
        ks = np.ascontiguousarray(k_scale, dtype=np.float32)
        vs = np.ascontiguousarray(v_scale, dtype=np.float32)
        seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
        B, q_len, Hq, D = q.shape
        _, Hkv, Lmax, _ = k8.shape
        if k8.shape != v8.shape or ks.shape != (Hkv,) or vs.shape != (Hkv,):
            raise ValueError("cache or scale shapes disagree")
        out = np.zeros((B, q_len, Hq, D), np.float64)
        lse = np.zeros((B, q_len, Hq), np.float64)
        rc = self.lib.fdo_attention_quant(B, q_len, Hq, Hkv, D, Lmax, KV_TYPES[kv_type], q, k8, v8, ks, vs, seqlens,
                                          float(scale), out, lse, int(nthreads))
        if rc <= 0:
            raise RuntimeError(f"fdo_attention_quant failed ({rc})")
        self.threads_used = rc
        return (out[:, 0], lse[:, 0]) if single else (out, lse)

    def split_attention(self, q, k, v, seqlens, scale, bounds, nthreads=0, want_parts=False):
        """Split-then-reduce form with token boundaries ``bounds`` (nsplit+1
        ascending positions). Returns (out, lse) or, with want_parts,
        (out, lse, part_o [B,Hq,nsplit,D], part_lse [B,Hq,nsplit])."""
        q, k, v, seqlens = self._prep(q, k, v, seqlens)
        B, Hq, Hkv, D, Lmax = self._shapes(q, k)
        bounds = np.ascontiguousarray(bounds, dtype=np.int32)
        n = len(bounds) - 1
        out = np.zeros((B, Hq, D), np.float64)
        lse = np.zeros((B, Hq), np.float64)
        po = np.zeros((B, Hq, n, D), np.float64) if want_parts else None
        pl = np.zeros((B, Hq, n), np.float64) if want_parts else None
        rc = self.lib.fdo_split_attention(
            B, Hq, Hkv, D, Lmax, q, k, v, seqlens, float(scale), n, bounds, out, lse,
            po.ctypes.data if want_parts else None, pl.ctypes.data if want_parts else None, int(nthreads))
        if rc <= 0:
            raise RuntimeError(f"fdo_split_attention failed ({rc})")
        self.threads_used = rc
        return (out, lse, po, pl) if want_parts else (out, lse)

    def combine(self, part_o, part_lse):
        """Final reduction alone: part_o [rows,nsplit,D], part_lse [rows,nsplit]."""
        po = np.ascontiguousarray(part_o, dtype=np.float64)
        pl = np.ascontiguousarray(part_lse, dtype=np.float64)
        rows, n, D = po.shape
        out = np.zeros((rows, D), np.float64)
        lse = np.zeros((rows,), np.float64)
        if self.lib.fdo_combine(rows, n, D, po, pl, out, lse) != 0:
            raise RuntimeError("fdo_combine failed")
        return out, lse


_default = None


def default() -> Oracle:
    """The oracle built from fd_oracle.c with no planted mistake."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def attention(q, k, v, seqlens, scale, nthreads=0):
    return default().attention(q, k, v, seqlens, scale, nthreads)


def split_attention(q, k, v, seqlens, scale, bounds, nthreads=0, want_parts=False):
    return default().split_attention(q, k, v, seqlens, scale, bounds, nthreads, want_parts)


def combine(part_o, part_lse):
    return default().combine(part_o, part_lse)


def attention_multi(q, k, v, seqlens, scale, nthreads=0):
    return default().attention_multi(q, k, v, seqlens, scale, nthreads)


def attention_quant(q, k8, v8, k_scale, v_scale, seqlens, scale, kv_type, nthreads=0):
    return default().attention_quant(q, k8, v8, k_scale, v_scale, seqlens, scale, kv_type, nthreads)


LIBRARY = _build.LIBRARY
SOURCE = _build.SOURCE
__all__ = ["Oracle", "default", "attention", "attention_multi", "attention_quant", "KV_TYPES", "split_attention", "combine", "LIBRARY", "SOURCE"]
