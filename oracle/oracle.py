"""ctypes wrapper of the C++ oracle (``kvq_oracle.cpp``) -- test infrastructure only.

Arrays cross as numpy buffers; bf16 inputs are widened to fp32 (exactly)
before they reach the oracle.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build_oracle

_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32


class OrcCache(ctypes.Structure):
    _fields_ = [("batch", _I32), ("kv_heads", _I32), ("head_dim", _I32), ("capacity", _I32),
                ("k_bits", _I32), ("v_bits", _I32), ("rotate_k", _I32), ("keep_ch0", _I32),
                ("rotate_v", _I32), ("v_clip", ctypes.c_float),
                ("k_codes", _P), ("k_scales", _P), ("k_ch0", _P), ("v_codes", _P), ("v_scales", _P),
                ("sink", _I32), ("recent", _I32), ("k_win", _P), ("v_win", _P), ("t_q", _P), ("t_k", _P),
                ("bucket_w", _I32), ("rope_inv_freq", _P)]


class OrcStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("k_elems", "v_elems", "k_exempt", "v_exempt", "k_clamped", "v_clamped", "groups_exempt")]


def lib():
    global _lib
    if _lib is None:
        so = build_oracle.build()
        L = ctypes.CDLL(so)
        L.orc_fwht.argtypes = [_P, _I32]
        L.orc_rotate.argtypes = [_P, _I32, _P]
        L.orc_transform.argtypes = [_P, _P, _I32, _P]
        L.orc_rope.argtypes = [_P, _I32, _P, ctypes.c_int64, _P]
        L.orc_select_buckets.argtypes = [ctypes.POINTER(OrcCache), _P, _I32, _P, _I32, _P, _P]
        L.orc_half_rn.argtypes = [ctypes.c_float]
        L.orc_half_rn.restype = ctypes.c_uint16
        L.orc_half_value.argtypes = [ctypes.c_uint16]
        L.orc_half_value.restype = ctypes.c_double
        L.orc_bf16_rn.argtypes = [ctypes.c_float]
        L.orc_bf16_rn.restype = ctypes.c_uint16
        L.orc_bf16_value.argtypes = [ctypes.c_uint16]
        L.orc_bf16_value.restype = ctypes.c_double
        L.orc_quantize_group.argtypes = [_P, _P, _I32, _I32, _P, _P, _P, _P, _P]
        L.orc_quantize_group.restype = _I32
        L.orc_quantize_group_clip.argtypes = [_P, _P, _I32, _I32, ctypes.c_float, _P, _P, _P, _P, _P]
        L.orc_quantize_group_clip.restype = _I32
        L.orc_quantize_append.argtypes = [ctypes.POINTER(OrcCache), _P, _P, _I32, _I32, ctypes.POINTER(OrcStats),
                                          _P, _P]
        L.orc_quantize_append.restype = _I32
        L.orc_unpack_codes.argtypes = [ctypes.POINTER(OrcCache), _I32, _I32, _I32, _I32, _P]
        L.orc_dequantize.argtypes = [ctypes.POINTER(OrcCache), _I32, _I32, _I32, _I32, _P, _P]
        L.orc_select.argtypes = [_P, _I32, _I32, _I32, _I32, _I32, _P, _I32, _P, _P]
        L.orc_attention.argtypes = [ctypes.POINTER(OrcCache), _P, _I32, _P, _P, ctypes.c_double, _P, _I32, _P]
        L.orc_dual_score.argtypes = [_P, _I32, _P, _P]
        L.orc_dual_score.restype = ctypes.c_double
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def as_f32(x: np.ndarray) -> np.ndarray:
    """fp32 values of an input array (bf16 bit patterns as uint16, or fp32)."""
    if x.dtype == np.uint16:
        return np.ascontiguousarray((x.astype(np.uint32) << 16).view(np.float32))
    return np.ascontiguousarray(x, dtype=np.float32)


def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalized fp64 Walsh-Hadamard butterflies (natural order)."""
    y = np.ascontiguousarray(x, dtype=np.float64).copy()
    lib().orc_fwht(_p(y), y.size)
    return y


def rotate(x: np.ndarray) -> np.ndarray:
    """fp32(FWHT(x)/sqrt(d)) of one row."""
    xi = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty_like(xi)
    lib().orc_rotate(_p(xi), xi.size, _p(out))
    return out


def transform(A: np.ndarray, x: np.ndarray) -> np.ndarray:
    """fp32 of the fp64 product A x (sum over j in order) of one row."""
    Ac = np.ascontiguousarray(A, dtype=np.float32)
    xi = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty_like(xi)
    lib().orc_transform(_p(Ac), _p(xi), xi.size, _p(out))
    return out


def rope(x: np.ndarray, inv_freq: np.ndarray, pos: int) -> np.ndarray:
    """Rotary embedding of one row at position pos (channel i paired with i + d/2)."""
    xi = np.ascontiguousarray(x, dtype=np.float32)
    fr = np.ascontiguousarray(inv_freq, dtype=np.float32)
    out = np.empty_like(xi)
    lib().orc_rope(_p(xi), xi.size, _p(fr), int(pos), _p(out))
    return out


def half_rn(x: float) -> int:
    return lib().orc_half_rn(float(x))


def half_value(h: int) -> float:
    return lib().orc_half_value(int(h))


def bf16_rn(x: float) -> int:
    return lib().orc_bf16_rn(float(x))


def bf16_value(h: int) -> float:
    return lib().orc_bf16_value(int(h))


def quantize_group(x, bits: int, include=None, clip: float = 1.0):
    """-> (s16 bits, z16 bits, codes, exempt flags, group_exempt, clamped count)"""
    xi = np.ascontiguousarray(x, dtype=np.float32)
    n = xi.size
    inc = None if include is None else np.ascontiguousarray(include, dtype=np.uint8)
    s = ctypes.c_uint16()
    z = ctypes.c_uint16()
    codes = np.zeros(n, np.uint8)
    ex = np.zeros(n, np.uint8)
    clamped = ctypes.c_int64(0)
    gex = lib().orc_quantize_group_clip(_p(xi), _p(inc), n, bits, float(clip), ctypes.byref(s), ctypes.byref(z),
                                        _p(codes), _p(ex), ctypes.byref(clamped))
    return s.value, z.value, codes, ex, gex, clamped.value


class Cache:
    """Host copy of the packed cache, written by the oracle."""

    def __init__(self, B, Hkv, d, capacity, k_bits, v_bits, rotate_k=1, keep_ch0=0, rotate_v=0, v_clip=1.0,
                 sink=0, recent=0, t_q=None, t_k=None, bucket_w=0, inv_freq=None):
        """rotate_k = 2 takes the caller's pair: t_q [Hkv][d][d] on queries and
        t_k [Hkv][d][d] (its inverse transpose) on keys, fp32 row-major.
        bucket_w > 0: keys and queries arrive before rotary embedding and are
        embedded relative to their bucket's anchor (inv_freq [d/2] fp32)."""
        self.B, self.Hkv, self.d, self.capacity = B, Hkv, d, capacity
        if rotate_k == 2:
            t_q = np.ascontiguousarray(t_q, dtype=np.float32).reshape(Hkv, d, d)
            t_k = np.ascontiguousarray(t_k, dtype=np.float32).reshape(Hkv, d, d)
        self.t_q, self.t_k = t_q, t_k
        self.bucket_w = bucket_w
        self.inv_freq = np.ascontiguousarray(inv_freq, dtype=np.float32) if bucket_w else None
        self.n_buckets = -(-capacity // bucket_w) if bucket_w else 1
        self.k_bits, self.v_bits, self.rotate_k, self.keep_ch0 = k_bits, v_bits, rotate_k, keep_ch0
        self.rotate_v, self.v_clip, self.sink, self.recent = rotate_v, v_clip, sink, recent
        w = B * Hkv * (sink + recent) * d
        self.k_win = np.zeros(w, np.uint16) if w else None  # bf16 windows
        self.v_win = np.zeros(w, np.uint16) if w else None
        blocked = -(-capacity // 128) * 128  # codes are stored in blocks of 128 tokens
        self.k_codes = np.zeros(B * Hkv * (d // 4) * blocked * (4 * k_bits // 8), np.uint8)
        self.k_scales = np.zeros(B * Hkv * (d // 32) * blocked * 2, np.uint16)
        self.k_ch0 = np.zeros(B * Hkv * capacity, np.uint16) if keep_ch0 else None
        self.v_codes = np.zeros(B * Hkv * d * blocked * v_bits // 8, np.uint8)  # channel rows per block
        self.v_scales = np.zeros(B * Hkv * capacity * (d // 32) * 2, np.uint16)
        self.struct = OrcCache(B, Hkv, d, capacity, k_bits, v_bits, rotate_k, keep_ch0, rotate_v, v_clip,
                               _p(self.k_codes), _p(self.k_scales), _p(self.k_ch0), _p(self.v_codes),
                               _p(self.v_scales), sink, recent, _p(self.k_win), _p(self.v_win),
                               _p(self.t_q) if rotate_k == 2 else None, _p(self.t_k) if rotate_k == 2 else None,
                               bucket_w, _p(self.inv_freq))

    def append(self, k_new: np.ndarray, v_new: np.ndarray, offset: int, want_exempt: bool = False):
        """k_new, v_new: [B][Hkv][n][d] (bf16 as uint16, or fp32)."""
        k = as_f32(k_new)
        v = as_f32(v_new)
        n_new = k.shape[2]
        st = OrcStats()
        kex = np.zeros(self.B * self.Hkv * n_new, np.uint8) if want_exempt else None
        vex = np.zeros(self.B * self.Hkv * n_new, np.uint8) if want_exempt else None
        rc = lib().orc_quantize_append(ctypes.byref(self.struct), _p(k), _p(v), n_new, offset, ctypes.byref(st),
                                       _p(kex), _p(vex))
        if rc != 0:
            raise ValueError("oracle rejected append arguments")
        stats = {f: getattr(st, f) for f, _ in OrcStats._fields_}
        if want_exempt:
            stats["k_row_exempt"] = kex.reshape(self.B, self.Hkv, n_new)
            stats["v_row_exempt"] = vex.reshape(self.B, self.Hkv, n_new)
        return stats

    def unpack(self, b, h, n, which):
        out = np.zeros(self.d, np.uint8)
        lib().orc_unpack_codes(ctypes.byref(self.struct), b, h, n, which, _p(out))
        return out

    def dequantize(self, b, h, n0, n):
        kh = np.zeros((n, self.d), np.float64)
        vh = np.zeros((n, self.d), np.float64)
        lib().orc_dequantize(ctypes.byref(self.struct), b, h, n0, n, _p(kh), _p(vh))
        return kh, vh

    def select_buckets(self, q: np.ndarray, lens: np.ndarray, keep: int):
        """-> (mask [B][nb][Hkv] uint32, energy [B][nb][Hkv][d/4]): one mask per bucket."""
        qf = as_f32(q)
        Hq = qf.shape[1]
        ln = np.ascontiguousarray(lens, dtype=np.int32)
        mask = np.zeros((self.B, self.n_buckets, self.Hkv), np.uint32)
        energy = np.zeros((self.B, self.n_buckets, self.Hkv, self.d // 4), np.float64)
        lib().orc_select_buckets(ctypes.byref(self.struct), _p(qf), Hq, _p(ln), keep, _p(mask), _p(energy))
        return mask, energy

    def attention(self, q: np.ndarray, lens: np.ndarray, mask: np.ndarray | None, scale: float,
                  rows: np.ndarray | None = None) -> np.ndarray:
        """q: [B][Hq][d]; returns [nrows][d] fp64 (all B*Hq rows when rows is None)."""
        qf = as_f32(q)
        Hq = qf.shape[1]
        ln = np.ascontiguousarray(lens, dtype=np.int32)
        mk = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint32)
        rw = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
        n = self.B * Hq if rw is None else rw.size
        out = np.zeros((n, self.d), np.float64)
        lib().orc_attention(ctypes.byref(self.struct), _p(qf), Hq, _p(ln), _p(mk), float(scale), _p(rw),
                            0 if rw is None else rw.size, _p(out))
        return out


def select(q: np.ndarray, Hkv: int, rotate: int, keep: int, t_q: np.ndarray | None = None):
    """-> (mask [B][Hkv] uint32, energy [B][Hkv][d/4] fp64); rotate = 2 takes
    the pair's query matrices t_q [Hkv][d][d]."""
    qf = as_f32(q)
    tq = np.ascontiguousarray(t_q, dtype=np.float32) if rotate == 2 else None
    B, Hq, d = qf.shape
    mask = np.zeros((B, Hkv), np.uint32)
    energy = np.zeros((B, Hkv, d // 4), np.float64)
    lib().orc_select(_p(qf), B, Hq, Hkv, d, rotate, _p(tq), keep, _p(mask), _p(energy))
    return mask, energy


def dual_score(T: np.ndarray, q: np.ndarray, k: np.ndarray) -> float:
    Tc = np.ascontiguousarray(T, dtype=np.float64)
    qc = np.ascontiguousarray(q, dtype=np.float64)
    kc = np.ascontiguousarray(k, dtype=np.float64)
    return lib().orc_dual_score(_p(Tc), Tc.shape[0], _p(qc), _p(kc))
