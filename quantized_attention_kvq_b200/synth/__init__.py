"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

The generator (``kvqgen.c``) is counter-based SplitMix64 + Box-Muller; it holds
none of the method's arithmetic.  Distributions follow the workload recipe:
q ~ N(0,1); V ~ N(0,1); K = N(0,1) * c[kv_head][channel] with
c = exp(0.5 * N(0,1)) and 4 outlier channels per KV head multiplied by 10.
Values are formed in fp64, rounded to fp32 and, for bf16 workloads, rounded
again (nearest-even) to bf16, which the kernels and the oracle both consume.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(os.path.dirname(_HERE), "lib", "libkvqgen.so")

TAG_Q, TAG_K, TAG_V, TAG_CHSCALE, TAG_LENS = 1, 2, 3, 4, 5

_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(LIB_PATH)
        u64, i64, i32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32
        lib.kvqgen_u64.restype = u64
        lib.kvqgen_u64.argtypes = [u64, u64]
        lib.kvqgen_key.restype = u64
        lib.kvqgen_key.argtypes = [u64, u64]
        lib.kvqgen_normal.restype = ctypes.c_double
        lib.kvqgen_normal.argtypes = [u64, u64]
        lib.kvqgen_fill.restype = None
        lib.kvqgen_fill.argtypes = [u64, u64, i64, ctypes.c_void_p, i64, i32, ctypes.c_void_p]
        lib.kvqgen_chscale.restype = None
        lib.kvqgen_chscale.argtypes = [u64, i32, ctypes.c_double, i32, ctypes.c_double, ctypes.c_void_p]
        lib.kvqgen_lengths.restype = None
        lib.kvqgen_lengths.argtypes = [u64, i32, i32, i32, ctypes.c_void_p]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def u64(key: int, n: int) -> int:
    return _load().kvqgen_u64(key, n)


def stream_key(seed: int, tag: int) -> int:
    return _load().kvqgen_key(seed, tag)


def normals(key: int, first: int, count: int, fmt: str = "f32", scale: np.ndarray | None = None) -> np.ndarray:
    """Normals ``first .. first+count-1`` of stream ``key`` (times ``scale[e % len(scale)]``)."""
    lib = _load()
    out = np.empty(count, dtype=np.uint16 if fmt == "bf16" else np.float32)
    sp, per = 0, 1
    if scale is not None:
        scale = np.ascontiguousarray(scale, dtype=np.float64)
        sp, per = _ptr(scale), scale.size
    lib.kvqgen_fill(key, first, count, sp, per, 1 if fmt == "bf16" else 0, _ptr(out))
    return out


def dual_pair(key: int, H: int, d: int = 128, spread: float = 0.35) -> tuple:
    """Caller inputs of the dual transform pair: per kv head an anisotropic
    invertible T = I + spread * N / sqrt(d) with its first d/2 columns doubled,
    and T's inverse transpose, both fp32 [H][d][d] (seeded normals N)."""
    z = normals(stream_key(key, 0x7A17), 0, H * d * d).astype(np.float64).reshape(H, d, d)
    tq = np.empty((H, d, d), np.float32)
    tk = np.empty((H, d, d), np.float32)
    for h in range(H):
        t = np.eye(d) + spread * z[h] / np.sqrt(d)
        t[:, : d // 2] *= 2.0
        tq[h] = t
        tk[h] = np.linalg.inv(t).T
    return tq, tk


def rope_inv_freq(base: float, d: int = 128) -> np.ndarray:
    """A model's rotary inverse frequencies base^(-2i/d), i < d/2, fp32."""
    return (base ** (-np.arange(0, d, 2, dtype=np.float64) / d)).astype(np.float32)


def channel_scales(key: int, d: int, sigma: float = 0.5, n_outliers: int = 4, mult: float = 10.0) -> np.ndarray:
    out = np.empty(d, dtype=np.float64)
    _load().kvqgen_chscale(key, d, sigma, n_outliers, mult, _ptr(out))
    return out


def lengths(key: int, count: int, lo: int, hi: int) -> np.ndarray:
    out = np.empty(count, dtype=np.int32)
    _load().kvqgen_lengths(key, count, lo, hi, _ptr(out))
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to fp32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


class Synth:
    """Inputs of one workload, drawn per (batch, kv-head) slice on demand.

    K and V are [B][Hkv][T][d]; element (b, h, n, c) uses counter
    ((b*Hkv + h)*T + n)*d + c of its tensor's stream, so any slice can be
    regenerated on its own.  q is [B][Hq][d].
    """

    def __init__(self, seed: int, B: int, Hq: int, Hkv: int, d: int, T: int, fmt: str,
                 len_range: tuple[int, int] | None = None):
        self.seed, self.B, self.Hq, self.Hkv, self.d, self.T, self.fmt = seed, B, Hq, Hkv, d, T, fmt
        self.kq = stream_key(seed, TAG_Q)
        self.kk = stream_key(seed, TAG_K)
        self.kv = stream_key(seed, TAG_V)
        kcs = stream_key(seed, TAG_CHSCALE)
        self.chscale = np.stack([channel_scales(u64(kcs, h + 1), d) for h in range(Hkv)])
        if len_range is None:
            self.lens = np.full(B, T, dtype=np.int32)
        else:
            self.lens = lengths(stream_key(seed, TAG_LENS), B, len_range[0], len_range[1])

    @property
    def np_dtype(self):
        return np.uint16 if self.fmt == "bf16" else np.float32

    def q(self) -> np.ndarray:
        return normals(self.kq, 0, self.B * self.Hq * self.d, self.fmt).reshape(self.B, self.Hq, self.d)

    def _first(self, b: int, h: int, n0: int) -> int:
        return ((b * self.Hkv + h) * self.T + n0) * self.d

    def k_slice(self, b: int, h: int, n0: int = 0, n: int | None = None) -> np.ndarray:
        n = self.T - n0 if n is None else n
        return normals(self.kk, self._first(b, h, n0), n * self.d, self.fmt, self.chscale[h]).reshape(n, self.d)

    def v_slice(self, b: int, h: int, n0: int = 0, n: int | None = None) -> np.ndarray:
        n = self.T - n0 if n is None else n
        return normals(self.kv, self._first(b, h, n0), n * self.d, self.fmt).reshape(n, self.d)

    def k_full(self) -> np.ndarray:
        out = np.empty((self.B, self.Hkv, self.T, self.d), dtype=self.np_dtype)
        for b in range(self.B):
            for h in range(self.Hkv):
                out[b, h] = self.k_slice(b, h)
        return out

    def v_full(self) -> np.ndarray:
        return normals(self.kv, 0, self.B * self.Hkv * self.T * self.d, self.fmt).reshape(
            self.B, self.Hkv, self.T, self.d)
