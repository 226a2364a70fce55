"""Thin ctypes binding of ``lib/libkvq.so`` (C ABI in ``include/kvq.h``).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  torch supplies device memory and the current CUDA stream.  There is
no CPU fallback; a missing library or a non-CUDA tensor raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

# KVQ_LIBRARY=checked selects the bounds-checked debug build of the same library
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib",
                        "libkvq_checked.so" if os.environ.get("KVQ_LIBRARY") == "checked" else "libkvq.so")

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA, KVQ_ERR_TIMEOUT = range(7)
KVQ_F32, KVQ_BF16, KVQ_F16 = 0, 1, 2

# every exported symbol the header declares
SYMBOLS = ("kvq_cache_sizes", "kvq_window_bytes", "kvq_quantize_append", "kvq_select_channels",
           "kvq_select_channels_at", "kvq_decode_workspace_bytes", "kvq_decode_attention", "kvq_decode_partials", "kvq_decode_combine",
           "kvq_decode_step_workspace_bytes",
           "kvq_decode_step_host", "kvq_decode_attention_static", "kvq_decode_attention_select",
           "kvq_decode_partials_select", "kvq_decode_status", "kvq_test_withhold_tile", "kvq_bounds_violations",
           "kvq_status_string")

_P = ctypes.c_void_p
_I32 = ctypes.c_int32


class KvqCacheStruct(ctypes.Structure):
    _fields_ = [("batch", _I32), ("kv_heads", _I32), ("head_dim", _I32), ("capacity", _I32),
                ("k_bits", _I32), ("v_bits", _I32), ("group_size", _I32), ("prune_granule", _I32),
                ("rotate_k", _I32), ("keep_ch0", _I32), ("rotate_v", _I32), ("v_clip", ctypes.c_float),
                ("k_codes", _P), ("k_scales", _P), ("k_ch0", _P), ("v_codes", _P), ("v_scales", _P),
                ("sink_tokens", _I32), ("recent_tokens", _I32), ("k_window", _P), ("v_window", _P),
                ("t_query", _P), ("t_key", _P), ("bucket_tokens", _I32), ("rope_inv_freq", _P)]


class KvqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        C = ctypes.POINTER(KvqCacheStruct)
        L.kvq_cache_sizes.argtypes = [C, ctypes.POINTER(ctypes.c_size_t)]
        L.kvq_cache_sizes.restype = ctypes.c_int
        L.kvq_window_bytes.argtypes = [C]
        L.kvq_window_bytes.restype = ctypes.c_size_t
        L.kvq_quantize_append.argtypes = [C, _P, _P, ctypes.c_int, _I32, _I32, _P]
        L.kvq_quantize_append.restype = ctypes.c_int
        L.kvq_select_channels.argtypes = [C, _P, ctypes.c_int, _I32, _I32, _P, _P]
        L.kvq_select_channels.restype = ctypes.c_int
        L.kvq_select_channels_at.argtypes = [C, _P, ctypes.c_int, _I32, _P, _I32, _P, _P]
        L.kvq_select_channels_at.restype = ctypes.c_int
        L.kvq_decode_workspace_bytes.argtypes = [C, _I32, _I32]
        L.kvq_decode_workspace_bytes.restype = ctypes.c_size_t
        L.kvq_decode_attention.argtypes = [C, _P, ctypes.c_int, _I32, _P, _I32, _P, ctypes.c_float, _P, _P,
                                           ctypes.c_size_t, _P]
        L.kvq_decode_attention.restype = ctypes.c_int
        L.kvq_decode_partials.argtypes = [C, _P, ctypes.c_int, _I32, _P, _I32, _P, ctypes.c_float, _P,
                                          ctypes.c_size_t, _P]
        L.kvq_decode_partials.restype = ctypes.c_int
        L.kvq_decode_combine.argtypes = [C, _I32, _P, _I32, _P, _P, ctypes.c_size_t, _P]
        L.kvq_decode_combine.restype = ctypes.c_int
        L.kvq_decode_step_workspace_bytes.argtypes = [C, ctypes.c_int, _I32, _I32]
        L.kvq_decode_step_workspace_bytes.restype = ctypes.c_size_t
        L.kvq_decode_step_host.argtypes = [C, _P, ctypes.c_int, _I32, _P, _I32, _I32, ctypes.c_float, _P, _P,
                                           ctypes.c_size_t, _P]
        L.kvq_decode_step_host.restype = ctypes.c_int
        L.kvq_decode_attention_static.argtypes = [C, _P, ctypes.c_int, _I32, _P, _I32, _P, ctypes.c_float, _P, _P]
        L.kvq_decode_attention_static.restype = ctypes.c_int
        L.kvq_decode_attention_select.argtypes = [C, _P, ctypes.c_int, _I32, _P, _I32, _I32, ctypes.c_float, _P,
                                                  _P, ctypes.c_size_t, _P]
        L.kvq_decode_attention_select.restype = ctypes.c_int
        L.kvq_decode_partials_select.argtypes = [C, _P, ctypes.c_int, _I32, _P, _I32, _I32, ctypes.c_float, _P,
                                                 ctypes.c_size_t, _P]
        L.kvq_decode_partials_select.restype = ctypes.c_int
        L.kvq_decode_status.argtypes = [C, _I32, _P, ctypes.c_size_t, _P]
        L.kvq_decode_status.restype = ctypes.c_int
        L.kvq_bounds_violations.argtypes = [_I32]
        L.kvq_bounds_violations.restype = ctypes.c_uint32
        L.kvq_test_withhold_tile.argtypes = [_I32]
        L.kvq_test_withhold_tile.restype = None
        L.kvq_status_string.argtypes = [ctypes.c_int]
        L.kvq_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().kvq_status_string(status).decode()


def _check(status: int, what: str):
    if status != KVQ_OK:
        raise KvqError(status, what)


def torch_dtype_code(t: torch.dtype) -> int:
    return {torch.float32: KVQ_F32, torch.bfloat16: KVQ_BF16, torch.float16: KVQ_F16}[t]


def _dev_ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def describe(B, H, capacity, k_bits, v_bits, rotate_k=1, keep_ch0=0, d=128, rotate_v=0, v_clip=1.0, sink=0,
             recent=0) -> KvqCacheStruct:
    d_ = KvqCacheStruct(B, H, d, capacity, k_bits, v_bits, 32, 4, rotate_k, keep_ch0, rotate_v, v_clip)
    d_.sink_tokens, d_.recent_tokens = sink, recent
    return d_


def cache_sizes(desc: KvqCacheStruct) -> list[int]:
    out = (ctypes.c_size_t * 5)()
    _check(lib().kvq_cache_sizes(ctypes.byref(desc), out), "kvq_cache_sizes")
    return list(out)


class KVQCache:
    """Packed quantized KV cache in device memory (torch-allocated, library-laid-out)."""

    def __init__(self, B: int, H: int, capacity: int, k_bits: int, v_bits: int, rotate_k: int = 1,
                 keep_ch0: int = 0, device="cuda", zero: bool = True, rotate_v: int = 0, v_clip: float = 1.0,
                 sink: int = 0, recent: int = 0, t_query: torch.Tensor | None = None,
                 t_key: torch.Tensor | None = None, bucket_tokens: int = 0,
                 rope_inv_freq: torch.Tensor | None = None):
        """rotate_k = 2 takes the caller's dual transform pair: t_query (T) and
        t_key (T^-T), fp32 device tensors [H][128][128], kept referenced here."""
        if rotate_k == 2 and (t_query is None or t_key is None):
            raise ValueError("rotate_k = 2 needs t_query and t_key")
        if rotate_k == 2 and (t_query.dtype != torch.float32 or t_key.dtype != torch.float32 or
                              tuple(t_query.shape) != (H, 128, 128) or tuple(t_key.shape) != (H, 128, 128)):
            raise ValueError("t_query and t_key are fp32 [H][128][128]")
        if bucket_tokens and (rope_inv_freq is None or rope_inv_freq.dtype != torch.float32 or
                              tuple(rope_inv_freq.shape) != (64,)):
            raise ValueError("bucket-relative RoPE needs rope_inv_freq, fp32 [64]")
        self.desc = describe(B, H, capacity, k_bits, v_bits, rotate_k, keep_ch0, rotate_v=rotate_v, v_clip=v_clip,
                             sink=sink, recent=recent)
        sizes = cache_sizes(self.desc)
        alloc = torch.zeros if zero else torch.empty
        self.k_codes = alloc(sizes[0], dtype=torch.uint8, device=device)
        self.k_scales = alloc(sizes[1], dtype=torch.uint8, device=device)
        self.k_ch0 = alloc(sizes[2], dtype=torch.uint8, device=device) if keep_ch0 else None
        self.v_codes = alloc(sizes[3], dtype=torch.uint8, device=device)
        self.v_scales = alloc(sizes[4], dtype=torch.uint8, device=device)
        self.desc.k_codes = _dev_ptr(self.k_codes)
        self.desc.k_scales = _dev_ptr(self.k_scales)
        self.desc.k_ch0 = _dev_ptr(self.k_ch0)
        self.desc.v_codes = _dev_ptr(self.v_codes)
        self.desc.v_scales = _dev_ptr(self.v_scales)
        wb = lib().kvq_window_bytes(ctypes.byref(self.desc)) if sink + recent else 0
        self.k_window = alloc(wb, dtype=torch.uint8, device=device) if wb else None  # bf16 token windows
        self.v_window = alloc(wb, dtype=torch.uint8, device=device) if wb else None
        self.desc.k_window = _dev_ptr(self.k_window)
        self.desc.v_window = _dev_ptr(self.v_window)
        self.t_query = t_query.contiguous() if rotate_k == 2 else None
        self.t_key = t_key.contiguous() if rotate_k == 2 else None
        self.desc.t_query = _dev_ptr(self.t_query)
        self.desc.t_key = _dev_ptr(self.t_key)
        self.rope_inv_freq = rope_inv_freq.contiguous() if bucket_tokens else None
        self.desc.bucket_tokens = bucket_tokens
        self.desc.rope_inv_freq = _dev_ptr(self.rope_inv_freq)
        self.n_buckets = capacity // bucket_tokens if bucket_tokens else 1
        self.B, self.H, self.capacity = B, H, capacity

    def sequence_desc(self, b: int) -> KvqCacheStruct:
        """Descriptor of sequence b alone (batch 1): every cache array is [B][...]
        with the sequence outermost, so this is a pointer offset per array."""
        per = [x // self.B for x in cache_sizes(self.desc)]
        d = describe(1, self.H, self.capacity, self.desc.k_bits, self.desc.v_bits, self.desc.rotate_k,
                     self.desc.keep_ch0, rotate_v=self.desc.rotate_v, v_clip=self.desc.v_clip,
                     sink=self.desc.sink_tokens, recent=self.desc.recent_tokens)
        d.k_codes = self.desc.k_codes + b * per[0]
        d.k_scales = self.desc.k_scales + b * per[1]
        d.k_ch0 = self.desc.k_ch0 + b * per[2] if self.desc.keep_ch0 else None
        d.v_codes = self.desc.v_codes + b * per[3]
        d.v_scales = self.desc.v_scales + b * per[4]
        if self.k_window is not None:
            wper = self.k_window.numel() // self.B
            d.k_window = self.desc.k_window + b * wper
            d.v_window = self.desc.v_window + b * wper
        d.t_query, d.t_key = self.desc.t_query, self.desc.t_key  # per kv head, shared by every sequence
        d.bucket_tokens, d.rope_inv_freq = self.desc.bucket_tokens, self.desc.rope_inv_freq
        return d

    def append_sequence(self, b: int, k_new: torch.Tensor, v_new: torch.Tensor, offset: int, stream=None):
        """Append [H][n_new][128] (or [1][H][n_new][128]) tokens to sequence b only."""
        d = self.sequence_desc(b)
        n_new = k_new.shape[-2]
        _check(lib().kvq_quantize_append(ctypes.byref(d), _dev_ptr(k_new), _dev_ptr(v_new),
                                         torch_dtype_code(k_new.dtype), n_new, offset, _stream(stream)),
               "kvq_quantize_append")

    # -- calls --------------------------------------------------------------
    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, offset: int, stream=None):
        """k_new, v_new: [B][H][n_new][128] (fp32 / bf16 / fp16) on the device."""
        n_new = k_new.shape[2] if k_new.dim() == 4 else 0
        _check(lib().kvq_quantize_append(ctypes.byref(self.desc), _dev_ptr(k_new), _dev_ptr(v_new),
                                         torch_dtype_code(k_new.dtype), n_new, offset, _stream(stream)),
               "kvq_quantize_append")

    def select(self, q: torch.Tensor, keep_groups: int, mask_out: torch.Tensor | None = None, stream=None):
        """q: [B][Hq][128]; returns mask [B][H] (int32 tensor holding uint32 bits)."""
        if mask_out is None:
            mask_out = torch.empty((self.B, self.H), dtype=torch.int32, device=q.device)
        _check(lib().kvq_select_channels(ctypes.byref(self.desc), _dev_ptr(q), torch_dtype_code(q.dtype),
                                         q.shape[1], keep_groups, _dev_ptr(mask_out), _stream(stream)),
               "kvq_select_channels")
        return mask_out

    def select_at(self, q: torch.Tensor, seq_lens: torch.Tensor, keep_groups: int,
                  mask_out: torch.Tensor | None = None, stream=None):
        """Selection for queries at positions seq_lens - 1; returns mask [B][nb][H]
        (nb buckets, 1 without bucket-relative RoPE)."""
        if mask_out is None:
            mask_out = torch.empty((self.B, self.n_buckets, self.H), dtype=torch.int32, device=q.device)
        _check(lib().kvq_select_channels_at(ctypes.byref(self.desc), _dev_ptr(q), torch_dtype_code(q.dtype),
                                            q.shape[1], _dev_ptr(seq_lens), keep_groups, _dev_ptr(mask_out),
                                            _stream(stream)),
               "kvq_select_channels_at")
        return mask_out

    def workspace_bytes(self, q_heads: int, max_len: int) -> int:
        return lib().kvq_decode_workspace_bytes(ctypes.byref(self.desc), q_heads, max_len)


    def decode(self, q: torch.Tensor, seq_lens: torch.Tensor, max_len: int, mask: torch.Tensor | None = None,
               softmax_scale: float | None = None, out: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """q: [B][Hq][128]; seq_lens: int32 [B] on the device; returns fp32 [B][Hq][128]."""
        Hq = q.shape[1]
        if softmax_scale is None:
            softmax_scale = 1.0 / math.sqrt(128)
        if out is None:
            out = torch.empty((self.B, Hq, 128), dtype=torch.float32, device=q.device)
        if workspace is None:
            workspace = torch.empty(max(self.workspace_bytes(Hq, max_len), 256), dtype=torch.uint8, device=q.device)
        _check(lib().kvq_decode_attention(ctypes.byref(self.desc), _dev_ptr(q), torch_dtype_code(q.dtype), Hq,
                                          _dev_ptr(seq_lens), max_len, _dev_ptr(mask), float(softmax_scale),
                                          _dev_ptr(out), _dev_ptr(workspace), workspace.numel(), _stream(stream)),
               "kvq_decode_attention")
        return out

    def decode_partials(self, q: torch.Tensor, seq_lens: torch.Tensor, max_len: int, mask, softmax_scale: float,
                        workspace: torch.Tensor, stream=None):
        _check(lib().kvq_decode_partials(ctypes.byref(self.desc), _dev_ptr(q), torch_dtype_code(q.dtype), q.shape[1],
                                         _dev_ptr(seq_lens), max_len, _dev_ptr(mask), float(softmax_scale),
                                         _dev_ptr(workspace), workspace.numel(), _stream(stream)),
               "kvq_decode_partials")

    def decode_select(self, q: torch.Tensor, seq_lens: torch.Tensor, max_len: int, keep_groups: int,
                      softmax_scale: float | None = None, out: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """decode() with the channel selection done inside the call (kvq_decode_attention_select)."""
        Hq = q.shape[1]
        if softmax_scale is None:
            softmax_scale = 1.0 / math.sqrt(128)
        if out is None:
            out = torch.empty((self.B, Hq, 128), dtype=torch.float32, device=q.device)
        if workspace is None:
            workspace = torch.empty(max(self.workspace_bytes(Hq, max_len), 256), dtype=torch.uint8, device=q.device)
        _check(lib().kvq_decode_attention_select(ctypes.byref(self.desc), _dev_ptr(q), torch_dtype_code(q.dtype), Hq,
                                                 _dev_ptr(seq_lens), max_len, keep_groups, float(softmax_scale),
                                                 _dev_ptr(out), _dev_ptr(workspace), workspace.numel(),
                                                 _stream(stream)),
               "kvq_decode_attention_select")
        return out

    def decode_partials_select(self, q: torch.Tensor, seq_lens: torch.Tensor, max_len: int, keep_groups: int,
                               softmax_scale: float, workspace: torch.Tensor, stream=None):
        _check(lib().kvq_decode_partials_select(ctypes.byref(self.desc), _dev_ptr(q), torch_dtype_code(q.dtype),
                                                q.shape[1], _dev_ptr(seq_lens), max_len, keep_groups,
                                                float(softmax_scale), _dev_ptr(workspace), workspace.numel(),
                                                _stream(stream)),
               "kvq_decode_partials_select")

    def decode_combine(self, q_heads: int, seq_lens: torch.Tensor, max_len: int, out: torch.Tensor,
                       workspace: torch.Tensor, stream=None):
        _check(lib().kvq_decode_combine(ctypes.byref(self.desc), q_heads, _dev_ptr(seq_lens), max_len,
                                        _dev_ptr(out), _dev_ptr(workspace), workspace.numel(), _stream(stream)),
               "kvq_decode_combine")

    def decode_status(self, q_heads: int, workspace: torch.Tensor, stream=None) -> int:
        """Status of the last split decode that used `workspace`: KVQ_OK or KVQ_ERR_TIMEOUT
        (synchronizes the stream)."""
        return lib().kvq_decode_status(ctypes.byref(self.desc), q_heads, _dev_ptr(workspace), workspace.numel(),
                                       _stream(stream))

    def step_workspace_bytes(self, dtype: torch.dtype, q_heads: int, max_len: int) -> int:
        return lib().kvq_decode_step_workspace_bytes(ctypes.byref(self.desc), torch_dtype_code(dtype), q_heads,
                                                     max_len)

    def decode_step_host(self, q_host: torch.Tensor, seq_lens: torch.Tensor, max_len: int, keep_groups: int,
                         softmax_scale: float, out_host: torch.Tensor, workspace: torch.Tensor, stream=None):
        """Host q in, host fp32 out (both CPU tensors, ideally pinned); asynchronous on the stream."""
        if q_host.is_cuda or out_host.is_cuda:
            raise ValueError("decode_step_host takes host tensors")
        _check(lib().kvq_decode_step_host(ctypes.byref(self.desc), q_host.data_ptr(), torch_dtype_code(q_host.dtype),
                                          q_host.shape[1], _dev_ptr(seq_lens), max_len, keep_groups,
                                          float(softmax_scale), out_host.data_ptr(), _dev_ptr(workspace),
                                          workspace.numel(), _stream(stream)),
               "kvq_decode_step_host")
