"""The allocation-free decode entry point (kvq_decode_attention_static).

It serves callers that cannot allocate device memory (an engine owning all
device memory in its own pool, or a decode loop that must not call cudaMalloc)
by keeping the split partials in a fixed array inside the library.  Its
output must match kvq_decode_attention's on the same inputs, on two calls in
a row (the second call reuses the array the first one left behind, with a
different shape), and sizes beyond the array are refused before any launch.
This file is collected last on purpose.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from kvq_testlib import assert_close_output, to_device
from quantized_attention_kvq_b200 import native, synth

pytestmark = pytest.mark.gpu


def call_static(cache, q, lens, max_len, mask, out):
    L = native.lib()
    return L.kvq_decode_attention_static(ctypes.byref(cache.desc), q.data_ptr(), native.torch_dtype_code(q.dtype),
                                         q.shape[1], lens.data_ptr(), max_len,
                                         None if mask is None else mask.data_ptr(), 1 / math.sqrt(128),
                                         out.data_ptr(), torch.cuda.current_stream().cuda_stream)


def make(seed, B, G, H, T, kb, vb, ch0):
    s = synth.Synth(seed, B, G * H, H, 128, T, "bf16")
    cache = native.KVQCache(B, H, T, kb, vb, 1, ch0)
    cache.append(to_device(s.k_full(), "bf16"), to_device(s.v_full(), "bf16"), 0)
    return cache, to_device(s.q(), "bf16")


def test_static_scratch_matches_workspace_entry_point_twice():
    cases = [
        # (seed, B, G, H, T, kb, vb, ch0, lens, keep)
        (41, 3, 4, 2, 2048, 4, 4, 0, [2048, 700, 1], 32),
        (42, 2, 8, 2, 1024, 4, 2, 1, [1000, 1024], 24),
    ]
    for seed, B, G, H, T, kb, vb, ch0, lens, keep in cases:
        cache, q = make(seed, B, G, H, T, kb, vb, ch0)
        lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
        mask = cache.select(q, keep) if keep < 32 else None
        want = cache.decode(q, lens_d, T, mask, 1 / math.sqrt(128))
        out = torch.full_like(want, float("nan"))
        assert call_static(cache, q, lens_d, T, mask, out) == native.KVQ_OK
        torch.cuda.synchronize()
        got, ref = out.cpu().numpy().reshape(-1, 128), want.cpu().numpy().reshape(-1, 128)
        assert np.isfinite(got).all()
        assert_close_output(got, ref.astype(np.float64), f"static scratch, case seed {seed}")


def test_static_scratch_refuses_sizes_beyond_its_array():
    # 512 sequences x 128 query heads: the workspace the library asks for is
    # well over the 16 MiB array (at least the B * Hq output rows of partials)
    B, H, Hq, cap = 512, 8, 128, 128
    cache = native.KVQCache(B, H, cap, 2, 2, 1, 0)
    need = cache.workspace_bytes(Hq, cap)
    assert need >= B * Hq * 128 * 4 > (16 << 20) + (8 << 20)
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.full((B,), cap, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, Hq, 128), dtype=torch.float32, device="cuda")
    assert call_static(cache, q, lens, cap, None, out) == native.KVQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert not out.any().item()  # nothing was enqueued
