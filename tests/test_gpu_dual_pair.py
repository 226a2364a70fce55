"""GPU parity of the caller-supplied dual transform pair (Dual-QK summary
Sec. 1, Sec. 3.1: T on queries, T^-T on keys, per kv head) against the CPU
oracle, through the C ABI.

The matrices are seeded inputs handed to both sides as the same fp32 arrays.
Codes, scales, zeros, channel 0 and the bf16 windows are bit-exact (both
sides sum the fp64 products in the same order, so the transformed rows are the
same fp32 values; near-ties counted as in the other append tests); masks are
bit-exact; outputs within max|o_gpu - o_ref| <= 2e-3 * max|o_ref|.
"""
import ctypes

import numpy as np
import pytest
import torch

from kvq_testlib import (assert_close_output, compare_cache_bytes, gpu_arrays, host_f32, mask_u32, oracle_arrays,
                         softmax_scale, to_device)
from oracle import oracle as orc
from quantized_attention_kvq_b200 import native, synth

pytestmark = pytest.mark.gpu
D = 128


def dense_pair(seed, H):
    """Per head an anisotropic, well-conditioned T and fp32 T^-T."""
    rng = np.random.default_rng(seed)
    tq = np.empty((H, D, D), np.float32)
    tk = np.empty((H, D, D), np.float32)
    for h in range(H):
        t = np.eye(D) + 0.35 * rng.standard_normal((D, D)) / np.sqrt(D)
        t[:, : D // 2] *= 2.0
        tq[h] = t
        tk[h] = np.linalg.inv(t).T
    return tq, tk


def draw(seed, B, Hq, H, T, fmt):
    s = synth.Synth(seed, B, Hq, H, D, T, "bf16" if fmt == "bf16" else "f32")
    q, k, v = s.q(), s.k_full(), s.v_full()
    if fmt == "f16":
        q, k, v = (x.astype(np.float16) for x in (q, k, v))
    return q, k, v


def build_pair(B, H, cap, kb, vb, ch0, k, v, fmt, tq, tk, offset=0, rotate_v=0, v_clip=1.0, sink=0, recent=0):
    gc = native.KVQCache(B, H, cap, kb, vb, 2, ch0, rotate_v=rotate_v, v_clip=v_clip, sink=sink, recent=recent,
                         t_query=torch.from_numpy(tq).cuda(), t_key=torch.from_numpy(tk).cuda())
    oc = orc.Cache(B, H, D, cap, kb, vb, 2, ch0, rotate_v, v_clip, sink, recent, tq, tk)
    gc.append(to_device(k, fmt), to_device(v, fmt), offset)
    st = oc.append(host_f32(k, fmt), host_f32(v, fmt), offset, want_exempt=True)
    torch.cuda.synchronize()
    T = k.shape[2]
    flags = {"k": np.zeros((B, H, cap), np.uint8), "v": np.zeros((B, H, cap), np.uint8)}
    flags["k"][:, :, offset:offset + T] = st["k_row_exempt"]
    flags["v"][:, :, offset:offset + T] = st["v_row_exempt"]
    return gc, oc, flags, (cap, kb, vb, st["k_elems"] + st["v_elems"])


@pytest.mark.parametrize("kb,vb,ch0,fmt,T,offset,cap", [
    (4, 4, 0, "f32", 200, 0, 256),
    (2, 2, 1, "bf16", 129, 7, 256),
    (4, 2, 1, "f16", 65, 63, 128),
    (2, 4, 0, "bf16", 1, 127, 128),
])
def test_append_bitexact_with_pair(kb, vb, ch0, fmt, T, offset, cap):
    B, H = 2, 3
    _, k, v = draw(1300 + T, B, H, H, T, fmt)
    tq, tk = dense_pair(T, H)
    gc, oc, flags, geom = build_pair(B, H, cap, kb, vb, ch0, k, v, fmt, tq, tk, offset)
    compare_cache_bytes(gpu_arrays(gc), oracle_arrays(oc), flags, geom)


@pytest.mark.parametrize("G,keep,fmt", [(1, 7, "f32"), (4, 19, "bf16"), (8, 24, "f16"), (16, 1, "bf16")])
def test_select_bitexact_with_pair(G, keep, fmt):
    B, H = 3, 2
    q, _, _ = draw(1400 + G, B, G * H, H, 1, fmt)
    tq, tk = dense_pair(G, H)
    gc = native.KVQCache(B, H, 128, 4, 4, 2, 0, t_query=torch.from_numpy(tq).cuda(),
                         t_key=torch.from_numpy(tk).cuda())
    m = mask_u32(gc.select(to_device(q, fmt), keep))
    ref, _ = orc.select(host_f32(q, fmt), H, 2, keep, tq)
    np.testing.assert_array_equal(m, ref)


@pytest.mark.parametrize("B,G,H,kb,vb,ch0,keep,fmt,rotv,sink,recent,lens", [
    (2, 4, 2, 2, 2, 1, 19, "bf16", 0, 0, 0, [1000, 129]),
    (1, 8, 1, 4, 4, 0, 32, "f32", 0, 0, 0, [2048]),
    (2, 2, 2, 4, 2, 1, 24, "f16", 1, 0, 0, [777, 1]),
    (1, 4, 2, 2, 2, 1, 19, "bf16", 1, 64, 256, [1000]),   # with the Dual-QK bf16 windows
])
def test_decode_with_pair_matches_oracle(B, G, H, kb, vb, ch0, keep, fmt, rotv, sink, recent, lens):
    T = 2048
    clip = 0.92 if rotv else 1.0
    q, k, v = draw(1500 + G + kb, B, G * H, H, T, fmt)
    if sink + recent:
        k, v = k[:, :, :lens[0]], v[:, :, :lens[0]]  # the ring holds the last tokens appended
    tq, tk = dense_pair(G + 10 * kb, H)
    gc, oc, flags, geom = build_pair(B, H, T, kb, vb, ch0, k, v, fmt, tq, tk, rotate_v=rotv, v_clip=clip,
                                     sink=sink, recent=recent)
    compare_cache_bytes(gpu_arrays(gc), oracle_arrays(oc), flags, geom)
    if sink + recent:
        assert np.array_equal(gc.k_window.cpu().numpy(), oc.k_win.view(np.uint8))
    qd = to_device(q, fmt)
    lens_np = np.array(lens, np.int32)
    lens_d = torch.from_numpy(lens_np).cuda()
    mask_d = gc.select(qd, keep) if keep < 32 else None
    ref_mask = None
    if keep < 32:
        ref_mask, _ = orc.select(host_f32(q, fmt), H, 2, keep, tq)
        np.testing.assert_array_equal(mask_u32(mask_d), ref_mask)
    out = gc.decode(qd, lens_d, T, mask_d, softmax_scale())
    again = gc.decode(qd, lens_d, T, mask_d, softmax_scale())
    torch.cuda.synchronize()
    assert torch.equal(out, again), "two identical decode calls differ"
    o_ref = oc.attention(host_f32(q, fmt), lens_np, ref_mask, softmax_scale())
    o_gpu = out.cpu().numpy().reshape(-1, D)
    for b in range(B):
        rows = slice(b * G * H, (b + 1) * G * H)
        if lens[b] == 0:
            assert not o_gpu[rows].any()
        else:
            assert_close_output(o_gpu[rows], o_ref[rows], f"sequence {b}")


def test_static_and_step_host_entry_points_with_pair():
    # the transformed queries live in the workspace of every decode entry point
    B, G, H, T = 2, 4, 2, 1024
    q, k, v = draw(1600, B, G * H, H, T, "bf16")
    tq, tk = dense_pair(77, H)
    gc, oc, _, _ = build_pair(B, H, T, 4, 2, 1, k, v, "bf16", tq, tk)
    qd = to_device(q, "bf16")
    lens_np = np.array([T, 300], np.int32)
    lens_d = torch.from_numpy(lens_np).cuda()
    mask_d = gc.select(qd, 19)
    ref = gc.decode(qd, lens_d, T, mask_d, softmax_scale())
    st = torch.empty_like(ref)
    rc = native.lib().kvq_decode_attention_static(ctypes.byref(gc.desc), qd.data_ptr(), native.KVQ_BF16, G * H,
                                                   lens_d.data_ptr(), T, mask_d.data_ptr(), softmax_scale(),
                                                   st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == native.KVQ_OK
    q_host = qd.cpu().pin_memory()
    out_host = torch.empty((B, G * H, D), dtype=torch.float32).pin_memory()
    ws = torch.empty(gc.step_workspace_bytes(torch.bfloat16, G * H, T), dtype=torch.uint8, device="cuda")
    gc.decode_step_host(q_host, lens_d, T, 19, softmax_scale(), out_host, ws)
    torch.cuda.synchronize()
    assert torch.equal(ref, st)
    assert torch.equal(out_host, ref.cpu())
    ref_mask, _ = orc.select(host_f32(q, "bf16"), H, 2, 19, tq)
    np.testing.assert_array_equal(mask_u32(mask_d), ref_mask)
    o_ref = oc.attention(host_f32(q, "bf16"), lens_np, ref_mask, softmax_scale())
    assert_close_output(ref.cpu().numpy().reshape(-1, D), o_ref, "pair")
