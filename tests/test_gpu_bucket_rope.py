"""GPU parity of bucket-relative RoPE (Dual-QK summary Sec. 3.4, App. C.4)
against the CPU oracle, through the C ABI.

The CUDA cache is bucket-major (bucket k of sequence b is sequence b * nb + k
of a cache of batch B * nb and capacity w); the oracle keeps the plain layout,
so its arrays are reordered bucket-major here before the bit-exact byte
comparison (near-ties counted as in the other append tests).  Per-bucket masks
are bit-exact; outputs within max|o_gpu - o_ref| <= 2e-3 * max|o_ref|.
"""
import numpy as np
import pytest
import torch

from kvq_testlib import (assert_close_output, compare_cache_bytes, gpu_arrays, host_f32, mask_u32, oracle_arrays,
                         softmax_scale, to_device)
from oracle import oracle as orc
from quantized_attention_kvq_b200 import native, synth

pytestmark = pytest.mark.gpu
D = 128


def inv_freq(base):
    return (base ** (-np.arange(0, D, 2) / D)).astype(np.float32)


def dense_pair(seed, H):
    rng = np.random.default_rng(seed)
    tq = np.empty((H, D, D), np.float32)
    tk = np.empty((H, D, D), np.float32)
    for h in range(H):
        t = np.eye(D) + 0.35 * rng.standard_normal((D, D)) / np.sqrt(D)
        tq[h], tk[h] = t, np.linalg.inv(t).T
    return tq, tk


def draw(seed, B, Hq, H, T, fmt):
    s = synth.Synth(seed, B, Hq, H, D, T, "bf16" if fmt == "bf16" else "f32")
    q, k, v = s.q(), s.k_full(), s.v_full()
    if fmt == "f16":
        q, k, v = (x.astype(np.float16) for x in (q, k, v))
    return q, k, v


def bucket_major(a: np.ndarray, B: int, H: int, nb: int) -> np.ndarray:
    """[B][H][nb chunks] -> [B][nb][H] chunks, chunks being a bucket's bytes."""
    return a.reshape(B, H, nb, -1).transpose(0, 2, 1, 3).reshape(-1)


def build(B, H, cap, w, kb, vb, rot, ch0, k, v, fmt, fr, tq=None, tk=None, rotv=0, clip=1.0, sink=0, recent=0):
    nb = cap // w
    gc = native.KVQCache(B, H, cap, kb, vb, rot, ch0, rotate_v=rotv, v_clip=clip, bucket_tokens=w,
                         rope_inv_freq=torch.from_numpy(fr).cuda(), sink=sink, recent=recent,
                         t_query=None if tq is None else torch.from_numpy(tq).cuda(),
                         t_key=None if tk is None else torch.from_numpy(tk).cuda())
    oc = orc.Cache(B, H, D, cap, kb, vb, rot, ch0, rotv, clip, sink, recent, tq, tk, bucket_w=w, inv_freq=fr)
    T = k.shape[2]
    for t0 in range(0, T, w):  # an append stays inside one bucket
        gc.append(to_device(k[:, :, t0:t0 + w], fmt), to_device(v[:, :, t0:t0 + w], fmt), t0)
    st = oc.append(host_f32(k, fmt), host_f32(v, fmt), 0, want_exempt=True)
    torch.cuda.synchronize()
    flags = {}
    for side in ("k", "v"):
        f = np.zeros((B, H, cap), np.uint8)
        f[:, :, :T] = st[f"{side}_row_exempt"]
        flags[side] = f.reshape(B, H, nb, w).transpose(0, 2, 1, 3).reshape(B * nb, H, w)
    ref = {name: bucket_major(a, B, H, nb) for name, a in oracle_arrays(oc).items()}
    compare_cache_bytes(gpu_arrays(gc), ref, flags, (w, kb, vb, st["k_elems"] + st["v_elems"]))
    return gc, oc


@pytest.mark.parametrize("kb,vb,rot,ch0,fmt,rotv", [
    (2, 2, 1, 1, "bf16", 0),
    (4, 4, 0, 0, "f32", 0),
    (4, 2, 2, 1, "f16", 1),
])
def test_bucket_rope_append_select_decode_match_oracle(kb, vb, rot, ch0, fmt, rotv):
    B, G, H, w, cap = 2, 4, 2, 256, 1024
    lens = [700, 1]
    T = max(lens)
    q, k, v = draw(1700 + kb + rot, B, G * H, H, T, fmt)
    fr = inv_freq(10000.0)
    tq, tk = dense_pair(5 + kb, H) if rot == 2 else (None, None)
    # one cache holding T tokens for every sequence; sequence 1 decodes 1 token
    gc, oc = build(B, H, cap, w, kb, vb, rot, ch0, k, v, fmt, fr, tq, tk, rotv, 0.92 if rotv else 1.0)
    qd = to_device(q, fmt)
    lens_np = np.array(lens, np.int32)
    lens_d = torch.from_numpy(lens_np).cuda()
    mask_d = gc.select_at(qd, lens_d, 19)
    ref_mask, _ = oc.select_buckets(host_f32(q, fmt), lens_np, 19)
    np.testing.assert_array_equal(mask_u32(mask_d).reshape(ref_mask.shape), ref_mask)
    assert len({int(m) for m in ref_mask[0, :3, 0]}) > 1  # buckets select differently here
    out = gc.decode(qd, lens_d, cap, mask_d, softmax_scale())
    again = gc.decode(qd, lens_d, cap, mask_d, softmax_scale())
    torch.cuda.synchronize()
    assert torch.equal(out, again)
    o_ref = oc.attention(host_f32(q, fmt), lens_np, ref_mask, softmax_scale())
    o_gpu = out.cpu().numpy().reshape(-1, D)
    for b in range(B):
        rows = slice(b * G * H, (b + 1) * G * H)
        assert_close_output(o_gpu[rows], o_ref[rows], f"sequence {b}")
    # no mask: every channel of every bucket
    full = gc.decode(qd, lens_d, cap, None, softmax_scale())
    torch.cuda.synchronize()
    assert_close_output(full.cpu().numpy().reshape(-1, D), oc.attention(host_f32(q, fmt), lens_np, None,
                                                                          softmax_scale()), "no mask")


def test_bucket_rope_lengths_at_bucket_edges():
    # lengths ending exactly on, just past and before bucket boundaries, and 0
    B, G, H, w, cap = 4, 2, 1, 128, 512
    lens = [128, 129, 511, 0]
    T = 512
    q, k, v = draw(1800, B, G * H, H, T, "bf16")
    fr = inv_freq(500.0)
    gc, oc = build(B, H, cap, w, 4, 2, 1, 0, k, v, "bf16", fr)
    qd = to_device(q, "bf16")
    lens_np = np.array(lens, np.int32)
    lens_d = torch.from_numpy(lens_np).cuda()
    mask_d = gc.select_at(qd, lens_d, 24)
    ref_mask, _ = oc.select_buckets(host_f32(q, "bf16"), lens_np, 24)
    np.testing.assert_array_equal(mask_u32(mask_d).reshape(ref_mask.shape)[:3], ref_mask[:3])
    out = gc.decode(qd, lens_d, cap, mask_d, softmax_scale())
    torch.cuda.synchronize()
    o_gpu = out.cpu().numpy().reshape(-1, D)
    o_ref = oc.attention(host_f32(q, "bf16"), lens_np, ref_mask, softmax_scale())
    for b in range(B):
        rows = slice(b * G * H, (b + 1) * G * H)
        if lens[b] == 0:
            assert not o_gpu[rows].any()
        else:
            assert_close_output(o_gpu[rows], o_ref[rows], f"sequence {b}")


@pytest.mark.parametrize("T,sink,recent,rot,keep", [(700, 64, 200, 1, 19), (1000, 16, 256, 2, 24), (200, 64, 256, 1, 32)])
def test_bucket_rope_with_bf16_windows_matches_oracle(T, sink, recent, rot, keep):
    # bf16 sink and recent windows together with bucket-relative RoPE: a window
    # token is scored over every channel with the query of the bucket it sits
    # in; the recent window here spans two buckets (Dual-QK Sec. 3.3 and 3.4)
    B, G, H, w, cap = 2, 4, 2, 256, 1024
    q, k, v = draw(1900 + T + rot, B, G * H, H, T, "bf16")
    fr = inv_freq(10000.0)
    tq, tk = dense_pair(7, H) if rot == 2 else (None, None)
    gc, oc = build(B, H, cap, w, 4, 2, rot, 1, k, v, "bf16", fr, tq, tk, sink=sink, recent=recent)
    # the windows are bit-exact (bf16 of the same embedded, transformed rows)
    assert np.array_equal(gc.k_window.cpu().numpy(), oc.k_win.view(np.uint8))
    assert np.array_equal(gc.v_window.cpu().numpy(), oc.v_win.view(np.uint8))
    qd = to_device(q, "bf16")
    lens_np = np.array([T, T], np.int32)  # the decode length is the tokens appended (the ring holds the last ones)
    lens_d = torch.from_numpy(lens_np).cuda()
    if keep < 32:
        mask_d = gc.select_at(qd, lens_d, keep)
        ref_mask, _ = oc.select_buckets(host_f32(q, "bf16"), lens_np, keep)
        np.testing.assert_array_equal(mask_u32(mask_d).reshape(ref_mask.shape), ref_mask)
    else:
        mask_d, ref_mask = None, None
    out = gc.decode(qd, lens_d, cap, mask_d, softmax_scale())
    sel = gc.decode_select(qd, lens_d, cap, keep, softmax_scale()) if keep < 32 else out
    torch.cuda.synchronize()
    assert torch.equal(out, sel)
    o_ref = oc.attention(host_f32(q, "bf16"), lens_np, ref_mask, softmax_scale())
    o_gpu = out.cpu().numpy().reshape(-1, D)
    for b in range(B):
        rows = slice(b * G * H, (b + 1) * G * H)
        assert_close_output(o_gpu[rows], o_ref[rows], f"sequence {b}")
