"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle on
small seeded inputs that span several tiles and ragged tails.

Codes, scales, zeros and channel-0 values must be bit-exact (near-ties
counted, within 1e-5 of the elements); masks bit-exact; attention outputs
within max|o_gpu - o_ref| <= 2e-3 * max|o_ref|.
"""
import numpy as np
import pytest
import torch

from kvq_testlib import (assert_close_output, compare_cache_bytes, gpu_arrays, host_f32, mask_u32, oracle_arrays,
                         softmax_scale, to_device)
from oracle import oracle as orc
from quantized_attention_kvq_b200 import native, synth

pytestmark = pytest.mark.gpu


def draw(seed, B, Hq, H, T, fmt):
    s = synth.Synth(seed, B, Hq, H, 128, T, "bf16" if fmt == "bf16" else "f32")
    q, k, v = s.q(), s.k_full(), s.v_full()
    if fmt == "f16":  # fp16 inputs: round the fp32 draws to fp16
        q, k, v = (x.astype(np.float16) for x in (q, k, v))
    return q, k, v


def build_both(B, H, cap, kb, vb, rot, ch0, k, v, fmt, offset=0, chunks=None, rotate_v=0, v_clip=1.0):
    """Append the same inputs through the C ABI and through the oracle.
    Returns (gpu cache, oracle cache, near-tie row flags, comparison geometry)."""
    gc = native.KVQCache(B, H, cap, kb, vb, rot, ch0, rotate_v=rotate_v, v_clip=v_clip)
    oc = orc.Cache(B, H, 128, cap, kb, vb, rot, ch0, rotate_v=rotate_v, v_clip=v_clip)
    T = k.shape[2]
    chunks = chunks or [T]
    flags = {"k": np.zeros((B, H, cap), np.uint8), "v": np.zeros((B, H, cap), np.uint8)}
    elems = 0
    t = 0
    for n in chunks:
        gc.append(to_device(k[:, :, t:t + n], fmt), to_device(v[:, :, t:t + n], fmt), offset + t)
        st = oc.append(host_f32(k[:, :, t:t + n], fmt), host_f32(v[:, :, t:t + n], fmt), offset + t,
                       want_exempt=True)
        flags["k"][:, :, offset + t:offset + t + n] = st["k_row_exempt"]
        flags["v"][:, :, offset + t:offset + t + n] = st["v_row_exempt"]
        elems += st["k_elems"] + st["v_elems"]
        t += n
    torch.cuda.synchronize()
    return gc, oc, flags, (cap, kb, vb, elems)


@pytest.mark.parametrize("kb,vb,rot,ch0,fmt,T,offset,cap", [
    (4, 4, 1, 0, "f32", 200, 0, 256),
    (4, 4, 1, 0, "bf16", 64, 64, 256),
    (2, 2, 1, 1, "bf16", 129, 7, 256),
    (4, 2, 1, 1, "bf16", 65, 0, 128),
    (2, 4, 0, 0, "f16", 33, 31, 128),
    (4, 2, 0, 1, "f32", 1, 127, 128),
    (2, 2, 0, 0, "bf16", 300, 100, 512),
])
def test_append_bitexact(kb, vb, rot, ch0, fmt, T, offset, cap):
    B, H = 2, 3
    _, k, v = draw(100 + T, B, H, H, T, fmt)
    gc, oc, flags, geom = build_both(B, H, cap, kb, vb, rot, ch0, k, v, fmt, offset)
    compare_cache_bytes(gpu_arrays(gc), oracle_arrays(oc), flags, geom)


@pytest.mark.parametrize("kb,vb,ch0,fmt,T,offset,cap,clip", [
    (4, 2, 1, "bf16", 200, 0, 256, 0.92),
    (2, 2, 0, "f32", 129, 7, 256, 0.92),
    (4, 4, 0, "f16", 64, 64, 128, 1.0),
    (2, 4, 1, "bf16", 33, 95, 128, 0.5),
])
def test_append_bitexact_rotated_clipped_values(kb, vb, ch0, fmt, T, offset, cap, clip):
    # values rotated like the keys and quantized with a clipping ratio on each
    # group's range (Dual-QK App. B.2)
    B, H = 2, 3
    _, k, v = draw(700 + T, B, H, H, T, fmt)
    gc, oc, flags, geom = build_both(B, H, cap, kb, vb, 1, ch0, k, v, fmt, offset, rotate_v=1, v_clip=clip)
    compare_cache_bytes(gpu_arrays(gc), oracle_arrays(oc), flags, geom)


def test_append_in_chunks_equals_one_append():
    B, H, T = 2, 2, 300
    _, k, v = draw(7, B, H, H, T, "bf16")
    whole, _, _, _ = build_both(B, H, 384, 4, 2, 1, 1, k, v, "bf16")
    parts, oc, flags, geom = build_both(B, H, 384, 4, 2, 1, 1, k, v, "bf16", chunks=[1, 63, 64, 100, 72])
    gw, gp = gpu_arrays(whole), gpu_arrays(parts)
    for name in gw:
        np.testing.assert_array_equal(gw[name], gp[name])
    compare_cache_bytes(gp, oracle_arrays(oc), flags, geom)


def test_append_stress_distributions():
    # heavy-tailed, low-rank and focused keys (gist.science explainer: the
    # distributions its quality study uses) still quantize bit-exactly
    rng = np.random.default_rng(11)
    B, H, T = 1, 2, 256
    heavy = rng.standard_t(1.5, (B, H, T, 128))
    low = rng.standard_normal((B, H, T, 4)) @ rng.standard_normal((4, 128))
    focused = rng.standard_normal((B, H, T, 128)) * 0.01
    focused[..., 3] += 50.0
    for x in (heavy, low, focused):
        k = x.astype(np.float32)
        v = np.flip(k, axis=2).copy()
        gc, oc, flags, geom = build_both(B, H, T, 4, 2, 1, 1, k, v, "f32")
        compare_cache_bytes(gpu_arrays(gc), oracle_arrays(oc), flags, geom)


@pytest.mark.parametrize("G,keep,rot,fmt", [(1, 7, 1, "f32"), (4, 19, 1, "bf16"), (8, 24, 1, "bf16"),
                                            (16, 1, 1, "bf16"), (4, 32, 1, "bf16"), (2, 13, 0, "f16"),
                                            (64, 20, 1, "bf16")])
def test_select_bitexact(G, keep, rot, fmt):
    B, H = 3, 2
    q, _, _ = draw(200 + G, B, G * H, H, 1, fmt)
    gc = native.KVQCache(B, H, 128, 4, 4, rot, 0)
    m = mask_u32(gc.select(to_device(q, fmt), keep))
    ref, _ = orc.select(host_f32(q, fmt), H, rot, keep)
    np.testing.assert_array_equal(m, ref)


def test_select_ties_keep_lower_groups():
    q = np.ones((1, 4, 128), np.float32)
    gc = native.KVQCache(1, 1, 128, 4, 4, 0, 0)
    assert int(mask_u32(gc.select(to_device(q, "f32"), 6))[0, 0]) == 0b111111


DECODE_CASES = [
    # B, G, H, kb, vb, rot, ch0, keep, fmt, T (capacity), lens
    (1, 1, 1, 4, 4, 1, 0, 32, "f32", 1024, [1024]),
    (2, 4, 2, 4, 4, 1, 0, 32, "bf16", 1536, [1500, 1]),
    (3, 4, 2, 2, 2, 1, 1, 19, "bf16", 1024, [1000, 33, 7]),
    (2, 8, 2, 4, 2, 1, 1, 24, "bf16", 2048, [2048, 1025]),
    (4, 2, 1, 2, 4, 0, 0, 9, "f16", 512, [0, 1, 129, 512]),
    (2, 16, 1, 4, 4, 1, 1, 32, "bf16", 256, [255, 256]),
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: f"B{c[0]}G{c[1]}k{c[3]}v{c[4]}ch0{c[6]}keep{c[7]}")
def test_decode_matches_oracle(case):
    B, G, H, kb, vb, rot, ch0, keep, fmt, T, lens = case
    q, k, v = draw(300 + T + G, B, G * H, H, T, fmt)
    gc, oc, flags, geom = build_both(B, H, T, kb, vb, rot, ch0, k, v, fmt)
    compare_cache_bytes(gpu_arrays(gc), oracle_arrays(oc), flags, geom)
    qd = to_device(q, fmt)
    lens_np = np.array(lens, np.int32)
    lens_d = torch.from_numpy(lens_np).cuda()
    mask_d = gc.select(qd, keep) if keep < 32 else None
    ref_mask = None
    if keep < 32:
        ref_mask, _ = orc.select(host_f32(q, fmt), H, rot, keep)
        np.testing.assert_array_equal(mask_u32(mask_d), ref_mask)
    out = gc.decode(qd, lens_d, T, mask_d, softmax_scale())
    again = gc.decode(qd, lens_d, T, mask_d, softmax_scale())
    torch.cuda.synchronize()
    assert torch.equal(out, again), "two identical decode calls differ"
    o_ref = oc.attention(host_f32(q, fmt), lens_np, ref_mask, softmax_scale())
    o_gpu = out.cpu().numpy().reshape(-1, 128)
    for b in range(B):
        rows = slice(b * G * H, (b + 1) * G * H)
        if lens[b] == 0:
            assert not o_gpu[rows].any()
        else:
            assert_close_output(o_gpu[rows], o_ref[rows], f"sequence {b}")


@pytest.mark.parametrize("B,G,H,kb,vb,ch0,keep,clip,lens", [
    (2, 4, 2, 2, 2, 1, 19, 0.92, [1000, 129]),
    (2, 8, 1, 4, 2, 1, 24, 0.92, [2048, 1]),
    (1, 1, 2, 4, 4, 0, 32, 1.0, [777]),
])
def test_decode_with_rotated_values_matches_oracle(B, G, H, kb, vb, ch0, keep, clip, lens):
    # the decode works in the rotated value basis; the combine rotates back
    T = 2048
    q, k, v = draw(900 + G + kb, B, G * H, H, T, "bf16")
    gc, oc, flags, geom = build_both(B, H, T, kb, vb, 1, ch0, k, v, "bf16", rotate_v=1, v_clip=clip)
    compare_cache_bytes(gpu_arrays(gc), oracle_arrays(oc), flags, geom)
    qd = to_device(q, "bf16")
    lens_np = np.array(lens, np.int32)
    lens_d = torch.from_numpy(lens_np).cuda()
    mask_d = gc.select(qd, keep) if keep < 32 else None
    ref_mask = orc.select(host_f32(q, "bf16"), H, 1, keep)[0] if keep < 32 else None
    out = gc.decode(qd, lens_d, T, mask_d, softmax_scale())
    torch.cuda.synchronize()
    o_ref = oc.attention(host_f32(q, "bf16"), lens_np, ref_mask, softmax_scale())
    o_gpu = out.cpu().numpy().reshape(-1, 128)
    for b in range(B):
        rows = slice(b * G * H, (b + 1) * G * H)
        assert_close_output(o_gpu[rows], o_ref[rows], f"sequence {b}")


@pytest.mark.parametrize("G,H,kb,vb,ch0,keep,rotv,sink,recent,L", [
    (4, 2, 2, 2, 1, 19, 1, 64, 256, 1000),   # the Dual-QK recipe: INT2, pruned keys, bf16 windows
    (1, 2, 4, 4, 0, 32, 0, 4, 8, 10),        # the whole sequence inside the windows
    (8, 1, 4, 2, 1, 24, 0, 16, 0, 300),      # sink only
    (2, 2, 4, 4, 0, 9, 0, 0, 100, 129),      # recent only
    (16, 1, 4, 4, 1, 32, 1, 3, 5, 2),        # shorter than the sink
])
def test_decode_with_bf16_windows_matches_oracle(G, H, kb, vb, ch0, keep, rotv, sink, recent, L):
    # window tokens come from bf16 copies of the rotated key and value, scored over
    # every channel; the others from the codes (Dual-QK Sec. 3.3); decode length =
    # tokens appended, as the ring holds the last `recent` of them
    T = 1024
    clip = 0.92 if rotv else 1.0
    q, k, v = draw(1100 + G + L, 1, G * H, H, T, "bf16")
    k, v = k[:, :, :L], v[:, :, :L]
    gc = native.KVQCache(1, H, T, kb, vb, 1, ch0, rotate_v=rotv, v_clip=clip, sink=sink, recent=recent)
    oc = orc.Cache(1, H, 128, T, kb, vb, 1, ch0, rotv, clip, sink, recent)
    gc.append(to_device(k, "bf16"), to_device(v, "bf16"), 0)
    oc.append(host_f32(k, "bf16"), host_f32(v, "bf16"), 0)
    torch.cuda.synchronize()
    # the bf16 windows are bit-exact (bf16 of the same fp32 rows)
    assert np.array_equal(gc.k_window.cpu().numpy(), oc.k_win.view(np.uint8))
    assert np.array_equal(gc.v_window.cpu().numpy(), oc.v_win.view(np.uint8))
    qd = to_device(q, "bf16")
    lens_np = np.array([L], np.int32)
    lens_d = torch.from_numpy(lens_np).cuda()
    mask_d = gc.select(qd, keep) if keep < 32 else None
    ref_mask = orc.select(host_f32(q, "bf16"), H, 1, keep)[0] if keep < 32 else None
    out = gc.decode(qd, lens_d, T, mask_d, softmax_scale())
    torch.cuda.synchronize()
    o_ref = oc.attention(host_f32(q, "bf16"), lens_np, ref_mask, softmax_scale())
    assert_close_output(out.cpu().numpy().reshape(-1, 128), o_ref, "bf16 windows")


def test_full_mask_is_bit_identical_to_no_mask_and_split_plan_is_exact():
    B, G, H, T = 2, 4, 2, 1024
    q, k, v = draw(9, B, G * H, H, T, "bf16")
    gc, _, _, _ = build_both(B, H, T, 4, 4, 1, 1, k, v, "bf16")
    qd = to_device(q, "bf16")
    lens = torch.tensor([1024, 700], dtype=torch.int32, device="cuda")
    full = torch.full((B, H), -1, dtype=torch.int32, device="cuda")
    a = gc.decode(qd, lens, T, None).cpu()
    b = gc.decode(qd, lens, T, full).cpu()
    c = gc.decode(qd, lens, T, gc.select(qd, 32)).cpu()
    assert torch.equal(a, b) and torch.equal(a, c)
    # a larger max_len changes the split plan, not the result beyond rounding
    gc2 = native.KVQCache(B, H, 2048, 4, 4, 1, 1)
    gc2.append(to_device(k, "bf16"), to_device(v, "bf16"), 0)
    d = gc2.decode(qd, lens, 2048, None).cpu()
    assert (a - d).abs().max().item() <= 1e-5 * a.abs().max().item()


def test_decode_step_host_matches_device_calls():
    B, G, H, T = 2, 4, 2, 512
    q, k, v = draw(13, B, G * H, H, T, "bf16")
    gc, _, _, _ = build_both(B, H, T, 2, 2, 1, 1, k, v, "bf16")
    qd = to_device(q, "bf16")
    lens = torch.tensor([512, 300], dtype=torch.int32, device="cuda")
    want = gc.decode(qd, lens, T, gc.select(qd, 19)).cpu()
    q_host = qd.cpu().pin_memory()
    out_host = torch.empty((B, G * H, 128), dtype=torch.float32).pin_memory()
    ws = torch.empty(gc.step_workspace_bytes(torch.bfloat16, G * H, T), dtype=torch.uint8, device="cuda")
    gc.decode_step_host(q_host, lens, T, 19, softmax_scale(), out_host, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_host, want)
