"""Full-size workloads on the GPU, in the launch configuration bench.py times
(same calls, same max_len, hence the same split plan), checked on sampled
(sequence, kv head) slices that the oracle recomputes on its own: the packed
bytes of the slice bit-exact, the selection masks bit-exact for every
sequence, and the decode outputs of the slice's query heads within
2e-3 * max|o_ref|.
"""
import math

import numpy as np
import pytest
import torch

from kvq_testlib import ATOL_REL, TIE_BUDGET, host_f32, mask_u32
from kvq_testlib import _token_of as token_of
from oracle import oracle as orc
from quantized_attention_kvq_b200 import native, synth, workloads

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def up(a, fmt):
    if fmt == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def slice_bytes(gc: native.KVQCache, b: int, h: int):
    """Packed bytes of (b, h) from the device cache, in the oracle's 1x1 layout."""
    B, H, cap = gc.B, gc.H, gc.capacity
    bh = b * H + h
    kw = 2 if gc.desc.k_bits == 4 else 1
    out = {
        "k_codes": gc.k_codes[bh * 32 * cap * kw:(bh + 1) * 32 * cap * kw],
        "k_scales": gc.k_scales[bh * 4 * cap * 4:(bh + 1) * 4 * cap * 4],
        "v_codes": gc.v_codes[bh * cap * 16 * gc.desc.v_bits:(bh + 1) * cap * 16 * gc.desc.v_bits],
        "v_scales": gc.v_scales[bh * cap * 16:(bh + 1) * cap * 16],
    }
    if gc.k_ch0 is not None:
        out["k_ch0"] = gc.k_ch0[bh * cap * 2:(bh + 1) * cap * 2]
    return {k: v.cpu().numpy() for k, v in out.items()}


def oracle_slice(wl, s, b, h, pair=None):
    tq, tk = (None, None) if pair is None else (pair[0][h:h + 1], pair[1][h:h + 1])
    c = orc.Cache(1, 1, 128, wl.capacity, wl.k_bits, wl.v_bits, wl.rotate_k, wl.keep_ch0, wl.rotate_v, wl.v_clip,
                  wl.sink, wl.recent, tq, tk)
    k = s.k_slice(b, h)[None, None]
    v = s.v_slice(b, h)[None, None]
    st = c.append(host_f32(k, wl.fmt), host_f32(v, wl.fmt), wl.offset, want_exempt=True)
    return c, st


def check_slice_bytes(got: dict, c: orc.Cache, st: dict, wl):
    ref = {"k_codes": c.k_codes, "k_scales": c.k_scales.view(np.uint8), "v_codes": c.v_codes,
           "v_scales": c.v_scales.view(np.uint8)}
    if c.k_ch0 is not None:
        ref["k_ch0"] = c.k_ch0.view(np.uint8)
    bad_rows = 0
    for name, r in ref.items():
        diff = np.nonzero(got[name] != r)[0]
        if diff.size:
            # every differing byte must sit in a token the oracle flagged as a near-tie
            # (a value-code byte holds several tokens: any of them may carry the tie)
            _, tok = token_of(name, diff, wl.capacity, wl.k_bits, wl.v_bits)
            span = 8 // wl.v_bits if name == "v_codes" else 1
            flags = st["k_row_exempt" if name.startswith("k_") else "v_row_exempt"][0, 0]
            ok = np.zeros(diff.size, bool)
            for i in range(span):
                t = tok + i - wl.offset
                inside = (t >= 0) & (t < wl.T)
                ok |= inside & flags[np.clip(t, 0, wl.T - 1)].astype(bool)
            assert ok.all(), f"{name}: {int((~ok).sum())} differing bytes outside near-tie tokens"
            bad_rows += np.unique(tok).size
    assert bad_rows <= TIE_BUDGET * (st["k_elems"] + st["v_elems"]) + 1


def build_cache(wl, s):
    gc = native.KVQCache(wl.B, wl.Hkv, wl.capacity, wl.k_bits, wl.v_bits, wl.rotate_k, wl.keep_ch0,
                         rotate_v=wl.rotate_v, v_clip=wl.v_clip, sink=wl.sink, recent=wl.recent)
    for b in range(wl.B):
        kd = up(np.stack([s.k_slice(b, h) for h in range(wl.Hkv)]), wl.fmt)
        vd = up(np.stack([s.v_slice(b, h) for h in range(wl.Hkv)]), wl.fmt)
        gc.append_sequence(b, kd, vd, wl.offset)
        torch.cuda.synchronize()
        del kd, vd
    return gc


def sampled_pairs(wl, n=2, seed=0):
    """First and last (sequence, kv head) plus up to n seeded others, all distinct."""
    rng = np.random.default_rng(seed + wl.id)
    pairs = {(0, 0), (wl.B - 1, wl.Hkv - 1)}
    want = min(n + 2, wl.B * wl.Hkv)
    for _ in range(100 * want):
        if len(pairs) >= want:
            break
        pairs.add((int(rng.integers(wl.B)), int(rng.integers(wl.Hkv))))
    return sorted(pairs)


@pytest.mark.parametrize("wid", [0, 1, 2, 4, 5, 7])
def test_decode_workload(wid):
    wl = workloads.by_id(wid)
    s = synth.Synth(workloads.BASE_SEED + wl.id, wl.B, wl.Hq, wl.Hkv, wl.d, wl.T, wl.fmt, wl.len_range)
    gc = build_cache(wl, s)
    q = s.q()
    qd = up(q, wl.fmt)
    lens = s.lens.astype(np.int32)
    lens_d = torch.from_numpy(lens).cuda()
    max_len = wl.T if wl.len_range is None else wl.capacity
    scale = 1.0 / math.sqrt(128)
    mask_d = None
    ref_mask = np.full((wl.B, wl.Hkv), 0xFFFFFFFF, np.uint32)
    if wl.keep_groups < 32:
        mask_d = gc.select(qd, wl.keep_groups)
        ref_mask, _ = orc.select(host_f32(q, wl.fmt), wl.Hkv, wl.rotate_k, wl.keep_groups)
        np.testing.assert_array_equal(mask_u32(mask_d), ref_mask)
        assert all(bin(int(m)).count("1") == wl.keep_groups for m in ref_mask.ravel())
    # the two halves bench.py times, then the one-call form: identical results
    ws = torch.empty(gc.workspace_bytes(wl.Hq, max_len), dtype=torch.uint8, device="cuda")
    out = torch.empty((wl.B, wl.Hq, 128), dtype=torch.float32, device="cuda")
    gc.decode_partials(qd, lens_d, max_len, mask_d, scale, ws)
    gc.decode_combine(wl.Hq, lens_d, max_len, out, ws)
    out2 = gc.decode(qd, lens_d, max_len, mask_d, scale)
    torch.cuda.synchronize()
    o_gpu = out.cpu().numpy()
    assert np.isfinite(o_gpu).all()
    G = wl.G
    qf = host_f32(q, wl.fmt)
    for b, h in sampled_pairs(wl):
        c, st = oracle_slice(wl, s, b, h)
        check_slice_bytes(slice_bytes(gc, b, h), c, st, wl)
        qs = qf[b:b + 1, h * G:(h + 1) * G]
        o_ref = c.attention(qs, lens[b:b + 1], ref_mask[b:b + 1, h:h + 1], scale)
        got = o_gpu[b, h * G:(h + 1) * G].astype(np.float64)
        err = np.abs(got - o_ref).max()
        assert err <= ATOL_REL * np.abs(o_ref).max(), (wl.name, b, h, err, np.abs(o_ref).max())
    diff = (out - out2).abs().reshape(wl.B, wl.Hq, 128).amax(dim=2)
    rows = torch.nonzero(diff).tolist()
    assert not rows, f"identical decode calls differ in {len(rows)} rows, e.g. {rows[:8]}, max {diff.max().item():.3e}"


@pytest.mark.parametrize("wid", [3, 6, 9])
def test_append_workload(wid):
    wl = workloads.by_id(wid)
    s = synth.Synth(workloads.BASE_SEED + wl.id, wl.B, wl.Hq, wl.Hkv, wl.d, wl.T, wl.fmt, wl.len_range)
    pair = synth.dual_pair(workloads.BASE_SEED + wl.id, wl.Hkv) if wl.rotate_k == 2 else None
    kw = {} if pair is None else dict(t_query=torch.from_numpy(pair[0]).cuda(), t_key=torch.from_numpy(pair[1]).cuda())
    gc = native.KVQCache(wl.B, wl.Hkv, wl.capacity, wl.k_bits, wl.v_bits, wl.rotate_k, wl.keep_ch0,
                         rotate_v=wl.rotate_v, v_clip=wl.v_clip, sink=wl.sink, recent=wl.recent, **kw)
    # one launch over the whole batch, as timed for the append workload
    kd = up(s.k_full(), wl.fmt)
    vd = up(s.v_full(), wl.fmt)
    gc.append(kd, vd, wl.offset)
    torch.cuda.synchronize()
    del kd, vd
    for b, h in sampled_pairs(wl, n=3):
        c, st = oracle_slice(wl, s, b, h, pair)
        check_slice_bytes(slice_bytes(gc, b, h), c, st, wl)
    # nothing before the offset was written
    cap, off = wl.capacity, wl.offset
    kw = 2 if wl.k_bits == 4 else 1
    kc = gc.k_codes.view(wl.B * wl.Hkv, cap // 128, 32 * 128 * kw)  # key blocks of 128 tokens
    assert not kc[:, :off // 128].any().item()
    assert kc[:, off // 128:].any().item()
    vc = gc.v_codes.view(wl.B * wl.Hkv, cap, -1)
    assert not vc[:, :off].any().item()


@pytest.mark.parametrize("wid", [8, 10])
def test_decode_bucket_workload(wid):
    """The whole Dual-QK recipe at 128K (Dual-QK summary Sec. 3.1, 3.3, 3.4): a
    dual transform pair, bucket-relative RoPE at w = 2048, values rotated and
    clipped, and for workload 10 the bf16 sink and recent windows.  The cache is
    built as bench.py builds it (one append per bucket); the decode runs as
    timed (selection inside the split half) and as selection then decode.
    Sampled (sequence, kv head) slices: the per-bucket masks bit-exact and the
    outputs within the bar, against an oracle cache of that slice alone (the
    bytes of bucket-major caches are compared bit-exactly at small sizes in
    test_gpu_bucket_rope.py)."""
    wl = workloads.by_id(wid)
    seed = workloads.BASE_SEED + wl.id
    s = synth.Synth(seed, wl.B, wl.Hq, wl.Hkv, wl.d, wl.T, wl.fmt, wl.len_range)
    tq, tk = synth.dual_pair(seed, wl.Hkv)
    fr = synth.rope_inv_freq(wl.rope_base)
    gc = native.KVQCache(wl.B, wl.Hkv, wl.capacity, wl.k_bits, wl.v_bits, wl.rotate_k, wl.keep_ch0,
                         rotate_v=wl.rotate_v, v_clip=wl.v_clip, sink=wl.sink, recent=wl.recent,
                         t_query=torch.from_numpy(tq).cuda(), t_key=torch.from_numpy(tk).cuda(),
                         bucket_tokens=wl.bucket, rope_inv_freq=torch.from_numpy(fr).cuda())
    for b in range(wl.B):
        kd = up(np.stack([s.k_slice(b, h) for h in range(wl.Hkv)]), wl.fmt)
        vd = up(np.stack([s.v_slice(b, h) for h in range(wl.Hkv)]), wl.fmt)
        for t0 in range(0, wl.T, wl.bucket):  # an append stays inside one bucket
            gc.append_sequence(b, kd[:, t0:t0 + wl.bucket].contiguous(), vd[:, t0:t0 + wl.bucket].contiguous(),
                               wl.offset + t0)
        torch.cuda.synchronize()
        del kd, vd
    q = s.q()
    qd = up(q, wl.fmt)
    lens = s.lens.astype(np.int32)
    lens_d = torch.from_numpy(lens).cuda()
    max_len = wl.T
    scale = 1.0 / math.sqrt(128)
    keep = wl.keep_groups
    ws = torch.empty(gc.workspace_bytes(wl.Hq, max_len), dtype=torch.uint8, device="cuda")
    out = torch.empty((wl.B, wl.Hq, 128), dtype=torch.float32, device="cuda")
    gc.decode_partials_select(qd, lens_d, max_len, keep, scale, ws)
    gc.decode_combine(wl.Hq, lens_d, max_len, out, ws)
    mask_d = gc.select_at(qd, lens_d, keep)
    out2 = gc.decode(qd, lens_d, max_len, mask_d, scale)
    torch.cuda.synchronize()
    assert torch.equal(out, out2), "selection inside the decode and selection then decode differ"
    o_gpu = out.cpu().numpy()
    assert np.isfinite(o_gpu).all()
    nb = wl.capacity // wl.bucket
    masks = mask_u32(mask_d).reshape(wl.B, nb, wl.Hkv)
    G = wl.G
    qf = host_f32(q, wl.fmt)
    for b, h in sampled_pairs(wl):
        c = orc.Cache(1, 1, 128, wl.capacity, wl.k_bits, wl.v_bits, wl.rotate_k, wl.keep_ch0, wl.rotate_v,
                      wl.v_clip, wl.sink, wl.recent, tq[h:h + 1], tk[h:h + 1], bucket_w=wl.bucket, inv_freq=fr)
        c.append(host_f32(s.k_slice(b, h)[None, None], wl.fmt), host_f32(s.v_slice(b, h)[None, None], wl.fmt),
                 wl.offset)
        qs = qf[b:b + 1, h * G:(h + 1) * G]
        ref_mask, _ = c.select_buckets(qs, lens[b:b + 1], keep)
        np.testing.assert_array_equal(masks[b, :, h], ref_mask[0, :, 0], err_msg=f"masks of ({b}, {h})")
        o_ref = c.attention(qs, lens[b:b + 1], ref_mask, scale)
        got = o_gpu[b, h * G:(h + 1) * G].astype(np.float64)
        err = np.abs(got - o_ref).max()
        assert err <= ATOL_REL * np.abs(o_ref).max(), (wl.name, b, h, err, np.abs(o_ref).max())
