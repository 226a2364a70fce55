"""GPU decode parity on numerically hard inputs, against the CPU oracle.

* Sharp queries: almost all of a query's energy in a few channels, a dynamic
  range of 10^4 between its largest and smallest channels -- the queries the
  Dual-QK transform is built to produce (Dual-QK summary, title and Sec. 3.1:
  the query basis concentrates query energy), here without a rotation
  (rotate_k = 0) and through a caller-supplied pair (rotate_k = 2) whose
  transformed query is the sharp vector.
* Value scales at the ends of fp16: values times 1e-4 (group scales near the
  fp16 subnormal range) and times 10^3 (group scales of hundreds), INT2 and
  INT4 (Dual-QK App. B.2: per-token asymmetric values with FP16 scale/zero).
* The gist.science explainer's key distributions (heavy-tailed, low-rank,
  focused) through the decode, not only the append.

Bar: max|o_gpu - o_ref| <= 2e-3 * max|o_ref| per sequence, the caches
bit-exact (near-ties counted) as in the other parity tests.
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


def sharp_queries(rng, B, Hq, n_hot=3, floor=1e-3):
    """Queries with n_hot channels of magnitude 2..20 and the rest ~ floor * N(0,1)."""
    q = (rng.standard_normal((B, Hq, D)) * floor).astype(np.float64)
    for b in range(B):
        for h in range(Hq):
            hot = rng.choice(D, n_hot, replace=False)
            q[b, h, hot] = rng.choice([-1.0, 1.0], n_hot) * rng.uniform(2.0, 20.0, n_hot)
    return q.astype(np.float32)


def keys_values(seed, B, H, T):
    s = synth.Synth(seed, B, H, H, D, T, "f32")
    return s.k_full(), s.v_full()


def run_decode(gc, oc, q, lens, keep, H, rot, tq=None):
    qd = to_device(q, "f32")
    lens_np = np.array(lens, np.int32)
    lens_d = torch.from_numpy(lens_np).cuda()
    mask_d = gc.select(qd, keep) if keep < 32 else None
    ref_mask = None
    if keep < 32:
        ref_mask, _ = orc.select(q, H, rot, keep, tq)
        np.testing.assert_array_equal(mask_u32(mask_d), ref_mask)
    out = gc.decode(qd, lens_d, max(lens), mask_d, softmax_scale())
    torch.cuda.synchronize()
    o_ref = oc.attention(q, lens_np, ref_mask, softmax_scale())
    return out.cpu().numpy().reshape(o_ref.shape), o_ref


def check_per_sequence(o_gpu, o_ref, B, rows_per_seq, what):
    o_gpu = o_gpu.reshape(B, rows_per_seq, D)
    o_ref = o_ref.reshape(B, rows_per_seq, D)
    for b in range(B):
        assert np.isfinite(o_gpu[b]).all(), f"{what}: non-finite output in sequence {b}"
        assert_close_output(o_gpu[b], o_ref[b], f"{what}, sequence {b}")


def build(B, H, T, kb, vb, rot, ch0, k, v, tq=None, tk=None, rotate_v=0, v_clip=1.0):
    kw = {}
    if rot == 2:
        kw = dict(t_query=torch.from_numpy(tq).cuda(), t_key=torch.from_numpy(tk).cuda())
    gc = native.KVQCache(B, H, T, kb, vb, rot, ch0, rotate_v=rotate_v, v_clip=v_clip, **kw)
    oc = orc.Cache(B, H, D, T, kb, vb, rot, ch0, rotate_v, v_clip, 0, 0, tq, tk)
    gc.append(to_device(k, "f32"), to_device(v, "f32"), 0)
    st = oc.append(k, v, 0, want_exempt=True)
    torch.cuda.synchronize()
    flags = {"k": st["k_row_exempt"], "v": st["v_row_exempt"]}
    compare_cache_bytes(gpu_arrays(gc), oracle_arrays(oc), flags, (T, kb, vb, st["k_elems"] + st["v_elems"]))
    return gc, oc


@pytest.mark.parametrize("G,H,kb,vb,ch0,keep,lens", [
    (4, 2, 4, 4, 0, 32, [1536, 200]),
    (4, 2, 2, 2, 1, 19, [1536, 1]),
    (8, 1, 4, 2, 1, 24, [1300]),
    (1, 2, 4, 4, 0, 7, [1536]),
])
def test_sharp_queries_without_rotation(G, H, kb, vb, ch0, keep, lens):
    rng = np.random.default_rng(40 + G + kb)
    B, T = len(lens), 1536
    k, v = keys_values(4000 + G, B, H, T)
    q = sharp_queries(rng, B, G * H)
    gc, oc = build(B, H, T, kb, vb, 0, ch0, k, v)
    o_gpu, o_ref = run_decode(gc, oc, q, lens, keep, H, 0)
    check_per_sequence(o_gpu, o_ref, B, G * H, "sharp queries, rotate_k = 0")


@pytest.mark.parametrize("G,H,kb,vb,ch0,keep", [(4, 2, 2, 2, 1, 19), (8, 1, 4, 2, 1, 24), (2, 2, 4, 4, 0, 32)])
def test_sharp_transformed_queries_through_dual_pair(G, H, kb, vb, ch0, keep):
    # q = T^-1 s with s sharp, so the transformed query T q is sharp (up to fp32 rounding)
    rng = np.random.default_rng(60 + G)
    B, T = 2, 1280
    tq, tk = synth.dual_pair(77 + G, H)
    s = sharp_queries(rng, B, G * H).astype(np.float64)
    q = np.empty_like(s)
    for b in range(B):
        for hq in range(G * H):
            q[b, hq] = tk[hq // G].astype(np.float64).T @ s[b, hq]  # T^-1 = (T^-T)^T
    q = q.astype(np.float32)
    k, v = keys_values(4100 + G, B, H, T)
    gc, oc = build(B, H, T, kb, vb, 2, ch0, k, v, tq, tk)
    o_gpu, o_ref = run_decode(gc, oc, q, [T, 777], keep, H, 2, tq)
    check_per_sequence(o_gpu, o_ref, B, G * H, "sharp transformed queries, dual pair")


@pytest.mark.parametrize("vscale", [1e-4, 1e3])
@pytest.mark.parametrize("G,kb,vb,keep,rotv", [(4, 4, 4, 32, 0), (4, 2, 2, 19, 0), (8, 4, 2, 24, 1)])
def test_extreme_value_scales(vscale, G, kb, vb, keep, rotv):
    # values times 1e-4 put the group scales near fp16's subnormal range; times
    # 1e3 makes scales of hundreds, so p * scale leaves fp16's normal range
    # unless the decode rescales it
    B, H, T = 2, 2, 1536
    k, v = keys_values(4200 + G + kb, B, H, T)
    v = (v.astype(np.float64) * vscale).astype(np.float32)
    q = synth.Synth(4300 + G, B, G * H, H, D, 1, "f32").q()
    gc, oc = build(B, H, T, kb, vb, 1, 1, k, v, rotate_v=rotv, v_clip=0.92 if rotv else 1.0)
    o_gpu, o_ref = run_decode(gc, oc, q, [T, 531], keep, H, 1)
    check_per_sequence(o_gpu, o_ref, B, G * H, f"values x {vscale:g}")


def test_peaked_attention_with_large_value_scales():
    # one token per sequence dominates the softmax (its key is a multiple of the
    # query), values of scale ~10^3: p reaches the top of its range on large scales
    B, G, H, T = 2, 4, 1, 1024
    rng = np.random.default_rng(91)
    k, v = keys_values(4400, B, H, T)
    v = (v.astype(np.float64) * 1e3).astype(np.float32)
    q = synth.Synth(4401, B, G * H, H, D, 1, "f32").q()
    for b in range(B):
        j = int(rng.integers(0, T))
        k[b, 0, j] = 4.0 * q[b, 0]
    gc, oc = build(B, H, T, 4, 4, 0, 0, k, v)
    o_gpu, o_ref = run_decode(gc, oc, q, [T, T], 32, H, 0)
    check_per_sequence(o_gpu, o_ref, B, G * H, "peaked attention, values x 1e3")


def stress_keys(kind, rng, B, H, T):
    if kind == "heavy":
        x = rng.standard_t(1.5, (B, H, T, D))
    elif kind == "low_rank":
        x = rng.standard_normal((B, H, T, 4)) @ rng.standard_normal((4, D))
    else:  # focused: one dominant channel over a small floor
        x = rng.standard_normal((B, H, T, D)) * 0.01
        x[..., 3] += 50.0
    return x.astype(np.float32)


@pytest.mark.parametrize("kind", ["heavy", "low_rank", "focused"])
@pytest.mark.parametrize("kb,vb,ch0,keep", [(4, 2, 1, 24), (2, 2, 1, 19)])
def test_stress_distributions_through_decode(kind, kb, vb, ch0, keep):
    rng = np.random.default_rng({"heavy": 5, "low_rank": 6, "focused": 7}[kind])
    B, G, H, T = 1, 4, 2, 1024
    k = stress_keys(kind, rng, B, H, T)
    v = np.flip(k, axis=2).copy()
    q = synth.Synth(4500 + kb, B, G * H, H, D, 1, "f32").q()
    gc, oc = build(B, H, T, kb, vb, 1, ch0, k, v)
    o_gpu, o_ref = run_decode(gc, oc, q, [T], keep, H, 1)
    check_per_sequence(o_gpu, o_ref, B, G * H, f"{kind} keys")
