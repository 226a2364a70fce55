"""Pins of the oracle's bucket-relative RoPE.

Source: Dual-QK summary Sec. 3.4 and App. C.4 -- stored keys are expressed
relative to local anchors, one every w tokens (w = 2048 on the pages), with
the same dual transform pair; the query takes a per-bucket adjustment, masks
may differ between buckets, and one softmax covers them all.

Readings pinned here: token n is embedded at offset n mod w; the query (at
position len - 1) at offset (len - 1) - w * k for bucket k; rotary embedding
pairs channel i with i + d/2.  The pins come from the mathematics of rotary
embedding (rotations that compose, preserve norms and depend only on the
position difference in a dot product), not from the oracle's own steps.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc

D = 128


def inv_freq(base=10000.0):
    return (base ** (-np.arange(0, D, 2) / D)).astype(np.float32)


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def abs_rope64(x, f, pos):
    """Absolute rotary embedding in fp64 (numpy's cos and sin)."""
    x = np.asarray(x, np.float64)
    th = float(pos) * f.astype(np.float64)
    c, s = np.cos(th), np.sin(th)
    a, b = x[: D // 2], x[D // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s])


def test_rope_pairs_channel_i_with_i_plus_half():
    f = inv_freq()
    for i in (0, 5, 63):
        e = np.zeros(D, np.float32)
        e[i] = 1.0
        out = orc.rope(e, f, 37).astype(np.float64)
        th = 37.0 * float(f[i])
        want = np.zeros(D)
        want[i], want[i + D // 2] = np.cos(th), np.sin(th)
        np.testing.assert_allclose(out, want, atol=2 ** -24)
    x = np.random.default_rng(0).standard_normal(D).astype(np.float32)
    assert np.array_equal(orc.rope(x, f, 0), x)  # position 0 is the identity


def test_rope_is_a_rotation_that_composes():
    rng = np.random.default_rng(1)
    f = inv_freq()
    for _ in range(10):
        x = rng.standard_normal(D).astype(np.float32)
        a, b = (int(v) for v in rng.integers(0, 5000, 2))
        ra = orc.rope(x, f, a).astype(np.float64)
        assert abs(np.linalg.norm(ra) - np.linalg.norm(x.astype(np.float64))) < 1e-5 * np.linalg.norm(x)
        two = orc.rope(orc.rope(x, f, a), f, b).astype(np.float64)
        np.testing.assert_allclose(two, orc.rope(x, f, a + b).astype(np.float64), atol=1e-5 * np.abs(x).max())


def test_dot_product_depends_on_the_position_difference_only():
    rng = np.random.default_rng(2)
    f = inv_freq()
    q = rng.standard_normal(D).astype(np.float32)
    k = rng.standard_normal(D).astype(np.float32)
    for p, n, anchor in ((5000, 4100, 4096), (2047, 0, 0), (9000, 2050, 2048)):
        rel = orc.rope(q, f, p - anchor).astype(np.float64) @ orc.rope(k, f, n - anchor).astype(np.float64)
        ab = abs_rope64(q, f, p) @ abs_rope64(k, f, n)
        assert abs(rel - ab) < 1e-4 * np.linalg.norm(q) * np.linalg.norm(k)


def test_zero_frequencies_are_the_plain_cache():
    # no rotation at any position: the bucketed cache is the plain one
    rng = np.random.default_rng(3)
    H, T = 2, 90
    k = rng.standard_normal((1, H, T, D)).astype(np.float32)
    v = rng.standard_normal((1, H, T, D)).astype(np.float32)
    q = rng.standard_normal((1, 2 * H, D)).astype(np.float32)
    zero = np.zeros(D // 2, np.float32)
    a = orc.Cache(1, H, D, 128, 4, 2, 1, 1, 0, 1.0, 4, 8, bucket_w=32, inv_freq=zero)
    b = orc.Cache(1, H, D, 128, 4, 2, 1, 1, 0, 1.0, 4, 8)
    a.append(k, v, 0)
    b.append(k, v, 0)
    for name in ("k_codes", "k_scales", "k_ch0", "k_win"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name
    lens = np.array([T], np.int32)
    ma, _ = a.select_buckets(q, lens, 19)
    mb, _ = orc.select(q, H, 1, 19)
    assert np.array_equal(ma, np.broadcast_to(mb[:, None, :], ma.shape))
    np.testing.assert_array_equal(a.attention(q, lens, ma, 0.09), b.attention(q, lens, mb, 0.09))


@pytest.mark.parametrize("rot,w", [(0, 16), (1, 7), (2, 32)])
def test_window_scores_equal_absolute_rope_scores(rot, w):
    # every token in the bf16 sink, several buckets, value rows one-hot so the
    # output is the softmax itself and ln p_n - ln p_0 = s_n - s_0: the
    # bucket-relative scores must be the absolute-position RoPE scores up to the
    # bf16 rounding of the stored keys; without the per-bucket query
    # adjustment they are not
    rng = np.random.default_rng(4 + rot)
    H, T, G = 2, 80, 2
    f = inv_freq(500.0)  # fast rotations, so positions matter over a few tokens
    k = rng.standard_normal((1, H, T, D)).astype(np.float32)
    v = np.zeros((1, H, T, D), np.float32)
    v[0, :, np.arange(T), np.arange(T)] = 1.0
    q = rng.standard_normal((1, H * G, D)).astype(np.float32)
    tq = tk = None
    if rot == 2:
        tq = np.empty((H, D, D), np.float32)
        tk = np.empty((H, D, D), np.float32)
        for h in range(H):
            t = np.eye(D) + 0.3 * rng.standard_normal((D, D)) / np.sqrt(D)
            tq[h], tk[h] = t, np.linalg.inv(t).T
    c = orc.Cache(1, H, D, 128, 4, 4, rot, 0, 0, 1.0, 128, 0, tq, tk, bucket_w=w, inv_freq=f)
    c.append(k, v, 0)
    scale = 1.0 / np.sqrt(D)
    out = c.attention(q, np.array([T], np.int32), None, scale)
    p = T - 1
    for hq in range(H * G):
        h = hq // G
        s_true = scale * np.array([abs_rope64(q[0, hq], f, p) @ abs_rope64(k[0, h, n], f, n) for n in range(T)])
        # without the adjustment: the query at its absolute position against anchored keys
        s_wrong = scale * np.array([abs_rope64(q[0, hq], f, p) @ abs_rope64(k[0, h, n], f, n % w) for n in range(T)])
        got = np.log(out[hq, :T]) - np.log(out[hq, 0])
        # per-score bound: bf16 rounding of each stored key element (relative
        # 2^-8), amplified by the pair's condition number, plus fp32 roundings
        cond = 1.0 if rot < 2 else np.linalg.cond(tq[h].astype(np.float64))
        kn = np.linalg.norm(k[0, h], axis=1).astype(np.float64)
        delta = scale * np.linalg.norm(q[0, hq]) * kn * (2.0 ** -8 * cond + 1e-5)
        want = s_true - s_true[0]
        assert np.all(np.abs(got - want) <= delta + delta[0] + 1e-9)
        assert np.max(np.abs((s_wrong - s_wrong[0]) - want)) > 10 * np.max(delta + delta[0])


def test_each_bucket_has_its_own_mask_and_query():
    # quantized tokens in three buckets: the oracle's output is the softmax
    # over tokens scored with their own bucket's query and mask, assembled
    # here from the dequantized rows
    rng = np.random.default_rng(6)
    H, G, w, T = 2, 2, 40, 100
    f = inv_freq(300.0)
    k = rng.standard_normal((1, H, T, D)).astype(np.float32)
    v = rng.standard_normal((1, H, T, D)).astype(np.float32)
    q = rng.standard_normal((1, H * G, D)).astype(np.float32)
    c = orc.Cache(1, H, D, 128, 4, 4, 1, 0, 0, 1.0, 0, 0, bucket_w=w, inv_freq=f)
    c.append(k, v, 0)
    lens = np.array([T], np.int32)
    mask, _ = c.select_buckets(q, lens, 13)
    assert mask.shape == (1, 4, H)  # ceil(128 / 40) buckets
    p = T - 1
    for kb in range(3):
        qk = np.stack([orc.rotate(orc.rope(q[0, hq], f, p - kb * w)) for hq in range(H * G)])[None]
        want, _ = orc.select(qk, H, 0, 13)
        assert np.array_equal(mask[:, kb], want)
    assert len({int(m) for m in mask[0, :3, 0]}) > 1  # the buckets' masks differ here
    out = c.attention(q, lens, mask, 0.1)
    for hq in range(H * G):
        h = hq // G
        khat, vhat = c.dequantize(0, h, 0, T)
        s = np.empty(T)
        for n in range(T):
            kb = n // w
            qr = orc.rotate(orc.rope(q[0, hq], f, p - kb * w)).astype(np.float64)
            sel = np.array([(int(mask[0, kb, h]) >> (ch // 4)) & 1 for ch in range(D)], bool)
            s[n] = 0.1 * (khat[n, sel] @ qr[sel])
        pr = np.exp(s - s.max())
        np.testing.assert_allclose(out[hq], (pr / pr.sum()) @ vhat, rtol=1e-10, atol=1e-12)
