"""Pins of the oracle's channel selection and decode attention.

Sources: Dual-QK summary Sec. 3.2 (keep the m channel groups with the
largest query norms under one shared mask; every key channel stays stored),
App. C.2 (query energy summed over the query heads of a GQA group), Sec. 3.4
(one global softmax), App. A (the mask only controls which key coordinates
are read); tq-kv abstract (scores taken from the codes).
"""
import numpy as np
import pytest

from oracle import oracle as orc


def rng_q(seed, B, Hq, d=128, scale=1.0):
    return (np.random.default_rng(seed).standard_normal((B, Hq, d)) * scale).astype(np.float32)


# ---------------------------------------------------------------- selection
def test_keep_all_sets_every_bit():
    m, _ = orc.select(rng_q(0, 3, 8), 2, 1, 32)
    assert np.all(m == 0xFFFFFFFF)


@pytest.mark.parametrize("keep", [1, 7, 19, 24, 31])
def test_selected_groups_dominate_the_rest(keep):
    q = rng_q(1, 4, 8)
    m, E = orc.select(q, 2, 1, keep)
    for b in range(4):
        for h in range(2):
            bits = np.array([(int(m[b, h]) >> p) & 1 for p in range(32)], bool)
            assert bits.sum() == keep
            assert E[b, h][bits].min() >= E[b, h][~bits].max()


def test_single_head_group_ranks_by_l2_norm_of_rotated_query():
    q = rng_q(2, 2, 3)
    m, E = orc.select(q, 3, 1, 10)  # G = 1
    for b in range(2):
        for h in range(3):
            qr = orc.rotate(q[b, h]).astype(np.float64)
            e = (qr.reshape(32, 4) ** 2).sum(1)
            np.testing.assert_allclose(E[b, h], e, rtol=1e-15)
            order = sorted(range(32), key=lambda p: (-e[p], p))[:10]
            assert int(m[b, h]) == sum(1 << p for p in order)


def test_gqa_energy_is_sum_over_query_heads():
    q = rng_q(3, 2, 8)
    _, Eg = orc.select(q, 2, 1, 5)   # G = 4
    _, E1 = orc.select(q, 8, 1, 5)   # G = 1, same query heads
    np.testing.assert_allclose(Eg, E1.reshape(2, 2, 4, 32).sum(2), rtol=1e-14)


def test_equal_energies_keep_lower_groups():
    q = np.ones((1, 2, 128), np.float32)
    m, _ = orc.select(q, 1, 0, 5)  # no rotation: every group has the same energy
    assert int(m[0, 0]) == 0b11111


def test_selection_without_rotation_uses_raw_query():
    q = np.zeros((1, 1, 128), np.float32)
    q[0, 0, 4 * 7 + 2] = 3.0
    q[0, 0, 4 * 20] = -2.0
    m, _ = orc.select(q, 1, 0, 2)
    assert int(m[0, 0]) == (1 << 7) | (1 << 20)


# ---------------------------------------------------------------- attention
def make_cache(seed, B=2, Hkv=2, n=40, k_bits=4, v_bits=4, rotate=1, ch0=0, capacity=None, kscale=1.0):
    rng = np.random.default_rng(seed)
    k = (rng.standard_normal((B, Hkv, n, 128)) * kscale).astype(np.float32)
    v = rng.standard_normal((B, Hkv, n, 128)).astype(np.float32)
    c = orc.Cache(B, Hkv, 128, capacity or n, k_bits, v_bits, rotate, ch0)
    c.append(k, v, 0)
    return c, k, v


def test_single_token_returns_its_value():
    c, _, _ = make_cache(10, n=1)
    q = rng_q(11, 2, 4)
    out = c.attention(q, np.array([1, 1]), None, 0.1).reshape(2, 4, 128)
    for b in range(2):
        for h in range(4):
            _, vh = c.dequantize(b, h // 2, 0, 1)
            np.testing.assert_allclose(out[b, h], vh[0], rtol=1e-15, atol=1e-15)


def test_identical_keys_average_the_values():
    rng = np.random.default_rng(12)
    n = 17
    k = np.repeat(rng.standard_normal((1, 1, 1, 128)).astype(np.float32), n, axis=2)
    v = rng.standard_normal((1, 1, n, 128)).astype(np.float32)
    c = orc.Cache(1, 1, 128, n, 2, 4, 1, 1)
    c.append(k, v, 0)
    out = c.attention(rng_q(13, 1, 1), np.array([n]), None, 0.3)
    _, vh = c.dequantize(0, 0, 0, n)
    np.testing.assert_allclose(out[0], vh.mean(0), rtol=1e-12, atol=1e-14)


def test_zero_scale_is_uniform_attention_over_the_sequence_length():
    c, _, _ = make_cache(14, n=30)
    q = rng_q(15, 2, 2)
    out = c.attention(q, np.array([30, 11]), None, 0.0).reshape(2, 2, 128)
    for b, n in [(0, 30), (1, 11)]:
        for h in range(2):
            _, vh = c.dequantize(b, h, 0, n)
            np.testing.assert_allclose(out[b, h], vh.mean(0), rtol=1e-12, atol=1e-14)


def test_empty_sequence_gives_zeros():
    c, _, _ = make_cache(16, n=8)
    out = c.attention(rng_q(17, 2, 2), np.array([0, 8]), None, 0.1).reshape(2, 2, 128)
    assert not out[0].any() and out[1].any()


def test_tokens_past_the_length_are_ignored():
    c1, k, v = make_cache(18, B=1, Hkv=1, n=20)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 12:] *= 5
    v2[:, :, 12:] += 3
    c2 = orc.Cache(1, 1, 128, 20, 4, 4, 1, 0)
    c2.append(k2, v2, 0)
    q = rng_q(19, 1, 1)
    np.testing.assert_array_equal(c1.attention(q, np.array([12]), None, 0.2), c2.attention(q, np.array([12]), None, 0.2))


def test_token_order_does_not_matter():
    c1, k, v = make_cache(20, B=1, Hkv=1, n=25)
    perm = np.random.default_rng(21).permutation(25)
    c2 = orc.Cache(1, 1, 128, 25, 4, 4, 1, 0)
    c2.append(k[:, :, perm], v[:, :, perm], 0)
    q = rng_q(22, 1, 1)
    np.testing.assert_allclose(c1.attention(q, np.array([25]), None, 0.2), c2.attention(q, np.array([25]), None, 0.2),
                               rtol=1e-12, atol=1e-14)


def test_output_is_linear_in_power_of_two_value_scaling():
    c1, k, v = make_cache(23, B=1, Hkv=1, n=20, v_bits=2)
    c2 = orc.Cache(1, 1, 128, 20, 4, 2, 1, 0)
    c2.append(k, v * 4, 0)
    q = rng_q(24, 1, 1)
    np.testing.assert_array_equal(4 * c1.attention(q, np.array([20]), None, 0.2),
                                  c2.attention(q, np.array([20]), None, 0.2))


def test_full_mask_equals_unpruned():
    c, _, _ = make_cache(25, ch0=1, k_bits=2, v_bits=2)
    q = rng_q(26, 2, 8)
    full = np.full((2, 2), 0xFFFFFFFF, np.uint32)
    np.testing.assert_array_equal(c.attention(q, np.array([40, 33]), None, 0.09),
                                  c.attention(q, np.array([40, 33]), full, 0.09))


@pytest.mark.parametrize("ch0", [0, 1])
def test_pruning_equals_zeroing_the_query_channels(ch0):
    # rotation off so the query seen by the scores is the input itself
    c, _, _ = make_cache(27, rotate=0, ch0=ch0)
    q = rng_q(28, 2, 4)
    mask, _ = orc.select(q, 2, 0, 13)
    qz = q.copy()
    for b in range(2):
        for h in range(4):
            m = int(mask[b, h // 2])
            for p in range(32):
                if not (m >> p) & 1:
                    qz[b, h, 4 * p:4 * p + 4] = 0
    lens = np.array([40, 29])
    np.testing.assert_array_equal(c.attention(q, lens, mask, 0.1), c.attention(qz, lens, None, 0.1))


def test_matches_materialized_matrices():
    c, _, _ = make_cache(29, ch0=1, k_bits=2, v_bits=4, kscale=2.0)
    q = rng_q(30, 2, 4)
    mask, _ = orc.select(q, 2, 1, 21)
    lens = np.array([40, 7])
    out = c.attention(q, lens, mask, 0.125).reshape(2, 4, 128)
    for b in range(2):
        for h in range(4):
            kh, vh = c.dequantize(b, h // 2, 0, lens[b])
            sel = np.repeat([(int(mask[b, h // 2]) >> p) & 1 for p in range(32)], 4).astype(bool)
            qr = orc.rotate(q[b, h]).astype(np.float64) * sel
            s = 0.125 * (kh @ qr)
            p = np.exp(s - s.max())
            np.testing.assert_allclose(out[b, h], p @ vh / p.sum(), rtol=1e-12, atol=1e-13)


def test_quantized_attention_approximates_exact_attention():
    # INT4 with a Hadamard rotation: attention over the decoded cache stays close
    # to fp64 attention over the original K, V (a dropped zero-point, a wrong
    # scale or a mis-packed code would not)
    c, k, v = make_cache(31, B=1, Hkv=1, n=256, kscale=1.0)
    q = rng_q(32, 1, 1)
    out = c.attention(q, np.array([256]), None, 1 / np.sqrt(128))[0]
    s = (k[0, 0].astype(np.float64) @ q[0, 0].astype(np.float64)) / np.sqrt(128)
    p = np.exp(s - s.max())
    exact = p @ v[0, 0].astype(np.float64) / p.sum()
    err = np.abs(out - exact).max() / np.abs(exact).max()
    assert err < 0.15, err
    # and INT4 beats INT2 on the same data
    c2 = orc.Cache(1, 1, 128, 256, 2, 2, 1, 0)
    c2.append(k, v, 0)
    out2 = c2.attention(q, np.array([256]), None, 1 / np.sqrt(128))[0]
    assert np.abs(out - exact).max() < np.abs(out2 - exact).max()


def test_row_subset_matches_full_output():
    c, _, _ = make_cache(33)
    q = rng_q(34, 2, 6)
    lens = np.array([40, 21])
    full = c.attention(q, lens, None, 0.1)
    rows = np.array([7, 0, 11, 3])
    np.testing.assert_array_equal(c.attention(q, lens, None, 0.1, rows=rows), full[rows])
