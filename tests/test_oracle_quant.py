"""Pins of the oracle's fp16/bf16 rounding, group quantizer and packed layout.

Sources: Dual-QK summary Sec. 3.3 (asymmetric per-token keys, channel 0 in
BF16 outside the range estimate, channel-major key rows), App. B.2
(per-token asymmetric values), App. C.3 (channel 0 narrows the range when it
sets an extremum); CASK-Q Method (scalar codes + FP16 scales); tq-kv abstract
(incremental append: earlier tokens are never re-quantized).
"""
import os

import numpy as np
import pytest
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_groups.txt")


def test_half_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 10.0 ** rng.integers(-9, 5, 4000),
        np.array([0.0, -0.0, 65504, 65519, 65520, -65520, 6.1e-5, 5.96e-8, 2.98e-8, 2.99e-8, 1e-9,
                  1.00048828125, 1.000244140625, 1.000732421875, 2049.0, 2051.0], np.float32)])
    for x in xs:
        want = np.float32(x).astype(np.float16).view(np.uint16)
        assert orc.half_rn(x) == int(want), x
        assert orc.half_value(int(want)) == float(np.float16(np.float32(x)))


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    xs = rng.standard_normal(5000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 5000)
    xs = np.concatenate([xs, np.array([1.00390625, 1.01171875, 1.0078125, 3.0e-39, -0.0], np.float32)])
    want = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for x, w in zip(xs, want):
        assert orc.bf16_rn(x) == int(w), x
        assert orc.bf16_value(int(w)) == float(torch.tensor(float(x)).to(torch.bfloat16).float())


def _golden_cases():
    cases = []
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        name, bits, vals, s, z, codes = [f.strip() for f in line.split("|")]
        cases.append((name, int(bits), [float(v) for v in vals.split()], float(s), float(z),
                      [int(c) for c in codes.split()]))
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c[0])
def test_hand_computed_groups(case):
    _, bits, vals, s, z, codes = case
    s16, z16, got, _, _, clamped = orc.quantize_group(np.array(vals, np.float32), bits)
    assert orc.half_value(s16) == s
    assert orc.half_value(z16) == z
    assert list(got) == codes
    assert clamped == 0


def test_codes_in_range_and_error_bound():
    rng = np.random.default_rng(2)
    for bits in (2, 4):
        L = (1 << bits) - 1
        for _ in range(300):
            x = (rng.standard_normal(32) * 10.0 ** rng.uniform(-3, 2)).astype(np.float32)
            s16, z16, codes, _, _, clamped = orc.quantize_group(x, bits)
            assert codes.max() <= L
            s, z = orc.half_value(s16), orc.half_value(z16)
            xhat = s * codes.astype(np.float64) + z
            # |x - xhat| <= s/2 up to the fp32/fp16 rounding of (x - z)/s, scale and zero
            bound = 0.5 * s + 1e-3 * (x.max() - x.min()) + abs(z - x.min()) + 1e-6 * np.abs(x)
            assert np.all(np.abs(x - xhat) <= bound)


def test_requantizing_dequantized_values_gives_same_codes():
    rng = np.random.default_rng(3)
    for bits in (2, 4):
        for _ in range(200):
            x = (rng.standard_normal(32) * 3).astype(np.float32)
            s16, z16, codes, _, _, _ = orc.quantize_group(x, bits)
            s, z = np.float32(orc.half_value(s16)), np.float32(orc.half_value(z16))
            # dequantized points lie on the grid, so dividing back lands on the code
            xhat = (np.float64(s) * codes + np.float64(z)).astype(np.float32)
            back = np.rint((xhat - z) / s)
            np.testing.assert_array_equal(back, codes)


def test_constant_group_gives_zero_codes():
    for bits in (2, 4):
        s16, z16, codes, _, _, _ = orc.quantize_group(np.full(32, -3.3, np.float32), bits)
        assert s16 == 0 and not codes.any()
        assert orc.half_value(z16) == float(np.float16(np.float32(-3.3)))


def _cache_with(k, v, k_bits, v_bits, rotate, ch0, capacity=None, offset=0):
    B, H, n, d = k.shape
    c = orc.Cache(B, H, d, capacity or n, k_bits, v_bits, rotate, ch0)
    st = c.append(k, v, offset)
    return c, st


def test_pack_unpack_roundtrip_matches_group_quantizer():
    rng = np.random.default_rng(4)
    for kb, vb, rot, ch0 in [(4, 4, 1, 0), (2, 2, 1, 1), (4, 2, 0, 1), (2, 4, 0, 0)]:
        k = (rng.standard_normal((2, 2, 5, 128)) * 2).astype(np.float32)
        v = rng.standard_normal((2, 2, 5, 128)).astype(np.float32)
        c, _ = _cache_with(k, v, kb, vb, rot, ch0, capacity=8, offset=2)
        for b in range(2):
            for h in range(2):
                for t in range(5):
                    kr = orc.rotate(k[b, h, t]) if rot else k[b, h, t]
                    want_k = []
                    for g in range(4):
                        inc = np.ones(32, np.uint8)
                        if ch0 and g == 0:
                            inc[0] = 0
                        want_k += list(orc.quantize_group(kr[32 * g:32 * g + 32], kb, inc)[2])
                    np.testing.assert_array_equal(c.unpack(b, h, t + 2, 0), want_k)
                    want_v = np.concatenate([orc.quantize_group(v[b, h, t, 32 * g:32 * g + 32], vb)[2]
                                             for g in range(4)])
                    np.testing.assert_array_equal(c.unpack(b, h, t + 2, 1), want_v)


def test_key_layout_is_channel_major_words():
    # one token, codes known: rotate off, values equal to their INT4 codes
    d = 128
    k = np.zeros((1, 1, 1, d), np.float32)
    for g in range(4):
        k[0, 0, 0, 32 * g:32 * g + 32] = np.arange(32) % 16
        k[0, 0, 0, 32 * g + 31] = 15  # max 15, min 0 -> scale 1, zero 0
    v = np.zeros_like(k)
    c, _ = _cache_with(k, v, 4, 4, 0, 0, capacity=256, offset=129)
    codes = (np.arange(d) % 32) % 16
    codes[31::32] = 15
    words = c.k_codes.view(np.uint16).reshape(2, 32, 128)  # [block of 128 tokens][group of 4 channels][token]
    for p in range(32):
        want = sum(int(codes[4 * p + i]) << (4 * i) for i in range(4))
        assert words[1, p, 1] == want  # token 129 = block 1, position 1
    words[1, :, 1] = 0
    assert not words.any()
    sc = c.k_scales.view(np.uint32).reshape(2, 4, 128)  # [block][group][token]
    assert sc[1, :, 1].all()
    sc[1, :, 1] = 0
    assert not sc.any()


def test_value_layout_is_channel_major_rows_with_swizzled_chunks():
    # INT2, rotation off, one token at position 129 = block 1, token 1 of the
    # block; value of channel ch is ch % 4, which is also its code (min 0, max 3)
    d = 128
    v = np.zeros((1, 1, 1, d), np.float32)
    v[0, 0, 0, :] = np.tile(np.array([0, 1, 2, 3], np.float32), 32)
    c, _ = _cache_with(np.zeros_like(v), v, 2, 2, 0, 0, capacity=256, offset=129)
    rows = c.v_codes.reshape(2, 128, 32)  # [block][channel][128 tokens x 2 bits]
    # hand-placed: token 1 is the second crumb (bits 2-3) of byte 0 of chunk 0;
    # chunk 0 of channels 4-7, 12-15, ... sits in the second 16-byte half of the row
    assert rows[1, 1, 0] == 1 << 2
    assert rows[1, 2, 0] == 2 << 2
    assert rows[1, 3, 0] == 3 << 2
    assert rows[1, 5, 16] == 1 << 2
    assert rows[1, 6, 16] == 2 << 2
    assert rows[1, 127, 16] == 3 << 2
    assert rows[1, 9, 0] == 1 << 2
    rows[1, :, 0] = 0
    rows[1, :, 16] = 0
    assert not rows.any()


def test_value_rows_share_bytes_between_tokens_without_clobbering():
    # INT4: tokens 32 and 33 of a block share byte 0 of chunk 1 (low, high nibble)
    d = 128
    v = np.zeros((1, 1, 2, d), np.float32)
    v[0, 0, 0, :] = np.tile(np.array([0, 15], np.float32), 64)  # codes 0, 15, 0, 15, ...
    v[0, 0, 1, :] = np.tile(np.array([15, 0], np.float32), 64)  # codes 15, 0, 15, 0, ...
    c = orc.Cache(1, 1, d, 128, 4, 4, 0, 0)
    c.append(np.zeros((1, 1, 1, d), np.float32), v[:, :, :1], 32)
    c.append(np.zeros((1, 1, 1, d), np.float32), v[:, :, 1:], 33)
    rows = c.v_codes.reshape(128, 64)  # [channel][128 tokens x 4 bits]
    # chunk 1 of channel ch lands at chunk position 1 ^ ((ch >> 1) & 3)
    assert rows[0, 16] == 0xF0   # ch 0: token 32 code 0, token 33 code 15
    assert rows[1, 16] == 0x0F   # ch 1: token 32 code 15, token 33 code 0
    assert rows[2, 0] == 0xF0    # ch 2: chunk position 0
    assert rows[5, 48] == 0x0F   # ch 5: chunk position 3
    assert rows[7, 32] == 0x0F   # ch 7: chunk position 2
    assert np.count_nonzero(rows) == 128
    assert list(c.unpack(0, 0, 32, 1)) == [0, 15] * 64
    assert list(c.unpack(0, 0, 33, 1)) == [15, 0] * 64


def test_channel0_outlier_is_excluded_from_range():
    rng = np.random.default_rng(5)
    k = rng.standard_normal((1, 1, 2, 128)).astype(np.float32)
    k[0, 0, 1] = k[0, 0, 0]
    k[0, 0, 1, 0] = 1000.0  # outlier only in channel 0 of token 1
    v = np.zeros_like(k)
    c, _ = _cache_with(k, v, 2, 2, 0, 1)
    sc = c.k_scales.reshape(4, 128, 2)  # [group][token (one block)][scale, zero]
    np.testing.assert_array_equal(sc[:, 0], sc[:, 1])
    np.testing.assert_array_equal(c.unpack(0, 0, 0, 0)[1:], c.unpack(0, 0, 1, 0)[1:])
    assert c.unpack(0, 0, 1, 0)[0] == 0
    assert orc.bf16_value(int(c.k_ch0[1])) == 1000.0
    # without the channel-0 rule the outlier widens group 0's range
    c2, _ = _cache_with(k, v, 2, 2, 0, 0)
    assert orc.half_value(int(c2.k_scales.reshape(4, 128, 2)[0, 1, 0])) > 100


def test_channel0_keeps_rotated_value_in_bf16():
    rng = np.random.default_rng(6)
    k = rng.standard_normal((1, 1, 3, 128)).astype(np.float32)
    c, _ = _cache_with(k, np.zeros_like(k), 4, 4, 1, 1)
    for t in range(3):
        assert int(c.k_ch0[t]) == orc.bf16_rn(orc.rotate(k[0, 0, t])[0])


def test_append_leaves_other_tokens_untouched_and_is_incremental():
    rng = np.random.default_rng(7)
    k = rng.standard_normal((2, 2, 12, 128)).astype(np.float32)
    v = rng.standard_normal((2, 2, 12, 128)).astype(np.float32)
    whole = orc.Cache(2, 2, 128, 16, 4, 2, 1, 1)
    whole.append(k, v, 0)
    parts = orc.Cache(2, 2, 128, 16, 4, 2, 1, 1)
    parts.append(k[:, :, :5], v[:, :, :5], 0)
    snap = parts.k_codes.copy()
    parts.append(k[:, :, 5:], v[:, :, 5:], 5)
    for name in ("k_codes", "k_scales", "k_ch0", "v_codes", "v_scales"):
        np.testing.assert_array_equal(getattr(whole, name), getattr(parts, name))
    # tokens 12..127 of the (single) key block were never written
    assert not whole.k_codes.view(np.uint16).reshape(2, 2, 32, 128)[..., 12:].any()
    assert snap.view(np.uint16).reshape(2, 2, 32, 128)[..., :5].any()


def test_append_rejects_overflowing_offset():
    c = orc.Cache(1, 1, 128, 4, 4, 4)
    with pytest.raises(ValueError):
        c.append(np.zeros((1, 1, 3, 128), np.float32), np.zeros((1, 1, 3, 128), np.float32), 2)


def test_tie_window_flags_exact_midpoints():
    # (x - z)/s = 0.5 exactly -> exempt
    _, _, _, ex, _, _ = orc.quantize_group(np.array([0, 0.5, 1, 3], np.float32), 2)
    assert list(ex) == [0, 1, 0, 0]


def test_signed_zero_extremes_are_canonical():
    a = orc.quantize_group(np.array([-0.0, 0.0, 0.0, -0.0], np.float32), 2)
    b = orc.quantize_group(np.array([0.0, -0.0, -0.0, 0.0], np.float32), 2)
    assert a[0] == b[0] == 0 and a[1] == b[1] == 0
