"""Pins of the oracle's value-side rotation and clipping ratio.

Sources: Dual-QK summary App. B.2 and Sec. 3.3 (values take a rotation
composed with a Hadamard transform and per-token asymmetric quantization with
a 0.92 clipping ratio; keys are not clipped).  The Hadamard part is built; the
ratio is read as scaling the group's minimum and maximum before the scale and
zero are formed, so values beyond the clipped range saturate.  The attention
output leaves the rotated basis through the same orthonormal transform, which
is its own inverse.
"""
import numpy as np
import pytest

from oracle import oracle as orc


def _groups(seed, n=200):
    rng = np.random.default_rng(seed)
    return [(rng.standard_normal(32) * rng.uniform(0.01, 30.0)).astype(np.float32) for _ in range(n)]


@pytest.mark.parametrize("bits", [2, 4])
def test_clip_one_is_the_unclipped_quantizer(bits):
    for x in _groups(10 + bits):
        a = orc.quantize_group(x, bits)
        b = orc.quantize_group(x, bits, clip=1.0)
        assert a[0] == b[0] and a[1] == b[1] and np.array_equal(a[2], b[2])


@pytest.mark.parametrize("bits,clip", [(2, 0.92), (4, 0.92), (2, 0.5)])
def test_clipping_saturates_the_extremes_and_spans_the_clipped_range(bits, clip):
    L = (1 << bits) - 1
    saturated = 0
    for x in _groups(20 + bits):
        mn, mx = float(x.min()), float(x.max())
        if not (mn < 0.0 < mx):
            continue
        s16, z16, codes, _, _, _ = orc.quantize_group(x, bits, clip=clip)
        s, z = orc.half_value(s16), orc.half_value(z16)
        # the range is the clipped one, up to the fp16 rounding of scale and zero
        assert abs(z - clip * mn) <= 2 ** -10 * abs(clip * mn) + 2 ** -24
        assert abs((z + L * s) - clip * mx) <= 2 ** -9 * (clip * (mx - mn)) + 2 ** -24
        # the extremes lie beyond the clipped range and saturate
        assert codes[int(np.argmax(x))] == L and codes[int(np.argmin(x))] == 0
        # every element sits within half a step of its value clamped into the range
        deq = s * codes.astype(np.float64) + z
        target = np.clip(x.astype(np.float64), z, z + L * s)
        assert np.all(np.abs(deq - target) <= 0.5 * s * (1 + 1e-3) + 1e-12)
        saturated += int((codes == 0).sum() + (codes == L).sum())
    assert saturated > 0


def _exact_attention(q_rot, khat, v, scale):
    s = scale * (khat @ q_rot)
    p = np.exp(s - s.max())
    return (p / p.sum()) @ v


@pytest.mark.parametrize("vb,clip", [(4, 1.0), (4, 0.92), (2, 0.92)])
def test_rotated_values_come_back_to_the_value_basis(vb, clip):
    # attention over rotated, quantized values, rotated back, against attention
    # over the unquantized values with the same scores: within the values'
    # reconstruction error, which the rotation leaves unchanged in 2-norm
    rng = np.random.default_rng(31 + vb)
    n, d = 96, 128
    k = rng.standard_normal((1, 1, n, d)).astype(np.float32)
    v = (rng.standard_normal((1, 1, n, d)) * 0.7 + 0.2).astype(np.float32)
    q = rng.standard_normal((1, 1, d)).astype(np.float32)
    scale = 1.0 / np.sqrt(d)
    c = orc.Cache(1, 1, d, 128, 4, vb, 1, 0, rotate_v=1, v_clip=clip)
    c.append(k, v, 0)
    out = c.attention(q, np.array([n], np.int32), None, scale)[0]
    khat, vhat_rot = c.dequantize(0, 0, 0, n)
    want = _exact_attention(orc.rotate(q[0, 0]).astype(np.float64), khat, v[0, 0].astype(np.float64), scale)
    # reconstruction error of every value row, measured in the rotated basis
    v_rot = np.stack([orc.rotate(v[0, 0, j]) for j in range(n)]).astype(np.float64)
    row_err = np.linalg.norm(vhat_rot - v_rot, axis=1)
    assert np.linalg.norm(out - want) <= row_err.max() * (1 + 1e-9) + 1e-12
    # and far closer than the same output left in the rotated basis
    assert np.linalg.norm(out - want) < 0.2 * np.linalg.norm(orc.rotate(out.astype(np.float32)) - want)


def test_unrotated_unclipped_values_are_the_plain_cache():
    rng = np.random.default_rng(5)
    k = rng.standard_normal((1, 2, 40, 128)).astype(np.float32)
    v = rng.standard_normal((1, 2, 40, 128)).astype(np.float32)
    a = orc.Cache(1, 2, 128, 128, 4, 2, 1, 1)
    b = orc.Cache(1, 2, 128, 128, 4, 2, 1, 1, rotate_v=0, v_clip=1.0)
    a.append(k, v, 3)
    b.append(k, v, 3)
    assert np.array_equal(a.v_codes, b.v_codes) and np.array_equal(a.v_scales, b.v_scales)
