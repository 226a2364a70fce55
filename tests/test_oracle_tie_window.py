"""Pins of the oracle's near-tie rule at group level and its row aggregation.

The byte-exact comparison of the packed cache lets a byte differ only in a
row the oracle flags: a code whose pre-rounding value (x - zero) / scale lies
within 1e-6 relative of a half-integer, or a group whose fp32 scale or fp32
minimum lies within 1e-6 relative of a midpoint between two neighbouring fp16
values (Dual-QK summary Sec. 3.3: FP16 scale and zero; the 1e-6 window is the
workload's tie rule).  The flags are checked here against midpoints taken from
numpy's own fp16 grid (np.nextafter in float16), not from the oracle's
exponent arithmetic, at normal and subnormal fp16 magnitudes, on both sides
of the window and at wrong-grid decoys.
"""
import numpy as np
import pytest

from oracle import oracle as orc

REL = 1e-6


def fp16_midpoints(x: float):
    """The two midpoints between the fp16 value nearest to x and its
    neighbours, from numpy's fp16 grid (float64, exact)."""
    h = np.float16(x)
    lo = np.nextafter(h, np.float16(-np.inf))
    hi = np.nextafter(h, np.float16(np.inf))
    return (float(lo) + float(h)) / 2.0, (float(h) + float(hi)) / 2.0


def near_midpoint(x: float) -> bool:
    a = abs(float(x))
    if a == 0.0 or a > 65504.0:
        return False
    return any(abs(a - m) <= REL * a for m in fp16_midpoints(a))


def _max_for_quotient(target: np.float32, L: int):
    """An fp32 max whose IEEE fp32 quotient by L is exactly target, or None."""
    mx = np.float32(target * np.float32(L))
    for _ in range(64):
        q = np.float32(mx / np.float32(L))
        if q == target:
            return mx
        mx = np.nextafter(mx, np.float32(np.inf) if q < target else np.float32(-np.inf))
    return None


def group_for_scale(target: np.float32, bits: int):
    """A 32-element fp32 group with minimum 0 whose fp32 scale
    (max - min) / L is exactly `target` (or, where no fp32 max gives that
    quotient, the nearest fp32 value above it that one does), the other
    elements on exact code points of the fp16 scale (so no element sits near
    a tie).  Returns (group, scale)."""
    L = (1 << bits) - 1
    mx = _max_for_quotient(target, L)
    while mx is None:  # one fp32 step at a time: far below the 2e-7 margins of the cases
        target = np.nextafter(target, np.float32(np.inf))
        mx = _max_for_quotient(target, L)
    s16 = np.float32(np.float16(target))
    x = np.zeros(32, np.float32)
    x[1] = mx
    for i in range(2, 32):
        j = i % L
        x[i] = np.float32(np.float64(s16) * j)  # exact: j has at most 4 bits
        if x[i] > mx:
            x[i] = 0.0
    return x, target


# (description, scale target): exact midpoints, inside and outside the window
NORMAL_MID = np.float32(1.5 + 2.0 ** -11)           # between 1.5 and 1.5 + 2^-10
SUB_MID = np.float32(3.5 * 2.0 ** -24)              # between fp16 subnormals 3 and 4 * 2^-24
LARGE_MID = np.float32(1000.0 + 0.25)               # quantum 0.5 at [512, 1024)


def _scaled(m, f):
    return np.float32(np.float64(m) * f)


SCALE_CASES = [
    ("normal, exact midpoint", NORMAL_MID, True),
    ("normal, 0.9e-6 above", _scaled(NORMAL_MID, 1 + 0.9e-6), True),
    ("normal, 0.9e-6 below", _scaled(NORMAL_MID, 1 - 0.9e-6), True),
    ("normal, 1.2e-6 above", _scaled(NORMAL_MID, 1 + 1.2e-6), False),
    ("normal, 1.2e-6 below", _scaled(NORMAL_MID, 1 - 1.2e-6), False),
    ("normal, on an fp16 value", np.float32(1.5), False),
    ("large, exact midpoint", LARGE_MID, True),
    ("large, 1.5e-6 above", _scaled(LARGE_MID, 1 + 1.5e-6), False),
    ("subnormal, exact midpoint", SUB_MID, True),
    ("subnormal, 0.9e-6 above", _scaled(SUB_MID, 1 + 0.9e-6), True),
    ("subnormal, 1.2e-6 above", _scaled(SUB_MID, 1 + 1.2e-6), False),
    # a midpoint of the grid a normal-number formula would give below 2^-14
    # (quantum 2^-33 here), but an integer multiple of the true subnormal
    # quantum 2^-24 plus a tiny offset: not near a true midpoint
    ("subnormal, wrong-grid decoy", np.float32(3.0 * 2.0 ** -24 + 2.0 ** -34), False),
    ("smallest subnormal midpoint", np.float32(0.5 * 2.0 ** -24), True),
    ("normal/subnormal boundary midpoint", np.float32(2.0 ** -14 - 2.0 ** -25), True),
]


@pytest.mark.parametrize("desc,target,want", SCALE_CASES, ids=[c[0] for c in SCALE_CASES])
@pytest.mark.parametrize("bits", [2, 4])
def test_group_flag_on_scale_near_fp16_midpoint(desc, target, want, bits):
    x, target = group_for_scale(target, bits)
    assert near_midpoint(target) == want, "case construction"
    s16, z16, codes, ex, gex, _ = orc.quantize_group(x, bits)
    assert orc.half_value(z16) == 0.0  # the zero (min 0) is never near a midpoint
    assert not ex.any(), "elements sit on exact code points"
    assert gex == int(want), desc


ZERO_CASES = [
    ("normal min at a midpoint", NORMAL_MID, True),
    ("negative min at a midpoint", np.float32(-NORMAL_MID), True),
    ("min 1.2e-6 off a midpoint", _scaled(NORMAL_MID, 1 + 1.2e-6), False),
    ("subnormal min at a midpoint", SUB_MID, True),
    ("min on an fp16 value", np.float32(-2.25), False),
    ("min beyond fp16 (saturates to -65504)", np.float32(-70000.0), False),
]


@pytest.mark.parametrize("desc,mn,want", ZERO_CASES, ids=[c[0] for c in ZERO_CASES])
def test_group_flag_on_zero_near_fp16_midpoint(desc, mn, want):
    # range 15 * 0.5 exactly: scale 0.5 (an fp16 value), so only the min decides
    x = np.full(32, mn, np.float32)
    x[1] = np.float32(np.float64(mn) + 7.5)
    s16, _, _, _, gex, _ = orc.quantize_group(x, 4)
    assert orc.half_value(s16) == 0.5
    assert near_midpoint(mn) == want
    assert gex == int(want), desc


def test_element_flag_window_is_relative_to_max_of_value_and_one():
    # (x - z)/s = k + 1/2 +- e: flagged when e <= 1e-6 * max(|v|, 1)
    s = np.float32(0.25)  # fp16-exact scale, zero 0
    for k, e, want in [(0, 0.0, True), (0, 0.9e-6, True), (0, 1.5e-6, False), (10, 0.9e-6 * 10.5, True),
                       (10, 1.2e-6 * 10.5, False)]:
        v = np.float32(k + 0.5 + e)
        xv = np.float32(v * s)  # exact: s is a power of two
        x = np.zeros(32, np.float32)
        x[1] = np.float32(15 * s)  # max -> scale (15 s)/15 = s exactly
        x[2] = xv
        _, z16, _, ex, gex, _ = orc.quantize_group(x, 4)
        assert gex == 0 and orc.half_value(z16) == 0.0
        assert bool(ex[2]) == want, (k, e)


def _row_with(groups):
    """A 128-channel row from four 32-channel groups."""
    return np.concatenate(groups).astype(np.float32)


def test_row_flags_aggregate_group_and_element_flags():
    # four tokens, rotation off so each row is stored as given; value rows are
    # plain and unflagged except token 3
    clean, _ = group_for_scale(np.float32(0.25), 4)
    flagged, _ = group_for_scale(NORMAL_MID, 4)
    tie = clean.copy()
    tie[5] = np.float32(2.5 * 0.25)  # (x - 0)/0.25 = 2.5 exactly: an element tie
    keys = np.stack([
        _row_with([clean, clean, clean, clean]),    # token 0: nothing flagged
        _row_with([clean, clean, flagged, clean]),  # token 1: group 2's scale at a midpoint
        _row_with([clean, tie, clean, clean]),      # token 2: one element tie
        _row_with([clean, clean, clean, clean]),    # token 3: key clean, value flagged
    ])
    vals = np.stack([keys[0], keys[0], keys[0], _row_with([flagged, clean, clean, clean])])
    c = orc.Cache(1, 1, 128, 128, 4, 4, 0, 0)
    st = c.append(keys[None, None], vals[None, None], 0, want_exempt=True)
    assert list(st["k_row_exempt"][0, 0]) == [0, 1, 1, 0]
    assert list(st["v_row_exempt"][0, 0]) == [0, 0, 0, 1]
    # every element of a flagged group counts as exempt, plus the tie element
    assert st["k_exempt"] == 32 + 1
    assert st["v_exempt"] == 32
    assert st["groups_exempt"] == 2
    assert st["k_elems"] == st["v_elems"] == 4 * 128


def test_row_flag_with_channel0_kept_counts_31_elements():
    # channel 0 outside group 0: a flagged group 0 contributes its 31 coded elements
    flagged, _ = group_for_scale(NORMAL_MID, 2)
    row = _row_with([flagged, flagged * 0, flagged * 0, flagged * 0])
    row[0] = 123.0  # channel 0 (kept in bf16) is outside the range; group 0's min/max unchanged
    c = orc.Cache(1, 1, 128, 128, 2, 2, 0, 1)
    st = c.append(row[None, None, None], np.zeros((1, 1, 1, 128), np.float32), 0, want_exempt=True)
    assert st["k_row_exempt"][0, 0, 0] == 1
    assert st["k_exempt"] == 31
    assert st["k_elems"] == 127
