"""Host-side checks of the C ABI (no GPU needed): the library loads and exports
every entry point include/kvq.h declares, sizes and plans follow the layout,
and bad arguments are rejected with the documented status before anything is
enqueued.  Every call here fails validation or is a pure host query, so no
kernel is ever launched with the placeholder pointers used below."""
import ctypes
import os
import re

import pytest

from quantized_attention_kvq_b200 import native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x100000  # 16-byte-aligned placeholder; only reaches calls that are rejected


@pytest.fixture(scope="module")
def L():
    from quantized_attention_kvq_b200 import build
    build.build_kvq()
    return native.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return sorted(set(re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    declared = header_functions()
    assert len(declared) >= 9
    assert sorted(native.SYMBOLS) == declared
    for name in declared:
        assert hasattr(L, name), name


def test_bounds_checked_build_exports_every_declared_symbol(L):
    # the debug build of the same sources (-DKVQ_BOUNDS_CHECK), built beside the library
    path = os.path.join(os.path.dirname(native.LIB_PATH), "libkvq_checked.so")
    if not os.path.exists(path):
        from quantized_attention_kvq_b200 import build
        build.build_kvq(checked=True)
    C = ctypes.CDLL(path)
    for name in header_functions():
        assert hasattr(C, name), name
    # the regular library has no checks compiled in
    L.kvq_bounds_violations.restype = ctypes.c_uint32
    assert L.kvq_bounds_violations(0) == 0xFFFFFFFF


def desc(**kw):
    d = native.describe(kw.pop("B", 2), kw.pop("H", 2), kw.pop("cap", 256), kw.pop("kb", 4), kw.pop("vb", 2),
                        kw.pop("rot", 1), kw.pop("ch0", 1))
    for k, v in kw.items():
        setattr(d, k, v)
    for f in ("k_codes", "k_scales", "k_ch0", "v_codes", "v_scales"):
        if getattr(d, f) is None:
            setattr(d, f, FAKE)
    return d


def test_cache_sizes_follow_layout(L):
    d = native.describe(3, 5, 128, 4, 2, 1, 1)
    assert native.cache_sizes(d) == [3 * 5 * 128 * 32 * 2, 3 * 5 * 128 * 16, 3 * 5 * 128 * 2,
                                     3 * 5 * 128 * 32, 3 * 5 * 128 * 16]
    d = native.describe(1, 1, 256, 2, 4, 0, 0)
    assert native.cache_sizes(d) == [256 * 32, 256 * 16, 0, 256 * 64, 256 * 16]
    # keys are stored in blocks of 128 tokens: other capacities are refused
    assert native.lib().kvq_cache_sizes(ctypes.byref(native.describe(1, 1, 192, 4, 4)),
                                        (ctypes.c_size_t * 5)()) == native.KVQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, native.KVQ_ERR_UNSUPPORTED), ("k_bits", 3, native.KVQ_ERR_UNSUPPORTED),
    ("v_bits", 8, native.KVQ_ERR_UNSUPPORTED), ("capacity", 100, native.KVQ_ERR_UNSUPPORTED),
    ("group_size", 64, native.KVQ_ERR_UNSUPPORTED), ("prune_granule", 8, native.KVQ_ERR_UNSUPPORTED),
    ("batch", 0, native.KVQ_ERR_INVALID_ARG), ("rotate_k", 3, native.KVQ_ERR_INVALID_ARG),
    ("rotate_k", -1, native.KVQ_ERR_INVALID_ARG), ("rotate_k", 2, native.KVQ_ERR_INVALID_ARG),
    ("k_codes", 0, native.KVQ_ERR_INVALID_ARG), ("k_ch0", 0, native.KVQ_ERR_INVALID_ARG),
    ("v_scales", FAKE + 4, native.KVQ_ERR_INVALID_ARG), ("rotate_v", 2, native.KVQ_ERR_INVALID_ARG),
    ("v_clip", 0.0, native.KVQ_ERR_INVALID_ARG), ("v_clip", 1.5, native.KVQ_ERR_INVALID_ARG),
    ("v_clip", float("nan"), native.KVQ_ERR_INVALID_ARG), ("v_clip", -0.5, native.KVQ_ERR_INVALID_ARG),
])
def test_bad_cache_rejected(L, field, value, status):
    d = desc()
    setattr(d, field, value)
    rc = L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, native.KVQ_BF16, 8, 0, None)
    assert rc == status


def test_rotated_clipped_values_are_accepted(L):
    # the flags leave the layout alone: same sizes, and the host checks pass
    # (the enqueue itself is left to the GPU tests)
    d = desc(rotate_v=1, v_clip=0.92)
    assert native.cache_sizes(d) == native.cache_sizes(desc())
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, native.KVQ_BF16, 8, 250, None) == \
        native.KVQ_ERR_CAPACITY


@pytest.mark.parametrize("sink,recent,kw,vw,status", [
    (-1, 0, None, None, native.KVQ_ERR_INVALID_ARG), (0, -3, None, None, native.KVQ_ERR_INVALID_ARG),
    (200, 100, FAKE, FAKE, native.KVQ_ERR_INVALID_ARG),          # more than the capacity
    (64, 0, 0, FAKE, native.KVQ_ERR_INVALID_ARG), (0, 8, FAKE, FAKE + 8, native.KVQ_ERR_INVALID_ARG),
])
def test_bad_windows_rejected(L, sink, recent, kw, vw, status):
    d = desc(sink_tokens=sink, recent_tokens=recent)
    if kw is not None:
        d.k_window, d.v_window = kw, vw
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, native.KVQ_BF16, 8, 0, None) == status


def test_window_sizes(L):
    d = native.describe(3, 2, 4096, 2, 2, 1, 1, sink=64, recent=256)
    assert L.kvq_window_bytes(ctypes.byref(d)) == 3 * 2 * 320 * 128 * 2
    assert L.kvq_window_bytes(ctypes.byref(native.describe(3, 2, 4096, 2, 2))) == 0
    big = native.describe(1, 1, 8192, 4, 4, sink=1024, recent=1025)
    big.k_window = big.v_window = FAKE
    for f in ("k_codes", "k_scales", "v_codes", "v_scales"):
        setattr(big, f, FAKE)
    assert L.kvq_quantize_append(ctypes.byref(big), FAKE, FAKE, native.KVQ_BF16, 8, 0, None) == \
        native.KVQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("tq,tk", [(None, FAKE), (FAKE, None), (FAKE + 4, FAKE), (FAKE, FAKE + 8)])
def test_transform_pair_pointers_checked(L, tq, tk):
    d = desc(rotate_k=2)
    d.t_query, d.t_key = tq, tk
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, native.KVQ_BF16, 8, 0, None) == \
        native.KVQ_ERR_INVALID_ARG
    ws = L.kvq_decode_workspace_bytes(ctypes.byref(d), 8, 256)
    assert L.kvq_decode_attention(ctypes.byref(d), FAKE, native.KVQ_BF16, 8, FAKE, 256, None, 0.088, FAKE, FAKE,
                                  ws, None) == native.KVQ_ERR_INVALID_ARG
    # the channel selection reads only the query matrices (called only where
    # they are bad, so nothing is enqueued)
    if tq != FAKE:
        rc = L.kvq_select_channels(ctypes.byref(d), FAKE, native.KVQ_BF16, 8, 4, FAKE, None)
        assert rc == native.KVQ_ERR_INVALID_ARG


def test_transform_pair_workspace_holds_the_transformed_queries(L):
    d = desc()
    p = desc(rotate_k=2)
    p.t_query = p.t_key = FAKE
    for q_heads in (8, 16):
        plain = L.kvq_decode_workspace_bytes(ctypes.byref(d), q_heads, 256)
        pair = L.kvq_decode_workspace_bytes(ctypes.byref(p), q_heads, 256)
        assert pair - plain == -(-d.batch * q_heads * 128 * 4 // 256) * 256
    # and the step entry point's workspace grows with it
    assert L.kvq_decode_step_workspace_bytes(ctypes.byref(p), native.KVQ_BF16, 8, 256) - \
        L.kvq_decode_step_workspace_bytes(ctypes.byref(d), native.KVQ_BF16, 8, 256) == \
        L.kvq_decode_workspace_bytes(ctypes.byref(p), 8, 256) - L.kvq_decode_workspace_bytes(ctypes.byref(d), 8, 256)


@pytest.mark.parametrize("w,sink,status", [(100, 0, native.KVQ_ERR_UNSUPPORTED), (128, 200, native.KVQ_ERR_UNSUPPORTED),
                                           (-128, 0, native.KVQ_ERR_INVALID_ARG)])
def test_bad_buckets_rejected(L, w, sink, status):
    d = desc(cap=512, bucket_tokens=w, sink_tokens=sink)
    d.rope_inv_freq = FAKE
    if sink:
        d.k_window = d.v_window = FAKE
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, native.KVQ_BF16, 8, 0, None) == status


def test_bucket_rope_host_checks(L):
    d = desc(cap=512, bucket_tokens=256)  # 384 does not divide 512: checked below
    # no frequencies
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, native.KVQ_BF16, 8, 0, None) == \
        native.KVQ_ERR_INVALID_ARG
    d.rope_inv_freq = FAKE
    # an append may not cross a bucket boundary
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, native.KVQ_BF16, 8, 250, None) == \
        native.KVQ_ERR_INVALID_ARG
    # the plain selection has no query positions
    assert L.kvq_select_channels(ctypes.byref(d), FAKE, native.KVQ_BF16, 8, 4, FAKE, None) == \
        native.KVQ_ERR_INVALID_ARG
    assert L.kvq_select_channels_at(ctypes.byref(d), FAKE, native.KVQ_BF16, 8, None, 4, FAKE, None) == \
        native.KVQ_ERR_INVALID_ARG
    many = desc(B=300, cap=128 * 256, bucket_tokens=128)  # 300 x 256 bucket rows
    many.rope_inv_freq = FAKE
    assert L.kvq_quantize_append(ctypes.byref(many), FAKE, FAKE, native.KVQ_BF16, 8, 0, None) == \
        native.KVQ_ERR_UNSUPPORTED
    # without buckets the batch alone is the grid row count
    wide = desc(B=65536, cap=128)
    assert L.kvq_quantize_append(ctypes.byref(wide), FAKE, FAKE, native.KVQ_BF16, 8, 0, None) == \
        native.KVQ_ERR_UNSUPPORTED
    assert L.kvq_select_channels(ctypes.byref(wide), FAKE, native.KVQ_BF16, 8, 4, FAKE, None) == \
        native.KVQ_ERR_UNSUPPORTED
    edge = desc(B=65535, cap=128)
    assert L.kvq_cache_sizes(ctypes.byref(edge), (ctypes.c_size_t * 5)()) == native.KVQ_OK
    odd = desc(cap=512, bucket_tokens=384)
    odd.rope_inv_freq = FAKE
    assert L.kvq_quantize_append(ctypes.byref(odd), FAKE, FAKE, native.KVQ_BF16, 8, 0, None) == \
        native.KVQ_ERR_UNSUPPORTED
    # same array sizes; the decode workspace holds the bucket batch's partials,
    # query rows and lengths
    assert native.cache_sizes(d) == native.cache_sizes(desc(cap=512))
    plain = L.kvq_decode_workspace_bytes(ctypes.byref(desc(cap=512)), 8, 512)
    ws = L.kvq_decode_workspace_bytes(ctypes.byref(d), 8, 512)
    B, H, G, nb = 2, 2, 4, 2
    extra = (B * nb - B) * H * G * (128 * 4 + 8)
    assert ws >= plain + extra + B * nb * 8 * 128 * 4 + B * nb * 4
    # a step's mask holds one word per bucket
    assert L.kvq_decode_step_workspace_bytes(ctypes.byref(d), native.KVQ_BF16, 8, 512) >= ws + B * nb * H * 4


def test_append_argument_checks(L):
    d = desc()
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, native.KVQ_BF16, 200, 100, None) == \
        native.KVQ_ERR_CAPACITY
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, native.KVQ_BF16, -1, 0, None) == \
        native.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE, FAKE, 7, 4, 0, None) == native.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_append(ctypes.byref(d), None, FAKE, native.KVQ_BF16, 4, 0, None) == \
        native.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_append(ctypes.byref(d), FAKE + 2, FAKE, native.KVQ_BF16, 4, 0, None) == \
        native.KVQ_ERR_INVALID_ARG
    # zero new tokens is an accepted no-op that enqueues nothing
    assert L.kvq_quantize_append(ctypes.byref(d), None, None, native.KVQ_BF16, 0, 256, None) == native.KVQ_OK
    assert L.kvq_quantize_append(None, FAKE, FAKE, native.KVQ_BF16, 4, 0, None) == native.KVQ_ERR_INVALID_ARG


def test_select_argument_checks(L):
    d = desc()
    for keep in (0, 33):
        assert L.kvq_select_channels(ctypes.byref(d), FAKE, native.KVQ_BF16, 8, keep, FAKE, None) == \
            native.KVQ_ERR_INVALID_ARG
    assert L.kvq_select_channels(ctypes.byref(d), FAKE, native.KVQ_BF16, 7, 4, FAKE, None) == \
        native.KVQ_ERR_INVALID_ARG
    assert L.kvq_select_channels(ctypes.byref(d), FAKE, native.KVQ_BF16, 8, 4, None, None) == \
        native.KVQ_ERR_INVALID_ARG
    assert L.kvq_select_channels(ctypes.byref(d), FAKE, native.KVQ_BF16, 2 * 128, 4, FAKE, None) == \
        native.KVQ_ERR_UNSUPPORTED


def test_decode_argument_checks(L):
    d = desc()
    ws = L.kvq_decode_workspace_bytes(ctypes.byref(d), 8, 256)
    assert ws > 0

    def call(q_heads=8, max_len=256, ws_bytes=ws, scale=0.088, wsp=FAKE, lens=FAKE):
        return L.kvq_decode_attention(ctypes.byref(d), FAKE, native.KVQ_BF16, q_heads, lens, max_len, None,
                                      scale, FAKE, wsp, ws_bytes, None)
    assert call(ws_bytes=ws - 1) == native.KVQ_ERR_WORKSPACE
    assert call(max_len=257) == native.KVQ_ERR_CAPACITY
    assert call(max_len=-1) == native.KVQ_ERR_INVALID_ARG
    assert call(q_heads=7) == native.KVQ_ERR_INVALID_ARG
    assert call(q_heads=6) == native.KVQ_ERR_UNSUPPORTED  # G = 3 not built
    assert call(q_heads=2 * 32) == native.KVQ_ERR_UNSUPPORTED  # G = 32 not built
    assert call(scale=float("nan")) == native.KVQ_ERR_INVALID_ARG
    assert call(wsp=None) == native.KVQ_ERR_INVALID_ARG
    assert call(lens=None) == native.KVQ_ERR_INVALID_ARG
    assert call(wsp=FAKE + 8) == native.KVQ_ERR_INVALID_ARG


def test_decode_step_host_argument_checks(L):
    d = desc()
    ws = L.kvq_decode_step_workspace_bytes(ctypes.byref(d), native.KVQ_BF16, 8, 256)
    assert ws > L.kvq_decode_workspace_bytes(ctypes.byref(d), 8, 256)
    rc = L.kvq_decode_step_host(ctypes.byref(d), FAKE, native.KVQ_BF16, 8, FAKE, 256, 19, 0.088, FAKE, FAKE,
                                ws - 1, None)
    assert rc == native.KVQ_ERR_WORKSPACE
    rc = L.kvq_decode_step_host(ctypes.byref(d), FAKE, native.KVQ_BF16, 8, FAKE, 256, 0, 0.088, FAKE, FAKE, ws, None)
    assert rc == native.KVQ_ERR_INVALID_ARG


@pytest.mark.parametrize("B,H,G,max_len", [(8, 8, 4, 32768), (4, 8, 4, 131072), (64, 8, 8, 16384), (1, 1, 1, 1024),
                                           (16, 8, 2, 12288), (2, 2, 16, 100), (1, 1, 1, 0), (3, 7, 8, 4096)])
def test_decode_workspace_holds_one_partial_per_slot_and_head(L, B, H, G, max_len):
    # the decode spreads all tiles over 148 persistent CTAs; a (sequence, kv head)
    # unit leaves at most one partial per CTA its tiles touch and per epilogue
    # group of that CTA (two groups taking alternate tiles when G <= 4, else
    # one), and consecutive units share at most one CTA, so B*H + 148 slots of
    # groups * G partial rows suffice
    d = native.describe(B, H, max(128, (max_len + 127) // 128 * 128), 4, 4)
    ws = L.kvq_decode_workspace_bytes(ctypes.byref(d), H * G, max_len)
    groups = 2 if G <= 4 else 1
    rows = (B * H + 148) * groups * G
    assert ws >= rows * (128 * 4 + 8)
    # two 256-byte aligned partial regions, the in-call masks ([B][H] words) and the status word
    assert ws <= rows * (128 * 4 + 8) + 512 + (B * H * 4 + 255) // 256 * 256 + 256


def test_status_strings(L):
    for s in range(7):
        assert native.status_string(s)
    assert "workspace" in native.status_string(native.KVQ_ERR_WORKSPACE)
    assert "gave up" in native.status_string(native.KVQ_ERR_TIMEOUT)


def test_decode_status_argument_checks(L):
    d = desc(cap=512)
    need = L.kvq_decode_workspace_bytes(ctypes.byref(d), 8, 512)
    assert need > 0
    assert L.kvq_decode_status(None, 8, FAKE, need, None) == native.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_status(ctypes.byref(d), 8, None, need, None) == native.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_status(ctypes.byref(d), 6, FAKE, need, None) == native.KVQ_ERR_UNSUPPORTED
    assert L.kvq_decode_status(ctypes.byref(d), 8, FAKE, need - 1, None) == native.KVQ_ERR_WORKSPACE
    # the hook only arms the next split decode of this thread; clearing it is harmless
    L.kvq_test_withhold_tile(-1)
