"""Host-side pieces of bench.py that set the reported roofline: the
algorithmic bytes of a decode step and of an append, and the key under which
an ncu traffic figure is recorded.  Per-token byte counts follow the cache
layout in include/kvq.h (codes, fp16 scale/zero pairs, bf16 channel 0)."""
import numpy as np

import bench
from quantized_attention_kvq_b200 import workloads


def test_decode_bytes_unpruned_int4():
    wl = workloads.by_id(1)
    masks = np.full((wl.B, wl.Hkv), 0xFFFFFFFF, np.uint32)
    lens = np.full(wl.B, wl.T, np.int32)
    got = bench.algorithmic_bytes(wl, masks, lens)
    # per token and kv head: 128 4-bit key codes, 4 key (scale, zero) pairs,
    # 128 4-bit value codes, 4 value pairs
    per = 128 * 4 // 8 + 4 * 4 + 128 * 4 // 8 + 4 * 4
    assert per == 160
    q = wl.B * wl.Hq * 128 * 2
    assert got["split_kernel"] == wl.B * wl.Hkv * wl.T * per + q
    assert got["step"] == got["split_kernel"] + wl.B * wl.Hq * 128 * 4


def test_decode_bytes_pruned_int2_with_channel0():
    wl = workloads.by_id(2)
    keep = (1 << 19) - 1  # prune groups 0..18: quantization groups 0, 1, 2 touched, channel 0 kept
    other = 0xFFFFFFFF ^ 1  # every prune group but 0: four quantization groups, channel 0 dropped
    masks = np.array([[keep, other] * (wl.Hkv // 2)] * wl.B, np.uint32)
    lens = np.arange(1, wl.B + 1, dtype=np.int32) * 1000
    got = bench.algorithmic_bytes(wl, masks, lens)
    per_keep = 19 * 4 * 2 // 8 + 3 * 4 + 2 + 128 * 2 // 8 + 4 * 4
    per_other = 31 * 4 * 2 // 8 + 4 * 4 + 128 * 2 // 8 + 4 * 4
    want = sum(int(n) * (wl.Hkv // 2) * (per_keep + per_other) for n in lens) + wl.B * wl.Hq * 128 * 2
    assert got["split_kernel"] == want


def test_append_bytes():
    wl = workloads.by_id(3)
    # per token and kv head: bf16 K and V rows in; 4-bit key codes, 2-bit value
    # codes and their (scale, zero) pairs out
    per = 2 * 128 * 2 + 128 * 4 // 8 + 16 + 128 * 2 // 8 + 16
    assert per == 640
    assert bench.append_algorithmic_bytes(wl) == wl.B * wl.Hkv * wl.T * per


def test_traffic_key_ignores_comments_and_layout():
    code = "int f(int a) { return a + 1; }"
    noisy = "// header\nint f(int a) {  /* add one */\n  return a + 1;  // done\n}\n"
    assert bench._code_tokens(code) == bench._code_tokens(noisy)
    assert bench._code_tokens(code) != bench._code_tokens(code.replace("+ 1", "+ 2"))


def test_recorded_traffic_only_for_its_workload():
    assert bench.recorded_traffic("no_such_workload") is None


def test_decode_bytes_with_bf16_windows():
    wl = workloads.by_id(7)
    masks = np.full((wl.B, wl.Hkv), (1 << 19) - 1, np.uint32)
    lens = np.array([wl.T, 300, 64, 10], np.int32)  # long, inside both windows, the sink alone, shorter than it
    got = bench.algorithmic_bytes(wl, masks, lens)
    per_code = 19 * 4 * 2 // 8 + 3 * 4 + 2 + 128 * 2 // 8 + 4 * 4
    windowed = [64 + 256, 300, 64, 10]  # tokens read as bf16 rows
    split = sum((int(n) - w) * per_code for n, w in zip(lens, windowed)) * wl.Hkv
    assert got["split_kernel"] == split + wl.B * wl.Hq * 128 * 2
    assert got["window"] == sum(windowed) * wl.Hkv * 2 * 128 * 2


def test_decode_bytes_with_rope_buckets():
    # each 2048-token bucket counts with its own mask; the split decode reads
    # one fp32 query row per (bucket holding tokens, query head)
    wl = workloads.by_id(8)
    nb = wl.capacity // wl.bucket
    keep = (1 << 19) - 1
    other = 0xFFFFFFFF ^ 1
    masks = np.zeros((wl.B, nb, wl.Hkv), np.uint32)
    masks[:, 0::2, :] = keep
    masks[:, 1::2, :] = other
    lens = np.array([wl.T, 2048, 2049, 1], np.int32)
    got = bench.algorithmic_bytes(wl, masks, lens)
    per = {keep: 19 * 4 * 2 // 8 + 3 * 4 + 2 + 128 * 2 // 8 + 4 * 4,
           other: 31 * 4 * 2 // 8 + 4 * 4 + 128 * 2 // 8 + 4 * 4}
    want = 0
    rows = 0
    for n in lens:
        used = -(-int(n) // wl.bucket)
        rows += used * wl.Hq
        for k in range(used):
            nk = min(int(n) - k * wl.bucket, wl.bucket)
            want += nk * wl.Hkv * per[keep if k % 2 == 0 else other]
    assert got["split_kernel"] == want + rows * 128 * 4
    assert got["window"] == 0
