"""The decode that selects its own query channels (kvq_decode_attention_select).

It must equal, bit for bit, kvq_select_channels (kvq_select_channels_at with
bucket-relative RoPE) followed by kvq_decode_attention with that mask: the
selection inside the call reads the query rows the decode prepares (each
bucket's embedded and transformed rows, or the pair-transformed rows), which
are the rows the separate selection computes (Dual-QK summary Sec. 3.2 and
App. C.2 for the selection, Sec. 3.4 for the buckets).  The split half
(kvq_decode_partials_select + kvq_decode_combine) must give the same output.
"""
import numpy as np
import pytest
import torch

from kvq_testlib import softmax_scale, to_device
from quantized_attention_kvq_b200 import native, synth

pytestmark = pytest.mark.gpu
D = 128


def inv_freq(base):
    return (base ** (-np.arange(0, D, 2) / D)).astype(np.float32)


@pytest.mark.parametrize("G,H,rot,keep,bucket,lens", [
    (4, 2, 1, 19, 0, [1536, 777]),
    (8, 1, 2, 24, 0, [1300, 1536]),
    (4, 2, 2, 19, 256, [1024, 700]),
    (2, 2, 1, 7, 512, [1024, 1]),
])
def test_selecting_decode_equals_select_then_decode(G, H, rot, keep, bucket, lens):
    B, T = len(lens), 1536 if not bucket else 1024
    s = synth.Synth(900 + G + rot + bucket, B, G * H, H, D, T, "bf16")
    kw = {}
    if rot == 2:
        tq, tk = synth.dual_pair(91 + G, H)
        kw.update(t_query=torch.from_numpy(tq).cuda(), t_key=torch.from_numpy(tk).cuda())
    if bucket:
        kw.update(bucket_tokens=bucket, rope_inv_freq=torch.from_numpy(inv_freq(1.0e6)).cuda())
    cache = native.KVQCache(B, H, T, 4, 2, rot, 1, **kw)
    k, v = to_device(s.k_full(), "bf16"), to_device(s.v_full(), "bf16")
    step = bucket or T
    for t0 in range(0, T, step):  # an append stays inside one bucket
        cache.append(k[:, :, t0:t0 + step].contiguous(), v[:, :, t0:t0 + step].contiguous(), t0)
    q = to_device(s.q(), "bf16")
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    scale = softmax_scale()

    if bucket:
        mask = torch.empty((B, cache.n_buckets, H), dtype=torch.int32, device="cuda")
        cache.select_at(q, lens_d, keep, mask)
    else:
        mask = torch.empty((B, H), dtype=torch.int32, device="cuda")
        cache.select(q, keep, mask)
    ref = cache.decode(q, lens_d, T, mask, scale).cpu().numpy()
    got = cache.decode_select(q, lens_d, T, keep, scale).cpu().numpy()
    np.testing.assert_array_equal(got, ref)

    ws = torch.empty(cache.workspace_bytes(G * H, T), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, G * H, D), dtype=torch.float32, device="cuda")
    cache.decode_partials_select(q, lens_d, T, keep, scale, ws)
    cache.decode_combine(G * H, lens_d, T, out, ws)
    np.testing.assert_array_equal(out.cpu().numpy(), ref)
