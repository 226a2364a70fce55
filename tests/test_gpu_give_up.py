"""The split decode's bounded waits: a give-up is reported and the GPU stays usable.

Every wait of the split decode on a shared-memory barrier is bounded (about a
second).  A test hook, kvq_test_withhold_tile, makes the first CTA leave one
tile's ring stage unfilled, so the roles waiting on it give up (no fault, no
trap: a flag that nothing sets).  The decode must then return; the outputs
that read that CTA's partials are NaN, the others are unchanged;
kvq_decode_status reports KVQ_ERR_TIMEOUT; and the next decode on the same
context is correct again with status KVQ_OK.
"""
import math

import numpy as np
import pytest
import torch

from kvq_testlib import to_device
from quantized_attention_kvq_b200 import native, synth

pytestmark = pytest.mark.gpu


def test_wait_give_up_is_reported_and_the_context_stays_usable():
    B, G, H, T = 4, 4, 8, 16384  # 4096 tiles: 28 per CTA, CTA 0 takes unit (0, 0) alone
    s = synth.Synth(777, B, G * H, H, 128, T, "bf16")
    cache = native.KVQCache(B, H, T, 4, 2, 1, 0)
    cache.append(to_device(s.k_full(), "bf16"), to_device(s.v_full(), "bf16"), 0)
    q = to_device(s.q(), "bf16")
    lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    ws = torch.empty(cache.workspace_bytes(G * H, T), dtype=torch.uint8, device="cuda")
    scale = 1 / math.sqrt(128)

    ref = cache.decode(q, lens, T, None, scale, workspace=ws).clone()
    assert cache.decode_status(G * H, ws) == native.KVQ_OK
    assert torch.isfinite(ref).all()

    native.lib().kvq_test_withhold_tile(5)
    out = cache.decode(q, lens, T, None, scale, workspace=ws)
    assert cache.decode_status(G * H, ws) == native.KVQ_ERR_TIMEOUT
    o = out.cpu().numpy().reshape(B, H, G, 128)
    r = ref.cpu().numpy().reshape(B, H, G, 128)
    assert np.isnan(o[0, 0]).all(), "the unit of the CTA that gave up"
    # units whose tiles no CTA range shared with CTA 0 are untouched
    np.testing.assert_array_equal(o[1:], r[1:])
    np.testing.assert_array_equal(o[0, 1:], r[0, 1:])

    # the hook is spent: the next decode is normal, on the same context
    again = cache.decode(q, lens, T, None, scale, workspace=ws)
    assert cache.decode_status(G * H, ws) == native.KVQ_OK
    np.testing.assert_array_equal(again.cpu().numpy(), ref.cpu().numpy())
