"""Runs small appends, selections and decodes (plain, with bf16 windows, and
with bucket-relative RoPE, the caller's pair and windows together)
through whichever library KVQ_LIBRARY selects, and prints a digest of the
cache bytes and outputs and the library's bounds-violation count as JSON.
Used by tests/test_gpu_bounds_checked.py in a child process."""
import hashlib
import json
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from kvq_testlib import to_device  # noqa: E402
from quantized_attention_kvq_b200 import native, synth  # noqa: E402


def main():
    L = native.lib()
    L.kvq_bounds_violations(1)
    h = hashlib.sha256()
    for (B, G, H, T, kb, vb, ch0, keep, sink, recent) in [(2, 4, 2, 1536, 4, 2, 1, 19, 0, 0),
                                                         (2, 8, 1, 1024, 2, 4, 0, 32, 64, 256)]:
        s = synth.Synth(4242 + G, B, G * H, H, 128, T, "bf16")
        cache = native.KVQCache(B, H, T, kb, vb, 1, ch0, sink=sink, recent=recent)
        cache.append(to_device(s.k_full(), "bf16"), to_device(s.v_full(), "bf16"), 0)
        q = to_device(s.q(), "bf16")
        lens = torch.tensor([T, T // 2 + 17][:B], dtype=torch.int32, device="cuda")
        out = cache.decode_select(q, lens, T, keep) if keep < 32 else cache.decode(q, lens, T)
        torch.cuda.synchronize()
        for t in (cache.k_codes, cache.v_codes, out):
            h.update(t.cpu().numpy().tobytes())
    # bucket-relative RoPE with bf16 windows and the caller's pair: appends bucket by bucket
    B, G, H, T, w = 2, 4, 2, 700, 256
    s = synth.Synth(4343, B, G * H, H, 128, T, "bf16")
    tq, tk = synth.dual_pair(4344, H)
    fr = synth.rope_inv_freq(1.0e6)
    cache = native.KVQCache(B, H, 1024, 2, 2, 2, 1, sink=64, recent=200, bucket_tokens=w,
                            rope_inv_freq=torch.from_numpy(fr).cuda(), t_query=torch.from_numpy(tq).cuda(),
                            t_key=torch.from_numpy(tk).cuda())
    k, v = to_device(s.k_full(), "bf16"), to_device(s.v_full(), "bf16")
    for t0 in range(0, T, w):
        cache.append(k[:, :, t0:t0 + w].contiguous(), v[:, :, t0:t0 + w].contiguous(), t0)
    q = to_device(s.q(), "bf16")
    lens = torch.tensor([T, T], dtype=torch.int32, device="cuda")
    out = cache.decode_select(q, lens, 1024, 19)
    torch.cuda.synchronize()
    for t in (cache.k_codes, cache.k_window, cache.v_window, out):
        h.update(t.cpu().numpy().tobytes())
    print(json.dumps({"digest": h.hexdigest(), "violations": int(L.kvq_bounds_violations(0))}))


if __name__ == "__main__":
    main()
