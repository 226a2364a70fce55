"""Five split-decode launches of one workload, for a profiler to capture.

    python -m quantized_attention_kvq_b200.profile_decode <workload id>

Builds the workload's cache with the append kernel (the same seeded inputs as
``bench.py``), runs the channel selection once when the workload prunes, then
launches ``kvq_decode_partials`` five times with a 256 MiB L2 flush before each
launch.  Under ``ncu -k regex:k_decode -s 2 -c 1`` the third launch is the one
captured.  Plain Python + torch for device memory; every step runs in the
library's kernels.
"""
from __future__ import annotations

import math
import sys

import numpy as np
import torch

from quantized_attention_kvq_b200 import native, synth, workloads


def main(wid: int) -> None:
    wl = workloads.by_id(wid)
    if wl.kind != "decode" or wl.bucket or wl.rotate_k == 2 or wl.sink + wl.recent:
        raise SystemExit("profile_decode covers the plain decode workloads")
    dev = torch.device("cuda", 0)
    s = synth.Synth(workloads.BASE_SEED + wl.id, wl.B, wl.Hq, wl.Hkv, wl.d, wl.T, wl.fmt, wl.len_range)

    def up(a):
        if wl.fmt == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    cache = native.KVQCache(wl.B, wl.Hkv, wl.capacity, wl.k_bits, wl.v_bits, wl.rotate_k, wl.keep_ch0, device=dev,
                            rotate_v=wl.rotate_v, v_clip=wl.v_clip)
    for b in range(wl.B):  # one sequence at a time keeps host memory small
        kd = up(np.stack([s.k_slice(b, h) for h in range(wl.Hkv)]))
        vd = up(np.stack([s.v_slice(b, h) for h in range(wl.Hkv)]))
        cache.append_sequence(b, kd, vd, wl.offset)
        torch.cuda.synchronize()
    qd = up(s.q())
    lens = torch.from_numpy(s.lens.astype(np.int32)).to(dev)
    max_len = int(wl.T if wl.len_range is None else wl.capacity)
    mask = cache.select(qd, wl.keep_groups) if wl.keep_groups < 32 else None
    ws = torch.empty(cache.workspace_bytes(wl.Hq, max_len), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(5):
        flush.zero_()
        cache.decode_partials(qd, lens, max_len, mask, 1 / math.sqrt(128), ws)
    torch.cuda.synchronize()
    print("ok")


if __name__ == "__main__":
    main(int(sys.argv[1]))
