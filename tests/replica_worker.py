"""One rank of the replica bench glue, run under torchrun with the gloo
backend on CPU by test_replicas.py (not collected by pytest itself).

Each rank checks the host-side pieces bench.py uses on N GPUs: a process
group from the torchrun environment, barriers, a seed of its own, the step
time as the max over ranks and the whole-job throughput; rank 0 prints what
it saw as one JSON line."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import bench  # noqa: E402
from quantized_attention_kvq_b200 import workloads  # noqa: E402


def main():
    rep = bench.Replicas(backend="gloo", timeout_s=60)
    wl = workloads.by_id(1)
    # every rank a different seed, rank 0 the single-GPU one
    seeds = [None] * rep.world
    rep.dist.all_gather_object(seeds, rep.seed(wl))
    rep.barrier()
    # per-rank "step times": the slowest rank sets the step
    my_ms = 1.0 + 0.5 * rep.rank
    ms = rep.max(my_ms, torch.device("cpu"))
    value = rep.whole_job(wl.B, ms)
    rep.barrier()
    if rep.rank == 0:
        print(json.dumps({"world": rep.world, "seeds": seeds, "ms": ms, "value": value,
                          "single_seed": workloads.BASE_SEED + wl.id}), flush=True)
    rep.close()


if __name__ == "__main__":
    main()
