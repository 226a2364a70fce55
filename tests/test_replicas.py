"""The multi-GPU path is replicas only: one process per GPU, each on its own
batch, no collective on the data path.  These run its host-side glue (and the
reference arm's rank handling) as two torchrun ranks over gloo on the CPU."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torchrun(script_args, nproc=2, timeout=180):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), *script_args]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


def json_lines(text):
    return [json.loads(l) for l in text.splitlines() if l.startswith("{")]


def test_two_ranks_max_step_time_whole_job_value_and_own_seeds():
    r = torchrun([os.path.join("tests", "replica_worker.py")])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1  # rank 0 alone prints
    got = lines[0]
    assert got["world"] == 2
    assert got["ms"] == 1.5  # the max of the ranks' 1.0 and 1.5 ms
    assert abs(got["value"] - 2 * 8 / 1.5e-3) < 1e-6  # both ranks' 8 sequences per max step
    assert got["seeds"][0] == got["single_seed"] and len(set(got["seeds"])) == 2


def test_reference_arm_runs_on_rank_zero_only():
    r = torchrun(["bench.py", "--impl", "reference", "--gpus", "2", "--workload", "0", "--steps", "2",
                  "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["value"] > 0
    assert lines[0]["e2e"]["h2d_bytes_per_step"] == 0
