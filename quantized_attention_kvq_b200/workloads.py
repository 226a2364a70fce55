"""The synthetic workloads of the quantized-KV decode path.

Each names its shapes, code widths and flags; inputs are drawn by
``synth.Synth`` with seed ``base_seed + id``.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    id: int
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int              # tokens drawn per sequence (= tokens appended)
    capacity: int       # cache capacity in tokens
    offset: int         # first token written by the append
    fmt: str            # "f32" or "bf16" inputs
    k_bits: int
    v_bits: int
    rotate_k: int
    keep_ch0: int
    keep_groups: int    # channel groups of 4 kept by the query-channel pruning (32 = none)
    len_range: tuple | None = None  # per-sequence lengths U[lo, hi] (ragged), else all T
    rotate_v: int = 0   # values rotated before quantization (decode output rotated back)
    v_clip: float = 1.0  # value clipping ratio on each group's min and max
    kind: str = "decode"  # what bench.py times: "decode" or "append"
    sink: int = 0       # bf16 window: the first tokens of each sequence
    recent: int = 0     # bf16 window: the most recent tokens of each sequence
    bucket: int = 0     # bucket-relative RoPE bucket width (0 = none); keys and queries drawn before RoPE
    rope_base: float = 1.0e6  # rotary base of the inverse frequencies (the Qwen3 value)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


WORKLOADS = [
    Workload(0, "tiny_int4", 1, 1, 1, 128, 1024, 1024, 0, "f32", 4, 4, 1, 0, 32),
    Workload(1, "gqa_int4_b8_h32x8_n32k", 8, 32, 8, 128, 32768, 32768, 0, "bf16", 4, 4, 1, 0, 32),
    Workload(2, "dualqk_int2_b4_h32x8_n128k_keep19", 4, 32, 8, 128, 131072, 131072, 0, "bf16", 2, 2, 1, 1, 19),
    Workload(3, "append_b16_h8_t4096_at8192", 16, 8, 8, 128, 4096, 12288, 8192, "bf16", 4, 2, 1, 0, 32,
             kind="append"),
    Workload(4, "ragged_b64_h64x8_n1k16k_keep24", 64, 64, 8, 128, 16384, 16384, 0, "bf16", 4, 2, 1, 1, 24,
             (1024, 16384)),
    # values rotated and clipped at 0.92 before INT2 quantization (Dual-QK App. B.2)
    Workload(5, "dualqk_int2_vrot_clip092_b4_h32x8_n128k_keep19", 4, 32, 8, 128, 131072, 131072, 0, "bf16", 2, 2,
             1, 1, 19, rotate_v=1, v_clip=0.92),
    Workload(6, "append_vrot_clip092_b16_h8_t4096_at8192", 16, 8, 8, 128, 4096, 12288, 8192, "bf16", 4, 2, 1, 0,
             32, rotate_v=1, v_clip=0.92, kind="append"),
    # and the first 64 and most recent 256 tokens kept in bf16 (Dual-QK Sec. 3.3)
    Workload(7, "dualqk_int2_vrot_win64x256_b4_h32x8_n128k_keep19", 4, 32, 8, 128, 131072, 131072, 0, "bf16", 2,
             2, 1, 1, 19, rotate_v=1, v_clip=0.92, sink=64, recent=256),
    # a caller-supplied dual transform pair on queries and keys (Dual-QK Sec. 3.1)
    # with bucket-relative RoPE at w = 2048 (Sec. 3.4)
    Workload(8, "dualqk_int2_pair_bucket2048_vrot_b4_h32x8_n128k_keep19", 4, 32, 8, 128, 131072, 131072, 0, "bf16",
             2, 2, 2, 1, 19, rotate_v=1, v_clip=0.92, bucket=2048),
    # the append through a caller-supplied dual transform pair (Dual-QK Sec. 3.1):
    # each key row taken through its kv head's 128 x 128 key matrix
    Workload(9, "append_pair_b16_h8_t4096_at8192", 16, 8, 8, 128, 4096, 12288, 8192, "bf16", 4, 2, 2, 0, 32,
             kind="append"),
    # the whole Dual-QK recipe: as 8, with the first 64 and the most recent 256
    # tokens kept in bf16 (Sec. 3.3 with Sec. 3.4)
    Workload(10, "dualqk_int2_pair_bucket2048_win64x256_vrot_b4_h32x8_n128k_keep19", 4, 32, 8, 128, 131072, 131072,
             0, "bf16", 2, 2, 2, 1, 19, rotate_v=1, v_clip=0.92, sink=64, recent=256, bucket=2048),
]

BASE_SEED = 0


def by_id(i: int) -> Workload:
    for w in WORKLOADS:
        if w.id == i:
            return w
    raise KeyError(f"no workload {i}")
