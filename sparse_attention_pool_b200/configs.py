"""The five workloads the path is measured and checked on.

Each names a decode or prefill step of CSA (block m = 4, top-k) plus HCA
(block m = 128) over one shared compressed KV head, head_dim 128, indexer
dim 64, inputs N(0, 1) in bf16.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    index: int          # seed = BASE_SEED + index
    mode: str           # "decode" or "prefill"
    B: int
    L: int              # tokens per sequence (max for ragged)
    H: int
    topk: int
    fp8: bool = False
    L_min: int | None = None   # ragged: lengths uniform in [L_min, L]
    d: int = 128
    d_idx: int = 128 // 2
    m_csa: int = 4
    m_hca: int = 128


WORKLOADS = [
    Workload("decode_b1_t4k_h8_k64", 0, "decode", 1, 4096, 8, 64),
    Workload("decode_b16_t64k_h64_k512", 1, "decode", 16, 65536, 64, 512),
    Workload("decode_b4_t1m_h64_k2048", 2, "decode", 4, 1048576, 64, 2048),
    Workload("prefill_b1_t128k_h64_k2048", 3, "prefill", 1, 131072, 64, 2048),
    Workload("ragged_fp8_b32_t64k-256k_h64_k1024", 4, "decode", 32, 262144, 64, 1024, fp8=True, L_min=65536),
]
BY_NAME = {w.name: w for w in WORKLOADS}
