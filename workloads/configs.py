"""The five named workloads and a small record type for ad-hoc shapes.

Sizes come from the models the UltraEP page measures on (Qwen3-235B-A22B,
section "Shared redundant slots manage dynamic replicas": 3 x 4096 x 1536 bf16
per expert) and the DeepSeek-V3 shape of the Waterfill page (section
"Experimental setup"), simulated as R expert-parallel ranks on one GPU.
"""
from __future__ import annotations

import dataclasses
from typing import Optional


@dataclasses.dataclass(frozen=True)
class WorkloadConfig:
    name: str
    R: int  # simulated EP ranks
    E: int  # logical experts
    K: int  # routed top-k per token
    T: int  # tokens per rank
    hidden: int  # bf16 row width of a hidden state
    ffn: int  # expert FFN width; one expert holds 3 * hidden * ffn weights
    S: int  # redundant slots per rank
    m: int  # minimum quota of a new replica
    zipf_s: float  # Zipf exponent of the per-layer expert popularity
    seed: int
    layers: int = 1
    shared_expert: bool = False  # one Waterfill shared-expert slot per token
    distinct: bool = True  # top-k experts of a token are distinct
    hot_frac: Optional[float] = None  # stress: share of assignments on one expert
    J: int = 16  # cap candidates of the quota solve
    waterfill_seed: int = 0x5EED_0F_1A7E12
    waterfill_bonus_permille: int = 10
    waterfill_all_ranks: bool = False  # Waterfill candidates: all ranks instead of visited ones
    sampled_rerouting: bool = False  # tokens sample an instance with probability quota/total
    sampling_seed: int = 0x5A3B_1E5EED

    @property
    def N(self) -> int:
        return self.R * self.T

    @property
    def A(self) -> int:
        return self.R * self.T * self.K

    @property
    def expert_elems(self) -> int:
        return 3 * self.hidden * self.ffn

    def replace(self, **kw) -> "WorkloadConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    # 8 experts on EP4 with one redundant slot per rank: the geometry of the
    # memory-management figure on the UltraEP page.
    "tiny": WorkloadConfig(
        name="tiny", R=4, E=8, K=2, T=1024, hidden=256, ffn=512, S=1, m=64,
        zipf_s=1.5, seed=1001,
    ),
    "qwen": WorkloadConfig(
        name="qwen", R=32, E=128, K=8, T=8192, hidden=4096, ffn=1536, S=1, m=1024,
        zipf_s=1.2, seed=2001,
    ),
    "dsv3": WorkloadConfig(
        name="dsv3", R=64, E=256, K=8, T=4096, hidden=7168, ffn=2048, S=2, m=1024,
        zipf_s=1.0, seed=3001, shared_expert=True,
    ),
    "sweep": WorkloadConfig(
        name="sweep", R=32, E=128, K=8, T=4096, hidden=4096, ffn=1536, S=1, m=1024,
        zipf_s=0.0, seed=4001, layers=94,
    ),
    "stress": WorkloadConfig(
        name="stress", R=72, E=256, K=8, T=16384, hidden=7168, ffn=2048, S=2, m=1024,
        zipf_s=1.1, seed=5001, distinct=False, hot_frac=0.4,
    ),
}


def get_config(name: str) -> WorkloadConfig:
    try:
        return CONFIGS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(CONFIGS)}") from None
