"""The five attention workloads this library is measured and checked on.

Each entry fixes the shapes, the masking, the input distribution and the chunk
schedule. Q, K, V are bf16 ``[B, H, N, d]`` with ``d`` contiguous; outputs are
O fp32 ``[B, Hq, N, d]`` and LSE fp32 ``[B, Hq, N]``.

Schedules:
  * ``chunks``  - KV split into ``kv_chunks`` pieces, each run as a partial
    attention, then merged; also run unchunked.
  * ``single``  - one unchunked pass.
  * ``ring``    - the sequence split into ``n_chunks`` Q/KV chunks; Q chunk ``i``
    visits KV chunk ``(i - s) mod n_chunks`` at ring step ``s`` (Ring Attention,
    "Ring Attention with Blockwise Parallel Transformers", section 3), skipping
    chunks that the causal mask hides entirely; per-chunk partials are merged.
  * ``grid2d``  - a ``grid x grid`` array of (Q chunk, KV chunk) cells (ATTENTION2D,
    section 3), merged per Q chunk in a seeded random order.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    schedule: str
    n_chunks: int = 1          # ring: Q/KV chunks; chunks: KV chunks; grid2d: chunks per axis
    stress: bool = False       # Q*8 and 1% of K rows *16 (frequent running-max rescales)
    seed: int = 0
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def chunk(self) -> int:
        return self.N // self.n_chunks

    @property
    def flops(self) -> float:
        return attention_flops(self.B, self.Hq, self.N, self.N, self.d, self.causal)


def attention_flops(B: int, Hq: int, Nq: int, Nkv: int, d: int, causal: bool) -> float:
    """Nominal forward FLOPs: 2*Nq*Nkv*d for Q.K^T plus the same for P.V, per head;
    halved for a causal square problem (the usual convention)."""
    f = 4.0 * B * Hq * Nq * Nkv * d
    return f / 2.0 if causal else f


CONFIGS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_chunks4", B=1, Hq=2, Hkv=2, N=256, d=64, causal=False,
                 schedule="chunks", n_chunks=4, seed=0,
                 description="B=1 H=2 N=256 d=64 non-causal; KV in 4 chunks of 64, merged; "
                             "also unchunked"),
        Workload("causal_4k", B=2, Hq=16, Hkv=16, N=4096, d=128, causal=True,
                 schedule="single", seed=1,
                 description="B=2 H=16 N=4096 d=128 causal, single pass"),
        Workload("ring_32k", B=1, Hq=32, Hkv=32, N=32768, d=128, causal=True,
                 schedule="ring", n_chunks=8, seed=2,
                 description="B=1 H=32 N=32768 d=128 causal; ring of 8 Q/KV chunks of 4096 "
                             "emulated on one GPU; partials merged"),
        Workload("gqa_128k", B=1, Hq=32, Hkv=8, N=131072, d=128, causal=True,
                 schedule="single", seed=3,
                 description="B=1 Hq=32 Hkv=8 N=131072 d=128 causal GQA, single pass"),
        Workload("grid2d_64k_stress", B=1, Hq=16, Hkv=16, N=65536, d=64, causal=False,
                 schedule="grid2d", n_chunks=4, stress=True, seed=4,
                 description="B=1 H=16 N=65536 d=64 non-causal; 4x4 grid of 16384-chunks; "
                             "Q*8, 1% of K rows *16; merge in seeded random order"),
    ]
}


def get(name: str) -> Workload:
    return CONFIGS[name]
