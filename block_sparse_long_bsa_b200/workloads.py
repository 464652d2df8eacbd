"""The five synthetic workloads of the block-sparse causal attention forward.

Each entry fixes shapes and the block-layout pattern as plain data; nothing
here computes anything.  ``heads``/``kv_heads`` are folded batch*head counts.

Pattern parameters (kinds as in ``include/bsa.h``):
  band_global : kept(i) = {i-window .. i} (clipped at 0), plus block 0 when
                global_first is set.  window=0, global_first=0 is the BSBR
                within-chunk (block-diagonal) term.
  dyadic      : band_global(window, global_first) plus i - 2^k for k >= kmin.
  random      : diagonal + block 0 + uniformly drawn earlier blocks up to a
                per-row count of round(density*(i+1)), seeded per layout head.
"""
from __future__ import annotations

from dataclasses import dataclass, field, asdict

PATTERN_BAND_GLOBAL = 0
PATTERN_DYADIC = 1
PATTERN_RANDOM = 2
PATTERN_EXPLICIT = 3


@dataclass(frozen=True)
class Pattern:
    kind: int
    window: int = 0
    global_first: int = 0
    dyadic_kmin: int = 2
    density: float = 0.0
    seed: int = 0


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_heads: int          # query heads per sequence
    kv_heads_per_seq: int
    n: int
    d: int
    B: int
    pattern: Pattern
    layout_heads: int     # 1 = one layout shared by all heads, else per head
    description: str = ""

    @property
    def heads(self) -> int:
        return self.batch * self.q_heads

    @property
    def kv_heads(self) -> int:
        return self.batch * self.kv_heads_per_seq

    @property
    def n_blocks(self) -> int:
        return -(-self.n // self.B)

    def as_dict(self):
        d = asdict(self)
        d["heads"] = self.heads
        d["kv_heads"] = self.kv_heads
        return d


LAYOUT_SEED = 17

WORKLOADS = {
    "tiny_band_global": Workload(
        "tiny_band_global", 1, 1, 1, 256, 64, 64,
        Pattern(PATTERN_BAND_GLOBAL, window=1, global_first=1), 1,
        "n=256, d=64, B=64: each query block keeps itself (causal), the "
        "previous block and block 0"),
    "bsbr_block_diagonal": Workload(
        "bsbr_block_diagonal", 2, 8, 8, 4096, 64, 128,
        Pattern(PATTERN_BAND_GLOBAL, window=0, global_first=0), 1,
        "BSBR within-chunk term: batch 2, 8 heads, n=4096, d=64, B=128, "
        "block-diagonal causal"),
    "band_global_32k": Workload(
        "band_global_32k", 1, 32, 32, 32768, 128, 128,
        Pattern(PATTERN_BAND_GLOBAL, window=2, global_first=1), 1,
        "sliding band + global block: 32 heads, n=32768, d=128, B=128, "
        "keeps i, i-1, i-2 and 0"),
    "bf1_dyadic_gqa_32k": Workload(
        "bf1_dyadic_gqa_32k", 1, 16, 8, 32768, 128, 64,
        Pattern(PATTERN_DYADIC, window=2, global_first=1, dyadic_kmin=2), 1,
        "BF1-style dyadic route with GQA: 16 query heads on 8 KV heads, "
        "n=32768, d=128, B=64"),
    "static_random_131k": Workload(
        "static_random_131k", 1, 8, 8, 131072, 128, 128,
        Pattern(PATTERN_RANDOM, density=0.1, seed=LAYOUT_SEED), 8,
        "static random block mask: 8 heads, n=131072, d=128, B=128, ~10% "
        "causal block density, seeded per head"),
}

ORDER = ["tiny_band_global", "bsbr_block_diagonal", "band_global_32k",
         "bf1_dyadic_gqa_32k", "static_random_131k"]

# The single-GPU benchmark headline: the BF1 dyadic route at 32K tokens.
HEADLINE = "bf1_dyadic_gqa_32k"
