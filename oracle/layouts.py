"""Oracle block layouts: which key blocks each query block keeps.

Test infrastructure (see the package docstring).  Written independently of the
C++ layout compiler; the two must agree bit for bit.

A layout maps (layout head h, query block i) to a set of key blocks j <= i.
Sources for each family:

* band + global first block -- "Block-Sparse Attention" (ai-model-reference),
  "How It Works": nearby diagonal blocks plus a few farther anchor blocks;
  "Block Sparse Attention in LLMs", section 5B (sliding window + global
  tokens).  window=0 without the global block is BSBR's within-chunk
  (block-diagonal) term ("bsbr", "Solution": ordinary attention inside each
  chunk under the within-chunk causal mask).
* dyadic -- "BF1: A Causal Dyadic Sparse-Attention Retrofit ...", Method and
  section 3.1: the self block (read causally), two local predecessors, the
  first block, and predecessors at dyadic offsets.  Offsets 2^k with k >= 2
  (1 and 2 are already the local predecessors); everything is a set, so
  overlaps are counted once.
* static random -- the same page's "static-random graph 17" control (section
  8; its generator is not published).  Our reading: the diagonal and block 0
  are always kept; row i keeps round-half-up(density * (i+1)) blocks in total
  (at least the mandatory ones, at most i+1), the rest drawn uniformly without
  replacement from {1..i-1} by a partial Fisher-Yates shuffle driven by
  SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014).  One stream per layout head, seeded with
  seed + (h+1)*GOLDEN mod 2^64, rows consumed in order.  density is handled
  as an integer number of parts per million so that no floating-point
  rounding decides a block count.
* explicit -- a caller's block mask M_B ("Block-Sparse Attention", "Math Or
  Compute Schema"), which must be causal at block level (j <= i).
"""
from __future__ import annotations

from collections import deque

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB

BAND_GLOBAL, DYADIC, RANDOM, EXPLICIT = 0, 1, 2, 3


class SplitMix64:
    """SplitMix64 as published: add the golden gamma, then two xor-shift-multiply
    rounds and a final xor-shift."""

    def __init__(self, state: int):
        self.state = state & MASK64

    def next(self) -> int:
        self.state = (self.state + GOLDEN) & MASK64
        z = self.state
        z = ((z ^ (z >> 30)) * MIX1) & MASK64
        z = ((z ^ (z >> 27)) * MIX2) & MASK64
        return z ^ (z >> 31)


def n_blocks(n: int, B: int) -> int:
    return -(-n // B)


def band_global_row(i: int, window: int, global_first: int) -> set:
    kept = set(range(max(0, i - window), i + 1))
    if global_first:
        kept.add(0)
    return kept


def dyadic_row(i: int, window: int, global_first: int, kmin: int) -> set:
    kept = band_global_row(i, window, global_first)
    k = kmin
    while i - (1 << k) >= 0:
        kept.add(i - (1 << k))
        k += 1
    return kept


def density_ppm(density: float) -> int:
    return int(round(density * 1_000_000))


def random_rows(nb: int, ppm: int, seed: int, head: int) -> list:
    """Kept sets of every query block of one layout head (static random)."""
    rng = SplitMix64(seed + (head + 1) * GOLDEN)
    rows = []
    for i in range(nb):
        mandatory = {0} if i == 0 else {0, i}
        target = (ppm * (i + 1) + 500_000) // 1_000_000
        total = min(i + 1, max(len(mandatory), target))
        draws = total - len(mandatory)
        cand = list(range(1, i))          # earlier blocks other than block 0
        for t in range(draws):
            j = t + rng.next() % (len(cand) - t)
            cand[t], cand[j] = cand[j], cand[t]
        rows.append(mandatory | set(cand[:draws]))
    return rows


def kept_sets(kind: int, n: int, B: int, layout_heads: int, window: int = 0,
              global_first: int = 0, dyadic_kmin: int = 2, density: float = 0.0,
              seed: int = 0, mask=None) -> list:
    """``result[h][i]`` = set of key blocks kept by query block i of layout head h."""
    nb = n_blocks(n, B)
    out = []
    for h in range(layout_heads):
        if kind == BAND_GLOBAL:
            out.append([band_global_row(i, window, global_first) for i in range(nb)])
        elif kind == DYADIC:
            out.append([dyadic_row(i, window, global_first, dyadic_kmin) for i in range(nb)])
        elif kind == RANDOM:
            out.append(random_rows(nb, density_ppm(density), seed, h))
        elif kind == EXPLICIT:
            rows = []
            for i in range(nb):
                row = set()
                for j in range(nb):
                    if mask[h][i][j]:
                        if j > i:
                            raise ValueError("explicit block mask is not causal")
                        row.add(j)
                rows.append(row)
            out.append(rows)
        else:
            raise ValueError(f"unknown pattern kind {kind}")
    return out


def kept_sets_for(workload) -> list:
    p = workload.pattern
    return kept_sets(p.kind, workload.n, workload.B, workload.layout_heads,
                     p.window, p.global_first, p.dyadic_kmin, p.density, p.seed)


def to_csr(sets: list):
    """Sorted CSR over rows (h, i) in order h-major: (row_ptr, col_idx) lists."""
    row_ptr, col_idx = [0], []
    for per_head in sets:
        for row in per_head:
            col_idx.extend(sorted(row))
            row_ptr.append(len(col_idx))
    return row_ptr, col_idx


def to_csc(sets: list):
    """The transposed layout over columns (h, j) in order h-major: for each key
    block j of layout head h, the query blocks i whose kept set holds j, in
    ascending order.  (col_ptr, row_idx) lists."""
    col_ptr, row_idx = [0], []
    for per_head in sets:
        nb = len(per_head)
        for j in range(nb):
            row_idx.extend(i for i in range(nb) if j in per_head[i])
            col_ptr.append(len(row_idx))
    return col_ptr, row_idx


def block_mask(sets_one_head: list):
    """Dense n_b x n_b 0/1 block mask M_B of one layout head."""
    nb = len(sets_one_head)
    return [[1 if j in sets_one_head[i] else 0 for j in range(nb)] for i in range(nb)]


def kept_token_pairs(sets_one_head: list, n: int, B: int) -> int:
    """Token pairs (t, u) with u <= t and block(u) kept by block(t)."""
    total = 0
    for i, row in enumerate(sets_one_head):
        rows_i = min(n, (i + 1) * B) - i * B
        for j in row:
            if j < i:
                total += rows_i * (min(n, (j + 1) * B) - j * B)
            elif j == i:
                total += rows_i * (rows_i + 1) // 2
    return total


def max_shortest_path(sets_one_head: list) -> int:
    """Largest BFS distance over all (source, reachable later block) pairs.

    Information moves from key block j to query block i in one layer when j is
    kept by i (self loops add nothing); the BF1 page calls the maximum of the
    shortest such path lengths the communication depth.
    """
    nb = len(sets_one_head)
    succ = [[] for _ in range(nb)]
    for i, row in enumerate(sets_one_head):
        for j in row:
            if j != i:
                succ[j].append(i)
    worst = 0
    for src in range(nb):
        dist = {src: 0}
        dq = deque([src])
        while dq:
            x = dq.popleft()
            for y in succ[x]:
                if y not in dist:
                    dist[y] = dist[x] + 1
                    dq.append(y)
        worst = max(worst, max(dist.values()))
    return worst
