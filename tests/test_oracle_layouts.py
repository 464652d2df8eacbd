"""Pins for the oracle's layout builder (CPU only).

Each check ties the oracle's kept-block sets to something other than the
oracle itself: values printed on the BF1 page, published SplitMix64 outputs,
hand-derived rows and closed-form counts, and structural invariants.
"""
import json
import math
import os

import pytest

from oracle import layouts as L
from block_sparse_long_bsa_b200.workloads import WORKLOADS, ORDER


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as fh:
        return json.load(fh)


def test_splitmix64_reference_outputs(golden_dir):
    g = _load(golden_dir, "splitmix64_vectors.json")
    for vec in g["vectors"]:
        rng = L.SplitMix64(vec["seed"])
        if "outputs_hex" in vec:
            got = [format(rng.next(), "016x") for _ in vec["outputs_hex"]]
            assert got == vec["outputs_hex"]
        else:
            got = [rng.next() for _ in vec["outputs"]]
            assert got == vec["outputs"]


def test_bf1_printed_reduction_and_depth(golden_dir):
    g = _load(golden_dir, "bf1_route_pins.json")
    n, B = g["n"], g["B"]
    sets = L.kept_sets(L.DYADIC, n, B, 1, window=2, global_first=1, dyadic_kmin=2)[0]
    assert len(sets) == 512
    dense_causal = n * (n + 1) // 2
    selected = L.kept_token_pairs(sets, n, B)
    ratio = dense_causal / selected
    assert round(ratio, g["printed_reduction_decimals"]) == g["printed_reduction"]
    assert L.max_shortest_path(sets) == g["printed_max_shortest_path"]


def test_bf1_reduction_rejects_wrong_readings(golden_dir):
    """The printed 26.98x separates token-level causal counting from the
    alternatives: a full B^2 diagonal block or a dropped global block miss it."""
    g = _load(golden_dir, "bf1_route_pins.json")
    n, B = g["n"], g["B"]
    sets = L.kept_sets(L.DYADIC, n, B, 1, window=2, global_first=1, dyadic_kmin=2)[0]
    full_diag = sum(len(r) for r in sets) * B * B
    assert round(n * (n + 1) / 2 / full_diag, 2) != g["printed_reduction"]
    no_global = L.kept_sets(L.DYADIC, n, B, 1, window=2, global_first=0, dyadic_kmin=2)[0]
    assert L.max_shortest_path(no_global) != g["printed_max_shortest_path"]


def test_hand_derived_rows(golden_dir):
    g = _load(golden_dir, "layout_rows.json")
    for case in g["cases"]:
        sets = L.kept_sets(case["kind"], case["n"], case["B"], 1, window=case["window"],
                           global_first=case["global_first"],
                           dyadic_kmin=case.get("dyadic_kmin", 2))[0]
        rows = [sorted(r) for r in sets]
        if "rows" in case:
            assert rows == case["rows"]
        if "first_rows" in case:
            assert rows[:len(case["first_rows"])] == case["first_rows"]
        if "row_511" in case:
            assert rows[511] == case["row_511"]
        if "nnz" in case:
            assert sum(len(r) for r in rows) == case["nnz"]
        if "row_len" in case:
            assert all(len(r) == case["row_len"] for r in rows)


def test_band_closed_form_counts():
    # row i keeps min(i, w) + 1 local blocks, plus block 0 when it lies outside the band
    for nb, w, gf in [(256, 2, 1), (37, 0, 0), (64, 5, 1), (9, 3, 0), (1, 2, 1)]:
        sets = L.kept_sets(L.BAND_GLOBAL, nb * 16, 16, 1, window=w, global_first=gf)[0]
        expect = sum(min(i, w) + 1 + (1 if gf and i > w else 0) for i in range(nb))
        assert sum(len(r) for r in sets) == expect


def test_dyadic_log_growth():
    """Selected pairs grow like n log n at fixed block width (BF1 section 3.2)."""
    B = 64
    ratios = []
    for n in [4096, 8192, 16384, 32768, 65536]:
        sets = L.kept_sets(L.DYADIC, n, B, 1, window=2, global_first=1)[0]
        pairs = L.kept_token_pairs(sets, n, B)
        ratios.append(pairs / (n * B * math.log2(n // B)))
    assert max(ratios) / min(ratios) < 1.5
    # and it is far from quadratic: doubling n should not double pairs/n
    assert ratios[-1] < 2 * ratios[0]


def test_random_layout_invariants():
    w = WORKLOADS["static_random_131k"]
    sets = L.kept_sets_for(w)
    assert len(sets) == 8
    ppm = L.density_ppm(w.pattern.density)
    assert ppm == 100_000
    total_blocks = 0
    for h, rows in enumerate(sets):
        for i, row in enumerate(rows):
            assert 0 in row and i in row
            assert all(0 <= j <= i for j in row)
            target = (ppm * (i + 1) + 500_000) // 1_000_000
            mand = 1 if i == 0 else 2
            assert len(row) == min(i + 1, max(mand, target))
        total_blocks += sum(len(r) for r in rows)
    nb = w.n_blocks
    density = total_blocks / (8 * nb * (nb + 1) / 2)
    assert abs(density - 0.10) < 0.002
    # heads draw from different streams
    assert sets[0] != sets[1]


def test_random_draws_are_uniform():
    """Chi-square check that the drawn earlier blocks are uniform over 1..i-1."""
    nb = 400
    sets = L.kept_sets(L.RANDOM, nb * 8, 8, 64, density=0.3, seed=5)
    i = nb - 1
    counts = [0] * i
    for h in range(64):
        for j in sets[h][i]:
            if j not in (0, i):
                counts[j] += 1
    draws = sum(counts[1:])
    expect = draws / (i - 1)
    chi2 = sum((c - expect) ** 2 / expect for c in counts[1:])
    dof = i - 2
    assert chi2 < dof + 6 * math.sqrt(2 * dof)


def test_explicit_mask_roundtrip_and_noncausal():
    dy = L.kept_sets(L.DYADIC, 40 * 4, 4, 1, window=2, global_first=1)[0]
    mask = [L.block_mask(dy)]
    ex = L.kept_sets(L.EXPLICIT, 40 * 4, 4, 1, mask=mask)[0]
    assert ex == dy
    bad = [[[1 if j <= i + (i == 3) else 0 for j in range(40)] for i in range(40)]]
    with pytest.raises(ValueError):
        L.kept_sets(L.EXPLICIT, 40 * 4, 4, 1, mask=bad)


def test_workload_nnz():
    expect = {"tiny_band_global": 9, "bsbr_block_diagonal": 32, "band_global_32k": 1018,
              "bf1_dyadic_gqa_32k": 5111}
    for name in ORDER:
        w = WORKLOADS[name]
        sets = L.kept_sets_for(w)
        if name in expect:
            assert sum(len(r) for r in sets[0]) == expect[name]
        rp, ci = L.to_csr(sets)
        assert rp[0] == 0 and rp[-1] == len(ci)
        assert len(rp) == w.layout_heads * w.n_blocks + 1


def test_p4_arithmetic(golden_dir):
    g = _load(golden_dir, "p4_arithmetic.json")
    assert round(g["n_32k"] ** 2 / 1e9, 2) == g["scores_32k_billions"]
    assert g["tokens_1m"] // g["block_1m"] == g["blocks_1m"]
    assert g["blocks_1m"] ** 2 // 1000 == g["dense_block_ops_thousands"]  # 952,576 printed as ~952k
    # the dense causal token-pair count the BF1 ratio divides into
    sets = L.kept_sets(L.BAND_GLOBAL, 1024, 64, 1, window=10 ** 6, global_first=1)[0]
    assert L.kept_token_pairs(sets, 1024, 64) == 1024 * 1025 // 2


# ------------------------------------------------------------ transposed layout
def _csc_columns(sets_one_head):
    col_ptr, row_idx = L.to_csc([sets_one_head])
    return [row_idx[col_ptr[j]:col_ptr[j + 1]] for j in range(len(col_ptr) - 1)]


def test_csc_hand_derived_columns(golden_dir):
    """The tiny band workload's columns, read off its rows by hand."""
    g = _load(golden_dir, "layout_rows.json")
    case = g["cases"][0]
    sets = L.kept_sets(case["kind"], case["n"], case["B"], 1, window=case["window"],
                       global_first=case["global_first"])[0]
    assert _csc_columns(sets) == case["cols"]


@pytest.mark.parametrize("nb,window,global_first", [(40, 2, 1), (33, 0, 0), (17, 5, 1), (9, 0, 1)])
def test_csc_band_closed_form(nb, window, global_first):
    """Inverting the band rule: key block j > 0 is kept by the query blocks
    j .. j + window (those inside the sequence); block 0 by the first window + 1
    blocks, or by every block when the global first block is kept."""
    sets = L.kept_sets(L.BAND_GLOBAL, nb * 64, 64, 1, window=window, global_first=global_first)[0]
    cols = _csc_columns(sets)
    for j in range(nb):
        if j == 0 and global_first:
            want = list(range(nb))
        else:
            want = list(range(j, min(nb, j + window + 1)))
        assert cols[j] == want, j


def test_csc_dyadic_closed_form():
    """Inverting BF1's route ("BF1 ...", Method, section 3.1): key block j > 0
    is kept by i = j, j + 1, j + 2 (self and the two local predecessors) and by
    i = j + 2^k for k >= 2; block 0 by every query block."""
    nb = 512
    sets = L.kept_sets(L.DYADIC, nb * 64, 64, 1, window=2, global_first=1, dyadic_kmin=2)[0]
    cols = _csc_columns(sets)
    assert cols[0] == list(range(nb))
    for j in range(1, nb):
        want = {j, j + 1, j + 2} | {j + (1 << k) for k in range(2, 10)}
        assert cols[j] == sorted(i for i in want if i < nb), j


@pytest.mark.parametrize("kind,kw", [
    (L.BAND_GLOBAL, dict(window=3, global_first=1)),
    (L.DYADIC, dict(window=2, global_first=1, dyadic_kmin=2)),
    (L.RANDOM, dict(density=0.3, seed=11)),
])
def test_csc_is_the_transposed_block_mask(kind, kw):
    """Columns of the transposed layout equal the nonzero rows of each column
    of the dense block mask M_B, transposed by numpy, for every layout head."""
    np = pytest.importorskip("numpy")
    sets = L.kept_sets(kind, 37 * 64, 64, 2, **kw)
    col_ptr, row_idx = L.to_csc(sets)
    nb = 37
    for h in range(2):
        mt = np.array(L.block_mask(sets[h]), dtype=np.uint8).T
        for j in range(nb):
            c = h * nb + j
            assert row_idx[col_ptr[c]:col_ptr[c + 1]] == [int(i) for i in np.nonzero(mt[j])[0]]
    assert col_ptr[-1] == sum(len(r) for s in sets for r in s)


def test_csc_pins_catch_a_planted_transpose():
    """A transposed layout built from the rows instead of the columns (the
    mistake a shared misreading would make on both sides) fails the closed form."""
    nb = 64
    sets = L.kept_sets(L.DYADIC, nb * 64, 64, 1, window=2, global_first=1, dyadic_kmin=2)[0]
    wrong = [sorted(sets[j]) for j in range(nb)]          # rows, not columns
    want5 = sorted(i for i in {5, 6, 7} | {5 + (1 << k) for k in range(2, 6)} if i < nb)
    assert wrong[5] != want5 and _csc_columns(sets)[5] == want5
