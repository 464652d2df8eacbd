"""Host-side checks of the C ABI (CPU only, no kernel launches).

* the shared library loads and exports every function include/bsa.h declares;
* the host layout compiler matches the oracle's independent builder bit for
  bit (row_ptr, col_idx) on every workload pattern and on edge cases;
* the longest-row-first order is a valid permutation in the stated order;
* invalid specs return the documented status codes.
"""
import os
import re
import subprocess

import numpy as np
import pytest

import block_sparse_long_bsa_b200 as bsa
from block_sparse_long_bsa_b200.workloads import WORKLOADS, ORDER
from oracle import layouts as OL

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_long_bsa_b200 import build
    build.build()
    return bsa.load_library()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "bsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|void|size_t|const char\*)\s+(bsa_\w+)\s*\(", text, flags=re.M)))


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert "bsa_forward" in declared and "bsa_build_layout" in declared
    out = subprocess.run(["nm", "-D", "--defined-only", bsa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (bsa_\w+)", out))
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    assert set(declared) == set(bsa.EXPORTED)


def _csr_from_lib(kind, n, B, L, **kw):
    lay = bsa.Layout(kind, n, B, L, -1, **kw)
    rp, ci = lay.csr()
    order = lay.order()
    lay.close()
    return rp, ci, order


@pytest.mark.parametrize("name", ORDER)
def test_layout_bit_exact_vs_oracle(lib, name):
    w = WORKLOADS[name]
    rp, ci, order = _csr_from_lib(w.pattern.kind, w.n, w.B, w.layout_heads,
                                  window=w.pattern.window, global_first=w.pattern.global_first,
                                  dyadic_kmin=w.pattern.dyadic_kmin, density=w.pattern.density,
                                  seed=w.pattern.seed)
    sets = OL.kept_sets_for(w)
    orp, oci = OL.to_csr(sets)
    np.testing.assert_array_equal(rp, np.array(orp, dtype=np.int32))
    np.testing.assert_array_equal(ci, np.array(oci, dtype=np.int32))
    _check_order(rp, order, w.layout_heads, w.n_blocks)


def _check_order(rp, order, L, nb):
    lens = np.diff(rp).reshape(L, nb)
    order = order.reshape(L, nb)
    for h in range(L):
        assert sorted(order[h].tolist()) == list(range(nb))
        ln = lens[h][order[h]]
        assert np.all(ln[:-1] >= ln[1:])
        # ties in length keep ascending block order
        for a in range(nb - 1):
            if ln[a] == ln[a + 1]:
                assert order[h][a] < order[h][a + 1]


@pytest.mark.parametrize("kind,n,B,L,kw", [
    (OL.BAND_GLOBAL, 1, 64, 1, dict(window=3, global_first=1)),          # single token
    (OL.BAND_GLOBAL, 1000, 64, 2, dict(window=0, global_first=0)),       # ragged, 16 blocks
    (OL.BAND_GLOBAL, 777, 128, 1, dict(window=50, global_first=1)),      # window wider than n
    (OL.DYADIC, 64 * 1000 + 5, 64, 1, dict(window=2, global_first=1, dyadic_kmin=2)),
    (OL.DYADIC, 4096, 64, 3, dict(window=0, global_first=0, dyadic_kmin=0)),
    (OL.RANDOM, 128 * 300, 128, 5, dict(density=0.25, seed=123456789)),
    (OL.RANDOM, 64 * 50, 64, 2, dict(density=0.0, seed=1)),
    (OL.RANDOM, 64 * 50 + 1, 64, 2, dict(density=1.0, seed=2 ** 64 - 1)),
])
def test_layout_edge_cases_bit_exact(lib, kind, n, B, L, kw):
    rp, ci, order = _csr_from_lib(kind, n, B, L, **kw)
    sets = OL.kept_sets(kind, n, B, L, **kw)
    lay = bsa.Layout(kind, n, B, L, -1, **kw)
    cp, ri = bsa.bsa_layout_csc(lay.handle)
    lay.close()
    ocp, ori = OL.to_csc(sets)
    np.testing.assert_array_equal(cp, np.array(ocp, dtype=np.int32))
    np.testing.assert_array_equal(ri, np.array(ori, dtype=np.int32))
    orp, oci = OL.to_csr(sets)
    np.testing.assert_array_equal(rp, np.array(orp, dtype=np.int32))
    np.testing.assert_array_equal(ci, np.array(oci, dtype=np.int32))
    _check_order(rp, order, L, OL.n_blocks(n, B))


def _segments_from_csc(col_ptr, L, nb, seg=16):
    """Columns cut into runs of at most `seg` entries, per layout head, stably
    sorted by run length (longest first)."""
    seg_ptr, out = [0], []
    for h in range(L):
        runs = []
        for j in range(nb):
            c0, c1 = col_ptr[h * nb + j], col_ptr[h * nb + j + 1]
            for e in range(c0, c1, seg):
                runs.append((j, e, min(seg, c1 - e)))
        runs.sort(key=lambda r: -r[2])          # Python's sort is stable
        out.extend(runs)
        seg_ptr.append(len(out))
    return np.array(seg_ptr, dtype=np.int32), np.array(out, dtype=np.int32).reshape(-1, 3)


@pytest.mark.parametrize("kind,n,B,L,kw", [
    (OL.DYADIC, 32768, 64, 1, dict(window=2, global_first=1, dyadic_kmin=2)),
    (OL.BAND_GLOBAL, 32768, 128, 1, dict(window=2, global_first=1)),
    (OL.RANDOM, 128 * 300, 128, 3, dict(density=0.3, seed=7)),
    (OL.BAND_GLOBAL, 1, 64, 1, dict(window=3, global_first=1)),
    (OL.RANDOM, 64 * 50, 64, 2, dict(density=0.0, seed=1)),
])
def test_gradient_work_segments_bit_exact(lib, kind, n, B, L, kw):
    sets = OL.kept_sets(kind, n, B, L, **kw)
    ocp, ori = OL.to_csc(sets)
    want_ptr, want = _segments_from_csc(ocp, L, OL.n_blocks(n, B))
    lay = bsa.Layout(kind, n, B, L, -1, **kw)
    seg_ptr, segs = bsa.bsa_layout_segments(lay.handle)
    lay.close()
    np.testing.assert_array_equal(seg_ptr, want_ptr)
    np.testing.assert_array_equal(segs, want)
    # every (column, query block) entry is covered exactly once
    covered = np.zeros(len(ori), dtype=np.int64)
    for j, e, c in segs:
        assert 1 <= c <= 16
        covered[e:e + c] += 1
    assert np.all(covered == 1)


def test_explicit_mask_bit_exact_and_noncausal(lib):
    nb, B = 20, 64
    rng = np.random.default_rng(0)
    mask = (rng.random((2, nb, nb)) < 0.3) & np.tri(nb, dtype=bool)[None]
    mask[1, 5, :] = False               # an empty row is allowed
    rp, ci, order = _csr_from_lib(OL.EXPLICIT, nb * B, B, 2, mask=mask.astype(np.uint8))
    sets = OL.kept_sets(OL.EXPLICIT, nb * B, B, 2, mask=mask.tolist())
    orp, oci = OL.to_csr(sets)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    bad = mask.copy()
    bad[0, 3, 7] = True
    with pytest.raises(bsa.BsaError) as ei:
        bsa.Layout(OL.EXPLICIT, nb * B, B, 2, -1, mask=bad.astype(np.uint8))
    assert ei.value.status == 4


@pytest.mark.parametrize("args,status", [
    (dict(kind=9, n=128, B=64), 1),
    (dict(kind=0, n=0, B=64), 2),
    (dict(kind=0, n=128, B=0), 2),
    (dict(kind=0, n=128, B=64, layout_heads=0), 2),
    (dict(kind=0, n=128, B=64, window=-1), 1),
    (dict(kind=1, n=128, B=64, dyadic_kmin=-1), 1),
    (dict(kind=2, n=128, B=64, density=1.5), 1),
    (dict(kind=2, n=128, B=64, density=float("nan")), 1),
    (dict(kind=3, n=128, B=64), 1),
])
def test_invalid_specs(lib, args, status):
    kw = dict(args)
    kind, n, B = kw.pop("kind"), kw.pop("n"), kw.pop("B")
    L = kw.pop("layout_heads", 1)
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_build_layout(kind, n, B, L, -1, **kw)
    assert ei.value.status == status
    assert bsa.bsa_last_error()


def test_forward_rejects_host_only_layout(lib):
    lay = bsa.Layout(OL.BAND_GLOBAL, 256, 64, 1, -1, window=1, global_first=1)
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_forward(16, 16, 16, lay.handle, 64, 256, 1, 1, 64, 0.125, 16, 16, 0)
    assert ei.value.status == 1
    lay.close()
    bsa.bsa_free(0)   # NULL is a no-op


C_PROGRAM = r"""
#include <stdio.h>
#include "bsa.h"

int main(void) {
  bsa_pattern spec = {0};
  bsa_layout* lay = NULL;
  const int32_t* row_ptr = NULL;
  const int32_t* col_idx = NULL;
  int rows = 0, nnz = 0, i;
  spec.kind = BSA_PATTERN_BAND_GLOBAL;
  spec.window = 1;
  spec.global_first = 1;
  if (bsa_build_layout(&spec, 256, 64, 1, -1, &lay) != BSA_OK) {
    printf("build: %s\n", bsa_last_error());
    return 1;
  }
  if (bsa_layout_csr(lay, &row_ptr, &col_idx, &rows, &nnz) != BSA_OK) return 2;
  printf("%d %d", rows, nnz);
  for (i = 0; i < nnz; ++i) printf(" %d", (int)col_idx[i]);
  printf("\n");
  /* a host-only layout is refused before anything is launched */
  printf("%d\n", bsa_forward(NULL, NULL, NULL, lay, 64, 256, 1, 1, 64, 0.125f, NULL, NULL, NULL) != BSA_OK);
  bsa_free(lay);
  bsa_free(NULL);
  return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    """include/bsa.h compiles as C99 with warnings as errors, and a C program
    linked against libbsa.so builds a host-only layout: the 4-block band
    layout with block 0 has rows {0}, {0,1}, {0,1,2}, {0,2,3}."""
    import shutil
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(bsa.LIB_PATH)
    inc = os.path.join(os.path.dirname(libdir), "include")
    res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", f"-I{inc}", str(src), "-o", str(exe),
                          f"-L{libdir}", "-lbsa", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.split("\n")[:2] == ["4 9 0 0 1 0 1 2 0 2 3", "1"]


def test_random_specs_bit_exact_sweep(lib):
    """A seeded sweep over every pattern family's parameters (sizes, ragged
    ends, block sizes, layout heads, windows, dyadic exponents, densities,
    seeds and explicit masks): CSR, longest-first order, transposed layout
    and gradient segments all equal the oracle's rules."""
    rng = np.random.default_rng(2024)
    for trial in range(40):
        kind = [OL.BAND_GLOBAL, OL.DYADIC, OL.RANDOM, OL.EXPLICIT][trial % 4]
        B = int(rng.choice([64, 128]))
        n = int(rng.integers(1, 40 * B))
        L = int(rng.integers(1, 4))
        nb = OL.n_blocks(n, B)
        if kind == OL.BAND_GLOBAL:
            kw = dict(window=int(rng.integers(0, 6)), global_first=int(rng.integers(0, 2)))
        elif kind == OL.DYADIC:
            kw = dict(window=int(rng.integers(0, 4)), global_first=int(rng.integers(0, 2)),
                      dyadic_kmin=int(rng.integers(0, 5)))
        elif kind == OL.RANDOM:
            kw = dict(density=float(rng.random()), seed=int(rng.integers(0, 2 ** 63)))
        else:
            mask = (rng.random((L, nb, nb)) < rng.random()) & np.tri(nb, dtype=bool)[None]
            kw = dict(mask=mask.astype(np.uint8))
        okw = dict(kw, mask=kw["mask"].astype(bool).tolist()) if kind == OL.EXPLICIT else kw
        rp, ci, order = _csr_from_lib(kind, n, B, L, **kw)
        sets = OL.kept_sets(kind, n, B, L, **okw)
        orp, oci = OL.to_csr(sets)
        label = f"trial {trial}: kind {kind} n {n} B {B} L {L} {kw if kind != OL.EXPLICIT else ''}"
        np.testing.assert_array_equal(rp, np.array(orp, dtype=np.int32), err_msg=label)
        np.testing.assert_array_equal(ci, np.array(oci, dtype=np.int32), err_msg=label)
        _check_order(rp, order, L, nb)
        lay = bsa.Layout(kind, n, B, L, -1, **kw)
        cp, ri = bsa.bsa_layout_csc(lay.handle)
        seg_ptr, segs = bsa.bsa_layout_segments(lay.handle)
        lay.close()
        ocp, ori = OL.to_csc(sets)
        np.testing.assert_array_equal(cp, np.array(ocp, dtype=np.int32), err_msg=label)
        np.testing.assert_array_equal(ri, np.array(ori, dtype=np.int32), err_msg=label)
        want_ptr, want = _segments_from_csc(ocp, L, nb)
        np.testing.assert_array_equal(seg_ptr, want_ptr, err_msg=label)
        np.testing.assert_array_equal(segs.reshape(-1, 3), want, err_msg=label)

@pytest.mark.parametrize("kind,n,B,L,kw", [
    (OL.DYADIC, 32768, 64, 1, dict(window=2, global_first=1, dyadic_kmin=2)),
    (OL.BAND_GLOBAL, 32768, 128, 1, dict(window=2, global_first=1)),
    (OL.RANDOM, 128 * 300, 128, 3, dict(density=0.3, seed=7)),
    (OL.BAND_GLOBAL, 1000, 64, 2, dict(window=0, global_first=0)),
    (OL.BAND_GLOBAL, 1, 64, 1, dict(window=3, global_first=1)),
    (OL.RANDOM, 64 * 50, 64, 2, dict(density=0.0, seed=1)),
])
def test_work_table_decodes_the_oracle_layout(lib, kind, n, B, L, kw):
    """Each entry of the forward's work table is (query block at that rank of
    the longest-first order, its first CSR entry, its kept-block count, whether
    its last kept block is the diagonal), read off the oracle's CSR; the
    longest-first order is checked on its own above."""
    lay = bsa.Layout(kind, n, B, L, -1, **kw)
    work = bsa.bsa_layout_work(lay.handle)
    order = lay.order()
    lay.close()
    nb = OL.n_blocks(n, B)
    rp, ci = OL.to_csr(OL.kept_sets(kind, n, B, L, **kw))
    assert work.shape == (L * nb, 4)
    for h in range(L):
        for rank in range(nb):
            row = int(order[h * nb + rank])
            r = h * nb + row
            start, length = rp[r], rp[r + 1] - rp[r]
            diag = int(length > 0 and ci[start + length - 1] == row)
            assert work[h * nb + rank].tolist() == [row, start, length, diag], (h, rank)
