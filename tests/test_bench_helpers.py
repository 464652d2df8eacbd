"""CPU checks of bench.py's bookkeeping: the headline's algorithmic work comes
from the compiled layout (the kept-pair count the BF1 page's 26.98x reduction
pins), and the ncu traffic figure is reported only while the profile's
recorded kernel hash matches the current kernel source."""
import os
import re

import pytest

import bench
import block_sparse_long_bsa_b200 as bsa


@pytest.fixture(scope="module", autouse=True)
def _lib():
    bsa.load_library()


def test_headline_work_from_the_layout():
    w = bench.WORKLOADS[bench.HEADLINE]
    lay = bsa.Layout.for_workload(w, -1)
    row_ptr, col_idx = lay.csr()
    pairs, flops, compulsory = bench.workload_work(w, row_ptr, col_idx)
    lay.close()
    assert pairs == 318_439_424                      # token pairs of the 32K dyadic route, 16 heads
    assert flops == 4 * w.d * pairs
    # q, o: 16 heads; k, v: 8 heads; bf16; plus the fp32 lse
    assert compulsory == 2 * (2 * 16 + 2 * 8) * 32768 * 128 + 4 * 16 * 32768


def test_traffic_only_while_the_profile_matches_the_source(tmp_path, monkeypatch):
    w = bench.HEADLINE
    src = os.path.join(bench.ROOT, "profiles", f"bsa_fwd_sm100a_{w}.md")
    text = open(src).read()
    sha = re.search(r"kernel_sha256:\s*([0-9a-f]{64})", text).group(1)
    tr = int(re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text).group(1))
    os.makedirs(tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # a profile recorded for the current source gives its traffic
    (tmp_path / "profiles" / f"bsa_fwd_sm100a_{w}.md").write_text(text.replace(sha, bench.kernel_sha()))
    assert bench.profiled_traffic(w) == tr
    # one recorded for another source gives none
    (tmp_path / "profiles" / f"bsa_fwd_sm100a_{w}.md").write_text(text.replace(sha, "0" * 64))
    assert bench.profiled_traffic(w) is None
    # no profile at all gives none
    os.remove(tmp_path / "profiles" / f"bsa_fwd_sm100a_{w}.md")
    assert bench.profiled_traffic(w) is None


def test_kernel_hash_covers_the_device_helpers_and_tensor_maps(tmp_path, monkeypatch):
    """A change to the included device helpers or to the tensor-map encoding
    (box shapes) changes the hash, so a profile taken before it is not reused."""
    import shutil
    copies = []
    for path in bench.KERNEL_SRCS:
        dst = tmp_path / os.path.basename(path)
        shutil.copy(path, dst)
        copies.append(str(dst))
    monkeypatch.setattr(bench, "KERNEL_SRCS", copies)
    base = bench.kernel_sha()
    for c in copies:
        with open(c, "a") as fh:
            fh.write("\n// edited\n")
        changed = bench.kernel_sha()
        assert changed != base, c
        base = changed
