"""Host logic of bench.py that feeds reported numbers: the DRAM-traffic record is used only while
the CUDA sources hash to the capture's, and the CPU-baseline slice covers whole responses and
groups of the first rows.  CPU only."""
import importlib.util
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(m)
    finally:
        sys.argv = argv
    return m


def test_traffic_record_needs_matching_sources_and_scales_by_rows(bench, tmp_path, monkeypatch):
    digest = bench.sources_hash()
    rec = tmp_path / "rec.md"
    H = 1536
    small_T = 5632
    small = 1_000_000_000 + 4 * H * small_T   # W part + hidden in / dH out
    rec.write_text(f"    traffic k_lm_fwd_dh {small} {small_T} {digest}\n"
                   f"    traffic k_lm_dw 99 {small_T} {'0' * 64}\n")
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(rec))
    # the per-row part is exact, the rest scales with the rows (rounds of clusters)
    assert bench.recorded_traffic("k_lm_fwd_dh", small_T, H) == small
    assert bench.recorded_traffic("k_lm_fwd_dh", 2 * small_T, H) == 2_000_000_000 + 4 * H * 2 * small_T
    assert bench.recorded_traffic("k_lm_dw", small_T, H) is None      # not modelled (and other sources)
    assert bench.recorded_traffic("k_gemm_pair", small_T, H) is None  # never captured
    rec.write_text(f"    traffic k_lm_fwd_dh {small} {small_T} {'1' * 64}\n")
    assert bench.recorded_traffic("k_lm_fwd_dh", small_T, H) is None  # captured on other sources


def test_sub_batch_covers_whole_groups_of_the_first_rows(bench):
    from workloads import make_batch, spec_for
    b = make_batch(spec_for("tiny"))
    off = b.resp_offsets.numpy()
    for nrows in (1, int(off[1]), int(off[3]) + 2, b.n_rows):
        new_off, new_goff, rew = bench.sub_batch(b, nrows)
        assert new_off[0] == 0 and new_off[-1] == nrows and np.all(np.diff(new_off) >= 0)
        R = len(new_off) - 1
        assert len(rew) == R and new_goff[0] == 0 and new_goff[-1] == R
        # every kept response starts where it starts in the full batch
        assert np.array_equal(new_off[:-1], off[:R])
