"""Host-side arithmetic of bench.py: the work and byte counts that the
roofline figures divide by, and the rule that ties a reported DRAM traffic
figure to the kernel sources it was measured on."""
import os
import shutil
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402


@pytest.mark.parametrize("n_chunks,chunk", [(1, 1), (3, 2), (7, 16), (24, 5), (1024, 16)])
def test_prefill_pairs_match_the_oracle_count(n_chunks, chunk):
    # the oracle's count is itself pinned to brute force over the mask
    assert bench.prefill_pairs(n_chunks, chunk) == oracle.prefill_pair_count(n_chunks, chunk)


@pytest.mark.parametrize("n_chunks,chunk", [(1, 1), (3, 2), (9, 7)])
def test_prefill_row_pairs_sum_to_the_total_and_match_the_mask(n_chunks, chunk):
    P = n_chunks * (chunk + 1)
    rows = [bench.prefill_row_pairs(p, chunk) for p in range(P)]
    assert sum(rows) == bench.prefill_pairs(n_chunks, chunk)
    for p in range(P):
        assert rows[p] == sum(oracle.gist_mask(p, t, chunk) for t in range(P))


def test_prefill_workload_flop_figure():
    p = synth.WORKLOADS["gist_prefill"]
    pairs = bench.prefill_pairs(p.n_chunks, p.chunk)
    assert pairs == 9_060_864
    assert 4 * p.head_dim * pairs * p.batch * p.n_q_heads == 296_906_391_552


def test_hierarchy_bytes_closed_form():
    h = synth.WORKLOADS["hier_1m"]
    s = h.l1
    row = s.head_dim * 2
    per_row = 2 * h.n_l2 * row + 2 * h.top_k2 * h.group * row + 2 * s.top_k * s.chunk * row + 2 * s.tail_len * row
    assert bench.hier_bytes(h) == s.rows * per_row + 2 * s.batch * s.n_q_heads * row
    assert abs(bench.hier_bytes(h) / 1e6 - 18.37) < 0.01


def test_decode_bytes_llama_shape():
    assert bench.algorithmic_bytes(synth.WORKLOADS["llama8b_decode"]) == 77_725_696


def test_traffic_is_reported_only_for_the_sources_it_was_measured_on(tmp_path, monkeypatch):
    # a copy of the repository layout bench.py reads: kernel sources + profiles
    csrc = tmp_path / "kv_cache_routing_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.KERNEL_SOURCES:
        shutil.copy(os.path.join(ROOT, "kv_cache_routing_b200", "csrc", f), csrc / f)
    (tmp_path / "profiles").mkdir()
    for f in os.listdir(os.path.join(ROOT, "profiles")):
        shutil.copy(os.path.join(ROOT, "profiles", f), tmp_path / "profiles" / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    t = bench.measured_traffic("llama8b_decode")
    if t is None:
        pytest.skip("the committed decode profile predates the current kernel sources")
    assert t > 0
    assert bench.measured_traffic("no_such_workload") is None
    # any edit of a kernel source voids the figure
    with open(csrc / bench.KERNEL_SOURCES[0], "a") as fh:
        fh.write("\n// edited\n")
    assert bench.measured_traffic("llama8b_decode") is None


def test_tensor_peak_prefers_the_sustained_measurement():
    v, kind = bench.tensor_peak()
    assert v > 0 and "sustained" in kind
