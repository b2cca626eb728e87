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
    # a profile stating these sources' digest (as a fresh capture would)
    import hashlib
    h = hashlib.sha256()
    for f in bench.KERNEL_SOURCES:
        h.update((csrc / f).read_bytes())
    (tmp_path / "profiles" / "fresh_capture.md").write_text(
        "# capture\n\nworkload: llama8b_decode\ndram_bytes_per_step: 80000000\nlaunches_per_step: 2\n"
        f"sources_sha256: {h.hexdigest()}\n")
    assert bench.measured_traffic("llama8b_decode") == 40_000_000    # per launch
    assert bench.traffic_source("llama8b_decode").endswith("fresh_capture.md")
    assert bench.measured_traffic("no_such_workload") is None
    # any edit of a kernel source voids the figure
    with open(csrc / bench.KERNEL_SOURCES[0], "a") as fh:
        fh.write("\n// edited\n")
    assert bench.measured_traffic("llama8b_decode") is None


def test_tensor_peak_prefers_the_sustained_measurement():
    v, kind = bench.tensor_peak()
    assert v > 0 and "sustained" in kind


def test_paged_bytes_full_sequences_equal_the_dense_step():
    ps = synth.WORKLOADS["llama8b_paged"]
    s = ps.base
    assert bench.paged_bytes(ps, np.full(s.batch, s.n_chunks)) == bench.algorithmic_bytes(s)


def test_paged_bytes_are_the_sum_of_one_sequence_problems():
    """A short sequence counts as the dense one-sequence problem with N = nb
    and k = min(k, nb)."""
    import dataclasses
    ps = synth.WORKLOADS["llama8b_paged"]
    s = dataclasses.replace(ps.base, batch=4)
    ps = dataclasses.replace(ps, base=s)
    counts = [0, 5, 700, s.n_chunks]
    want = sum(bench.algorithmic_bytes(dataclasses.replace(s, batch=1, n_chunks=n, top_k=min(s.top_k, n)))
               for n in counts)
    assert bench.paged_bytes(ps, np.array(counts)) == want


def test_levels_bytes_at_depth_two_are_the_two_level_bytes():
    h = synth.WORKLOADS["hier_1m"]
    hl = synth.LevelsShape(h.l1, (h.group,), (h.top_k2,))
    assert hl.counts == [h.l1.n_chunks, h.n_l2]
    assert bench.levels_bytes(hl) == bench.hier_bytes(h)


def test_suffix_flops_by_position():
    """Per selection row (b, hk, p): scores 2 G N d, attention 4 G d over the
    mode's gists + k c raw tokens + the p + 1 suffix tokens."""
    import dataclasses
    base = synth.WORKLOADS["suffix_stage2"].base
    for mode, gists in ((synth.ALL_GISTS, base.n_chunks), (synth.SELECTED_PAIRS, base.top_k),
                        (synth.SR_ONLY, 0), (synth.UNSELECTED_GISTS, base.n_chunks - base.top_k)):
        s = dataclasses.replace(base, tail_len=3, mode=mode)
        G, d = s.group, s.head_dim
        want = s.rows * sum(2 * G * s.n_chunks * d + 4 * G * d * (gists + s.top_k * s.chunk + p + 1)
                            for p in range(3))
        assert bench.suffix_flops(synth.SuffixShape(s)) == want


def test_suffix_workspace_is_the_decode_plan_of_its_selection_rows():
    """On the CUDA-core passes (fp32, d = 64) the suffix forward's workspace
    is the decode workspace of a batch of B * S rows."""
    import kv_cache_routing_b200 as gsa
    for B, S in ((1, 5), (2, 64), (3, 1)):
        d = gsa.decode_desc(B, 8, 2, 64, 300, 8, 12, S, gsa.GSA_F32)
        rows = gsa.decode_desc(B * S, 8, 2, 64, 300, 8, 12, S, gsa.GSA_F32)
        assert gsa.gsa_suffix_workspace_size(d) == gsa.gsa_decode_workspace_size(rows) > 0


def test_levels_workspace_holds_every_level():
    """The workspace holds every level's scores (top level: all its gists;
    lower levels: the children of the selection above), selection and the
    partials of every pass: at least the score and selection regions."""
    import kv_cache_routing_b200 as gsa
    l1 = gsa.decode_desc(2, 8, 2, 128, 4096, 16, 8, 64, gsa.GSA_BF16)
    rows = 2 * 2
    for g, k in (((8,), (16,)), ((8, 8), (16, 4)), ((8, 8, 4), (16, 8, 2))):
        n = [4096]
        for gg in g:
            n.append(-(-n[-1] // gg))
        ks = (8,) + k
        nv = [ks[i + 1] * g[i] for i in range(len(g))] + [n[-1]]
        floor = rows * 4 * (sum(nv) + sum(ks))
        assert gsa.gsa_levels_workspace_size(gsa.levels_desc(l1, g, k)) >= floor
