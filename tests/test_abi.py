"""CPU-side checks of the C-ABI library: it loads without a GPU, exports every
function the header declares, and rejects bad arguments on the host before
touching the device (no compute calls here)."""
import ctypes
import os
import re

import pytest

import kv_cache_routing_b200 as gsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "gsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gsa_\w+)\s*\(", text)))


def test_library_exports_every_declared_function():
    declared = _header_functions()
    assert set(declared) == set(gsa.EXPORTS)
    L = ctypes.CDLL(gsa.LIB_PATH)
    for name in declared:
        assert hasattr(L, name), name


def test_status_strings():
    for code in range(8):
        assert gsa.status_string(code).startswith("GSA_")
    assert "unknown" in gsa.status_string(99)


def _desc(**kw):
    base = dict(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, n_chunks=100, chunk=16, top_k=4, tail_len=8,
                dtype=gsa.GSA_BF16, mode=gsa.GSA_ALL_GISTS, scale=0.0)
    base.update(kw)
    return gsa.decode_desc(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), gsa.GSA_ERR_SHAPE),
    (dict(n_q_heads=6), gsa.GSA_ERR_SHAPE),
    (dict(n_q_heads=24, n_kv_heads=2), gsa.GSA_ERR_SHAPE),    # G = 12
    (dict(top_k=101), gsa.GSA_ERR_ARG),
    (dict(top_k=-1), gsa.GSA_ERR_ARG),
    (dict(chunk=0), gsa.GSA_ERR_ARG),
    (dict(tail_len=-3), gsa.GSA_ERR_ARG),
    (dict(dtype=7), gsa.GSA_ERR_DTYPE),
    (dict(mode=5), gsa.GSA_ERR_ARG),
    (dict(mode=gsa.GSA_SELECTED_PAIRS, top_k=0, tail_len=0), gsa.GSA_ERR_ARG),   # empty context
    (dict(mode=gsa.GSA_SR_ONLY, top_k=0, tail_len=0), gsa.GSA_ERR_ARG),          # empty context
    (dict(mode=4), gsa.GSA_ERR_ARG),
    (dict(batch=0), gsa.GSA_ERR_SHAPE),
])
def test_descriptor_validation(kw, code):
    d = _desc(**kw)
    assert gsa.gsa_decode_workspace_size(d) == 0
    with pytest.raises(gsa.GsaError) as e:
        gsa.gsa_score(d, 1 << 20, 1 << 21, 1 << 22, stream=0)
    assert e.value.status == code


def test_pointer_and_workspace_checks_happen_before_launch():
    d = _desc()
    n = gsa.gsa_decode_workspace_size(d)
    assert n > 0 and n % 256 == 0
    A = 1 << 20
    ptrs = [A * (i + 1) for i in range(7)]
    with pytest.raises(gsa.GsaError) as e:      # misaligned q
        gsa.gsa_decode_step(d, ptrs[0] + 4, *ptrs[1:], None, None, A * 9, A * 10, stream=0, ws_bytes=n)
    assert e.value.status == gsa.GSA_ERR_ALIGN
    with pytest.raises(gsa.GsaError) as e:      # missing workspace
        gsa.gsa_decode_step(d, *ptrs, None, None, A * 9, None, stream=0, ws_bytes=0)
    assert e.value.status == gsa.GSA_ERR_WORKSPACE
    with pytest.raises(gsa.GsaError) as e:      # workspace too small
        gsa.gsa_decode_step(d, *ptrs, None, None, A * 9, A * 10, stream=0, ws_bytes=n - 256)
    assert e.value.status == gsa.GSA_ERR_WORKSPACE
    with pytest.raises(gsa.GsaError) as e:      # workspace not 256-byte aligned
        gsa.gsa_decode_step(d, *ptrs, None, None, A * 9, A * 10 + 16, stream=0, ws_bytes=n)
    assert e.value.status == gsa.GSA_ERR_WORKSPACE
    with pytest.raises(gsa.GsaError) as e:      # null output
        gsa.gsa_decode_step(d, *ptrs, None, None, None, A * 10, stream=0, ws_bytes=n)
    assert e.value.status == gsa.GSA_ERR_ARG


def test_hier_validation():
    l1 = _desc(n_chunks=160, top_k=8)
    ok = gsa.hier_desc(l1, 10, 16, 2)
    assert gsa.gsa_hier_workspace_size(ok) > 0
    assert gsa.gsa_hier_workspace_size(gsa.hier_desc(l1, 11, 16, 2)) == 0       # n_l2 != ceil(N/group)
    assert gsa.gsa_hier_workspace_size(gsa.hier_desc(l1, 10, 16, 0)) == 0       # k2 = 0
    assert gsa.gsa_hier_workspace_size(gsa.hier_desc(_desc(n_chunks=160, top_k=40), 10, 16, 2)) == 0  # k1 > cands
    assert gsa.gsa_hier_workspace_size(gsa.hier_desc(_desc(n_chunks=160, mode=gsa.GSA_SELECTED_PAIRS), 10, 16, 2)) == 0


def test_prefill_validation():
    with pytest.raises(gsa.GsaError) as e:
        gsa.gsa_gist_prefill(gsa.prefill_desc(1, 8, 2, 128, 4, 16, gsa.GSA_F32), 1 << 20, 1 << 21, 1 << 22,
                             1 << 23, stream=0)
    assert e.value.status == gsa.GSA_ERR_DTYPE
    with pytest.raises(gsa.GsaError) as e:
        gsa.gsa_gist_prefill(gsa.prefill_desc(1, 8, 2, 96, 4, 16), 1 << 20, 1 << 21, 1 << 22, 1 << 23, stream=0)
    assert e.value.status == gsa.GSA_ERR_SHAPE


def test_launch_counts_follow_the_path():
    """One launch on the tensor-core path (bf16, d = 128); the CUDA-core path
    runs a gist pass and an unfold pass (one when there are no gists), and its
    hierarchy three passes; -1 for an invalid descriptor.  Host only."""
    assert gsa.gsa_decode_launch_count(_desc()) == 1
    assert gsa.gsa_decode_launch_count(_desc(dtype=gsa.GSA_F32)) == 2
    assert gsa.gsa_decode_launch_count(_desc(head_dim=64)) == 2
    assert gsa.gsa_decode_launch_count(_desc(head_dim=64, n_chunks=0, top_k=0)) == 1
    # SR-only is one step; the unselected-gists step scores, selects, then attends
    assert gsa.gsa_decode_launch_count(_desc(mode=gsa.GSA_SR_ONLY)) == 1
    assert gsa.gsa_decode_launch_count(_desc(mode=gsa.GSA_UNSELECTED_GISTS)) == 3
    assert gsa.gsa_decode_launch_count(_desc(mode=gsa.GSA_UNSELECTED_GISTS, dtype=gsa.GSA_F32)) == 4
    assert gsa.gsa_decode_launch_count(_desc(mode=gsa.GSA_UNSELECTED_GISTS, top_k=0)) == 1


def test_topp_arguments_are_checked_before_launch():
    d = _desc(top_k=8)
    for p, code in [(0.0, gsa.GSA_ERR_ARG), (1.5, gsa.GSA_ERR_ARG), (float("nan"), gsa.GSA_ERR_ARG)]:
        with pytest.raises(gsa.GsaError) as e:
            gsa.gsa_topp(d, p, 1 << 20, 1 << 21, None, stream=0)
        assert e.value.status == code
    with pytest.raises(gsa.GsaError) as e:
        gsa.gsa_topp(_desc(n_chunks=4000, top_k=3000), 0.5, 1 << 20, 1 << 21, None, stream=0)
    assert e.value.status == gsa.GSA_ERR_SHAPE
    with pytest.raises(gsa.GsaError) as e:
        gsa.gsa_topp(d, 0.5, (1 << 20) + 4, 1 << 21, None, stream=0)
    assert e.value.status == gsa.GSA_ERR_ALIGN
    with pytest.raises(gsa.GsaError):
        gsa.gsa_decode_launch_count(_desc(head_dim=96))
    l1 = _desc(n_chunks=160, top_k=8)
    assert gsa.gsa_hier_launch_count(gsa.hier_desc(l1, 10, 16, 2)) == 1
    assert gsa.gsa_hier_launch_count(gsa.hier_desc(_desc(n_chunks=160, top_k=8, dtype=gsa.GSA_F32), 10, 16, 2)) == 3
    with pytest.raises(gsa.GsaError):
        gsa.gsa_hier_launch_count(gsa.hier_desc(l1, 11, 16, 2))


def test_every_benchmark_decode_workload_takes_the_one_launch_path():
    """The Llama-shaped step, the six compression-ratio sweeps and the
    1M-token hierarchy all fit the tensor-core path (TMEM columns, selection
    size, one children tile and one raw tile), so none silently falls back to
    the CUDA-core passes.  Host only."""
    import synth
    from gsa_check import desc_of
    for name, w in synth.WORKLOADS.items():
        if isinstance(w, synth.DecodeShape) and w.dtype == "bf16" and w.head_dim == 128:
            assert gsa.gsa_decode_launch_count(desc_of(w)) == 1, name
        elif isinstance(w, synth.HierShape):
            hd = gsa.hier_desc(desc_of(w.l1), w.n_l2, w.group, w.top_k2)
            assert gsa.gsa_hier_launch_count(hd) == 1, name
        elif isinstance(w, synth.LevelsShape):
            ld = gsa.levels_desc(desc_of(w.l1), w.groups, w.top_ks)
            assert gsa.gsa_levels_launch_count(ld) == 1, name


def test_host_buffer_step_argument_checks():
    """Missing host buffers, or a host selection without a device one, are
    refused before anything is enqueued."""
    desc = gsa.decode_desc(1, 4, 1, 64, 8, 4, 2, 2, gsa.GSA_F32)
    dev_args = [1 << 20] * 7
    for q_host, idx_out, idx_host, out_host in ((None, None, None, 1 << 20), (1 << 20, None, None, None),
                                                (1 << 20, None, 1 << 20, 1 << 20)):
        with pytest.raises(gsa.GsaError) as e:
            gsa.gsa_decode_step_host(desc, q_host, *dev_args, idx_out, idx_host, 1 << 20, out_host, 1 << 20,
                                     stream=0, ws_bytes=1 << 30)
        assert e.value.status == gsa.GSA_ERR_ARG


def test_levels_path_choice():
    """The any-depth hierarchy takes the one-launch tensor-core step only for
    bf16, d = 128, at most four levels, every children tile within 128 rows
    (and, beyond two levels, groups that are whole TMA runs), k1 c <= 128."""
    bf = lambda N, c, k1: gsa.decode_desc(1, 32, 8, 128, N, c, k1, 64, gsa.GSA_BF16)
    cases = [
        (bf(4096, 16, 8), (8, 8), (16, 4), 1),
        (bf(4096, 16, 8), (16,), (8,), 1),                  # two levels through the same entry point
        (bf(4096, 16, 8), (5, 8), (16, 4), 4),              # a group of 5 is not a whole TMA run
        (bf(4096, 16, 8), (8, 8), (32, 4), 4),              # 32 x 8 = 256 children at level 1
        (bf(4096, 16, 16), (8, 8), (16, 4), 4),             # 16 x 16 = 256 raw rows
        (bf(65536, 16, 8), (8, 8, 8, 8), (8, 8, 8, 4), 6),  # five levels
        (gsa.decode_desc(1, 8, 2, 64, 4096, 16, 8, 64, gsa.GSA_F32), (8, 8), (16, 4), 4),
    ]
    for l1, groups, ks, launches in cases:
        assert gsa.gsa_levels_launch_count(gsa.levels_desc(l1, groups, ks)) == launches, (groups, ks)
