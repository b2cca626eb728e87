"""Hierarchy of any depth (gsa_levels_decode) against the fp64 oracle on
identical seeded inputs: three levels on the bf16 / d = 128 shape of the
Llama-style step, four levels in fp32 / d = 64.

Selections are compared level by level with the decidability rule of the
flat step (exact where the k-th and (k+1)-th candidate scores are more than
twice the fp32 score bound apart, else a valid top-k of the candidates the
GPU's own selection one level up yields); the output is compared with the
oracle's step evaluated for the GPU's selections."""
import numpy as np
import pytest
import torch

import kv_cache_routing_b200 as gsa
import oracle
import synth
from synth import DecodeShape, LevelsShape

from gsa_check import check_out, desc_of, dev, host, tdtype, workspace

SHAPES = {
    # 65536 raw tokens, 4096 -> 512 -> 64 gists, k = 8 / 16 / 4
    "l3_bf16": LevelsShape(DecodeShape(2, 32, 8, 128, 4096, 16, 8, 64, "bf16", n_needles=4), (8, 8), (16, 4)),
    # four levels on the tensor-core path: 8192 -> 1024 -> 128 -> 16 gists, k = 8 / 16 / 8 / 4
    "l4_bf16": LevelsShape(DecodeShape(1, 32, 8, 128, 8192, 16, 8, 64, "bf16", n_needles=4), (8, 8, 8), (16, 8, 4)),
    # 2000 chunks, 2000 -> 400 -> 100 -> 25 gists, k = 6 / 12 / 6 / 3
    "l4_f32": LevelsShape(DecodeShape(2, 4, 2, 64, 2000, 8, 6, 16, "f32", n_needles=3), (5, 4, 4), (12, 6, 3)),
}


def _desc(h):
    return gsa.levels_desc(desc_of(h.l1), h.groups, h.top_ks)


def _run_gpu(h, x):
    s = h.l1
    desc = _desc(h)
    ws = workspace(gsa.gsa_levels_workspace_size(desc))
    ks = (s.top_k,) + tuple(h.top_ks)
    idx = [torch.full((s.batch, s.n_kv_heads, k), -7, dtype=torch.int32, device="cuda") for k in ks]
    out = torch.empty((s.batch, s.n_q_heads, s.head_dim), dtype=tdtype(s.dtype), device="cuda")
    kg = [dev(a) for a in x.k_g]
    vg = [dev(a) for a in x.v_g]
    gsa.gsa_levels_decode(desc, dev(x.q), kg, vg, dev(x.k_raw), dev(x.v_raw), dev(x.k_tail), dev(x.v_tail), idx, out,
                          ws)
    torch.cuda.synchronize()
    assert gsa.gsa_workspace_error(ws) == 0
    return [i.cpu().numpy() for i in idx], host(out)


def _check_levels(h, x, idx, label):
    s = h.l1
    n = h.counts
    L = len(n)
    ks = (s.top_k,) + tuple(h.top_ks)
    groups = tuple(h.groups)
    undecidable = 0
    for lv in range(L - 1, -1, -1):
        sc = oracle.gist_scores(x.q, x.k_g[lv])
        eps = oracle.score_error_bound(x.q, x.k_g[lv])
        for b in range(s.batch):
            for hk in range(s.n_kv_heads):
                if lv == L - 1:
                    cand = np.arange(n[lv])
                else:
                    g = groups[lv]
                    par = idx[lv + 1][b, hk]
                    cand = np.array([j for p in par for j in range(p * g, min((p + 1) * g, n[lv]))])
                row = sc[b, hk, cand]
                k = ks[lv]
                got = idx[lv][b, hk]
                order = np.lexsort((cand, -row))
                want = np.sort(cand[order[:k]])
                gap = row[order[k - 1]] - row[order[k]] if k < len(cand) else np.inf
                if gap > 2 * eps[b, hk]:
                    assert got.tolist() == want.tolist(), f"{label} level {lv + 1} ({b},{hk}): {got} != {want}"
                else:
                    undecidable += 1
                    assert np.all(np.diff(got) > 0) and set(got.tolist()) <= set(cand.tolist()), label
                    rest = np.setdiff1d(cand, got)
                    if len(rest):
                        pos = {j: i for i, j in enumerate(cand.tolist())}
                        gs = row[[pos[j] for j in got.tolist()]]
                        rs = row[[pos[j] for j in rest.tolist()]]
                        assert gs.min() >= rs.max() - 2 * eps[b, hk], f"{label} level {lv + 1} not a top-k"
    return undecidable


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(SHAPES))
def test_levels_decode_matches_oracle(name):
    h = SHAPES[name]
    x = synth.levels_inputs(h, 9500 + len(name))
    idx, out = _run_gpu(h, x)
    und = _check_levels(h, x, idx, name)
    ks = (h.l1.top_k,) + tuple(h.top_ks)
    _, want = oracle.hier_levels(x.q, x.k_g, x.v_g, x.k_raw, x.v_raw, x.k_tail, x.v_tail, h.groups, ks,
                                 given=idx)
    check_out(out, want, h.l1.dtype, name)
    print(f"{name}: {und} undecidable (row, level) selections")


@pytest.mark.gpu
def test_levels_depth_two_matches_the_two_level_oracle():
    """Two levels through gsa_levels_decode: the two-level oracle's step."""
    h2 = synth.WORKLOADS["hier_1m"]
    l1 = DecodeShape(1, 32, 8, 128, 8192, 16, 8, 128, "bf16", n_needles=8)
    h = LevelsShape(l1, (16,), (8,))
    x = synth.levels_inputs(h, 9601)
    idx, out = _run_gpu(h, x)
    _check_levels(h, x, idx, "depth 2")
    t = dict(q=x.q, k_g2=x.k_g[1], v_g2=x.v_g[1], k_g1=x.k_g[0], v_g1=x.v_g[0], k_raw=x.k_raw, v_raw=x.v_raw,
             k_tail=x.k_tail, v_tail=x.v_tail)
    _, _, want = oracle.hier_decode(t, 16, 8, 8, given=(idx[1], idx[0]))
    check_out(out, want, "bf16", "depth 2")
    assert h2.group == 16


def test_levels_paths():
    """bf16 with d = 128 and every level's children within one tile: one
    tensor-core launch (up to four levels); otherwise the CUDA-core passes."""
    for name, launches in (("l3_bf16", 1), ("l4_bf16", 1), ("l4_f32", 5)):
        assert gsa.gsa_levels_launch_count(_desc(SHAPES[name])) == launches, name
    five = LevelsShape(DecodeShape(1, 32, 8, 128, 65536, 16, 8, 64, "bf16"), (8, 8, 8, 8), (8, 8, 8, 4))
    assert gsa.gsa_levels_launch_count(_desc(five)) == 6


def test_levels_descriptor_checks():
    """Host-side validation: depth 1 or beyond the maximum, a zero group, a
    top-level k above its gist count, a lower k above the fewest candidates."""
    l1 = gsa.decode_desc(1, 4, 2, 64, 100, 4, 5, 8, gsa.GSA_F32)
    ok = gsa.levels_desc(l1, (10, 5), (4, 2))          # 100 -> 10 -> 2 gists
    assert gsa.gsa_levels_workspace_size(ok) > 0
    assert gsa.gsa_levels_launch_count(ok) == 4
    bad = [gsa.levels_desc(l1, (10, 0), (4, 2)),         # zero group
           gsa.levels_desc(l1, (10, 5), (4, 3)),         # top k 3 > 2 gists
           gsa.levels_desc(l1, (10, 5), (9, 1)),         # 9 > one group of 5 candidates
           gsa.levels_desc(gsa.decode_desc(1, 4, 2, 64, 100, 4, 41, 8, gsa.GSA_F32), (10, 5), (4, 2))]   # k1 41 > 40
    d1 = gsa.levels_desc(l1, (10,), (4,))
    d1.levels = 1
    d9 = gsa.levels_desc(l1, (10,), (4,))
    d9.levels = 9
    for d in bad + [d1, d9]:
        assert gsa.gsa_levels_workspace_size(d) == 0
        with pytest.raises(gsa.GsaError):
            gsa.gsa_levels_launch_count(d)
        with pytest.raises(gsa.GsaError) as e:
            gsa.gsa_levels_decode(d, 1 << 20, [1 << 20] * 3, [1 << 20] * 3, 1 << 20, 1 << 20, 1 << 20, 1 << 20,
                                  None, 1 << 20, 1 << 20, stream=0, ws_bytes=1 << 30)
        assert e.value.status == gsa.GSA_ERR_ARG
    # a valid descriptor with a missing level pointer fails the same way, before any device work
    with pytest.raises(gsa.GsaError) as e:
        gsa.gsa_levels_decode(ok, 1 << 20, [1 << 20, None, 1 << 20], [1 << 20] * 3, 1 << 20, 1 << 20, 1 << 20,
                              1 << 20, None, 1 << 20, 1 << 20, stream=0, ws_bytes=1 << 30)
    assert e.value.status == gsa.GSA_ERR_ARG
