"""GPU parity of top-p (nucleus) selection and of variable-size selections.

gsa_topp is compared with the oracle's top-p on the GPU's own fp32 scores
(widened exactly to fp64), so the ranking is the same data on both sides; the
cut depends on a sum of fp32 weights against p, so a row is held to the exact
oracle answer when the oracle's fp64 prefix masses lie clear of p (margin
1e-4), and otherwise to a cut one place either way with the same order.  The
whole top-p decode step is checked the same way for the selection and
against the oracle's attention over the GPU's selection for the output."""
import dataclasses

import numpy as np
import pytest
import torch

import kv_cache_routing_b200 as gsa
import oracle
import synth
from synth import ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS, DecodeShape

from gsa_check import check_out, desc_of, dev, host, tdtype, upload, workspace

pytestmark = pytest.mark.gpu

MARGIN = 1e-4


def _scale(s):
    return s.scale if s.scale > 0 else 1.0 / np.sqrt(s.head_dim)


def check_topp(scores32, p, kmax, scale, idx_gpu, cnt_gpu, label):
    """Rows decided by the fp64 masses must match exactly.  On the others the
    GPU's cut must be valid within the margin: the fp64 prefix mass at its
    cut reaches p - margin and the one before it stays below p + margin (so
    a cut among weights too small to move an fp32 sum is accepted), and the
    set is that prefix of the same order.  Returns the undecided rows."""
    s = scores32.astype(np.float64).reshape(-1, scores32.shape[-1])
    want_idx, want_cnt = oracle.topp(s, p, kmax, scale)
    got_idx = idx_gpu.reshape(-1, kmax)
    got_cnt = cnt_gpu.reshape(-1)
    undecided = 0
    for r in range(s.shape[0]):
        order = np.lexsort((np.arange(s.shape[1]), -s[r]))
        w = np.exp(scale * (s[r] - s[r].max()))
        cum = np.cumsum(w[order]) / w.sum()
        m = int(want_cnt[r])
        clear = (m == kmax or cum[m - 1] >= p + MARGIN) and (m == 1 or cum[m - 2] <= p - MARGIN)
        g = int(got_cnt[r])
        if clear:
            assert g == m, f"{label} row {r}: count {g} != {m}"
            assert got_idx[r].tolist() == want_idx[r].tolist(), f"{label} row {r}"
        else:
            undecided += 1
            assert 1 <= g <= kmax, f"{label} row {r}: count {g}"
            assert g == kmax or cum[g - 1] >= p - MARGIN, f"{label} row {r}: count {g} short of p"
            assert g == 1 or cum[g - 2] <= p + MARGIN, f"{label} row {r}: count {g} past p"
            assert got_idx[r, :g].tolist() == np.sort(order[:g]).tolist(), f"{label} row {r}"
            assert (got_idx[r, g:] == -1).all()
    return undecided


@pytest.mark.parametrize("n,kmax,p,scale", [(2048, 64, 0.3, 0.09), (2048, 64, 0.9, 0.09), (300, 300, 0.5, 1.0),
                                            (4096, 256, 0.99, 0.02), (100, 8, 0.95, 0.05), (17, 17, 1.0, 0.3)])
def test_topp_kernel(n, kmax, p, scale):
    rng = np.random.default_rng(n + kmax)
    rows = 24
    s = (rng.standard_normal((rows, n)) * 20).astype(np.float32)
    s[::5, 3] = s[::5, 40 % n]                               # exact ties
    sc = torch.from_numpy(s).cuda()
    desc = gsa.decode_desc(rows, 1, 1, 128, n, 16, kmax, 0, gsa.GSA_BF16, scale=scale)
    idx = torch.full((rows, kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    gsa.gsa_topp(desc, p, sc, idx, cnt)
    torch.cuda.synchronize()
    check_topp(s, p, kmax, scale, idx.cpu().numpy(), cnt.cpu().numpy(), f"topp n={n} p={p}")


TOPP_SHAPES = {
    "llama_rows_bf16": DecodeShape(2, 32, 8, 128, 2048, 16, 64, 64, "bf16", ALL_GISTS, n_needles=16),
    "f32_d64": DecodeShape(2, 8, 2, 64, 500, 8, 40, 10, "f32", ALL_GISTS, n_needles=6),
}


@pytest.mark.parametrize("name", sorted(TOPP_SHAPES))
@pytest.mark.parametrize("mode", [ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS])
@pytest.mark.parametrize("p", [0.5, 0.95])
def test_decode_step_topp(name, mode, p):
    s = dataclasses.replace(TOPP_SHAPES[name], mode=mode)
    x = synth.decode_inputs(s, 3100 + int(100 * p))
    t = x.tensors()
    d = upload(x)
    desc = desc_of(s)
    ws = workspace(gsa.gsa_decode_workspace_size(desc))
    kmax = s.top_k
    idx = torch.full((s.batch, s.n_kv_heads, kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((s.batch, s.n_kv_heads), -7, dtype=torch.int32, device="cuda")
    sc = torch.empty((s.batch, s.n_kv_heads, s.n_chunks), dtype=torch.float32, device="cuda")
    out = torch.empty((s.batch, s.n_q_heads, s.head_dim), dtype=tdtype(s.dtype), device="cuda")
    gsa.gsa_decode_step_topp(desc, p, d["q"], d["k_gist"], d["v_gist"], d["k_raw"], d["v_raw"], d["k_tail"],
                             d["v_tail"], idx, cnt, sc, out, ws)
    torch.cuda.synchronize()
    assert gsa.gsa_workspace_error(ws) == 0
    s32 = sc.cpu().numpy()
    eps = oracle.score_error_bound(x.q, x.k_gist)
    assert np.max(np.abs(s32 - oracle.gist_scores(x.q, x.k_gist)) - eps[..., None]) <= 0
    gi = idx.cpu().numpy()
    check_topp(s32, p, kmax, _scale(s), gi, cnt.cpu().numpy(), f"{name} mode {mode}")
    check_out(host(out), oracle.unfold_attn(t, gi.astype(np.int32), mode, s.scale), s.dtype,
              f"{name} mode {mode} p {p}")


@pytest.mark.parametrize("dt,d", [("bf16", 128), ("f32", 64)])
def test_unfold_attn_padded_selection(dt, d):
    """Selections padded with -1 (variable size per row) on both paths."""
    s = DecodeShape(3, 8, 2, d, 400, 8, 12, 9, dt, ALL_GISTS)
    x = synth.decode_inputs(s, 91)
    t = x.tensors()
    dd = upload(x)
    rng = np.random.default_rng(8)
    idx = np.full((3, 2, 12), -1, np.int32)
    for b in range(3):
        for hk in range(2):
            m = int(rng.integers(0, 13))
            idx[b, hk, :m] = np.sort(rng.permutation(400)[:m])
    for mode in (ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS):
        sm = dataclasses.replace(s, mode=mode)
        dm = desc_of(sm)
        ws = workspace(gsa.gsa_decode_workspace_size(dm))
        out = torch.empty((3, 8, d), dtype=tdtype(dt), device="cuda")
        gsa.gsa_unfold_attn(dm, dd["q"], dd["k_gist"], dd["v_gist"], dd["k_raw"], dd["v_raw"], dd["k_tail"],
                            dd["v_tail"], dev(idx), out, None, ws)
        torch.cuda.synchronize()
        assert gsa.gsa_workspace_error(ws) == 0
        check_out(host(out), oracle.unfold_attn(t, idx, mode), dt, f"padded {dt} mode {mode}")
