"""Decode over a paged, multi-document raw cache (gsa_decode_step_paged)
against the fp64 oracle on identical seeded inputs.

The inputs: a pool of documents in scrambled page order, sequences drawn as
runs of documents (so they share pages), each cut to its own chunk count,
with decoy gists past every sequence's end that would win the routing if
they were scored.  Both GPU paths are covered: the tensor-core step (bf16,
d = 128) and the CUDA-core passes (fp32, d = 64), in all four context rules.
"""
import dataclasses

import numpy as np
import pytest
import torch

import kv_cache_routing_b200 as gsa
import oracle
import synth
from synth import ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS, DecodeShape, PagedShape

from gsa_check import check_out, desc_of, dev, host, tdtype, workspace

MODES = [ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS]

# tensor-core path: llama-8B heads, 1000-chunk sequences of 12..80-chunk documents
PAGED_TC = PagedShape(DecodeShape(4, 32, 8, 128, 1000, 16, 16, 64, "bf16", n_needles=16),
                      n_docs=40, doc_min=12, doc_max=80, spare_pages=7)
# CUDA-core path: fp32, d = 64, G = 4, k > 32
PAGED_CC = PagedShape(DecodeShape(3, 8, 2, 64, 700, 8, 40, 32, "f32", n_needles=40),
                      n_docs=25, doc_min=5, doc_max=60, spare_pages=3)


def _upload(x):
    d = {k: dev(v) for k, v in x.tensors().items()}
    d["k_pages"], d["v_pages"] = dev(x.k_pages), dev(x.v_pages)
    d["table"] = torch.from_numpy(x.table).cuda()
    d["nch"] = torch.from_numpy(x.seq_chunks).cuda()
    return d


def _gpu_paged(s, x, d, ws=None, with_nch=True):
    desc = desc_of(s)
    if ws is None:
        ws = workspace(gsa.gsa_decode_workspace_size(desc))
    B, Hkv, N, k = s.batch, s.n_kv_heads, s.n_chunks, s.top_k
    idx = torch.full((B, Hkv, max(k, 1)), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, Hkv, N), float("nan"), dtype=torch.float32, device="cuda")
    out = torch.empty((B, s.n_q_heads, s.head_dim), dtype=tdtype(s.dtype), device="cuda")
    gsa.gsa_decode_step_paged(desc, d["q"], d["k_gist"], d["v_gist"], d["k_pages"], d["v_pages"],
                              x.k_pages.shape[0], d["table"], d["nch"] if with_nch else None, d["k_tail"],
                              d["v_tail"], idx, sc, out, ws)
    torch.cuda.synchronize()
    return ws, idx[..., :k].cpu().numpy(), sc.cpu().numpy().astype(np.float64), host(out)


def _slice(x, b, n, kr, vr):
    sl = lambda a: np.ascontiguousarray(a[b:b + 1, :, :n])
    return dict(q=np.ascontiguousarray(x.q[b:b + 1]), k_gist=sl(x.k_gist), v_gist=sl(x.v_gist), k_raw=sl(kr),
                v_raw=sl(vr), k_tail=np.ascontiguousarray(x.k_tail[b:b + 1]),
                v_tail=np.ascontiguousarray(x.v_tail[b:b + 1]))


def _check(s, x, idx, sc, out, label):
    """Scores within the fp32 bound (-inf past each sequence's end); the
    selection exact where decidable, else a valid top-k, padded with -1 past
    a short sequence's chunks; the output against the oracle's attention over
    the GPU's own selection, sequence by sequence (one-sequence problems with
    N = nb: the pins show that this is the paged problem)."""
    s_ex, idx_ex, out_ex = oracle.decode_paged(x.tensors(), x.k_pages, x.v_pages, x.table, s.top_k, s.mode,
                                               s.scale, seq_chunks=x.seq_chunks)
    eps = oracle.score_error_bound(x.q, x.k_gist)
    kr, vr = x.dense_raw()
    k = s.top_k
    for b in range(s.batch):
        n = int(x.seq_chunks[b])
        kk = min(k, n)
        assert np.all(sc[b, :, n:] == -np.inf), f"{label} b={b}: scores past the end"
        if n:
            assert np.max(np.abs(sc[b, :, :n] - s_ex[b, :, :n]) - eps[b][:, None]) <= 0, f"{label} b={b}: scores"
        for hk in range(s.n_kv_heads):
            g = idx[b, hk]
            assert np.all(g[kk:] == -1), f"{label} ({b},{hk}): padding {g}"
            row = s_ex[b, hk, :n]
            gap = oracle.topk_gap(row[None], kk)[0] if n else np.inf
            if gap > 2 * eps[b, hk]:
                assert g.tolist() == idx_ex[b, hk].tolist(), f"{label} ({b},{hk}): {g} != {idx_ex[b, hk]}"
            else:
                sel = g[:kk]
                assert np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() < n, f"{label} ({b},{hk})"
                rest = np.setdiff1d(np.arange(n), sel)
                if len(rest):
                    assert row[sel].min() >= row[rest].max() - 2 * eps[b, hk], f"{label} ({b},{hk}) not a top-k"
        want = oracle.unfold_attn(_slice(x, b, n, kr, vr), idx[b:b + 1].astype(np.int32), s.mode, s.scale)
        check_out(out[b:b + 1], want, s.dtype, f"{label} b={b}")
    return idx_ex


@pytest.mark.gpu
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("shape", ["tc", "cc"])
def test_paged_decode_matches_oracle(shape, mode):
    ps = PAGED_TC if shape == "tc" else PAGED_CC
    ps = dataclasses.replace(ps, base=dataclasses.replace(ps.base, mode=mode))
    x = synth.paged_inputs(ps, 9100 + mode)
    ws, idx, sc, out = _gpu_paged(ps.base, x, _upload(x))
    assert gsa.gsa_workspace_error(ws) == 0
    _check(ps.base, x, idx, sc, out, f"{shape} mode {mode}")


@pytest.mark.gpu
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("shape", ["tc", "cc"])
def test_paged_short_and_empty_sequences(shape, mode):
    """Chunk counts 0, 1, k - 1, k and N in one batch: a short sequence
    selects all of its chunks and pads with -1; an empty one keeps its tail."""
    ps = PAGED_TC if shape == "tc" else PAGED_CC
    base = dataclasses.replace(ps.base, mode=mode, batch=5)
    ps = dataclasses.replace(ps, base=base)
    k, N = base.top_k, base.n_chunks
    x = synth.paged_inputs(ps, 9200 + mode, seq_chunks=[0, 1, k - 1, k, N])
    ws, idx, sc, out = _gpu_paged(base, x, _upload(x))
    assert gsa.gsa_workspace_error(ws) == 0
    _check(base, x, idx, sc, out, f"{shape} short mode {mode}")
    assert np.all(idx[0] == -1)
    assert np.all(idx[1, :, 0] == 0) and np.all(idx[1, :, 1:] == -1)


@pytest.mark.gpu
@pytest.mark.parametrize("shape", ["tc", "cc"])
def test_paged_identity_table_equals_dense_step(shape):
    """A pool that is the dense cache itself (page b*N + j holds chunk j of
    sequence b) and full-length sequences: the paged step gives the dense
    step's selection and output bit for bit (same kernels, same order)."""
    ps = PAGED_TC if shape == "tc" else PAGED_CC
    s = dataclasses.replace(ps.base, batch=2)
    x = synth.decode_inputs(s, 9300)
    B, Hkv, N, c, d = s.batch, s.n_kv_heads, s.n_chunks, s.chunk, s.head_dim
    pool_k = np.ascontiguousarray(x.k_raw.transpose(0, 2, 1, 3, 4).reshape(B * N, Hkv, c, d))
    pool_v = np.ascontiguousarray(x.v_raw.transpose(0, 2, 1, 3, 4).reshape(B * N, Hkv, c, d))
    dd = {k: dev(v) for k, v in x.tensors().items()}
    table = torch.arange(B * N, dtype=torch.int32, device="cuda").reshape(B, N)
    desc = desc_of(s)
    res = []
    for paged in (False, True):
        ws = workspace(gsa.gsa_decode_workspace_size(desc))
        idx = torch.empty((B, Hkv, s.top_k), dtype=torch.int32, device="cuda")
        out = torch.empty((B, s.n_q_heads, d), dtype=tdtype(s.dtype), device="cuda")
        if paged:
            gsa.gsa_decode_step_paged(desc, dd["q"], dd["k_gist"], dd["v_gist"], dev(pool_k), dev(pool_v), B * N,
                                      table, None, dd["k_tail"], dd["v_tail"], idx, None, out, ws)
        else:
            gsa.gsa_decode_step(desc, dd["q"], dd["k_gist"], dd["v_gist"], dd["k_raw"], dd["v_raw"], dd["k_tail"],
                                dd["v_tail"], idx, None, out, ws)
        torch.cuda.synchronize()
        assert gsa.gsa_workspace_error(ws) == 0
        res.append((idx.cpu().numpy(), host(out)))
    np.testing.assert_array_equal(res[0][0], res[1][0])
    np.testing.assert_array_equal(res[0][1], res[1][1])


@pytest.mark.gpu
@pytest.mark.parametrize("shape", ["tc", "cc"])
def test_page_outside_the_pool_is_flagged_not_faulted(shape):
    """A table entry past the pool (for a chunk that is selected) is clamped
    into the pool and flagged in the workspace error word."""
    ps = PAGED_TC if shape == "tc" else PAGED_CC
    s = dataclasses.replace(ps.base, batch=1, n_chunks=64, top_k=64, mode=SR_ONLY)
    ps = dataclasses.replace(ps, base=s, n_docs=4, doc_min=16, doc_max=20)
    x = synth.paged_inputs(ps, 9400, seq_chunks=[64])
    d = _upload(x)
    d["table"][0, 5] = x.k_pages.shape[0] + 3
    ws, idx, _, out = _gpu_paged(s, x, d)
    assert gsa.gsa_workspace_error(ws) & gsa.GSA_WS_ERR_INDEX
    assert np.all(np.isfinite(out))


def test_paged_argument_checks():
    """Host-side checks (no device work): a pool of no pages, a missing table,
    a chunk-count array with an empty tail, a misaligned table."""
    desc = gsa.decode_desc(1, 4, 1, 64, 8, 4, 2, 0, gsa.GSA_F32, ALL_GISTS)
    p = [1 << 20] * 3
    args = lambda n_pages, table, nch: (desc, *p, 1 << 20, 1 << 20, n_pages, table, nch, None, None, None, None,
                                        1 << 20, 1 << 21)
    for a, want in ((args(0, 1 << 20, None), gsa.GSA_ERR_ARG), (args(4, None, None), gsa.GSA_ERR_ARG),
                    (args(4, 1 << 20, 1 << 20), gsa.GSA_ERR_ARG), (args(4, (1 << 20) + 2, None), gsa.GSA_ERR_ALIGN)):
        with pytest.raises(gsa.GsaError) as e:
            gsa.gsa_decode_step_paged(*a, stream=0, ws_bytes=1 << 30)
        assert e.value.status == want
