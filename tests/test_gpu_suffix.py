"""Stage-2 selective-finetuning forward (gsa_suffix_attn) against the fp64
oracle on identical seeded inputs: every suffix position selects its own
chunks and attends causally to the suffix before it.  Covered: bf16 with
d = 128 (Llama-style heads, k = 16) and fp32 with d = 64 (k > 32), all four
context rules.  Selections follow the decidability rule of the decode tests;
outputs are compared with the oracle's step for the GPU's own selection."""
import dataclasses

import numpy as np
import pytest
import torch

import kv_cache_routing_b200 as gsa
import oracle
import synth
from synth import ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS, DecodeShape, SuffixShape

from gsa_check import check_out, desc_of, dev, host, tdtype, workspace

MODES = [ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS]
SHAPES = {
    "bf16": SuffixShape(DecodeShape(2, 32, 8, 128, 1024, 16, 16, 256, "bf16", n_needles=16)),
    "f32": SuffixShape(DecodeShape(1, 4, 2, 64, 300, 8, 40, 100, "f32", n_needles=40)),
}


def _run(ss, x):
    s = ss.base
    desc = desc_of(s)
    ws = workspace(gsa.gsa_suffix_workspace_size(desc))
    B, S, Hkv, N, k = s.batch, s.tail_len, s.n_kv_heads, s.n_chunks, s.top_k
    idx = torch.full((B, Hkv, S, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, Hkv, S, N), float("nan"), dtype=torch.float32, device="cuda")
    out = torch.empty((B, S, s.n_q_heads, s.head_dim), dtype=tdtype(s.dtype), device="cuda")
    gsa.gsa_suffix_attn(desc, dev(x.q), dev(x.k_gist), dev(x.v_gist), dev(x.k_raw), dev(x.v_raw), dev(x.k_suf),
                        dev(x.v_suf), idx, sc, out, ws)
    torch.cuda.synchronize()
    assert gsa.gsa_workspace_error(ws) == 0
    return idx.cpu().numpy(), sc.cpu().numpy().astype(np.float64), host(out)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", list(SHAPES))
def test_suffix_forward_matches_oracle(name, mode):
    ss = SuffixShape(dataclasses.replace(SHAPES[name].base, mode=mode))
    s = ss.base
    x = synth.suffix_inputs(ss, 9700 + mode)
    idx, sc, out = _run(ss, x)
    s_ex, idx_ex, out_ex = oracle.suffix_attn(x.q, x.k_gist, x.v_gist, x.k_raw, x.v_raw, x.k_suf, x.v_suf,
                                              s.top_k, mode)
    k = s.top_k
    undecidable = []
    for p in range(s.tail_len):
        eps = oracle.score_error_bound(np.ascontiguousarray(x.q[:, p]), x.k_gist)   # [B, Hkv]
        assert np.max(np.abs(sc[:, :, p] - s_ex[:, :, p]) - eps[..., None]) <= 0, f"{name} p={p}: scores"
        gap = oracle.topk_gap(s_ex[:, :, p], k)
        for b in range(s.batch):
            for hk in range(s.n_kv_heads):
                got, want = idx[b, hk, p], idx_ex[b, hk, p]
                if gap[b, hk] > 2 * eps[b, hk]:
                    assert got.tolist() == want.tolist(), f"{name} mode {mode} ({b},{hk},{p}): {got} != {want}"
                else:
                    undecidable.append(p)
                    row = s_ex[b, hk, p]
                    assert np.all(np.diff(got) > 0)
                    rest = np.setdiff1d(np.arange(s.n_chunks), got)
                    assert row[got].min() >= row[rest].max() - 2 * eps[b, hk]
    # outputs: the oracle's step for the GPU's selection where it differs
    for p in sorted(set(undecidable)):
        t = dict(q=np.ascontiguousarray(x.q[:, p]), k_gist=x.k_gist, v_gist=x.v_gist, k_raw=x.k_raw,
                 v_raw=x.v_raw, k_tail=np.ascontiguousarray(x.k_suf[:, :, :p + 1]),
                 v_tail=np.ascontiguousarray(x.v_suf[:, :, :p + 1]))
        out_ex[:, p] = oracle.unfold_attn(t, np.ascontiguousarray(idx[:, :, p]), mode)
    check_out(out, out_ex, s.dtype, f"{name} mode {mode}")
    print(f"{name} mode {mode}: {len(undecidable)} undecidable selections of {s.batch * s.n_kv_heads * s.tail_len}")


@pytest.mark.gpu
def test_suffix_of_one_token_is_the_decode_step():
    """S = 1 through gsa_suffix_attn gives gsa_decode_step's selection, and
    its output within the tolerance (different passes: the decode step runs
    on the tensor-core kernel)."""
    s = dataclasses.replace(synth.WORKLOADS["llama8b_decode"], batch=2, tail_len=1)
    x = synth.decode_inputs(s, 9801)
    d = {k: dev(v) for k, v in x.tensors().items()}
    desc = desc_of(s)
    ws = workspace(max(gsa.gsa_suffix_workspace_size(desc), gsa.gsa_decode_workspace_size(desc)))
    idx_a = torch.empty((2, 8, 1, 16), dtype=torch.int32, device="cuda")
    out_a = torch.empty((2, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
    gsa.gsa_suffix_attn(desc, d["q"], d["k_gist"], d["v_gist"], d["k_raw"], d["v_raw"], d["k_tail"], d["v_tail"],
                        idx_a, None, out_a, ws)
    torch.cuda.synchronize()
    ws.zero_()
    idx_b = torch.empty((2, 8, 16), dtype=torch.int32, device="cuda")
    out_b = torch.empty((2, 32, 128), dtype=torch.bfloat16, device="cuda")
    gsa.gsa_decode_step(desc, d["q"], d["k_gist"], d["v_gist"], d["k_raw"], d["v_raw"], d["k_tail"], d["v_tail"],
                        idx_b, None, out_b, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx_a[:, :, 0].cpu().numpy(), idx_b.cpu().numpy())
    check_out(host(out_a)[:, 0], host(out_b), "bf16", "S = 1")


def test_suffix_descriptor_checks():
    """An empty suffix and too many selection rows are refused on the host."""
    d0 = gsa.decode_desc(1, 4, 2, 64, 16, 4, 2, 0, gsa.GSA_F32)
    assert gsa.gsa_suffix_workspace_size(d0) == 0
    with pytest.raises(gsa.GsaError):
        gsa.gsa_suffix_launch_count(d0)
    big = gsa.decode_desc(8, 32, 8, 128, 64, 16, 4, 1024, gsa.GSA_BF16)   # 65536 rows
    assert gsa.gsa_suffix_workspace_size(big) == 0
    ok = gsa.decode_desc(1, 4, 2, 64, 16, 4, 2, 8, gsa.GSA_F32, UNSELECTED_GISTS)
    assert gsa.gsa_suffix_launch_count(ok) == 3
    with pytest.raises(gsa.GsaError) as e:
        gsa.gsa_suffix_attn(big, *([1 << 20] * 7), None, None, 1 << 20, 1 << 20, stream=0, ws_bytes=1 << 30)
    assert e.value.status == gsa.GSA_ERR_SHAPE
