"""Device-side error reporting, without a GPU fault.

A cross-CTA wait of the one-launch decode step is made to run out: the
row's ticket word in the workspace is preset half the 32-bit counter range
away, so the merging CTA's wrap-aware wait can never see the full count, and
the wait limit is shortened through the diagnostics setter.  The kernel must
finish its launch normally and flag GSA_WS_ERR_TIMEOUT in the workspace
error word; a fresh zero-filled workspace then gives oracle-exact results.
The library's own error words (prefill, workspace-less calls) read 0 after
normal calls."""
import pytest
import torch

import kv_cache_routing_b200 as gsa
import oracle
import synth
from synth import ALL_GISTS, DecodeShape

from gsa_check import check_out, check_selection, desc_of, gpu_decode_step, tdtype, upload, workspace

pytestmark = pytest.mark.gpu

WS_TICKETS = 64          # byte offset of the tickets [2][rows] in a decode workspace (the error word is at 0)


def test_cross_cta_wait_runs_out_and_is_flagged():
    s = DecodeShape(2, 8, 2, 128, 300, 16, 8, 32, "bf16", ALL_GISTS, n_needles=8)
    desc = desc_of(s)
    assert gsa.gsa_decode_launch_count(desc) == 1          # the one-launch tensor-core step
    x = synth.decode_inputs(s, 777)
    d = upload(x)
    ws = workspace(gsa.gsa_decode_workspace_size(desc))
    ws.view(torch.int32)[WS_TICKETS // 4] = -2 ** 31       # row 0's ticket: 0x80000000
    idx = torch.empty((s.batch, s.n_kv_heads, s.top_k), dtype=torch.int32, device="cuda")
    out = torch.empty((s.batch, s.n_q_heads, s.head_dim), dtype=tdtype(s.dtype), device="cuda")
    gsa.gsa_set_wait_limit_ns(20_000_000)                 # 20 ms
    try:
        gsa.gsa_decode_step(desc, d["q"], d["k_gist"], d["v_gist"], d["k_raw"], d["v_raw"], d["k_tail"],
                            d["v_tail"], idx, None, out, ws)
        torch.cuda.synchronize()                           # the launch ends by itself
        flags = gsa.gsa_workspace_error(ws)
    finally:
        gsa.gsa_set_wait_limit_ns(0)
    assert flags & gsa.GSA_WS_ERR_TIMEOUT
    # the merging CTA left the row's counters at zero after giving up
    assert int(ws.view(torch.int32)[WS_TICKETS // 4]) == 0
    # a fresh workspace: exact again
    t = x.tensors()
    s_ex, idx_ex, out_ex = oracle.decode(t, s.top_k, s.mode, s.scale)
    idx2, sc2, out2 = gpu_decode_step(s, d)
    eps = oracle.score_error_bound(x.q, x.k_gist)
    assert check_selection(idx2, s_ex, eps, s.top_k, "after timeout") == 0
    check_out(out2, out_ex, s.dtype, "after timeout")


def test_library_error_words_read_zero_after_normal_calls():
    p = synth.PrefillShape(1, 4, 2, 128, 24, 16)
    x = synth.prefill_inputs(p, 5)
    dd = {k: v for k, v in upload(x).items()}
    desc = gsa.prefill_desc(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.n_chunks, p.chunk, gsa.GSA_BF16)
    out = torch.empty((p.batch, p.n_q_heads, p.positions, p.head_dim), dtype=torch.bfloat16, device="cuda")
    gsa.gsa_gist_prefill(desc, dd["q"], dd["k"], dd["v"], out)
    s = synth.WORKLOADS["tiny_f32"]
    xd = synth.decode_inputs(s, 3)
    dq = upload(xd)
    sc = torch.empty((s.batch, s.n_kv_heads, s.n_chunks), dtype=torch.float32, device="cuda")
    gsa.gsa_score(desc_of(s), dq["q"], dq["k_gist"], sc)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
