"""gsa_decode_step_noalloc: the decode step for callers that cannot allocate
device memory (its scratch is a fixed array inside the library).

Collected last on purpose, so that a run stopping at the first failure has
already run every other test.  The GPU test compares it, through the C ABI,
with gsa_decode_step on a caller-provided zero-filled workspace, on two
calls in a row (the second call reuses the array the first one left
behind).  Both run the same plan and the same kernels on the same inputs, so
the selections and the outputs must be bit-identical: any stale partial or
counter left in the shared array would show.  It covers both paths: the
tensor-core step (bf16, d = 128) and the CUDA-core passes (fp32, d = 64)."""
import dataclasses

import numpy as np
import pytest
import torch

import kv_cache_routing_b200 as gsa
import synth

from gsa_check import desc_of, host, tdtype, upload, workspace

STATIC_BYTES = 8 << 20


def test_rejects_workspace_beyond_the_static_array():
    big = gsa.decode_desc(16, 32, 8, 128, 65536, 16, 64, 128, gsa.GSA_BF16)
    assert gsa.gsa_decode_workspace_size(big) > STATIC_BYTES
    with pytest.raises(gsa.GsaError) as e:
        gsa.gsa_decode_step_noalloc(big, *([1 << 20] * 7), None, None, 1 << 21, stream=0)
    assert e.value.status == gsa.GSA_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny_f32", "llama8b_decode"])
def test_noalloc_matches_workspace_entry_point_twice(name):
    s = synth.WORKLOADS[name]
    if s.batch > 4:
        s = dataclasses.replace(s, batch=4)
    desc = desc_of(s)
    assert gsa.gsa_decode_workspace_size(desc) <= STATIC_BYTES
    x = synth.decode_inputs(s, 4242)
    d = upload(x)
    ws = workspace(gsa.gsa_decode_workspace_size(desc))

    def run(noalloc):
        idx = torch.full((s.batch, s.n_kv_heads, s.top_k), -1, dtype=torch.int32, device="cuda")
        out = torch.empty((s.batch, s.n_q_heads, s.head_dim), dtype=tdtype(s.dtype), device="cuda")
        args = (d["q"], d["k_gist"], d["v_gist"], d["k_raw"], d["v_raw"], d["k_tail"], d["v_tail"], idx, None, out)
        if noalloc:
            gsa.gsa_decode_step_noalloc(desc, *args)
        else:
            gsa.gsa_decode_step(desc, *args, ws)
        torch.cuda.synchronize()
        return idx.cpu().numpy(), host(out)

    idx_ref, out_ref = run(False)
    assert gsa.gsa_workspace_error(ws) == 0
    for _ in range(2):
        idx, out = run(True)
        np.testing.assert_array_equal(idx, idx_ref)
        np.testing.assert_array_equal(out, out_ref)
    # the scratch array's error word (read and cleared with the library's others)
    assert gsa.gsa_device_error() == 0
