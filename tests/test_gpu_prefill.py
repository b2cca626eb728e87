"""GPU parity of the gist-causal prefill (tcgen05 kernel) against the oracle."""
import numpy as np
import pytest
import torch

import kv_cache_routing_b200 as gsa
import oracle
import synth
from synth import PrefillShape

from gsa_check import TOL, host, upload

pytestmark = pytest.mark.gpu


def run_prefill(p: PrefillShape, seed: int, label: str, sample: int = 0):
    """Compare every query row (sample=0) or `sample` random rows plus edge rows."""
    x = synth.prefill_inputs(p, seed)
    d = upload(x)
    P = p.positions
    desc = gsa.prefill_desc(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.n_chunks, p.chunk, gsa.GSA_BF16,
                            p.scale)
    out = torch.full((p.batch, p.n_q_heads, P, p.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((p.batch, p.n_q_heads, P), float("nan"), dtype=torch.float32, device="cuda")
    gsa.gsa_gist_prefill(desc, d["q"], d["k"], d["v"], out, lse)
    torch.cuda.synchronize()
    if sample:
        rng = np.random.default_rng(seed)
        rows = [(rng.integers(p.batch), rng.integers(p.n_q_heads), rng.integers(P)) for _ in range(sample)]
        c1 = p.chunk + 1
        for pos in (0, 1, p.chunk - 1, p.chunk, c1, 2 * c1 - 1, P - c1, P - 2, P - 1):   # chunk edges, gists
            rows.append((p.batch - 1, p.n_q_heads - 1, pos))
        rows = np.array(rows, np.int64)
    else:
        rows = np.array([(b, h, t) for b in range(p.batch) for h in range(p.n_q_heads) for t in range(P)], np.int64)
    want = oracle.prefill_rows(x.tensors(), p.n_chunks, p.chunk, rows, p.scale)
    got = host(out)[rows[:, 0], rows[:, 1], rows[:, 2]]
    err = np.max(np.abs(got - want))
    assert err <= TOL["bf16"], f"{label}: max abs err {err:.3e}"
    # lse: the natural-log normaliser, checked through the output's own definition
    assert np.all(np.isfinite(lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]])), f"{label}: lse not finite"
    return err


@pytest.mark.parametrize("shape", [
    PrefillShape(1, 4, 2, 128, 24, 16),      # 4 query tiles, one gist tile
    PrefillShape(1, 2, 1, 128, 3, 2),        # the slide-7 case, three chunks of two
    PrefillShape(1, 2, 2, 128, 1, 16),       # single chunk: plain causal
    PrefillShape(2, 4, 1, 128, 40, 1),       # c = 1: 64 chunks per query tile
    PrefillShape(1, 2, 1, 128, 5, 127),      # c = 127: one chunk per tile
    PrefillShape(1, 4, 2, 128, 300, 16),     # three gist tiles for the last query tiles
    PrefillShape(1, 8, 2, 128, 700, 7),      # ragged last tile, six gist tiles
    PrefillShape(1, 6, 2, 128, 100, 16),     # G = 3: the last head pair has one head
    PrefillShape(2, 8, 2, 128, 400, 16),     # 464 work items: several per persistent CTA
])
def test_prefill_small_exhaustive(shape):
    run_prefill(shape, 11 + shape.n_chunks, f"prefill N={shape.n_chunks} c={shape.chunk}")


def test_prefill_full_size_sampled():
    name = "gist_prefill"
    run_prefill(synth.WORKLOADS[name], synth.seed_for(name), name, sample=768)


def test_prefill_full_size_exhaustive_with_lse():
    """Every query row of the full-size prefill (2 x 32 heads x 17408
    positions) against the oracle, output and log-normaliser, one head at a
    time.  lse is fp32 from an fp32 logit sum: within 1e-3."""
    name = "gist_prefill"
    p = synth.WORKLOADS[name]
    x = synth.prefill_inputs(p, synth.seed_for(name))
    d = upload(x)
    P = p.positions
    desc = gsa.prefill_desc(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.n_chunks, p.chunk, gsa.GSA_BF16,
                            p.scale)
    out = torch.full((p.batch, p.n_q_heads, P, p.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((p.batch, p.n_q_heads, P), float("nan"), dtype=torch.float32, device="cuda")
    gsa.gsa_gist_prefill(desc, d["q"], d["k"], d["v"], out, lse)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    got_o, got_l = host(out), lse.cpu().numpy().astype(np.float64)
    worst_o = worst_l = 0.0
    t = x.tensors()
    for b in range(p.batch):
        for h in range(p.n_q_heads):
            rows = np.stack([np.full(P, b), np.full(P, h), np.arange(P)], axis=1).astype(np.int64)
            want_o, want_l = oracle.prefill_rows(t, p.n_chunks, p.chunk, rows, p.scale, with_lse=True)
            worst_o = max(worst_o, float(np.max(np.abs(got_o[b, h] - want_o))))
            worst_l = max(worst_l, float(np.max(np.abs(got_l[b, h] - want_l))))
    print(f"{name}: every row, max |out err| {worst_o:.3e}, max |lse err| {worst_l:.3e}")
    assert worst_o <= TOL["bf16"]
    assert worst_l <= 1e-3


def test_prefill_lse_matches_oracle_normaliser():
    """lse[p] = log sum_t exp(scale q.k_t) over the allowed keys: with V = 1 the
    output is 1 everywhere, and lse equals the oracle's log-normaliser."""
    p = PrefillShape(1, 2, 1, 128, 20, 16)
    x = synth.prefill_inputs(p, 99)
    d = upload(x)
    desc = gsa.prefill_desc(1, 2, 1, 128, 20, 16)
    out = torch.empty((1, 2, p.positions, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 2, p.positions), dtype=torch.float32, device="cuda")
    gsa.gsa_gist_prefill(desc, d["q"], d["k"], d["v"], out, lse)
    torch.cuda.synchronize()
    # log-normaliser from the oracle: softmax output with V = e_i one-hots is the
    # weight vector; use the identity lse = log(sum exp(l)) computed by torch on
    # the mask the oracle defines
    q = synth.widen(x.q, "bf16")[0]
    k = synth.widen(x.k, "bf16")[0, 0]
    P = p.positions
    mask = np.array([[oracle.gist_mask(a, t, 16) for t in range(P)] for a in range(P)])
    logits = torch.from_numpy(np.einsum("hpd,td->hpt", q, k) / np.sqrt(128.0))
    logits[:, ~torch.from_numpy(mask)] = -float("inf")
    want = torch.logsumexp(logits, dim=-1).numpy()
    assert np.max(np.abs(lse.cpu().numpy()[0] - want)) < 2e-3
