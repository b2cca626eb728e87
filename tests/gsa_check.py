"""Helpers shared by the GPU parity tests: device upload, calls through the
C-ABI binding, and the comparison rules against the fp64 oracle.

Comparison rules
  * selected indices: bit-exact on every decidable row, i.e. where the gap
    between the k-th and (k+1)-th exact score exceeds twice the fp32 rounding
    bound of a score; on an undecidable row the GPU set must be a valid top-k
    for some scores within that bound (min over the set >= max over the rest
    minus twice the bound);
  * outputs: max |gpu - oracle| <= 1e-5 for fp32 inputs, 2e-2 for bf16.
"""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_routing_b200 as gsa
import oracle

TOL = {"f32": 1e-5, "bf16": 2e-2}


def dev(a: np.ndarray) -> torch.Tensor:
    """Host array -> device tensor (bf16 bit patterns become torch.bfloat16)."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def dtype_code(dt: str) -> int:
    return gsa.GSA_F32 if dt == "f32" else gsa.GSA_BF16


def tdtype(dt: str):
    return torch.float32 if dt == "f32" else torch.bfloat16


def desc_of(s) -> gsa.DecodeDesc:
    return gsa.decode_desc(s.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, s.n_chunks, s.chunk, s.top_k,
                           s.tail_len, dtype_code(s.dtype), s.mode, s.scale)


def workspace(nbytes: int) -> torch.Tensor:
    """Zero-filled, 256-byte aligned device workspace."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device="cuda")


def upload(x) -> dict:
    return {k: dev(v) for k, v in x.tensors().items()}


def gpu_decode_step(s, d: dict, ws=None):
    desc = desc_of(s)
    if ws is None:
        ws = workspace(gsa.gsa_decode_workspace_size(desc))
    B, Hkv, N, k = s.batch, s.n_kv_heads, s.n_chunks, s.top_k
    idx = torch.full((B, Hkv, max(k, 1)), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, Hkv, max(N, 1)), float("nan"), dtype=torch.float32, device="cuda")
    out = torch.empty((B, s.n_q_heads, s.head_dim), dtype=tdtype(s.dtype), device="cuda")
    gsa.gsa_decode_step(desc, d["q"], d["k_gist"], d["v_gist"], d["k_raw"], d["v_raw"], d["k_tail"], d["v_tail"],
                        idx, sc, out, ws)
    torch.cuda.synchronize()
    assert gsa.gsa_workspace_error(ws) == 0
    return idx[..., :k].cpu().numpy(), sc[..., :N].cpu().numpy().astype(np.float64), host(out)


def check_selection(idx_gpu, scores_exact, eps_row, k, label=""):
    """Decidability rule; returns the number of undecidable rows."""
    rows = scores_exact.reshape(-1, scores_exact.shape[-1])
    want = oracle.topk(rows, k)
    got = idx_gpu.reshape(-1, k)
    gap = oracle.topk_gap(rows, k)
    eps = np.asarray(eps_row).reshape(-1)
    undecidable = 0
    for r in range(rows.shape[0]):
        if gap[r] > 2 * eps[r]:
            assert got[r].tolist() == want[r].tolist(), f"{label} row {r}: {got[r]} != {want[r]}"
        else:
            undecidable += 1
            g = got[r]
            assert len(set(g.tolist())) == k and np.all(np.diff(g) > 0), f"{label} row {r} invalid set"
            rest = np.setdiff1d(np.arange(rows.shape[1]), g)
            if len(rest) and k:
                assert rows[r, g].min() >= rows[r, rest].max() - 2 * eps[r], f"{label} row {r} not a top-k"
    return undecidable


def check_out(out_gpu, out_exact, dt, label=""):
    err = np.max(np.abs(out_gpu - out_exact)) if out_gpu.size else 0.0
    assert err <= TOL[dt], f"{label}: max abs err {err:.3e} > {TOL[dt]}"
    return err
