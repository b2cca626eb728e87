"""GSA oracle — TEST INFRASTRUCTURE ONLY.

Python marshalling around ``gsa_oracle.c`` (plain C, fp64).  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package; the CUDA library and its binding never do.

Inputs are numpy arrays in their storage type (fp32, or bf16 bit patterns in
uint16); the C code widens each element exactly to double.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16, F64 = 0, 1, 2
ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS = 0, 1, 2, 3
_DT = {"f32": F32, "bf16": BF16, "f64": F64}


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` (gcc -O2, IEEE fp64, OpenMP over rows)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    L = ctypes.CDLL(_LIB)
    i, i64, d, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    sig = {
        "oracle_gist_scores": [i, i, i, i, i, i, vp, vp, vp],
        "oracle_topk": [i, i, i, vp, vp],
        "oracle_topk_gap": [i, i, i, vp, vp],
        "oracle_topp": [i, i, i, d, d, vp, vp, vp],
        "oracle_score_error_bound": [i, i, i, i, i, i, vp, vp, vp],
        "oracle_decode": [i, i, i, i, i, i, i, i, i, d, i] + [vp] * 10,
        "oracle_unfold_attn": [i, i, i, i, i, i, i, i, i, d, i] + [vp] * 10,
        "oracle_decode_paged": [i, i, i, i, i, i, i, i, i, d, i] + [vp] * 12,
        "oracle_hier_decode": [i, i, i, i, i, i, i, i, i, i, i, d, i] + [vp] * 12 + [i],
        "oracle_hier_levels": [i, i, i, i, i, i, i, vp, vp, vp, d, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, i],
        "oracle_suffix_attn": [i, i, i, i, i, i, i, i, i, d, i] + [vp] * 10,
        "oracle_gist_mask": [i64, i64, i],
        "oracle_prefill_pair_count": [i, i],
        "oracle_prefill_rows": [i, i, i, i, i, i, d, i, vp, vp, vp, i64, vp, vp, vp],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = None
    L.oracle_gist_mask.restype = i
    L.oracle_prefill_pair_count.restype = i64
    _lib = L
    return L


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _dtcode(a: np.ndarray) -> int:
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(a.dtype)


# --- step 1: routing scores -------------------------------------------------
def gist_scores(q: np.ndarray, k_gist: np.ndarray) -> np.ndarray:
    """q [B,Hq,d], k_gist [B,Hkv,N,d] -> s [B,Hkv,N] fp64."""
    B, Hq, d = q.shape
    _, Hkv, N, _ = k_gist.shape
    s = np.empty((B, Hkv, N), np.float64)
    _load().oracle_gist_scores(B, Hq, Hkv, d, N, _dtcode(q), _p(q), _p(k_gist), _p(s))
    return s


# --- step 2: selection ------------------------------------------------------
def topk(scores: np.ndarray, k: int) -> np.ndarray:
    """scores [..., N] fp64 -> idx [..., k] int32, ascending; ties -> lowest index."""
    s = np.ascontiguousarray(scores, np.float64)
    N = s.shape[-1]
    rows = int(np.prod(s.shape[:-1])) if s.ndim > 1 else 1
    idx = np.empty(s.shape[:-1] + (k,), np.int32)
    _load().oracle_topk(rows, N, k, _p(s), _p(idx))
    return idx


def topp(scores: np.ndarray, p: float, kmax: int, scale: float):
    """Top-p selection of each row of scores [..., N] (fp64): the shortest
    prefix of the top-k order whose softmax(scale * s) mass reaches p, cut at
    kmax.  Returns (idx [..., kmax] int32 ascending then -1, count [...])."""
    s = np.ascontiguousarray(scores, np.float64)
    N = s.shape[-1]
    rows = int(np.prod(s.shape[:-1])) if s.ndim > 1 else 1
    idx = np.empty(s.shape[:-1] + (kmax,), np.int32)
    cnt = np.empty(s.shape[:-1], np.int32)
    _load().oracle_topp(rows, N, kmax, float(p), float(scale), _p(s), _p(idx), _p(cnt))
    return idx, cnt


def topk_gap(scores: np.ndarray, k: int) -> np.ndarray:
    s = np.ascontiguousarray(scores, np.float64)
    N = s.shape[-1]
    rows = int(np.prod(s.shape[:-1])) if s.ndim > 1 else 1
    gap = np.empty(s.shape[:-1], np.float64)
    _load().oracle_topk_gap(rows, N, k, _p(s), _p(gap))
    return gap


def score_error_bound(q: np.ndarray, k_gist: np.ndarray) -> np.ndarray:
    """Per (b, hk): bound on |fp32 score - exact score| for any summation order."""
    B, Hq, d = q.shape
    _, Hkv, N, _ = k_gist.shape
    eps = np.empty((B, Hkv), np.float64)
    _load().oracle_score_error_bound(B, Hq, Hkv, d, N, _dtcode(q), _p(q), _p(k_gist), _p(eps))
    return eps


# --- steps 1-4: decode --------------------------------------------------------
def decode(t: dict, top_k: int, mode: int = ALL_GISTS, scale: float = 0.0):
    """Flat decode step.  t: q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail.
    Returns (scores [B,Hkv,N], idx [B,Hkv,k], out [B,Hq,d]) in fp64 / int32."""
    q, kg = t["q"], t["k_gist"]
    B, Hq, d = q.shape
    _, Hkv, N, c, _ = t["k_raw"].shape
    W = t["k_tail"].shape[2]
    s = np.empty((B, Hkv, N), np.float64)
    idx = np.empty((B, Hkv, top_k), np.int32)
    out = np.empty((B, Hq, d), np.float64)
    _load().oracle_decode(B, Hq, Hkv, d, N, c, top_k, W, mode, scale, _dtcode(q), _p(q), _p(kg),
                          _p(t["v_gist"]), _p(t["k_raw"]), _p(t["v_raw"]), _p(t["k_tail"]),
                          _p(t["v_tail"]), _p(s), _p(idx), _p(out))
    return s, idx, out


def decode_paged(t: dict, k_pages: np.ndarray, v_pages: np.ndarray, table: np.ndarray, top_k: int,
                 mode: int = ALL_GISTS, scale: float = 0.0, seq_chunks=None):
    """Flat decode step over a paged raw cache.  t holds q, k_gist, v_gist
    [B,Hkv,N,d], k_tail, v_tail; chunk j of sequence b is page table[b, j] of
    the pools k_pages / v_pages [pages, Hkv, c, d]; seq_chunks [B] (or None)
    gives the chunks of each sequence.  Returns (scores, idx, out)."""
    q, kg = t["q"], t["k_gist"]
    B, Hq, d = q.shape
    _, Hkv, N, _ = kg.shape
    c = k_pages.shape[2]
    W = t["k_tail"].shape[2]
    table = np.ascontiguousarray(table, np.int32)
    nch = None if seq_chunks is None else np.ascontiguousarray(seq_chunks, np.int32)
    s = np.empty((B, Hkv, N), np.float64)
    idx = np.empty((B, Hkv, top_k), np.int32)
    out = np.empty((B, Hq, d), np.float64)
    _load().oracle_decode_paged(B, Hq, Hkv, d, N, c, top_k, W, mode, scale, _dtcode(q), _p(q), _p(kg),
                                _p(t["v_gist"]), _p(k_pages), _p(v_pages), _p(table), _p(nch),
                                _p(t["k_tail"]), _p(t["v_tail"]), _p(s), _p(idx), _p(out))
    return s, idx, out


def unfold_attn(t: dict, idx: np.ndarray, mode: int = ALL_GISTS, scale: float = 0.0, with_lse: bool = False):
    """Hybrid attention for a given selection; returns out [B,Hq,d] (and lse [B,Hq])."""
    q = t["q"]
    B, Hq, d = q.shape
    _, Hkv, N, c, _ = t["k_raw"].shape
    W = t["k_tail"].shape[2]
    k = idx.shape[-1]
    idx = np.ascontiguousarray(idx, np.int32)
    out = np.empty((B, Hq, d), np.float64)
    lse = np.empty((B, Hq), np.float64)
    _load().oracle_unfold_attn(B, Hq, Hkv, d, N, c, k, W, mode, scale, _dtcode(q), _p(q),
                               _p(t["k_gist"]), _p(t["v_gist"]), _p(t["k_raw"]), _p(t["v_raw"]),
                               _p(t["k_tail"]), _p(t["v_tail"]), _p(idx), _p(out), _p(lse))
    return (out, lse) if with_lse else out


def hier_decode(t: dict, group: int, top_k2: int, top_k1: int, scale: float = 0.0, given=None):
    """t: q, k_g2, v_g2, k_g1, v_g1, k_raw, v_raw, k_tail, v_tail.
    Returns (idx2 [B,Hkv,k2], idx1 [B,Hkv,k1], out [B,Hq,d]).  given=(idx2, idx1)
    evaluates the attention for that selection instead of selecting."""
    q = t["q"]
    B, Hq, d = q.shape
    _, Hkv, N1, c, _ = t["k_raw"].shape
    n_l2 = t["k_g2"].shape[2]
    W = t["k_tail"].shape[2]
    if given is None:
        idx2 = np.empty((B, Hkv, top_k2), np.int32)
        idx1 = np.empty((B, Hkv, top_k1), np.int32)
    else:
        idx2 = np.ascontiguousarray(given[0], np.int32).copy()
        idx1 = np.ascontiguousarray(given[1], np.int32).copy()
    out = np.empty((B, Hq, d), np.float64)
    _load().oracle_hier_decode(B, Hq, Hkv, d, N1, c, top_k1, W, n_l2, group, top_k2, scale,
                               _dtcode(q), _p(q), _p(t["k_g2"]), _p(t["v_g2"]), _p(t["k_g1"]),
                               _p(t["v_g1"]), _p(t["k_raw"]), _p(t["v_raw"]), _p(t["k_tail"]),
                               _p(t["v_tail"]), _p(idx2), _p(idx1), _p(out), 0 if given is None else 1)
    return idx2, idx1, out


def suffix_attn(q, k_gist, v_gist, k_raw, v_raw, k_suf, v_suf, top_k: int, mode: int = ALL_GISTS,
                scale: float = 0.0):
    """Stage-2 forward: q [B,S,Hq,d] (position-major), k_suf / v_suf
    [B,Hkv,S,d].  Returns (scores [B,Hkv,S,N], idx [B,Hkv,S,k], out [B,S,Hq,d])."""
    B, S, Hq, d = q.shape
    _, Hkv, N, c, _ = k_raw.shape
    sc = np.empty((B, Hkv, S, N), np.float64)
    idx = np.empty((B, Hkv, S, top_k), np.int32)
    out = np.empty((B, S, Hq, d), np.float64)
    _load().oracle_suffix_attn(B, Hq, Hkv, d, N, c, top_k, S, mode, scale, _dtcode(q), _p(q), _p(k_gist),
                               _p(v_gist), _p(k_raw), _p(v_raw), _p(k_suf), _p(v_suf), _p(sc), _p(idx), _p(out))
    return sc, idx, out


def hier_levels(q, k_g, v_g, k_raw, v_raw, k_tail, v_tail, groups, top_ks, scale: float = 0.0, given=None):
    """Hierarchy of any depth: k_g / v_g are lists of the gist tensors of
    levels 1..L ([B,Hkv,n_l,d], level 1 one gist per chunk), groups[l-1] the
    level-l gists per level-(l+1) gist (L-1 values), top_ks[l-1] the
    selection size at level l (L values).  Returns ([idx_l], out).  given: a
    list of L selections to evaluate the step for instead of selecting."""
    B, Hq, d = q.shape
    Hkv = k_raw.shape[1]
    c = k_raw.shape[3]
    W = k_tail.shape[2]
    L = len(k_g)
    assert len(v_g) == L and len(groups) == L - 1 and len(top_ks) == L
    n = np.array([g.shape[2] for g in k_g], np.int32)
    grp = np.array(list(groups) + [0], np.int32)
    kk = np.array(top_ks, np.int32)
    if given is None:
        idx = [np.empty((B, Hkv, int(t)), np.int32) for t in top_ks]
    else:
        idx = [np.ascontiguousarray(g, np.int32).copy() for g in given]
    out = np.empty((B, Hq, d), np.float64)
    arr = lambda xs: (ctypes.c_void_p * len(xs))(*[x.ctypes.data for x in xs])
    for x in list(k_g) + list(v_g):
        assert x.flags["C_CONTIGUOUS"]
    _load().oracle_hier_levels(B, Hq, Hkv, d, c, W, L, _p(n), _p(grp), _p(kk), scale, _dtcode(q), _p(q),
                               arr(k_g), arr(v_g), _p(k_raw), _p(v_raw), _p(k_tail), _p(v_tail), arr(idx),
                               _p(out), 0 if given is None else 1)
    return idx, out


# --- prefill ------------------------------------------------------------------
def gist_mask(p: int, t: int, chunk: int) -> bool:
    return bool(_load().oracle_gist_mask(p, t, chunk))


def prefill_pair_count(n_chunks: int, chunk: int) -> int:
    return int(_load().oracle_prefill_pair_count(n_chunks, chunk))


def prefill_rows(t: dict, n_chunks: int, chunk: int, rows: np.ndarray, scale: float = 0.0, with_lse: bool = False):
    """rows: int64 [n, 3] of (b, h, p).  Returns out [n, d] fp64 (and the
    natural-log normaliser lse [n] of each row's softmax)."""
    q, k, v = t["q"], t["k"], t["v"]
    B, Hq, P, d = q.shape
    Hkv = k.shape[1]
    assert P == n_chunks * (chunk + 1)
    rows = np.ascontiguousarray(rows, np.int64)
    out = np.empty((rows.shape[0], d), np.float64)
    lse = np.empty(rows.shape[0], np.float64) if with_lse else None
    _load().oracle_prefill_rows(B, Hq, Hkv, d, n_chunks, chunk, scale, _dtcode(q), _p(q), _p(k),
                                _p(v), rows.shape[0], _p(rows), _p(out), _p(lse))
    return (out, lse) if with_lse else out
