"""Seeded synthetic inputs for the GSA decode / prefill workloads.

This package only produces numbers: standard normals from a counter-based
generator (``synth.c``), needle planting along a query direction, and the
workload shape table.  It holds none of the attention method's arithmetic and
is imported by both sides of every parity check (the CUDA library's callers
and the oracle's callers), so the two see byte-identical inputs.

Storage conventions (host numpy arrays):
  * fp32 tensors are ``numpy.float32``;
  * bf16 tensors are ``numpy.uint16`` holding the bf16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        lib.synth_u64.restype = u64
        lib.synth_u64.argtypes = [u64, u64, u64]
        for name in ("synth_normal_f64", "synth_normal_f32", "synth_normal_bf16"):
            f = getattr(lib, name)
            f.restype = None
            f.argtypes = [u64, u64, u64, i64, vp]
        for name in ("synth_round_f32", "synth_round_bf16"):
            f = getattr(lib, name)
            f.restype = None
            f.argtypes = [vp, i64, vp]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def normal(seed: int, stream: int, shape, dtype: str, offset: int = 0) -> np.ndarray:
    """Standard normals for (seed, stream), element i of the flattened shape
    taking counter ``offset + i``.  dtype: 'f64' | 'f32' | 'bf16'."""
    lib = _load()
    n = int(np.prod(shape)) if len(shape) else 1
    if dtype == "f64":
        out = np.empty(shape, np.float64)
        lib.synth_normal_f64(seed, stream, offset, n, _ptr(out))
    elif dtype == "f32":
        out = np.empty(shape, np.float32)
        lib.synth_normal_f32(seed, stream, offset, n, _ptr(out))
    elif dtype == "bf16":
        out = np.empty(shape, np.uint16)
        lib.synth_normal_bf16(seed, stream, offset, n, _ptr(out))
    else:
        raise ValueError(dtype)
    return out


def u64(seed: int, stream: int, i: int) -> int:
    return int(_load().synth_u64(seed, stream, i))


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values to the storage dtype (fp32 RNE; bf16 RNE via fp32)."""
    x = np.ascontiguousarray(x, np.float64)
    lib = _load()
    if dtype == "f32":
        out = np.empty(x.shape, np.float32)
        lib.synth_round_f32(_ptr(x), x.size, _ptr(out))
    elif dtype == "bf16":
        out = np.empty(x.shape, np.uint16)
        lib.synth_round_bf16(_ptr(x), x.size, _ptr(out))
    else:
        raise ValueError(dtype)
    return out


def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values to fp64 (bf16 bits -> fp32 -> fp64)."""
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# ---------------------------------------------------------------------------
# Workload shapes
# ---------------------------------------------------------------------------
ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS = 0, 1, 2, 3

# stream ids, one per generated tensor
S_Q, S_KG, S_VG, S_KR, S_VR, S_KT, S_VT, S_NEEDLE_IDX, S_NEEDLE_NOISE = range(1, 10)
S_KG2, S_VG2, S_NEEDLE2_NOISE = 10, 11, 12
S_PQ, S_PK, S_PV = 20, 21, 22
S_PAGE_K, S_PAGE_V, S_PAGE_ORDER, S_DOC, S_SEQ_LEN = 30, 31, 32, 33, 34
S_LEVEL_K, S_LEVEL_V, S_LEVEL_NOISE = 40, 50, 60   # + level
S_SUF_Q, S_SUF_K, S_SUF_V = 70, 71, 72


@dataclass(frozen=True)
class DecodeShape:
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_chunks: int          # N gists, one per chunk
    chunk: int             # c raw tokens per chunk
    top_k: int
    tail_len: int          # W uncompressed local tokens after the chunks
    dtype: str = "bf16"    # 'f32' | 'bf16'
    mode: int = ALL_GISTS
    n_needles: int = 0
    needle_alpha: float = 3.0
    scale: float = 0.0     # <= 0: 1/sqrt(head_dim)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def rows(self) -> int:
        return self.batch * self.n_kv_heads


@dataclass(frozen=True)
class HierShape:
    l1: DecodeShape        # level-1 gists, raw chunks, tail; l1.top_k = k1
    n_l2: int              # level-2 (meta) gists
    group: int             # level-1 gists per level-2 gist
    top_k2: int


@dataclass(frozen=True)
class PrefillShape:
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_chunks: int
    chunk: int
    dtype: str = "bf16"
    scale: float = 0.0

    @property
    def positions(self) -> int:
        return self.n_chunks * (self.chunk + 1)


@dataclass(frozen=True)
class LevelsShape:
    """A gist hierarchy of depth L = len(groups) + 1: level 1 is l1's gists
    (one per chunk); groups[i] level-(i+1) gists make one level-(i+2) gist;
    top_ks[i] is the selection size at level i + 2 (l1.top_k at level 1)."""
    l1: DecodeShape
    groups: tuple
    top_ks: tuple

    @property
    def counts(self) -> list:
        n = [self.l1.n_chunks]
        for g in self.groups:
            n.append(-(-n[-1] // g))
        return n


@dataclass(frozen=True)
class SuffixShape:
    """The forward pass of a suffix of S = base.tail_len tokens after N
    compressed chunks (stage-2 selective finetuning): every suffix position
    selects its own chunks; the suffix attends causally to itself."""
    base: DecodeShape


@dataclass(frozen=True)
class PagedShape:
    """A batch of sequences whose raw chunks live in a shared page pool.

    The pool holds n_docs documents of doc_min..doc_max chunks each (one page
    per chunk, all KV heads in the page) in a scrambled page order; each
    sequence is a run of documents drawn from the pool (so sequences share
    pages) cut to its chunk count, between 3/4 N and N unless given."""
    base: DecodeShape      # n_chunks = N, the most chunks a sequence has
    n_docs: int
    doc_min: int
    doc_max: int
    spare_pages: int = 0   # pool pages that no document uses


# The five workloads (shapes, dtypes, needles).
WORKLOADS = {
    "tiny_f32": DecodeShape(1, 4, 1, 64, 128, 16, 4, 16, "f32", ALL_GISTS, n_needles=4),
    "llama8b_decode": DecodeShape(8, 32, 8, 128, 2048, 16, 16, 64, "bf16", ALL_GISTS, n_needles=16),
    # compression-ratio sweep: 131072 raw tokens, k*c = 2048 unfolded tokens
    "sweep_c8_all": DecodeShape(4, 32, 8, 128, 16384, 8, 256, 128, "bf16", ALL_GISTS, n_needles=256),
    "sweep_c16_all": DecodeShape(4, 32, 8, 128, 8192, 16, 128, 128, "bf16", ALL_GISTS, n_needles=128),
    "sweep_c32_all": DecodeShape(4, 32, 8, 128, 4096, 32, 64, 128, "bf16", ALL_GISTS, n_needles=64),
    "sweep_c8_pairs": DecodeShape(4, 32, 8, 128, 16384, 8, 256, 128, "bf16", SELECTED_PAIRS, n_needles=256),
    "sweep_c16_pairs": DecodeShape(4, 32, 8, 128, 8192, 16, 128, 128, "bf16", SELECTED_PAIRS, n_needles=128),
    "sweep_c32_pairs": DecodeShape(4, 32, 8, 128, 4096, 32, 64, 128, "bf16", SELECTED_PAIRS, n_needles=64),
    "hier_1m": HierShape(DecodeShape(1, 32, 8, 128, 65536, 16, 8, 128, "bf16", ALL_GISTS, n_needles=8),
                         n_l2=4096, group=16, top_k2=8),
    "gist_prefill": PrefillShape(2, 32, 8, 128, 1024, 16, "bf16"),
    # three levels over 1M raw tokens: 65536 -> 4096 -> 256 gists, k = 8 at every level
    "hier3_1m": LevelsShape(DecodeShape(1, 32, 8, 128, 65536, 16, 8, 128, "bf16", ALL_GISTS, n_needles=8),
                            groups=(16, 16), top_ks=(8, 8)),
    # the fixed latency of the one-launch step: a 2048-token context (8 rows, 128 gists), about 1 MB
    "decode_floor": DecodeShape(1, 32, 8, 128, 128, 16, 4, 64, "bf16", ALL_GISTS, n_needles=4),
    # stage-2 forward: a 512-token suffix after 2048 chunks of 16 (Llama-style heads)
    "suffix_stage2": SuffixShape(DecodeShape(2, 32, 8, 128, 2048, 16, 16, 512, "bf16", ALL_GISTS, n_needles=16)),
    # the Llama-shaped step over a shared page pool of 32..160-chunk documents
    # (KV-cache reuse), sequences of 1536..2048 chunks
    "llama8b_paged": PagedShape(DecodeShape(8, 32, 8, 128, 2048, 16, 16, 64, "bf16", ALL_GISTS, n_needles=16),
                                n_docs=48, doc_min=32, doc_max=160),
}

# workload -> index in the published config list (seeds 20260422 + 100*cfg + rep)
CONFIG_INDEX = {"tiny_f32": 1, "llama8b_decode": 2, "sweep_c8_all": 3, "sweep_c16_all": 3,
                "sweep_c32_all": 3, "sweep_c8_pairs": 3, "sweep_c16_pairs": 3,
                "sweep_c32_pairs": 3, "hier_1m": 4, "gist_prefill": 5, "llama8b_paged": 6,
                "hier3_1m": 7, "suffix_stage2": 8,
                "decode_floor": 9}


def seed_for(workload: str, rep: int = 0) -> int:
    return 20260422 + 100 * CONFIG_INDEX[workload] + rep


def _distinct_draws(seed: int, stream: int, base: int, count: int, modulus: int) -> list:
    """`count` distinct values in [0, modulus) from successive draws."""
    assert count <= modulus
    out, seen, i = [], set(), 0
    while len(out) < count:
        v = u64(seed, stream, base + i) % modulus
        i += 1
        if v not in seen:
            seen.add(v)
            out.append(v)
    return out


def _needle_keys(q_wide: np.ndarray, b: int, hk: int, G: int, alpha: float, noise: np.ndarray) -> np.ndarray:
    """alpha * qbar/|qbar| + 0.1 * noise, qbar = sum of the group's query heads."""
    qbar = q_wide[b, hk * G:(hk + 1) * G, :].sum(axis=0)
    return alpha * qbar / np.linalg.norm(qbar) + 0.1 * noise


@dataclass
class DecodeInputs:
    shape: DecodeShape
    q: np.ndarray
    k_gist: np.ndarray
    v_gist: np.ndarray
    k_raw: np.ndarray
    v_raw: np.ndarray
    k_tail: np.ndarray
    v_tail: np.ndarray
    needles: np.ndarray = field(default=None)   # [rows, n_needles] chunk ids

    def tensors(self):
        return dict(q=self.q, k_gist=self.k_gist, v_gist=self.v_gist, k_raw=self.k_raw,
                    v_raw=self.v_raw, k_tail=self.k_tail, v_tail=self.v_tail)


def decode_inputs(s: DecodeShape, seed: int) -> DecodeInputs:
    B, Hq, Hkv, d, N, c, W = s.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, s.n_chunks, s.chunk, s.tail_len
    dt = s.dtype
    q = normal(seed, S_Q, (B, Hq, d), dt)
    kg = normal(seed, S_KG, (B, Hkv, N, d), dt)
    vg = normal(seed, S_VG, (B, Hkv, N, d), dt)
    kr = normal(seed, S_KR, (B, Hkv, N, c, d), dt)
    vr = normal(seed, S_VR, (B, Hkv, N, c, d), dt)
    kt = normal(seed, S_KT, (B, Hkv, W, d), dt)
    vt = normal(seed, S_VT, (B, Hkv, W, d), dt)
    needles = np.zeros((B * Hkv, s.n_needles), np.int64)
    if s.n_needles:
        qw = widen(q, dt)
        G = s.group
        for b in range(B):
            for hk in range(Hkv):
                row = b * Hkv + hk
                ids = _distinct_draws(seed, S_NEEDLE_IDX, row * 1_000_003, s.n_needles, N)
                needles[row] = ids
                noise = normal(seed, S_NEEDLE_NOISE, (s.n_needles, d), "f64",
                               offset=row * s.n_needles * d)
                for t, j in enumerate(ids):
                    kg[b, hk, j] = round_to(_needle_keys(qw, b, hk, G, s.needle_alpha, noise[t]), dt)
    return DecodeInputs(s, q, kg, vg, kr, vr, kt, vt, needles)


@dataclass
class HierInputs:
    shape: HierShape
    q: np.ndarray
    k_g2: np.ndarray
    v_g2: np.ndarray
    k_g1: np.ndarray
    v_g1: np.ndarray
    k_raw: np.ndarray
    v_raw: np.ndarray
    k_tail: np.ndarray
    v_tail: np.ndarray
    needles: np.ndarray = field(default=None)

    def tensors(self):
        return dict(q=self.q, k_g2=self.k_g2, v_g2=self.v_g2, k_g1=self.k_g1, v_g1=self.v_g1,
                    k_raw=self.k_raw, v_raw=self.v_raw, k_tail=self.k_tail, v_tail=self.v_tail)


def hier_inputs(h: HierShape, seed: int) -> HierInputs:
    """Level-1 tensors as for flat decode (without needles), plus level-2 gists.
    Needles go into distinct level-2 groups: one level-1 chunk per needle group
    gets the needle key, and so does that group's level-2 gist."""
    s = h.l1
    base = decode_inputs(replace(s, n_needles=0), seed)
    B, Hkv, d, dt = s.batch, s.n_kv_heads, s.head_dim, s.dtype
    kg2 = normal(seed, S_KG2, (B, Hkv, h.n_l2, d), dt)
    vg2 = normal(seed, S_VG2, (B, Hkv, h.n_l2, d), dt)
    needles = np.zeros((B * Hkv, s.n_needles), np.int64)
    if s.n_needles:
        qw = widen(base.q, dt)
        G = s.group
        for b in range(B):
            for hk in range(Hkv):
                row = b * Hkv + hk
                groups = _distinct_draws(seed, S_NEEDLE_IDX, row * 1_000_003, s.n_needles, h.n_l2)
                noise1 = normal(seed, S_NEEDLE_NOISE, (s.n_needles, d), "f64", offset=row * s.n_needles * d)
                noise2 = normal(seed, S_NEEDLE2_NOISE, (s.n_needles, d), "f64", offset=row * s.n_needles * d)
                for t, g in enumerate(groups):
                    lo = g * h.group
                    width = min(h.group, s.n_chunks - lo)
                    j = lo + u64(seed, S_NEEDLE_IDX, 7_777_777 + row * 1_000_003 + t) % width
                    needles[row, t] = j
                    base.k_gist[b, hk, j] = round_to(_needle_keys(qw, b, hk, G, s.needle_alpha, noise1[t]), dt)
                    kg2[b, hk, g] = round_to(_needle_keys(qw, b, hk, G, s.needle_alpha, noise2[t]), dt)
    return HierInputs(h, base.q, kg2, vg2, base.k_gist, base.v_gist, base.k_raw, base.v_raw,
                      base.k_tail, base.v_tail, needles)


@dataclass
class PrefillInputs:
    shape: PrefillShape
    q: np.ndarray   # [B, Hq, P, d]
    k: np.ndarray   # [B, Hkv, P, d]
    v: np.ndarray

    def tensors(self):
        return dict(q=self.q, k=self.k, v=self.v)


def prefill_inputs(p: PrefillShape, seed: int) -> PrefillInputs:
    P = p.positions
    q = normal(seed, S_PQ, (p.batch, p.n_q_heads, P, p.head_dim), p.dtype)
    k = normal(seed, S_PK, (p.batch, p.n_kv_heads, P, p.head_dim), p.dtype)
    v = normal(seed, S_PV, (p.batch, p.n_kv_heads, P, p.head_dim), p.dtype)
    return PrefillInputs(p, q, k, v)


@dataclass
class PagedInputs:
    shape: PagedShape
    q: np.ndarray
    k_gist: np.ndarray       # [B, Hkv, N, d]; entries past a sequence's chunk count are decoys
    v_gist: np.ndarray
    k_pages: np.ndarray      # [pages, Hkv, c, d]
    v_pages: np.ndarray
    table: np.ndarray        # [B, N] int32 page of chunk j of sequence b; -1 past its chunk count
    seq_chunks: np.ndarray   # [B] int32
    k_tail: np.ndarray
    v_tail: np.ndarray

    def tensors(self):
        return dict(q=self.q, k_gist=self.k_gist, v_gist=self.v_gist, k_tail=self.k_tail, v_tail=self.v_tail)

    def dense_raw(self):
        """The raw cache gathered per sequence, [B, Hkv, N, c, d] (zeros past
        each sequence's chunk count)."""
        B, N = self.table.shape
        P, Hkv, c, d = self.k_pages.shape
        kr = np.zeros((B, Hkv, N, c, d), self.k_pages.dtype)
        vr = np.zeros_like(kr)
        for b in range(B):
            n = int(self.seq_chunks[b])
            kr[b, :, :n] = self.k_pages[self.table[b, :n]].transpose(1, 0, 2, 3)
            vr[b, :, :n] = self.v_pages[self.table[b, :n]].transpose(1, 0, 2, 3)
        return kr, vr


def paged_inputs(ps: PagedShape, seed: int, seq_chunks=None) -> PagedInputs:
    s = ps.base
    B, Hq, Hkv, d, N, c, W, dt = (s.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, s.n_chunks, s.chunk,
                                  s.tail_len, s.dtype)
    span = ps.doc_max - ps.doc_min + 1
    doc_len = [ps.doc_min + u64(seed, S_DOC, i) % span for i in range(ps.n_docs)]
    P = sum(doc_len) + ps.spare_pages
    order = np.argsort(np.array([u64(seed, S_PAGE_ORDER, i) for i in range(P)], np.uint64), kind="stable")
    starts = np.concatenate([[0], np.cumsum(doc_len)])
    if seq_chunks is None:
        seq_chunks = [N - u64(seed, S_SEQ_LEN, b) % (N // 4 + 1) for b in range(B)]
    seq_chunks = np.asarray(seq_chunks, np.int32)
    assert seq_chunks.shape == (B,) and np.all((seq_chunks >= 0) & (seq_chunks <= N))
    table = np.full((B, N), -1, np.int32)
    for b in range(B):
        pages, t = [], 0
        while len(pages) < seq_chunks[b]:
            doc = u64(seed, S_DOC, 1_000_003 * (b + 1) + t) % ps.n_docs
            t += 1
            pages.extend(order[starts[doc]:starts[doc] + doc_len[doc]].tolist())
        table[b, :seq_chunks[b]] = pages[:seq_chunks[b]]
    q = normal(seed, S_Q, (B, Hq, d), dt)
    kg = normal(seed, S_KG, (B, Hkv, N, d), dt)
    vg = normal(seed, S_VG, (B, Hkv, N, d), dt)
    kp = normal(seed, S_PAGE_K, (P, Hkv, c, d), dt)
    vp = normal(seed, S_PAGE_V, (P, Hkv, c, d), dt)
    kt = normal(seed, S_KT, (B, Hkv, W, d), dt)
    vt = normal(seed, S_VT, (B, Hkv, W, d), dt)
    qw = widen(q, dt)
    G = s.group
    for b in range(B):
        n = int(seq_chunks[b])
        for hk in range(Hkv):
            row = b * Hkv + hk
            # needles among the sequence's chunks; every gist past its end is a
            # decoy that would win the routing if it were scored
            m = min(s.n_needles, n)
            ids = _distinct_draws(seed, S_NEEDLE_IDX, row * 1_000_003, m, n) if m else []
            noise = normal(seed, S_NEEDLE_NOISE, (max(m, 1) + N - n, d), "f64", offset=row * (N + 1) * d)
            for t, j in enumerate(ids):
                kg[b, hk, j] = round_to(_needle_keys(qw, b, hk, G, s.needle_alpha, noise[t]), dt)
            for t, j in enumerate(range(n, N)):
                kg[b, hk, j] = round_to(_needle_keys(qw, b, hk, G, 2 * s.needle_alpha, noise[max(m, 1) + t]), dt)
    return PagedInputs(ps, q, kg, vg, kp, vp, table, seq_chunks, kt, vt)


@dataclass
class LevelsInputs:
    shape: LevelsShape
    q: np.ndarray
    k_g: list            # level 1 first, [B, Hkv, n_l, d]
    v_g: list
    k_raw: np.ndarray
    v_raw: np.ndarray
    k_tail: np.ndarray
    v_tail: np.ndarray
    needles: np.ndarray  # [rows, n_needles] level-1 chunk of each needle chain


def levels_inputs(h: LevelsShape, seed: int) -> LevelsInputs:
    """Level-1 tensors as for flat decode, upper-level gists drawn per level.
    Each needle is a chain: a level-1 chunk and every ancestor of it get a
    needle key, the chains in distinct top-level gists, so the descent can
    follow each chain to its chunk."""
    s = h.l1
    base = decode_inputs(replace(s, n_needles=0), seed)
    B, Hkv, d, dt = s.batch, s.n_kv_heads, s.head_dim, s.dtype
    n = h.counts
    L = len(n)
    kg, vg = [base.k_gist], [base.v_gist]
    for lv in range(1, L):
        kg.append(normal(seed, S_LEVEL_K + lv, (B, Hkv, n[lv], d), dt))
        vg.append(normal(seed, S_LEVEL_V + lv, (B, Hkv, n[lv], d), dt))
    needles = np.zeros((B * Hkv, s.n_needles), np.int64)
    if s.n_needles:
        qw = widen(base.q, dt)
        G = s.group
        for b in range(B):
            for hk in range(Hkv):
                row = b * Hkv + hk
                tops = _distinct_draws(seed, S_NEEDLE_IDX, row * 1_000_003, s.n_needles, n[-1])
                for t, top in enumerate(tops):
                    node = top
                    for lv in range(L - 1, -1, -1):
                        noise = normal(seed, S_LEVEL_NOISE + lv, (d,), "f64",
                                       offset=(row * s.n_needles + t) * d)
                        kg[lv][b, hk, node] = round_to(_needle_keys(qw, b, hk, G, s.needle_alpha, noise), dt)
                        if lv == 0:
                            break
                        g = h.groups[lv - 1]
                        lo = node * g
                        width = min(g, n[lv - 1] - lo)
                        node = lo + u64(seed, S_NEEDLE_IDX, 5_555_555 + (row * s.n_needles + t) * L + lv) % width
                    needles[row, t] = node
    return LevelsInputs(h, base.q, kg, vg, base.k_raw, base.v_raw, base.k_tail, base.v_tail, needles)


@dataclass
class SuffixInputs:
    shape: SuffixShape
    q: np.ndarray        # [B, S, Hq, d]
    k_gist: np.ndarray
    v_gist: np.ndarray
    k_raw: np.ndarray
    v_raw: np.ndarray
    k_suf: np.ndarray    # [B, Hkv, S, d]
    v_suf: np.ndarray


def suffix_inputs(ss: SuffixShape, seed: int) -> SuffixInputs:
    """Gists and raw chunks as for decode (needles along each sequence's
    common query direction); the suffix queries of a sequence share that
    direction: q[b, p, h] = q0[b, h] + 0.5 * noise[b, p, h]."""
    s = ss.base
    B, Hq, Hkv, d, S, dt = s.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, s.tail_len, s.dtype
    base = decode_inputs(replace(s, tail_len=0), seed)
    q0 = widen(base.q, dt)
    noise = normal(seed, S_SUF_Q, (B, S, Hq, d), "f64")
    q = round_to(q0[:, None] + 0.5 * noise, dt)
    ks = normal(seed, S_SUF_K, (B, Hkv, S, d), dt)
    vs = normal(seed, S_SUF_V, (B, Hkv, S, d), dt)
    return SuffixInputs(ss, q, base.k_gist, base.v_gist, base.k_raw, base.v_raw, ks, vs)
