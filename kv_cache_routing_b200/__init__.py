"""Python binding of libgsa.so — the GSA decode hot path on B200 (sm_100a).

Argument marshalling only: every entry point takes the same arguments as the
C function of the same name in ``include/gsa.h``, with torch tensors (or raw
integer device addresses) in place of pointers, and raises ``GsaError`` on a
non-OK status.  All work runs in the CUDA kernels of libgsa.so; there is no
fallback path.  ``stream`` defaults to torch's current stream.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgsa.so")

GSA_OK, GSA_ERR_ARG, GSA_ERR_SHAPE, GSA_ERR_DTYPE, GSA_ERR_ALIGN, GSA_ERR_WORKSPACE, GSA_ERR_CUDA, \
    GSA_ERR_TIMEOUT = range(8)
GSA_F32, GSA_BF16 = 0, 1
GSA_ALL_GISTS, GSA_SELECTED_PAIRS, GSA_SR_ONLY, GSA_UNSELECTED_GISTS = 0, 1, 2, 3
GSA_WS_ERR_TIMEOUT, GSA_WS_ERR_INDEX = 1, 2

# Every function the C header declares (checked by the tests).
EXPORTS = ("gsa_decode_workspace_size", "gsa_hier_workspace_size", "gsa_score", "gsa_topk",
           "gsa_unfold_attn", "gsa_decode_step", "gsa_hier_decode", "gsa_gist_prefill",
           "gsa_workspace_error", "gsa_status_string", "gsa_decode_step_noalloc", "gsa_decode_launch_count",
           "gsa_hier_launch_count", "gsa_device_error", "gsa_set_wait_limit_ns", "gsa_topp",
           "gsa_decode_step_topp", "gsa_decode_step_paged",
           "gsa_levels_workspace_size", "gsa_levels_decode", "gsa_levels_launch_count",
           "gsa_suffix_workspace_size", "gsa_suffix_launch_count", "gsa_suffix_attn", "gsa_decode_step_host")


class GsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class DecodeDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("n_chunks", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("tail_len", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("mode", ctypes.c_int), ("scale", ctypes.c_float)]


class HierDesc(ctypes.Structure):
    _fields_ = [("l1", DecodeDesc), ("n_l2", ctypes.c_int32), ("group", ctypes.c_int32),
                ("top_k2", ctypes.c_int32)]


GSA_MAX_LEVELS = 8


class LevelsDesc(ctypes.Structure):
    _fields_ = [("l1", DecodeDesc), ("levels", ctypes.c_int32),
                ("group", ctypes.c_int32 * (GSA_MAX_LEVELS - 1)), ("top_k", ctypes.c_int32 * (GSA_MAX_LEVELS - 1))]


class PrefillDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("n_chunks", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("dtype", ctypes.c_int), ("scale", ctypes.c_float)]


_lib = None
_SIG = None


def _signatures():
    vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    pd, ph, pp = ctypes.POINTER(DecodeDesc), ctypes.POINTER(HierDesc), ctypes.POINTER(PrefillDesc)
    return {
        "gsa_decode_workspace_size": (sz, [pd]),
        "gsa_hier_workspace_size": (sz, [ph]),
        "gsa_score": (st, [pd, vp, vp, vp, vp]),
        "gsa_topk": (st, [pd, vp, vp, vp]),
        "gsa_unfold_attn": (st, [pd] + [vp] * 10 + [vp, sz, vp]),
        "gsa_decode_step": (st, [pd] + [vp] * 11 + [sz, vp]),
        "gsa_decode_step_noalloc": (st, [pd] + [vp] * 10 + [vp]),
        "gsa_hier_decode": (st, [ph] + [vp] * 13 + [sz, vp]),
        "gsa_gist_prefill": (st, [pp, vp, vp, vp, vp, vp, vp]),
        "gsa_workspace_error": (st, [vp, ctypes.POINTER(ctypes.c_uint32), vp]),
        "gsa_device_error": (st, [ctypes.POINTER(ctypes.c_uint32), vp]),
        "gsa_topp": (st, [pd, ctypes.c_float, vp, vp, vp, vp]),
        "gsa_decode_step_topp": (st, [pd, ctypes.c_float] + [vp] * 11 + [sz, vp]),
        "gsa_decode_step_paged": (st, [pd] + [vp] * 5 + [ctypes.c_int32] + [vp] * 8 + [sz, vp]),
        "gsa_set_wait_limit_ns": (st, [ctypes.c_uint64]),
        "gsa_status_string": (ctypes.c_char_p, [st]),
        "gsa_decode_launch_count": (ctypes.c_int, [pd]),
        "gsa_levels_workspace_size": (sz, [ctypes.POINTER(LevelsDesc)]),
        "gsa_levels_decode": (st, [ctypes.POINTER(LevelsDesc)] + [vp] * 10 + [sz, vp]),
        "gsa_levels_launch_count": (ctypes.c_int, [ctypes.POINTER(LevelsDesc)]),
        "gsa_suffix_workspace_size": (sz, [pd]),
        "gsa_suffix_launch_count": (ctypes.c_int, [pd]),
        "gsa_suffix_attn": (st, [pd] + [vp] * 10 + [vp, sz, vp]),
        "gsa_decode_step_host": (st, [pd] + [vp] * 13 + [sz, vp]),
        "gsa_hier_launch_count": (ctypes.c_int, [ph]),
    }


class _Lib:
    """libgsa.so with argument types attached on first use of each symbol."""

    def __init__(self, path):
        self._dll = ctypes.CDLL(path)
        self._sig = _signatures()

    def __getattr__(self, name):
        f = getattr(self._dll, name)
        res, args = self._sig[name]
        f.restype = res
        f.argtypes = args
        setattr(self, name, f)
        return f


def lib() -> "_Lib":
    """Load libgsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m kv_cache_routing_b200.build`")
        _lib = _Lib(LIB_PATH)
    return _lib


def status_string(status: int) -> str:
    return lib().gsa_status_string(status).decode()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != GSA_OK:
        raise GsaError(status, where)


def _nbytes(ws):
    if ws is None:
        return 0
    return ws.numel() * ws.element_size()


def decode_desc(batch, n_q_heads, n_kv_heads, head_dim, n_chunks, chunk, top_k, tail_len,
                dtype=GSA_BF16, mode=GSA_ALL_GISTS, scale=0.0) -> DecodeDesc:
    return DecodeDesc(batch, n_q_heads, n_kv_heads, head_dim, n_chunks, chunk, top_k, tail_len,
                      dtype, mode, scale)


def hier_desc(l1: DecodeDesc, n_l2, group, top_k2) -> HierDesc:
    return HierDesc(l1, n_l2, group, top_k2)


def levels_desc(l1: DecodeDesc, groups, top_ks) -> LevelsDesc:
    """groups[i]: level-(i+1) gists per level-(i+2) gist; top_ks[i]: the
    selection size at level i + 2 (level 1: l1.top_k)."""
    assert len(groups) == len(top_ks) and 1 <= len(groups) < GSA_MAX_LEVELS
    g = (ctypes.c_int32 * (GSA_MAX_LEVELS - 1))(*groups)
    k = (ctypes.c_int32 * (GSA_MAX_LEVELS - 1))(*top_ks)
    return LevelsDesc(l1, len(groups) + 1, g, k)


def prefill_desc(batch, n_q_heads, n_kv_heads, head_dim, n_chunks, chunk, dtype=GSA_BF16,
                 scale=0.0) -> PrefillDesc:
    return PrefillDesc(batch, n_q_heads, n_kv_heads, head_dim, n_chunks, chunk, dtype, scale)


def gsa_decode_workspace_size(desc: DecodeDesc) -> int:
    return int(lib().gsa_decode_workspace_size(ctypes.byref(desc)))


def gsa_hier_workspace_size(desc: HierDesc) -> int:
    return int(lib().gsa_hier_workspace_size(ctypes.byref(desc)))


def gsa_score(desc, q, k_gist, scores, stream=None):
    _check(lib().gsa_score(ctypes.byref(desc), _ptr(q), _ptr(k_gist), _ptr(scores), _stream(stream)),
           "gsa_score")


def gsa_topk(desc, scores, idx, stream=None):
    _check(lib().gsa_topk(ctypes.byref(desc), _ptr(scores), _ptr(idx), _stream(stream)), "gsa_topk")


def gsa_unfold_attn(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx, out, lse, ws,
                    stream=None, ws_bytes=None):
    nb = _nbytes(ws) if ws_bytes is None else ws_bytes
    _check(lib().gsa_unfold_attn(ctypes.byref(desc), _ptr(q), _ptr(k_gist), _ptr(v_gist), _ptr(k_raw),
                                 _ptr(v_raw), _ptr(k_tail), _ptr(v_tail), _ptr(idx), _ptr(out), _ptr(lse),
                                 _ptr(ws), nb, _stream(stream)), "gsa_unfold_attn")


def gsa_decode_step(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx_out, scores_out, out, ws,
                    stream=None, ws_bytes=None):
    nb = _nbytes(ws) if ws_bytes is None else ws_bytes
    _check(lib().gsa_decode_step(ctypes.byref(desc), _ptr(q), _ptr(k_gist), _ptr(v_gist), _ptr(k_raw),
                                 _ptr(v_raw), _ptr(k_tail), _ptr(v_tail), _ptr(idx_out), _ptr(scores_out),
                                 _ptr(out), _ptr(ws), nb, _stream(stream)), "gsa_decode_step")


def gsa_decode_step_noalloc(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx_out, scores_out, out,
                            stream=None):
    """gsa_decode_step for callers that cannot allocate: the scratch is a fixed
    8 MiB device array inside the library (see include/gsa.h)."""
    _check(lib().gsa_decode_step_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k_gist), _ptr(v_gist), _ptr(k_raw),
                                         _ptr(v_raw), _ptr(k_tail), _ptr(v_tail), _ptr(idx_out), _ptr(scores_out),
                                         _ptr(out), _stream(stream)), "gsa_decode_step_noalloc")


def gsa_hier_decode(desc, q, k_g2, v_g2, k_g1, v_g1, k_raw, v_raw, k_tail, v_tail, idx2_out, idx1_out, out,
                    ws, stream=None, ws_bytes=None):
    nb = _nbytes(ws) if ws_bytes is None else ws_bytes
    _check(lib().gsa_hier_decode(ctypes.byref(desc), _ptr(q), _ptr(k_g2), _ptr(v_g2), _ptr(k_g1), _ptr(v_g1),
                                 _ptr(k_raw), _ptr(v_raw), _ptr(k_tail), _ptr(v_tail), _ptr(idx2_out),
                                 _ptr(idx1_out), _ptr(out), _ptr(ws), nb, _stream(stream)), "gsa_hier_decode")


def gsa_gist_prefill(desc, q, k, v, out, lse=None, stream=None):
    _check(lib().gsa_gist_prefill(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                  _stream(stream)), "gsa_gist_prefill")


def gsa_decode_launch_count(desc) -> int:
    """Kernel launches one gsa_decode_step with `desc` enqueues."""
    n = lib().gsa_decode_launch_count(ctypes.byref(desc))
    if n < 0:
        raise GsaError(1, "gsa_decode_launch_count")
    return int(n)


def gsa_hier_launch_count(desc) -> int:
    """Kernel launches one gsa_hier_decode with `desc` enqueues."""
    n = lib().gsa_hier_launch_count(ctypes.byref(desc))
    if n < 0:
        raise GsaError(1, "gsa_hier_launch_count")
    return int(n)


def gsa_workspace_error(ws, stream=None) -> int:
    """Workspace error word (0 or GSA_WS_ERR_* flags)."""
    flags = ctypes.c_uint32(0)
    lib().gsa_workspace_error(_ptr(ws), ctypes.byref(flags), _stream(stream))
    return int(flags.value)


def gsa_device_error(stream=None) -> int:
    """Reads and clears the library's own device error words (entry points
    without a workspace, the prefill, the no-allocation scratch): 0 or an OR
    of GSA_WS_ERR_* flags."""
    flags = ctypes.c_uint32(0)
    st = lib().gsa_device_error(ctypes.byref(flags), _stream(stream))
    if st not in (GSA_OK, GSA_ERR_TIMEOUT, GSA_ERR_ARG):
        raise GsaError(st, "gsa_device_error")
    return int(flags.value)


def gsa_set_wait_limit_ns(ns: int):
    """Diagnostics: limit of the cross-CTA waits of a decode launch (0: default)."""
    _check(lib().gsa_set_wait_limit_ns(int(ns)), "gsa_set_wait_limit_ns")


def gsa_topp(desc, top_p, scores, idx, count=None, stream=None):
    _check(lib().gsa_topp(ctypes.byref(desc), float(top_p), _ptr(scores), _ptr(idx), _ptr(count), _stream(stream)),
           "gsa_topp")


def gsa_decode_step_topp(desc, top_p, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx_out, count_out,
                         scores_out, out, ws, stream=None, ws_bytes=None):
    nb = _nbytes(ws) if ws_bytes is None else ws_bytes
    _check(lib().gsa_decode_step_topp(ctypes.byref(desc), float(top_p), _ptr(q), _ptr(k_gist), _ptr(v_gist),
                                      _ptr(k_raw), _ptr(v_raw), _ptr(k_tail), _ptr(v_tail), _ptr(idx_out),
                                      _ptr(count_out), _ptr(scores_out), _ptr(out), _ptr(ws), nb, _stream(stream)),
           "gsa_decode_step_topp")


def gsa_decode_step_paged(desc, q, k_gist, v_gist, k_pages, v_pages, n_pages, block_table, seq_chunks, k_tail,
                          v_tail, idx_out, scores_out, out, ws, stream=None, ws_bytes=None):
    """Decode step over a paged raw cache: k_pages / v_pages [n_pages, Hkv, c, d],
    block_table int32 [B, N], seq_chunks int32 [B] or None."""
    nb = _nbytes(ws) if ws_bytes is None else ws_bytes
    _check(lib().gsa_decode_step_paged(ctypes.byref(desc), _ptr(q), _ptr(k_gist), _ptr(v_gist), _ptr(k_pages),
                                       _ptr(v_pages), int(n_pages), _ptr(block_table), _ptr(seq_chunks),
                                       _ptr(k_tail), _ptr(v_tail), _ptr(idx_out), _ptr(scores_out), _ptr(out),
                                       _ptr(ws), nb, _stream(stream)), "gsa_decode_step_paged")


def gsa_levels_workspace_size(desc: LevelsDesc) -> int:
    return int(lib().gsa_levels_workspace_size(ctypes.byref(desc)))


def gsa_levels_launch_count(desc: LevelsDesc) -> int:
    n = lib().gsa_levels_launch_count(ctypes.byref(desc))
    if n < 0:
        raise GsaError(1, "gsa_levels_launch_count")
    return int(n)


def gsa_levels_decode(desc, q, k_gists, v_gists, k_raw, v_raw, k_tail, v_tail, idx_out, out, ws, stream=None,
                      ws_bytes=None):
    """Hierarchy of any depth.  k_gists / v_gists: sequences of the L levels'
    gist tensors, level 1 first; idx_out: None or a sequence of L nullable
    selection tensors."""
    L = len(k_gists)
    arr = lambda xs: (ctypes.c_void_p * L)(*[_ptr(x) for x in xs])
    nb = _nbytes(ws) if ws_bytes is None else ws_bytes
    _check(lib().gsa_levels_decode(ctypes.byref(desc), _ptr(q), arr(k_gists), arr(v_gists), _ptr(k_raw), _ptr(v_raw),
                                   _ptr(k_tail), _ptr(v_tail), None if idx_out is None else arr(idx_out), _ptr(out),
                                   _ptr(ws), nb, _stream(stream)), "gsa_levels_decode")


def gsa_suffix_workspace_size(desc) -> int:
    return int(lib().gsa_suffix_workspace_size(ctypes.byref(desc)))


def gsa_suffix_launch_count(desc) -> int:
    n = lib().gsa_suffix_launch_count(ctypes.byref(desc))
    if n < 0:
        raise GsaError(1, "gsa_suffix_launch_count")
    return int(n)


def gsa_suffix_attn(desc, q, k_gist, v_gist, k_raw, v_raw, k_suffix, v_suffix, idx_out, scores_out, out, ws,
                    stream=None, ws_bytes=None):
    """Stage-2 forward over a suffix of desc.tail_len tokens: q / out
    [B, S, Hq, d], k_suffix / v_suffix [B, Hkv, S, d]."""
    nb = _nbytes(ws) if ws_bytes is None else ws_bytes
    _check(lib().gsa_suffix_attn(ctypes.byref(desc), _ptr(q), _ptr(k_gist), _ptr(v_gist), _ptr(k_raw), _ptr(v_raw),
                                 _ptr(k_suffix), _ptr(v_suffix), _ptr(idx_out), _ptr(scores_out), _ptr(out), _ptr(ws),
                                 nb, _stream(stream)), "gsa_suffix_attn")


def gsa_decode_step_host(desc, q_host, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx_out, idx_host, out,
                         out_host, ws, stream=None, ws_bytes=None):
    """gsa_decode_step with q_host / out_host (and idx_host) in host memory
    (page-locked tensors or raw addresses): copy in, step, copy out, one call."""
    nb = _nbytes(ws) if ws_bytes is None else ws_bytes
    _check(lib().gsa_decode_step_host(ctypes.byref(desc), _ptr(q_host), _ptr(q), _ptr(k_gist), _ptr(v_gist),
                                      _ptr(k_raw), _ptr(v_raw), _ptr(k_tail), _ptr(v_tail), _ptr(idx_out),
                                      _ptr(idx_host), _ptr(out), _ptr(out_host), _ptr(ws), nb, _stream(stream)),
           "gsa_decode_step_host")
