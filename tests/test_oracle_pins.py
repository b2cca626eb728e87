"""Pins for the fp64 oracle: worked examples printed on the pages, closed
forms, brute force and library routines (torch SDPA in fp64, numpy sorts).

None of these retypes the oracle's own formulas: attention is checked against
``torch.nn.functional.scaled_dot_product_attention`` over an explicitly
assembled key list or a boolean mask, selection against ``numpy.lexsort``,
scores against one-hot closed forms, the prefill mask against the slide's
table and a pair-count closed form.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import DecodeShape, HierShape, ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS


def sdpa(qv, K, V, scale, mask=None, causal=False):
    """Library attention in fp64: qv [..., L, d], K/V [..., S, d]."""
    q = torch.as_tensor(qv, dtype=torch.float64)
    k = torch.as_tensor(K, dtype=torch.float64)
    v = torch.as_tensor(V, dtype=torch.float64)
    m = None if mask is None else torch.as_tensor(mask, dtype=torch.bool)
    return torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=m, is_causal=causal, scale=scale).numpy()


def small_shape(**kw):
    base = dict(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=8, n_chunks=6, chunk=3, top_k=2,
                tail_len=2, dtype="f32", mode=ALL_GISTS)
    base.update(kw)
    return DecodeShape(**base)


# ---------------------------------------------------------------- scores ----
def test_score_one_hot_queries_pick_gist_columns():
    """q_h = e_{i_h}: the group score of gist j is the sum of Kg[j, i_h] over
    the group's heads; heads of the other KV head do not contribute."""
    B, Hq, Hkv, d, N = 1, 4, 2, 8, 5
    kg = synth.normal(11, 1, (B, Hkv, N, d), "f64")
    q = np.zeros((B, Hq, d))
    cols = [1, 6, 3, 0]             # head h -> one-hot column; heads 0,1 -> kv 0; 2,3 -> kv 1
    for h, i in enumerate(cols):
        q[0, h, i] = 1.0
    s = oracle.gist_scores(q, kg)
    np.testing.assert_array_equal(s[0, 0], kg[0, 0, :, 1] + kg[0, 0, :, 6])
    np.testing.assert_array_equal(s[0, 1], kg[0, 1, :, 3] + kg[0, 1, :, 0])


def test_score_error_bound_covers_fp32_evaluation():
    """Higham's inner-product bound holds for a float32 evaluation of the same sum."""
    sh = small_shape(head_dim=64, n_chunks=40)
    x = synth.decode_inputs(sh, 5)
    s = oracle.gist_scores(x.q, x.k_gist)
    eps = oracle.score_error_bound(x.q, x.k_gist)
    G = sh.group
    for b in range(sh.batch):
        for hk in range(sh.n_kv_heads):
            q32 = x.q[b, hk * G:(hk + 1) * G].astype(np.float32)
            for j in range(sh.n_chunks):
                acc = np.float32(0)
                for g in range(G):
                    for i in range(sh.head_dim):
                        acc = np.float32(acc + np.float32(q32[g, i] * x.k_gist[b, hk, j, i]))
                assert abs(float(acc) - s[b, hk, j]) <= eps[b, hk]


def test_score_error_bound_closed_form_by_hand():
    """Higham's inner-product bound gamma_n * sum |q_i k_i| evaluated by hand
    for inputs of known sign and magnitude.

    G = 1, d = 4, q = (1, -2, 3, -4); gist 0 has k = (1, 1, 1, 1) (sum of
    |q_i k_i| = 10), gist 1 has k = (0.5, -0.5, 0.5, -0.5) (sum 5).  The row
    bound is the larger one: n = G d = 4 products, u = 2^-24,
        gamma_4 = 4u / (1 - 4u) = 2.384185791015625e-07 / 0.9999997615814209
                = 2.3841863594e-07,
        eps = 10 * gamma_4 = 2.3841863594e-06.
    A bound built with another n, or without the absolute values, misses it."""
    q = np.array([[[1.0, -2.0, 3.0, -4.0]]])
    kg = np.array([[[[1.0, 1.0, 1.0, 1.0], [0.5, -0.5, 0.5, -0.5]]]])
    eps = oracle.score_error_bound(q, kg)
    assert eps.shape == (1, 1)
    assert eps[0, 0] == pytest.approx(2.3841863594e-06, rel=1e-9)


def test_score_error_bound_counts_every_product_of_the_group():
    """The number of products in a routing score is G * d: with all entries
    equal to 1 the bound is n * gamma_n, n = G * d, so (G = 2, d = 64) and
    (G = 1, d = 128) give the same bound, and doubling d at G = 1 multiplies
    it by 2 * gamma_128 / gamma_64, just above 4 (hand value 4.00001525890...)."""
    def bound(G, d):
        q = np.ones((1, G, d))
        kg = np.ones((1, 1, 3, d))
        return oracle.score_error_bound(q, kg)[0, 0]
    assert bound(2, 64) == pytest.approx(bound(1, 128), rel=1e-12)
    # 128 gamma_128 / (64 gamma_64) = 2 * (128u / (1 - 128u)) / (64u / (1 - 64u)) = 4 (1 - 64u) / (1 - 128u)
    assert bound(1, 128) / bound(1, 64) == pytest.approx(4.0000152589055, rel=1e-11)
    # n = 64: 64u = 3.814697265625e-06, gamma_64 = 3.8147118...e-06, 64 gamma_64 = 2.44141556...e-04
    assert bound(1, 64) == pytest.approx(2.4414155633e-04, rel=1e-8)


# ------------------------------------------------------------- selection ----
def test_topk_worked_example(golden):
    rows = dict(r.split(None, 1) for r in golden("topk_slide10.txt"))
    scores = np.array([float(v) for v in rows["scores"].split()])
    k = int(rows["k"])
    want = [int(v) for v in rows["selected"].split()]
    assert oracle.topk(scores[None], k)[0].tolist() == want


@pytest.mark.parametrize("N,k,seed", [(1, 1, 0), (7, 3, 1), (50, 10, 2), (64, 64, 3), (200, 17, 4)])
def test_topk_matches_lexsort_with_ties(N, k, seed):
    rng = np.random.default_rng(seed)
    s = rng.integers(-3, 4, size=(5, N)).astype(np.float64)   # many exact ties
    got = oracle.topk(s, k)
    for r in range(5):
        order = np.lexsort((np.arange(N), -s[r]))               # score desc, index asc
        want = np.sort(order[:k])
        assert got[r].tolist() == want.tolist()


def test_topk_invariants_and_nan():
    rng = np.random.default_rng(9)
    s = rng.standard_normal((3, 100))
    s[1, [5, 50]] = np.nan
    idx = oracle.topk(s, 98)
    for r in range(3):
        assert len(set(idx[r].tolist())) == 98 and np.all(np.diff(idx[r]) > 0)
        assert idx[r].min() >= 0 and idx[r].max() < 100
    assert 5 not in idx[1] and 50 not in idx[1]
    assert oracle.topk(s, 100)[0].tolist() == list(range(100))


def test_topk_gap():
    s = np.array([[0.1, 0.8, 0.7, 0.2]])
    assert oracle.topk_gap(s, 2)[0] == pytest.approx(0.5)
    assert math.isinf(oracle.topk_gap(s, 4)[0])


def test_topk_gap_ties_and_empty_selection():
    """A tie across the k-th / (k+1)-th place leaves no margin (gap 0, the row
    is undecidable at any precision); a tie inside the selected set does not
    matter; k = 0 selects nothing and has no boundary (gap infinite)."""
    s = np.array([[0.5, 0.2, 0.5, 0.5],        # k = 2: 0.5, 0.5 | 0.5, 0.2 -> gap 0
                  [0.3, 0.5, 0.5, 0.1]])       # k = 2: 0.5, 0.5 | 0.3      -> gap 0.2
    gap = oracle.topk_gap(s, 2)
    assert gap[0] == 0.0
    assert gap[1] == pytest.approx(0.2)
    assert math.isinf(oracle.topk_gap(s, 0)[0]) and math.isinf(oracle.topk_gap(s, 0)[1])
    # the tie at the boundary still resolves to the lower indices
    assert oracle.topk(s, 2)[0].tolist() == [0, 2]


# -------------------------------------------------------------- attention ---
def _all_keys(x, b, hk):
    """[all gists, all raw tokens chunk by chunk, tail] for one (b, hk), fp64."""
    dt = x.shape.dtype
    N, c, d = x.shape.n_chunks, x.shape.chunk, x.shape.head_dim
    K = np.concatenate([synth.widen(x.k_gist[b, hk], dt), synth.widen(x.k_raw[b, hk], dt).reshape(N * c, d),
                        synth.widen(x.k_tail[b, hk], dt)])
    V = np.concatenate([synth.widen(x.v_gist[b, hk], dt), synth.widen(x.v_raw[b, hk], dt).reshape(N * c, d),
                        synth.widen(x.v_tail[b, hk], dt)])
    return K, V


@pytest.mark.parametrize("mode", [ALL_GISTS, SELECTED_PAIRS])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_full_selection_is_full_attention(mode, dtype):
    """k = N: both modes reduce to softmax attention over every gist, every raw
    token and the tail."""
    sh = small_shape(top_k=6, mode=mode, dtype=dtype)
    x = synth.decode_inputs(sh, 21)
    _, idx, out = oracle.decode(x.tensors(), sh.top_k, mode)
    assert (idx == np.arange(6)).all()
    G = sh.group
    for b in range(sh.batch):
        for hk in range(sh.n_kv_heads):
            K, V = _all_keys(x, b, hk)
            qv = synth.widen(x.q[b, hk * G:(hk + 1) * G], dtype)
            np.testing.assert_allclose(out[b, hk * G:(hk + 1) * G], sdpa(qv, K, V, 1 / math.sqrt(8)),
                                       rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", [ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS])
def test_partial_selection_is_masked_attention(mode):
    """k < N: the gathered context equals full attention under a boolean mask
    that keeps the selected chunks' raw tokens and the tail, and of the gists:
    all (ALL_GISTS), the selected ones (SELECTED_PAIRS), none (SR_ONLY) or
    the unselected ones (UNSELECTED_GISTS); the selection itself equals a
    lexsort top-k."""
    sh = small_shape(n_chunks=9, chunk=4, top_k=3, tail_len=3, mode=mode)
    x = synth.decode_inputs(sh, 33)
    s, idx, out = oracle.decode(x.tensors(), sh.top_k, mode, scale=0.3)
    N, c, G = sh.n_chunks, sh.chunk, sh.group
    for b in range(sh.batch):
        for hk in range(sh.n_kv_heads):
            order = np.lexsort((np.arange(N), -s[b, hk]))
            assert idx[b, hk].tolist() == sorted(order[:3].tolist())
            sel = np.zeros(N, bool)
            sel[idx[b, hk]] = True
            gist_keep = {ALL_GISTS: np.ones(N, bool), SELECTED_PAIRS: sel, SR_ONLY: np.zeros(N, bool),
                         UNSELECTED_GISTS: ~sel}[mode]
            mask = np.concatenate([gist_keep, np.repeat(sel, c), np.ones(sh.tail_len, bool)])
            K, V = _all_keys(x, b, hk)
            qv = synth.widen(x.q[b, hk * G:(hk + 1) * G], "f32")
            want = sdpa(qv, K, V, 0.3, mask=np.broadcast_to(mask, (G, mask.size)))
            np.testing.assert_allclose(out[b, hk * G:(hk + 1) * G], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", [SR_ONLY, UNSELECTED_GISTS])
def test_full_selection_without_gists_is_raw_and_tail_attention(mode):
    """k = N: SR_ONLY keeps no gist and UNSELECTED_GISTS has no unselected
    chunk left, so both reduce to softmax attention over every raw token and
    the tail (library SDPA over that key list)."""
    sh = small_shape(top_k=6, mode=mode)
    x = synth.decode_inputs(sh, 23)
    _, idx, out = oracle.decode(x.tensors(), sh.top_k, mode)
    N, c, d, G = sh.n_chunks, sh.chunk, sh.head_dim, sh.group
    for b in range(sh.batch):
        for hk in range(sh.n_kv_heads):
            K = np.concatenate([synth.widen(x.k_raw[b, hk], "f32").reshape(N * c, d),
                                synth.widen(x.k_tail[b, hk], "f32")])
            V = np.concatenate([synth.widen(x.v_raw[b, hk], "f32").reshape(N * c, d),
                                synth.widen(x.v_tail[b, hk], "f32")])
            qv = synth.widen(x.q[b, hk * G:(hk + 1) * G], "f32")
            np.testing.assert_allclose(out[b, hk * G:(hk + 1) * G], sdpa(qv, K, V, 1 / math.sqrt(d)),
                                       rtol=0, atol=1e-12)


def test_empty_selection_of_the_gist_rules():
    """k = 0: UNSELECTED_GISTS keeps every gist and equals ALL_GISTS (both are
    every gist plus the tail); SR_ONLY keeps the tail alone."""
    sh = small_shape(top_k=0, tail_len=3)
    x = synth.decode_inputs(sh, 25)
    t = x.tensors()
    _, _, a = oracle.decode(t, 0, ALL_GISTS)
    _, _, u = oracle.decode(t, 0, UNSELECTED_GISTS)
    np.testing.assert_array_equal(a, u)
    _, _, r = oracle.decode(t, 0, SR_ONLY)
    G, d = sh.group, sh.head_dim
    for b in range(sh.batch):
        for hk in range(sh.n_kv_heads):
            qv = synth.widen(x.q[b, hk * G:(hk + 1) * G], "f32")
            want = sdpa(qv, synth.widen(x.k_tail[b, hk], "f32"), synth.widen(x.v_tail[b, hk], "f32"),
                        1 / math.sqrt(d))
            np.testing.assert_allclose(r[b, hk * G:(hk + 1) * G], want, rtol=0, atol=1e-12)


def test_unfold_attn_lse_is_library_logsumexp():
    """lse output = torch.logsumexp of the scaled logits over the assembled context."""
    sh = small_shape(n_chunks=7, top_k=3, tail_len=4)
    x = synth.decode_inputs(sh, 45)
    for mode in (ALL_GISTS, SELECTED_PAIRS):
        _, idx, _ = oracle.decode(x.tensors(), sh.top_k, mode, scale=0.7)
        _, lse = oracle.unfold_attn(x.tensors(), idx, mode, scale=0.7, with_lse=True)
        G, c = sh.group, sh.chunk
        for b in range(sh.batch):
            for hk in range(sh.n_kv_heads):
                sel = idx[b, hk]
                gl = np.arange(sh.n_chunks) if mode == ALL_GISTS else sel
                K = np.concatenate([x.k_gist[b, hk][gl], x.k_raw[b, hk][sel].reshape(-1, sh.head_dim),
                                    x.k_tail[b, hk]]).astype(np.float64)
                for g in range(G):
                    logits = 0.7 * torch.from_numpy(K) @ torch.from_numpy(x.q[b, hk * G + g].astype(np.float64))
                    assert lse[b, hk * G + g] == pytest.approx(torch.logsumexp(logits, 0).item(), abs=1e-12)


def test_unfold_attn_equals_decode_for_same_selection():
    sh = small_shape()
    x = synth.decode_inputs(sh, 41)
    for mode in (ALL_GISTS, SELECTED_PAIRS):
        _, idx, out = oracle.decode(x.tensors(), sh.top_k, mode)
        np.testing.assert_array_equal(oracle.unfold_attn(x.tensors(), idx, mode), out)


def test_empty_selection_is_tail_attention_and_single_key_returns_value():
    sh = small_shape(top_k=0, mode=SELECTED_PAIRS, tail_len=5)
    x = synth.decode_inputs(sh, 43)
    _, _, out = oracle.decode(x.tensors(), 0, SELECTED_PAIRS)
    G = sh.group
    for b in range(sh.batch):
        for hk in range(sh.n_kv_heads):
            want = sdpa(x.q[b, hk * G:(hk + 1) * G].astype(np.float64), x.k_tail[b, hk].astype(np.float64),
                        x.v_tail[b, hk].astype(np.float64), 1 / math.sqrt(8))
            np.testing.assert_allclose(out[b, hk * G:(hk + 1) * G], want, rtol=0, atol=1e-12)
    sh1 = small_shape(top_k=0, mode=SELECTED_PAIRS, tail_len=1)
    x1 = synth.decode_inputs(sh1, 44)
    _, _, out1 = oracle.decode(x1.tensors(), 0, SELECTED_PAIRS)
    for b in range(2):
        for h in range(4):
            np.testing.assert_array_equal(out1[b, h], x1.v_tail[b, h // 2, 0].astype(np.float64))


def test_weights_sum_to_one():
    sh = small_shape(n_chunks=12, top_k=4)
    x = synth.decode_inputs(sh, 47)
    t = x.tensors()
    for name in ("v_gist", "v_raw", "v_tail"):
        t[name] = np.ones_like(t[name])
    for mode in (ALL_GISTS, SELECTED_PAIRS):
        _, _, out = oracle.decode(t, sh.top_k, mode)
        np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


def test_strong_needles_are_always_selected():
    """needle gist key = alpha * qbar/|qbar| + noise with alpha = 3*sqrt(d):
    every planted needle chunk is in the selected set (k = #needles)."""
    sh = DecodeShape(2, 8, 2, 64, 300, 4, 6, 4, "bf16", ALL_GISTS, n_needles=6, needle_alpha=3 * 8.0)
    x = synth.decode_inputs(sh, 51)
    _, idx, _ = oracle.decode(x.tensors(), sh.top_k)
    for r in range(sh.rows):
        assert sorted(x.needles[r].tolist()) == idx.reshape(sh.rows, -1)[r].tolist()


# -------------------------------------------------------------- hierarchy ---
def _hier_small(n1=40, group=4, c=2, k2=3, k1=4, W=2, seed=61, d=8):
    n2 = -(-n1 // group)
    h = HierShape(DecodeShape(1, 4, 2, d, n1, c, k1, W, "f32", ALL_GISTS), n_l2=n2, group=group, top_k2=k2)
    return h, synth.hier_inputs(h, seed)


def test_hier_full_level2_selection_equals_flat_selection():
    """k2 = n_l2: every level-1 gist is a candidate, so the level-1 selection
    equals flat top-k1, and the context is every meta-gist + every gist + raw
    of the selection + tail."""
    h, x = _hier_small(n1=39, group=4, k2=10)
    t = x.tensors()
    idx2, idx1, out = oracle.hier_decode(t, h.group, h.top_k2, h.l1.top_k)
    assert idx2[0, 0].tolist() == list(range(10))
    flat_s = oracle.gist_scores(x.q, x.k_g1)
    np.testing.assert_array_equal(idx1, oracle.topk(flat_s, h.l1.top_k))
    G, c, d = 2, h.l1.chunk, h.l1.head_dim
    for hk in range(2):
        sel = idx1[0, hk]
        K = np.concatenate([x.k_g2[0, hk], x.k_g1[0, hk], x.k_raw[0, hk][sel].reshape(-1, d), x.k_tail[0, hk]])
        V = np.concatenate([x.v_g2[0, hk], x.v_g1[0, hk], x.v_raw[0, hk][sel].reshape(-1, d), x.v_tail[0, hk]])
        want = sdpa(x.q[0, hk * G:(hk + 1) * G].astype(np.float64), K.astype(np.float64), V.astype(np.float64),
                    1 / math.sqrt(d))
        np.testing.assert_allclose(out[0, hk * G:(hk + 1) * G], want, rtol=0, atol=1e-12)


def test_hier_slide11_parent_child_mapping(golden):
    """Slide 11: 100 raw tokens per gist, 10 gists per meta-gist.  Forcing the
    level-2 selection to G2 makes the candidates exactly g11..g20."""
    rows = dict(r.split(None, 1) for r in golden("hierarchy_slide11.txt"))
    c, n1, group = int(rows["chunk"]), int(rows["n_gists"]), int(rows["group"])
    lo, hi = (int(v) for v in rows["G2_children_range0"].split())
    assert int(rows["n_meta"]) == n1 // group
    d = 4
    h = HierShape(DecodeShape(1, 1, 1, d, n1, c, 3, 1, "f32", ALL_GISTS), n_l2=n1 // group, group=group, top_k2=1)
    x = synth.hier_inputs(h, 71)
    x.q[...] = np.float32([1.0, 0.5, -0.25, 0.125])
    x.k_g2[0, 0, 1] = np.float32(50.0) * x.q[0, 0]          # G2 (0-based 1) dominates level 2
    idx2, idx1, out = oracle.hier_decode(x.tensors(), group, 1, 3)
    assert idx2[0, 0].tolist() == [1]
    assert all(lo <= j < hi for j in idx1[0, 0])
    s1 = oracle.gist_scores(x.q, x.k_g1)[0, 0, lo:hi]
    assert idx1[0, 0].tolist() == sorted((lo + np.lexsort((np.arange(10), -s1))[:3]).tolist())
    sel = idx1[0, 0]
    K = np.concatenate([x.k_g2[0, 0], x.k_g1[0, 0, lo:hi], x.k_raw[0, 0][sel].reshape(-1, d), x.k_tail[0, 0]])
    V = np.concatenate([x.v_g2[0, 0], x.v_g1[0, 0, lo:hi], x.v_raw[0, 0][sel].reshape(-1, d), x.v_tail[0, 0]])
    want = sdpa(x.q[0].astype(np.float64), K.astype(np.float64), V.astype(np.float64), 0.5)
    np.testing.assert_allclose(out[0], want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- prefill ---
def _slide7_names(c=2, n=3):
    names = []
    for j in range(n):
        names += [f"x{j * c + u + 1}" for u in range(c)] + [f"g{j + 1}"]
    return names


def test_mask_matches_slide7_table(golden):
    names = _slide7_names()
    pos = {nm: p for p, nm in enumerate(names)}
    for line in golden("gist_mask_slide7.txt"):
        kind, rest = line.split(None, 1)
        qn, keys = rest.split(":")
        allowed = set(keys.split())
        p = pos[qn]
        got = {names[t] for t in range(len(names)) if oracle.gist_mask(p, t, 2)}
        assert got == allowed, (kind, qn, got, allowed)


def test_mask_layout_slide3(golden):
    rows = dict(r.split() for r in golden("layout_slide3.txt"))
    c = int(rows["chunk"])
    g1, t17, g2, t33 = (int(rows[k]) for k in ("gist1", "token17", "gist2", "token33"))
    assert [t for t in range(g1 + 1) if oracle.gist_mask(g1, t, c)] == list(range(int(rows["token1"]), int(rows["token16"]) + 1)) + [g1]
    assert [t for t in range(t17 + 1) if oracle.gist_mask(t17, t, c)] == [g1, t17]
    assert [t for t in range(g2 + 1) if oracle.gist_mask(g2, t, c)] == [g1] + list(range(t17, int(rows["token32"]) + 1)) + [g2]
    assert [t for t in range(t33 + 1) if oracle.gist_mask(t33, t, c)] == [g1, g2, t33]
    assert oracle.gist_mask(int(rows["gist3"]), g2, c)


def _pairs_closed_form(N, c):
    """gist->earlier gists + gist->self + gist->own raw + raw->earlier gists + raw->own-chunk causal."""
    return N * (N - 1) // 2 + N + N * c + c * N * (N - 1) // 2 + N * c * (c + 1) // 2


@pytest.mark.parametrize("N,c", [(1, 1), (1, 5), (3, 2), (4, 1), (7, 3), (12, 16)])
def test_pair_count_closed_form_small(N, c):
    assert oracle.prefill_pair_count(N, c) == _pairs_closed_form(N, c)


def test_pair_count_full_prefill_size():
    assert _pairs_closed_form(1024, 16) == 9_060_864
    assert oracle.prefill_pair_count(1024, 16) == 9_060_864


def test_mask_c1_closed_form():
    """c = 1: x_j (p = 2j) sees g_i for i < j and itself; g_j (p = 2j+1) sees g_i
    for i < j, x_j and itself."""
    N = 6
    for p in range(2 * N):
        j = p // 2
        want = {2 * i + 1 for i in range(j)} | {p}
        if p % 2 == 1:
            want |= {2 * j}
        assert {t for t in range(2 * N) if oracle.gist_mask(p, t, 1)} == want


def test_prefill_single_chunk_is_causal_attention():
    """N = 1: the mask is the plain causal mask over the c + 1 positions."""
    p = synth.PrefillShape(1, 2, 1, 8, 1, 6, "f32")
    x = synth.prefill_inputs(p, 81)
    P = p.positions
    rows = np.array([(0, h, t) for h in range(2) for t in range(P)], np.int64)
    out = oracle.prefill_rows(x.tensors(), 1, 6, rows).reshape(2, P, 8)
    k = np.repeat(x.k.astype(np.float64), 2, axis=1)[0]
    v = np.repeat(x.v.astype(np.float64), 2, axis=1)[0]
    want = sdpa(x.q[0].astype(np.float64), k, v, 1 / math.sqrt(8), causal=True)
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)


def test_prefill_matches_sdpa_under_slide7_mask(golden):
    """Masked library attention with the slide-7 table (c = 2, three chunks),
    grouped-query heads: head h reads KV head h // (Hq / Hkv)."""
    names = _slide7_names()
    pos = {nm: p for p, nm in enumerate(names)}
    P = len(names)
    M = np.zeros((P, P), bool)
    for line in golden("gist_mask_slide7.txt"):
        qn, keys = line.split(None, 1)[1].split(":")
        for kn in keys.split():
            M[pos[qn], pos[kn]] = True
    p = synth.PrefillShape(1, 4, 2, 8, 3, 2, "bf16")
    x = synth.prefill_inputs(p, 91)
    rows = np.array([(0, h, t) for h in range(4) for t in range(P)], np.int64)
    out = oracle.prefill_rows(x.tensors(), 3, 2, rows, scale=0.2).reshape(4, P, 8)
    k = np.repeat(synth.widen(x.k, "bf16"), 2, axis=1)[0]
    v = np.repeat(synth.widen(x.v, "bf16"), 2, axis=1)[0]
    want = sdpa(synth.widen(x.q, "bf16")[0], k, v, 0.2, mask=np.broadcast_to(M, (4, P, P)))
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)


def test_hier_given_selection_reproduces_own_selection():
    """Evaluating the attention for the oracle's own selection gives the same output."""
    h, x = _hier_small(n1=41, group=4, k2=3, k1=5)
    t = x.tensors()
    idx2, idx1, out = oracle.hier_decode(t, h.group, h.top_k2, h.l1.top_k)
    _, _, out2 = oracle.hier_decode(t, h.group, h.top_k2, h.l1.top_k, given=(idx2, idx1))
    np.testing.assert_array_equal(out, out2)


# ------------------------------------------------------------------ top-p ----
def test_topp_slide10_scores_by_hand():
    """Slide 10's scores 0.1 / 0.8 / 0.7 / 0.2 under softmax with scale 1.
    By hand: e^0.1 = 1.1051709, e^0.8 = 2.2255409, e^0.7 = 2.0137527,
    e^0.2 = 1.2214028, sum 6.5658673, so the masses are 0.168321, 0.338957,
    0.306700, 0.186022.  In score order (g2, g3, g4, g1) they accumulate to
    0.338957, 0.645657, 0.831679, 1."""
    s = np.array([[0.1, 0.8, 0.7, 0.2]])
    cases = [(0.30, [1]), (0.60, [1, 2]), (0.65, [1, 2, 3]), (0.83, [1, 2, 3]), (0.84, [0, 1, 2, 3])]
    for p, want in cases:
        idx, cnt = oracle.topp(s, p, 4, 1.0)
        assert cnt[0] == len(want), p
        assert idx[0, :cnt[0]].tolist() == want, p
        assert (idx[0, cnt[0]:] == -1).all()
    # cut at kmax: p = 0.9 would need all four
    idx, cnt = oracle.topp(s, 0.9, 2, 1.0)
    assert cnt[0] == 2 and idx[0].tolist() == [1, 2]


def test_topp_uniform_mass_closed_form():
    """scale 0 makes every chunk weigh 1/N: the count is ceil(p N), taken in
    the top-k order (lexsort)."""
    rng = np.random.default_rng(3)
    s = rng.standard_normal((4, 10))
    for p, m in [(0.35, 4), (0.05, 1), (0.5, 5), (0.91, 10)]:
        idx, cnt = oracle.topp(s, p, 10, 0.0)
        assert (cnt == m).all(), p
        for r in range(4):
            want = np.sort(np.lexsort((np.arange(10), -s[r]))[:m])
            assert idx[r, :m].tolist() == want.tolist()


def test_topp_is_the_shortest_prefix_reaching_p():
    """Invariants on random rows against library routines (softmax of the
    scaled scores, lexsort order): the selected mass reaches p, the mass
    without the last chunk of the prefix does not, and the set is that prefix."""
    rng = np.random.default_rng(11)
    s = rng.standard_normal((50, 64)) * 3.0
    s[::7, 5] = s[::7, 9]                      # ties
    scale = 0.7
    for p in (0.2, 0.5, 0.9, 0.99):
        idx, cnt = oracle.topp(s, p, 64, scale)
        for r in range(50):
            w = np.exp(scale * (s[r] - s[r].max()))
            w /= w.sum()
            order = np.lexsort((np.arange(64), -s[r]))
            m = int(cnt[r])
            assert w[order[:m]].sum() >= p - 1e-12
            assert m == 1 or w[order[:m - 1]].sum() < p
            assert idx[r, :m].tolist() == np.sort(order[:m]).tolist()


def test_padded_selection_equals_the_compacted_one():
    """A selection padded with -1 (variable size, as top-p returns it) attends
    exactly the context of its non-negative entries."""
    sh = small_shape(n_chunks=9, chunk=4, top_k=4, tail_len=3)
    x = synth.decode_inputs(sh, 47)
    t = x.tensors()
    full = np.array([[[1, 4, 6, 8], [0, 2, 3, 7]], [[2, 5, -1, -1], [8, -1, -1, -1]]], np.int32)
    for mode in (ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS):
        out = oracle.unfold_attn(t, full, mode, 0.4)
        for b in range(2):
            for hk in range(2):
                kept = full[b, hk][full[b, hk] >= 0]
                one = {k: v[b:b + 1, hk:hk + 1].copy() for k, v in t.items()}
                one["q"] = t["q"][b:b + 1, hk * sh.group:(hk + 1) * sh.group].copy()
                sub = dataclasses.replace(sh, top_k=len(kept))
                want = oracle.unfold_attn(one, kept.reshape(1, 1, -1), mode, 0.4)
                np.testing.assert_array_equal(out[b, hk * sh.group:(hk + 1) * sh.group], want[0])


# ------------------------------------------------------------ paged cache ----
def _paged_small(seq_chunks=None, mode=ALL_GISTS, k=3, dt="f32", seed=71):
    base = small_shape(n_chunks=10, top_k=k, mode=mode, dtype=dt, n_needles=2)
    ps = synth.PagedShape(base, n_docs=4, doc_min=2, doc_max=5, spare_pages=2)
    return ps, synth.paged_inputs(ps, seed, seq_chunks)


@pytest.mark.parametrize("mode", [ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS])
def test_paged_full_sequences_equal_the_gathered_dense_cache(mode):
    """Every sequence N chunks long: decoding over the page pool equals
    decoding over the raw cache gathered through the table by numpy
    indexing (bit for bit: the same keys in the same order)."""
    ps, x = _paged_small([10, 10], mode)
    kr, vr = x.dense_raw()
    t = dict(x.tensors(), k_raw=kr, v_raw=vr)
    s0, i0, o0 = oracle.decode(t, 3, mode)
    s1, i1, o1 = oracle.decode_paged(x.tensors(), x.k_pages, x.v_pages, x.table, 3, mode,
                                     seq_chunks=x.seq_chunks)
    np.testing.assert_array_equal(s0, s1)
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_array_equal(o0, o1)


@pytest.mark.parametrize("mode", [ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS])
@pytest.mark.parametrize("chunks", [(7, 10), (2, 0), (1, 5)])
def test_paged_short_sequence_is_the_truncated_problem(mode, chunks):
    """Sequence b with nb < N chunks: its scores, selection and output are
    those of a one-sequence dense problem with N = nb and k = min(k, nb)
    (sliced arrays), its scores past nb are -inf and its selection is padded
    with -1; the decoy gists past nb (needles twice as strong) are ignored."""
    ps, x = _paged_small(list(chunks), mode)
    kr, vr = x.dense_raw()
    s1, i1, o1 = oracle.decode_paged(x.tensors(), x.k_pages, x.v_pages, x.table, 3, mode,
                                     seq_chunks=x.seq_chunks)
    G = ps.base.group
    for b, n in enumerate(chunks):
        kk = min(3, n)
        sl = lambda a: np.ascontiguousarray(a[b:b + 1, :, :n])
        t = dict(q=np.ascontiguousarray(x.q[b:b + 1]), k_gist=sl(x.k_gist), v_gist=sl(x.v_gist),
                 k_raw=sl(kr), v_raw=sl(vr), k_tail=np.ascontiguousarray(x.k_tail[b:b + 1]),
                 v_tail=np.ascontiguousarray(x.v_tail[b:b + 1]))
        s0, i0, o0 = oracle.decode(t, kk, mode)
        np.testing.assert_array_equal(s1[b, :, :n], s0[0])
        assert np.all(s1[b, :, n:] == -np.inf)
        np.testing.assert_array_equal(i1[b, :, :kk], i0[0])
        assert np.all(i1[b, :, kk:] == -1)
        np.testing.assert_array_equal(o1[b], o0[0])


def test_paged_sequences_sharing_a_document_see_the_same_raw_keys():
    """Two sequences whose tables name the same page read the same bytes: a
    pool page changed in place changes the output of both and nothing else."""
    ps, x = _paged_small([10, 10], SR_ONLY, k=10)
    common = sorted(set(x.table[0].tolist()) & set(x.table[1].tolist()))
    assert common, "the draw gives the two sequences a shared document"
    _, _, o0 = oracle.decode_paged(x.tensors(), x.k_pages, x.v_pages, x.table, 10, SR_ONLY)
    vp = x.v_pages.copy()
    vp[common[0]] += 1.0
    _, _, o1 = oracle.decode_paged(x.tensors(), x.k_pages, vp, x.table, 10, SR_ONLY)
    assert np.all(np.abs(o1 - o0).max(axis=(1, 2)) > 0)
    unused = sorted(set(range(x.k_pages.shape[0])) - set(x.table[x.table >= 0].tolist()))
    assert unused
    vp = x.v_pages.copy()
    vp[unused] += 1.0
    _, _, o2 = oracle.decode_paged(x.tensors(), x.k_pages, vp, x.table, 10, SR_ONLY)
    np.testing.assert_array_equal(o2, o0)


# ---------------------------------------------------- deeper hierarchy -----
def _levels(x, h):
    return oracle.hier_levels(x.q, x.k_g, x.v_g, x.k_raw, x.v_raw, x.k_tail, x.v_tail, h.groups,
                              (h.l1.top_k,) + tuple(h.top_ks))


def test_levels_depth_two_is_the_two_level_hierarchy():
    """L = 2 is the two-level step (pinned above) bit for bit."""
    h2, x2 = _hier_small(n1=41, group=4, k2=3, k1=4)
    hl = synth.LevelsShape(h2.l1, (4,), (3,))
    idx, out = oracle.hier_levels(x2.q, [x2.k_g1, x2.k_g2], [x2.v_g1, x2.v_g2], x2.k_raw, x2.v_raw, x2.k_tail,
                                  x2.v_tail, hl.groups, (4, 3))
    i2, i1, o = oracle.hier_decode(x2.tensors(), 4, 3, 4)
    np.testing.assert_array_equal(idx[1], i2)
    np.testing.assert_array_equal(idx[0], i1)
    np.testing.assert_array_equal(out, o)


def test_levels_three_worked_example_by_hand():
    """Eight chunks, groups of two at both levels (n = 8, 4, 2), k = 1 at
    every level, q = e0 so a score is the key's first coordinate.  Level 3
    scores (1, 5) pick gist 1, whose children are level-2 gists 2, 3; these
    score (2, 3) and 3 wins although gists 0, 1 score 9 (they are not
    candidates); its children, chunks 6 and 7, score (1, 4): chunk 7.  The
    context is level-3 {0, 1}, level-2 {2, 3}, level-1 {6, 7}, chunk 7's raw
    token and the tail, listed here by hand for library SDPA."""
    d = 4
    h = synth.LevelsShape(DecodeShape(1, 1, 1, d, 8, 1, 1, 1, "f32"), (2, 2), (1, 1))
    x = synth.levels_inputs(h, 83)
    x.q[...] = np.float32([1, 0, 0, 0])
    for lv, first in ((0, [8, 8, 8, 8, 8, 8, 1, 4]), (1, [9, 9, 2, 3]), (2, [1, 5])):
        x.k_g[lv][0, 0, :, 0] = np.float32(first)
    idx, out = _levels(x, h)
    assert [i[0, 0].tolist() for i in idx] == [[7], [3], [1]]
    K = np.concatenate([x.k_g[2][0, 0, [0, 1]], x.k_g[1][0, 0, [2, 3]], x.k_g[0][0, 0, [6, 7]], x.k_raw[0, 0, 7],
                        x.k_tail[0, 0]])
    V = np.concatenate([x.v_g[2][0, 0, [0, 1]], x.v_g[1][0, 0, [2, 3]], x.v_g[0][0, 0, [6, 7]], x.v_raw[0, 0, 7],
                        x.v_tail[0, 0]])
    want = sdpa(x.q[0].astype(np.float64), K.astype(np.float64), V.astype(np.float64), 0.5)
    np.testing.assert_allclose(out[0], want, rtol=0, atol=1e-12)


def test_levels_with_every_upper_group_selected_and_silent_is_flat_decode():
    """Depth 4, every upper level selects all of its candidates and its gist
    keys point against the query (logits near -1e4: weight exactly 0 in
    fp64): the candidates of level 1 are all gists, so the step is the flat
    decode step (pinned above) over the level-1 gists."""
    d, n1 = 8, 50
    h = synth.LevelsShape(DecodeShape(2, 2, 2, d, n1, 3, 5, 2, "f32", n_needles=0), (4, 3, 2), (13, 5, 3))
    assert h.counts == [50, 13, 5, 3]
    x = synth.levels_inputs(h, 84)
    qw = x.q.astype(np.float64)
    for lv in (1, 2, 3):
        for b in range(2):
            for hk in range(2):
                x.k_g[lv][b, hk, :] = (-1e4 * qw[b, hk] / np.linalg.norm(qw[b, hk])).astype(np.float32)
    idx, out = _levels(x, h)
    for lv, cnt in ((1, 13), (2, 5), (3, 3)):
        assert np.all(idx[lv] == np.arange(cnt))
    t = dict(q=x.q, k_gist=x.k_g[0], v_gist=x.v_g[0], k_raw=x.k_raw, v_raw=x.v_raw, k_tail=x.k_tail,
             v_tail=x.v_tail)
    _, i_flat, o_flat = oracle.decode(t, 5, ALL_GISTS)
    np.testing.assert_array_equal(idx[0], i_flat)
    np.testing.assert_allclose(out, o_flat, rtol=0, atol=1e-13)


def test_levels_selection_follows_the_tree_and_finds_needle_chains():
    """Each level's selection lies among the children of the level above's,
    ascending and distinct; the planted needle chains are found at every
    level (one needle chunk per selected top-level gist)."""
    h = synth.LevelsShape(DecodeShape(2, 4, 2, 16, 300, 2, 4, 3, "f32", n_needles=3), (5, 4), (6, 3))
    x = synth.levels_inputs(h, 85)
    idx, _ = _levels(x, h)
    for lv in (0, 1):
        g = h.groups[lv]
        for r in range(4):
            b, hk = divmod(r, 2)
            sel, par = idx[lv][b, hk], idx[lv + 1][b, hk]
            assert np.all(np.diff(sel) > 0)
            assert set((sel // g).tolist()) <= set(par.tolist())
    for r in range(4):
        b, hk = divmod(r, 2)
        assert set(x.needles[r].tolist()) <= set(idx[0][b, hk].tolist())


def test_levels_given_selection_reproduces_own_selection():
    h = synth.LevelsShape(DecodeShape(1, 4, 2, 16, 120, 2, 4, 3, "f32", n_needles=2), (4, 3), (5, 3))
    x = synth.levels_inputs(h, 86)
    idx, out = _levels(x, h)
    idx2, out2 = oracle.hier_levels(x.q, x.k_g, x.v_g, x.k_raw, x.v_raw, x.k_tail, x.v_tail, h.groups,
                                    (h.l1.top_k,) + tuple(h.top_ks), given=idx)
    np.testing.assert_array_equal(out, out2)


# ------------------------------------------- stage-2 suffix forward --------
def _suffix_small(mode=ALL_GISTS, S=5, k=2, seed=91, dt="f32"):
    ss = synth.SuffixShape(small_shape(n_chunks=7, top_k=k, tail_len=S, mode=mode, dtype=dt, n_needles=1))
    return ss, synth.suffix_inputs(ss, seed)


@pytest.mark.parametrize("mode", [ALL_GISTS, SELECTED_PAIRS, SR_ONLY, UNSELECTED_GISTS])
def test_suffix_position_is_a_decode_step_with_the_causal_tail(mode):
    """Suffix position p is the decode step (pinned above) of query q[:, p]
    with the suffix tokens 0..p as the tail: scores, selection and output
    bit for bit."""
    ss, x = _suffix_small(mode)
    sc, idx, out = oracle.suffix_attn(x.q, x.k_gist, x.v_gist, x.k_raw, x.v_raw, x.k_suf, x.v_suf, 2, mode)
    for p in range(ss.base.tail_len):
        t = dict(q=np.ascontiguousarray(x.q[:, p]), k_gist=x.k_gist, v_gist=x.v_gist, k_raw=x.k_raw,
                 v_raw=x.v_raw, k_tail=np.ascontiguousarray(x.k_suf[:, :, :p + 1]),
                 v_tail=np.ascontiguousarray(x.v_suf[:, :, :p + 1]))
        s0, i0, o0 = oracle.decode(t, 2, mode)
        np.testing.assert_array_equal(sc[:, :, p], s0)
        np.testing.assert_array_equal(idx[:, :, p], i0)
        np.testing.assert_array_equal(out[:, p], o0)


def test_suffix_slide10_worked_example():
    """Slide 10: four chunks whose gists score 0.1, 0.8, 0.7, 0.2 against the
    suffix token; top-2 unfolds chunks 2 and 3 (0-based 1, 2).  The context
    (every gist, the raw tokens of chunks 1 and 2, the suffix so far) is
    listed here by hand for library SDPA."""
    d, c = 4, 2
    ss = synth.SuffixShape(DecodeShape(1, 1, 1, d, 4, c, 2, 2, "f32"))
    x = synth.suffix_inputs(ss, 92)
    x.q[...] = np.float32([1, 0, 0, 0])
    x.k_gist[0, 0, :, 0] = np.float32([0.1, 0.8, 0.7, 0.2])
    x.k_gist[0, 0, :, 1:] = 0
    sc, idx, out = oracle.suffix_attn(x.q, x.k_gist, x.v_gist, x.k_raw, x.v_raw, x.k_suf, x.v_suf, 2)
    np.testing.assert_allclose(sc[0, 0, 0], np.float32([0.1, 0.8, 0.7, 0.2]), rtol=0, atol=0)
    assert idx[0, 0].tolist() == [[1, 2], [1, 2]]
    for p in range(2):
        K = np.concatenate([x.k_gist[0, 0], x.k_raw[0, 0, [1, 2]].reshape(-1, d), x.k_suf[0, 0, :p + 1]])
        V = np.concatenate([x.v_gist[0, 0], x.v_raw[0, 0, [1, 2]].reshape(-1, d), x.v_suf[0, 0, :p + 1]])
        want = sdpa(x.q[0, p].astype(np.float64), K.astype(np.float64), V.astype(np.float64), 0.5)
        np.testing.assert_allclose(out[0, p], want, rtol=0, atol=1e-12)


def test_suffix_is_causal():
    """Changing suffix token t's key and value changes the outputs of
    positions >= t and leaves the earlier ones bit for bit."""
    ss, x = _suffix_small(S=6)
    _, _, o0 = oracle.suffix_attn(x.q, x.k_gist, x.v_gist, x.k_raw, x.v_raw, x.k_suf, x.v_suf, 2)
    ks, vs = x.k_suf.copy(), x.v_suf.copy()
    ks[:, :, 3] += 1.0
    vs[:, :, 3] -= 2.0
    _, _, o1 = oracle.suffix_attn(x.q, x.k_gist, x.v_gist, x.k_raw, x.v_raw, ks, vs, 2)
    np.testing.assert_array_equal(o1[:, :3], o0[:, :3])
    assert np.all(np.abs(o1[:, 3:] - o0[:, 3:]).max(axis=(2, 3)) > 0)


def test_prefill_lse_is_library_logsumexp():
    """The prefill rows' log-normaliser is torch.logsumexp of the scaled
    logits over the keys the slide-7 mask allows (mask from the slide's
    table, not from the oracle)."""
    c, n = 2, 3
    p = synth.PrefillShape(1, 2, 1, 8, n, c, "f32", 0.3)
    x = synth.prefill_inputs(p, 93)
    P = p.positions
    rows = np.array([(0, h, t) for h in range(2) for t in range(P)], np.int64)
    _, lse = oracle.prefill_rows(x.tensors(), n, c, rows, 0.3, with_lse=True)
    names = _slide7_names(c, n)
    allowed = {"x1": ["x1"], "x2": ["x1", "x2"], "g1": ["x1", "x2", "g1"], "x3": ["g1", "x3"],
               "x4": ["g1", "x3", "x4"], "g2": ["g1", "x3", "x4", "g2"], "x5": ["g1", "g2", "x5"],
               "x6": ["g1", "g2", "x5", "x6"], "g3": ["g1", "g2", "x5", "x6", "g3"]}
    k = torch.from_numpy(x.k[0, 0].astype(np.float64))
    for i, (_, h, t) in enumerate(rows):
        keys = [names.index(nm) for nm in allowed[names[t]]]
        logits = 0.3 * (k[keys] @ torch.from_numpy(x.q[0, h, t].astype(np.float64)))
        assert lse[i] == pytest.approx(torch.logsumexp(logits, 0).item(), abs=1e-12)


def test_topp_ties_take_the_lower_index_first():
    """Equal scores enter the prefix lowest index first: scores (1, 3, 1, 3, 1)
    with scale ln 2 give weights (2, 8, 2, 8, 2) / 22.  In order 1, 3, 0, 2, 4
    the masses accumulate to 8/22, 16/22, 18/22, 20/22, 1, so p = 0.8 stops at
    the third chunk (index 0, the lowest of the tied ones), p = 0.85 at the
    fourth (index 2)."""
    s = np.array([[1.0, 3.0, 1.0, 3.0, 1.0]])
    for p, want in ((0.30, [1]), (0.70, [1, 3]), (0.80, [0, 1, 3]), (0.85, [0, 1, 2, 3]), (0.95, [0, 1, 2, 3, 4])):
        idx, cnt = oracle.topp(s, p, 5, math.log(2.0))
        assert idx[0, :cnt[0]].tolist() == want, p
        assert (idx[0, cnt[0]:] == -1).all()


def test_levels_ragged_groups_reduce_to_the_two_level_step():
    """Ragged groups at every level (301 -> 61 -> 16 gists: the last groups
    hold 1 and 1 children).  With every level-3 gist selected and its keys
    silenced (weight exactly 0 in fp64), the three-level step is the
    two-level step (pinned above) over levels 2 and 1, bit for bit."""
    d = 8
    h = synth.LevelsShape(DecodeShape(1, 2, 2, d, 301, 2, 4, 3, "f32", n_needles=0), (5, 4), (6, 16))
    assert h.counts == [301, 61, 16]
    x = synth.levels_inputs(h, 87)
    qw = x.q.astype(np.float64)
    for hk in range(2):
        x.k_g[2][0, hk, :] = (-1e4 * qw[0, hk] / np.linalg.norm(qw[0, hk])).astype(np.float32)
    idx, out = _levels(x, h)
    assert np.all(idx[2] == np.arange(16))
    t = dict(q=x.q, k_g2=x.k_g[1], v_g2=x.v_g[1], k_g1=x.k_g[0], v_g1=x.v_g[0], k_raw=x.k_raw, v_raw=x.v_raw,
             k_tail=x.k_tail, v_tail=x.v_tail)
    i2, i1, o = oracle.hier_decode(t, 5, 6, 4)
    np.testing.assert_array_equal(idx[1], i2)
    np.testing.assert_array_equal(idx[0], i1)
    np.testing.assert_allclose(out, o, rtol=0, atol=1e-13)
