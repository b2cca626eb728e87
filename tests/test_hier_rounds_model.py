"""Host model of the tensor-core step's hierarchy rounds, checked against the
oracle's descent on CPU.

The kernel descends one 128-row tile per level: round 0 lays out the
children of the top level's selection group after group (rows past a short
last group are empty), the tile's scores become selection keys (an empty row
the lowest key), the next round selects among the first kp * g rows and maps
each selected row back to its gist (parent[row / g] * g + row % g), and the
last round takes the raw tokens of the level-1 selection.  Selections live in
two shared buffers that rounds use in turn.  This model follows those index
rules (not the oracle's candidate lists) and must reach the oracle's
selections at every level, on many ragged shapes, including the case where
the tile is full and where the last group is short.
"""
import numpy as np
import pytest

import oracle
import synth
from synth import DecodeShape, LevelsShape

TILE = 128


def _order_keys(scores: np.ndarray) -> np.ndarray:
    """Monotone 32-bit keys of fp32 scores (an empty row gets 0, below all)."""
    f = scores.astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    neg = (u >> 31) == 1
    return np.where(neg, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)


def _top_k_positions(keys: np.ndarray, k: int) -> np.ndarray:
    """Exact top-k of the keys, ties to the lower position, ascending."""
    pos = np.arange(len(keys))
    order = np.lexsort((pos, -keys.astype(np.int64)))
    return np.sort(order[:k])


def model_descent(scores_by_level, counts, groups, ks):
    """scores_by_level[l]: the exact fp64 scores of level l + 1's gists (one
    row).  Returns the selection of every level (level 1 first) the way the
    kernel's rounds produce it."""
    L = len(counts)
    bufs = [None, None]                                  # the two shared selection buffers
    sel = {}
    # round 0: the top level's selection over all its gists
    top = _top_k_positions(_order_keys(scores_by_level[L - 1]), ks[L - 1])
    sel[L] = top
    bufs[0] = top
    for rd in range(1, L):
        lv = L - rd                                      # level selected this round
        par = bufs[(rd - 1) & 1]
        g, nch = groups[lv - 1], counts[lv - 1]
        kp = len(par)
        # the children tile of round rd - 1
        keys = np.zeros(TILE, np.uint64)
        child_of = np.full(TILE, -1)
        for r in range(min(TILE, kp * g)):
            child = par[r // g] * g + r % g
            if child < nch:
                child_of[r] = child
                keys[r] = _order_keys(np.array([scores_by_level[lv - 1][child]]))[0]
        n = min(TILE, kp * g)
        picked = _top_k_positions(keys[:n], ks[lv - 1])
        assert np.all(child_of[picked] >= 0), "an empty row was selected"
        out = np.array([par[p // g] * g + p % g for p in picked])
        sel[lv] = out
        bufs[rd & 1] = out
    return [sel[l] for l in range(1, L + 1)]


@pytest.mark.parametrize("n1,groups,top_ks,k1,seed", [
    (4096, (8, 8), (16, 4), 8, 1),          # full tiles at every level
    (301, (5, 4), (6, 3), 4, 2),            # ragged groups at both levels
    (1000, (8, 8, 8), (16, 8, 2), 8, 3),    # four levels
    (999, (7, 3, 5), (9, 4, 2), 5, 4),      # four levels, ragged everywhere
    (130, (2,), (64,), 16, 5),              # two levels, a full 128-row children tile
    (8192, (16, 16), (8, 8), 8, 6),         # the three-level workload's groups
])
def test_kernel_rounds_reach_the_oracle_selections(n1, groups, top_ks, k1, seed):
    h = LevelsShape(DecodeShape(2, 4, 2, 16, n1, 2, k1, 2, "f32", n_needles=2), groups, top_ks)
    x = synth.levels_inputs(h, 700 + seed)
    ks = (k1,) + tuple(top_ks)
    idx, _ = oracle.hier_levels(x.q, x.k_g, x.v_g, x.k_raw, x.v_raw, x.k_tail, x.v_tail, groups, ks)
    scores = [oracle.gist_scores(x.q, kg) for kg in x.k_g]     # [B, Hkv, n_l] per level
    counts = h.counts
    for b in range(2):
        for hk in range(2):
            per_level = [sc[b, hk] for sc in scores]
            got = model_descent(per_level, counts, groups, ks)
            for lv in range(len(counts)):
                assert got[lv].tolist() == idx[lv][b, hk].tolist(), (lv + 1, b, hk)
