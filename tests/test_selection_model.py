"""Step-by-step host models of the two selections the decode kernels run on
the GPU (the threshold selection for k <= 32 and the radix select on keys in
registers), checked against numpy's lexsort on many inputs, adversarial ones
included.

These models pin the algorithms' reasoning, not the CUDA code: that tau is a
lower bound of the k-th largest key, that the flood test fires only when it
must, and that the radix passes (starting below the bits every key shares,
with digits narrower than 8 bits at the end) always land on the k-th largest
key.  The GPU tests compare the kernels themselves with the oracle.

The selection is the one the pages' routing step needs (gist.science
explainer, section 2 "Methodology", selective unfolding: the k best-scoring
chunks), with the tie rule and output order the library documents: ties to
the lowest index, indices ascending.
"""
import numpy as np

NT = 128          # threads of the unfold warp group
WARP = 32


def order_key(x: np.ndarray) -> np.ndarray:
    """Monotone fp32 -> u32 map (larger score, larger key); -0 and +0 share a
    key, NaN maps to 0, below every number."""
    f = np.asarray(x, np.float32)
    u = f.view(np.uint32).copy()
    u[f == 0] = 0
    neg = (u & 0x80000000) != 0
    k = np.where(neg, ~u, u | 0x80000000).astype(np.uint32)
    k[np.isnan(f)] = 0
    return k


def expected(keys: np.ndarray, k: int) -> np.ndarray:
    """The k largest keys, ties to the lower position, ascending (library sort)."""
    pos = np.arange(len(keys))
    order = np.lexsort((pos, -keys.astype(np.int64)))
    return np.sort(order[:k])


def clz32(v: int) -> int:
    return 32 - int(v).bit_length()


def threshold_model(keys: np.ndarray, k: int):
    """Returns (selection or None on a flood, tau, candidate count)."""
    n = len(keys)
    pos = np.arange(n)
    tmax = np.zeros(NT, np.uint64)
    for t in range(NT):
        mine = keys[t::NT]
        if len(mine):
            tmax[t] = mine.max()
    # each warp: the k-th largest of its 32 lane maxima; tau: the largest bound
    tau = max(np.sort(tmax[w:w + WARP])[::-1][k - 1] for w in range(0, NT, WARP))
    cand = pos[keys >= tau]
    if len(cand) > NT:
        return None, int(tau), len(cand)
    comp = (keys[cand].astype(np.uint64) << np.uint64(32)) | (~cand.astype(np.uint32)).astype(np.uint64)
    rank = np.array([(comp > c).sum() for c in comp])
    sel = cand[rank < k]
    assert len(sel) == k
    return np.sort(sel), int(tau), len(cand)


def radix_model(keys: np.ndarray, k: int) -> np.ndarray:
    kmin, kmax = int(keys.min()), int(keys.max())
    common = clz32(kmin ^ kmax)
    pmask = ((0xFFFFFFFF << (32 - common)) & 0xFFFFFFFF) if common > 0 else 0
    prefix = kmax & pmask
    kk = k
    left = 32 - common
    passes = 0
    while left > 0:
        width = min(8, left)
        shift = left - width
        dmask = (1 << width) - 1
        live = (keys.astype(np.int64) & pmask) == prefix
        hist = np.bincount(((keys[live].astype(np.int64) >> shift) & dmask), minlength=256)
        above, digit, above_digit = 0, None, None
        for b in range(255, -1, -1):          # bins in descending order, as the warp scan
            if above < kk <= above + hist[b]:
                digit, above_digit = b, above
            above += hist[b]
        assert digit is not None and digit <= dmask
        prefix |= digit << shift
        pmask |= dmask << shift
        kk -= above_digit
        left -= width
        passes += 1
    assert pmask == 0xFFFFFFFF or common == 32
    T = prefix
    gt = keys > T
    eq = keys == T
    take = gt | (eq & (np.cumsum(eq) <= kk))
    sel = np.nonzero(take)[0]
    assert len(sel) == k
    return sel


def cases(rng, n_cases=120):
    for i in range(n_cases):
        n = int(rng.choice([2, 3, 31, 129, 700, 2048, 3000, 4096]))
        k = int(rng.integers(1, min(n - 1, 300) + 1)) if n > 2 else 1
        kind = i % 6
        if kind == 0:
            x = rng.standard_normal(n)                       # mixed signs: no shared prefix
        elif kind == 1:
            x = np.abs(rng.standard_normal(n)) + 1e-3         # all positive: sign shared
        elif kind == 2:
            x = 3.0 + rng.random(n) * 0.5                     # one binade: long shared prefix
        elif kind == 3:
            x = rng.integers(0, 5, n).astype(np.float64)      # few values: runs of ties
        elif kind == 4:
            x = -np.abs(rng.standard_normal(n)) - 1.0         # all negative
        else:
            x = rng.standard_normal(n)
            x[rng.integers(0, n, max(1, n // 10))] = np.nan   # NaN ranks lowest
            x[rng.integers(0, n, max(1, n // 10))] = -0.0     # -0 equals +0
            x[rng.integers(0, n, max(1, n // 10))] = 0.0
        yield order_key(x.astype(np.float32)), k


def test_radix_model_matches_library_sort():
    rng = np.random.default_rng(11)
    for keys, k in cases(rng):
        np.testing.assert_array_equal(radix_model(keys, k), expected(keys, k))


def test_radix_model_all_keys_equal_needs_no_pass():
    keys = np.full(1000, 0x9F00AA55, np.uint32)
    np.testing.assert_array_equal(radix_model(keys, 37), np.arange(37))


def test_radix_model_narrow_last_digit():
    """Keys sharing 5 leading bits leave 27 bits: digits of 8, 8, 8 and 3."""
    rng = np.random.default_rng(12)
    keys = (np.uint32(0b10110) << np.uint32(27)) | rng.integers(0, 1 << 27, 3000).astype(np.uint32)
    keys[5] = np.uint32(0b10110) << np.uint32(27)            # the smallest possible, makes the prefix exactly 5 bits
    keys[6] = (np.uint32(0b10110) << np.uint32(27)) | np.uint32((1 << 27) - 1)
    assert clz32(int(keys.min()) ^ int(keys.max())) == 5
    for k in (1, 2, 64, 1500, 2999):
        np.testing.assert_array_equal(radix_model(keys, k), expected(keys, k))


def test_threshold_model_is_exact_or_reports_a_flood():
    rng = np.random.default_rng(13)
    floods = 0
    for keys, k in cases(rng, 180):
        k = min(k, 32, len(keys) - 1) if len(keys) > 1 else 1
        if k < 1:
            continue
        sel, tau, m = threshold_model(keys, k)
        # tau bounds the k-th largest key from below
        assert tau <= int(np.sort(keys)[::-1][k - 1])
        if sel is None:
            floods += 1
            assert m > NT
        else:
            np.testing.assert_array_equal(sel, expected(keys, k))
    assert floods > 0            # the tie-heavy inputs do reach the fallback


def test_threshold_model_flood_on_equal_keys():
    keys = np.full(2048, 7, np.uint32)
    sel, tau, m = threshold_model(keys, 16)
    assert sel is None and m == 2048
    np.testing.assert_array_equal(radix_model(keys, 16), np.arange(16))
