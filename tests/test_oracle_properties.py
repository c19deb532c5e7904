"""Property checks of the oracle's selection rules on random small inputs (hypothesis, fixed
derandomised examples so runs are reproducible). Each property is one the rule must satisfy
whatever its implementation: bounds, symmetry, coverage and minimality of cuts, monotonicity in
alpha, the median by brute force, and token-level coverage of the vertical-slash merge."""
import math

import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import crisp_oracle as O

SETTINGS = settings(max_examples=60, derandomize=True, deadline=None)


def _dist(xs):
    p = np.asarray(xs, dtype=np.float64) + 1e-9
    return p / p.sum()


vec = st.lists(st.floats(min_value=0.0, max_value=1.0, allow_nan=False), min_size=3, max_size=24)


@SETTINGS
@given(vec, vec)
def test_jsd_bounds_and_symmetry(a, b):
    n = min(len(a), len(b))
    p, q = _dist(a[:n]), _dist(b[:n])
    j = O.jsd(p, q)
    assert -1e-15 <= j <= math.log(2.0) + 1e-12
    assert math.isclose(j, O.jsd(q, p), rel_tol=1e-12, abs_tol=1e-15)
    assert abs(O.jsd(p, p)) < 1e-15


@SETTINGS
@given(vec, st.floats(min_value=0.05, max_value=0.999))
def test_gamma_direction_covers_and_is_minimal(xs, gamma):
    p = _dist(xs)
    nb = p.shape[0]
    kept_inner, cut = O.gamma_keep_direction(p, gamma)
    # brute force: walk the (p desc, j asc) order until the running sum reaches gamma * total
    order = sorted(range(nb), key=lambda j: (-p[j], j))
    target, acc, prefix = gamma * p.sum(), 0.0, []
    for j in order:
        prefix.append(j)
        acc += p[j]
        if acc >= target:
            break
    assert kept_inner == sorted(j for j in prefix if 1 <= j <= nb - 2)
    assert cut == p[prefix[-1]]
    assert sum(p[j] for j in prefix[:-1]) < target     # no shorter prefix reaches the target


@SETTINGS
@given(vec, st.floats(min_value=0.0, max_value=3.0), st.floats(min_value=0.0, max_value=3.0))
def test_keep_rule_shrinks_as_alpha_grows(xs, a1, a2):
    p = _dist(xs)
    lo, hi = sorted((a1, a2))
    for floor in ("mean", "median"):
        assert set(O.keep_blocks(p, hi, floor=floor)) <= set(O.keep_blocks(p, lo, floor=floor))


@SETTINGS
@given(vec)
def test_median_floor_by_sorting(xs):
    p = _dist(xs)
    inner = sorted(p[1:-1])
    m = len(inner)
    want = inner[m // 2] if m % 2 else 0.5 * (inner[m // 2 - 1] + inner[m // 2])
    assert math.isclose(O.median_floor(p), want, rel_tol=1e-15)


@SETTINGS
@given(st.integers(min_value=3, max_value=12), st.data())
def test_merge_covers_every_token_of_kept_diagonals(nb, data):
    B = 8  # the mapping is the same at any block size; small blocks keep the brute force cheap
    keep_v = data.draw(st.lists(st.integers(1, nb - 2), unique=True, max_size=nb - 2))
    keep_s = data.draw(st.lists(st.integers(1, nb - 2), unique=True, max_size=nb - 2))
    lists = O.merge_vertical_slash(keep_v, keep_s, nb)
    slash = set(keep_s) | {0, nb - 1}
    for qb in range(nb):
        sel = set(lists[qb].tolist())
        assert lists[qb].tolist() == sorted(sel) and all(0 <= j <= qb for j in sel)
        assert 0 in sel and qb in sel
        for j in set(keep_v) | {nb - 1}:
            if j <= qb:
                assert j in sel
        # every (query token, key token) pair on a kept diagonal falls in a selected block
        for i in range(qb * B, qb * B + B):
            for m in slash:
                for o in range(m * B, m * B + B):
                    if i - o >= 0:
                        assert (i - o) // B in sel, (qb, i, m, o)
