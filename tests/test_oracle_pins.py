"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: a brute-force loop, a
library routine (torch SDPA in fp64 with an explicit mask), a closed form, a hand-built case
from the paper's described failure modes, or an invariant that any correct implementation
must satisfy. A plausible mistake in the oracle (a dropped term, a wrong index or sign, a
transposed operand, the wrong direction of a comparison) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import crisp_oracle as O
from dynamic_block_sparse_proxy_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "noise_floor_cases.json")


def f64(t):
    return t.to(torch.float64).numpy()


def sdpa_masked(q, k, v, mask):
    """Library reference: torch fp64 scaled-dot-product attention with an explicit bool mask."""
    tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(mask)[None, None])
    return out[0, 0].numpy()


def block_mask(lists, n, B):
    m = np.zeros((n, n), dtype=bool)
    for qb, kbs in enumerate(lists):
        for kb in kbs:
            m[qb * B:(qb + 1) * B, kb * B:(kb + 1) * B] = True
    return m & np.tril(np.ones((n, n), dtype=bool))


# ---------------------------------------------------------------------------- attention pins
def test_attention_bruteforce_loop_tiny():
    """All blocks selected == a naive per-element loop (tiny n, d)."""
    rng = np.random.default_rng(0)
    n, d, B = 48, 6, 8
    q, k, v = rng.normal(size=(n, d)), rng.normal(size=(n, d)), rng.normal(size=(n, d))
    lists = [np.arange(qb + 1) for qb in range(n // B)]
    o, lse = O.attention_head(q, k, v, lists, B)
    for i in range(n):
        logits = [sum(q[i, c] * k[j, c] for c in range(d)) / math.sqrt(d) for j in range(i + 1)]
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        z = sum(w)
        for c in range(d):
            ref = sum(w[j] * v[j, c] for j in range(i + 1)) / z
            assert abs(o[i, c] - ref) < 1e-12
        assert abs(lse[i] - (mx + math.log(z))) < 1e-12


@pytest.mark.parametrize("n", [128, 256, 512, 1024, 1, 77, 129, 300, 1000])
def test_all_blocks_equals_sdpa_dense(n):
    # lengths that are not a multiple of 128 have a partial last block (R11)
    q, k, v = (f64(t[0]) for t in W.random_qkv(1, 1, n, seed=n))
    lists = [np.arange(qb + 1) for qb in range(-(-n // 128))]
    o, _ = O.attention_head(q, k, v, lists)
    ref = sdpa_masked(q, k, v, np.tril(np.ones((n, n), dtype=bool)))
    assert np.max(np.abs(o - ref)) < 1e-12
    assert np.max(np.abs(O.dense_causal_attention(q, k, v) - ref)) < 1e-12


def test_random_index_set_equals_masked_sdpa():
    rng = np.random.default_rng(3)
    n, B = 1024, 128
    q, k, v = (f64(t[0]) for t in W.random_qkv(1, 1, n, seed=7))
    nb = n // B
    lists = []
    for qb in range(nb):
        s = {qb} | {int(j) for j in rng.choice(qb + 1, size=min(qb + 1, 3), replace=False)}
        lists.append(np.array(sorted(s)))
    o, _ = O.attention_head(q, k, v, lists, B)
    ref = sdpa_masked(q, k, v, block_mask(lists, n, B))
    assert np.max(np.abs(o - ref)) < 1e-12


def test_selected_all_two_ways_is_dense():
    """tau>1 with gamma=1 (all PE) and alpha=0 with tau=0 (all VS) both select every block."""
    n = 1024
    q, k, v = W.random_qkv(1, 1, n, seed=11)
    q, k, v = f64(q[0]), f64(k[0]), f64(v[0])
    dense = O.dense_causal_attention(q, k, v)
    for kw in (dict(tau_proxy=2.0, gamma=1.0), dict(tau_proxy=0.0, alpha=0.0)):
        sel = O.select_head(q, k, **kw)
        assert sel["route"] == (1 if kw["tau_proxy"] == 0.0 else 0)
        for qb, kb in enumerate(sel["lists"]):
            assert np.array_equal(kb, np.arange(qb + 1))
        o, _ = O.attention_head(q, k, v, sel["lists"])
        assert np.max(np.abs(o - dense)) < 1e-12


# ---------------------------------------------------------------------------- proxy / pooling
@pytest.mark.parametrize("n,seed,scale", [(256, 0, 1.0), (1024, 1, 3.0), (4096, 2, 0.3), (300, 3, 1.0),
                                          (1000, 4, 2.0), (4097, 5, 0.5)])
def test_mass_identities(n, seed, scale):
    q, k, _ = W.random_qkv(1, 1, n, seed=seed, q_scale=scale)
    q, k = f64(q[0]), f64(k[0])
    sel = O.select_head(q, k)
    assert sel["p_v"].shape == (-(-n // 128),)
    assert abs(sel["p_v"].sum() - 1.0) < 1e-12
    assert abs(sel["p_s"].sum() - 1.0) < 1e-12
    assert 0.0 <= sel["c_struct"] <= 1.0
    if n % 128 == 0:   # the anchor windows are then exactly the first and last blocks
        assert abs(sel["c_struct"] - (sel["p_v"][0] + sel["p_v"][-1])) < 1e-12
    assert np.all(sel["p_v"] >= 0) and np.all(sel["p_s"] >= 0)


@pytest.mark.parametrize("n", [256, 640, 2048, 300, 1000, 4097])
def test_uniform_proxy_closed_forms(n):
    """Q_last = 0: every visible key gets 1/(i_r+1); check C, p_v and p_s by counting."""
    B, d = 128, 128
    rng = np.random.default_rng(n)
    q = rng.normal(size=(n, d))
    q[n - B:] = 0.0
    k = rng.normal(size=(n, d))
    sel = O.select_head(q, k)
    rows = n - B + np.arange(B)
    c = np.mean([(128 + r + 1) / (n - B + r + 1) for r in range(B)])
    assert abs(sel["c_struct"] - c) < 1e-12
    nb = -(-n // B)
    pv = np.zeros(nb)
    for i in rows:
        for b in range(nb):
            lo, hi = b * B, min(b * B + B, i + 1)
            pv[b] += max(hi - lo, 0) / (i + 1) / B
    assert np.max(np.abs(sel["p_v"] - pv)) < 1e-12
    ps = np.zeros(nb)
    for i in rows:
        for o in range(i + 1):               # offset o reaches key i-o
            ps[o // B] += 1.0 / (i + 1) / B
    assert np.max(np.abs(sel["p_s"] - ps)) < 1e-12


@pytest.mark.parametrize("kb", [0, 3, 6])
def test_spike_is_one_hot(kb):
    """One key (first of block kb) with a dominant logit: p_v and p_s are one-hot where predicted."""
    n, B, d = 1024, 128, 128
    rng = np.random.default_rng(kb)
    w = rng.normal(size=d)
    q = rng.normal(size=(n, d)) * 0.01
    q[n - B:] = w
    k = rng.normal(size=(n, d)) * 0.01
    k[kb * B] = 400.0 * w / (w @ w) * math.sqrt(d)        # logit ~ 400 for every proxy row
    sel = O.select_head(q, k)
    nb = n // B
    ev = np.eye(nb)[kb]
    es = np.eye(nb)[nb - 1 - kb]
    assert np.max(np.abs(sel["p_v"] - ev)) < 1e-9
    assert np.max(np.abs(sel["p_s"] - es)) < 1e-9


def test_causality_of_proxy():
    """A key after every proxy row's position cannot exist; a key inside the last block is seen
    only by rows at or after it (reading: the proxy is causal)."""
    n, B, d = 512, 128, 128
    q = np.zeros((n, d))
    q[n - B:, 0] = 1.0
    k = np.zeros((n, d))
    j = n - B + 40
    k[j, 0] = 500.0
    a = O.proxy_attention(q[n - B:], k, n)
    assert np.all(a[:40, j] == 0.0)
    assert np.all(a[40:, j] > 0.99)
    assert np.all(a[np.arange(B)[:, None] < (np.arange(n)[None, :] - (n - B))] == 0.0)


# ---------------------------------------------------------------------------- noise floor pins
def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_hand_built_mu():
    g = _golden()["hand_built_mu"]
    p = np.array(g["p"])
    assert abs(O.noise_floor(p) - g["mu"]) < 1e-15
    assert O.keep_blocks(p, g["alpha"]) == g["keep"]
    lists = O.merge_vertical_slash(g["keep"], [], len(p))
    assert 0 in lists[-1] and 9 in lists[-1] and 2 in lists[-1] and 5 in lists[-1]


def test_keep_rule_is_strict():
    """A block whose mass equals alpha*mu exactly is not kept (strict '>')."""
    p = np.array([0.5, 0.0625, 0.0625, 0.0625, 0.0625, 0.25])   # mu = 0.25/4 = 0.0625 exactly
    assert O.noise_floor(p) == 0.0625
    assert O.keep_blocks(p, 1.0) == []
    assert O.keep_blocks(p, 0.5) == [1, 2, 3, 4]


def test_sink_only_collapse():
    g = _golden()["sink_only_collapse"]
    nb = g["n_blocks"]
    p = np.full(nb, 0.01 / 7)
    p[0], p[-1], p[g["signal_block"]] = g["p0"], g["p_last"], g["signal_mass"]
    assert abs(p.sum() - 1.0) < 1e-12
    kept, _, _ = O.gamma_cut(p, g["gamma"], 1.0)
    assert sorted(kept.tolist()) == g["gamma_keeps"]
    assert abs(O.noise_floor(p) - g["mu"]) < 1e-15
    assert O.keep_blocks(p, 1.0) == g["alpha_mu_keeps"]
    # FlexPrefill's per-direction rule is the same gamma cut on one direction: it keeps only the
    # sink anchor, so no inner block survives
    inner, cut = O.gamma_keep_direction(p, g["gamma"])
    assert inner == [j for j in g["gamma_keeps"] if 0 < j < nb - 1] == [] and cut == g["p0"]


def test_o_n_noise_growth():
    g = _golden()["o_n_noise"]
    for nb, want_gamma, want_mu in zip(g["n_blocks"], g["gamma_non_anchor_count"], g["alpha_mu_count"]):
        p = np.full(nb, g["background_total"] / (nb - 6))
        sig = [nb // 5, 2 * nb // 5, 3 * nb // 5, 4 * nb // 5]
        p[0], p[-1] = g["p0"], g["p_last"]
        p[sig] = g["signal_mass"]
        assert abs(p.sum() - 1.0) < 1e-12
        kept, _, _ = O.gamma_cut(p, g["gamma"], 1.0)
        non_anchor = [j for j in kept.tolist() if 0 < j < nb - 1]
        assert len(non_anchor) == want_gamma
        # the same count through FlexPrefill's per-direction rule
        assert len(O.gamma_keep_direction(p, g["gamma"])[0]) == want_gamma
        keep = O.keep_blocks(p, 1.0)
        assert len(keep) == want_mu and keep == sorted(sig)


def test_min_blocks_top_up():
    p = np.array([0.5, 0.30, 0.01, 0.02, 0.02, 0.01, 0.0, 0.14])
    # mu = (1-0.5-0.14)/6 = 0.06: only block 1 passes
    assert O.keep_blocks(p, 1.0) == [1]
    # top-up takes the largest remaining, ties to the lower index: 3 before 4, then 2 before 5
    assert O.keep_blocks(p, 1.0, min_blocks=3) == [1, 3, 4]
    assert O.keep_blocks(p, 1.0, min_blocks=4) == [1, 2, 3, 4]
    assert O.keep_blocks(p, 1.0, min_blocks=99) == [1, 2, 3, 4, 5, 6]


# ---------------------------------------------------------------------------- PE pins
@pytest.mark.parametrize("nb,gamma", [(16, 0.95), (10, 0.9), (33, 0.8)])
def test_pe_uniform_closed_form(nb, gamma):
    """Zero-mean query blocks make every pooled row uniform, 1/(qb+1); the global cut keeps
    rows 0..R-1 whole (R = floor(gamma*N_b)) and the first ceil((gamma*N_b-R)(R+1)) of row R."""
    B, d = 128, 128
    rng = np.random.default_rng(nb)
    half = rng.integers(-8, 9, size=(nb, B // 2, d)) / 8.0     # exact in bf16/fp32/fp64
    q = np.concatenate([half, -half], axis=1).reshape(nb * B, d)
    k = rng.normal(size=(nb * B, d))
    lists, P, _ = O.pe_select(q, k, B, gamma)
    R = int(math.floor(gamma * nb))
    t = int(math.ceil((gamma * nb - R) * (R + 1) - 1e-9))
    for qb in range(nb):
        assert np.allclose(P[qb, : qb + 1], 1.0 / (qb + 1), rtol=0, atol=1e-15)
        if qb < R:
            want = set(range(qb + 1))
        elif qb == R:
            want = set(range(min(t, qb + 1)))
        else:
            want = set()
        want |= {j for j in (0, qb - 1, qb) if j >= 0}
        assert set(lists[qb].tolist()) == want, qb


def test_pe_cut_bruteforce_small():
    """The global cut equals an exhaustive search for the smallest mass-covering set."""
    rng = np.random.default_rng(5)
    for _ in range(20):
        x = rng.random(7) ** 3
        x /= x.sum()
        gamma = float(rng.uniform(0.3, 0.99))
        kept, _, _ = O.gamma_cut(x, gamma, 1.0)
        best = None
        for mask in range(1 << 7):
            idx = [i for i in range(7) if mask >> i & 1]
            if x[idx].sum() >= gamma and (best is None or len(idx) < len(best)):
                best = idx
        assert len(kept) == len(best)
        # the cut takes the largest values
        assert x[kept].min() >= np.sort(x)[::-1][len(best) - 1] - 1e-15


# ---------------------------------------------------------------------------- merge coverage
@pytest.mark.parametrize("seed", range(6))
def test_merge_covers_kept_diagonals_and_verticals(seed):
    """Token-level brute force (B=4): every causal pair on a kept diagonal or in a kept vertical
    block lies in a kept block, and every kept block is justified by some rule."""
    rng = np.random.default_rng(seed)
    B = 4
    nb = int(rng.integers(3, 17))
    n = nb * B
    inner = list(range(1, nb - 1))
    keep_v = sorted(rng.choice(inner, size=rng.integers(0, len(inner) + 1), replace=False).tolist())
    keep_s = sorted(rng.choice(inner, size=rng.integers(0, len(inner) + 1), replace=False).tolist())
    lists = O.merge_vertical_slash(keep_v, keep_s, nb)
    kept = np.zeros((nb, nb), dtype=bool)
    for qb, kb in enumerate(lists):
        kept[qb, kb] = True
    slash_m = set(keep_s) | {0, nb - 1}
    vert = set(keep_v) | {0, nb - 1}
    justified = np.zeros_like(kept)
    for i in range(n):
        for j in range(i + 1):
            on_diag = (i - j) // B in slash_m
            in_vert = j // B in vert
            if on_diag or in_vert:
                assert kept[i // B, j // B], (i, j)
                justified[i // B, j // B] = True
    assert np.array_equal(kept, justified)


def test_small_nb_keeps_everything():
    for n in (128, 256):
        q, k, _ = W.random_qkv(1, 1, n, seed=n)
        for tau in (0.0, 2.0):
            sel = O.select_head(f64(q[0]), f64(k[0]), tau_proxy=tau)
            for qb, kb in enumerate(sel["lists"]):
                assert np.array_equal(kb, np.arange(qb + 1))


# ---------------------------------------------------------------------------- generator sanity
def _select_workload(w):
    q, k, v, meta = W.generate(w)
    G = w.h_q // w.h_kv
    out = []
    for h in range(w.h_q):
        out.append(O.select_head(f64(q[h]), f64(k[h // G])))
    return out, meta


def test_tiny_workload_routes_vs_and_finds_planted_verticals():
    sels, meta = _select_workload(W.WORKLOADS["tiny_1h_4k"])
    s = sels[0]
    assert s["route"] == 1 and s["c_struct"] > 0.9
    assert set(meta["vertical_blocks"][0]) <= set(s["keep_v"])


def test_llama_geometry_routing_at_reduced_length():
    w = W.WORKLOADS["llama8b_32k"].scaled(4096)
    sels, meta = _select_workload(w)
    for h, s in enumerate(sels):
        assert s["route"] == int(meta["concentrated"][h]), (h, s["c_struct"])
        if meta["concentrated"][h]:
            assert set(meta["vertical_blocks"][h // 4]) <= set(s["keep_v"])


def test_llama_geometry_slash_plants_found():
    """At 64k tokens the planted verticals are always kept and most planted slash offsets are
    kept in the slash direction (each diagonal is planted on a quarter of the rows, so a few
    fall under the floor on some heads)."""
    w = W.WORKLOADS["llama8b_128k"].scaled(65536)
    sels, meta = _select_workload(w)
    found = total = 0
    for h, s in enumerate(sels):
        assert s["route"] == int(meta["concentrated"][h])
        if meta["concentrated"][h]:
            offs = meta["slash_offsets"][h // 4]
            found += len({o // 128 for o in offs} & set(s["keep_s"]))
            total += len(offs)
            assert set(meta["vertical_blocks"][h // 4]) <= set(s["keep_v"])
    assert found >= 0.8 * total, (found, total)


def test_qwen_geometry_sink_dominates_concentrated_heads():
    w = W.WORKLOADS["qwen7b_128k"].scaled(16384)
    sels, meta = _select_workload(w)
    for h, s in enumerate(sels):
        assert s["route"] == int(meta["concentrated"][h])
        if meta["concentrated"][h]:
            assert s["p_v"][0] > 0.9


# ------------------------------------------------------------------ FlexPrefill rules, median floor
def test_jsd_closed_forms():
    p = np.array([0.2, 0.3, 0.5])
    assert O.jsd(p, p) == 0.0
    # disjoint supports: ln 2 (natural log)
    assert math.isclose(O.jsd(np.array([1.0, 0.0]), np.array([0.0, 1.0])), math.log(2.0), rel_tol=1e-15)
    # hand value: p = (1, 0), q = (1/2, 1/2), m = (3/4, 1/4)
    # KL(p||m) = ln(4/3); KL(q||m) = (1/2) ln(2/3) + (1/2) ln 2
    want = 0.5 * math.log(4 / 3) + 0.5 * (0.5 * math.log(2 / 3) + 0.5 * math.log(2.0))
    assert math.isclose(O.jsd(np.array([1.0, 0.0]), np.array([0.5, 0.5])), want, rel_tol=1e-14)
    rng = np.random.default_rng(1)
    a, b = rng.random(7), rng.random(7)
    a, b = a / a.sum(), b / b.sum()
    assert math.isclose(O.jsd(a, b), O.jsd(b, a), rel_tol=1e-14)
    assert 0.0 < O.jsd(a, b) < math.log(2.0)


def test_pooled_estimate_hand_case():
    # d = 2, B = 2: mean query (sqrt(2) ln 3, 0) against block means (1, 0) and (0, 1) gives
    # logits (ln 3, 0) after the 1/sqrt(d) scale, i.e. a_bar = (3/4, 1/4)
    qbar = np.array([math.sqrt(2.0) * math.log(3.0), 0.0])
    q_last = np.stack([qbar + [0.5, -1.0], qbar - [0.5, -1.0]])   # mean is qbar
    k = np.array([[1.0, 0.0], [1.0, 0.0], [0.0, 1.0], [0.0, 1.0]])
    np.testing.assert_allclose(O.pooled_estimate(q_last, k, 2), [0.75, 0.25], rtol=1e-14)
    # identical key blocks: uniform
    np.testing.assert_allclose(O.pooled_estimate(q_last, np.ones((6, 2)), 2), np.full(3, 1 / 3), rtol=1e-14)


def test_gamma_keep_direction_hand_cases():
    p = np.array([0.5, 0.1, 0.3, 0.1])
    assert O.gamma_keep_direction(p, 0.8) == ([2], 0.3)         # {0, 2} reach 0.8; 0 is an anchor
    assert O.gamma_keep_direction(p, 0.85) == ([1, 2], 0.1)     # the tie at 0.1 goes to j=1 first
    assert O.gamma_keep_direction(p, 0.95) == ([1, 2], 0.1)     # 0.1 at j=3 only comes after
    assert O.gamma_keep_direction(p, 1.0)[0] == [1, 2]
    # a target scaled by the direction's own total
    assert O.gamma_keep_direction(2 * p, 0.8) == ([2], 0.6)


def test_median_floor_and_keep():
    p = np.array([0.4, 0.1, 0.3, 0.05, 0.15])                   # inner 0.1, 0.3, 0.05 -> 0.1
    assert O.median_floor(p) == 0.1
    assert O.keep_blocks(p, 1.0, floor="median") == [2]
    assert O.keep_blocks(p, 0.4, floor="median") == [1, 2, 3]   # 0.05 > 0.04
    q = np.array([0.5, 0.1, 0.2, 0.04, 0.06, 0.1])              # inner even: (0.06 + 0.1) / 2
    assert math.isclose(O.median_floor(q), 0.08, rel_tol=1e-15)
    # the mean floor of the same inner mass differs: (1 - 0.5 - 0.1) / 4 = 0.1
    assert math.isclose(O.noise_floor(q), 0.1, rel_tol=1e-14)
    assert O.keep_blocks(q, 1.0, floor="median") == [1, 2]       # j = 5 is the last anchor
    assert O.keep_blocks(q, 1.0, floor="mean") == [2]


def test_flexprefill_rules_on_planted_heads():
    """JSD is large on planted-concentrated heads and small on diffuse ones. On a sink-dominated
    head the per-direction gamma cut stops at the sink block (the mass-cliff collapse the CRISP
    paper describes, §4), so no inner vertical block survives; gamma = 1 keeps every block that
    carries mass."""
    w = W.WORKLOADS["llama8b_32k"].scaled(4096)
    q, k, v, meta = W.generate(w)
    G = w.h_q // w.h_kv
    nb = w.n // 128
    for h in (0, 2):
        s = O.select_head(q[h].double().numpy(), k[h // G].double().numpy(), route_rule="jsd",
                          vs_rule="gamma")
        assert s["route"] == int(meta["concentrated"][h]), s["jsd"]
        if s["route"]:
            assert s["jsd"] > 0.3
            assert s["p_v"][0] >= 0.95 and s["keep_v"] == []
        else:
            assert s["jsd"] < 0.01
    s = O.select_head(q[0].double().numpy(), k[0].double().numpy(), route_rule="jsd", vs_rule="gamma",
                      gamma=1.0)
    assert s["keep_v"] == [j for j in range(1, nb - 1) if s["p_v"][j] > 0]
    # with a target below the sink's share but above it plus the planted blocks' mass, the
    # planted verticals come first among the inner blocks
    pv = s["p_v"]
    inner_planted = sorted(meta["vertical_blocks"][0])
    g = (pv[0] + pv[nb - 1] + pv[inner_planted].sum() * 0.999) / pv.sum()
    kept, _ = O.gamma_keep_direction(pv, g)
    assert set(kept) <= set(inner_planted)


def test_block_mean_of_a_partial_block():
    x = np.arange(2 * 300, dtype=np.float64).reshape(300, 2)
    m = O.block_mean(x, 128)
    assert m.shape == (3, 2)
    np.testing.assert_allclose(m[2], x[256:300].mean(axis=0))   # 44 rows, not 128
    np.testing.assert_allclose(O.pool_blocks(np.ones(300), 128), [128, 128, 44])


# ---------------------------------------------------------------- pooled scores, non-uniform rows
def _pooled_case():
    with open(os.path.join(os.path.dirname(__file__), "golden", "pooled_scores_case.json")) as f:
        g = json.load(f)
    named = {"ln 3": math.log(3.0), "ln 2": math.log(2.0), "-ln 2": -math.log(2.0)}
    a = np.array([named.get(x, x) for x in g["a"]], dtype=np.float64)
    b = np.array(g["b"], dtype=np.float64)
    nb, B = g["n_blocks"], g["B"]
    rng = np.random.default_rng(7)
    qbar = np.stack([math.sqrt(2.0) * a, math.sqrt(2.0) * b], axis=1)
    kbar = np.stack([np.arange(nb, dtype=np.float64), np.ones(nb)], axis=1)
    dq, dk = rng.normal(size=(nb, 2)), rng.normal(size=(nb, 2))
    q = np.stack([qbar + dq, qbar - dq], axis=1).reshape(nb * B, 2)   # block means are qbar
    k = np.stack([kbar + dk, kbar - dk], axis=1).reshape(nb * B, 2)
    frac = lambda x: float(eval(x)) if isinstance(x, str) else float(x)  # noqa: E731
    P = [[frac(x) for x in row] for row in g["P"]]
    return g, q, k, P


def _pooled_case_holds() -> bool:
    """The golden pooled matrix and every golden gamma cut, against the oracle."""
    g, q, k, P = _pooled_case()
    got = O.pooled_scores(q, k, g["B"])
    for qb, row in enumerate(P):
        if not np.allclose(got[qb, : qb + 1], row, rtol=0, atol=1e-12):
            return False
        if np.any(got[qb, qb + 1:] != 0.0):
            return False
    for cut in g["cuts"]:
        lists, _, _ = O.pe_select(q, k, g["B"], cut["gamma"])
        if [x.tolist() for x in lists] != cut["lists"]:
            return False
    return True


def test_pooled_scores_hand_case():
    """Non-uniform pooled rows with closed forms (the 1/sqrt(d) scale, the operand order
    Qbar . Kbar and the inclusive causal mask all show), and three gamma cuts derived by hand."""
    assert _pooled_case_holds()


def _mean_pool(x, B):
    n = x.shape[0]
    return np.stack([x[i:min(i + B, n)].mean(axis=0) for i in range(0, n, B)])


def _softmax_causal(s):
    nb = s.shape[0]
    causal = np.tril(np.ones((nb, nb), dtype=bool))
    s = np.where(causal, s, -np.inf)
    e = np.where(causal, np.exp(s - s.max(axis=1, keepdims=True)), 0.0)
    return e / e.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("mistake", ["transposed", "unscaled", "sum_pooled_q", "strict_mask"])
def test_pooled_scores_hand_case_catches_plausible_mistakes(monkeypatch, mistake):
    """Each plausible slip in pooled_scores, planted on the CPU, fails the hand case above."""
    def bad(q, k, B):
        d = q.shape[1]
        qb, kb = _mean_pool(q, B), _mean_pool(k, B)
        if mistake == "transposed":
            s = (kb @ qb.T) / np.sqrt(d)
        elif mistake == "unscaled":
            s = qb @ kb.T
        elif mistake == "sum_pooled_q":
            s = (B * qb @ kb.T) / np.sqrt(d)
        else:  # kb < qb only: the diagonal block left out (row 0 then keeps its one entry)
            s = (qb @ kb.T) / np.sqrt(d)
            s = s - np.where(np.eye(s.shape[0], dtype=bool), 1e3, 0.0) * (np.arange(s.shape[0]) > 0)[:, None]
        return _softmax_causal(s)

    monkeypatch.setattr(O, "pooled_scores", bad)
    assert not _pooled_case_holds()
    if mistake == "transposed":
        # the index lists alone already differ: the gamma = 0.55 and 0.7 cuts keep (4, 1)
        g, q, k, _ = _pooled_case()
        got = [[x.tolist() for x in O.pe_select(q, k, g["B"], c["gamma"])[0]] for c in g["cuts"]]
        assert any(gl != c["lists"] for gl, c in zip(got, g["cuts"]))


# ---------------------------------------------------------------------------------------------
# FP8 (E4M3) quantisation of the attention logits' operands
# ---------------------------------------------------------------------------------------------
def test_e4m3_codes_from_the_format_definition():
    """Values whose codes follow from the format (bias 7, 3 mantissa bits, subnormals m * 2^-9,
    largest finite 448), including ties to the even code and saturation."""
    cases = {1.0: 0x38, 448.0: 0x7E, 0.5: 0x30, 2.0 ** -6: 0x08, 2.0 ** -9: 0x01,
             1.0625: 0x38,          # halfway between 1.0 (even) and 1.125
             1.1875: 0x3A,          # halfway between 1.125 and 1.25 (even)
             500.0: 0x7E, 1e6: 0x7E, -1.0: 0xB8, -448.0: 0xFE,
             3 * 2.0 ** -10: 0x02,  # halfway between 1 and 2 subnormal units (2 is even)
             2.0 ** -10: 0x00,      # halfway between 0 (even) and the smallest subnormal
             2.0 ** -11: 0x00, 240.0: 0x77, 0.0: 0x00}
    for v, code in cases.items():
        assert int(O.e4m3_encode(np.float32(v))) == code, (v, hex(int(O.e4m3_encode(np.float32(v)))), hex(code))
    assert O.e4m3_decode(np.array([0x7E]))[0] == 448.0 and O.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9


def test_e4m3_round_trip_and_library_cast():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert (O.e4m3_encode(O.e4m3_decode(codes)) == codes).all()
    rng = np.random.default_rng(0)
    y = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(0, 1, 20000),
                        rng.normal(0, 0.01, 20000)]).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (O.e4m3_encode(y) == ref).all()


def test_quantize_blocks_fp8_properties():
    rng = np.random.default_rng(1)
    n, B = 300, 128   # a partial last block
    x = torch.from_numpy(rng.normal(0, 2, (n, 128))).to(torch.bfloat16).double().numpy()
    x[128:256] = 0.0  # an all-zero block
    codes, scales = O.quantize_blocks_fp8(x, B)
    assert scales[1] == 1.0 and (codes[128:256] == 0).all()
    deq = O.dequantize_blocks_fp8(codes, scales, B)
    for b in (0, 2):
        blk = slice(b * B, min(n, (b + 1) * B))
        amax = np.abs(x[blk]).max()
        # the element at the block's amax lands on the largest code
        i = np.unravel_index(np.abs(x[blk]).argmax(), x[blk].shape)
        assert (codes[blk][i] & 0x7F) == 0x7E
        assert scales[b] == np.float32(np.float32(amax) / np.float32(448.0))
        # every value within half a unit of its binade (2^-4 relative) or of the subnormal step
        err = np.abs(deq[blk] - x[blk])
        bound = np.maximum(np.abs(x[blk]) * 2.0 ** -4, 2.0 ** -10 * scales[b]) * (1 + 1e-6)
        assert (err <= bound).all()
