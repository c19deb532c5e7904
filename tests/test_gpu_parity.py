"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same seeded inputs.

Selection (routes, p_v/p_s, C_struct, per-query-block lists) must agree outside the 1e-5 tie
band; attention on the GPU's own index set must be within 2e-2 max / 2e-3 mean abs of fp64.
Small workloads are checked in full; the full-size workloads (as the benchmark launches them)
are checked on every head's selection where the oracle is fast enough, and on sampled query
blocks for attention.
"""
import numpy as np
import pytest
import torch

import dynamic_block_sparse_proxy_b200 as crisp
from dynamic_block_sparse_proxy_b200 import build as B
from dynamic_block_sparse_proxy_b200 import workloads as W
from oracle import crisp_oracle as O

from tests import parity as PT

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()
    crisp.lib()


def dev():
    return torch.device("cuda:0")


def run_select(q, k, params, ws=None):
    ws = ws if ws is not None else crisp.workspace(q.shape[0], k.shape[0], q.shape[1], q.device)
    idx = crisp.select(q, k, params, ws=ws, debug=True)
    crisp.check_status(ws, "select")
    return idx, ws


def all_lists(idx, heads):
    return {h: idx.lists(h) for h in heads}


def sample_blocks(nb, heads, per_head, seed):
    rng = np.random.default_rng(seed)
    out = []
    for h in heads:
        picks = {0, nb - 1}
        if nb > 2:
            picks |= set(rng.choice(np.arange(1, nb - 1), size=min(per_head, nb - 2), replace=False).tolist())
        out += [(h, int(qb)) for qb in sorted(picks)]
    return out


# ------------------------------------------------------------------------------ device plumbing
def test_timeout_selftest_reports_and_context_survives():
    ws = torch.zeros(4096, dtype=torch.uint8, device=dev())
    assert crisp.selftest_timeout(ws, 2_000_000) == -5
    assert crisp.get_status(ws) == 0
    q, k, v = (t.to(dev()) for t in W.random_qkv(1, 1, 256, seed=1))
    o, _ = crisp.dense_prefill(q, k, v)
    torch.cuda.synchronize()
    ref = O.dense_causal_attention(PT.f64(q[0]), PT.f64(k[0]), PT.f64(v[0]))
    assert np.max(np.abs(PT.f64(o[0]) - ref)) < 2e-2


@pytest.mark.parametrize("n,hq,hkv", [(128, 1, 1), (256, 2, 1), (384, 1, 1), (640, 3, 1), (896, 7, 1), (1024, 4, 2),
                                        (1, 1, 1), (77, 2, 1), (129, 3, 1), (300, 4, 2), (1000, 7, 1), (4097, 8, 2)])
def test_dense_matches_oracle(n, hq, hkv):
    q, k, v = (t.to(dev()) for t in W.random_qkv(hq, hkv, n, seed=n + hq))
    ws = crisp.workspace(hq, hkv, n, dev())
    o, lse = crisp.dense_prefill(q, k, v, ws=ws)
    crisp.check_status(ws)
    nb = -(-n // 128)  # a length that is not a multiple of 128 ends in a partial block
    lists = {h: [list(range(qb + 1)) for qb in range(nb)] for h in range(hq)}
    blocks = [(h, qb) for h in range(hq) for qb in range(nb)]
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, lists, blocks, hq // hkv))


# ------------------------------------------------------------------------------ small workloads, full
def test_tiny_workload_selection_and_attention():
    w = W.WORKLOADS["tiny_1h_4k"]
    q, k, v, meta = W.generate(w)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    params = crisp.Params()
    idx, ws = run_select(q, k, params)
    sels = PT.oracle_select_heads(q, k, params, [0])
    PT.compare_selection(idx, sels, w.n // 128, name="tiny_1h_4k")
    assert int(idx.route[0]) == 1
    o, lse = crisp.sparse_prefill(q, k, v, idx, ws=ws)
    crisp.check_status(ws)
    nb = w.n // 128
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, all_lists(idx, [0]),
                                                       [(0, qb) for qb in range(nb)], 1))
    # one-call prefill gives the same output bit for bit
    o2, lse2, idx2 = crisp.prefill(q, k, v, params, ws=ws)
    crisp.check_status(ws)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("name,n", [("llama8b_32k", 4096), ("qwen7b_128k", 2048), ("llama8b_128k", 8192)])
def test_scaled_workloads_full(name, n):
    w = W.WORKLOADS[name].scaled(n)
    q, k, v, meta = W.generate(w)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    params = crisp.Params()
    idx, ws = run_select(q, k, params)
    heads = list(range(w.h_q))
    sels = PT.oracle_select_heads(q, k, params, heads)
    PT.compare_selection(idx, sels, n // 128, name=f"{name} at n={n}")
    o, lse = crisp.sparse_prefill(q, k, v, idx, ws=ws)
    crisp.check_status(ws)
    blocks = sample_blocks(n // 128, heads, 3, seed=n)
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, all_lists(idx, heads), blocks,
                                                       w.h_q // w.h_kv))


# ------------------------------------------------------------------------------ edge cases
@pytest.mark.parametrize("n", [128, 256, 384])
@pytest.mark.parametrize("tau", [0.0, 2.0])
def test_tiny_block_counts(n, tau):
    q, k, v = (t.to(dev()) for t in W.random_qkv(2, 1, n, seed=n))
    params = crisp.Params(tau_proxy=tau)
    idx, ws = run_select(q, k, params)
    sels = PT.oracle_select_heads(q, k, params, [0, 1])
    PT.compare_selection(idx, sels, n // 128, name=f"random n={n} tau={tau}")
    o, lse = crisp.sparse_prefill(q, k, v, idx, ws=ws)
    crisp.check_status(ws)
    nb = n // 128
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, all_lists(idx, [0, 1]),
                                                       [(h, qb) for h in (0, 1) for qb in range(nb)], 2))


@pytest.mark.parametrize("kw", [dict(tau_proxy=0.0, alpha=0.0), dict(tau_proxy=2.0, gamma=1.0)])
def test_select_everything_equals_dense(kw):
    n = 2048
    q, k, v = (t.to(dev()) for t in W.random_qkv(4, 2, n, seed=3))
    params = crisp.Params(**kw)
    ws = crisp.workspace(4, 2, n, dev())
    o, lse, idx = crisp.prefill(q, k, v, params, ws=ws)
    od, lsed = crisp.dense_prefill(q, k, v, ws=ws)
    crisp.check_status(ws)
    nb = n // 128
    for h in range(4):
        assert idx.lists(h) == [list(range(qb + 1)) for qb in range(nb)]
    assert torch.equal(o, od)
    assert torch.allclose(lse, lsed, atol=0, rtol=0)


def test_min_blocks_variant():
    w = W.WORKLOADS["llama8b_32k"].scaled(4096)
    q, k, v, _ = W.generate(w)
    q, k = q.to(dev()), k.to(dev())
    params = crisp.Params(min_blocks=8)
    idx, _ = run_select(q, k, params)
    sels = PT.oracle_select_heads(q, k, params, list(range(w.h_q)))
    PT.compare_selection(idx, sels, w.n // 128, name="min_blocks=8 llama8b_32k at n=4096")


def test_pe_uniform_closed_form_on_gpu():
    """Zero-mean query blocks make every pooled row exactly uniform: the GPU cut must keep rows
    0..R-1 whole and the first ceil((gamma*N_b-R)(R+1)) blocks of row R, like the oracle."""
    nb, gamma = 16, 0.95
    rng = np.random.default_rng(0)
    half = rng.integers(-8, 9, size=(2, nb, 64, 128)) / 8.0
    qn = np.concatenate([half, -half], axis=2).reshape(2, nb * 128, 128)
    q = torch.from_numpy(qn).to(torch.bfloat16).to(dev())
    k = torch.randn(1, nb * 128, 128, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).to(dev())
    params = crisp.Params(tau_proxy=2.0, gamma=gamma)
    idx, _ = run_select(q, k, params)
    sels = PT.oracle_select_heads(q, k, params, [0, 1])
    for h in (0, 1):
        assert idx.lists(h) == [x.tolist() for x in sels[h]["lists"]]


@pytest.mark.parametrize("n,hq,hkv,mixed", [(2048, 4, 2, False), (1152, 3, 1, False), (640, 1, 1, False),
                                            (1920, 14, 2, True), (1152, 5, 1, True), (1000, 4, 2, True),
                                            (2177, 3, 1, False)])
def test_user_index_through_sparse_prefill(n, hq, hkv, mixed):
    # random strictly ascending lists with the diagonal block; odd group sizes and odd block
    # counts pair a head's adjacent query blocks in one CTA
    q, k, v = (t.to(dev()) for t in W.random_qkv(hq, hkv, n, seed=5))
    nb = -(-n // 128)  # partial last block when n is not a multiple of 128
    rng = np.random.default_rng(9)
    cap = nb * (nb + 1) // 2
    row_ptr = np.zeros((hq, nb + 1), dtype=np.int32)
    cols = np.zeros((hq, cap), dtype=np.int32)
    lists = {}
    for h in range(hq):
        lists[h] = []
        pos = 0
        for qb in range(nb):
            sel = sorted({qb} | set(rng.choice(qb + 1, size=min(qb + 1, 4), replace=False).tolist()))
            lists[h].append(sel)
            cols[h, pos:pos + len(sel)] = sel
            pos += len(sel)
            row_ptr[h, qb + 1] = pos
    # a mixed route splits each group into classes that are scheduled apart
    route = torch.from_numpy(rng.integers(0, 2, size=hq).astype(np.int32)) if mixed else torch.zeros(hq, dtype=torch.int32)
    idx = crisp.Index(route.to(dev()), torch.zeros(hq, device=dev()),
                      torch.from_numpy(row_ptr).to(dev()), torch.from_numpy(cols).to(dev()))
    ws = crisp.workspace(hq, hkv, n, dev())
    o, lse = crisp.sparse_prefill(q, k, v, idx, ws=ws)
    crisp.check_status(ws)
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, lists,
                                                       [(h, qb) for h in range(hq) for qb in range(nb)], hq // hkv))


def _dense_index(hq, nb):
    cap = nb * (nb + 1) // 2
    row_ptr = np.zeros((hq, nb + 1), dtype=np.int32)
    cols = np.zeros((hq, cap), dtype=np.int32)
    for h in range(hq):
        pos = 0
        for qb in range(nb):
            cols[h, pos:pos + qb + 1] = np.arange(qb + 1)
            pos += qb + 1
            row_ptr[h, qb + 1] = pos
    return row_ptr, cols


@pytest.mark.parametrize("corrupt", ["out_of_range", "not_ascending", "duplicate", "row_too_long", "row_beyond_cap"])
def test_malformed_index_is_reported(corrupt):
    # A malformed user index never reads outside K/V: the kernel reports CRISP_ERR_DEVICE_CHECK.
    n, hq = 1024, 4
    q, k, v = (t.to(dev()) for t in W.random_qkv(hq, 2, n, seed=3))
    nb = n // 128
    row_ptr, cols = _dense_index(hq, nb)
    qb = 5
    beg = row_ptr[3, qb]
    if corrupt == "out_of_range":
        cols[3, beg + 2] = 99
    elif corrupt == "not_ascending":
        cols[3, beg + 2], cols[3, beg + 3] = cols[3, beg + 3], cols[3, beg + 2]
    elif corrupt == "duplicate":
        cols[3, beg + 2] = cols[3, beg + 1]
    elif corrupt == "row_too_long":
        row_ptr[3, qb + 1] += 5  # row qb claims more entries than blocks 0..qb
    else:
        row_ptr[3, nb] = cols.shape[1] + 3  # last row ends past the head's column array
    idx = crisp.Index(torch.zeros(hq, dtype=torch.int32, device=dev()), torch.zeros(hq, device=dev()),
                      torch.from_numpy(row_ptr).to(dev()), torch.from_numpy(cols).to(dev()))
    ws = crisp.workspace(hq, 2, n, dev())
    crisp.sparse_prefill(q, k, v, idx, ws=ws)
    assert crisp.get_status(ws) == -7
    assert crisp.get_status(ws) == 0  # read and cleared
    # a head pair without malformed rows is unaffected
    lists = {0: [list(range(b + 1)) for b in range(nb)]}
    o, lse = crisp.sparse_prefill(q, k, v, idx, ws=ws)
    crisp.get_status(ws)
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, lists, [(0, b) for b in range(nb)], 2))


def test_bad_arguments_raise():
    q, k, v = (t.to(dev()) for t in W.random_qkv(2, 1, 256, seed=1))
    with pytest.raises(crisp.CrispError):
        crisp.select(q, k, crisp.Params(alpha=-1.0))
    with pytest.raises(ValueError):
        crisp.select(q.float(), k)
    ws = torch.zeros(1024, dtype=torch.uint8, device=dev())
    with pytest.raises(crisp.CrispError) as e:
        crisp.select(q, k, ws=ws)
    assert e.value.code == -3
    assert crisp.get_status(ws) == 0


# ------------------------------------------------------------- FlexPrefill rules, median floor, alpha
RULES = {
    "flexprefill": crisp.Params.flexprefill(),
    "jsd_route_only": crisp.Params(route_rule=1),
    "gamma_vs_only": crisp.Params(vs_rule=1),
    "median_floor": crisp.Params(floor_rule=1),
    "median_floor_min8": crisp.Params(floor_rule=1, min_blocks=8),
    "alpha_1.25": crisp.Params(alpha=1.25),
    "alpha_1.5": crisp.Params(alpha=1.5),
    "flexprefill_gamma_0.9": crisp.Params.flexprefill(gamma=0.9),
}


@pytest.mark.parametrize("rule", sorted(RULES))
@pytest.mark.parametrize("name,n", [("llama8b_32k", 8192), ("qwen7b_128k", 4096)])
def test_rule_variants_match_oracle(rule, name, n):
    params = RULES[rule]
    w = W.WORKLOADS[name].scaled(n)
    q, k, v, meta = W.generate(w)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    idx, ws = run_select(q, k, params)
    heads = list(range(w.h_q))
    sels = PT.oracle_select_heads(q, k, params, heads)
    nb = w.n // 128
    PT.compare_selection(idx, sels, nb, name=f"{rule} {name} at n={n}")
    G = w.h_q // w.h_kv
    if params.route_rule:
        for h in heads:
            assert int(idx.route[h]) == int(meta["concentrated"][h]), (h, float(idx.debug[h, 2 * nb + 4]))
    o, lse = crisp.sparse_prefill(q, k, v, idx, ws=ws)
    crisp.check_status(ws)
    ah = [0, 2, w.h_q - 1]
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, all_lists(idx, ah),
                                                       sample_blocks(nb, ah, 3, seed=n), G))


def test_flexprefill_full_128k():
    """The baseline rules at the 128k Llama geometry: routes follow the planted structure, and
    the gamma rule collapses sink-dominated Vertical-Slash heads onto their anchors."""
    w = W.WORKLOADS["llama8b_128k"]
    q, k, v, meta = W.generate(w, device=dev())
    params = crisp.Params.flexprefill()
    ws = crisp.workspace(w.h_q, w.h_kv, w.n, dev())
    idx = crisp.Index.empty(w.h_q, w.n, dev(), debug=True)
    o, lse, idx = crisp.prefill(q, k, v, params, index=idx, ws=ws)
    crisp.check_status(ws)
    nb = w.n // 128
    heads = [0, 1, 2, 3, 12, 13, 30, 31]
    sels = PT.oracle_select_heads(q, k, params, heads)
    PT.compare_selection(idx, sels, nb, name="flexprefill llama8b_128k")
    for h in range(w.h_q):
        assert int(idx.route[h]) == int(meta["concentrated"][h])
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, all_lists(idx, [0, 2]),
                                                       sample_blocks(nb, [0, 2], 1, seed=3), w.h_q // w.h_kv))


# ------------------------------------------------------------------ lengths not a multiple of 128
def _ragged(name, n):
    """The workload's generator at the next multiple of 128, cut to n tokens."""
    w = W.WORKLOADS[name].scaled(-(-n // 128) * 128)
    q, k, v, meta = W.generate(w)
    cut = lambda t: t[:, :n].contiguous().to(dev())  # noqa: E731
    return w, cut(q), cut(k), cut(v)


@pytest.mark.parametrize("name,n,rules", [("tiny_1h_4k", 300, "crisp"), ("tiny_1h_4k", 200, "crisp"),
                                          ("llama8b_32k", 4000, "crisp"), ("qwen7b_128k", 3001, "crisp"),
                                          ("llama8b_32k", 4000, "flexprefill"), ("qwen7b_128k", 2177, "median_floor"),
                                          ("llama8b_32k", 4095, "crisp"), ("llama8b_32k", 3969, "crisp")])
def test_ragged_selection_and_attention(name, n, rules):
    params = {"crisp": crisp.Params(), "flexprefill": crisp.Params.flexprefill(),
              "median_floor": crisp.Params(floor_rule=1)}[rules]
    w, q, k, v = _ragged(name, n)
    nb = -(-n // 128)
    ws = crisp.workspace(w.h_q, w.h_kv, n, dev())
    idx = crisp.Index.empty(w.h_q, n, dev(), debug=True)
    o, lse, idx = crisp.prefill(q, k, v, params, index=idx, ws=ws)
    crisp.check_status(ws)
    heads = list(range(w.h_q))
    sels = PT.oracle_select_heads(q, k, params, heads)
    PT.compare_selection(idx, sels, nb, name=f"ragged {name} n={n} {rules}")
    G = w.h_q // w.h_kv
    ah = sorted({0, w.h_q // 2, w.h_q - 1})
    blocks = [(h, qb) for h in ah for qb in sorted({0, nb // 2, nb - 2, nb - 1}) if qb >= 0]
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, all_lists(idx, ah), blocks, G))


def test_varlen_batch_equals_single_sequences():
    """A packed batch gives, for every sequence, exactly what crisp_prefill gives for that sequence
    alone (same kernels, same inputs), and the oracle agrees on sampled blocks."""
    import dataclasses
    lens = [300, 1024, 128, 0, 2177]
    seqs = []
    for i, n in enumerate(lens):
        if n == 0:
            seqs.append(None)
            continue
        w = dataclasses.replace(W.WORKLOADS["llama8b_32k"].scaled(-(-n // 128) * 128), seed=100 + i)
        q, k, v, _ = W.generate(w)
        seqs.append(tuple(t[:, :n].contiguous() for t in (q, k, v)))
    parts = [s for s in seqs if s is not None]
    q, k, v = (torch.cat([s[j] for s in parts], dim=1).to(dev()) for j in range(3))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    params = crisp.Params()
    o, lse = crisp.prefill_varlen(q, k, v, cu, params)
    torch.cuda.synchronize()
    G = q.shape[0] // k.shape[0]
    for i, n in enumerate(lens):
        if n == 0:
            continue
        qs, ks, vs = (t.to(dev()) for t in seqs[i])
        ws = crisp.workspace(qs.shape[0], ks.shape[0], n, dev())
        os_, ls_, idx = crisp.prefill(qs, ks, vs, params, ws=ws)
        crisp.check_status(ws)
        b, e = int(cu[i]), int(cu[i + 1])
        assert torch.equal(o[:, b:e], os_), i
        assert torch.equal(lse[:, b:e], ls_), i
        nb = -(-n // 128)
        heads = [0, 17]
        PT.assert_attention_ok(PT.compare_attention_blocks(qs, ks, vs, os_, ls_, all_lists(idx, heads),
                                                           [(h, qb) for h in heads for qb in {0, nb - 1}], G))


# ------------------------------------------------------------------------------ full-size workloads
def _full(name, sel_heads, attn_per_head, attn_heads=None, seed=0):
    w = W.WORKLOADS[name]
    q, k, v, meta = W.generate(w, device=dev())
    params = crisp.Params()
    ws = crisp.workspace(w.h_q, w.h_kv, w.n, dev())
    idx = crisp.Index.empty(w.h_q, w.n, dev(), debug=True)
    o, lse, idx = crisp.prefill(q, k, v, params, index=idx, ws=ws)
    crisp.check_status(ws, name)
    nb = w.n // 128
    sels = PT.oracle_select_heads(q, k, params, sel_heads)
    log = []
    PT.compare_selection(idx, sels, nb, log, name=name)
    G = w.h_q // w.h_kv
    for h in sel_heads:
        assert int(idx.route[h]) == int(meta["concentrated"][h])
    attn_heads = attn_heads if attn_heads is not None else sel_heads
    lists = all_lists(idx, attn_heads)
    blocks = sample_blocks(nb, attn_heads, attn_per_head, seed=seed)
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, lists, blocks, G))
    return idx, meta


def test_llama_32k_full():
    _full("llama8b_32k", list(range(32)), 2)


def test_llama_128k_full():
    idx, meta = _full("llama8b_128k", list(range(32)), 1, attn_heads=[0, 1, 2, 3, 12, 13, 30, 31])
    found = total = 0
    for h in range(32):
        if meta["concentrated"][h]:
            rows = idx.lists(h)
            last = set(rows[-1])
            verts = set(meta["vertical_blocks"][h // 4])
            assert verts <= last, h
            for off in meta["slash_offsets"][h // 4]:
                total += 1
                found += (1023 - off // 128) in last
    assert found >= 0.8 * total


def test_qwen_128k_full():
    _full("qwen7b_128k", list(range(28)), 1, attn_heads=[0, 4, 5, 6, 27])


def test_llama_512k_all_heads():
    """Selection of every head at 512k against the oracle (the PE heads' global cuts run over
    8,390,656 pooled entries each); attention on sampled query blocks of three heads."""
    _full("llama8b_512k", list(range(32)), 1, attn_heads=[0, 2, 31])
