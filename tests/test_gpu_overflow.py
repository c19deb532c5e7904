"""The softmax reference handling of both tcgen05 kernels, on inputs that force it.

Both kernels exponentiate a key block against the row reference of the blocks before it and redo
the block against its own maximum (rescaling what was accumulated) only when its exponentials
would sum past 2^64, i.e. when its logits lie more than 64 / log2(e) ~ 44.4 nats above that
reference. These inputs plant one key block whose logits sit 60 or 100 nats above the first
block the walk meets (100 nats overflow fp32 outright), and check the attention output against
the fp64 oracle (2e-2 max / 2e-3 mean abs), in both CTA tile modes (two heads at one query block,
and two adjacent query blocks of one head), through a user index, the dense entry point and
selection; and the proxy's block masses and lists against the oracle when the spike lies inside
a 16-block proxy chunk after its first block.
"""
import numpy as np
import pytest
import torch

import dynamic_block_sparse_proxy_b200 as crisp
from dynamic_block_sparse_proxy_b200 import build as B
from dynamic_block_sparse_proxy_b200 import workloads as W

from tests import parity as PT

LOG2E = 1.4426950408889634


@pytest.fixture(scope="module")
def built():
    B.build()
    crisp.lib()


def dev():
    return torch.device("cuda:0")


def _dense_lists(nb):
    return [list(range(qb + 1)) for qb in range(nb)]


def _index_from_lists(lists_by_head, nb, route):
    hq = len(lists_by_head)
    cap = nb * (nb + 1) // 2
    row_ptr = np.zeros((hq, nb + 1), dtype=np.int32)
    cols = np.zeros((hq, cap), dtype=np.int32)
    for h, lists in enumerate(lists_by_head):
        pos = 0
        for qb, sel in enumerate(lists):
            cols[h, pos:pos + len(sel)] = sel
            pos += len(sel)
            row_ptr[h, qb + 1] = pos
    return crisp.Index(torch.tensor(route, dtype=torch.int32, device=dev()), torch.zeros(hq, device=dev()),
                       torch.from_numpy(row_ptr).to(dev()), torch.from_numpy(cols).to(dev()))


def _gap_log2(q, k, h, kv, first_kb, spike_kb, rows):
    """log2 of the spiked block's sum of exponentials against the largest logit of the walk's
    first block (the quantity the kernels test against 2^64), smallest over the query rows."""
    qq = q[h].double()[rows[0]:rows[1]]
    kk = k[kv].double()
    s = qq @ kk.T / np.sqrt(128.0)
    first = s[:, first_kb * 128:(first_kb + 1) * 128].max(dim=1).values
    spike = torch.logsumexp(s[:, spike_kb * 128:(spike_kb + 1) * 128], dim=1)
    return float(((spike - first) * LOG2E).min())


@pytest.mark.parametrize("gap", [60.0, 100.0])
def test_spiked_inputs_pass_the_redo_threshold(gap):
    """CPU check of the construction: on every spiked query row the spiked block's exponentials
    sum past 2^64 times the first block's largest one, so the GPU tests below take the redo path."""
    q, k, v = W.spiked_qkv(2, 1, 1024, [3], [gap, 0.0], seed=11)
    assert _gap_log2(q, k, 0, 0, 0, 3, (512, 640)) > 64.0 + 8.0
    assert _gap_log2(q, k, 1, 0, 0, 3, (512, 640)) < 16.0
    # proxy rows: the spiked block against the first block of its 16-block chunk
    n = 4096
    q, k, v = W.spiked_qkv(4, 2, n, [5, 20], [gap, 0.0, gap, 0.0], seed=7, q_rows=(n - 128, n))
    assert _gap_log2(q, k, 0, 0, 0, 5, (n - 128, n)) > 64.0 + 8.0
    assert _gap_log2(q, k, 2, 1, 16, 20, (n - 128, n)) > 64.0 + 8.0


@pytest.mark.gpu
@pytest.mark.parametrize("gap", [60.0, 100.0])
@pytest.mark.parametrize("hq,n,gaps_of", [(2, 1024, "both"), (2, 1024, "first"), (1, 1024, "first"),
                                          (3, 1152, "mixed"), (1, 1000, "first"), (2, 1000, "both")])
def test_attention_redo_through_user_index(built, gap, hq, n, gaps_of):
    """Head-pair tiles (hq = 2), same-head two-query-block tiles (hq = 1) and both (hq = 3), at a
    length that is a multiple of 128 and a ragged one; one or both tiles of a CTA redo."""
    gaps = {"both": [gap] * hq, "first": [gap] + [0.0] * (hq - 1), "mixed": [gap, 0.0, gap][:hq]}[gaps_of]
    q, k, v = W.spiked_qkv(hq, 1, n, [3, 6], gaps, seed=int(gap) + hq)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    nb = -(-n // 128)
    lists = {h: _dense_lists(nb) for h in range(hq)}
    # a sparse list for the last head: the spike comes after two unrelated blocks
    lists[hq - 1] = [sorted({0, qb} | ({2, 3} if qb >= 3 else set()) | ({6} if qb >= 6 else set()))
                     for qb in range(nb)]
    idx = _index_from_lists([lists[h] for h in range(hq)], nb, [1] * hq)
    ws = crisp.workspace(hq, 1, n, dev())
    o, lse = crisp.sparse_prefill(q, k, v, idx, ws=ws)
    crisp.check_status(ws)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    blocks = [(h, qb) for h in range(hq) for qb in range(nb)]
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, lists, blocks, hq))


@pytest.mark.parametrize("keys", [(0, 64), (64, 128), (0, 16), (112, 128)])
def test_half_block_spikes_pass_the_redo_threshold(keys):
    """CPU check of the construction below: a spike on part of a block's keys alone lifts that
    block's exponentials past the redo threshold against the first block."""
    q, k, v = W.spiked_qkv(2, 1, 1024, [3, 6], [60.0, 100.0], seed=5, keys=keys)
    _, k0, _ = W.spiked_qkv(2, 1, 1024, [3, 6], [60.0, 100.0], seed=5, keys=(0, 0))  # no spike
    moved = (k.float() - k0.float()).abs().amax(dim=-1)[0]  # per key: touched by the spike?
    for kb in (3, 6):
        blk = moved[kb * 128:(kb + 1) * 128] > 0
        assert blk[keys[0]:keys[1]].all() and blk.sum() == keys[1] - keys[0]
    for h in range(2):
        assert _gap_log2(q, k, h, 0, 0, 3, (512, 640)) > 64.0 + 8.0


@pytest.mark.gpu
@pytest.mark.parametrize("keys", [(0, 64), (64, 128), (0, 16), (112, 128)])
@pytest.mark.parametrize("hq,n", [(2, 1024), (1, 1000)])
def test_attention_redo_by_key_range(built, keys, hq, n):
    """The spike sits in only part of a block's keys (its first or its second 64 keys, or 16 of
    them), at 60 and 100 nats, on a dense walk and a sparse one: the redo moves the reference
    whichever keys carry the spike."""
    q, k, v = W.spiked_qkv(hq, 1, n, [3, 6], [60.0, 100.0][:hq], seed=5, keys=keys)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    nb = -(-n // 128)
    lists = {h: _dense_lists(nb) for h in range(hq)}
    lists[hq - 1] = [sorted({0, qb} | ({2, 3} if qb >= 3 else set()) | ({6} if qb >= 6 else set()))
                     for qb in range(nb)]
    idx = _index_from_lists([lists[h] for h in range(hq)], nb, [1] * hq)
    ws = crisp.workspace(hq, 1, n, dev())
    o, lse = crisp.sparse_prefill(q, k, v, idx, ws=ws)
    crisp.check_status(ws)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    blocks = [(h, qb) for h in range(hq) for qb in range(nb)]
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, lists, blocks, hq))


@pytest.mark.gpu
@pytest.mark.parametrize("gap", [60.0, 100.0])
def test_dense_attention_redo(built, gap):
    hq, n = 4, 2048
    q, k, v = W.spiked_qkv(hq, 2, n, [5, 9], [gap, 0.0, gap, gap], seed=3)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    ws = crisp.workspace(hq, 2, n, dev())
    o, lse = crisp.dense_prefill(q, k, v, ws=ws)
    crisp.check_status(ws)
    nb = n // 128
    lists = {h: _dense_lists(nb) for h in range(hq)}
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, lists,
                                                       [(h, qb) for h in range(hq) for qb in range(nb)], 2))


@pytest.mark.gpu
@pytest.mark.parametrize("gap", [60.0, 100.0])
@pytest.mark.parametrize("n,spikes", [(4096, [5, 20]), (4000, [5, 29]), (2048, [1, 14])])
def test_proxy_redo_inside_a_chunk(built, gap, n, spikes):
    """The proxy rows (the last 128 queries) meet a spiked block after the first block of its
    16-block chunk: block masses, routes and lists match the oracle; attention on the result too."""
    hq = 4
    q, k, v = W.spiked_qkv(hq, 2, n, spikes, [gap, 0.0, gap, 0.0], seed=7, q_rows=(n - 128, n))
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    params = crisp.Params()
    ws = crisp.workspace(hq, 2, n, dev())
    idx = crisp.Index.empty(hq, n, dev(), debug=True)
    o, lse, idx = crisp.prefill(q, k, v, params, index=idx, ws=ws)
    crisp.check_status(ws)
    nb = -(-n // 128)
    sels = PT.oracle_select_heads(q, k, params, list(range(hq)))
    PT.compare_selection(idx, sels, nb, name=f"spiked proxy n={n} gap={gap}")
    lists = {h: idx.lists(h) for h in range(hq)}
    blocks = [(h, qb) for h in range(hq) for qb in sorted({0, spikes[0], spikes[1], nb - 2, nb - 1})]
    PT.assert_attention_ok(PT.compare_attention_blocks(q, k, v, o, lse, lists, blocks, 2))
