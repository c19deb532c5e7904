"""The FP8 variant of the attention logits (crisp_sparse_prefill_fp8qk) against the oracle.

Two separate checks, so that the oracle never takes an input from the GPU:
- the quantisation itself: the E4M3 codes and per-block scales the library leaves in its buffer
  equal, bit for bit, the oracle's per-block quantisation (quantize_blocks_fp8) of the same bf16
  Q and K;
- the attention: the kernel's output equals the exact fp64 attention of the oracle's dequantised
  Q and K (and the same V) on the same index set, within the bf16 kernel's tolerance (2e-2 max /
  2e-3 mean abs on O, 5e-3 on the LSE), since the kernel computes that attention up to its own
  fp32 accumulation and bf16 P.
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


@pytest.fixture(scope="module")
def built():
    B.build()
    crisp.lib()


def dev():
    return torch.device("cuda:0")


def _dequantised(x: torch.Tensor) -> tuple[torch.Tensor, np.ndarray, np.ndarray]:
    """Oracle quantisation of every head of x [heads, n, d] (bf16): (fp64 dequantised values,
    codes [heads, n, d], scales [heads, N_b])."""
    codes, scales, deq = [], [], []
    for h in range(x.shape[0]):
        c, s = O.quantize_blocks_fp8(PT.f64(x[h]))
        codes.append(c)
        scales.append(s)
        deq.append(O.dequantize_blocks_fp8(c, s))
    return torch.from_numpy(np.stack(deq)), np.stack(codes), np.stack(scales)


@pytest.mark.parametrize("name,n", [("tiny_1h_4k", 4096), ("llama8b_32k", 8192), ("llama8b_32k", 3001)])
def test_fp8_codes_and_scales_bit_exact(built, name, n):
    w = W.WORKLOADS[name].scaled(-(-n // 128) * 128)
    q, k, v, _ = W.generate(w)
    q, k, v = (t[:, :n].contiguous() for t in (q, k, v))
    qd, kd, vd = q.to(dev()), k.to(dev()), v.to(dev())
    idx = crisp.select(qd, kd, crisp.Params()) if n >= 128 else None
    o, lse, buf = crisp.sparse_prefill_fp8qk(qd, kd, vd, idx)
    torch.cuda.synchronize()
    q8, k8, qs, ks = crisp.fp8qk_views(buf, w.h_q, w.h_kv, n)
    for x, codes, scales in ((q, q8, qs), (k, k8, ks)):
        _, oc, osc = _dequantised(x)
        gc = codes.cpu().numpy()
        bad = np.nonzero(gc != oc)
        assert bad[0].size == 0, (name, n, bad[0][:5], bad[1][:5], gc[bad][:5], oc[bad][:5])
        assert np.array_equal(scales.cpu().numpy(), osc), (name, n)


def _edge_blocks() -> torch.Tensor:
    """Two heads of 640 rows whose blocks reach the quantiser's special cases: all zeros, all
    negative zeros (scale 1 and codes 0 either way), one large value beside values a million times
    smaller (subnormal and zero codes), and a block whose maximum is exactly 448, so that values
    pass unscaled and those halfway between E4M3 neighbours, subnormal and normal, positive and
    negative, are settled by the ties-to-even rule."""
    n, d = 640, 128
    g = torch.Generator().manual_seed(3)
    x = torch.randn(2, n, d, generator=g)
    x[0, 0:128] = 0.0
    x[0, 128:256] = -0.0
    x[0, 256:384] *= 1e-3
    x[0, 300, 5] = 1e3
    t = torch.zeros(128, d)
    t[0, 0] = 448.0
    halfway = [(m + 0.5) * 2.0 ** -9 for m in range(8)] + [1.0625, 1.1875, 17.0, 19.0, 104.0, 0.0146484375]
    for i, val in enumerate(halfway):
        t[1 + i, :] = val
        t[40 + i, :] = -val
    x[1, 128:256] = t
    return x.to(torch.bfloat16)


def test_fp8_codes_edge_blocks_bit_exact(built):
    q = _edge_blocks()
    k = _edge_blocks()[:1].flip(1).contiguous()
    v = torch.randn(1, q.shape[1], 128, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    qd, kd, vd = q.to(dev()), k.to(dev()), v.to(dev())
    ws = crisp.workspace(2, 1, q.shape[1], dev())
    idx = crisp.select(qd, kd, crisp.Params(), ws=ws)
    o, lse, buf = crisp.sparse_prefill_fp8qk(qd, kd, vd, idx, ws=ws)
    crisp.check_status(ws)
    q8, k8, qs, ks = crisp.fp8qk_views(buf, 2, 1, q.shape[1])
    for x, codes, scales in ((q, q8, qs), (k, k8, ks)):
        _, oc, osc = _dequantised(x)
        gc = codes.cpu().numpy()
        bad = np.nonzero(gc != oc)
        assert bad[0].size == 0, (bad[0][:5], bad[1][:5], bad[2][:5], gc[bad][:5], oc[bad][:5])
        assert np.array_equal(scales.cpu().numpy(), osc)
    assert torch.isfinite(o.float()).all()


@pytest.mark.parametrize("name,n", [("tiny_1h_4k", 4096), ("llama8b_32k", 8192), ("llama8b_32k", 3001)])
def test_fp8_attention_matches_dequantised_oracle(built, name, n):
    w = W.WORKLOADS[name].scaled(-(-n // 128) * 128)
    q, k, v, _ = W.generate(w)
    q, k, v = (t[:, :n].contiguous() for t in (q, k, v))
    qd, kd, vd = q.to(dev()), k.to(dev()), v.to(dev())
    ws = crisp.workspace(w.h_q, w.h_kv, n, dev())
    idx = crisp.select(qd, kd, crisp.Params(), ws=ws)
    o, lse, _ = crisp.sparse_prefill_fp8qk(qd, kd, vd, idx, ws=ws)
    crisp.check_status(ws)
    qq, _, _ = _dequantised(q)
    kq, _, _ = _dequantised(k)
    nb = -(-n // 128)
    G = w.h_q // w.h_kv
    heads = sorted({0, w.h_q // 2, w.h_q - 1})
    lists = {h: idx.lists(h) for h in heads}
    blocks = [(h, qb) for h in heads for qb in sorted({0, nb // 2, nb - 2, nb - 1}) if qb >= 0]
    PT.assert_attention_ok(PT.compare_attention_blocks(qq, kq, v, o, lse, lists, blocks, G))


def test_fp8_dense_index_equals_dense_oracle(built):
    """Every causal block selected: the FP8 kernel against dense causal attention of the
    dequantised inputs (two heads sharing one kv-head, so both CTA tile pairings run)."""
    n, hq, hkv = 1024, 2, 1
    q, k, v = W.random_qkv(hq, hkv, n, seed=11)
    nb = n // 128
    cap = nb * (nb + 1) // 2
    row_ptr = torch.tensor([[qb * (qb + 1) // 2 for qb in range(nb + 1)]] * hq, dtype=torch.int32)
    cols = torch.tensor([[kb for qb in range(nb) for kb in range(qb + 1)]] * hq, dtype=torch.int32)
    idx = crisp.Index(torch.ones(hq, dtype=torch.int32, device=dev()), torch.zeros(hq, device=dev()),
                      row_ptr.to(dev()), cols.to(dev()))
    assert cols.shape[1] == cap
    o, lse, _ = crisp.sparse_prefill_fp8qk(q.to(dev()), k.to(dev()), v.to(dev()), idx)
    torch.cuda.synchronize()
    qq, _, _ = _dequantised(q)
    kq, _, _ = _dequantised(k)
    lists = {h: [list(range(qb + 1)) for qb in range(nb)] for h in range(hq)}
    blocks = [(h, qb) for h in range(hq) for qb in range(nb)]
    PT.assert_attention_ok(PT.compare_attention_blocks(qq, kq, v, o, lse, lists, blocks, hq // hkv))
