"""crisp_select_noalloc against crisp_select, through the C ABI.

Some callers cannot allocate device memory: a serving engine whose memory manager owns every
device byte, or a latency-critical path that cannot afford the device synchronisation an
allocation implies. They call crisp_select_noalloc, which keeps its scratch in a fixed array
inside the library instead of a caller-provided workspace. Its index must equal crisp_select's
exactly on consecutive calls over different inputs of the same shape (the array keeps the
previous call's contents, so nothing stale may leak through), and shapes that need more scratch
than the array holds must be refused before anything is launched.
"""
import ctypes

import pytest
import torch

import dynamic_block_sparse_proxy_b200 as crisp
from dynamic_block_sparse_proxy_b200 import build as B
from dynamic_block_sparse_proxy_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _entry():
    B.build()
    f = crisp.lib().crisp_select_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.POINTER(crisp._Params), ctypes.POINTER(crisp._Index), ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _call(f, q, k, params, index, status):
    h_q, n, d = q.shape
    p, ix = params.c(), index.c()
    stream = ctypes.c_void_p(torch.cuda.current_stream(q.device).cuda_stream)
    return f(q.data_ptr(), k.data_ptr(), h_q, k.shape[0], n, d, ctypes.byref(p), ctypes.byref(ix),
             status.data_ptr() if status is not None else None, stream)


def _same_index(a, b, nb):
    assert torch.equal(a.route, b.route)
    assert torch.equal(a.c_struct, b.c_struct)
    assert torch.equal(a.row_ptr, b.row_ptr)
    assert torch.equal(a.debug, b.debug)
    for h in range(a.route.numel()):
        used = int(a.row_ptr[h, nb])
        assert torch.equal(a.cols[h, :used], b.cols[h, :used]), h


def test_noalloc_select_matches_select_on_consecutive_calls():
    """Per shape: planted inputs, then different inputs of the same shape (all heads diffuse, so
    every head takes the other route and its scratch regions hold other values), then the
    planted inputs again; each call must equal crisp_select on its own inputs."""
    dev = torch.device("cuda:0")
    f = _entry()
    cases = [(W.WORKLOADS["llama8b_32k"].scaled(4096), crisp.Params()),
             (W.WORKLOADS["qwen7b_128k"].scaled(2048), crisp.Params(min_blocks=4))]
    for w, params in cases:
        q, k, _, _ = W.generate(w)
        q2, k2, _ = W.random_qkv(w.h_q, w.h_kv, w.n, seed=w.n + 1)
        inputs = [(q.to(dev), k.to(dev)), (q2.to(dev), k2.to(dev))]
        refs = []
        for qq, kk in inputs:
            refs.append(crisp.select(qq, kk, params, debug=True))
        torch.cuda.synchronize()
        assert not torch.equal(refs[0].route, refs[1].route)
        for which in (0, 1, 0):
            qq, kk = inputs[which]
            got = crisp.Index.empty(w.h_q, w.n, dev, debug=True)
            status = torch.zeros(1, dtype=torch.int32, device=dev)
            assert _call(f, qq, kk, params, got, status) == 0
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            _same_index(refs[which], got, w.n // 128)


def test_noalloc_select_refuses_shapes_beyond_its_array():
    dev = torch.device("cuda:0")
    f = _entry()
    w = W.WORKLOADS["llama8b_128k"]
    # 32 heads at 128k tokens need far more than 32 MiB of scratch: refused before any launch
    assert crisp.workspace_size(w.h_q, w.h_kv, w.n) > (32 << 20)
    q = torch.empty(w.h_q, w.n, w.d, dtype=torch.bfloat16, device=dev)
    k = torch.empty(w.h_kv, w.n, w.d, dtype=torch.bfloat16, device=dev)
    idx = crisp.Index.empty(w.h_q, w.n, dev)
    assert _call(f, q, k, crisp.Params(), idx, None) == -3
