"""C-ABI checks that need no GPU: the library loads, exports every declared entry point, sizes
its workspace, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest
import torch

import dynamic_block_sparse_proxy_b200 as crisp
from dynamic_block_sparse_proxy_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "crisp.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return crisp.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(crisp_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(crisp.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in crisp.STATUS_NAMES.items():
        assert L.crisp_status_string(code).decode() == name
    assert L.crisp_status_string(12345).decode() == "CRISP_ERR_UNKNOWN"


def test_workspace_size(L):
    p = crisp.Params().c()
    small = L.crisp_workspace_size(1, 1, 4096, 128, ctypes.byref(p))
    big = L.crisp_workspace_size(32, 8, 131072, 128, ctypes.byref(p))
    assert 0 < small < big
    # dominated by the per-head pooled-score and column arrays: 2 * 4 B * h_q * N_b(N_b+1)/2
    nb = 131072 // 128
    assert big > 8 * 32 * nb * (nb + 1) // 2
    assert big % 256 == 0
    for bad in [(1, 1, 4096, 64), (1, 1, 100, 128), (3, 2, 4096, 128), (0, 1, 4096, 128), (1, 1, 0, 128)]:
        assert L.crisp_workspace_size(*bad, ctypes.byref(p)) == 0
    q = crisp.Params(block=64).c()
    assert L.crisp_workspace_size(1, 1, 4096, 128, ctypes.byref(q)) == 0


def _idx(route=1, c=1, rp=1, cols=1):
    return crisp._Index(0x1000 if route else None, 0x1000 if c else None, 0x1000 if rp else None,
                        0x1000 if cols else None, None)


def test_select_rejects_bad_arguments_before_launch(L):
    p = crisp.Params().c()
    ws = 0x100000
    big = 1 << 40
    fake = 0x10000
    ix = _idx()
    cases = [
        ((None, fake, 1, 1, 4096, 128, ctypes.byref(p), ctypes.byref(ix), ws, big, None), crisp.STATUS_NAMES[-1]),
        ((fake, fake, 1, 1, 4096, 64, ctypes.byref(p), ctypes.byref(ix), ws, big, None), crisp.STATUS_NAMES[-2]),
        ((fake, fake, 1, 1, 100, 128, ctypes.byref(p), ctypes.byref(ix), ws, big, None), crisp.STATUS_NAMES[-2]),
        ((fake, fake, 3, 2, 4096, 128, ctypes.byref(p), ctypes.byref(ix), ws, big, None), crisp.STATUS_NAMES[-2]),
        ((fake, fake, 1, 1, 4096, 128, None, ctypes.byref(ix), ws, big, None), crisp.STATUS_NAMES[-1]),
        ((fake, fake, 1, 1, 4096, 128, ctypes.byref(p), None, ws, big, None), crisp.STATUS_NAMES[-1]),
        ((fake, fake, 1, 1, 4096, 128, ctypes.byref(p), ctypes.byref(_idx(rp=0)), ws, big, None), crisp.STATUS_NAMES[-1]),
        ((fake, fake, 1, 1, 4096, 128, ctypes.byref(p), ctypes.byref(ix), ws, 1024, None), crisp.STATUS_NAMES[-3]),
        ((fake, fake, 1, 1, 4096, 128, ctypes.byref(p), ctypes.byref(ix), ws + 8, big, None), crisp.STATUS_NAMES[-1]),
        ((fake + 2, fake, 1, 1, 4096, 128, ctypes.byref(p), ctypes.byref(ix), ws, big, None), crisp.STATUS_NAMES[-1]),
    ]
    for args, want in cases:
        assert crisp.STATUS_NAMES[L.crisp_select(*args)] == want, args
    for bad in (crisp.Params(alpha=-1.0), crisp.Params(gamma=0.0), crisp.Params(min_blocks=-1),
                crisp.Params(tau_proxy=float("nan")), crisp.Params(anchors=64), crisp.Params(route_rule=2),
                crisp.Params(vs_rule=-1), crisp.Params(floor_rule=3), crisp.Params(tau_jsd=-0.5),
                crisp.Params(tau_jsd=float("inf"))):
        bp = bad.c()
        rc = L.crisp_select(fake, fake, 1, 1, 4096, 128, ctypes.byref(bp), ctypes.byref(ix), ws, big, None)
        assert rc in (-1, -2), bad


def test_lengths_not_multiple_of_128(L):
    # any length sizes a workspace; selection needs n >= 128 (the proxy takes the last 128 queries)
    # (fake pointers only with arguments refused before any launch)
    p = crisp.Params().c()
    assert L.crisp_workspace_size(2, 1, 1000, 128, None) > 0
    assert L.crisp_workspace_size(2, 1, 1000, 128, ctypes.byref(p)) > 0
    assert L.crisp_workspace_size(2, 1, 100, 128, ctypes.byref(p)) == 0
    assert L.crisp_workspace_size(2, 1, 100, 128, None) > 0
    ix = _idx()
    assert L.crisp_select(0x10000, 0x10000, 2, 1, 100, 128, ctypes.byref(p), ctypes.byref(ix), 0x100000,
                          1 << 40, None) == -2


def test_selection_beyond_8192_blocks_is_unsupported(L):
    p = crisp.Params().c()
    ix = _idx()
    n = 128 * 8193
    rc = L.crisp_select(0x10000, 0x10000, 1, 1, n, 128, ctypes.byref(p), ctypes.byref(ix), 0x100000, 1 << 40, None)
    assert rc == -2
    rc = L.crisp_select_noalloc(0x10000, 0x10000, 1, 1, n, 128, ctypes.byref(p), ctypes.byref(ix), None, None)
    assert rc == -2


def test_attention_entry_points_reject_bad_arguments(L):
    fake, ws, big = 0x10000, 0x100000, 1 << 40
    ix = _idx()
    assert L.crisp_sparse_prefill(fake, fake, None, 1, 1, 4096, 128, ctypes.byref(ix), fake, None, ws, big, None) == -1
    assert L.crisp_sparse_prefill(fake, fake, fake, 1, 1, 4096, 128, ctypes.byref(_idx(cols=0)), fake, None, ws, big,
                                  None) == -1
    assert L.crisp_sparse_prefill(fake, fake, fake, 1, 1, 4096, 128, ctypes.byref(ix), None, None, ws, big, None) == -1
    assert L.crisp_sparse_prefill(fake, fake, fake, 1, 1, 4096, 128, ctypes.byref(ix), fake, None, ws, 10, None) == -3
    # (fake pointers only with arguments refused before any launch)
    assert L.crisp_dense_prefill(fake, fake, fake, 1, 1, 4096, 64, fake, None, ws, big, None) == -2
    assert L.crisp_dense_prefill(fake, fake, fake, 2, 4, 4096, 128, fake, None, ws, big, None) == -2
    p = crisp.Params().c()
    assert L.crisp_prefill(fake, fake, fake, 1, 1, 4096, 128, ctypes.byref(p), fake, None, None, ws, 10, None) == -3
    assert L.crisp_prefill(fake, fake, fake, 1, 1, 4096, 128, None, fake, None, None, ws, big, None) == -1
    assert L.crisp_get_status(None, None) == -1
    assert L.crisp_selftest_timeout(None, 0, 10, None) == -1


def test_overflowing_sizes_are_refused(L):
    p = crisp.Params().c()
    # N_b (N_b+1)/2 beyond 2^31 entries per head
    assert L.crisp_workspace_size(1, 1, 128 * 70000, 128, ctypes.byref(p)) == 0


def test_compute_calls_fail_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(crisp, "_lib", None)
    monkeypatch.setattr(crisp, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        crisp.lib()


def test_binding_sizes_the_index_by_ceil_blocks_and_checks_it():
    assert crisp.n_blocks(300) == 3 and crisp.n_blocks(256) == 2 and crisp.n_blocks(1) == 1
    # an index the library would overrun is refused before any call (CPU tensors fail the check too)
    import torch
    h_q, n = 2, 300
    small = crisp.Index(torch.zeros(h_q, dtype=torch.int32), torch.zeros(h_q), torch.zeros(h_q, 3, dtype=torch.int32),
                        torch.zeros(h_q, 3, dtype=torch.int32))
    with pytest.raises(ValueError):
        small.check(h_q, n)


def test_varlen_refuses_bad_batches_before_launch(L):
    # (fake pointers only with arguments refused before any launch)
    p = crisp.Params().c()
    fake, ws, big = 0x10000, 0x100000, 1 << 40
    I32 = ctypes.c_int32

    def call(cu, total, ws_bytes=big):
        arr = (I32 * len(cu))(*cu)
        return L.crisp_prefill_varlen(fake, fake, fake, 2, 1, total, arr, len(cu) - 1, 128, ctypes.byref(p), fake,
                                      None, ws, ws_bytes, None)

    assert L.crisp_prefill_varlen(fake, fake, fake, 2, 1, 512, None, 2, 128, ctypes.byref(p), fake, None, ws, big,
                                  None) == -1
    assert call([1, 256, 512], 512) == -1          # does not start at 0
    assert call([0, 256, 500], 512) == -1          # does not end at total
    assert call([0, 300, 256, 512], 512) == -1     # decreasing
    assert call([0, 50, 512], 512) == -2           # a sequence shorter than 128 tokens
    assert call([0, 256, 512], 512, ws_bytes=100) == -3
    assert call([0, 0, 0], 0) == -1                # nothing to do (total = 0)


def test_params_pack_into_the_c_struct():
    p = crisp.Params.flexprefill(gamma=0.9, tau_jsd=0.2).c()
    assert (p.block, p.anchors, p.route_rule, p.vs_rule, p.floor_rule) == (128, 128, 1, 1, 0)
    assert abs(p.gamma - 0.9) < 1e-7 and abs(p.tau_jsd - 0.2) < 1e-7
    assert ctypes.sizeof(crisp._Params) == 40  # 10 four-byte fields, as in include/crisp.h
    q = crisp.Params(floor_rule=1, min_blocks=8).c()
    assert (q.floor_rule, q.min_blocks, q.route_rule) == (1, 8, 0)


def test_binding_refuses_outputs_of_the_wrong_shape_before_calling():
    import torch
    q = torch.zeros(2, 256, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        crisp._check_out(q, torch.zeros(2, 256, 128, dtype=torch.float32), None)     # dtype
    with pytest.raises(ValueError):
        crisp._check_out(q, torch.zeros(2, 256, 128, dtype=torch.bfloat16), None)    # not on the GPU
    with pytest.raises(ValueError):
        crisp._qkv_shape(q, q)                                                       # CPU tensors


def test_workspace_grows_with_length_including_partial_blocks(L):
    sizes = [L.crisp_workspace_size(4, 2, n, 128, None) for n in (1, 127, 128, 129, 1000, 1024, 1025)]
    assert all(s > 0 and s % 256 == 0 for s in sizes)
    assert sizes == sorted(sizes)
    assert sizes[2] == L.crisp_workspace_size(4, 2, 128, 128, None) and sizes[3] > sizes[2]


def test_fp8qk_buffer_size_and_argument_checks(L):
    """The FP8 entry points: the buffer size follows the layout crisp.h documents (and the binding's
    views mirror it), and a missing, misaligned or short buffer is refused before any launch."""
    def layout(h_q, h_kv, n):
        nb = -(-n // 128)
        off = 0
        for nbytes in (h_q * n * 128, h_kv * n * 128, h_q * nb * 4, h_kv * nb * 4):
            off = -(-(off + nbytes) // 256) * 256
        return off
    for h_q, h_kv, n in ((32, 8, 131072), (28, 4, 3001), (1, 1, 1), (4, 2, 300)):
        assert L.crisp_fp8qk_buffer_size(h_q, h_kv, n, 128) == layout(h_q, h_kv, n)
    assert L.crisp_fp8qk_buffer_size(1, 1, 4096, 64) == 0
    buf = torch.zeros(layout(4, 2, 300), dtype=torch.uint8)
    q8, k8, qs, ks = crisp.fp8qk_views(buf, 4, 2, 300)
    assert q8.shape == (4, 300, 128) and k8.shape == (2, 300, 128) and qs.shape == (4, 3) and ks.shape == (2, 3)
    assert ks.data_ptr() + ks.numel() * 4 <= buf.data_ptr() + buf.numel()
    fake, ws, big = 0x10000, 0x100000, 1 << 40
    ix = _idx()
    assert L.crisp_sparse_prefill_fp8qk(fake, fake, fake, 1, 1, 4096, 128, ctypes.byref(ix), fake, None, ws, big,
                                        None, big, None) == -1
    assert L.crisp_sparse_prefill_fp8qk(fake, fake, fake, 1, 1, 4096, 128, ctypes.byref(ix), fake, None, ws, big,
                                        fake + 16, big, None) == -1
    assert L.crisp_sparse_prefill_fp8qk(fake, fake, fake, 1, 1, 4096, 128, ctypes.byref(ix), fake, None, ws, big,
                                        ws, 100, None) == -3
