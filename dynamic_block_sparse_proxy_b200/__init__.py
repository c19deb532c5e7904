"""CRISP sparse prefill on B200: a thin Python binding over libcrisp.so.

Every step of selection and attention runs in the library's CUDA kernels; this module only
marshals torch tensors (device memory, current stream) into the C ABI declared in
include/crisp.h. There is no CPU fallback: without the built library (or without a CUDA
device) every compute call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcrisp.so")

OK = 0
STATUS_NAMES = {
    0: "CRISP_OK", -1: "CRISP_ERR_INVALID_ARG", -2: "CRISP_ERR_UNSUPPORTED", -3: "CRISP_ERR_WORKSPACE",
    -4: "CRISP_ERR_CUDA", -5: "CRISP_ERR_DEVICE_TIMEOUT", -6: "CRISP_ERR_OVERFLOW", -7: "CRISP_ERR_DEVICE_CHECK",
}
EXPORTED = ["crisp_workspace_size", "crisp_select", "crisp_sparse_prefill", "crisp_prefill",
            "crisp_dense_prefill", "crisp_get_status", "crisp_status_string", "crisp_selftest_timeout",
            "crisp_select_noalloc", "crisp_prefill_varlen", "crisp_fp8qk_buffer_size", "crisp_sparse_prefill_fp8qk"]


class CrispError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({code})")
        self.code = code


class _Params(ctypes.Structure):
    _fields_ = [("block", ctypes.c_int32), ("anchors", ctypes.c_int32), ("tau_proxy", ctypes.c_float),
                ("alpha", ctypes.c_float), ("gamma", ctypes.c_float), ("min_blocks", ctypes.c_int32),
                ("route_rule", ctypes.c_int32), ("tau_jsd", ctypes.c_float), ("vs_rule", ctypes.c_int32),
                ("floor_rule", ctypes.c_int32)]


class _Index(ctypes.Structure):
    _fields_ = [("route", ctypes.c_void_p), ("c_struct", ctypes.c_void_p), ("row_ptr", ctypes.c_void_p),
                ("cols", ctypes.c_void_p), ("debug", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libcrisp.so (built in-tree); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m dynamic_block_sparse_proxy_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        P, I = ctypes.POINTER(_Params), ctypes.POINTER(_Index)
        L.crisp_workspace_size.argtypes = [i32, i32, i32, i32, P]
        L.crisp_workspace_size.restype = sz
        L.crisp_select.argtypes = [vp, vp, i32, i32, i32, i32, P, I, vp, sz, vp]
        L.crisp_sparse_prefill.argtypes = [vp, vp, vp, i32, i32, i32, i32, I, vp, vp, vp, sz, vp]
        L.crisp_prefill.argtypes = [vp, vp, vp, i32, i32, i32, i32, P, vp, vp, I, vp, sz, vp]
        L.crisp_dense_prefill.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, sz, vp]
        L.crisp_prefill_varlen.argtypes = [vp, vp, vp, i32, i32, i32, ctypes.POINTER(ctypes.c_int32), i32, i32, P,
                                           vp, vp, vp, sz, vp]
        L.crisp_get_status.argtypes = [vp, vp]
        L.crisp_status_string.argtypes = [i32]
        L.crisp_status_string.restype = ctypes.c_char_p
        L.crisp_selftest_timeout.argtypes = [vp, sz, ctypes.c_uint64, vp]
        L.crisp_fp8qk_buffer_size.argtypes = [i32, i32, i32, i32]
        L.crisp_fp8qk_buffer_size.restype = sz
        L.crisp_sparse_prefill_fp8qk.argtypes = [vp, vp, vp, i32, i32, i32, i32, I, vp, vp, vp, sz, vp, sz, vp]
        for name in ("crisp_select", "crisp_sparse_prefill", "crisp_prefill", "crisp_dense_prefill",
                     "crisp_get_status", "crisp_selftest_timeout", "crisp_prefill_varlen",
                     "crisp_sparse_prefill_fp8qk"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


@dataclasses.dataclass
class Params:
    """CRISP parameters (paper §3.2, §4, §5). block and anchors must be 128.

    route_rule / vs_rule / floor_rule select the FlexPrefill baseline rules (JSD router,
    per-direction gamma cut) and the median noise floor; 0 is CRISP's own rule."""
    block: int = 128
    anchors: int = 128
    tau_proxy: float = 0.5
    alpha: float = 1.0
    gamma: float = 0.95
    min_blocks: int = 0
    route_rule: int = 0
    tau_jsd: float = 0.1
    vs_rule: int = 0
    floor_rule: int = 0

    @staticmethod
    def flexprefill(**kw) -> "Params":
        """FlexPrefill's rules as the CRISP paper describes them (JSD router, gamma per direction)."""
        return Params(route_rule=1, vs_rule=1, **kw)

    def c(self) -> _Params:
        return _Params(self.block, self.anchors, self.tau_proxy, self.alpha, self.gamma, self.min_blocks,
                       self.route_rule, self.tau_jsd, self.vs_rule, self.floor_rule)


@dataclasses.dataclass
class Index:
    """Per-head selection result on the device (CSR over query blocks)."""
    route: torch.Tensor      # int32 [h_q]
    c_struct: torch.Tensor   # float32 [h_q]
    row_ptr: torch.Tensor    # int32 [h_q, N_b+1]
    cols: torch.Tensor       # int32 [h_q, N_b(N_b+1)/2]
    debug: torch.Tensor | None = None  # float32 [h_q, 2*N_b+5]

    @staticmethod
    def empty(h_q: int, n: int, device, debug: bool = False) -> "Index":
        nb = n_blocks(n)
        i32 = dict(device=device, dtype=torch.int32)
        return Index(torch.empty(h_q, **i32), torch.empty(h_q, device=device, dtype=torch.float32),
                     torch.empty(h_q, nb + 1, **i32), torch.empty(h_q, nb * (nb + 1) // 2, **i32),
                     torch.empty(h_q, 2 * nb + 5, device=device, dtype=torch.float32) if debug else None)

    def check(self, h_q: int, n: int, need_select_fields: bool = True):
        """Raise unless every array is a contiguous device tensor large enough for (h_q, n): the
        library writes and reads these sizes without seeing the tensors."""
        nb = n_blocks(n)
        want = [("row_ptr", self.row_ptr, torch.int32, (h_q, nb + 1)),
                ("cols", self.cols, torch.int32, (h_q, nb * (nb + 1) // 2))]
        if need_select_fields:
            want += [("route", self.route, torch.int32, (h_q,)), ("c_struct", self.c_struct, torch.float32, (h_q,))]
        elif self.route is not None:  # attention reads it to schedule heads
            want.append(("route", self.route, torch.int32, (h_q,)))
            if self.debug is not None:
                want.append(("debug", self.debug, torch.float32, (h_q, 2 * nb + 5)))
        for name, t, dt, shape in want:
            if t is None or not t.is_cuda or t.dtype != dt or not t.is_contiguous() or tuple(t.shape) != shape:
                raise ValueError(f"index.{name} must be a contiguous {dt} CUDA tensor of shape {shape}")

    def c(self) -> _Index:
        return _Index(self.route.data_ptr(), self.c_struct.data_ptr(), self.row_ptr.data_ptr(),
                      self.cols.data_ptr(), self.debug.data_ptr() if self.debug is not None else None)

    def lists(self, h: int) -> list:
        """Host copy of head h's per-query-block key-block lists (for inspection and tests)."""
        rp = self.row_ptr[h].cpu().tolist()
        cols = self.cols[h].cpu()
        return [cols[rp[i]:rp[i + 1]].tolist() for i in range(len(rp) - 1)]


def n_blocks(n: int) -> int:
    """Number of 128-token blocks; a length that is not a multiple of 128 ends in a partial block."""
    return -(-n // 128)


def _check_out(q, o, lse):
    if not o.is_cuda or o.dtype != torch.bfloat16 or not o.is_contiguous() or o.shape != q.shape:
        raise ValueError("o must be a contiguous bf16 CUDA tensor shaped like q")
    if lse is not None and (not lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous()
                            or tuple(lse.shape) != (q.shape[0], q.shape[1])):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor of shape [h_q, n]")


def _check(code: int, where: str):
    if code != OK:
        raise CrispError(code, where)


def _stream(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _qkv_shape(q, k, v=None):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t is None:
            continue
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous 3-D bf16 CUDA tensor")
    h_q, n, d = q.shape
    h_kv = k.shape[0]
    if k.shape[1:] != (n, d) or (v is not None and v.shape != k.shape):
        raise ValueError("q [h_q,n,d], k and v [h_kv,n,d] shapes disagree")
    return h_q, h_kv, n, d


def workspace_size(h_q: int, h_kv: int, n: int, d: int = 128, params: Params | None = None) -> int:
    """Workspace bytes for this shape; without params any length counts (attention alone runs at
    any n, selection needs a multiple of 128)."""
    if params is None:
        return int(lib().crisp_workspace_size(h_q, h_kv, n, d, None))
    p = params.c()
    return int(lib().crisp_workspace_size(h_q, h_kv, n, d, ctypes.byref(p)))


def workspace(h_q: int, h_kv: int, n: int, device, d: int = 128) -> torch.Tensor:
    """Device workspace for this shape, zero-filled (the status word must start at zero)."""
    nbytes = workspace_size(h_q, h_kv, n, d)
    if nbytes == 0:
        raise CrispError(-2, "workspace_size")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def select(q, k, params: Params | None = None, index: Index | None = None, ws: torch.Tensor | None = None,
           debug: bool = False) -> Index:
    """Route every q-head and build its key-block lists (crisp_select)."""
    h_q, h_kv, n, d = _qkv_shape(q, k)
    params = params or Params()
    ws = ws if ws is not None else workspace(h_q, h_kv, n, q.device, d)
    index = index or Index.empty(h_q, n, q.device, debug=debug)
    index.check(h_q, n)
    p, ix = params.c(), index.c()
    _check(lib().crisp_select(q.data_ptr(), k.data_ptr(), h_q, h_kv, n, d, ctypes.byref(p), ctypes.byref(ix),
                              ws.data_ptr(), ws.numel(), _stream(q)), "crisp_select")
    return index


def sparse_prefill(q, k, v, index: Index, o=None, lse=None, ws=None, want_lse: bool = True):
    """Block-sparse causal attention over `index` (crisp_sparse_prefill). Returns (o, lse)."""
    h_q, h_kv, n, d = _qkv_shape(q, k, v)
    ws = ws if ws is not None else workspace(h_q, h_kv, n, q.device, d)
    o = o if o is not None else torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(h_q, n, device=q.device, dtype=torch.float32)
    _check_out(q, o, lse)
    index.check(h_q, n, need_select_fields=False)
    ix = index.c()
    _check(lib().crisp_sparse_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), h_q, h_kv, n, d, ctypes.byref(ix),
                                      o.data_ptr(), lse.data_ptr() if lse is not None else None, ws.data_ptr(),
                                      ws.numel(), _stream(q)), "crisp_sparse_prefill")
    return o, lse


def prefill(q, k, v, params: Params | None = None, index: Index | None = None, o=None, lse=None, ws=None,
            want_lse: bool = True, keep_index: bool = True):
    """Selection + block-sparse attention (crisp_prefill). Returns (o, lse, index or None)."""
    h_q, h_kv, n, d = _qkv_shape(q, k, v)
    params = params or Params()
    ws = ws if ws is not None else workspace(h_q, h_kv, n, q.device, d)
    o = o if o is not None else torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(h_q, n, device=q.device, dtype=torch.float32)
    if index is None and keep_index:
        index = Index.empty(h_q, n, q.device)
    _check_out(q, o, lse)
    if index is not None:
        index.check(h_q, n)
    p = params.c()
    ix = ctypes.byref(index.c()) if index is not None else None
    _check(lib().crisp_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), h_q, h_kv, n, d, ctypes.byref(p),
                               o.data_ptr(), lse.data_ptr() if lse is not None else None, ix, ws.data_ptr(),
                               ws.numel(), _stream(q)), "crisp_prefill")
    return o, lse, index


def prefill_varlen(q, k, v, cu_seqlens, params: Params | None = None, o=None, lse=None, ws=None,
                   want_lse: bool = True):
    """crisp_prefill over independent sequences packed along the tokens (crisp_prefill_varlen).
    cu_seqlens: host sequence of n_seqs+1 offsets into the token axis. Returns (o, lse)."""
    h_q, h_kv, total, d = _qkv_shape(q, k, v)
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    params = params or Params()
    longest = max((b - a for a, b in zip(cu[:-1], cu[1:])), default=0)
    ws = ws if ws is not None else workspace(h_q, h_kv, max(longest, 1), q.device, d)
    o = o if o is not None else torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(h_q, total, device=q.device, dtype=torch.float32)
    _check_out(q, o, lse)
    arr = (ctypes.c_int32 * len(cu))(*cu)
    p = params.c()
    _check(lib().crisp_prefill_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), h_q, h_kv, total, arr, len(cu) - 1,
                                      d, ctypes.byref(p), o.data_ptr(), lse.data_ptr() if lse is not None else None,
                                      ws.data_ptr(), ws.numel(), _stream(q)), "crisp_prefill_varlen")
    return o, lse


def dense_prefill(q, k, v, o=None, lse=None, ws=None, want_lse: bool = True):
    """Dense causal attention with the same kernel (crisp_dense_prefill). Returns (o, lse)."""
    h_q, h_kv, n, d = _qkv_shape(q, k, v)
    ws = ws if ws is not None else workspace(h_q, h_kv, n, q.device, d)
    o = o if o is not None else torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(h_q, n, device=q.device, dtype=torch.float32)
    _check_out(q, o, lse)
    _check(lib().crisp_dense_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), h_q, h_kv, n, d, o.data_ptr(),
                                     lse.data_ptr() if lse is not None else None, ws.data_ptr(), ws.numel(),
                                     _stream(q)), "crisp_dense_prefill")
    return o, lse


def fp8qk_buffer(h_q: int, h_kv: int, n: int, device, d: int = 128) -> torch.Tensor:
    """Device buffer for the E4M3 codes and scales of crisp_sparse_prefill_fp8qk."""
    nbytes = int(lib().crisp_fp8qk_buffer_size(h_q, h_kv, n, d))
    if nbytes == 0:
        raise CrispError(-2, "crisp_fp8qk_buffer_size")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def fp8qk_views(buf: torch.Tensor, h_q: int, h_kv: int, n: int, d: int = 128):
    """(Q codes [h_q, n, d] uint8, K codes [h_kv, n, d] uint8, Q scales [h_q, N_b] float32,
    K scales [h_kv, N_b] float32) inside an fp8qk buffer, in the layout crisp.h documents."""
    nb = -(-n // 128)
    offs, off = [], 0
    for nbytes in (h_q * n * d, h_kv * n * d, h_q * nb * 4, h_kv * nb * 4):
        offs.append(off)
        off = -(-(off + nbytes) // 256) * 256
    q8 = buf[offs[0]:offs[0] + h_q * n * d].view(h_q, n, d)
    k8 = buf[offs[1]:offs[1] + h_kv * n * d].view(h_kv, n, d)
    qs = buf[offs[2]:offs[2] + h_q * nb * 4].view(torch.float32).view(h_q, nb)
    ks = buf[offs[3]:offs[3] + h_kv * nb * 4].view(torch.float32).view(h_kv, nb)
    return q8, k8, qs, ks


def sparse_prefill_fp8qk(q, k, v, index: Index, o=None, lse=None, ws=None, fp8_buf=None, want_lse: bool = True):
    """Block-sparse causal attention with E4M3 logits (crisp_sparse_prefill_fp8qk): Q and K are
    quantised per head and 128-row block into fp8_buf, then S = Q K^T runs on the codes.
    Returns (o, lse, fp8_buf)."""
    h_q, h_kv, n, d = _qkv_shape(q, k, v)
    ws = ws if ws is not None else workspace(h_q, h_kv, n, q.device, d)
    fp8_buf = fp8_buf if fp8_buf is not None else fp8qk_buffer(h_q, h_kv, n, q.device, d)
    o = o if o is not None else torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(h_q, n, device=q.device, dtype=torch.float32)
    _check_out(q, o, lse)
    index.check(h_q, n, need_select_fields=False)
    ix = index.c()
    _check(lib().crisp_sparse_prefill_fp8qk(q.data_ptr(), k.data_ptr(), v.data_ptr(), h_q, h_kv, n, d,
                                            ctypes.byref(ix), o.data_ptr(),
                                            lse.data_ptr() if lse is not None else None, ws.data_ptr(),
                                            ws.numel(), fp8_buf.data_ptr(), fp8_buf.numel(), _stream(q)),
           "crisp_sparse_prefill_fp8qk")
    return o, lse, fp8_buf


def get_status(ws: torch.Tensor) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    return int(lib().crisp_get_status(ws.data_ptr(), _stream(ws)))


def check_status(ws: torch.Tensor, where: str = "device"):
    _check(get_status(ws), where)


def selftest_timeout(ws: torch.Tensor, limit_ns: int) -> int:
    """Run the device timeout self-test (a wait nothing satisfies) and return the status it left."""
    _check(lib().crisp_selftest_timeout(ws.data_ptr(), ws.numel(), limit_ns, _stream(ws)), "crisp_selftest_timeout")
    return get_status(ws)


__all__ = ["Params", "Index", "CrispError", "lib", "workspace_size", "workspace", "select", "sparse_prefill",
           "prefill", "dense_prefill", "get_status", "check_status", "selftest_timeout", "fp8qk_buffer",
           "fp8qk_views", "sparse_prefill_fp8qk",
           "EXPORTED", "LIB_PATH"]
