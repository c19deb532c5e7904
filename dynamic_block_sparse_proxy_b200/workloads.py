"""Seeded synthetic prefill workloads (bf16 Q, K, V) for the CRISP sparse-prefill path.

This module only draws random tensors with a planted attention structure; it holds none of
the selection or attention arithmetic, so the CUDA path and the CPU oracle can both consume
its output without sharing any of the method.

The structure mirrors what the CRISP paper describes for Vertical-Slash heads ("CRISP:
Cliff-awaRe Input-adaptive Sparse Prefilling with Structural-Mass-Motivated Routing", §3.2 and
§4): an attention sink on the first keys, task-relevant vertical key blocks, diagonal (slash)
dependencies at fixed offsets, and a recency bias; Pooled-Estimation heads are diffuse.

Recipe (per workload, seed fixed):
  * planted directions have squared norm sqrt(d), so adding w_q*u to a query and w_k*u to a key
    raises that query-key logit (q.k/sqrt(d)) by exactly w_q*w_k;
  * base Q and K are N(0,1) rotated by RoPE (rotate-half convention, base theta); planted
    terms are added after RoPE, except recency, which is a shared pre-RoPE vector;
  * sink: the first 16 keys of every kv-head get +sink_w*u; concentrated q-heads get +3u;
  * vertical: n_vertical random key blocks in [1, N_b-2] per kv-head get +3u on all 128 keys;
  * slash: n_slash offsets per kv-head in [2B, n/2), multiples of 4 but not of B; one code
    sequence c_i (|c_i|^2 = sqrt(d)) per kv-head; offset a serves query positions i with
    i % n_slash == a, and c_i is added x slash_w to q_i of the concentrated heads and to
    k_{i-off_a}, so each query and key carries at most one code (more codes per vector would
    raise every logit's noise far above the planted gaps);
  * recency: a shared vector v (|v|^2 = sqrt(d)) x2 on concentrated q and on all k, pre-RoPE;
  * within each GQA group the first `conc_per_group` q-heads are concentrated, the rest are
    diffuse: Q = RoPE(N(0,1))/2 with nothing planted;
  * V is N(0,1).
"""
from __future__ import annotations

import dataclasses

import torch

BLOCK = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n: int
    h_q: int
    h_kv: int
    d: int
    theta: float
    conc_per_group: int
    sink_w: float
    n_vertical: int
    n_slash: int
    recency: bool
    seed: int
    slash_w: float = 4.0
    sink_tokens: int = 16

    def scaled(self, n: int) -> "Workload":
        """Same generator at another sequence length (vertical count capped by N_b-2)."""
        nb = n // BLOCK
        return dataclasses.replace(self, name=f"{self.name}@n{n}", n=n,
                                   n_vertical=min(self.n_vertical, max(nb - 2, 0)),
                                   n_slash=self.n_slash if n >= 8 * BLOCK else 0)


# The five workloads: a tiny single-head case, Llama-3.1-8B attention geometry (32 q / 8 kv
# heads, d=128, RoPE theta 5e5) at 32k, 128k and 512k tokens, and Qwen2.5-7B geometry
# (28 q / 4 kv heads, RoPE theta 1e6) at 128k.
WORKLOADS = {
    "tiny_1h_4k": Workload("tiny_1h_4k", 4096, 1, 1, 128, 1e4, 1, 6.0, 4, 0, False, 0),
    "llama8b_32k": Workload("llama8b_32k", 32768, 32, 8, 128, 5e5, 2, 6.0, 8, 0, True, 1),
    "llama8b_128k": Workload("llama8b_128k", 131072, 32, 8, 128, 5e5, 2, 6.0, 16, 4, True, 2),
    "qwen7b_128k": Workload("qwen7b_128k", 131072, 28, 4, 128, 1e6, 5, 8.0, 16, 4, True, 3),
    "llama8b_512k": Workload("llama8b_512k", 524288, 32, 8, 128, 5e5, 2, 6.0, 32, 4, True, 4),
}

DEFAULT_PARAMS = dict(block=128, anchors=128, tau_proxy=0.5, alpha=1.0, gamma=0.95, min_blocks=0)


def _planted_direction(g: torch.Generator, d: int, device) -> torch.Tensor:
    v = torch.randn(d, generator=g, device=device, dtype=torch.float32)
    return v * (d ** 0.25) / v.norm()


def _rope(x: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotate-half RoPE over the last dim of x[..., n, d] (positions 0..n-1)."""
    n, d = x.shape[-2], x.shape[-1]
    half = d // 2
    inv = theta ** (-torch.arange(0, half, device=x.device, dtype=torch.float64) * 2.0 / d)
    ang = torch.arange(n, device=x.device, dtype=torch.float64)[:, None] * inv[None, :]
    cos = ang.cos().to(torch.float32)
    sin = ang.sin().to(torch.float32)
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def concentrated_heads(w: Workload) -> list[bool]:
    g = w.h_q // w.h_kv
    return [(h % g) < w.conc_per_group for h in range(w.h_q)]


def generate(w: Workload, device="cpu"):
    """Return (q, k, v, meta): bf16 q[h_q,n,d], k/v[h_kv,n,d] on `device`, plus the planted truth.

    The random stream is a torch.Generator on `device` seeded with w.seed, so CPU and GPU
    draws differ; parity tests always hand the very same tensors to both sides.
    """
    assert w.n % BLOCK == 0 and w.h_q % w.h_kv == 0
    n, d, hq, hkv = w.n, w.d, w.h_q, w.h_kv
    nb = n // BLOCK
    G = hq // hkv
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    f32 = dict(device=device, dtype=torch.float32)

    u = _planted_direction(g, d, device)
    rec = _planted_direction(g, d, device) if w.recency else None
    conc = concentrated_heads(w)

    # keys
    k = torch.randn(hkv, n, d, generator=g, **f32)
    if rec is not None:
        k += 2.0 * rec
    k = _rope(k, w.theta)
    k[:, : w.sink_tokens] += w.sink_w * u
    verticals, slashes = [], []
    for kv in range(hkv):
        if w.n_vertical > 0 and nb > 2:
            perm = torch.randperm(nb - 2, generator=g, device=device)[: w.n_vertical] + 1
            vb = sorted(int(x) for x in perm.tolist())
        else:
            vb = []
        verticals.append(vb)
        for b in vb:
            k[kv, b * BLOCK:(b + 1) * BLOCK] += 3.0 * u
        offs = []
        while len(offs) < w.n_slash:
            lo, hi = 2 * BLOCK // 4, max(n // 8, 2 * BLOCK // 4 + 2)
            off = 4 * int(torch.randint(lo, hi, (1,), generator=g, device=device).item())
            if off % BLOCK != 0 and off not in offs:
                offs.append(off)
        slashes.append(offs)

    # queries
    q = torch.empty(hq, n, d, **f32)
    for h in range(hq):
        z = torch.randn(n, d, generator=g, **f32)
        if conc[h]:
            if rec is not None:
                z += 2.0 * rec
            q[h] = _rope(z, w.theta) + 3.0 * u
        else:
            q[h] = _rope(z, w.theta) * 0.5

    # slash plants: per kv-group one code sequence c_i (|c_i|^2 = sqrt(d)); offset a serves the
    # query positions i with i % 4 == a (offsets are multiples of 4), so each query and each key
    # carries at most one code and q_i . k_{i-off_a} rises by slash_w^2.
    for kv in range(hkv):
        offs = slashes[kv]
        if not offs:
            continue
        c = torch.randn(n, d, generator=g, **f32)
        c *= (d ** 0.25) / c.norm(dim=-1, keepdim=True)
        pos = torch.arange(n, device=device)
        off_of = torch.tensor(offs, device=device)[pos % len(offs)]
        src_q = pos >= off_of                                    # q_i has a partner key
        kpos = pos + off_of                                      # key j pairs with query j+off
        has = kpos < n
        k[kv, has] += w.slash_w * c[kpos[has]]
        for h in range(kv * G, (kv + 1) * G):
            if conc[h]:
                q[h, src_q] += w.slash_w * c[src_q]
    v = torch.randn(hkv, n, d, generator=g, **f32)
    meta = dict(concentrated=conc, vertical_blocks=verticals, slash_offsets=slashes)
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), meta)


def random_qkv(h_q: int, h_kv: int, n: int, d: int = 128, seed: int = 0, device="cpu",
               q_scale: float = 1.0):
    """Plain N(0,1) bf16 tensors (no planted structure) for edge-case tests."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    f32 = dict(device=device, dtype=torch.float32)
    q = torch.randn(h_q, n, d, generator=g, **f32) * q_scale
    k = torch.randn(h_kv, n, d, generator=g, **f32)
    v = torch.randn(h_kv, n, d, generator=g, **f32)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def spiked_qkv(h_q: int, h_kv: int, n: int, spike_blocks, gaps, d: int = 128, seed: int = 0, device="cpu",
               q_rows=None, keys=(0, BLOCK)):
    """N(0,1) bf16 tensors with one planted direction u (|u|^2 = sqrt(d)): every key of the
    `spike_blocks` gets +w_k u and the queries of head h get +(gaps[h] / w_k) u, so that head's
    logits against the spiked keys rise by gaps[h] nats (q . k / sqrt(d) grows by w_q w_k).
    `q_rows` limits the query term to a row range (e.g. the last 128 rows) and `keys` the spike to
    a range of key offsets inside each spiked block. Edge-case inputs for the softmax reference
    handling: a spike far above the first key block a walk meets."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn(h_q, n, d, generator=g)
    k = torch.randn(h_kv, n, d, generator=g)
    v = torch.randn(h_kv, n, d, generator=g)
    u = _planted_direction(g, d, "cpu")
    w_k = 8.0
    for kb in spike_blocks:
        k[:, min(n, kb * BLOCK + keys[0]):min(n, kb * BLOCK + keys[1])] += w_k * u
    lo, hi = q_rows if q_rows is not None else (0, n)
    for h in range(h_q):
        q[h, lo:hi] += (float(gaps[h]) / w_k) * u
    return tuple(t.to(torch.bfloat16).to(device) for t in (q, k, v))


def proxy_flops(w: Workload) -> float:
    """Tensor FLOPs of the proxy logits (last query block against all keys) for one layer."""
    return 2.0 * w.h_q * BLOCK * w.n * w.d


def block_pair_flops(d: int = 128) -> float:
    """FLOPs of one (query block, key block) attention tile: QK^T plus PV, full tile."""
    return 4.0 * BLOCK * BLOCK * d


__all__ = ["Workload", "WORKLOADS", "DEFAULT_PARAMS", "generate", "random_qkv", "spiked_qkv",
           "concentrated_heads", "proxy_flops", "block_pair_flops", "BLOCK"]
