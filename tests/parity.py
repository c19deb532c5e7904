"""Comparison helpers between the CUDA path (through the C ABI) and the fp64 oracle.

Rules (the tolerances of the parity contract):
  * routes and index sets must match exactly, except where a score lies within 1e-5 relative of
    its threshold (the oracle reports those entries as ties; they may go either way and are
    logged);
  * attention output on identical index sets: max abs error <= 2e-2 and mean abs error <= 2e-3
    against the fp64 oracle; LSE within 5e-3 absolute.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import crisp_oracle as O

ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
LSE_ABS = 5e-3
P_REL = 2e-4     # relative agreement of the block masses p_v, p_s (fp32 path vs fp64)
# Accuracy of the JSD value itself (not a tie band: the route decision uses the 1e-5 band of the
# oracle). a_bar and a_hat carry fp32 rounding of relative size ~1e-6; the JSD of two nearby
# distributions is a sum of squared differences, so its relative error grows by about p/|p-q|
# (~20-50x on diffuse heads, where JSD ~ 2e-3).
JSD_REL = 2e-4

# Every compare_selection call appends one record here; the session summary prints them and,
# with CRISP_TIE_LOG set, writes them to that JSON file.
TIE_LOG: list[dict] = []


def f32(x: float) -> float:
    """The C ABI takes fp32 parameters; the oracle receives the same rounded values."""
    return float(np.float32(x))


def oracle_params(params) -> dict:
    return dict(block=params.block, anchors=params.anchors, tau_proxy=f32(params.tau_proxy),
                alpha=f32(params.alpha), gamma=f32(params.gamma), min_blocks=params.min_blocks,
                route_rule="jsd" if params.route_rule else "cstruct", tau_jsd=f32(params.tau_jsd),
                vs_rule="gamma" if params.vs_rule else "floor", floor="median" if params.floor_rule else "mean")


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def oracle_select_heads(q, k, params, heads):
    """Oracle selection for the given q-heads; q, k may live on any device."""
    G = q.shape[0] // k.shape[0]
    out = {}
    kcache = {}
    for h in heads:
        kv = h // G
        if kv not in kcache:
            kcache = {kv: f64(k[kv])}
        out[h] = O.select_head(f64(q[h]), kcache[kv], **oracle_params(params))
    return out


def compare_selection(index, sels: dict, nb: int, log: list | None = None, name: str | None = None) -> dict:
    """Assert GPU routes/lists agree with the oracle outside the tie band; return tie counts.

    The ties found (routing statistics inside the band, Vertical-Slash blocks inside the band,
    Pooled-Estimation entries where the GPU and the oracle differ inside the band) are logged
    per (head, block) in TIE_LOG under `name`."""
    route = index.route.cpu().numpy()
    cst = index.c_struct.cpu().numpy()
    dbg = index.debug.cpu().numpy() if index.debug is not None else None
    stats = dict(route_ties=0, vs_tie_blocks=0, pe_tie_entries=0, pe_differing=0, heads=0)
    rec = dict(name=name or "unnamed", nb=nb, heads=sorted(int(h) for h in sels), route_ties=[],
               vs_ties=[], pe_tie_entries={}, pe_differing=[])
    TIE_LOG.append(rec)
    for h, s in sels.items():
        stats["heads"] += 1
        assert abs(float(cst[h]) - s["c_struct"]) <= 1e-5 * max(1.0, s["c_struct"]) + 1e-6, (h, cst[h], s["c_struct"])
        if dbg is not None and "jsd" in s:
            assert abs(float(dbg[h, 2 * nb + 4]) - s["jsd"]) <= JSD_REL * max(s["jsd"], 1e-3), (h, dbg[h, 2 * nb + 4], s["jsd"])
        if s["route_tie"]:
            stats["route_ties"] += 1
            rec["route_ties"].append(int(h))
            if log is not None:
                log.append(f"head {h}: routing statistic within the tie band of its threshold")
            continue
        assert int(route[h]) == s["route"], (h, route[h], s["route"], s["c_struct"])
        if dbg is not None:
            for name, off in (("p_v", 0), ("p_s", nb)):
                g = dbg[h, off:off + nb].astype(np.float64)
                o = s[name]
                err = np.abs(g - o)
                bad = err > P_REL * np.maximum(o, 1e-6 * o.max()) + 1e-12
                assert not bad.any(), (h, name, np.nonzero(bad)[0][:5], g[bad][:5], o[bad][:5])
        gl = index_lists(index, h)
        ol = s["lists"]
        assert len(gl) == nb
        for qb in range(nb):
            g = gl[qb]
            assert g == sorted(set(g)) and all(0 <= x <= qb for x in g), (h, qb, g)
        if s["route"] == 1 and nb >= 3:
            tv, ts = set(s.get("vs_ties_v", [])), set(s.get("vs_ties_s", []))
            stats["vs_tie_blocks"] += len(tv) + len(ts)
            rec["vs_ties"] += [[int(h), "v", int(j)] for j in sorted(tv)] + [[int(h), "s", int(j)] for j in sorted(ts)]
            lo = O.merge_vertical_slash(sorted(set(s["keep_v"]) - tv), sorted(set(s["keep_s"]) - ts), nb)
            hi = O.merge_vertical_slash(sorted(set(s["keep_v"]) | tv), sorted(set(s["keep_s"]) | ts), nb)
            for qb in range(nb):
                g = set(gl[qb])
                assert set(lo[qb].tolist()) <= g <= set(hi[qb].tolist()), (h, qb, sorted(g ^ set(ol[qb].tolist())))
            if not tv and not ts:
                for qb in range(nb):
                    assert gl[qb] == ol[qb].tolist(), (h, qb)
        elif s["route"] == 0:
            ties = s.get("pe_ties")
            stats["pe_tie_entries"] += int(ties.sum()) if ties is not None else 0
            if ties is not None and ties.any():
                rec["pe_tie_entries"][str(int(h))] = int(ties.sum())
            for qb in range(nb):
                diff = set(gl[qb]) ^ set(ol[qb].tolist())
                for kb in diff:
                    assert ties is not None and ties[qb, kb], (h, qb, kb, "outside the tie band")
                    rec["pe_differing"].append([int(h), int(qb), int(kb), "gpu" if kb in gl[qb] else "oracle"])
                stats["pe_differing"] += len(diff)
        else:
            for qb in range(nb):
                assert gl[qb] == ol[qb].tolist()
    rec["counts"] = dict(stats)
    if log is not None and (stats["vs_tie_blocks"] or stats["pe_differing"]):
        log.append(f"ties: {stats}")
    return stats


def tie_summary_lines(max_entries: int = 6) -> list[str]:
    """One line per logged comparison: counts, then the first (head, block) entries."""
    out = []
    for r in TIE_LOG:
        ent = [f"h{h}:{d}{j}" for h, d, j in r["vs_ties"][:max_entries]]
        ent += [f"h{h}:({qb},{kb})->{side}" for h, qb, kb, side in r["pe_differing"][:max_entries]]
        ent += [f"h{h}:route" for h in r["route_ties"]]
        out.append(f"{r['name']}: heads={len(r['heads'])} route_ties={len(r['route_ties'])} "
                   f"vs_tie_blocks={len(r['vs_ties'])} pe_tie_entries={sum(r['pe_tie_entries'].values())} "
                   f"pe_differing={len(r['pe_differing'])}" + (f" [{' '.join(ent)}]" if ent else ""))
    return out


def index_lists(index, h: int):
    return index.lists(h)


def compare_attention_blocks(q, k, v, o, lse, lists: dict, blocks, G: int, B: int = 128):
    """Oracle attention for (h, qb) pairs on the GPU's own lists (lists[h][qb]).
    Returns (max_abs, mean_abs, max_lse_abs)."""
    errs, lerrs = [], []
    cache = {}
    for h, qb in blocks:
        kv = h // G
        if kv not in cache:
            cache = {kv: (f64(k[kv]), f64(v[kv]))}
        kk, vv = cache[kv]
        ro, rl = O.attention_block(f64(q[h, qb * B:(qb + 1) * B]), kk, vv, lists[h][qb], qb, B)
        errs.append(np.abs(f64(o[h, qb * B:(qb + 1) * B]) - ro))
        if lse is not None:
            gl = lse[h, qb * B:(qb + 1) * B].cpu().numpy().astype(np.float64)
            lerrs.append(np.max(np.abs(gl - rl)))
    e = np.concatenate([x.ravel() for x in errs])
    return float(e.max()), float(e.mean()), float(max(lerrs) if lerrs else 0.0)


def assert_attention_ok(stats):
    mx, mean, lmx = stats
    assert mx <= ATTN_MAX_ABS, stats
    assert mean <= ATTN_MEAN_ABS, stats
    assert lmx <= LSE_ABS, stats
