"""Benchmark: CRISP sparse prefill (selection + block-sparse attention) for one attention layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama8b_128k] [--impl crisp|reference]

One step = one full pass of the hot path over one layer: index selection for every q-head
(crisp_select) followed by block-sparse causal attention over the selected blocks
(crisp_sparse_prefill), on seeded synthetic bf16 inputs already resident in HBM. The metric is
prefill tokens per second per layer, n / step time, summed over ranks (each rank runs its own
independent layer; no collective on the data path, weak scaling).

Rank 0 prints one JSON line. With --impl reference the fp64 CPU oracle runs instead, on a
bounded sample of the same workload, extrapolated to the same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dynamic_block_sparse_proxy_b200 as crisp  # noqa: E402  (the library loads on first use)
from dynamic_block_sparse_proxy_b200 import workloads as W  # noqa: E402

METRIC = "prefill tokens/s per layer (select+sparse attn) at 128k; % bf16 peak, % HBM BW"
DEFAULT_WORKLOAD = "llama8b_128k"
# kernels per step: proxy pass, 2 for routing (row statistics, block masses + route), 5 for the PE
# path (Q_bar, scores, row softmax, two histogram levels), 3 for the merge, attention
KERNELS_PER_STEP = 12
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time: every rank takes part, in the same order, so ranks never diverge."""
    if world <= 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, n: int, steps: int, total_s: float) -> float:
    """Whole-job throughput: every rank processes `steps` layers of n tokens in the slowest rank's time."""
    return world * n * steps / total_s


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        # raw samples go to the temp directory (or CRISP_CLOCKS_DIR); the JSON line carries the summary
        self.path = os.path.join(os.environ.get("CRISP_CLOCKS_DIR", tempfile.gettempdir()),
                                 f"crisp_clocks_rank{gpu_index}_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        with open(self.path) as f:
            return self.summarise(f)

    @staticmethod
    def summarise(lines) -> dict:
        """Median SM clock, the maximum clock and the throttle reasons seen active, from
        `nvidia-smi --query-gpu=<QUERY> --format=csv,noheader,nounits` lines."""
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- byte / flop models
def select_bytes(w, n_pe_heads: int, total_pairs: int) -> float:
    """Algorithmic HBM bytes of selection: K once, the last query block of every head, the
    whole Q of the Pooled-Estimation heads, and the written index (row_ptr + cols)."""
    nb = -(-w.n // 128)
    k_bytes = w.h_kv * w.n * w.d * 2
    qlast = w.h_q * 128 * w.d * 2
    qpe = n_pe_heads * w.n * w.d * 2
    idx = 4 * (w.h_q * (nb + 1) + total_pairs)
    return float(k_bytes + qlast + qpe + idx)


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attention launch, and the sum
# over the selection kernels of one step, on the 128k workload, from a three-metric ncu capture
# of this command's own timed step. Each figure belongs to the kernel sources it was taken on
# (SHA-256 of the source, or of the selection sources in order); for any other source or workload
# the bench reports null.
ATTN_TRAFFIC = {"workload": "llama8b_128k",
                "source_sha256": "ba1487bcdca357eb7fce544ca872009ae1c3018bfa02d2e0dae827cb830a4843",
                "bytes": 2.72104e9 + 1.05506e9}
SELECT_SOURCES = ["proxy_pass.cu", "route_threshold.cu", "pe_cut.cu", "merge.cu", "sm100.cuh", "crisp_internal.h"]
SELECT_TRAFFIC = {"workload": "llama8b_128k",
                  "source_sha256": "134f564212b438969b5fb4cbf1ab7a41180d81fd7597859c5e87466119bcc3a3",
                  "bytes": 1282.67e6 + 87.71e6}


def _sources_sha(names):
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "dynamic_block_sparse_proxy_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attn_traffic(w):
    if w.name != ATTN_TRAFFIC["workload"] or _sources_sha(["sparse_attn.cu"]) != ATTN_TRAFFIC["source_sha256"]:
        return None
    return ATTN_TRAFFIC["bytes"]


def select_traffic(w):
    if w.name != SELECT_TRAFFIC["workload"] or _sources_sha(SELECT_SOURCES) != SELECT_TRAFFIC["source_sha256"]:
        return None
    return SELECT_TRAFFIC["bytes"]


# Index-selection rules: CRISP's own (default), the FlexPrefill baseline the CRISP paper compares
# against, and CRISP's variants (median floor, the speed-focused alpha values).
RULES = {
    "crisp": crisp.Params(),
    "flexprefill": crisp.Params.flexprefill(),
    "crisp_median": crisp.Params(floor_rule=1),
    "crisp_alpha1.25": crisp.Params(alpha=1.25),
    "crisp_alpha1.5": crisp.Params(alpha=1.5),
}


def rule_config(p) -> dict:
    out = {"tau_proxy": p.tau_proxy, "alpha": p.alpha, "gamma": p.gamma, "min_blocks": p.min_blocks}
    if p.route_rule:
        out.update(route="jsd", tau_jsd=p.tau_jsd)
    if p.vs_rule:
        out["vs"] = "gamma per direction"
    if p.floor_rule:
        out["floor"] = "median"
    return out


def bench_config(w, args, world: int) -> dict:
    """The workload line both arms (CUDA and oracle) report."""
    return {"workload": w.name, "n": w.n, "h_q": w.h_q, "h_kv": w.h_kv, "d": w.d, "block": 128,
            "rules": args.rules, **rule_config(RULES[args.rules]),
            "parallelism": f"independent layer per rank x{world}",
            "l2": "flushed before every step (256 MB write); inputs also exceed L2"}


def oracle_kwargs(p) -> dict:
    return dict(tau_proxy=p.tau_proxy, alpha=p.alpha, gamma=p.gamma, min_blocks=p.min_blocks,
                route_rule="jsd" if p.route_rule else "cstruct", tau_jsd=p.tau_jsd,
                vs_rule="gamma" if p.vs_rule else "floor", floor="median" if p.floor_rule else "mean")


def attn_flops(total_pairs: int, d: int = 128) -> float:
    return W.block_pair_flops(d) * total_pairs


# ---------------------------------------------------------------------------- GPU arm
def run_crisp(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = W.WORKLOADS[args.workload]
    if args.n:
        w = w.scaled(args.n)
    q, k, v, meta = W.generate(w, device=dev)
    params = RULES[args.rules]
    ws = crisp.workspace(w.h_q, w.h_kv, w.n, dev)
    idx = crisp.Index.empty(w.h_q, w.n, dev)
    o = torch.empty_like(q)
    lse = torch.empty(w.h_q, w.n, device=dev, dtype=torch.float32)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2
    stream = torch.cuda.current_stream(dev)

    def step():
        crisp.select(q, k, params, index=idx, ws=ws)
        crisp.sparse_prefill(q, k, v, idx, o=o, lse=lse, ws=ws)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    crisp.check_status(ws, "warmup")
    nb = -(-w.n // 128)
    total_pairs = int(idx.row_ptr[:, nb].sum().item())
    n_pe = int((idx.route == 0).sum().item())

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        crisp.select(q, k, params, index=idx, ws=ws)
        ev[i][1].record(stream)
        crisp.sparse_prefill(q, k, v, idx, o=o, lse=lse, ws=ws)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    crisp.check_status(ws, "timed")
    t_sel = np.array([ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]) / 1e3
    t_att = np.array([ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]) / 1e3
    t_step = t_sel + t_att
    total_s = float(t_step.sum())
    total_s = max_over_ranks(total_s, world, dev)

    # dense causal attention with the same kernel on the same inputs (after the timed region)
    dense = None
    if args.dense:
        od = torch.empty_like(q)
        lsed = torch.empty_like(lse)
        crisp.dense_prefill(q, k, v, o=od, lse=lsed, ws=ws)
        d_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.dense_steps)]
        sampler_d = ClockSampler(local)
        torch.cuda.synchronize()
        sampler_d.start()
        time.sleep(0.3)
        for e0, e1 in d_ev:
            flush.fill_(7)
            e0.record(stream)
            crisp.dense_prefill(q, k, v, o=od, lse=lsed, ws=ws)
            e1.record(stream)
        torch.cuda.synchronize()
        clocks_d = sampler_d.stop()
        crisp.check_status(ws, "dense")
        dense_s = float(np.mean([e0.elapsed_time(e1) for e0, e1 in d_ev])) / 1e3
        dense = {"dense_attn_ms": dense_s * 1e3, "dense_pairs": w.h_q * nb * (nb + 1) // 2,
                 "dense_tflops": attn_flops(w.h_q * nb * (nb + 1) // 2, w.d) / dense_s / 1e12,
                 "steps": args.dense_steps, "clocks": clocks_d}
        del od, lsed
        dense["torch_sdpa"] = torch_sdpa_reference(q, k, v, w, nb, args.dense_steps, flush, stream)

    # the FP8 variant of the logits on the same inputs and index (after the timed region; the
    # headline stays bf16): its attention time, including the quantisation of Q and K, and how far
    # its output lies from the bf16 kernel's
    fp8 = None
    if args.fp8:
        buf = crisp.fp8qk_buffer(w.h_q, w.h_kv, w.n, dev)
        o8, l8 = torch.empty_like(q), torch.empty_like(lse)
        crisp.sparse_prefill_fp8qk(q, k, v, idx, o=o8, lse=l8, ws=ws, fp8_buf=buf)
        f_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.dense_steps)]
        torch.cuda.synchronize()
        for e0, e1 in f_ev:
            flush.fill_(3)
            e0.record(stream)
            crisp.sparse_prefill_fp8qk(q, k, v, idx, o=o8, lse=l8, ws=ws, fp8_buf=buf)
            e1.record(stream)
        torch.cuda.synchronize()
        crisp.check_status(ws, "fp8qk")
        f_s = float(np.mean([e0.elapsed_time(e1) for e0, e1 in f_ev])) / 1e3
        dev_abs = (o8.float() - o.float()).abs()
        fp8 = {"attn_ms": f_s * 1e3, "tflops": attn_flops(total_pairs, w.d) / f_s / 1e12,
               "speedup_vs_bf16": float(t_att.mean()) / f_s, "max_abs_vs_bf16": float(dev_abs.max()),
               "mean_abs_vs_bf16": float(dev_abs.mean()), "steps": args.dense_steps,
               "what": "S = Q K^T on E4M3 codes with per-(head, 128-row block) scales; P, V and O as in "
                       "the bf16 kernel; the time includes quantising Q and K"}
        del buf, o8, l8, dev_abs

    e2e = None
    if args.e2e:
        e2e = e2e_pipelined(w, q, k, v, params, idx, ws, max(8, min(args.steps, 16)), dev, stream)
        e2e_s = max_over_ranks(e2e.pop("seconds_per_step"), world, dev)
        e2e.update(value=job_tokens_per_s(world, w.n, 1, e2e_s), ms_per_step=e2e_s * 1e3)

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    pk, src = peaks()
    mean_att = float(t_att.mean())
    mean_sel = float(t_sel.mean())
    fl = attn_flops(total_pairs, w.d)
    achieved_tf = fl / mean_att / 1e12
    sustained = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    sb = select_bytes(w, n_pe, total_pairs)
    sel_gbs = sb / mean_sel / 1e9
    dense_pairs = w.h_q * nb * (nb + 1) // 2
    out = {
        "metric": METRIC,
        "value": job_tokens_per_s(world, w.n, args.steps, total_s),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_s / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded planted-structure generator)",
        "config": bench_config(w, args, world),
        # The attention launch lasts tens of milliseconds and the timed region well under a
        # second, at clocks near the maximum: the burst figure is the denominator, and the
        # sustained one (a seconds-long GEMM loop at a lower clock under the power cap) is beside it.
        "roofline": {"bound": "tensor", "kernel": "sparse_attn", "achieved": achieved_tf,
                     "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved_tf / pk["bf16_tflops"],
                     "peak_kind": f"bf16 burst ({src})",
                     "frac_of_sustained": achieved_tf / sustained, "traffic": attn_traffic(w),
                     "flops_per_launch": fl, "selected_pairs": total_pairs,
                     "density": total_pairs / dense_pairs},
        "select_roofline": {"bound": "hbm", "achieved": sel_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                            "frac": sel_gbs / pk["hbm_gbs"], "bytes_per_launch": sb,
                            "traffic": select_traffic(w), "ms": mean_sel * 1e3, "pe_heads": n_pe},
        "attn_ms": mean_att * 1e3,
        "select_ms": mean_sel * 1e3,
        "e2e": e2e,
        "fp8_qk_variant": fp8,
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": clocks,
    }
    if dense is not None:
        dense["sparse_attn_ms"] = mean_att * 1e3
        dense["sparse_step_ms"] = (mean_att + mean_sel) * 1e3
        dense["attn_speedup"] = dense["dense_attn_ms"] / (mean_att * 1e3)
        dense["step_speedup"] = dense["dense_attn_ms"] / ((mean_att + mean_sel) * 1e3)
        out["sparse_vs_dense"] = dense
    if args.cpu_baseline:
        out["cpu_baseline"] = oracle_baseline(w, q, k, v, idx, args.cpu_seconds, params=params)
    print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------------------- end to end
def torch_sdpa_reference(q, k, v, w, nb, steps: int, flush, stream) -> dict:
    """An outside reference for the dense number: PyTorch's own causal scaled-dot-product attention
    (whichever backend it picks) on the same inputs, timed like the dense leg. FLOPs are counted as
    for the dense leg (full diagonal tiles), so the two TFLOP/s figures compare directly."""
    import torch.nn.functional as F
    try:
        qs, ks, vs = q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0)
        with torch.cuda.stream(stream):
            F.scaled_dot_product_attention(qs, ks, vs, is_causal=True, enable_gqa=True)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            torch.cuda.synchronize()
            for e0, e1 in ev:
                flush.fill_(5)
                e0.record(stream)
                F.scaled_dot_product_attention(qs, ks, vs, is_causal=True, enable_gqa=True)
                e1.record(stream)
            torch.cuda.synchronize()
        sec = float(np.mean([e0.elapsed_time(e1) for e0, e1 in ev])) / 1e3
        return {"ms": sec * 1e3, "tflops": attn_flops(w.h_q * nb * (nb + 1) // 2, w.d) / sec / 1e12,
                "call": "torch.nn.functional.scaled_dot_product_attention(is_causal=True, enable_gqa=True)"}
    except Exception as e:  # a missing backend is reported, not fatal
        return {"unavailable": f"{type(e).__name__}: {e}"[:200]}


def e2e_pipelined(w, q, k, v, params, idx, ws, steps: int, dev, stream) -> dict:
    """The metric end to end through the public API with host buffers: every step copies its Q, K
    and V from pinned host memory, selects (crisp.select), attends one kv-group at a time
    (crisp.sparse_prefill on the group's heads and index rows) and copies each group's output back
    to pinned host memory as soon as that group is done. Two sets of device inputs and outputs let
    step i+1's uploads run during step i's attention, as a prefill pipeline over layers would. One
    warm-up step runs to completion first; the timed region then covers `steps` steps from the
    first step's upload (nothing else running) to the last step's download, so every timed step's
    copies lie inside it and the pipeline fills once."""
    G = w.h_q // w.h_kv
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
    qd = [torch.empty_like(q) for _ in range(2)]
    kd = [torch.empty_like(k) for _ in range(2)]
    vd = [torch.empty_like(v) for _ in range(2)]
    od = [torch.empty_like(q) for _ in range(2)]
    lsed = [torch.empty(w.h_q, w.n, device=dev, dtype=torch.float32) for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_free = [None, None]   # attention of the last step that read input buffer b
    out_free = [None, None]  # download of the last step that wrote output buffer b
    gidx = [crisp.Index(idx.route[g * G:(g + 1) * G], idx.c_struct[g * G:(g + 1) * G],
                        idx.row_ptr[g * G:(g + 1) * G], idx.cols[g * G:(g + 1) * G]) for g in range(w.h_kv)]
    total = steps + 1
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    for i in range(total):
        b = i % 2
        if i == 1:
            torch.cuda.synchronize()  # the warm-up step is done
            t0.record(up)  # timed region starts with step 1's first upload
        with torch.cuda.stream(up):
            if in_free[b] is not None:
                up.wait_event(in_free[b])
            qd[b].copy_(qh, non_blocking=True)
            kd[b].copy_(kh, non_blocking=True)
            vd[b].copy_(vh, non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(up)
        stream.wait_event(ready)
        if out_free[b] is not None:
            stream.wait_event(out_free[b])
        crisp.select(qd[b], kd[b], params, index=idx, ws=ws)
        for g in range(w.h_kv):
            hs = slice(g * G, (g + 1) * G)
            crisp.sparse_prefill(qd[b][hs], kd[b][g:g + 1], vd[b][g:g + 1], gidx[g], o=od[b][hs], lse=lsed[b][hs],
                                 ws=ws)
            done = torch.cuda.Event()
            done.record(stream)
            down.wait_event(done)
            with torch.cuda.stream(down):
                oh[b][hs].copy_(od[b][hs], non_blocking=True)
        in_free[b] = torch.cuda.Event()
        in_free[b].record(stream)
        out_free[b] = torch.cuda.Event()
        out_free[b].record(down)
    down.wait_stream(stream)
    t1.record(down)
    torch.cuda.synchronize()
    crisp.check_status(ws, "e2e")
    h2d = (q.numel() + k.numel() + v.numel()) * 2
    d2h = q.numel() * 2
    return {"unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "seconds_per_step": t0.elapsed_time(t1) / 1e3 / steps, "steps": steps,
            "how": "pinned host Q/K/V uploaded and O downloaded inside the timed region every step; "
                   "uploads of step i+1 overlap step i's attention (two device buffer sets), O is "
                   "downloaded per kv-group as each group's attention finishes"}


# ---------------------------------------------------------------------------- CPU oracle arm
def oracle_baseline(w, q, k, v, idx, budget_s: float, seed: int = 0, params=None) -> dict:
    """Time the fp64 oracle on a bounded sample of the workload and extrapolate to one layer:
    selection of one Vertical-Slash and one Pooled-Estimation head (scaled by the head counts),
    and attention on a sample of query blocks (scaled by selected block pairs)."""
    from oracle import crisp_oracle as O

    G = w.h_q // w.h_kv
    nb = -(-w.n // 128)
    route = idx.route.cpu().numpy() if idx is not None else None
    conc = W.concentrated_heads(w)
    # one head of each kind the workload has (a one-head workload has only one)
    vs_head = next((h for h in range(w.h_q) if conc[h]), None)
    pe_head = next((h for h in range(w.h_q) if not conc[h]), None)
    heads = [h for h in (vs_head, pe_head) if h is not None]
    f64 = lambda t: t.detach().cpu().to(torch.float64).numpy()  # noqa: E731
    sel, times = {}, {}
    for h in heads:
        qh, kh = f64(q[h]), f64(k[h // G])
        t0 = time.perf_counter()
        sel[h] = O.select_head(qh, kh, **oracle_kwargs(params or crisp.Params()))
        times[h] = time.perf_counter() - t0
    n_vs = int(route.sum()) if route is not None else sum(conc)
    n_pe = w.h_q - n_vs
    t_vs = times[vs_head if vs_head is not None else pe_head]
    t_pe = times[pe_head if pe_head is not None else vs_head]
    sel_layer = t_vs * n_vs + t_pe * n_pe
    # attention sample: query blocks of both heads until the budget is used
    rng = np.random.default_rng(seed)
    pairs_done, t_attn = 0, 0.0
    kcache = {}
    start = time.perf_counter()
    while time.perf_counter() - start < budget_s:
        h = int(rng.choice(heads))
        qb = int(rng.integers(0, nb))
        lists = sel[h]["lists"]
        kv = h // G
        if kv not in kcache:
            kcache[kv] = (f64(k[kv]), f64(v[kv]))
        kk, vv = kcache[kv]
        t0 = time.perf_counter()
        O.attention_block(f64(q[h, qb * 128:(qb + 1) * 128]), kk, vv, lists[qb], qb)
        t_attn += time.perf_counter() - t0
        pairs_done += len(lists[qb])
    if idx is not None:
        total_pairs = int(idx.row_ptr[:, nb].sum().item())
    else:
        # no GPU index (the oracle arm alone): the layer's selected pairs from the oracle's own
        # lists of the timed heads, each standing for the heads of its kind
        per = {h: sum(len(x) for x in sel[h]["lists"]) for h in heads}
        total_pairs = per[vs_head if vs_head is not None else pe_head] * n_vs + \
            per[pe_head if pe_head is not None else vs_head] * n_pe
    attn_layer = t_attn / max(pairs_done, 1) * total_pairs
    layer_s = sel_layer + attn_layer
    try:
        from threadpoolctl import threadpool_info
        cores = max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:
        cores = os.cpu_count() or 1
    return {"value": w.n / layer_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": (f"selection of head(s) {heads} (planted-concentrated first) timed in full and "
                       f"scaled by {n_vs} VS / {n_pe} PE-routed heads; attention on {pairs_done} sampled "
                       f"block pairs ({t_attn:.1f}s) scaled to {total_pairs} selected pairs"),
            "extrapolated_layer_s": layer_s}


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    if args.n:
        w = w.scaled(args.n)
    torch.manual_seed(0)
    q, k, v, meta = W.generate(w, device="cuda" if torch.cuda.is_available() else "cpu")
    vals = []
    t0 = time.perf_counter()
    base = None
    for i in range(args.warmup + args.steps):
        b = oracle_baseline(w, q, k, v, None, args.cpu_seconds / max(1, args.steps + args.warmup), seed=i,
                            params=RULES[args.rules])
        if i >= args.warmup:
            vals.append(b["value"])
            base = b
    value = float(np.mean(vals))
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": w.n / value * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": bench_config(w, args, world),
           "impl": "reference",
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": base["cores"], "kind": "oracle",
                            "sample": base["sample"]},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "wall_s": time.perf_counter() - t0}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="crisp", choices=["crisp", "reference"])
    ap.add_argument("--rules", default="crisp", choices=sorted(RULES),
                    help="index-selection rules (the headline metric uses CRISP's own)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-fp8", dest="fp8", action="store_false",
                    help="skip the FP8-logits variant leg (run after the timed region)")
    ap.add_argument("--no-dense", dest="dense", action="store_false",
                    help="skip the dense-attention comparison run after the timed region")
    ap.add_argument("--dense-steps", type=int, default=2)
    ap.add_argument("--n", type=int, default=0, help="run the workload's generator at another length")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_crisp(args)


if __name__ == "__main__":
    main()
