#!/usr/bin/env python
"""Benchmark of CRISP sparse prefill on B200 (one JSON line on rank 0).

A step is one pass of the whole hot path over one synthetic input: route
(proxy map, block scores, C_struct), select (VS / PE selection, tile lists)
and block-sparse attention. The dense baseline (same attention kernel over
every causal tile) is timed beside it for the speedup.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama_512k]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample
  python bench.py --sweep out.jsonl      # N x diffuse-fraction x alpha sweep

Multi-GPU (torchrun): every rank runs its own replica (independent input,
seed + rank); the path has no exchange step, so there is no collective on
the data path. Timing is the max over ranks of CUDA-event time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse prefill attention ms, speedup vs own dense kernel at 128k/512k; TC util"
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        loaded = [x for x in sm if x > 0.5 * (mx or max(sm))] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(values, device):
    """Element-wise max of a list of floats over all ranks (identity when not
    distributed). Each rank times its own replica; the job's time is the
    slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def sum_over_ranks(values, device):
    """Element-wise sum of a list of numbers over all ranks (identity when
    not distributed): the whole job's tiles and heads under head sharding."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()]


def rank_problem(w, args, rank, world):
    """The workload this rank runs and the KV heads it owns: with --shard
    replicas every rank runs its own whole problem (seed + rank); with
    --shard heads rank r runs KV heads kv_head_range(H_kv, N, r) of one
    problem with their query heads (same seed on every rank)."""
    from dynamic_block_sparse_qk_b200.shard import kv_head_range
    if args.shard == "heads":
        kv = kv_head_range(w.h_kv, world, rank)
        g = w.h_q // w.h_kv
        return w.with_(seed=args.seed), list(kv), w.with_(h_q=len(kv) * g, h_kv=len(kv))
    wr = w.with_(seed=args.seed + rank)
    return wr, None, wr


def launches_per_step(router: str, n_blocks: int) -> dict:
    """Kernels of this library launched by one call of each stage."""
    route = 2 + (2 if router == "jsd" else 0)      # proxy stats (+ merge), scores (+ C_struct route),
    #                                                 JSD only: K pool, JSD route
    if n_blocks * (n_blocks + 1) // 2 <= 256 * 257 // 2:
        select = 5                                  # vs select, K/Q pool, PE logits, one-CTA PE cut, tiles
    else:
        select = 9                                  # vs select, K/Q pool, PE logits/normalise,
        #                                             3 x hist (+ cut), tie count (+ scan), tiles
    return {"route": route, "select": select, "attention": 1, "total": route + select + 1}


def workload_config(w, args) -> dict:
    """The config block both arms report for a workload and its hyper-parameters."""
    return {"workload": w.name, "batch": w.batch, "h_q": w.h_q, "h_kv": w.h_kv,
            "head_dim": w.head_dim, "seq_len": w.seqlen, "block": w.block,
            "diffuse_frac": w.diffuse_frac, "alpha": args.alpha, "gamma": args.gamma,
            "router": args.router, "vs_rule": args.vs_rule, "granularity": args.granularity,
            **({"lengths": list(w.lengths)} if w.lengths is not None else {})}


def stage_algorithmic_bytes(w, pattern, tiles: int) -> dict:
    """HBM bytes the routing and selection stages must move at least once
    (algorithmic, not measured). Routing reads K once per KV head (the proxy
    is bound by its exp2 work, so this only says how far from HBM-bound it
    is). Selection reads Q of the PE heads and K of the KV heads with a PE
    query head once (block-mean pooling), passes once over each PE head's
    N_b(N_b+1)/2 fp32 estimate entries (the gamma cut), and writes the tile
    lists: 4 bytes per executed tile and per query block (counts). The
    kernels pass over the estimate more than once (logits, normalisation,
    three radix levels, ties, tile builder); those repeats are the
    implementation's, not the algorithm's, and are not counted."""
    g = w.h_q // w.h_kv
    d2 = w.head_dim * 2
    route = sum(w.length(b) * w.h_kv * d2 for b in range(w.batch))
    select = 4 * int(tiles)
    for b in range(w.batch):
        n = w.length(b)
        nb = -(-n // w.block)
        pe = [h for h in range(w.h_q) if pattern[b * w.h_q + h] == 1]
        select += (len(pe) + len({h // g for h in pe})) * n * d2 + len(pe) * nb * (nb + 1) // 2 * 4
        select += w.h_q * nb * 4
    return {"route": route, "select": select}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the sparse attention kernel, from an ncu capture of this bench's own
# command on a B200 (1 pass; profiles/attn_tc_sparse_llama512k_dram.md).
# Valid for the default hyper-parameters of the workload and the kernel as
# captured; any other configuration reports null.
ATTN_DRAM_BYTES = {"llama_512k": 156_760_839_168 + 4_371_607_040}


def attn_traffic(w, args):
    if (args.alpha, args.gamma, args.router, args.vs_rule, args.granularity) != (1.0, 0.95, "cstruct", "alpha", "tile"):
        return None
    if args.shard != "replicas" or w.lengths is not None:
        return None
    return ATTN_DRAM_BYTES.get(w.name)


def executed_flops(tile_cnt_sum: int, block: int, d: int) -> float:
    """4 * B^2 * d per executed tile (QK^T and PV); diagonal tiles count in full."""
    return float(tile_cnt_sum) * 4.0 * block * block * d


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import dynamic_block_sparse_qk_b200 as C
    from synthetic import WORKLOADS, make_qkv

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w_full, kv_heads, w = rank_problem(WORKLOADS[args.workload], args, rank, world)
    q, k, v, meta = make_qkv(w_full, device=str(dev), heads_kv=kv_heads)
    lens = None if w.lengths is None else torch.tensor(list(w.lengths), dtype=torch.int32, device=dev)
    p = C.params_for(q, k, block=w.block, alpha=args.alpha, gamma=args.gamma, router=args.router,
                     vs_rule=args.vs_rule, seq_lens=lens, granularity=args.granularity)
    ws = C.alloc_workspace(p, dev)
    bh, nb = p.batch * p.h_q, p.n_blocks
    pattern = torch.empty(bh, dtype=torch.int32, device=dev)
    score = torch.empty(bh, dtype=torch.float32, device=dev)
    p_v = torch.empty(bh, nb, dtype=torch.float32, device=dev)
    p_s = torch.empty(bh, nb, dtype=torch.float32, device=dev)
    tidx = torch.empty(bh, nb, nb, dtype=torch.int32, device=dev)
    tcnt = torch.empty(bh, nb, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if in_bytes < 4 * L2_BYTES else None
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs: evs[0].record(stream)
        C.crisp_route(p, q, k, ws, pattern, score, p_v, p_s, stream=stream)
        if evs: evs[1].record(stream)
        C.crisp_select(p, q, k, pattern, p_v, p_s, ws, want_mask=False, tile_idx=tidx, tile_cnt=tcnt,
                       stream=stream)
        if evs: evs[2].record(stream)
        C.crisp_sparse_prefill(p, q, k, v, tidx, tcnt, ws, o=o, lse=lse, stream=stream)
        if evs: evs[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status = C.crisp_get_device_status(ws)
    cnt_sum = int(tcnt.sum().item())
    n_vs = int((pattern == 0).sum().item())
    nbv = [-(-w.length(b) // w.block) for b in range(w.batch)]        # each sequence's blocks
    causal_tiles = p.h_q * sum(x * (x + 1) // 2 for x in nbv)
    stage_bytes = stage_algorithmic_bytes(w, pattern.cpu().tolist(), cnt_sum)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            step(evs[i])
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    per = [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(3)] for i in range(args.steps)]
    step_ms = [sum(x) for x in per]
    ms_local = statistics.mean(step_ms)
    stages = {n: statistics.mean(x[j] for x in per) for j, n in enumerate(("route", "select", "attend"))}

    # dense baseline: same kernel, every causal tile (1 warm-up + args.dense_steps timed)
    od = torch.empty_like(q)
    dts = []
    if args.dense_steps > 0:
        C.crisp_dense_prefill(p, q, k, v, ws, o=od, lse=lse, stream=stream)
        torch.cuda.synchronize(dev)
    for _ in range(args.dense_steps):
        if flush is not None:
            flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        C.crisp_dense_prefill(p, q, k, v, ws, o=od, lse=lse, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        dts.append(e0.elapsed_time(e1))
    dense_ms = statistics.mean(dts) if dts else float("nan")
    del od

    ms, dense_ms, attend_ms = max_over_ranks([ms_local, dense_ms, stages["attend"]], dev)
    if args.shard == "heads":
        # the job's work is the sum of the ranks' slices; its time the slowest rank's
        cnt_sum, causal_tiles, n_vs, bh_all = (int(x) for x in sum_over_ranks(
            [cnt_sum, causal_tiles, n_vs, p.batch * p.h_q], dev))
        stages["attend"] = attend_ms
    else:
        bh_all = p.batch * p.h_q

    # end-to-end through the public API with host buffers (H2D inputs, D2H output)
    e2e = None
    if not args.no_e2e:
        hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
        hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hq.copy_(q)
        hk.copy_(k)
        hv.copy_(v)
        torch.cuda.synchronize(dev)

        # the public host-input entry point, the C ABI's crisp_prefill_host:
        # per KV head, copies in, the three stages and the copy out, overlapped
        # across KV heads; its device workspace is allocated once, like the
        # device path's
        hp = dict(block=w.block, alpha=args.alpha, gamma=args.gamma, router=args.router,
                  vs_rule=args.vs_rule, granularity=args.granularity)
        hws = C.host_workspace(hq, hk, kv_per_chunk=1, device=dev, **hp)

        def e2e_step():
            C.prefill_from_host(hq, hk, hv, ho, seq_lens=None if w.lengths is None else list(w.lengths),
                                kv_per_chunk=1, device=dev, ws=hws, **hp)

        e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], dev)[0]
        # bytes that cross PCIe: with lengths, only each sequence's own rows
        rows = sum(w.length(b) for b in range(w.batch))
        h2d = rows * (w.h_q + 2 * w.h_kv) * w.head_dim * q.element_size()
        d2h = rows * w.h_q * w.head_dim * o.element_size()
        e2e = {"value": round(e2e_ms, 3), "unit": "ms", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "path": "crisp_prefill_host, C ABI (pinned host Q/K/V in, O out; copies overlapped per KV head)"}
        del hq, hk, hv, ho, hws

    peaks = _peaks()
    flops = executed_flops(cnt_sum, w.block, w.head_dim)
    attn_tflops = flops / (stages["attend"] * 1e-3) / 1e12
    dense_tflops = executed_flops(causal_tiles, w.block, w.head_dim) / (dense_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"] if stages["attend"] > 50 else peaks["bf16_tflops"]
    line = {
        "metric": METRIC, "value": round(ms, 3), "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": False,
        "scaling": "strong" if args.shard == "heads" else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {**workload_config(w_full, args),
                   "parallelism": f"{'kv_heads' if args.shard == 'heads' else 'replicas'}{world}",
                   "l2": "flushed between steps" if flush is not None else
                         f"inputs ({in_bytes / 2**30:.1f} GiB) larger than L2"},
        "stages_ms": {k_: round(v_, 3) for k_, v_ in stages.items()},
        "dense_ms": round(dense_ms, 3),
        "speedup_vs_dense": round(dense_ms / ms, 3),
        "speedup_attend_only": round(dense_ms / stages["attend"], 3),
        "route_select_frac": round((stages["route"] + stages["select"]) / ms, 4),
        "density": round(cnt_sum / causal_tiles, 5), "vs_heads": n_vs, "heads": bh_all,
        "executed_tiles": cnt_sum,
        "attend_tflops": round(attn_tflops, 1), "dense_tflops": round(dense_tflops, 1),
        "roofline": {"bound": "tensor", "kernel": "attention (sparse)", "achieved": round(attn_tflops, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(attn_tflops / peak, 4),
                     "frac_of_burst": round(attn_tflops / peaks["bf16_tflops"], 4),
                     "frac_of_spec_2250": round(attn_tflops / 2250.0, 4),
                     "peak_source": f"{peaks['source']} bf16 "
                                    f"{'sustained' if peak == peaks['bf16_tflops_sustained'] else 'burst'}",
                     "traffic": attn_traffic(w_full, args),
                     "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
                     "algorithmic_bytes": int(in_bytes + o.numel() * o.element_size() + lse.numel() * 4)},
        "stage_hbm": {k_: {"algorithmic_bytes": int(v_),
                           "achieved_gbs": round(v_ / (stages[k_] * 1e-3) / 1e9, 1),
                           "frac_of_hbm": round(v_ / (stages[k_] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
                      for k_, v_ in stage_bytes.items()},
        "e2e": e2e,
        "gpu_launches": launches_per_step(args.router, nb)["total"] * args.steps,
        "device_status": status,
        "clocks": clk.summary(),
    }
    return line


# ----------------------------------------------------------------------------- sweep
def time_point(C, p, q, k, v, ws, timed, dev) -> dict:
    """Per-stage CUDA-event times of one prefill configuration (route,
    select, attend; each the mean of timed()'s repetitions), its tile
    density and the attention kernel's TFLOP/s on executed tiles."""
    import torch
    out = {}

    def route():
        out["r"] = C.crisp_route(p, q, k, ws)

    def select():
        r = out["r"]
        out["s"] = C.crisp_select(p, q, k, r[0], r[2], r[3], ws, want_mask=False)

    def attend():
        s_ = out["s"]
        out["a"] = C.crisp_sparse_prefill(p, q, k, v, s_[1], s_[2], ws, want_lse=False)

    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        t_route = timed(route)
        t_select = timed(select)
        t_attend = timed(attend)
    pattern, tcnt = out["r"][0], out["s"][2]
    nb = p.n_blocks
    causal = p.batch * p.h_q * nb * (nb + 1) // 2
    tiles = int(tcnt.sum())
    status = C.crisp_get_device_status(ws)
    return {"route_ms": round(t_route, 4), "select_ms": round(t_select, 4), "attend_ms": round(t_attend, 4),
            "total_ms": round(t_route + t_select + t_attend, 4), "density": round(tiles / causal, 5),
            "executed_tiles": tiles, "vs_heads": int((pattern == 0).sum()), "heads": p.batch * p.h_q,
            "attend_tflops": round(tiles * 4 * p.block ** 2 * p.head_dim / (t_attend * 1e-3) / 1e12, 1),
            "device_status": status, "clocks": clk.summary(), "_pattern": pattern.clone()}


def _event_timer(dev, reps, graphs=False):
    """timed(fn): mean CUDA-event time of `reps` runs of fn after one
    warm-up. With graphs, fn (a sequence of library calls) is captured once
    into a CUDA graph and the graph is replayed, so the time is the GPU's
    alone, without the host's per-call overhead (how a serving loop that
    captures its prefill runs it); the outputs fn stores stay valid."""
    import torch
    stream = torch.cuda.current_stream(dev)
    keep = []

    def timed(fn):
        fn()
        torch.cuda.synchronize(dev)
        run = fn
        if graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="relaxed"):
                fn()
            keep.append(g)
            run = g.replay
            run()
            torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            run()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps
    return timed


# The pages' latency comparison (CRISP page, Section 5.3 and Table 4): CRISP
# at alpha 1.0 / 1.25 / 1.5 against FlexPrefill (JSD routing, gamma-cumsum VS
# index) at gamma 0.95 / 0.97, plus the first ablation (C_struct routing with
# the gamma VS index, Table 5's Abl.1).
COMPARE_METHODS = {
    "crisp_alpha1.0": dict(router="cstruct", vs_rule="alpha", alpha=1.0, gamma=0.95),
    "crisp_alpha1.25": dict(router="cstruct", vs_rule="alpha", alpha=1.25, gamma=0.95),
    "crisp_alpha1.5": dict(router="cstruct", vs_rule="alpha", alpha=1.5, gamma=0.95),
    "flexprefill_gamma0.95": dict(router="jsd", vs_rule="gamma", alpha=1.0, gamma=0.95),
    "flexprefill_gamma0.97": dict(router="jsd", vs_rule="gamma", alpha=1.0, gamma=0.97),
    "abl1_cstruct_gamma0.95": dict(router="cstruct", vs_rule="gamma", alpha=1.0, gamma=0.95),
}


def run_compare(args, out_path):
    """CRISP vs FlexPrefill on the named workloads: per method the stage
    times, density, speedup over the dense kernel (timed once per workload)
    and the routes' agreement with C_struct routing. One JSON line each."""
    import torch
    import dynamic_block_sparse_qk_b200 as C
    from synthetic import WORKLOADS, make_qkv

    dev = torch.device("cuda", 0)
    timed = _event_timer(dev, max(1, args.steps), graphs=args.graphs)
    for name in args.compare_workloads.split(","):
        w = WORKLOADS[name].with_(seed=args.seed)
        q, k, v, _ = make_qkv(w, device=str(dev))
        base = C.params_for(q, k, block=w.block)
        ws = C.alloc_workspace(base, dev)
        dense_ms = timed(lambda: C.crisp_dense_prefill(base, q, k, v, ws, want_lse=False))
        ref_pattern = None
        for meth, kw in COMPARE_METHODS.items():
            p = C.params_for(q, k, block=w.block, **kw)
            pt = time_point(C, p, q, k, v, ws, timed, dev)
            pat = pt.pop("_pattern")
            if ref_pattern is None:
                ref_pattern = pat
            rec = {"workload": w.name, "method": meth, **kw, **pt, "dense_ms": round(dense_ms, 4),
                   "timing": "cuda_graph" if args.graphs else "eager",
                   "speedup_vs_dense": round(dense_ms / pt["total_ms"], 3),
                   "speedup_attend_only": round(dense_ms / pt["attend_ms"], 3),
                   "route_agreement_with_cstruct": round(float((pat == ref_pattern).float().mean()), 4)}
            with open(out_path, "a") as fo:
                fo.write(json.dumps(rec) + "\n")
            print(json.dumps(rec), flush=True)
        del q, k, v, ws
        torch.cuda.empty_cache()


SWEEP_N = (8192, 16384, 32768, 65536, 131072, 262144, 524288)
SWEEP_F = (0.0, 0.25, 0.5)
SWEEP_ALPHA = (0.5, 1.0, 2.0)


def run_sweep(args, out_path):
    """Llama-shaped sweep: sequence length x diffuse-head fraction x alpha.

    One JSON line per point: per-stage ms (route, select, attend), dense ms
    (same kernel, every causal tile, once per (N, f)), speedup, selected-tile
    density and the agreement of the C_struct and JSD routers on the heads.
    Points already present in out_path are skipped, so an interrupted sweep
    resumes where it stopped."""
    import torch
    import dynamic_block_sparse_qk_b200 as C
    from synthetic import make_qkv, sweep_workload

    done = set()
    if os.path.exists(out_path):
        with open(out_path) as f:
            for line in f:
                try:
                    d = json.loads(line)
                    done.add((d["seq_len"], d["diffuse_frac"], d["alpha"], d.get("vs_rule", "alpha"),
                              d.get("granularity", "tile")))
                except (ValueError, KeyError):
                    pass
    dev = torch.device("cuda", 0)
    timed = _event_timer(dev, max(1, args.steps), graphs=args.graphs)

    ns = tuple(int(x) for x in args.sweep_n.split(",")) if args.sweep_n else SWEEP_N
    fs = tuple(float(x) for x in args.sweep_f.split(",")) if args.sweep_f else SWEEP_F
    alphas = tuple(float(x) for x in args.sweep_alpha.split(",")) if args.sweep_alpha else SWEEP_ALPHA
    for n in ns:
        for f in fs:
            todo = [a for a in alphas if (n, f, a, args.vs_rule, args.granularity) not in done]
            if not todo:
                continue
            w = sweep_workload(n, f).with_(seed=args.seed)
            q, k, v, _ = make_qkv(w, device=str(dev))
            base = C.params_for(q, k, block=w.block)
            ws = C.alloc_workspace(base, dev)
            dense_ms = timed(lambda: C.crisp_dense_prefill(base, q, k, v, ws))
            pj = C.params_for(q, k, block=w.block, router="jsd")
            pat_j = C.crisp_route(pj, q, k, ws)[0].clone()
            for a in todo:
                p = C.params_for(q, k, block=w.block, alpha=a, vs_rule=args.vs_rule, granularity=args.granularity)
                pt = time_point(C, p, q, k, v, ws, timed, dev)
                pat = pt.pop("_pattern")
                rec = {"seq_len": n, "diffuse_frac": f, "alpha": a, "vs_rule": args.vs_rule, "granularity": args.granularity,
                       "workload": w.name,
                       "timing": "cuda_graph" if args.graphs else "eager",
                       **pt, "dense_ms": round(dense_ms, 4),
                       "speedup_vs_dense": round(dense_ms / pt["total_ms"], 3),
                       "cstruct_jsd_agreement": round(float((pat == pat_j).float().mean()), 4)}
                with open(out_path, "a") as fo:
                    fo.write(json.dumps(rec) + "\n")
                print(json.dumps(rec), flush=True)
            del q, k, v, ws
            torch.cuda.empty_cache()


# ----------------------------------------------------------------------------- CPU oracle
def oracle_inputs(w):
    """CPU inputs of the oracle sample: one VS and one PE query head and their KV heads."""
    from synthetic import make_qkv, head_kinds
    diffuse = set(head_kinds(w)["diffuse"])
    vs_head = next(h for h in range(w.h_q) if h not in diffuse)
    pe_head = min(diffuse) if diffuse else None
    heads = [vs_head] + ([pe_head] if pe_head is not None else [])
    q, k, v, _ = make_qkv(w, heads_q=heads)
    return {"q": q, "k": k, "v": v, "heads": heads, "vs_head": vs_head, "pe_head": pe_head,
            "n_diffuse": len(diffuse)}


def oracle_sample(w, args, inp, budget_s: float):
    """Times the float64 oracle on a bounded sample of the workload and
    extrapolates to one full prefill (ms). Returns (ms, description, threads)."""
    import numpy as np
    import oracle as O

    g = w.h_q // w.h_kv
    prm = O.CrispParams(block=w.block, alpha=args.alpha, gamma=args.gamma, router=args.router,
                        vs_rule=args.vs_rule, granularity=args.granularity)
    nb = w.n_blocks
    sel_ms, tiles, attn_ms_per_tile = {}, {}, []
    t_start = time.perf_counter()
    for i, h in enumerate(inp["heads"]):
        qh = O.bf16_to_f64(inp["q"][0, i])
        kh = O.bf16_to_f64(inp["k"][0, h // g])
        vh = O.bf16_to_f64(inp["v"][0, h // g])
        t0 = time.perf_counter()
        r = O.head_route_and_select(qh, kh, prm)
        sel_ms[h] = (time.perf_counter() - t0) * 1e3
        tiles[h] = int(r["mask"].sum())
        rng = np.random.default_rng(h)
        for qb in sorted(set([nb - 1] + [int(x) for x in rng.integers(0, nb, size=3)])):
            if attn_ms_per_tile and time.perf_counter() - t_start > budget_s:
                break                                      # at least one query block is always timed
            t0 = time.perf_counter()
            O.masked_attention_rows(qh, kh, vh, r["mask"], w.block, prm.scale(w.head_dim), [qb],
                                    r.get("vs_tokens"))
            attn_ms_per_tile.append((time.perf_counter() - t0) * 1e3 / max(int(r["mask"][qb].sum()), 1))
    n_pe = inp["n_diffuse"]
    n_vs = w.h_q - n_pe
    vs_h, pe_h = inp["vs_head"], inp["pe_head"]
    total_sel = sel_ms[vs_h] * n_vs + (sel_ms[pe_h] * n_pe if pe_h is not None else 0.0)
    total_tiles = tiles[vs_h] * n_vs + (tiles[pe_h] * n_pe if pe_h is not None else 0)
    ms = total_sel + statistics.mean(attn_ms_per_tile) * total_tiles
    desc = (f"oracle route+select timed on {len(inp['heads'])} heads (1 VS, 1 PE), attention on "
            f"{len(attn_ms_per_tile)} sampled query blocks; extrapolated to {w.h_q} heads and "
            f"{total_tiles} executed tiles")
    try:
        from threadpoolctl import threadpool_info
        threads = max([x.get("num_threads", 1) for x in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count()
    return ms, desc, threads


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def run_reference(args):
    from synthetic import WORKLOADS
    w = WORKLOADS[args.workload].with_(seed=args.seed)
    inp = oracle_inputs(w)
    vals, desc, threads = [], "", 1
    for i in range(args.warmup + args.steps):
        ms, desc, threads = oracle_sample(w, args, inp, budget_s=args.cpu_budget)
        if i >= args.warmup:
            vals.append(ms)
    v = statistics.mean(vals)
    return {"metric": METRIC, "value": round(v, 1), "unit": "ms", "n_gpus": 0, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(v, 1), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {**workload_config(w, args), "parallelism": "host cores"},
            "cpu_baseline": {"value": round(v, 1), "unit": "ms", "cores": threads, "kind": "oracle",
                             "cpu": cpu_model(), "sample": desc + " (extrapolated)"},
            "e2e": {"value": round(v, 1), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- driver
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--dense-steps", type=int, default=2)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama_512k")
    ap.add_argument("--alpha", type=float, default=1.0)
    ap.add_argument("--gamma", type=float, default=0.95)
    ap.add_argument("--router", default="cstruct")
    ap.add_argument("--vs-rule", default="alpha", choices=["alpha", "alpha_median", "gamma"])
    ap.add_argument("--granularity", default="tile", choices=["tile", "token"],
                    help="VS mask: selected blocks as whole tiles, or slash blocks as diagonal bands")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: independent replicas per rank (weak scaling), or one problem split by "
                         "KV-head groups (strong scaling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--sweep", default=None, help="write the N x f x alpha sweep to this JSONL file")
    ap.add_argument("--sweep-n", default=None, help="comma-separated sequence lengths (default: all)")
    ap.add_argument("--sweep-f", default=None, help="comma-separated diffuse-head fractions (default: all)")
    ap.add_argument("--sweep-alpha", default=None, help="comma-separated alpha values (default: 0.5,1,2)")
    ap.add_argument("--graphs", action="store_true",
                    help="sweep / compare: time each stage as a replayed CUDA graph (GPU time only)")
    ap.add_argument("--compare", default=None,
                    help="write the CRISP vs FlexPrefill latency comparison to this JSONL file")
    ap.add_argument("--compare-workloads", default="qwen_131k,llama_512k",
                    help="comma-separated workloads of the comparison")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args, args.sweep)
        return
    if args.compare:
        run_compare(args, args.compare)
        return

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    line = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from synthetic import WORKLOADS
        w = WORKLOADS[args.workload].with_(seed=args.seed)
        if w.batch == 1:
            ms, desc, threads = oracle_sample(w, args, oracle_inputs(w), budget_s=args.cpu_budget)
            line["cpu_baseline"] = {"value": round(ms, 1), "unit": "ms", "cores": threads, "kind": "oracle",
                                    "cpu": cpu_model(), "sample": desc + " (extrapolated)"}
        else:   # the sampler extrapolates one sequence's heads; batches are not sampled
            line["cpu_baseline"] = None
            line["cpu_baseline_note"] = "oracle sample covers single-sequence workloads only"
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
