"""Benchmark of the EntmaxKV support-aware paged α-entmax decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one decode token for every (sequence, KV head) unit of the
workload: cache append + tail-page metadata, bounding-box page scores, top-k
page selection, sparse α-entmax attention (scores over the selected K, τ,
support-only V).  Inputs are resident in HBM; L2 is flushed (256 MiB read)
between steps.  Prints one JSON line on rank 0.

Workload (default): the clustered 128k-context decode — batch 4, 32 query /
8 KV heads, d = 128, page size 16, bf16 cache, top-k k = 256, α = 1.5.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "entmax decode steps/s per (batch×KV-head) at 128k ctx; HBM GB/s vs roofline"
UNIT = "(sequence×KV-head) decode steps/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0

# dram__bytes_read.sum + dram__bytes_write.sum per launch from one ncu capture
# of the bench workload's shape, keyed by a hash of the kernel's sources (a
# changed kernel has no measured traffic until it is captured again)
SCORE_FILES = ("score.cu", "common.cuh", "kernels.cuh")
DECODE_FILES = ("decode_fused.cu", "decode.cuh", "common.cuh", "kernels.cuh")
SCORE_TRAFFIC = {"d0d585139e2ad614": 137794048}   # profiles/score_kernel_clustered_128k.md
DECODE_TRAFFIC = {"f4f00457b9e63761": 56003584}   # profiles/fused_decode_kernel_clustered_128k.md


def kernel_hash(files=SCORE_FILES):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "sparse_kv_cache_kmax_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_timing(elapsed_s: float, units_done: int, group=None):
    """Max elapsed time over ranks and total units over ranks (whole job)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return elapsed_s, units_done
    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([elapsed_s], dtype=torch.float64, device=dev)
    u = torch.tensor([units_done], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(u, op=dist.ReduceOp.SUM, group=group)
    return float(t.item()), int(u.item())


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = uuid
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50"], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        mhz, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                if self.uuid and parts[1] != self.uuid:
                    continue
                try:
                    mhz.append(float(parts[2]))
                    mx.append(float(parts[3]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[6:10]):
                    if val.lower() == "active":
                        reasons.add(name)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(mhz)}


class L2Flush:
    """Evicts the 126 MB L2 between timed steps by reading a 256 MiB buffer
    (a read leaves clean lines, so the next step pays no write-back)."""

    def __init__(self, dev):
        self.buf = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def zero_(self):
        torch.sum(self.buf, dim=0, out=self.sink)


# ---------------------------------------------------------------- bytes
def algorithmic_bytes(inp, eng, support_pages, support_tokens):
    """Bytes one step must move: metadata rows, q, ub, selected K, V of
    support pages, outputs, and the append (tail page + new rows + metadata).
    The decode kernel's own bytes count V token by token (the union of the
    group heads' support), as the method needs them; the kernel reads whole
    support pages, which the measured traffic shows."""
    wl = inp["workload"]
    es = inp["k_pool"].element_size()
    d, S, G = wl.head_dim, wl.page_size, wl.group
    lens = inp["seq_lens"].tolist()
    pages = [-(-L // S) for L in lens]
    units_pages = sum(pages) * wl.num_kv_heads
    meta = units_pages * 2 * d * es
    q = wl.batch * wl.num_q_heads * d * es
    ub = units_pages * 4
    n_sel = eng.n_sel.to(torch.int64)
    sel_tokens = int(n_sel.sum()) * S                     # full pages (tail rounding ignored)
    selK = sel_tokens * d * es
    supV = int(support_pages) * S * d * es
    out = wl.batch * wl.num_q_heads * d * 4
    append = wl.units * (S * d * es + 2 * d * es + 4 * d * es)
    supV_tok = int(support_tokens) * d * es
    return {"meta": meta, "q": q, "ub": ub, "sel_k": selK, "support_v": supV, "out": out,
            "append": append, "score_kernel": meta + q + ub,
            "decode_kernel": selK + supV_tok + q + out,
            "step": meta + q + selK + supV + out + append}


# ---------------------------------------------------------------- our arm
def run_ours(args):
    from sparse_kv_cache_kmax_b200 import binding as Bd
    from sparse_kv_cache_kmax_b200.engine import DecodeEngine
    from sparse_kv_cache_kmax_b200.workloads import WORKLOADS, make_inputs

    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    Bd.lib()                                   # fail loudly if the library is missing

    wl = WORKLOADS[args.workload]
    inp = make_inputs(wl, seed=3000 + rank, device=dev, n_new=1)
    q, k_new, v_new = inp["q"], inp["k_new"][0], inp["v_new"][0]
    alpha, k = args.alpha, args.k or wl.topk
    eng = DecodeEngine(inp["k_pool"], inp["v_pool"], inp["page_table"], inp["seq_lens"], wl.num_q_heads,
                       policy="topk", k=k, alpha=alpha)
    eng.build_meta()
    cache, seqs, Hq = eng.cache, eng.seqs, wl.num_q_heads
    scale = float(np.float32(wl.scale))
    ub = torch.empty(wl.batch, wl.num_kv_heads, inp["max_pages"], device=dev)
    dec_ws = Bd.workspace(Bd.ekv_workspace_bytes(Bd.EKV_OP_ENTMAX_DECODE, cache, seqs, Hq, k), dev)
    n_tk = Bd.ekv_workspace_bytes(Bd.EKV_OP_SELECT_TOPK, cache, seqs, Hq, k)
    tk_ws = Bd.workspace(n_tk, dev) if n_tk else None
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def stage_step(ev):
        ev[0].record(stream)
        Bd.ekv_append(cache, seqs, k_new, v_new, stream)
        ev[1].record(stream)
        Bd.ekv_score_pages(cache, seqs, q, scale, ub, stream)
        ev[2].record(stream)
        Bd.ekv_select_topk(seqs, wl.num_kv_heads, wl.page_size, ub, k, eng.sel, eng.n_sel, stream, ws=tk_ws)
        ev[3].record(stream)
        Bd.ekv_entmax_decode(cache, seqs, q, scale, alpha, eng.sel, eng.n_sel, k, eng.out, dec_ws, stream=stream)
        ev[4].record(stream)

    def timed(step_fn, n_events, steps, warmup):
        for _ in range(warmup):
            flush.zero_()
            step_fn([torch.cuda.Event(enable_timing=True) for _ in range(n_events)])
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_events)] for _ in range(steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            flush.zero_()
            step_fn(evs[i])
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(n_events - 1)] for i in range(steps)])
        return per                              # ms, [steps, stages]

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        uuid = None

    # headline: the whole step as one C-ABI call (its kernels chain with
    # programmatic dependent launch), CUDA events at step boundaries only
    def fused_step(ev):
        ev[0].record(stream)
        eng.step(q, k_new, v_new, stream)
        ev[1].record(stream)

    with ClockSampler(uuid) as clk:
        per_step = timed(fused_step, 2, args.steps, args.warmup)[:, 0]
    step_ms = float(per_step.mean())
    total_s = float(per_step.sum()) / 1e3
    max_s, units_all = reduce_timing(total_s, wl.units * args.steps)
    value = units_all / max_s
    clocks = clk.summary()
    # breakdown: the same stages as separate calls with events between them
    per = timed(stage_step, 5, max(3, min(args.steps, 300)), args.warmup)
    stages = per.mean(axis=0)

    # support statistics of the last step (untimed): pages whose V the step read
    words = (k * wl.page_size + 31) // 32
    bits = torch.zeros(wl.batch, Hq, words, dtype=torch.int32, device=dev)
    cnt = torch.zeros(wl.batch, Hq, dtype=torch.int32, device=dev)
    tau_last = torch.zeros(wl.batch, Hq, device=dev)
    Bd.ekv_entmax_decode(cache, seqs, q, scale, alpha, eng.sel, eng.n_sel, k, eng.out, dec_ws,
                         tau=tau_last, support_count=cnt, support_bits=bits)
    cert = torch.zeros(wl.batch, Hq, dtype=torch.int32, device=dev)
    Bd.ekv_exactness_certificate(seqs, wl.num_kv_heads, wl.page_size, alpha, ub, eng.sel, eng.n_sel, tau_last, cert)
    tok = ((bits.view(torch.int32).unsqueeze(-1) >> torch.arange(32, device=dev, dtype=torch.int32)) & 1)
    tok = tok.view(wl.batch, wl.num_kv_heads, wl.group, -1).amax(dim=2)          # union over the group
    page_sup = tok.view(wl.batch, wl.num_kv_heads, k, wl.page_size).amax(dim=-1)
    support_pages = int(page_sup.sum())
    support_tokens = int(tok.sum())
    nb = algorithmic_bytes(inp, eng, support_pages, support_tokens)

    # per-kernel rooflines from the staged timing; the headline one is the
    # kernel with the largest time (the launch list's largest share)
    peak, peak_kind = hbm_peak()
    kern = {}
    for name, idx, key, table, files in (("score", 1, "score_kernel", SCORE_TRAFFIC, SCORE_FILES),
                                         ("decode", 3, "decode_kernel", DECODE_TRAFFIC, DECODE_FILES)):
        ms = float(stages[idx])
        ach = nb[key] / (ms * 1e-3) / 1e9
        kern[name] = {"us": ms * 1e3, "algorithmic_bytes": nb[key], "achieved": ach, "frac": ach / peak,
                      "traffic": table.get(kernel_hash(files))}
    kern["topk"] = {"us": float(stages[2]) * 1e3, "bound": "latency (1 MiB of scores)"}
    kern["append"] = {"us": float(stages[0]) * 1e3, "bound": "latency (one page per unit)"}
    dom = max(("score", "decode"), key=lambda n: kern[n]["us"])
    dom_name = {"score": "score (bounding-box page scores)",
                "decode": "decode (fused: scores on selected K, tau, support V)"}[dom]
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": f"{wl.name}: batch {wl.batch}, {wl.num_q_heads} q / {wl.num_kv_heads} KV heads, "
                               f"d {wl.head_dim}, context {wl.context}, page size {wl.page_size}",
                   "policy": "topk", "k": k, "alpha": alpha, "global_batch": wl.batch * world,
                   "seq_len": wl.context, "parallelism": f"replicas x{world} (units sharded, no collective)",
                   "l2": "flushed between steps (256 MiB read)"},
        "steps_per_s": 1e3 / step_ms,
        "stages_us": {"append": stages[0] * 1e3, "score": stages[1] * 1e3, "topk": stages[2] * 1e3,
                      "decode": stages[3] * 1e3, "sum": float(stages.sum()) * 1e3,
                      "note": "separate calls with events between stages (no launch overlap)"},
        "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": kern[dom]["achieved"],
                     "peak": peak, "unit": "GB/s", "frac": kern[dom]["frac"],
                     "peak_kind": f"{peak_kind} copy bandwidth", "traffic": kern[dom]["traffic"],
                     "algorithmic_bytes": kern[dom]["algorithmic_bytes"]},
        "kernels": kern,
        "step_roofline": {"bytes": nb["step"], "achieved_gbs": nb["step"] / (step_ms * 1e-3) / 1e9,
                          "frac": nb["step"] / (step_ms * 1e-3) / 1e9 / peak,
                          "breakdown": {kk: v for kk, v in nb.items() if kk not in ("step", "score_kernel")}},
        "certificate": certificate_stats(cert, inp, wl, alpha, k),
        "support": {"mean_sel_pages": float(eng.n_sel.float().mean()), "support_pages_per_unit":
                    support_pages / wl.units, "mean_support_tokens_per_head": float(cnt.float().mean())},
        "gpu_launches": Bd.ekv_step_kernel_count(cache, seqs, eng.params, Hq) * args.steps,
        "clocks": clocks,
    }

    result["softmax_full_cache"] = bench_softmax(args, wl, inp, eng, dev, flush, peak, step_ms)
    if not args.quick:
        result["gauss"] = bench_policy(args, wl, inp, "gauss", dev, flush)
        result["full_cache"] = bench_policy(args, wl, inp, "full", dev, flush)
        result["full_cache_dense_v"] = bench_policy(args, wl, inp, "full", dev, flush, dense_v=True)
        result["e2e"] = bench_e2e(args, wl, inp, eng, dev, flush, world)
    if rank == 0 and world == 1 and not args.quick:
        result["cpu_baseline"] = cpu_baseline(wl, inp, k, alpha, budget_s=args.cpu_seconds)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def bench_policy(args, wl, inp, policy, dev, flush, dense_v=False):
    """Whole-step timing (one ekv_decode_step call) of another policy."""
    from sparse_kv_cache_kmax_b200.engine import DecodeEngine

    eng = DecodeEngine(inp["k_pool"], inp["v_pool"], inp["page_table"], inp["seq_lens"], wl.num_q_heads,
                       policy=policy, k=wl.topk, delta=wl.delta if wl.delta is not None else 0.5,
                       alpha=args.alpha, dense_v=dense_v)
    eng.build_meta()
    steps = max(3, min(args.steps, 200 if policy == "full" else args.steps))
    for _ in range(args.warmup):
        flush.zero_()
        eng.step(inp["q"], inp["k_new"][0], inp["v_new"][0])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        eng.step(inp["q"], inp["k_new"][0], inp["v_new"][0])
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    res = {"ms_per_step": ms, "value": wl.units / (ms * 1e-3), "unit": UNIT, "steps": steps,
           "mean_sel_pages": float(eng.n_sel.float().mean()) if policy != "full" else float(inp["max_pages"])}
    if policy == "full":
        es = inp["k_pool"].element_size()
        kv = sum(int(L) for L in inp["seq_lens"].tolist()) * wl.num_kv_heads * wl.head_dim * es
        res["k_bytes"] = kv
        res["dense_v"] = bool(dense_v)
    return res


def certificate_stats(cert, inp, wl, alpha, k):
    """Exactness certificate at the bench's budget, and the budget the doubling
    adaptive decode needs until every head is certified (untimed)."""
    from sparse_kv_cache_kmax_b200.engine import DecodeEngine
    eng = DecodeEngine(inp["k_pool"], inp["v_pool"], inp["page_table"], inp["seq_lens"], wl.num_q_heads,
                       policy="topk", k=k, alpha=alpha)
    eng.build_meta()
    _, k_needed = eng.decode_adaptive(inp["q"], k0=k)
    return {"certified_heads_frac_at_k": float(cert.float().mean()), "k": k,
            "adaptive_k_all_certified": int(k_needed)}


def bench_softmax(args, wl, inp, eng, dev, flush, peak, sparse_step_ms):
    """The full-cache softmax decode ([EntmaxKV] §4's baseline, split over
    pages) on the same cache: time, roofline on the K and V bytes it must read,
    and the sparse entmax step's speedup over it."""
    from sparse_kv_cache_kmax_b200 import binding as Bd
    if wl.dtype != "bf16":
        return {"unavailable": "bf16 caches only"}
    P = inp["max_pages"]
    out = torch.empty(wl.batch, wl.num_q_heads, wl.head_dim, device=dev)
    ws = Bd.workspace(Bd.ekv_workspace_bytes(Bd.EKV_OP_SOFTMAX_DECODE, eng.cache, eng.seqs, wl.num_q_heads, P), dev)
    scale = float(np.float32(wl.scale))
    steps = max(3, min(args.steps, 100))
    for _ in range(args.warmup):
        flush.zero_()
        Bd.ekv_softmax_decode(eng.cache, eng.seqs, inp["q"], scale, None, None, P, out, ws)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        Bd.ekv_softmax_decode(eng.cache, eng.seqs, inp["q"], scale, None, None, P, out, ws)
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    es = inp["k_pool"].element_size()
    tokens = sum(int(L) for L in inp["seq_lens"].tolist())
    nbytes = 2 * tokens * wl.num_kv_heads * wl.head_dim * es
    ach = nbytes / (ms * 1e-3) / 1e9
    return {"ms_per_step": ms, "value": wl.units / (ms * 1e-3), "unit": UNIT, "steps": steps,
            "algorithmic_bytes": nbytes, "achieved_gbs": ach, "frac": ach / peak,
            "sparse_entmax_step_speedup": ms / sparse_step_ms,
            "kernel": "softmax_split_kernel (all pages, K and V, split over pages)",
            "dropped_mass": dropped_mass(wl, inp, eng, dev, out, ws, scale)}


def dropped_mass(wl, inp, eng, dev, out_full_sm, ws_sm, scale):
    """Quality of the kept set (untimed; [EntmaxKV] §3–§4): under the same
    top-k pages, the softmax weight left outside them (1 − e^(lse_sel − lse_full))
    and its output error, against the entmax output error (zero whenever the
    kept pages hold the support).  Errors are per (sequence, query head) row:
    max_i |o_i − ô_i| / max_i |ô_i|."""
    from sparse_kv_cache_kmax_b200 import binding as Bd
    P, k, Hq = inp["max_pages"], eng.cap, wl.num_q_heads
    alpha = eng.params.alpha
    lse_full = torch.empty(wl.batch, Hq, device=dev)
    lse_sel = torch.empty(wl.batch, Hq, device=dev)
    out_sel = torch.empty_like(out_full_sm)
    Bd.ekv_softmax_decode(eng.cache, eng.seqs, inp["q"], scale, None, None, P, out_full_sm, ws_sm, lse=lse_full)
    ws_k = Bd.workspace(Bd.ekv_workspace_bytes(Bd.EKV_OP_SOFTMAX_DECODE, eng.cache, eng.seqs, Hq, k), dev)
    Bd.ekv_softmax_decode(eng.cache, eng.seqs, inp["q"], scale, eng.sel, eng.n_sel, k, out_sel, ws_k, lse=lse_sel)
    ent_full = torch.empty_like(out_full_sm)
    ent_sel = torch.empty_like(out_full_sm)
    ws_f = Bd.workspace(Bd.ekv_workspace_bytes(Bd.EKV_OP_ENTMAX_DECODE, eng.cache, eng.seqs, Hq, P), dev)
    Bd.ekv_entmax_decode(eng.cache, eng.seqs, inp["q"], scale, alpha, None, None, P, ent_full, ws_f)
    ws_s = Bd.workspace(Bd.ekv_workspace_bytes(Bd.EKV_OP_ENTMAX_DECODE, eng.cache, eng.seqs, Hq, k), dev)
    Bd.ekv_entmax_decode(eng.cache, eng.seqs, inp["q"], scale, alpha, eng.sel, eng.n_sel, k, ent_sel, ws_s)
    torch.cuda.synchronize()

    def rel(a, b):
        return ((a - b).abs().amax(-1) / b.abs().amax(-1).clamp_min(1e-6)).flatten()

    drop = (1.0 - torch.exp(lse_sel.double() - lse_full.double())).flatten()
    e_sm, e_ent = rel(out_sel, out_full_sm), rel(ent_sel, ent_full)
    return {"k": int(k), "softmax_dropped_mass_mean": float(drop.mean()), "softmax_dropped_mass_max": float(drop.max()),
            "softmax_rel_err_median": float(e_sm.median()), "softmax_rel_err_max": float(e_sm.max()),
            "entmax_rel_err_median": float(e_ent.median()), "entmax_rel_err_max": float(e_ent.max())}


def bench_e2e(args, wl, inp, eng, dev, flush, world):
    """Same step through the public one-call API with host buffers: pinned
    H2D of q, k_new, v_new, the step, and D2H of the output, per step."""
    q_h = inp["q"].cpu().pin_memory()
    k_h = inp["k_new"][0].cpu().pin_memory()
    v_h = inp["v_new"][0].cpu().pin_memory()
    out_h = torch.empty(eng.out.shape, dtype=eng.out.dtype).pin_memory()
    q_d, k_d, v_d = torch.empty_like(inp["q"]), torch.empty_like(inp["k_new"][0]), torch.empty_like(inp["v_new"][0])
    steps = max(3, min(args.steps, 500))

    def one():
        q_d.copy_(q_h, non_blocking=True)
        k_d.copy_(k_h, non_blocking=True)
        v_d.copy_(v_h, non_blocking=True)
        eng.step(q_d, k_d, v_d)
        out_h.copy_(eng.out, non_blocking=True)

    for _ in range(args.warmup):
        flush.zero_()
        one()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        one()
        ev[i][1].record()
    torch.cuda.synchronize()
    total = sum(a.elapsed_time(b) for a, b in ev) / 1e3
    max_s, units_all = reduce_timing(total, wl.units * steps)
    h2d = q_h.numel() * q_h.element_size() + 2 * k_h.numel() * k_h.element_size()
    d2h = out_h.numel() * out_h.element_size()
    return {"value": units_all / max_s, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": total / steps * 1e3, "steps": steps}


# ---------------------------------------------------------------- the oracle, timed
def oracle_step_units(wl, host_units, k, alpha, budget_s):
    """Run the oracle's decode step on host copies of some units until
    budget_s of CPU time is spent; returns (unit-steps done, seconds)."""
    import oracle as O

    scale = float(np.float32(wl.scale))
    done, t0 = 0, time.perf_counter()
    while True:
        for (kp, vp, n_valid, qg, meta) in host_units:
            # append: refresh the tail page's metadata
            last = len(n_valid) - 1
            tail = O.page_metadata(kp[last:last + 1], n_valid[last:last + 1], wl.dtype)
            for f in meta:
                meta[f][last] = tail[f][0]
            ub = O.bbox_upper_bound(qg, meta["kmax"], meta["kmin"], scale)
            sel = O.select_topk(O.page_scores(ub), k)
            Ks = np.concatenate([kp[p, : n_valid[p]] for p in sel])
            Vs = np.concatenate([vp[p, : n_valid[p]] for p in sel])
            O.entmax_attention(qg, Ks, Vs, scale, alpha)
            done += 1
            if time.perf_counter() - t0 >= budget_s:
                return done, time.perf_counter() - t0


def host_units_sample(wl, inp, n_units):
    import oracle as O

    units = []
    for u in range(n_units):
        b, h = divmod(u, wl.num_kv_heads)
        L = int(inp["seq_lens"][b])
        P = -(-L // wl.page_size)
        ids = inp["page_table"][b, :P].long()
        kp = inp["k_pool"][ids, h].double().cpu().numpy()
        vp = inp["v_pool"][ids, h].double().cpu().numpy()
        n_valid = np.minimum(wl.page_size, L - wl.page_size * np.arange(P))
        qg = inp["q"][b, h * wl.group:(h + 1) * wl.group].double().cpu().numpy()
        meta = O.page_metadata(kp, n_valid, wl.dtype)
        units.append((kp, vp, n_valid, qg, meta))
    return units


def cpu_baseline(wl, inp, k, alpha, budget_s=15.0):
    from threadpoolctl import threadpool_limits

    units = host_units_sample(wl, inp, 2)
    with threadpool_limits(1):
        done, secs = oracle_step_units(wl, units, k, alpha, budget_s)
    return {"value": done / secs, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"float64 numpy oracle, 1 thread: {done} unit-steps (append + scores + top-k + "
                      f"entmax attention) cycling over units 0-1 of {wl.name}, {secs:.1f} s"}


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    from sparse_kv_cache_kmax_b200.workloads import WORKLOADS, make_inputs, scaled_down

    world, rank, local = dist_env()
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    k = args.k or wl.topk
    # inputs are drawn on the host here (the reference arm needs no GPU); the
    # sampled units all live in sequence 0, so one sequence of the shape is drawn
    inp = make_inputs(scaled_down(args.workload, batch=1), seed=3000, device="cpu")
    units = host_units_sample(wl, inp, 2)
    from threadpoolctl import threadpool_limits

    # each step is a bounded sample of the workload: one unit-step of the
    # oracle (append, scores, top-k, entmax attention), cycling over the units
    import oracle as O  # noqa: F401  (the reference arm runs the oracle)

    done, secs = 0, 0.0
    with threadpool_limits(1):
        for i in range(args.warmup + args.steps):
            unit = [units[i % len(units)]]
            d, s_ = oracle_step_units(wl, unit, k, args.alpha, 0.0)
            if i >= args.warmup:
                done += d
                secs += s_
    value = done / secs
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / max(1, done) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name}: batch {wl.batch}, {wl.num_q_heads} q / {wl.num_kv_heads} KV heads, "
                               f"d {wl.head_dim}, context {wl.context}, page size {wl.page_size}",
                   "policy": "topk", "k": k, "alpha": args.alpha, "global_batch": wl.batch,
                   "seq_len": wl.context, "parallelism": "none (host oracle)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"float64 numpy oracle, 1 thread, one unit-step per step cycling "
                                   f"over units 0-1 of {wl.name}: {done} unit-steps in {secs:.1f} s"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))


# ---------------------------------------------------------------- kernel microbench
def run_kernel(args):
    """Launch one stage repeatedly on inputs of the workload's shape that only
    hold what that stage reads (a few hundred MB): the case ncu captures."""
    from sparse_kv_cache_kmax_b200 import binding as Bd
    from sparse_kv_cache_kmax_b200.workloads import WORKLOADS

    wl = WORKLOADS[args.workload]
    if args.shape:
        bb, hq, hkv = (int(x) for x in args.shape.split(","))
        wl = dataclasses.replace(wl, batch=bb, num_q_heads=hq, num_kv_heads=hkv)
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(11)
    B, Hkv, Hq, d, S = wl.batch, wl.num_kv_heads, wl.num_q_heads, wl.head_dim, wl.page_size
    P = wl.max_pages
    k = args.k or wl.topk
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    page_table = torch.arange(B * P, dtype=torch.int32, device=dev).view(B, P)
    seq_lens = torch.full((B,), wl.context, dtype=torch.int32, device=dev)
    q = torch.randn(B, Hq, d, generator=g, device=dev).to(dt)
    scale = float(np.float32(wl.scale))
    stream = torch.cuda.current_stream()
    if args.kernel == "copy":
        src = torch.empty(B * P * Hkv * 2 * d, dtype=dt, device=dev).normal_(generator=g)
        dst = torch.empty_like(src)

        def launch():
            dst.copy_(src)
        nbytes = 2 * src.numel() * src.element_size()
    elif args.kernel in ("score", "gauss", "topk"):
        kv = torch.empty(1, Hkv, S, d, dtype=dt, device=dev)          # never read by these stages
        lo = torch.randn(Hkv, B * P, 1, d, generator=g, device=dev)           # head-major [Hkv, pages, 2, d]
        box = torch.cat([lo + 0.5, lo - 0.5], dim=2).to(dt).contiguous()
        mom = torch.cat([lo, torch.rand(Hkv, B * P, 1, d, generator=g, device=dev)], dim=2).to(dt).contiguous()
        cache = Bd.make_cache(kv, kv, box, mom)
        cache.num_phys_pages = B * P
        seqs = Bd.make_seqs(page_table, seq_lens)
        ub = torch.randn(B, Hkv, P, generator=g, device=dev)
        sel = torch.zeros(B, Hkv, max(k, P), dtype=torch.int32, device=dev)
        n_sel = torch.zeros(B, Hkv, dtype=torch.int32, device=dev)
        tau_hat = torch.zeros(B, Hq, device=dev)
        n_tk = Bd.ekv_workspace_bytes(Bd.EKV_OP_SELECT_TOPK, cache, seqs, Hq, k)
        tk_ws = Bd.workspace(n_tk, dev) if n_tk else None
        gws = Bd.workspace(Bd.ekv_workspace_bytes(Bd.EKV_OP_SELECT_GAUSS, cache, seqs, Hq, P), dev)

        def launch():
            if args.kernel == "score":
                Bd.ekv_score_pages(cache, seqs, q, scale, ub, stream)
            elif args.kernel == "topk":
                Bd.ekv_select_topk(seqs, Hkv, S, ub, k, sel, n_sel, stream, ws=tk_ws)
            else:
                Bd.ekv_select_gauss(cache, seqs, q, scale, args.alpha, wl.delta or 0.5, P, sel, n_sel, tau_hat,
                                    gws, stream)
        nbytes = B * P * Hkv * 2 * d * box.element_size()
    else:  # decode: only the k selected pages of every unit exist in the pools
        kpool = torch.randn(B * k, Hkv, S, d, generator=g, device=dev).to(dt)
        vpool = torch.randn(B * k, Hkv, S, d, generator=g, device=dev).to(dt)
        meta = torch.empty(1, Hkv, 2, d, dtype=dt, device=dev)
        cache = Bd.make_cache(kpool, vpool, meta, meta)
        pt = torch.zeros(B, P, dtype=torch.int32, device=dev)
        pt[:, :k] = torch.arange(B * k, dtype=torch.int32, device=dev).view(B, k)
        seqs = Bd.make_seqs(pt, seq_lens)
        sel = torch.arange(k, dtype=torch.int32, device=dev).expand(B, Hkv, k).contiguous()
        n_sel = torch.full((B, Hkv), k, dtype=torch.int32, device=dev)
        out = torch.empty(B, Hq, d, device=dev)
        ws = Bd.workspace(Bd.ekv_workspace_bytes(Bd.EKV_OP_ENTMAX_DECODE, cache, seqs, Hq, k), dev)

        def launch():
            Bd.ekv_entmax_decode(cache, seqs, q, scale, args.alpha, sel, n_sel, k, out, ws, stream=stream)
        nbytes = B * Hkv * k * S * d * kpool.element_size()
    flush = L2Flush(dev)
    for _ in range(args.warmup):
        flush.zero_()
        launch()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record()
        launch()
        ev[i][1].record()
    torch.cuda.synchronize()
    us = float(np.mean([a.elapsed_time(b) for a, b in ev])) * 1e3
    print(json.dumps({"kernel": args.kernel, "workload": wl.name, "us": us, "bytes": nbytes,
                      "gbs": nbytes / (us * 1e-6) / 1e9}))


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="clustered_128k")
    p.add_argument("--alpha", type=float, default=1.5)
    p.add_argument("--k", type=int, default=0)
    p.add_argument("--cpu-seconds", type=float, default=15.0)
    p.add_argument("--quick", action="store_true", help="top-k step only (no other policies, e2e or CPU leg)")
    p.add_argument("--kernel", choices=["score", "gauss", "topk", "decode", "copy"],
                   help="time one stage alone on inputs holding only what it reads ('copy': a plain "
                        "device copy of the stage's bytes, for reference)")
    p.add_argument("--shape", default="", help="kernel mode: override 'batch,q_heads,kv_heads'")
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.kernel:
        run_kernel(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
