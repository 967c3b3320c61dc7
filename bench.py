"""Benchmark of the EntmaxKV support-aware paged α-entmax decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one decode token for every (sequence, KV head) unit of the
workload: cache append + tail-page metadata, bounding-box page scores, top-k
page selection, sparse α-entmax attention (scores over the selected K, τ,
support-only V), as one ekv_decode_step call.  Inputs are resident in HBM;
L2 is flushed (256 MiB read) between steps.  Prints one JSON line on rank 0.

Headline workload: the clustered 128k-context decode — batch 4, 32 query /
8 KV heads, d = 128, page size 16, bf16 cache, top-k k = 256, α = 1.5.  The
default run adds the Gaussian policy and the full-cache decodes on the same
cache, the end-to-end figure through host buffers, every other workload of
the set (``workloads``) and the float64 oracle timed on the host
(``cpu_baseline``); ``--quick`` keeps the headline line only.
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
import tempfile
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
kHostLead = 100_000  # device cycles (~50 µs) of delay before each staged stage

# dram__bytes_read.sum + dram__bytes_write.sum per launch from one ncu capture
# of the clustered 128k shape, keyed by a hash of the kernel's sources (a
# changed kernel has no measured traffic until it is captured again)
SCORE_FILES = ("score.cu", "common.cuh")
DECODE_FILES = ("decode_fused.cu", "decode.cuh", "common.cuh")
SCORE_TRAFFIC = {"d6a06f8bdcde3139": 134715392}
DECODE_TRAFFIC = {"546c3d7b8f786b33": 35236864}


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
        self.path = os.path.join(tempfile.gettempdir(), f"ekv_clocks_{os.getpid()}_{id(self)}.csv")

    def __enter__(self):
        try:
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
def step_bytes(inp, policy, n_sel, support_pages, support_tokens):
    """Bytes one step must move, and each kernel's share (per-unit bytes ×
    the units of the step): the metadata rows the
    selection reads (box for top-k, mean/var for the Gaussian policy; none
    for the full cache), q, the page scores, the selected K, the V rows of the
    support (token by token for the decode kernel, as the method needs them;
    page by page for the step, the pages that hold support), the output and
    the append (tail page + new rows + its metadata rows)."""
    wl = inp["workload"]
    es = inp["k_pool"].element_size()
    d, S = wl.head_dim, wl.page_size
    pages = sum(-(-int(L) // S) for L in inp["seq_lens"].tolist()) * wl.num_kv_heads
    meta = 0 if policy == "full" else pages * 2 * d * es
    q = wl.batch * wl.num_q_heads * d * es
    ub = pages * 4 if policy == "topk" else 0
    sel_k = int(n_sel) * S * d * es
    sup_v_pages = int(support_pages) * S * d * es
    sup_v_tok = int(support_tokens) * d * es
    out = wl.batch * wl.num_q_heads * d * 4
    append = wl.units * (S * d * es + 2 * d * es + 4 * d * es)
    return {"meta": meta, "q": q, "ub": ub, "sel_k": sel_k, "support_v": sup_v_pages, "out": out,
            "append": append, "select_kernel": meta + q + ub,
            "decode_kernel": sel_k + sup_v_tok + q + out,
            "step": meta + q + sel_k + sup_v_pages + out + append}


# ---------------------------------------------------------------- one timed line
class Line:
    """One workload × policy × α through the library, timed the way the
    headline is: whole steps (one ekv_decode_step call each, L2 flushed
    between steps) and a staged breakdown (the same kernels as separate calls
    with events between them)."""

    def __init__(self, wl, inp, policy, alpha, dev, flush, *, k=None, delta=None, cap=None, dense_v=False):
        from sparse_kv_cache_kmax_b200 import binding as Bd
        from sparse_kv_cache_kmax_b200.engine import DecodeEngine
        from sparse_kv_cache_kmax_b200.workloads import gauss_cap

        self.Bd, self.wl, self.inp, self.policy, self.alpha = Bd, wl, inp, policy, alpha
        self.dev, self.flush = dev, flush
        if policy == "gauss" and cap is None:
            cap = gauss_cap(wl, inp["max_pages"])
        self.eng = DecodeEngine(inp["k_pool"], inp["v_pool"], inp["page_table"], inp["seq_lens"], wl.num_q_heads,
                                policy=policy, k=k, delta=delta, alpha=alpha, cap=cap, dense_v=dense_v)
        self.eng.build_meta()
        self.k, self.delta, self.cap, self.dense_v = k, delta, self.eng.cap, dense_v
        self.scale = float(np.float32(wl.scale))
        self.q, self.k_new, self.v_new = inp["q"], inp["k_new"][0], inp["v_new"][0]
        e, Hq = self.eng, wl.num_q_heads
        self.ub = torch.empty(wl.batch, wl.num_kv_heads, inp["max_pages"], device=dev)
        self.dec_ws = Bd.workspace(Bd.ekv_workspace_bytes(Bd.EKV_OP_ENTMAX_DECODE, e.cache, e.seqs, Hq, self.cap), dev)
        n_tk = Bd.ekv_workspace_bytes(Bd.EKV_OP_SELECT_TOPK, e.cache, e.seqs, Hq, k or 1) if policy == "topk" else 0
        self.tk_ws = Bd.workspace(n_tk, dev) if n_tk else None
        self.g_ws = (Bd.workspace(Bd.ekv_workspace_bytes(Bd.EKV_OP_SELECT_GAUSS, e.cache, e.seqs, Hq, self.cap), dev)
                     if policy == "gauss" else None)
        self.tau_hat = torch.empty(wl.batch, Hq, device=dev)
        self.stream = torch.cuda.current_stream()

    # one whole step: the public one-call API
    def step(self, ev):
        ev[0].record(self.stream)
        self.eng.step(self.q, self.k_new, self.v_new, self.stream)
        ev[1].record(self.stream)

    # the same kernels as separate calls: append | selection | decode.  Each
    # stage's events bracket only its own launches: a short device-side delay
    # (no memory traffic) runs first, so the host has queued the stage's
    # launches before the device reaches its start event, and the time
    # between the events is the kernels' own device time, not the host's
    # call overhead.
    def staged(self, ev):
        Bd, e, st, wl = self.Bd, self.eng, self.stream, self.wl
        hold = lambda: torch.cuda._sleep(kHostLead)
        hold()
        ev[0].record(st)
        Bd.ekv_append(e.cache, e.seqs, self.k_new, self.v_new, st)
        ev[1].record(st)
        if self.policy == "topk":
            hold()
            ev[2].record(st)
            Bd.ekv_score_pages(e.cache, e.seqs, self.q, self.scale, self.ub, st)
            ev[3].record(st)
            hold()
            ev[4].record(st)
            Bd.ekv_select_topk(e.seqs, wl.num_kv_heads, wl.page_size, self.ub, self.k, e.sel, e.n_sel, st,
                               ws=self.tk_ws)
            ev[5].record(st)
        elif self.policy == "gauss":
            hold()
            ev[2].record(st)
            Bd.ekv_select_gauss(e.cache, e.seqs, self.q, self.scale, self.alpha, self.delta, self.cap, e.sel, e.n_sel,
                                self.tau_hat, self.g_ws, st)
            ev[3].record(st)
            ev[4].record(st)
            ev[5].record(st)
        else:
            for i in (2, 3, 4, 5):
                ev[i].record(st)
        hold()
        ev[6].record(st)
        full = self.policy == "full"
        Bd.ekv_entmax_decode(e.cache, e.seqs, self.q, self.scale, self.alpha, None if full else e.sel,
                             None if full else e.n_sel, self.cap, e.out, self.dec_ws, dense_v=self.dense_v, stream=st)
        ev[7].record(st)

    def timed(self, fn, n_events, steps, warmup, world=1, pairs=False):
        for _ in range(warmup):
            self.flush.zero_()
            fn([torch.cuda.Event(enable_timing=True) for _ in range(n_events)])
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_events)] for _ in range(steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            self.flush.zero_()
            fn(evs[i])
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        if pairs:  # events (0,1), (2,3), …: one interval per stage
            return np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(0, n_events, 2)]
                             for i in range(steps)])
        return np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(n_events - 1)] for i in range(steps)])

    def support(self):
        """Support of the last step's selection (untimed): pages and tokens
        whose V a step reads (union over each unit's query heads)."""
        Bd, e, wl = self.Bd, self.eng, self.wl
        Hq, S = wl.num_q_heads, wl.page_size
        full = self.policy == "full"
        words = (self.cap * S + 31) // 32
        bits = torch.zeros(wl.batch, Hq, words, dtype=torch.int32, device=self.dev)
        cnt = torch.zeros(wl.batch, Hq, dtype=torch.int32, device=self.dev)
        tau = torch.zeros(wl.batch, Hq, device=self.dev)
        Bd.ekv_entmax_decode(e.cache, e.seqs, self.q, self.scale, self.alpha, None if full else e.sel,
                             None if full else e.n_sel, self.cap, e.out, self.dec_ws, tau=tau, support_count=cnt,
                             support_bits=bits)
        tok = (bits.unsqueeze(-1) >> torch.arange(32, device=self.dev, dtype=torch.int32)) & 1
        tok = tok.view(wl.batch, wl.num_kv_heads, wl.group, -1).amax(dim=2)
        page_sup = tok[..., : self.cap * S].reshape(wl.batch, wl.num_kv_heads, self.cap, S).amax(dim=-1)
        if full:
            n_sel = sum(-(-int(L) // S) for L in self.inp["seq_lens"].tolist()) * wl.num_kv_heads
        else:
            n_sel = int(e.n_sel.sum())
        return {"n_sel": n_sel, "support_pages": int(page_sup.sum()), "support_tokens": int(tok.sum()),
                "mean_support_tokens_per_head": float(cnt.float().mean()), "tau": tau}

    def measure(self, steps, warmup, peak, world=1, uuid=None):
        with ClockSampler(uuid) as clk:
            per_step = self.timed(self.step, 2, steps, warmup, world)[:, 0]
        clocks = clk.summary()
        staged = self.timed(self.staged, 8, max(3, min(steps, 200)), warmup, pairs=True).mean(axis=0)
        sup = self.support()
        nb = step_bytes(self.inp, self.policy, sup["n_sel"], sup["support_pages"], sup["support_tokens"])
        step_ms = float(per_step.mean())
        sel_name = {"topk": "score", "gauss": "gauss_select", "full": None}[self.policy]
        kern = {"append": {"us": float(staged[0]) * 1e3, "bound": "latency (one page per unit)"}}
        if self.policy == "topk":
            kern["score"] = {"us": float(staged[1]) * 1e3}
            kern["topk"] = {"us": float(staged[2]) * 1e3, "bound": "latency (scores from L2)"}
        elif self.policy == "gauss":
            kern["gauss_select"] = {"us": float(staged[1]) * 1e3,
                                    "note": "page statistics + tau-hat + filter (three kernels)"}
        kern["decode"] = {"us": float(staged[3]) * 1e3}
        for name, key in ((sel_name, "select_kernel"), ("decode", "decode_kernel")):
            if name is None:
                continue
            us = kern[name]["us"]
            ach = nb[key] / (us * 1e-6) / 1e9
            kern[name].update({"algorithmic_bytes": nb[key], "achieved": ach, "frac": ach / peak})
        dom = max((n for n in (sel_name, "decode") if n), key=lambda n: kern[n]["us"])
        return {
            "ms_per_step": step_ms, "value": self.wl.units / (step_ms * 1e-3), "unit": UNIT, "steps": int(steps),
            "total_s": float(per_step.sum()) / 1e3,
            "stages_us": {"append": staged[0] * 1e3, "select": (staged[1] + staged[2]) * 1e3,
                          "decode": staged[3] * 1e3, "sum": float(staged.sum()) * 1e3},
            "kernels": kern, "dominant": dom,
            "step_roofline": {"bytes": nb["step"], "achieved_gbs": nb["step"] / (step_ms * 1e-3) / 1e9,
                              "frac": nb["step"] / (step_ms * 1e-3) / 1e9 / peak,
                              "breakdown": {kk: v for kk, v in nb.items() if kk not in ("step",)}},
            "support": {"mean_sel_pages": sup["n_sel"] / self.wl.units,
                        "support_pages_per_unit": sup["support_pages"] / self.wl.units,
                        "mean_support_tokens_per_head": sup["mean_support_tokens_per_head"]},
            "clocks": clocks, "tau": sup["tau"],
        }


def short_line(m):
    """The fields of a secondary line in the JSON (no tensors)."""
    dom = m["dominant"]
    return {"ms_per_step": m["ms_per_step"], "value": m["value"], "unit": m["unit"], "steps": m["steps"],
            "step_frac": m["step_roofline"]["frac"], "dominant_kernel": dom,
            "dominant_frac": m["kernels"][dom].get("frac"),
            "kernels_us": {n: v["us"] for n, v in m["kernels"].items()},
            "mean_sel_pages": m["support"]["mean_sel_pages"], "clocks": m["clocks"]}


# ---------------------------------------------------------------- our arm
def run_ours(args):
    from sparse_kv_cache_kmax_b200 import binding as Bd
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

    # the oracle's host threads start before any GPU work
    cpu_pool = None
    if rank == 0 and world == 1 and not args.quick:
        from concurrent.futures import ThreadPoolExecutor
        cpu_pool = ThreadPoolExecutor(max_workers=cpu_threads())

    wl = WORKLOADS[args.workload]
    inp = make_inputs(wl, seed=3000 + rank, device=dev, n_new=1)
    alpha, k = args.alpha, args.k or wl.topk
    flush = L2Flush(dev)
    peak, peak_kind = hbm_peak()
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        uuid = None

    line = Line(wl, inp, "topk", alpha, dev, flush, k=k)
    m = line.measure(args.steps, args.warmup, peak, world, uuid)
    max_s, units_all = reduce_timing(m["total_s"], wl.units * args.steps)
    value = units_all / max_s
    eng = line.eng
    kern = m["kernels"]
    dom = m["dominant"]
    files = {"score": SCORE_FILES, "decode": DECODE_FILES}
    tables = {"score": SCORE_TRAFFIC, "decode": DECODE_TRAFFIC}
    for name in ("score", "decode"):
        kern[name]["traffic"] = tables[name].get(kernel_hash(files[name]))
    dom_name = {"score": "score (bounding-box page scores)",
                "decode": "decode (scores on the selected K, tau, support V: one launch)"}[dom]
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": f"{wl.name}: batch {wl.batch}, {wl.num_q_heads} q / {wl.num_kv_heads} KV heads, "
                               f"d {wl.head_dim}, context {wl.context}, page size {wl.page_size}",
                   "policy": "topk", "k": k, "alpha": alpha, "global_batch": wl.batch * world,
                   "seq_len": wl.context, "parallelism": f"replicas x{world} (units sharded, no collective)",
                   "l2": "flushed between steps (256 MiB read)"},
        "steps_per_s": 1e3 / m["ms_per_step"],
        "stages_us": dict(m["stages_us"], note="separate calls, each bracketed by its own events after a "
                                               "device-side delay that lets the host queue it (no launch overlap)"),
        "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": kern[dom]["achieved"],
                     "peak": peak, "unit": "GB/s", "frac": kern[dom]["frac"],
                     "peak_kind": f"{peak_kind} copy bandwidth", "traffic": kern[dom]["traffic"],
                     "algorithmic_bytes": kern[dom]["algorithmic_bytes"]},
        "kernels": kern,
        "step_roofline": m["step_roofline"],
        "support": m["support"],
        "gpu_launches": Bd.ekv_step_kernel_count(eng.cache, eng.seqs, eng.params, wl.num_q_heads) * args.steps,
        "clocks": m["clocks"],
    }
    cert = torch.zeros(wl.batch, wl.num_q_heads, dtype=torch.int32, device=dev)
    Bd.ekv_score_pages(eng.cache, eng.seqs, inp["q"], line.scale, line.ub)
    Bd.ekv_exactness_certificate(eng.seqs, wl.num_kv_heads, wl.page_size, alpha, line.ub, eng.sel, eng.n_sel,
                                 m["tau"], cert)
    result["certificate"] = certificate_stats(cert, inp, wl, alpha, k)
    result["softmax_full_cache"] = bench_softmax(args, wl, inp, eng, dev, flush, peak, m["ms_per_step"])
    dm = result["softmax_full_cache"].get("dropped_mass", {})
    result["headline_exactness"] = {
        "certified_heads_frac": result["certificate"]["certified_heads_frac_at_k"],
        "entmax_rel_err_vs_full_cache_median": dm.get("entmax_rel_err_median"),
        "entmax_rel_err_vs_full_cache_max": dm.get("entmax_rel_err_max"),
        "note": "top-k k keeps a fixed budget: heads whose support reaches past the kept pages differ from "
                "the full-cache output; the adaptive budget and the Gaussian policy are the exact-output points"}
    if not args.quick:
        g = Line(wl, inp, "gauss", alpha, dev, flush, delta=wl.delta if wl.delta is not None else 0.5)
        gm = g.measure(max(3, min(args.steps, 200)), args.warmup, peak)
        result["gauss"] = dict(short_line(gm), delta=g.delta, cap=g.cap, stages_us=gm["stages_us"],
                               support=gm["support"])
        del g
        for key, dense in (("full_cache", False), ("full_cache_dense_v", True)):
            f = Line(wl, inp, "full", alpha, dev, flush, dense_v=dense)
            fm = f.measure(max(3, min(args.steps, 100)), args.warmup, peak)
            kb = sum(int(L) for L in inp["seq_lens"].tolist()) * wl.num_kv_heads * wl.head_dim * \
                inp["k_pool"].element_size()
            nbytes = kb * (2 if dense else 1) + (0 if dense else fm["step_roofline"]["breakdown"]["support_v"])
            result[key] = dict(short_line(fm), dense_v=dense, k_bytes=kb, algorithmic_bytes=nbytes,
                               achieved_gbs=nbytes / (fm["kernels"]["decode"]["us"] * 1e-6) / 1e9,
                               frac=nbytes / (fm["kernels"]["decode"]["us"] * 1e-6) / 1e9 / peak)
            del f
        result["e2e"] = bench_e2e(args, wl, inp, eng, dev, flush, world)
        if world == 1:
            result["workloads"] = other_workloads(args, wl, dev, flush, peak, uuid)
    if cpu_pool is not None:
        result["cpu_baseline"] = cpu_baseline(wl, inp, k, alpha, cpu_pool, budget_s=args.cpu_seconds)
        cpu_pool.shutdown()
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def run_line(args):
    """One line of the default run alone (one policy on one workload), on the
    workload's own inputs: the command the per-line ncu summaries use."""
    from sparse_kv_cache_kmax_b200 import binding as Bd
    from sparse_kv_cache_kmax_b200.workloads import WORKLOADS, make_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    Bd.lib()
    wl = WORKLOADS[args.workload]
    inp = make_inputs(wl, seed=3000, device=dev, n_new=1)
    flush = L2Flush(dev)
    peak, _ = hbm_peak()
    policy = {"topk": "topk", "gauss": "gauss", "full": "full", "dense": "full"}[args.line]
    kw = {"k": args.k or wl.topk} if policy == "topk" else (
        {"delta": wl.delta if wl.delta is not None else 0.5} if policy == "gauss" else {"dense_v": args.line == "dense"})
    ln = Line(wl, inp, policy, args.alpha, dev, flush, **kw)
    m = ln.measure(args.steps, args.warmup, peak)
    print(json.dumps(dict(short_line(m), line=args.line, workload=wl.name, alpha=args.alpha)))


# (workload, policy, alpha, budget) of the other lines in the default run
OTHER_LINES = [
    ("clustered_128k", "topk", 1.25, None),
    ("clustered_128k", "topk", 2.0, None),
    ("gqa_32k", "topk", 1.5, None),
    ("short_scattered", "topk", 1.5, None),
    ("long_512k", "topk", 1.5, None),
    ("long_512k", "gauss", 1.5, None),
    ("ctx_1m", "topk", 1.5, None),
    ("ctx_1m", "gauss", 1.5, None),
]


def other_workloads(args, head_wl, dev, flush, peak, uuid):
    """Every other configuration of the workload set, one line each, measured
    the way the headline is (whole steps, L2 flushed, staged breakdown)."""
    from sparse_kv_cache_kmax_b200.workloads import WORKLOADS, make_inputs

    out, cur, inp = {}, None, None
    for name, policy, alpha, _ in OTHER_LINES:
        wl = WORKLOADS[name]
        if name != cur:
            inp = None
            torch.cuda.empty_cache()
            inp = make_inputs(wl, seed=3000, device=dev, n_new=1)
            cur = name
        kw = {"k": wl.topk} if policy == "topk" else {"delta": wl.delta}
        ln = Line(wl, inp, policy, alpha, dev, flush, **kw)
        mm = ln.measure(max(3, min(args.steps, 200)), args.warmup, peak, 1, uuid)
        key = f"{name}/{policy}" + (f" k={wl.topk}" if policy == "topk" else f" delta={wl.delta}") + f"/alpha={alpha}"
        out[key] = short_line(mm)
        del ln
    torch.cuda.empty_cache()
    return out


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
            "entmax_rel_err_median": float(e_ent.median()), "entmax_rel_err_max": float(e_ent.max()),
            "entmax_heads_exact_frac": float((e_ent <= 1e-5).float().mean())}


def bench_e2e(args, wl, inp, eng, dev, flush, world):
    """Same step through the public one-call API with host buffers: the
    step's inputs (q, k_new, v_new) staged in one pinned host buffer and
    copied to the device in one H2D copy, the step, and the D2H copy of the
    output, every step."""
    parts = [inp["q"], inp["k_new"][0], inp["v_new"][0]]
    sizes = [t.numel() for t in parts]
    stage_h = torch.cat([t.reshape(-1) for t in parts]).cpu().pin_memory()
    stage_d = torch.empty_like(stage_h, device=dev)
    offs = [0, sizes[0], sizes[0] + sizes[1]]
    q_d, k_d, v_d = (stage_d[o:o + n].view(t.shape) for o, n, t in zip(offs, sizes, parts))
    out_h = torch.empty(eng.out.shape, dtype=eng.out.dtype).pin_memory()
    steps = max(3, min(args.steps, 500))

    def one():
        stage_d.copy_(stage_h, non_blocking=True)
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
    h2d = stage_h.numel() * stage_h.element_size()
    d2h = out_h.numel() * out_h.element_size()
    return {"value": units_all / max_s, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": total / steps * 1e3, "steps": steps}


# ---------------------------------------------------------------- the oracle, timed
def cpu_threads():
    """Host threads of the oracle's timed leg: one per core, at most 32 (each
    holds its own copy of a unit's metadata)."""
    return max(1, min(os.cpu_count() or 1, 32))


def oracle_step_units(wl, host_units, k, alpha, budget_s, meta=None):
    """Run the oracle's decode step on host copies of some units until
    budget_s of time is spent (at least one unit-step); returns (unit-steps
    done, seconds).  meta: per-unit metadata dicts this caller owns (the
    append refreshes their tail page)."""
    import oracle as O

    scale = float(np.float32(wl.scale))
    done, t0 = 0, time.perf_counter()
    while True:
        for i, (kp, vp, n_valid, qg, meta0) in enumerate(host_units):
            md = meta0 if meta is None else meta[i]
            # append: refresh the tail page's metadata
            last = len(n_valid) - 1
            tail = O.page_metadata(kp[last:last + 1], n_valid[last:last + 1], wl.dtype)
            for f in md:
                md[f][last] = tail[f][0]
            ub = O.bbox_upper_bound(qg, md["kmax"], md["kmin"], scale)
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


def oracle_threaded(wl, units, k, alpha, pool, n_threads, budget_s):
    """The oracle on n_threads host threads at once, each cycling over the
    sampled units with its own metadata copies, for budget_s; returns
    (unit-steps, wall seconds)."""
    metas = [[{f: a.copy() for f, a in u[4].items()} for u in units] for _ in range(n_threads)]
    t0 = time.perf_counter()
    futs = [pool.submit(oracle_step_units, wl, units[i % len(units):] + units[:i % len(units)], k, alpha, budget_s,
                        metas[i][i % len(units):] + metas[i][:i % len(units)]) for i in range(n_threads)]
    done = sum(f.result()[0] for f in futs)
    return done, time.perf_counter() - t0


def cpu_baseline(wl, inp, k, alpha, pool, budget_s=15.0):
    """The oracle as it stands, timed on this host: every thread of the pool
    at once, and one thread alone (BLAS limited to one thread per worker)."""
    from threadpoolctl import threadpool_limits

    n_threads = pool._max_workers
    units = host_units_sample(wl, inp, min(8, wl.units))
    with threadpool_limits(1):
        done_n, secs_n = oracle_threaded(wl, units, k, alpha, pool, n_threads, budget_s)
        done_1, secs_1 = oracle_step_units(wl, units[:1], k, alpha, budget_s / 2)
    return {"value": done_n / secs_n, "unit": UNIT, "cores": n_threads, "kind": "oracle",
            "host_cores": os.cpu_count(),
            "sample": f"float64 numpy oracle on {n_threads} host threads at once (one BLAS thread each): "
                      f"{done_n} unit-steps (append + scores + top-k + entmax attention) cycling over units "
                      f"0-{len(units) - 1} of {wl.name}, {secs_n:.1f} s wall",
            "single_thread": {"value": done_1 / secs_1, "cores": 1,
                              "sample": f"{done_1} unit-steps of unit 0 in {secs_1:.1f} s"}}


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    from concurrent.futures import ThreadPoolExecutor

    from threadpoolctl import threadpool_limits

    from sparse_kv_cache_kmax_b200.workloads import WORKLOADS, make_inputs, scaled_down

    world, rank, local = dist_env()
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    k = args.k or wl.topk
    n_threads = cpu_threads()
    pool = ThreadPoolExecutor(max_workers=n_threads)
    # inputs are drawn on the host here (the reference arm needs no GPU); the
    # sampled units live in the first sequences, so only those are drawn
    n_units = min(8, wl.units)
    nb = -(-n_units // wl.num_kv_heads)
    inp = make_inputs(scaled_down(args.workload, batch=nb), seed=3000, device="cpu")
    units = host_units_sample(wl, inp, n_units)
    import oracle as O  # noqa: F401  (the reference arm runs the oracle)

    # each step is a bounded sample of the workload: one unit-step of the
    # oracle (append, scores, top-k, entmax attention) on every host thread
    done, secs = 0, 0.0
    metas = [[{f: a.copy() for f, a in u[4].items()} for u in units] for _ in range(n_threads)]
    with threadpool_limits(1):
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            futs = [pool.submit(oracle_step_units, wl, [units[(i + j) % n_units]], k, args.alpha, 0.0,
                                [metas[j][(i + j) % n_units]]) for j in range(n_threads)]
            d = sum(f.result()[0] for f in futs)
            if i >= args.warmup:
                done += d
                secs += time.perf_counter() - t0
    pool.shutdown()
    value = done / secs
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name}: batch {wl.batch}, {wl.num_q_heads} q / {wl.num_kv_heads} KV heads, "
                               f"d {wl.head_dim}, context {wl.context}, page size {wl.page_size}",
                   "policy": "topk", "k": k, "alpha": args.alpha, "global_batch": wl.batch,
                   "seq_len": wl.context, "parallelism": f"none (host oracle, {n_threads} threads)",
                   "l2": "not applicable (host)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": n_threads, "kind": "oracle",
                         "sample": f"float64 numpy oracle, {n_threads} host threads, one unit-step per thread per "
                                   f"step over units 0-{n_units - 1} of {wl.name}: {done} unit-steps in "
                                   f"{secs:.1f} s"},
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
    p.add_argument("--line", choices=["topk", "gauss", "full", "dense"],
                   help="run one line of the default output alone: this policy on --workload")
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.kernel:
        run_kernel(args)
    elif args.line:
        run_line(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
