"""Benchmark of the complete sparse-prefill call: page-affinity grouping followed by
union attention, on one seeded synthetic prefill chunk per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4b] [--impl reference]

A step = qup_sparse_group + qup_sparse_prefill_attn over the whole chunk (inputs
resident in HBM). Each timed step is bracketed by CUDA events on the launching
stream; an untimed write of a buffer twice the L2 size precedes every timed step.
Under torchrun every rank runs its own independent chunk (weak scaling, no data
collective); the timed region is bracketed by a barrier and the max over ranks
is reported.

Metric: selected-edge TFLOP/s = 4 * d * E / t, E = (query head, token) pairs
inside each query's own causal support (union padding and masked slots are not
counted). The JSON line also carries us/call of each kernel, unique-KV GB/s,
logical page visits and masked slots, the roofline of the attention kernel,
the fp64 CPU oracle timed on a bounded sample, and an end-to-end number through
host buffers.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from query_union_paged_b200 import workloads as W  # noqa: E402

METRIC = "selected-edge TFLOP/s of the complete sparse-prefill call (group + union attention)"
CONFIG_DEFAULT = "4b"


# ------------------------------------------------------------------ workload accounting

def selected_edges_per_row(w, topk=None) -> np.ndarray:
    """|A_i| for every (Q head, query): tokens of the row's distinct pages with t < kv_len, t <= q_pos."""
    topk = w.topk if topk is None else topk
    Hq, Nq, K = topk.shape
    E = np.zeros((Hq, Nq), np.int64)
    srt = np.sort(topk, axis=2)
    first = np.ones_like(srt, dtype=bool)
    first[:, :, 1:] = srt[:, :, 1:] != srt[:, :, :-1]
    valid = first & (srt >= 0)
    start = srt.astype(np.int64) * w.T
    hi = np.minimum(np.minimum(start + w.T, w.kv_len), w.q_pos[None, :, None].astype(np.int64) + 1)
    cnt = np.clip(hi - start, 0, None)
    E = np.where(valid, cnt, 0).sum(axis=2)
    return E


def unique_kv_pages(w) -> int:
    g = w.Hq // w.Hkv
    n = 0
    for h in range(w.Hkv):
        rows = w.topk[h * g:(h + 1) * g].reshape(-1)
        n += np.unique(rows[rows >= 0]).size
    return n


def union_topk(w, groups) -> np.ndarray:
    """[Hq][Nq][Kmax] TopK rows holding each query's group union (host copy of the groups)."""
    n_groups = groups.n_groups.cpu().numpy()
    gp_all, up_all = groups.group_ptr.cpu().numpy(), groups.union_ptr.cpu().numpy()
    members, pages = groups.members.cpu().numpy(), groups.union_pages.cpu().numpy()
    g = w.Hq // w.Hkv
    kmax = max(1, max(int(np.diff(up_all[h, :n_groups[h] + 1]).max(initial=0)) for h in range(w.Hkv)))
    out = np.full((w.Hq, w.Nq, kmax), -1, np.int32)
    for h in range(w.Hkv):
        gp, up = gp_all[h], up_all[h]
        for k in range(int(n_groups[h])):
            u = pages[up[k]:up[k + 1]]
            for m in members[h, gp[k]:gp[k + 1]]:
                out[h * g:(h + 1) * g, m, :u.size] = u
    return out


# ------------------------------------------------------------------ ranks

def max_over_ranks(total_ms: float, world: int, device) -> float:
    """The slowest rank's device time (every rank calls this, in the same order)."""
    if world <= 1:
        return total_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([total_ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flop_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processed its own chunk in the slowest rank's time."""
    return world * flop_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ environment helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _code_only(src: str) -> str:
    """Source text without // comments and blank lines: what the compiler turns into the kernel."""
    lines = []
    for line in src.splitlines():
        code = re.sub(r"//.*$", "", line).rstrip()
        if code.strip():
            lines.append(code)
    return "\n".join(lines)


def kernel_source_hash() -> str:
    """Hash of the attention kernel's code (comments excluded): a recorded ncu capture counts only
    while it matches."""
    h = hashlib.sha256()
    for name in ("union_attn.cu", "ptx.cuh", "internal.h"):
        with open(os.path.join(ROOT, "query_union_paged_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload_name: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "union_attn_traffic.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    src = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", txt)
    if not src or src.group(1) != kernel_source_hash():
        return None
    m = re.search(rf"^\|\s*{re.escape(workload_name)}\s*\|\s*([0-9.e+]+)\s*\|", txt, re.M)
    return float(m.group(1)) if m else None


# kernels of one step: the fused grouping kernel, the fused bundling kernel (which also orders
# the bundles), union attention (a memset of the look-back status words precedes them); union
# support adds its mask rewrite and the bundle rebuild (bitset and bundling kernels)
LAUNCHES_PER_STEP = 3
LAUNCHES_UNION_SUPPORT = 3


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples taken during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle leg

def oracle_sample(w, target_s: float = 12.0, seed: int = 0):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload's rows.

    Returns (TFLOP/s over the sample's selected edges, threads, description).
    """
    import oracle
    E = selected_edges_per_row(w)
    rng = np.random.default_rng(seed)
    order = rng.permutation(w.Hq * w.Nq)
    threads = os.cpu_count() or 1
    # calibrate on a small slice, then size the sample for ~target_s
    n0 = min(order.size, 64 * threads)
    rows = np.sort(order[:n0]).astype(np.int64)
    t0 = time.perf_counter()
    oracle.sparse_attn_workload(w, rows=rows, nthreads=threads)
    dt0 = max(time.perf_counter() - t0, 1e-3)
    n = int(min(order.size, max(n0, n0 * target_s / dt0)))
    rows = np.sort(order[:n]).astype(np.int64)
    t0 = time.perf_counter()
    oracle.sparse_attn_workload(w, rows=rows, nthreads=threads)
    dt = time.perf_counter() - t0
    edges = int(E.reshape(-1)[rows].sum())
    tflops = 4.0 * w.d * edges / dt / 1e12
    return tflops, threads, f"{n} of {w.Hq * w.Nq} (query head, query) rows, {edges} selected edges, {dt:.1f} s"


def group_reference_sample(w, max_group: int, window: int, repeats: int = 3):
    """Time the CPU grouping reference (oracle.group, plain C) on the whole workload: one thread,
    and one call per query window spread over a thread pool (groups never cross a window, so the
    windows are independent calls; ctypes releases the GIL during each).  Median of `repeats`.
    The counters of the windowed calls are checked against the single call's."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    topk = np.ascontiguousarray(w.topk)
    starts = list(range(0, w.Nq, window))
    slices = [np.ascontiguousarray(topk[:, a:a + window, :]) for a in starts]
    threads = os.cpu_count() or 1

    def one():
        return oracle.group(topk, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, max_group, window)

    def windowed(pool):
        return list(pool.map(lambda t: oracle.group(t, w.Hq, w.Hkv, t.shape[1], w.num_logical_pages,
                                                     max_group, window), slices))

    t1 = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        ref = one()
        t1.append(time.perf_counter() - t0)
    tn = []
    with ThreadPoolExecutor(max_workers=threads) as pool:
        for _ in range(repeats):
            t0 = time.perf_counter()
            parts = windowed(pool)
            tn.append(time.perf_counter() - t0)
    match = bool(np.array_equal(sum(pt["counters"] for pt in parts), ref["counters"]))
    return {"single_thread_us": round(statistics.median(t1) * 1e6, 1),
            "threads_over_windows_us": round(statistics.median(tn) * 1e6, 1),
            "threads": threads, "windows": len(starts), "counters_match": match}


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=CONFIG_DEFAULT, choices=sorted(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--window", type=int, default=None)
    ap.add_argument("--max-group", type=int, default=None)
    ap.add_argument("--bundle-window", type=int, default=None)
    ap.add_argument("--union-support", action="store_true",
                    help="every row of a group attends to its group's whole union (qup_union_support)")
    ap.add_argument("--page-major", action="store_true",
                    help="direct KV-page union: page-major items and partial results merged by lse")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--select", choices=["refine", "reuse"], default=None,
                    help="also time the proxy-query page selector (qup_pivot_select) on indexer inputs of the "
                         "workload's shape (128-wide index vectors, groups of 16, 4 x TopK candidates)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank)

    import torch
    import torch.distributed as dist
    import query_union_paged_b200 as qup

    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))

    w = W.make(args.config)
    max_group = args.max_group or w.max_group
    window = args.window or w.window
    bundle_window = args.bundle_window if args.bundle_window is not None else w.bundle_window
    dev = {}
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    dev["Q"] = t(w.Q).view(torch.bfloat16) if w.q_dtype == W.DT_BF16 else t(w.Q)
    dev["K"] = t(w.Kc).view(torch.bfloat16) if w.kv_dtype == W.DT_BF16 else t(w.Kc)
    dev["V"] = t(w.Vc).view(torch.bfloat16) if w.kv_dtype == W.DT_BF16 else t(w.Vc)
    ks = t(w.k_scale) if w.k_scale is not None else None
    vs = t(w.v_scale) if w.v_scale is not None else None
    topk, page_table, q_pos = t(w.topk), t(w.page_table), t(w.q_pos)
    ws_bytes, cap = qup.group_workspace(w.Hq, w.Hkv, w.Nq, w.K, w.num_logical_pages, max_group, window)
    groups = qup.alloc_groups(w.Hq, w.Hkv, w.Nq, cap, ws_bytes, dev["Q"].device)
    groups.bundle_window = bundle_window
    O = torch.empty_like(dev["Q"])
    stream = torch.cuda.current_stream()

    items = None
    if args.page_major:
        items = qup.page_major_items(topk, w.Hq, w.Hkv, w.num_logical_pages, w.T)

    def step(ev=None):
        if args.page_major:  # items (timed as the grouping call), then attention and the merge
            if ev is not None:
                ev[0].record(stream)
            qup.page_major_items(topk, w.Hq, w.Hkv, w.num_logical_pages, w.T, out=items)
            if ev is not None:
                ev[1].record(stream)
            qup.page_major_attn(dev["Q"], dev["K"], dev["V"], page_table, items, q_pos, w.kv_len, k_scale=ks,
                                v_scale=vs, out=O, num_logical_pages=w.num_logical_pages)
            if ev is not None:
                ev[2].record(stream)
            return
        if ev is not None:
            ev[0].record(stream)
        qup.sparse_group(topk, w.Hq, w.Hkv, w.num_logical_pages, max_group, window, out=groups)
        if args.union_support:
            qup.union_support(groups, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, max_group)
        if ev is not None:
            ev[1].record(stream)
        qup.sparse_prefill_attn(dev["Q"], dev["K"], dev["V"], page_table, groups, q_pos, w.kv_len,
                                k_scale=ks, v_scale=vs, topk=topk, out=O,
                                num_logical_pages=w.num_logical_pages)
        if ev is not None:
            ev[2].record(stream)

    l2 = torch.cuda.get_device_properties(local_rank).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device="cuda")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert qup.get_error() == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for k in range(args.steps):
            flush.zero_()  # untimed: every timed step starts with a cold L2
            step(evs[k])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    code = qup.get_error()
    if code:
        raise RuntimeError(f"device error {code} during the timed steps")
    # the same steps with a warm L2 (no flush between them), reported beside the cold numbers
    wevs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for k in range(args.steps):
        step(wevs[k])
    torch.cuda.synchronize()
    w_group = [wevs[k][0].elapsed_time(wevs[k][1]) for k in range(args.steps)]
    w_attn = [wevs[k][1].elapsed_time(wevs[k][2]) for k in range(args.steps)]
    t_group = [evs[k][0].elapsed_time(evs[k][1]) for k in range(args.steps)]
    t_attn = [evs[k][1].elapsed_time(evs[k][2]) for k in range(args.steps)]
    t_step = [a + b for a, b in zip(t_group, t_attn)]
    total_ms = max_over_ranks(sum(t_step), world, "cuda")

    # ---- work accounting (with union support, a row's edges are those of its group's union)
    E = int(selected_edges_per_row(w, union_topk(w, groups) if args.union_support else None).sum())
    flop = 4.0 * w.d * E
    n_uniq = unique_kv_pages(w)
    uniq_bytes = n_uniq * w.kv_page_bytes()
    if args.page_major:  # the grouping counters of the same selection, for the work accounting
        qup.sparse_group(topk, w.Hq, w.Hkv, w.num_logical_pages, max_group, window, out=groups)
    ctr = groups.counters.cpu().numpy().sum(axis=0)
    bctr = groups.bcounters.cpu().numpy().sum(axis=0)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(flop, world, ms_per_step)
    attn_ms = statistics.mean(t_attn)
    peaks = measured_peaks()
    # contraction dtype: bf16 MMAs for bf16 KV, tf32 for fp32, fp8 for E4M3 (nominal 2x bf16)
    mma_peak = {W.DT_BF16: peaks["bf16_tflops"], W.DT_F32: peaks["bf16_tflops"] / 2,
                W.DT_E4M3: peaks["bf16_tflops"] * 2}[w.kv_dtype]
    attn_tflops = flop / (attn_ms * 1e-3) / 1e12

    # ---- the upstream selector, timed alone (not part of the step or its metric)
    select = None
    if args.select:
        prefix = int(w.q_pos.min())
        base_p = (prefix + w.Nq + w.T - 1) // w.T
        inp = W.indexer_inputs(7, w.Nq, w.Hkv, 128, prefix, w.T, extra_pages=max(0, w.num_logical_pages - base_p))
        qi = torch.from_numpy(inp.q_bits).cuda().view(torch.bfloat16)
        pk = torch.from_numpy(inp.k_bits).cuda().view(torch.bfloat16)
        qp = torch.from_numpy(inp.q_pos).cuda()
        G, C, Ks = 16, min(256, 4 * w.K), w.K
        sel_out = torch.empty((w.Hq, w.Nq, Ks), dtype=torch.int32, device="cuda")
        refine = args.select == "refine"
        for _ in range(3):
            qup.pivot_select(qi, pk, qp, w.Hq // w.Hkv, w.T, G, C, Ks, refine=refine, out=sel_out)
        sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for k in range(args.steps):
            flush.zero_()
            sev[k][0].record(stream)
            qup.pivot_select(qi, pk, qp, w.Hq // w.Hkv, w.T, G, C, Ks, refine=refine, out=sel_out)
            sev[k][1].record(stream)
        torch.cuda.synchronize()
        assert qup.get_error() == 0
        groups_n = (w.Nq + G - 1) // G
        scan_macs = w.Hkv * sum(min(inp.num_logical_pages, int(inp.q_pos[g0:g0 + G].max()) // w.T + 1)
                                for g0 in range(0, w.Nq, G)) * 128
        select = {"variant": args.select, "group_size": G, "n_cand": C, "topk": Ks, "index_dim": 128,
                  "us_per_call": round(statistics.median([a.elapsed_time(b) for a, b in sev]) * 1e3, 2),
                  "proxy_scan_macs": int(scan_macs), "groups": groups_n * w.Hkv,
                  "refine_macs": int(w.Hkv * w.Nq * C * 128) if refine else 0}

    # ---- end to end through host buffers (pinned), copies inside the timed region
    e2e = None if args.page_major else run_e2e(args, w, qup, dev, ks, vs, groups, max_group, window, stream, O, flop)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {W.DT_BF16: "bf16", W.DT_F32: "f32", W.DT_E4M3: "e4m3"}[w.kv_dtype],
        "data": "synthetic (seeded; shapes of the pages' prefill chunks)",
        "config": {"workload": w.name, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "d": w.d,
                   "page_tokens": w.T, "topk": w.K, "kv_len": w.kv_len, "max_group": max_group,
                   "window": window, "bundle_window": bundle_window,
                   "support": "group union" if args.union_support else "own TopK row",
                   "execution": "page-major items, partial results merged by lse" if args.page_major
                   else "query unions (bundles of page-affine groups)",
                   "l2": "flushed before every timed step (2x L2 write)",
                   "parallelism": f"replicas x{world} (independent chunks)"},
        "us_per_call": {"group": round(statistics.median(t_group) * 1e3, 2),
                        "attn": round(statistics.median(t_attn) * 1e3, 2),
                        "complete": round(statistics.median(t_step) * 1e3, 2),
                        "attn_min": round(min(t_attn) * 1e3, 2), "attn_max": round(max(t_attn) * 1e3, 2)},
        "warm_l2_us_per_call": {"group": round(statistics.median(w_group) * 1e3, 2),
                                "attn": round(statistics.median(w_attn) * 1e3, 2),
                                "complete": round(statistics.median([a + b for a, b in zip(w_group, w_attn)]) * 1e3, 2)},
        "work": {"selected_edges": E, "flop": flop, "unique_kv_pages": n_uniq,
                 "unique_kv_bytes": uniq_bytes, "logical_page_visits": int(ctr[0]),
                 "masked_row_slots": int(ctr[1]), "masked_query_slots": int(ctr[2]),
                 "page_edges": int(ctr[3]), "bundles": int(bctr[1]),
                 "bundle_page_visits": int(bctr[0]),
                 "streamed_kv_bytes": int(bctr[0]) * w.kv_page_bytes()},
        **({"page_major": {"items": int(items.arrays["n_items"].sum().item()), "tile_pages": items.tile_pages,
                           "streamed_kv_bytes": int(items.arrays["n_items"].sum().item()) * items.tile_pages *
                           w.kv_page_bytes(),
                           "partial_results": int(items.arrays["row_off"][-1].item()),
                           "partial_bytes_written_and_read": 2 * int(items.arrays["row_off"][-1].item()) * 4 * (w.d + 1)}}
           if args.page_major else {}),
        "roofline": {"kernel": "union_attn_kernel", "bound": "tensor",
                     "achieved": round(attn_tflops, 2), "peak": round(mma_peak, 1), "unit": "TFLOP/s",
                     "frac": round(attn_tflops / mma_peak, 4),
                     "traffic": profiled_traffic(w.name),
                     "peak_source": peaks["source"] + " bf16 burst" +
                     ("" if w.kv_dtype == W.DT_BF16 else " x nominal dtype ratio"),
                     "unique_kv_gbs": round(uniq_bytes / (attn_ms * 1e-3) / 1e9, 1),
                     "hbm_frac_unique_kv": round(uniq_bytes / (attn_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
        **({"select": select} if select else {}),
        "gpu_launches": (LAUNCHES_PER_STEP + (LAUNCHES_UNION_SUPPORT if args.union_support else 0)) * args.steps,
        "e2e": e2e,
    }
    if rank == 0:
        line["clocks"] = clk.summary()
        if world == 1 and not args.no_cpu_baseline:
            tf, cores, desc = oracle_sample(w)
            line["cpu_baseline"] = {"value": round(tf, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                    "sample": desc,
                                    "group_reference": group_reference_sample(w, max_group, window)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(args, w, qup, dev, ks, vs, groups, max_group, window, stream, O_ref, flop):
    """Same metric through the public calls with host (pinned) inputs and output.

    Every step copies its inputs (Q, TopK, q_pos, page table) from pinned host memory and reads
    its output O back into pinned host memory.  Steps are pipelined over three streams with two
    device buffers per input and output: the copies in of step k+1 and the read-back of step k-1
    run while step k computes (the device has separate copy engines for each direction).
    """
    import torch
    host = {"Q": dev["Q"].cpu().pin_memory(), "topk": torch.from_numpy(w.topk).pin_memory(),
            "q_pos": torch.from_numpy(w.q_pos).pin_memory(),
            "page_table": torch.from_numpy(w.page_table).pin_memory()}
    d_in = [{k: torch.empty_like(v, device="cuda") for k, v in host.items()} for _ in range(2)]
    O = [torch.empty_like(d_in[0]["Q"]) for _ in range(2)]
    O_host = [torch.empty_like(host["Q"]).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = O[0].numel() * O[0].element_size()
    s_in, s_comp, s_out = torch.cuda.Stream(), stream, torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in comp_done + out_done:
        e.record(s_comp)

    def step(k):
        b = k & 1
        s_in.wait_event(comp_done[b])      # step k-2 has finished reading input slot b
        with torch.cuda.stream(s_in):
            for key in host:
                d_in[b][key].copy_(host[key], non_blocking=True)
        in_ready[b].record(s_in)
        s_comp.wait_event(in_ready[b])
        s_comp.wait_event(out_done[b])     # step k-2's output in slot b has been read back
        di = d_in[b]
        qup.sparse_group(di["topk"], w.Hq, w.Hkv, w.num_logical_pages, max_group, window, out=groups,
                         stream=s_comp)
        if args.union_support:
            qup.union_support(groups, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, max_group, stream=s_comp)
        qup.sparse_prefill_attn(di["Q"], dev["K"], dev["V"], di["page_table"], groups, di["q_pos"],
                                w.kv_len, k_scale=ks, v_scale=vs, topk=di["topk"], out=O[b],
                                num_logical_pages=w.num_logical_pages, stream=s_comp)
        comp_done[b].record(s_comp)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            O_host[b].copy_(O[b], non_blocking=True)
        out_done[b].record(s_out)

    for k in range(3):
        step(k)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(3, args.steps)
    e0.record(s_comp)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for k in range(n):
        step(k)
    s_comp.wait_stream(s_out)
    s_comp.wait_stream(s_in)
    e1.record(s_comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    # the output read back through host memory is the device path's output
    if not torch.equal(O_host[(n - 1) & 1], O_ref.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident run")
    return {"value": round(flop / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "pipelined": "copies in, compute and read-back on three streams, two buffers each"}


def run_reference(args, rank):
    """The fp64 CPU oracle as it stands, timed on the host cores on a bounded sample of the workload."""
    if rank != 0:
        return
    w = W.make(args.config)
    vals = []
    desc = None
    cores = os.cpu_count() or 1
    for k in range(args.warmup + args.steps):
        tf, cores, desc = oracle_sample(w, target_s=2.0, seed=k)
        if k >= args.warmup:
            vals.append(tf)
    value = statistics.mean(vals)
    flop_per_step = 4.0 * w.d * float(selected_edges_per_row(w).sum())
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(flop_per_step / (value * 1e12) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes of the pages' prefill chunks)",
        "config": {"workload": w.name, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "d": w.d, "page_tokens": w.T,
                   "topk": w.K, "kv_len": w.kv_len, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
