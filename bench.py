"""Decode-step benchmark of libbytecross on the Llama-3.1-8B shape.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on stdout (rank 0).  A step is one batch-1 decode step through
the whole hot path.  The headline cell is mode `both` (rp 0.5, rkv 0.3, page
16, 1 sink page, 256 recent tokens) at 32K context: that mode runs every
kernel of the path (norm+select, gathered GEMVs with the rotary/append
epilogue, page scores and select, split-K attention and combine, SwiGLU,
LM head).  The line also carries every mode (dense/act/kv/both) at 2K, 8K,
32K, 64K and 128K context, with decode tok/s, byte-account bytes per step,
achieved GB/s and the fraction of the measured HBM peak, plus the measured
mode crossings against the byte-account n*.

Inputs are synthetic (random bf16 weights N(0, 0.02), keys N(0,1) with four
outlier channels x8, values N(0,1)), resident in HBM before timing.  Every
step reads more than 6 GB, far beyond the 126 MB L2, so no flush is needed.
With N > 1 each rank runs an independent replica (no collective on the data
path); time is the max over ranks and value sums the tokens of all ranks.

--impl reference times the fp64 CPU oracle (the checker, as it stands) on a
bounded sample of the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tok/s per mode (dense/act/KV/both), 2K–128K ctx; HBM GB/s vs B200 peak"
HEAD_MODE, HEAD_CTX = "both", 32768
KEEP = dict(rp=0.5, rkv=0.3, sinks=1, recent=16)
CONTEXTS = (131072, 65536, 32768, 8192, 2048)         # descending: every cell sees pristine synthetic KV
FORCED = dict(sinks=1, recent=16)                     # 1 sink page, 16 recent pages = 256 tokens
# Bench cells: name -> (library mode, keep arguments).  The keep pairs are the
# ones the ByteCross README times (rp 0.7 / 0.5, rkv 0.3 / 0.5).
CELLS = {
    "dense": ("dense", {}),
    "act": ("act", dict(rp=0.5)),
    "kv": ("kv", dict(rkv=0.3, **FORCED)),
    "both": ("both", dict(rp=0.5, rkv=0.3, **FORCED)),
    # the pages' KV window baseline: the kv mode with no scored pages
    # (K = |F|: the sink page and the 16 recent pages)
    "window": ("kv", dict(rkv=1e-6, **FORCED)),
    # the same window computed by the masked dense baseline: every KV byte
    # read, an additive mask keeping the window's pages
    "masked": ("masked", dict(FORCED)),
    # the pages' own KV mode: one selection after prefill (16 observation
    # positions per query head), then steps over the frozen pages
    "snap": ("snap", dict(rkv=0.3, **FORCED)),
    "act@0.7": ("act", dict(rp=0.7)),
    "kv@0.5": ("kv", dict(rkv=0.5, **FORCED)),
    "both@0.7/0.3": ("both", dict(rp=0.7, rkv=0.3, **FORCED)),
    "both@0.5/0.5": ("both", dict(rp=0.5, rkv=0.5, **FORCED)),
}
DEFAULT_CELLS = ["dense", "act", "kv", "both", "window", "masked", "snap", "act@0.7", "kv@0.5",
                 "both@0.7/0.3", "both@0.5/0.5"]
MODE_KW = {name: kw for name, (_, kw) in CELLS.items()}
SNAP_OBS = 16
# the keep pairs whose act-vs-kv crossings are located: (rp, rkv) -> (act cell, kv cell)
CROSS_CELLS = {(0.7, 0.3): ("act@0.7", "kv"), (0.5, 0.3): ("act", "kv"), (0.5, 0.5): ("act", "kv@0.5")}
# the crossing sweep: 2K, then 4K to 128K in 4K steps, each context timed in
# every sweep cell back to back (a block), blocks repeated
SWEEP_CONTEXTS = tuple([2048] + [4096 * i for i in range(1, 33)])
SWEEP_CELLS = ("dense", "act@0.7", "act", "kv", "kv@0.5")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def dist_init(n_gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
        return dist.get_rank(), ws, int(os.environ.get("LOCAL_RANK", "0"))
    return 0, 1, 0


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws, dev):
    """Slowest rank's value (the job's time); one all-reduce, timing only."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, ws, dev):
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def replica_throughput(tokens_per_rank, seconds, ws, dev):
    """Whole-job throughput of independent replicas: all ranks' tokens over
    the slowest rank's time."""
    return sum_over_ranks(tokens_per_rank, ws, dev) / max_over_ranks(seconds, ws, dev)


class Clocks:
    """nvidia-smi samples of this GPU, kept with host timestamps."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.samples = []
        self.windows = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 7:
                self.samples.append((time.time(), parts))

    def window(self, t0, t1):
        self.windows.append((t0, t1))

    def summary(self):
        if self.proc:
            self.proc.terminate()
        inside = [p for (t, p) in self.samples if any(a <= t <= b for a, b in self.windows)]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[0]) for p in inside if num(p[0]) is not None]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for p in inside for i in range(4) if p[3 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(inside[0][1]),
                "reasons": reasons, "samples": len(inside),
                "power_w_max": max((num(p[2]) or 0) for p in inside)}


def record_traffic(csv_path, key="k_gemv_gateup", kernel="k_gemv", source="gemv.cu"):
    """Writes profiles/traffic.json from an ncu raw-page CSV export
    (`ncu -i rep --page raw --csv`) of `--only-kernel gemv_gateup`: the mean
    DRAM bytes read + written per captured launch of `kernel`, stamped with
    the kernel source's hash so a later change of the source voids it."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    hdr, units = rows[0], rows[1]
    scale = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    ir, iw, ik = hdr.index("dram__bytes_read.sum"), hdr.index("dram__bytes_write.sum"), hdr.index("Kernel Name")
    per = [float(r[ir].replace(",", "")) * scale[units[ir]] + float(r[iw].replace(",", "")) * scale[units[iw]]
           for r in rows[2:] if r[ik].split("(")[0].split("<")[0].split()[-1] == kernel]
    if not per:
        raise SystemExit(f"no {kernel} launches in {csv_path}")
    src = os.path.join(ROOT, "activation_kv_sparsity_b200", "csrc", source)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    p = os.path.join(ROOT, "profiles", "traffic.json")
    d = json.load(open(p)) if os.path.exists(p) else {}
    d[key] = {"source": source, "source_sha": sha, "dram_bytes_per_launch": round(sum(per) / len(per)),
              "launches": len(per), "capture": "ncu --set full --clock-control none -k regex:k_gemv -s 3 -c 1 "
                                               "python bench.py --only-kernel gemv_gateup --steps 3 --warmup 3"}
    json.dump(d, open(p, "w"), indent=1)
    return d[key]


def traffic_record(kernel):
    """DRAM bytes per launch from the committed ncu summary, valid only while
    the kernel source is unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, "activation_kv_sparsity_b200", "csrc", rec["source"])
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return rec["dram_bytes_per_launch"] if sha == rec["source_sha"] else None


# ------------------------------------------------------------------ our arm

def cell_kw(name):
    """Full keep arguments of a cell (ratios default to 1, the forced pages
    to the benchmark's 1 sink page and 16 recent pages)."""
    kw = dict(rp=1.0, rkv=1.0, **FORCED)
    kw.update(CELLS[name][1])
    return kw


def run_ours(args, rank, ws, local):
    import torch
    import activation_kv_sparsity_b200 as bc
    from synth import LLAMA_8B, kv_chunks, make_weights, obs_queries

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = LLAMA_8B
    contexts = sorted(set(args.contexts), reverse=True)
    sweep_ctx = sorted((n for n in SWEEP_CONTEXTS if n <= max(contexts)), reverse=True) if args.sweep_blocks else []
    steps, warm = args.steps, args.warmup
    sw_steps = min(steps, args.sweep_steps)
    max_ctx = max(contexts + sweep_ctx) + warm + steps + 32
    w = make_weights(cfg, seed=0, device=dev)
    model = bc.Model(cfg, w, max_ctx)

    def refill():
        # the synthetic cache up to the longest context (each pass over the
        # contexts runs from long to short, so every cell reads pristine KV)
        model.reset(0)
        for k, v in kv_chunks(cfg, max(contexts + sweep_ctx), seed=1, device=dev):
            model.append(k, v)
        torch.cuda.synchronize()
    refill()
    stream = model.stream
    logits = torch.empty(cfg["vocab"], device=dev)
    toks = [(1 + 7919 * i) % cfg["vocab"] for i in range(warm + steps)]
    props = torch.cuda.get_device_properties(dev)
    clocks = Clocks(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local))
    peak, peak_kind = peaks()

    q_obs = obs_queries(cfg, SNAP_OBS, device=dev) if "snap" in args.modes else None
    snap_select_ms = {}
    host_enqueue = {}

    def time_cell(name, n, k_steps):
        lib, kw = CELLS[name]
        model.reset(n)
        if lib == "snap":
            # the selection is paid once per prefill: timed apart from the steps
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            model.snap_select(q_obs, **kw)
            s1.record(stream)
            torch.cuda.synchronize()
            snap_select_ms[n] = s0.elapsed_time(s1)
        for i in range(warm):
            model.step(toks[i], lib, logits, **kw)
        torch.cuda.synchronize()
        barrier(ws)
        l0 = model.launches()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.time()
        e0.record(stream)
        h0 = time.perf_counter()
        for i in range(k_steps):
            model.step(toks[warm + i], lib, logits, **kw)
        host_enqueue[(name, n)] = (time.perf_counter() - h0) * 1e3 / k_steps
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.window(t0, time.time())
        barrier(ws)
        ms = max_over_ranks(e0.elapsed_time(e1) / k_steps, ws, dev)
        return ms, model.launches() - l0

    def step_bytes(name, n, k_steps):
        """Byte account of the timed steps (contexts n+warm .. n+warm+k_steps-1), averaged."""
        lib, _ = CELLS[name]
        kw = cell_kw(name)
        if lib == "snap":
            # the step right after the selection at n, plus every token
            # appended since (each is read: frozen partial page, new pages)
            base = bc.byte_account(cfg, "snap", n, **kw)
            tok_bytes = cfg["n_layers"] * cfg["n_kv_heads"] * 2 * cfg["head_dim"] * 2
            return base, base["impl_total_bytes"] + tok_bytes * (warm + (k_steps - 1) / 2.0)
        accs = [bc.byte_account(cfg, lib, n + warm + i, **kw) for i in range(k_steps)]
        return accs[0], sum(a["impl_total_bytes"] for a in accs) / k_steps

    def time_e2e(n):
        # end to end through the public host-buffer entry point, at context n
        host_logits = torch.empty(cfg["vocab"], pin_memory=True)
        model.reset(n)
        kwh = MODE_KW[HEAD_MODE]
        for i in range(warm):
            model.step_host(toks[i], HEAD_MODE, host_logits, **kwh)
        barrier(ws)
        t0 = time.perf_counter()
        for i in range(steps):
            model.step_host(toks[warm + i], HEAD_MODE, host_logits, **kwh)
        secs = time.perf_counter() - t0
        return {"value": round(replica_throughput(steps, secs, ws, dev), 2), "unit": "tok/s",
                "h2d_bytes_per_step": 4, "d2h_bytes_per_step": 4 * cfg["vocab"],
                "note": "bc_decode_step_host: token id passed by value in the launch, logits copied to "
                        "pinned host memory, stream synchronised every step; wall clock"}

    e2e = None
    cells = {}
    for n in contexts:
        if n == HEAD_CTX or (e2e is None and n == min(contexts)):
            e2e = time_e2e(n)
        for name in args.modes:
            ms, launches = time_cell(name, n, steps)
            acc, nbytes = step_bytes(name, n, steps)
            gbs = nbytes / (ms * 1e-3) / 1e9
            cells[(name, n)] = dict(mode=name, context=n, ms_per_step=round(ms, 4),
                                    tok_s=round(1000.0 / ms, 2), bytes_per_step=nbytes,
                                    gbs=round(gbs, 1), frac_of_measured_peak=round(gbs / peak, 4),
                                    paper_bound=round(acc["bound"], 4), launches_per_step=launches // steps,
                                    host_enqueue_ms=round(host_enqueue[(name, n)], 4))
            if CELLS[name][0] == "snap":
                cells[(name, n)]["selection_ms_once"] = round(snap_select_ms[n], 3)
    for n in contexts:
        if ("dense", n) not in cells:
            continue
        d = cells[("dense", n)]
        for name in args.modes:
            c = cells.get((name, n))
            if c is None or name == "dense":
                continue
            c["speedup_vs_dense"] = round(d["ms_per_step"] / c["ms_per_step"], 4)
            # the bound a pure byte count allows: dense bytes over this cell's bytes
            c["byte_bound_vs_dense"] = round(d["bytes_per_step"] / c["bytes_per_step"], 4)
        if ("window", n) in cells and ("masked", n) in cells:
            cells[("window", n)]["speedup_vs_masked_dense"] = round(
                cells[("masked", n)]["ms_per_step"] / cells[("window", n)]["ms_per_step"], 4)

    # the crossing sweep: blocks of every sweep cell at every context
    sweep = []
    for b in range(args.sweep_blocks):
        refill()
        block = {}
        for n in sweep_ctx:
            for name in SWEEP_CELLS:
                ms, _ = time_cell(name, n, sw_steps)
                block[(name, n)] = {"ms_per_step": ms, "bytes_per_step": step_bytes(name, n, sw_steps)[1]}
        sweep.append(block)

    # the batched step: B sequences of equal length in lock step, each with
    # its own cache, against B batch-1 steps of the same context and mode
    batch_rows = []
    if args.batch_ctx and args.batch_ctx in contexts:
        n_b = args.batch_ctx
        for B in args.batches:
            bt = bc.Batch(cfg, w, B, n_b + warm + steps + 8)
            chunks = [list(kv_chunks(cfg, n_b, seed=1 + b, device=dev)) for b in range(B)]
            for i in range(len(chunks[0])):
                bt.append(torch.stack([chunks[b][i][0] for b in range(B)]),
                          torch.stack([chunks[b][i][1] for b in range(B)]))
            del chunks
            blog = torch.empty(B, cfg["vocab"], device=dev)
            for name in ("act", "both"):
                lib, kw = CELLS[name]
                bt.reset(n_b)
                for i in range(warm):
                    bt.step([(toks[i] + b) % cfg["vocab"] for b in range(B)], lib, blog, **kw)
                torch.cuda.synchronize()
                l0 = bt.launches()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(bt.stream)
                for i in range(steps):
                    bt.step([(toks[warm + i] + b) % cfg["vocab"] for b in range(B)], lib, blog, **kw)
                e1.record(bt.stream)
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1) / steps
                t1 = cells[(name, n_b)]["ms_per_step"] if (name, n_b) in cells else None
                batch_rows.append({"batch": B, "mode": name, "context": n_b, "ms_per_step": round(ms, 4),
                                   "tok_s": round(1000.0 * B / ms, 2),
                                   "ms_per_step_batch1": t1,
                                   "speedup_vs_separate_steps": round(B * t1 / ms, 3) if t1 else None,
                                   "launches_per_step": (bt.launches() - l0) // steps})
            bt.close()
            del bt
            torch.cuda.empty_cache()

    head = cells.get((HEAD_MODE, HEAD_CTX)) or cells.get((HEAD_MODE, contexts[0])) or next(iter(cells.values()))
    head_ctx = head["context"]
    head_launches = head["launches_per_step"] * steps

    # roofline of the dominant kernel of the headline step: the gathered
    # gate/up GEMV (k = ceil(0.5 * 4096) rows of 28672 bf16), timed alone
    # over the 32 layers' weights with the step's launch configuration
    kq = math.ceil(0.5 * cfg["hidden"] - 1e-9)
    d_out = 2 * cfg["intermediate"]
    idx = torch.sort(torch.randperm(cfg["hidden"], device=dev)[:kq])[0].to(torch.int32)
    xin = torch.randn(cfg["hidden"], device=dev)
    y = torch.empty(d_out, device=dev)
    scratch = torch.zeros(bc.bc_gemv_scratch_bytes(d_out), dtype=torch.uint8, device=dev)
    wgu = w["wgu_t"]
    it = [0]

    def launch_gu():
        bc.gemv(wgu[it[0] % cfg["n_layers"]], xin, idx, y, scratch)
        it[0] += 1
    # 4 x 32 launches over the 32 layers' weights, replayed from a CUDA graph
    gemv_ms = graph_timed(launch_gu, 4, 4 * cfg["n_layers"], dev)
    gemv_bytes = kq * d_out * 2 + kq * 8            # weight rows + index/activation reads
    achieved = gemv_bytes / (gemv_ms * 1e-3) / 1e9

    clk = clocks.summary()
    result = {
        "metric": METRIC,
        "value": round(replica_throughput(steps, head["ms_per_step"] * steps / 1000.0, ws, dev), 2),
        "unit": "tok/s",
        "n_gpus": ws,
        "steps": steps,
        "warmup": warm,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 weights/KV, fp32 accumulate",
        "data": "synthetic (seeded random weights and KV, resident in HBM)",
        "config": {"workload": f"Llama-3.1-8B-shaped decode, 1 sequence, {head_ctx // 1024}K context, mode {HEAD_MODE} "
                               f"(rp 0.5, rkv 0.3, page 16, 1 sink page, 256 recent tokens)",
                   "global_batch": ws, "seq_len": head_ctx, "parallelism": f"replicas x{ws}",
                   "l2": "no flush: every step reads > 6 GB, inputs far larger than the 126 MB L2"},
        "gpu_launches": head_launches,
        "roofline": {"kernel": "k_gemv (gate/up, 2048 of 4096 rows gathered, 28672 cols)", "bound": "hbm",
                     "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic_record("k_gemv_gateup"),
                     "launch_ms": round(gemv_ms, 5), "algorithmic_bytes_per_launch": gemv_bytes},
        "step_roofline": {"bytes_per_step": head["bytes_per_step"], "gbs": head["gbs"],
                          "frac": head["frac_of_measured_peak"]},
        "clocks": clk,
        "e2e": e2e,
        "modes": [cells[k] for k in sorted(cells, key=lambda k: (k[1], k[0]))],
        "crossings": crossing_report(bc, cfg, cells, contexts, sweep, sweep_ctx, sw_steps),
        "batched": {"rows": batch_rows,
                    "note": "bc_batch_step: B sequences, each with its own synthetic cache and tokens, decoding in "
                            "lock step; the projections read the union of the batch's kept rows once, the LM head "
                            "once; compared with B batch-1 steps of the same mode and context"},
    }
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args, w, head_ctx)
    model.close()
    return result


def crossing_report(bc, cfg, cells, contexts, sweep, sweep_ctx, sw_steps):
    """Per keep pair: the paper-form n* (Equation 5), this implementation's
    byte crossing, the crossings measured in every sweep block, and the
    cost-aware prediction fitted on the sweep with its error."""
    out = {"sweep": {"contexts": sorted(sweep_ctx), "cells": list(SWEEP_CELLS), "blocks": len(sweep),
                     "steps_per_cell": sw_steps,
                     "note": "each block times every sweep cell at every context back to back (contexts "
                             "descending); a crossing is where t(act) - t(kv) turns non-negative, linearly "
                             "interpolated between neighbouring contexts"}}
    fit = None
    if sweep:
        asc = sorted(sweep_ctx)
        mean_cells = {(c, n): {"ms_per_step": statistics.mean(b[(c, n)]["ms_per_step"] for b in sweep),
                               "bytes_per_step": sweep[0][(c, n)]["bytes_per_step"]}
                      for c in SWEEP_CELLS for n in asc}
        fit = cost_aware_fit(mean_cells, asc, SWEEP_CELLS)
        out["sweep"]["ms_mean"] = {c: [round(mean_cells[(c, n)]["ms_per_step"], 4) for n in asc]
                                   for c in SWEEP_CELLS}
        if fit:
            out["cost_aware_fit"] = {"fit_gbs": round(1.0 / fit[0], 1),
                                     "fixed_cost_ms": {c: round(v * 1e3, 4) for c, v in fit[1].items()}}
    pairs = {}
    for (rp, rkv), (ca, ck) in CROSS_CELLS.items():
        acc = bc.byte_account(cfg, "both", 1024, rp=rp, rkv=rkv)
        row = {"act_cell": ca, "kv_cell": ck, "n_star_tokens": round(acc["n_star"], 1),
               "n_star_impl_tokens": impl_crossing(bc, cfg, rp, rkv)}
        if sweep:
            asc = sorted(sweep_ctx)
            diffs = [[(n, b[(ca, n)]["ms_per_step"] - b[(ck, n)]["ms_per_step"]) for n in asc] for b in sweep]
            per_block = [crossing_of(dd) for dd in diffs]
            row["measured_tokens_per_block"] = per_block
            found = [x for x in per_block if x is not None]
            row["measured_tokens"] = round(statistics.mean(found), 1) if found else None
            if found:
                row["measured_range_tokens"] = [min(found), max(found)]
            else:
                # no sign change inside the sweep: say on which side the crossing lies
                if all(dd[0][1] >= 0 for dd in diffs):
                    row["measured_outside_sweep"] = f"below {asc[0]} tokens (kv already faster at the first context)"
                elif all(dd[-1][1] < 0 for dd in diffs):
                    row["measured_outside_sweep"] = f"above {asc[-1]} tokens (act still faster at the last context)"
                row["diff_ms_first_last"] = [[round(dd[0][1], 4), round(dd[-1][1], 4)] for dd in diffs]
            if fit:
                pred = predicted_crossing(bc, cfg, fit[0], fit[1], ca, ck)
                row["cost_aware_predicted_tokens"] = pred
                if pred is not None and found:
                    row["prediction_error_tokens"] = round(pred - row["measured_tokens"], 1)
        pairs[f"{rp}/{rkv}"] = row
    out["pairs"] = pairs
    # the coarse cells of the main sweep, for reference (the headline keep pair)
    out["coarse_act_vs_kv"] = measured_crossing(cells, contexts)
    out["coarse_act_vs_kv"]["cost_aware_prediction"] = cost_aware_prediction(cells, contexts, cfg, bc)
    return out


def impl_crossing(bc, cfg, rp, rkv, sinks=1, recent=16):
    """Context at which the act and kv steps of this library move the same
    bytes (bc_byte_account's implementation form), by bisection."""
    def diff(n):
        a = bc.byte_account(cfg, "act", n, rp=rp, sinks=sinks, recent=recent)["impl_total_bytes"]
        k = bc.byte_account(cfg, "kv", n, rkv=rkv, sinks=sinks, recent=recent)["impl_total_bytes"]
        return a - k          # negative while the projection branch moves fewer bytes
    lo, hi = 1, 1 << 21
    if diff(lo) >= 0 or diff(hi) <= 0:
        return None
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if diff(mid) < 0:
            lo = mid
        else:
            hi = mid
    return hi


def cost_aware_fit(cells, contexts, kinds):
    """The pages' cost-aware model restated for this library: per cell kind,
    step time = byte-account bytes / B + c (one bandwidth B for all kinds,
    one fixed per-step kernel cost c per kind), fitted by least squares over
    the sampled contexts.  Returns (1/B in s per GB, {kind: c in s}) or None
    when a cell is missing."""
    import numpy as np
    kinds = list(kinds)
    if len(contexts) < 2 or not all((m, n) in cells for m in kinds for n in contexts):
        return None
    rows, ys = [], []
    for j, m in enumerate(kinds):
        for n in contexts:
            c = cells[(m, n)]
            rows.append([c["bytes_per_step"] / 1e9] + [1.0 if k == j else 0.0 for k in range(len(kinds))])
            ys.append(c["ms_per_step"] * 1e-3)
    sol, *_ = np.linalg.lstsq(np.array(rows), np.array(ys), rcond=None)
    return sol[0], dict(zip(kinds, sol[1:]))


def predicted_crossing(bc, cfg, inv_bw, costs, act_cell, kv_cell):
    """Context (tokens) at which the fitted act and kv step times meet, by bisection."""
    def t(cell, n):
        return bc.byte_account(cfg, CELLS[cell][0], n, **cell_kw(cell))["impl_total_bytes"] / 1e9 * inv_bw \
            + costs[cell]
    lo, hi = 1, 1 << 21
    if (t(act_cell, lo) - t(kv_cell, lo)) * (t(act_cell, hi) - t(kv_cell, hi)) > 0:
        return None
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if t(act_cell, mid) < t(kv_cell, mid):
            lo = mid
        else:
            hi = mid
    return hi


def cost_aware_prediction(cells, contexts, cfg, bc):
    """The cost-aware fit over the dense, act and kv cells of the main
    contexts and its predicted act-vs-kv crossing (rp 0.5, rkv 0.3)."""
    fit = cost_aware_fit(cells, contexts, ("dense", "act", "kv"))
    if fit is None:
        return None
    inv_bw, costs = fit
    return {"fit_gbs": round(1.0 / inv_bw, 1),
            "fixed_cost_ms": {m: round(v * 1e3, 4) for m, v in costs.items()},
            "predicted_act_vs_kv_tokens": predicted_crossing(bc, cfg, inv_bw, costs, "act", "kv")}


def crossing_of(diff):
    """First context where diff = t(act) - t(kv) turns from negative to
    non-negative, linearly interpolated (the README's convention for latency
    crossings); diff is [(context, ms)] ascending.  None if it never does."""
    for (n0, d0), (n1, d1) in zip(diff, diff[1:]):
        if d0 < 0 <= d1:
            return round(n0 + (n1 - n0) * (-d0) / (d1 - d0), 1)
    return None


def measured_crossing(cells, contexts, act="act", kv="kv"):
    """Context where the KV branch starts to beat the projection branch over
    the sampled contexts."""
    ctx = sorted(contexts)
    if not all((act, n) in cells and (kv, n) in cells for n in ctx):
        return {"act_vs_kv_tokens": None}
    diff = [(n, cells[(act, n)]["ms_per_step"] - cells[(kv, n)]["ms_per_step"]) for n in ctx]
    got = crossing_of(diff)
    if got is not None:
        return {"act_vs_kv_tokens": got, "keep": f"{act} vs {kv}"}
    return {"act_vs_kv_tokens": None, "diff_ms": diff}


# ------------------------------------------------------------------ the oracle on the host

def oracle_sample(w_host, cache, n_ctx, mode, layer, lm_rows, token=7):
    """Runs one layer of a decode step and a slice of the LM head in the fp64
    oracle; returns seconds for each part."""
    from oracle import decoder as od
    from synth import LLAMA_8B
    cfg = LLAMA_8B
    kw = MODE_KW[mode]
    cache.n = n_ctx
    t0 = time.perf_counter()
    x = od.decode_step(cfg, w_host, cache, token, mode, layers=range(layer, layer + 1),
                       x_in=od.bf16_to_f64(w_host["embed"][token]), **kw)
    t1 = time.perf_counter()
    xf = od.rms_norm(x, w_host["final_norm"], cfg["rms_eps"])
    _ = od.bf16_to_f64(w_host["lm_head"][:lm_rows]) @ xf
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def host_sample_inputs(w_dev, n_ctx, n_layers):
    """Host copies of what the oracle sample needs: the first n_layers'
    weights, the LM head slice, and a KV cache of those layers drawn from the
    input generator (the same recipe and seed as the timed cache; the oracle
    never reads the library's pool)."""
    from oracle import decoder as od
    from synth import LLAMA_8B, bf16_bits, kv_chunks
    cfg = LLAMA_8B
    wh = {}
    for name in ("attn_norm", "mlp_norm", "wqkv_t", "wo_t", "wgu_t", "wd_t"):
        wh[name] = bf16_bits(w_dev[name][:n_layers])
    wh["embed"] = bf16_bits(w_dev["embed"][:16])
    wh["final_norm"] = bf16_bits(w_dev["final_norm"])
    wh["lm_head"] = bf16_bits(w_dev["lm_head"][: cfg["vocab"] // 32])
    small = dict(cfg, n_layers=n_layers)
    cache = od.Cache(small, n_ctx + 1)
    for k, v in kv_chunks(small, n_ctx, seed=1, device=w_dev["embed"].device):
        cache.extend(bf16_bits(k), bf16_bits(v))
    cache.n = n_ctx
    return wh, cache


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count()


def cpu_baseline(args, w_dev, n_ctx):
    """The oracle as it stands, on the host cores: layers 0-11 of one decode
    step of the headline cell plus 1/32 of the LM head each (about 10 s of
    CPU work), scaled to a full step."""
    from synth import LLAMA_8B
    cfg = LLAMA_8B
    nl = 12
    wh, cache = host_sample_inputs(w_dev, n_ctx, nl)
    layer_s, head_s = [], 0.0
    for l in range(nl):
        a, b = oracle_sample(wh, cache, n_ctx, HEAD_MODE, l, cfg["vocab"] // 32)
        layer_s.append(a)
        head_s += b / nl
    step_s = statistics.mean(layer_s) * cfg["n_layers"] + head_s * 32
    return {"value": round(1.0 / step_s, 5), "unit": "tok/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"fp64 oracle, {HEAD_MODE} mode at {n_ctx} context: layers 0-{nl - 1} of one step "
                      f"(mean {statistics.mean(layer_s):.2f} s/layer) and 1/32 of the LM head, timed; the value "
                      f"extrapolates them to {cfg['n_layers']} layers + the whole head ({head_s * 32:.2f} s)",
            "seconds_timed": round(sum(layer_s) + head_s * nl, 2),
            "seconds_per_step_extrapolated": round(step_s, 2)}


def run_reference(args, rank, ws, local):
    """The oracle arm.  Each timed step is a bounded sample of the headline
    cell's decode step: one decoder layer (layers 0-3 in turn) and 1/32 of
    the LM head, i.e. 1/32 of a step's work; ``value`` counts a sample as
    1/32 of a token, and ``ms_per_step`` is the time of one sample as timed,
    so that ``steps * ms_per_step`` is the timed region."""
    import torch
    from synth import LLAMA_8B, kv_chunks, make_weights
    cfg = LLAMA_8B
    nl = 4
    n_ctx = HEAD_CTX
    frac = 1.0 / cfg["n_layers"]          # a sample's share of a step (one layer; 1/32 of the head)
    # inputs: drawn with the same generators; on the host when no GPU
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    small = dict(cfg, n_layers=nl)
    w = make_weights(small, seed=0, device=dev)
    from oracle import decoder as od
    from synth import bf16_bits
    cache = od.Cache(small, n_ctx + 1)
    for k, v in kv_chunks(small, n_ctx, seed=1, device=dev):
        cache.extend(bf16_bits(k), bf16_bits(v))
    wh = {name: bf16_bits(t) for name, t in w.items() if name not in ("embed", "lm_head")}
    wh["embed"] = bf16_bits(w["embed"][:16])
    wh["lm_head"] = bf16_bits(w["lm_head"][: cfg["vocab"] // cfg["n_layers"]])
    del w
    times = []
    for i in range(args.warmup + args.steps):
        a, b = oracle_sample(wh, cache, n_ctx, HEAD_MODE, i % nl, cfg["vocab"] // cfg["n_layers"])
        if i >= args.warmup:
            times.append(a + b)
    sample_s = statistics.mean(times)
    val = round(frac / sample_s, 6)
    sample = (f"fp64 oracle, {HEAD_MODE} mode at {n_ctx} context; one timed step = one decoder layer "
              f"(layers 0-{nl - 1} in turn) + 1/{cfg['n_layers']} of the LM head = 1/{cfg['n_layers']} of a "
              f"decode step, counted as 1/{cfg['n_layers']} token")
    return {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tok/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(sample_s * 1000, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"Llama-3.1-8B-shaped decode, 1 sequence, {n_ctx // 1024}K context, mode {HEAD_MODE} "
                               f"(rp 0.5, rkv 0.3, page 16, 1 sink page, 256 recent tokens)",
                   "global_batch": 1, "seq_len": n_ctx, "parallelism": "host cores"},
        "tokens_per_timed_step": frac,
        "timed_seconds": round(sum(times), 2),
        "full_step_ms_extrapolated": round(sample_s / frac * 1000, 1),
        "cpu_baseline": {"value": val, "unit": "tok/s", "cores": cpu_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def graph_timed(launch, warmup, steps, dev):
    """Milliseconds per launch of `steps` back-to-back launches replayed
    from one CUDA graph (no host launch cost between them), after `warmup`
    direct launches.  launch() must enqueue on the current stream."""
    import torch
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        for _ in range(warmup):
            launch()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for _ in range(steps):
            launch()
    gr.replay()
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    gr.replay()
    e1.record(cur)
    torch.cuda.synchronize()
    del gr
    return e0.elapsed_time(e1) / steps


def run_kernel_only(args, local):
    """Times one kernel alone on a small case (for profiler captures): the
    gathered gate/up GEMV of one layer (235 MB dense, 117 MB at rp 0.5) or
    the dense split-K attention of one layer at 128K context (537 MB)."""
    import torch
    import activation_kv_sparsity_b200 as bc
    from synth import LLAMA_8B
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = LLAMA_8B
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    stream = torch.cuda.current_stream(dev)
    if args.only_kernel == "snap":
        # the once-after-prefill scorer of 2 layers at 32K context, 16
        # observation positions (64 queries per kv head): 2 passes over the keys
        from synth import kv_chunks, make_weights, obs_queries
        c2 = dict(cfg, n_layers=2)
        n = 32768
        w = make_weights(c2, seed=0, device=dev)
        model = bc.Model(c2, w, n + 8)
        for k, v in kv_chunks(c2, n, seed=1, device=dev):
            model.append(k, v)
        q_obs = obs_queries(c2, 16, device=dev)
        flops = 2 * c2["n_layers"] * c2["n_heads"] * 16 * n * c2["head_dim"]   # one pass over the keys, 2 per FMA

        def launch():
            model.snap_select(q_obs, rkv=0.3, sinks=1, recent=16)
        for _ in range(args.warmup):
            launch()
        torch.cuda.synchronize()
        # the selection ends by reading the scorer's status word (a host
        # sync), so it is timed on the device: CUPTI kernel timestamps, from
        # a selection's first kernel's start to its last kernel's end
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            for _ in range(args.steps):
                launch()
            torch.cuda.synchronize()
        ev = sorted((e for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA
                     and e.name.split("(")[0].split("<")[0].split("::")[-1] in
                     ("k_snap", "k_snap_tc", "k_snap_merge", "k_snap_mass", "k_page_select", "k_page_select_cta")),
                    key=lambda e: e.time_range.start)
        per = 4 * c2["n_layers"]
        if len(ev) != per * args.steps:
            return {"kernel": "snap", "error": f"{len(ev)} kernels traced, expected {per * args.steps}"}
        spans = [ev[i * per + per - 1].time_range.end - ev[i * per].time_range.start for i in range(args.steps)]
        kern = {}
        for e in ev:
            nm = e.name.split("(")[0]
            kern.setdefault(nm, []).append(e.time_range.end - e.time_range.start)
        ms = sum(spans) / len(spans) / 1000.0
        keys = c2["n_layers"] * c2["n_kv_heads"] * n * c2["head_dim"] * 2     # key bytes read (one pass)
        return {"kernel": "snap", "ms_per_selection": round(ms, 4), "flops": flops,
                "tflops": round(flops / (ms * 1e-3) / 1e12, 2), "key_bytes": keys,
                "key_gbs": round(keys / (ms * 1e-3) / 1e9, 1),
                "us_per_kernel": {k: round(sum(v) / len(v), 2) for k, v in kern.items()},
                "note": "2 layers at 32K: the scorer (one pass over the keys), the chunk merge, the page masses "
                        "and the page select; device span per selection (CUPTI); tcgen05 M128 N256 K16, keys by "
                        "tensor copies, hi/lo-split queries"}
    if args.only_kernel == "gemv_batch":
        return run_batch_gemv(args, dev, stream, cfg)
    if args.only_kernel in ("gemv_gateup", "gemv_gateup_dense"):
        d, d_out = cfg["hidden"], 2 * cfg["intermediate"]
        W = (torch.randn(d, d_out, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        if args.only_kernel == "gemv_gateup":
            k = math.ceil(0.5 * d - 1e-9)
            idx = torch.sort(torch.randperm(d, device=dev, generator=g)[:k])[0].to(torch.int32)
        else:
            k, idx = d, None
        x = torch.randn(d, generator=g, device=dev)
        y = torch.empty(d_out, device=dev)
        scratch = torch.zeros(bc.bc_gemv_scratch_bytes(d_out), dtype=torch.uint8, device=dev)
        nbytes = k * d_out * 2 + k * 8

        def launch():
            bc.gemv(W, x, idx, y, scratch)
    elif args.only_kernel in ("select", "select_wide"):
        # the exact top-k of the projection branch alone: 2048 of 4096
        # (q/k/v, o, gate/up inputs) or 7168 of 14336 (the down input)
        n = 4096 if args.only_kernel == "select" else 14336
        k = math.ceil(0.5 * n - 1e-9)
        vs = torch.randn(64, n, generator=g, device=dev)
        idx = torch.empty(k, dtype=torch.int32, device=dev)
        nbytes = 0
        it = [0]

        def launch():
            bc.select_topk(vs[it[0] % 64], k, idx)
            it[0] += 1
    elif args.only_kernel == "attention_short":
        # the both@32K attention: 615 of 2049 pages per kv head (the sink,
        # the 16 recent pages and 598 others), 8 layers' pools in turn so
        # that no launch finds its pages in L2 (40 MB a launch, 1.07 GB of pools)
        Hkv, G, hd, n_tok, nl = cfg["n_kv_heads"], cfg["n_heads"] // cfg["n_kv_heads"], cfg["head_dim"], 32769, 8
        P = -(-n_tok // 16)
        K = math.ceil(0.3 * P - 1e-9)
        pools = torch.randn(nl, Hkv, P, 2, 16, hd, generator=g, device=dev).to(torch.bfloat16)
        lists = torch.zeros(nl, Hkv, P, dtype=torch.int32, device=dev)
        for l in range(nl):
            for h in range(Hkv):
                mid = torch.randperm(P - 17, generator=g, device=dev)[:K - 17] + 1
                sel = torch.cat([torch.tensor([0], device=dev), mid, torch.arange(P - 16, P, device=dev)])
                lists[l, h, :K] = torch.sort(sel)[0].to(torch.int32)
        q = torch.randn(Hkv * G, hd, generator=g, device=dev)
        out = torch.empty(Hkv * G, hd, device=dev)
        scratch = torch.zeros(bc.bc_attention_scratch_bytes(Hkv * G, hd), dtype=torch.uint8, device=dev)
        nbytes = Hkv * (K * 16 - (P * 16 - n_tok)) * 2 * hd * 2
        it = [0]

        def launch():
            l = it[0] % nl
            it[0] += 1
            bc.attention(q, pools[l], Hkv, G, hd, P, lists[l], K, n_tok, out, scratch)
    else:
        Hkv, G, hd, n_tok = cfg["n_kv_heads"], cfg["n_heads"] // cfg["n_kv_heads"], cfg["head_dim"], 131073
        P = -(-n_tok // 16)
        pool = torch.randn(Hkv, P, 2, 16, hd, generator=g, device=dev).to(torch.bfloat16)
        q = torch.randn(Hkv * G, hd, generator=g, device=dev)
        out = torch.empty(Hkv * G, hd, device=dev)
        scratch = torch.zeros(bc.bc_attention_scratch_bytes(Hkv * G, hd), dtype=torch.uint8, device=dev)
        nbytes = Hkv * n_tok * 2 * hd * 2

        def launch():
            bc.attention(q, pool, Hkv, G, hd, P, None, P, n_tok, out, scratch)
    ms = graph_timed(launch, args.warmup, args.steps, dev)
    peak, kind = peaks()
    if not nbytes:
        return {"kernel": args.only_kernel, "us_per_launch": round(ms * 1e3, 3),
                "note": "launches back to back on one stream (programmatic dependent launch)"}
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": args.only_kernel, "ms_per_launch": round(ms, 5), "algorithmic_bytes": nbytes,
            "gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "peak": peak, "peak_kind": kind,
            "note": "includes the fused combine" if args.only_kernel.startswith("attention") else ""}


def run_batch_gemv(args, dev, stream, cfg):
    """The gate/up projection of one layer (4096 -> 28672 columns, rp 0.5)
    for a batch of B sequences (--batches; 1, 2, 4, 8 by default): one batched GEMV over the union
    of their kept channels against B separate gathered GEMVs.  The
    selections are the library's own top-k of the synthetic batch
    activations.  L2 is flushed (a 256 MB write) before every timed launch,
    so the separate GEMVs cannot reuse each other's rows from L2."""
    import torch
    import activation_kv_sparsity_b200 as bc
    from synth import batch_activations
    d, d_out = cfg["hidden"], 2 * cfg["intermediate"]
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    W = (torch.randn(d, d_out, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    k = math.ceil(0.5 * d - 1e-9)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peak, kind = peaks()

    def timed(fn):
        ev = []
        for i in range(args.warmup + args.steps):
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            if i >= args.warmup:
                ev.append((e0, e1))
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    rows = []
    for B in args.batches:
        X = batch_activations(B, d, device=dev).contiguous()
        idx = torch.empty(B, k, dtype=torch.int32, device=dev)
        for b in range(B):
            bc.select_topk(X[b], k, idx[b], stream)
        y = torch.empty(B, d_out, device=dev)
        ys = torch.empty(B, d_out, device=dev)
        nu = torch.zeros(1, dtype=torch.int32, device=dev)
        scratch = torch.empty(bc.bc_gemv_batch_scratch_bytes(d, d_out, B), dtype=torch.uint8, device=dev)
        s1 = torch.zeros(bc.bc_gemv_scratch_bytes(d_out), dtype=torch.uint8, device=dev)
        ms_b = timed(lambda: bc.gemv_batch(W, X, idx, y, scratch, nu, stream))

        def separate():
            for b in range(B):
                bc.gemv(W, X[b], idx[b], ys[b], s1, stream)
        ms_s = timed(separate)
        u = int(nu.item())
        nbytes = u * d_out * 2 + B * (k * 4 + d * 4 + d_out * 4)
        gbs = nbytes / (ms_b * 1e-3) / 1e9
        keep = u / d
        rows.append({"batch": B, "union_rows": u, "union_keep": round(keep, 4),
                     "ms_batched": round(ms_b, 5), "ms_separate": round(ms_s, 5),
                     "speedup_vs_separate": round(ms_s / ms_b, 3), "algorithmic_bytes": nbytes,
                     "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                     "weight_rows_separate_over_union": round(B * k / u, 3),
                     "crossover_batch_tokens_rkv0.3": round(bc.crossover_batch(cfg, keep, 0.3, B), 1)})
    return {"kernel": "gemv_batch", "peak": peak, "peak_kind": kind, "rows": rows,
            "note": "gate/up of one layer, rp 0.5, batch activations with a shared component (union ~92% at 4); "
                    "L2 flushed before each timed launch; batched = union + GEMV (+ split reduce)"}


GEMV_SITES = ["qkv", "o", "gate_up", "down"]


def site_of(kernel: str, gemvs_seen: int) -> str:
    """Step site of a traced kernel: GEMVs come in projection order within a
    layer, a selection kernel belongs to the GEMV after it."""
    if "k_gemv" in kernel:
        return GEMV_SITES[gemvs_seen % 4]
    if "k_page_select" in kernel:
        return "page_select"
    if "k_pages" in kernel:
        return "page_scores"
    if "k_select" in kernel:
        return "sel_" + GEMV_SITES[gemvs_seen % 4]
    if "k_attn" in kernel:
        return "attn"
    return kernel


def run_timeline(args, local):
    """Per-site cost of one decode step, from the kernel timestamps CUPTI
    records (torch.profiler): with programmatic dependent launch a kernel's
    CTAs start before its predecessor ends, so each site is charged the time
    from the previous kernel's end to its own end."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    import activation_kv_sparsity_b200 as bc
    from synth import LLAMA_8B, kv_chunks, make_weights
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = LLAMA_8B
    mode, n = args.timeline, args.contexts[0]
    w = make_weights(cfg, seed=0, device=dev)
    model = bc.Model(cfg, w, n + args.warmup + 8)
    for k, v in kv_chunks(cfg, n, seed=1, device=dev):
        model.append(k, v)
    logits = torch.empty(cfg["vocab"], device=dev)
    for i in range(args.warmup):
        model.step(1 + i, mode, logits, **MODE_KW[mode])
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        model.step(7, mode, logits, **MODE_KW[mode])
        torch.cuda.synchronize()
    ev = [e for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA
          and "k_" in e.name.split("(")[0]]
    ev.sort(key=lambda e: e.time_range.start)
    L = cfg["n_layers"]
    if not ev or "k_lmhead" not in ev[-1].name:
        return {"error": f"the step's last kernel is not the LM head ({len(ev)} traced)"}
    cost = {}
    gemvs = 0
    prev = ev[0].time_range.start
    for e in ev[:-1]:
        name = e.name.split("(")[0]
        site = site_of(name, gemvs)
        gemvs += "k_gemv" in name
        cost[site] = cost.get(site, 0.0) + e.time_range.end - prev
        prev = e.time_range.end
    span = (ev[-1].time_range.end - ev[0].time_range.start) / 1000.0
    out = {"mode": mode, "context": n, "step_ms": round(span, 4), "kernels": len(ev),
           "us_per_layer": {k: round(v / L, 2) for k, v in cost.items()},
           "lm_head_us": round((ev[-1].time_range.end - prev) / 1.0, 2),
           "note": "CUPTI kernel timestamps; each site charged from the previous kernel's end to its own end"}
    model.close()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--contexts", type=int, nargs="+", default=list(CONTEXTS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--modes", nargs="+", default=list(DEFAULT_CELLS), choices=list(CELLS),
                    help="bench cells timed at every --contexts value")
    ap.add_argument("--sweep-blocks", type=int, default=2,
                    help="blocks of the 2K-128K crossing sweep in 4K steps (0: no sweep)")
    ap.add_argument("--sweep-steps", type=int, default=8, help="timed steps per sweep cell (at most --steps)")
    ap.add_argument("--batch-ctx", type=int, default=8192,
                    help="context of the batched-step cells (one of --contexts; 0: none)")
    ap.add_argument("--batches", type=int, nargs="+", default=[1, 2, 4, 8])
    ap.add_argument("--timeline", choices=("dense", "act", "kv", "both"),
                    help="per-site cost of one step in this mode at the first --contexts value")
    ap.add_argument("--record-traffic", metavar="NCU_RAW_CSV",
                    help="write profiles/traffic.json from an ncu raw CSV of --only-kernel gemv_gateup")
    ap.add_argument("--only-kernel", choices=("gemv_gateup", "gemv_gateup_dense", "attention", "attention_short", "snap",
                                              "gemv_batch", "select", "select_wide"),
                    help="time one kernel alone on a small case (profiler captures)")
    args = ap.parse_args()
    if args.record_traffic:
        print(json.dumps(record_traffic(args.record_traffic)))
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        # the oracle arm runs on rank 0 alone; other ranks exit without work
        if int(os.environ.get("RANK", "0")) == 0:
            print(json.dumps(run_reference(args, 0, int(os.environ.get("WORLD_SIZE", "1")),
                                           int(os.environ.get("LOCAL_RANK", "0")))))
        return
    rank, ws, local = dist_init(args.gpus)
    if args.only_kernel:
        print(json.dumps(run_kernel_only(args, local)))
        return
    if args.timeline:
        print(json.dumps(run_timeline(args, local)))
        return
    res = run_ours(args, rank, ws, local)
    if rank == 0:
        print(json.dumps(res))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
