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
MODE_KW = {"dense": dict(), "act": dict(rp=0.5), "kv": dict(rkv=0.3, sinks=1, recent=16),
           "both": dict(rp=0.5, rkv=0.3, sinks=1, recent=16),
           # the pages' KV window baseline: the kv mode with no scored pages
           # (K = |F|: the sink page and the 16 recent pages)
           "window": dict(rkv=1e-6, sinks=1, recent=16),
           # the pages' own KV mode: one selection after prefill (16 observation
           # positions per query head), then steps over the frozen pages
           "snap": dict(rkv=0.3, sinks=1, recent=16)}
SNAP_OBS = 16
LIB_MODE = {"window": "kv"}                          # bench cells that run a library mode
CROSS_PAIRS = ((0.7, 0.3), (0.5, 0.3), (0.5, 0.5))


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

def run_ours(args, rank, ws, local):
    import torch
    import activation_kv_sparsity_b200 as bc
    from synth import LLAMA_8B, kv_chunks, make_weights, obs_queries

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = LLAMA_8B
    contexts = sorted(set(args.contexts), reverse=True)
    steps, warm = args.steps, args.warmup
    max_ctx = max(contexts) + warm + steps + 32
    w = make_weights(cfg, seed=0, device=dev)
    model = bc.Model(cfg, w, max_ctx)
    for k, v in kv_chunks(cfg, max(contexts), seed=1, device=dev):
        model.append(k, v)
    torch.cuda.synchronize()
    stream = model.stream
    logits = torch.empty(cfg["vocab"], device=dev)
    toks = [(1 + 7919 * i) % cfg["vocab"] for i in range(warm + steps)]
    props = torch.cuda.get_device_properties(dev)
    clocks = Clocks(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local))
    peak, peak_kind = peaks()

    q_obs = obs_queries(cfg, SNAP_OBS, device=dev) if "snap" in args.modes else None
    snap_select_ms = {}

    def time_cell(mode, n):
        kw = MODE_KW[mode]
        lib = LIB_MODE.get(mode, mode)
        model.reset(n)
        if mode == "snap":
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
        for i in range(steps):
            model.step(toks[warm + i], lib, logits, **kw)
        host_enqueue[(mode, n)] = (time.perf_counter() - h0) * 1e3 / steps
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.window(t0, time.time())
        barrier(ws)
        ms = max_over_ranks(e0.elapsed_time(e1) / steps, ws, dev)
        return ms, model.launches() - l0

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
    host_enqueue = {}
    for n in contexts:
        if n == HEAD_CTX or (e2e is None and n == min(contexts)):
            e2e = time_e2e(n)
        for mode in args.modes:
            ms, launches = time_cell(mode, n)
            kw = dict(KEEP)
            kw.update(MODE_KW[mode])
            # the timed steps run at contexts n+warm .. n+warm+steps-1: average their byte accounts
            accs = [bc.byte_account(cfg, LIB_MODE.get(mode, mode), n + warm + i, **kw) for i in range(steps)]
            acc = dict(accs[0])
            acc["impl_total_bytes"] = sum(a["impl_total_bytes"] for a in accs) / steps
            if mode == "snap":
                # the step right after the selection at n, plus every token
                # appended since (each is read: frozen partial page, new pages)
                base = bc.byte_account(cfg, "snap", n, **kw)["impl_total_bytes"]
                tok_bytes = cfg["n_layers"] * cfg["n_kv_heads"] * 2 * cfg["head_dim"] * 2
                acc["impl_total_bytes"] = base + tok_bytes * (warm + (steps - 1) / 2.0)
            gbs = acc["impl_total_bytes"] / (ms * 1e-3) / 1e9
            cells[(mode, n)] = dict(mode=mode, context=n, ms_per_step=round(ms, 4),
                                    tok_s=round(1000.0 / ms, 2), bytes_per_step=acc["impl_total_bytes"],
                                    gbs=round(gbs, 1), frac_of_measured_peak=round(gbs / peak, 4),
                                    paper_bound=round(acc["bound"], 4), launches_per_step=launches // steps,
                                    host_enqueue_ms=round(host_enqueue[(mode, n)], 4))
            if mode == "snap":
                cells[(mode, n)]["selection_ms_once"] = round(snap_select_ms[n], 3)
    for n in contexts:
        if ("dense", n) not in cells:
            continue
        d = cells[("dense", n)]["ms_per_step"]
        for mode in ("act", "kv", "both", "window", "snap"):
            if (mode, n) in cells:
                cells[(mode, n)]["speedup_vs_dense"] = round(d / cells[(mode, n)]["ms_per_step"], 4)

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
    for l in range(4):
        bc.gemv(wgu[l], xin, idx, y, scratch, stream)
    torch.cuda.synchronize()
    reps = 4
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        for l in range(cfg["n_layers"]):
            bc.gemv(wgu[l], xin, idx, y, scratch, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    gemv_ms = e0.elapsed_time(e1) / (reps * cfg["n_layers"])
    gemv_bytes = kq * d_out * 2 + kq * 8            # weight rows + index/activation reads
    achieved = gemv_bytes / (gemv_ms * 1e-3) / 1e9

    # attention at the headline context: dense page list of one layer
    # (second kernel of interest), timed through the single-kernel entry
    # point over 8 layers' pages
    attn = None

    clk = clocks.summary()
    # measured crossing against the byte account: the paper form (Equation 5)
    # and this implementation's bytes (which add the page bounds the scorer reads)
    crossings = {}
    for rp, rkv in CROSS_PAIRS:
        acc = bc.byte_account(cfg, "both", 1024, rp=rp, rkv=rkv)
        crossings[f"{rp}/{rkv}"] = {"n_star_tokens": round(acc["n_star"], 1),
                                    "n_star_impl_tokens": impl_crossing(bc, cfg, rp, rkv)}
    cross_measured = measured_crossing(cells, contexts)
    cross_measured["cost_aware_prediction"] = cost_aware_prediction(cells, contexts, cfg, bc)

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
        "crossings": {"byte_account": crossings, "measured": cross_measured},
    }
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args, w, head_ctx)
    del attn
    model.close()
    return result


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


def cost_aware_prediction(cells, contexts, cfg, bc):
    """The pages' cost-aware prediction restated for this library: per mode,
    step time = byte-account bytes / B + c (one bandwidth B for all modes,
    one fixed per-step kernel cost c per mode), fitted by least squares over
    the sampled contexts; the predicted crossing is where the act and kv fits
    meet.  Returns the fit and the predicted crossing in tokens."""
    import numpy as np
    modes = [m for m in ("dense", "act", "kv") if all((m, n) in cells for n in contexts)]
    if len(modes) < 3:
        return None
    rows, ys = [], []
    for j, m in enumerate(modes):
        for n in contexts:
            c = cells[(m, n)]
            r = [c["bytes_per_step"] / 1e9] + [1.0 if k == j else 0.0 for k in range(len(modes))]
            rows.append(r)
            ys.append(c["ms_per_step"] * 1e-3)
    sol, *_ = np.linalg.lstsq(np.array(rows), np.array(ys), rcond=None)
    inv_bw, costs = sol[0], dict(zip(modes, sol[1:]))
    kw = dict(KEEP)

    def t(mode, n):
        return bc.byte_account(cfg, mode, n, **kw)["impl_total_bytes"] / 1e9 * inv_bw + costs[mode]
    lo, hi = 1, 1 << 21
    if (t("act", lo) - t("kv", lo)) * (t("act", hi) - t("kv", hi)) > 0:
        pred = None
    else:
        while hi - lo > 1:
            mid = (lo + hi) // 2
            if t("act", mid) < t("kv", mid):
                lo = mid
            else:
                hi = mid
        pred = hi
    return {"fit_gbs": round(1.0 / inv_bw, 1),
            "fixed_cost_ms": {m: round(v * 1e3, 4) for m, v in costs.items()},
            "predicted_act_vs_kv_tokens": pred}


def measured_crossing(cells, contexts):
    """Context where the KV branch starts to beat the projection branch,
    interpolated linearly between the sampled contexts (the README's
    convention for latency crossings)."""
    ctx = sorted(contexts)
    if not all(("act", n) in cells and ("kv", n) in cells for n in ctx):
        return {"act_vs_kv_tokens": None}
    diff = [(n, cells[("act", n)]["ms_per_step"] - cells[("kv", n)]["ms_per_step"]) for n in ctx]
    for (n0, d0), (n1, d1) in zip(diff, diff[1:]):
        if d0 < 0 <= d1:
            return {"act_vs_kv_tokens": round(n0 + (n1 - n0) * (-d0) / (d1 - d0), 1),
                    "keep": "rp 0.5 (act) vs rkv 0.3 (kv)"}
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
    """The oracle as it stands, on the host cores: layers 0-3 of one decode
    step of the headline cell plus 1/32 of the LM head, scaled to a full step."""
    from synth import LLAMA_8B
    cfg = LLAMA_8B
    nl = 4
    wh, cache = host_sample_inputs(w_dev, n_ctx, nl)
    layer_s, head_s = [], 0.0
    for l in range(nl):
        a, b = oracle_sample(wh, cache, n_ctx, HEAD_MODE, l, cfg["vocab"] // 32)
        layer_s.append(a)
        head_s += b / nl
    step_s = statistics.mean(layer_s) * cfg["n_layers"] + head_s * 32
    return {"value": round(1.0 / step_s, 5), "unit": "tok/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"fp64 oracle, {HEAD_MODE} mode at {n_ctx} context: layers 0-{nl - 1} of one step "
                      f"(mean {statistics.mean(layer_s):.2f} s/layer) x {cfg['n_layers']} layers + 1/32 of the "
                      f"LM head x 32 ({head_s * 32:.2f} s)",
            "seconds_per_step": round(step_s, 2)}


def run_reference(args, rank, ws, local):
    """The oracle arm: each step is a bounded sample (one layer of the
    headline cell's step, rotating over layers 0-3, plus 1/32 of the LM head),
    scaled to a full step."""
    import torch
    from synth import LLAMA_8B, kv_chunks, make_weights
    cfg = LLAMA_8B
    nl = 4
    n_ctx = HEAD_CTX
    # inputs: drawn with the same generators; on the host when no GPU
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    small = dict(cfg, n_layers=nl)
    w = make_weights(small, seed=0, device=dev)

    class _Pool:          # the oracle reads token-major KV, filled from the draw
        pass
    from oracle import decoder as od
    from synth import bf16_bits
    cache = od.Cache(small, n_ctx + 1)
    for k, v in kv_chunks(small, n_ctx, seed=1, device=dev):
        cache.extend(bf16_bits(k), bf16_bits(v))
    wh = {name: bf16_bits(t) for name, t in w.items() if name not in ("embed", "lm_head")}
    wh["embed"] = bf16_bits(w["embed"][:16])
    wh["lm_head"] = bf16_bits(w["lm_head"][: cfg["vocab"] // 32])
    del w
    times = []
    for i in range(args.warmup + args.steps):
        a, b = oracle_sample(wh, cache, n_ctx, HEAD_MODE, i % nl, cfg["vocab"] // 32)
        if i >= args.warmup:
            times.append(a * cfg["n_layers"] + b * 32)
    step_s = statistics.mean(times)
    val = round(1.0 / step_s, 5)
    return {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tok/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_s * 1000, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"Llama-3.1-8B-shaped decode, 1 sequence, {n_ctx // 1024}K context, mode {HEAD_MODE} "
                               f"(rp 0.5, rkv 0.3, page 16, 1 sink page, 256 recent tokens)",
                   "global_batch": 1, "seq_len": n_ctx, "parallelism": "host cores"},
        "cpu_baseline": {"value": val, "unit": "tok/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": "per step: one layer of the step (layers 0-3 in turn) x 32 + 1/32 of the LM head x 32"},
        "e2e": {"value": val, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


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
        flops = 2 * 2 * c2["n_layers"] * c2["n_heads"] * 16 * n * c2["head_dim"]   # two passes, 2 per FMA

        def launch():
            model.snap_select(q_obs, rkv=0.3, sinks=1, recent=16)
        for _ in range(args.warmup):
            launch()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(model.stream)
        for _ in range(args.steps):
            launch()
        e1.record(model.stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        return {"kernel": "snap", "ms_per_selection": round(ms, 4), "flops": flops,
                "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                "note": "2 layers at 32K, both passes and the page select; mma.sync m16n8k16, bf16 keys, hi/lo-split queries"}
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
            bc.gemv(W, x, idx, y, scratch, stream)
    else:
        Hkv, G, hd, n_tok = cfg["n_kv_heads"], cfg["n_heads"] // cfg["n_kv_heads"], cfg["head_dim"], 131073
        P = -(-n_tok // 16)
        pool = torch.randn(Hkv, P, 2, 16, hd, generator=g, device=dev).to(torch.bfloat16)
        q = torch.randn(Hkv * G, hd, generator=g, device=dev)
        out = torch.empty(Hkv * G, hd, device=dev)
        scratch = torch.zeros(bc.bc_attention_scratch_bytes(Hkv * G, hd), dtype=torch.uint8, device=dev)
        nbytes = Hkv * n_tok * 2 * hd * 2

        def launch():
            bc.attention(q, pool, Hkv, G, hd, P, None, P, n_tok, out, scratch, stream)
    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        launch()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    peak, kind = peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": args.only_kernel, "ms_per_launch": round(ms, 5), "algorithmic_bytes": nbytes,
            "gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "peak": peak, "peak_kind": kind,
            "note": "includes the combine kernel" if args.only_kernel == "attention" else ""}


def run_batch_gemv(args, dev, stream, cfg):
    """The gate/up projection of one layer (4096 -> 28672 columns, rp 0.5)
    for a batch of B = 1, 2, 4, 8 sequences: one batched GEMV over the union
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
    for B in (1, 2, 4, 8):
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
    ap.add_argument("--modes", nargs="+", default=["dense", "act", "kv", "both", "window", "snap"],
                    choices=["dense", "act", "kv", "both", "window", "snap"])
    ap.add_argument("--timeline", choices=("dense", "act", "kv", "both"),
                    help="per-site cost of one step in this mode at the first --contexts value")
    ap.add_argument("--record-traffic", metavar="NCU_RAW_CSV",
                    help="write profiles/traffic.json from an ncu raw CSV of --only-kernel gemv_gateup")
    ap.add_argument("--only-kernel", choices=("gemv_gateup", "gemv_gateup_dense", "attention", "snap", "gemv_batch"),
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
