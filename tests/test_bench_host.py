"""Host-side logic of the benchmark, on CPU: the measured crossing's linear
interpolation, the cost-aware fit (it must recover a bandwidth and per-mode
fixed costs it was built from, and predict the crossing of that model), the
byte-account crossing by bisection, the per-site labels of a traced step,
the clocks record of the timed windows and the source-hash check of the
roofline's DRAM traffic."""
import pytest

import activation_kv_sparsity_b200 as bc
import bench
from synth import LLAMA_8B

CTX = (2048, 8192, 32768, 65536, 131072)


def test_measured_crossing_interpolates_linearly():
    cells = {}
    for n, (a, k) in zip(CTX, [(3.0, 3.7), (3.2, 4.0), (3.6, 4.1), (4.3, 4.4), (5.5, 5.0)]):
        cells[("act", n)] = {"ms_per_step": a}
        cells[("kv", n)] = {"ms_per_step": k}
    got = bench.measured_crossing(cells, CTX)["act_vs_kv_tokens"]
    # act - kv: -0.1 at 64K, +0.5 at 128K -> 65536 + 65536 * 0.1 / 0.6
    assert got == pytest.approx(65536 + 65536 * 0.1 / 0.6, abs=0.1)


def test_measured_crossing_absent():
    cells = {(m, n): {"ms_per_step": 1.0 if m == "act" else 2.0} for m in ("act", "kv") for n in CTX}
    assert bench.measured_crossing(cells, CTX)["act_vs_kv_tokens"] is None
    assert bench.measured_crossing({}, CTX) == {"act_vs_kv_tokens": None}


def _model_cells(bw_gbs, cost_ms):
    cells = {}
    for m in ("dense", "act", "kv"):
        for n in CTX:
            b = bc.byte_account(LLAMA_8B, m, n, **{k: v for k, v in bench.KEEP.items()
                                                  if m != "dense" or k in ("sinks", "recent")})["impl_total_bytes"]
            cells[(m, n)] = {"bytes_per_step": b, "ms_per_step": b / (bw_gbs * 1e9) * 1e3 + cost_ms[m]}
    return cells


def test_cost_aware_fit_recovers_its_model():
    costs = {"dense": 1.3, "act": 1.9, "kv": 1.6}
    cells = _model_cells(6700.0, costs)
    fit = bench.cost_aware_prediction(cells, CTX, LLAMA_8B, bc)
    assert fit["fit_gbs"] == pytest.approx(6700.0, rel=1e-6)
    for m, c in costs.items():
        assert fit["fixed_cost_ms"][m] == pytest.approx(c, abs=1e-3)
    n = fit["predicted_act_vs_kv_tokens"]

    def t(mode, ctx):
        kw = dict(bench.KEEP)
        return bc.byte_account(LLAMA_8B, mode, ctx, **kw)["impl_total_bytes"] / 6700e9 * 1e3 + costs[mode]
    assert t("act", n - 1) < t("kv", n - 1) and t("act", n) >= t("kv", n)


def test_cost_aware_fit_needs_all_modes():
    cells = _model_cells(6700.0, {"dense": 1.0, "act": 1.0, "kv": 1.0})
    del cells[("kv", 2048)]
    assert bench.cost_aware_prediction(cells, CTX, LLAMA_8B, bc) is None


def test_impl_crossing_is_where_the_byte_counts_meet():
    n = bench.impl_crossing(bc, LLAMA_8B, 0.5, 0.3)

    def diff(ctx):
        a = bc.byte_account(LLAMA_8B, "act", ctx, rp=0.5)["impl_total_bytes"]
        k = bc.byte_account(LLAMA_8B, "kv", ctx, rkv=0.3)["impl_total_bytes"]
        return a - k
    assert diff(n - 1) < 0 <= diff(n)
    # the paper form's n* (Equation 5) is below it: the page bounds cost the KV branch bytes
    assert bc.byte_account(LLAMA_8B, "both", 0, rp=0.5, rkv=0.3)["n_star"] < n


def test_site_labels_follow_the_projection_order():
    names = ["k_select_cta", "k_gemv", "k_pages", "k_page_select_cta", "k_attn", "k_select_cta", "k_gemv",
             "k_select_cta", "k_gemv", "k_select", "k_gemv", "k_lmhead"]
    sites, gemvs = [], 0
    for nm in names:
        sites.append(bench.site_of(nm, gemvs))
        gemvs += "k_gemv" in nm
    assert sites == ["sel_qkv", "qkv", "page_scores", "page_select", "attn", "sel_o", "o", "sel_gate_up",
                     "gate_up", "sel_down", "down", "k_lmhead"]


def test_crossing_of_first_sign_change():
    assert bench.crossing_of([(0, -2.0), (10, -1.0), (20, 1.0), (30, -1.0)]) == pytest.approx(15.0)
    assert bench.crossing_of([(0, 1.0), (10, 2.0)]) is None
    assert bench.crossing_of([(0, -1.0), (10, 0.0)]) == pytest.approx(10.0)


def test_sweep_fit_recovers_costs_and_predicts_every_pair():
    """The sweep's cost-aware model (one bandwidth, a fixed cost per cell
    kind) is recovered from cells built from it, its predicted crossing per
    keep pair is where the model's act and kv times meet, and the crossing
    measured on those cells by linear interpolation lies within one sweep
    step of it."""
    costs = {"dense": 1.30, "act@0.7": 1.80, "act": 1.90, "kv": 1.60, "kv@0.5": 1.55}
    ctx = sorted(bench.SWEEP_CONTEXTS)
    cells = {}
    for c in bench.SWEEP_CELLS:
        lib = bench.CELLS[c][0]
        for n in ctx:
            b = bc.byte_account(LLAMA_8B, lib, n, **bench.cell_kw(c))["impl_total_bytes"]
            cells[(c, n)] = {"bytes_per_step": b, "ms_per_step": b / 6600e9 * 1e3 + costs[c]}
    inv_bw, fitted = bench.cost_aware_fit(cells, ctx, bench.SWEEP_CELLS)
    assert 1.0 / inv_bw == pytest.approx(6600.0, rel=1e-6)
    for c, v in costs.items():
        assert fitted[c] * 1e3 == pytest.approx(v, abs=1e-6)
    for (rp, rkv), (ca, ck) in bench.CROSS_CELLS.items():
        pred = bench.predicted_crossing(bc, LLAMA_8B, inv_bw, fitted, ca, ck)
        meas = bench.crossing_of([(n, cells[(ca, n)]["ms_per_step"] - cells[(ck, n)]["ms_per_step"]) for n in ctx])
        if pred is None or pred > max(ctx):
            assert meas is None
            continue
        assert abs(meas - pred) <= 4096, (rp, rkv, meas, pred)


def test_crossing_report_names_a_crossing_outside_the_sweep():
    """When the kv branch is already faster at the sweep's first context the
    report says the crossing lies below it instead of leaving it blank."""
    ctx = [2048, 4096, 8192]
    block = {}
    for n in ctx:
        block[("act@0.7", n)] = {"ms_per_step": 4.0, "bytes_per_step": 1e9}
        block[("kv", n)] = {"ms_per_step": 3.9, "bytes_per_step": 1e9}
        for c in ("dense", "act", "kv@0.5"):
            block[(c, n)] = {"ms_per_step": 4.0, "bytes_per_step": 1e9}
    rep = bench.crossing_report(bc, LLAMA_8B, {}, [], [block], ctx, 8)
    row = rep["pairs"]["0.7/0.3"]
    assert row["measured_tokens"] is None
    assert row["measured_outside_sweep"].startswith("below 2048")


def test_clock_summary_keeps_samples_inside_the_timed_windows():
    """The clocks record: median SM clock and the throttle reasons seen
    while timing, samples outside the windows ignored."""
    c = bench.Clocks.__new__(bench.Clocks)          # no nvidia-smi process
    c.proc = None
    c.windows = [(10.0, 20.0)]
    idle = ["Not Active"] * 4

    def row(mhz, reasons):
        return [str(mhz), "1965", "900"] + reasons
    c.samples = [(5.0, row(700, ["Active"] * 4)),                     # before the window
                 (11.0, row(1965, idle)),
                 (12.0, row(1900, ["Not Active", "Not Active", "Not Active", "Active"])),
                 (13.0, row(1965, idle)),
                 (25.0, row(500, ["Active", "Not Active", "Not Active", "Not Active"]))]   # after it
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_without_samples():
    c = bench.Clocks.__new__(bench.Clocks)
    c.proc, c.windows, c.samples = None, [(0.0, 1.0)], []
    assert c.summary()["reasons"] == ["no samples"]


def test_traffic_record_is_void_once_the_source_changes(tmp_path, monkeypatch):
    """The roofline's DRAM traffic is reported only while the kernel source
    still hashes to the one the ncu capture was taken of."""
    import hashlib
    import json
    csrc = tmp_path / "activation_kv_sparsity_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "gemv.cu"
    src.write_text("// kernel v1\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    rec = {"k_gemv_gateup": {"source": "gemv.cu", "source_sha": sha, "dram_bytes_per_launch": 123}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k_gemv_gateup") == 123
    assert bench.traffic_record("k_other") is None
    src.write_text("// kernel v2\n")
    assert bench.traffic_record("k_gemv_gateup") is None
