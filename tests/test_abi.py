"""The C ABI without a GPU: the library loads, exports every declared symbol,
validates arguments on the host, and its byte account agrees with the
oracle's (and so with the values the ByteCross README prints)."""
import ctypes as C
import json
import os
import re

import pytest

import activation_kv_sparsity_b200 as bc
from oracle import byte_account as ba
from synth import LLAMA_8B, TINY

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bytecross.h")
GOLD = json.load(open(os.path.join(ROOT, "tests", "golden", "byte_account.json")))


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"BC_API\s+[\w\s\*]+?\b(bc_\w+)\s*\(", text)


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 20
    lib = C.CDLL(bc.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_no_undeclared_exports():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", bc.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line and line.split()[-1].startswith("bc_")}
    assert exported == set(declared_symbols())


def _cfg(d, max_ctx=4096):
    return bc.config(d, max_ctx)


def test_size_queries():
    c = _cfg(LLAMA_8B, 131072 + 64)
    P = (131072 + 64 + 15) // 16
    assert bc.bc_kv_pool_bytes(C.byref(c)) == 32 * 8 * P * 2 * 16 * 128 * 2
    assert bc.bc_meta_pool_bytes(C.byref(c)) == 32 * 8 * P * 2 * 128 * 2
    assert 0 < bc.bc_workspace_bytes(C.byref(c)) < 256 << 20
    bad = _cfg(dict(TINY, head_dim=96, hidden=768))
    assert bc.bc_kv_pool_bytes(C.byref(bad)) == 0
    assert bc.bc_workspace_bytes(C.byref(bad)) == 0


@pytest.mark.parametrize("field,value", [("page", 32), ("head_dim", 80), ("n_kv_heads", 3), ("hidden", 500),
                                         ("max_ctx", 0), ("rms_eps", 0.0)])
def test_model_create_rejects_bad_config(field, value):
    c = _cfg(TINY)
    setattr(c, field, value)
    w = bc.bc_weights(*([C.c_void_p(256)] * 9))
    h = C.c_void_p()
    st = bc.bc_model_create(C.byref(c), C.byref(w), C.c_void_p(256), C.c_void_p(256), C.c_void_p(256),
                            1 << 30, None, C.byref(h))
    assert st == bc.BC_EINVAL
    assert bc.bc_last_error()
    assert h.value is None


def test_model_create_rejects_null_and_small_workspace():
    c = _cfg(TINY)
    w = bc.bc_weights(*([C.c_void_p(256)] * 9))
    h = C.c_void_p()
    assert bc.bc_model_create(C.byref(c), C.byref(w), None, C.c_void_p(256), C.c_void_p(256), 1 << 30, None,
                              C.byref(h)) == bc.BC_EINVAL
    w0 = bc.bc_weights(*([C.c_void_p(256)] * 8 + [None]))
    assert bc.bc_model_create(C.byref(c), C.byref(w0), C.c_void_p(256), C.c_void_p(256), C.c_void_p(256), 1 << 30,
                              None, C.byref(h)) == bc.BC_EINVAL
    assert bc.bc_model_create(C.byref(c), C.byref(w), C.c_void_p(256), C.c_void_p(256), C.c_void_p(256), 16,
                              None, C.byref(h)) == bc.BC_ENOMEM
    assert bc.bc_model_create(C.byref(c), C.byref(w), C.c_void_p(260), C.c_void_p(256), C.c_void_p(256), 1 << 30,
                              None, C.byref(h)) == bc.BC_EINVAL


def test_single_kernel_entries_validate_on_host():
    assert bc.bc_gemv_scratch_bytes(300) == 0
    assert bc.bc_gemv(None, 4, 256, None, None, 4, None, None, 0, None) == bc.BC_EINVAL
    assert bc.bc_select_topk(C.c_void_p(256), 20000, 5, C.c_void_p(256), None) == bc.BC_EINVAL
    assert bc.bc_select_topk(C.c_void_p(256), 100, 0, C.c_void_p(256), None) == bc.BC_EINVAL
    p = C.c_void_p(256)
    assert bc.bc_attention(p, p, 8, 4, 96, 10, None, 1, 16, p, p, 1 << 20, None) == bc.BC_EINVAL


def test_batched_gemv_validates_on_host():
    p = C.c_void_p(256)
    big = 1 << 30
    assert bc.bc_gemv_batch_scratch_bytes(4096, 300, 4) == 0
    assert bc.bc_gemv_batch_scratch_bytes(4096, 512, 9) == 0
    assert bc.bc_gemv_batch_scratch_bytes(20000, 512, 2) == 0
    assert bc.bc_gemv_batch_scratch_bytes(4096, 512, 4) > 4 * 4096 * 4
    # batch out of range, d_out not a multiple of 256, k > d_in, no idx with
    # k < d_in, scratch too small: rejected before any launch
    assert bc.bc_gemv_batch(p, 64, 256, p, p, 8, 0, p, None, p, big, None) == bc.BC_EINVAL
    assert bc.bc_gemv_batch(p, 64, 256, p, p, 8, 9, p, None, p, big, None) == bc.BC_EINVAL
    assert bc.bc_gemv_batch(p, 64, 300, p, p, 8, 2, p, None, p, big, None) == bc.BC_EINVAL
    assert bc.bc_gemv_batch(p, 64, 256, p, p, 65, 2, p, None, p, big, None) == bc.BC_EINVAL
    assert bc.bc_gemv_batch(p, 64, 256, p, None, 8, 2, p, None, p, big, None) == bc.BC_EINVAL
    assert bc.bc_gemv_batch(None, 64, 256, p, p, 8, 2, p, None, p, big, None) == bc.BC_EINVAL
    need = bc.bc_gemv_batch_scratch_bytes(64, 256, 2)
    assert bc.bc_gemv_batch(p, 64, 256, p, p, 8, 2, p, None, p, need - 1, None) == bc.BC_ENOMEM


MODELS = {k: dict(v, page=16) for k, v in GOLD["models"].items()}


@pytest.mark.parametrize("case", GOLD["crossover_k"], ids=lambda c: f"{c['model']}-{c['rp']}-{c['rkv']}")
def test_library_crossover_matches_printed(case):
    got = bc.byte_account(MODELS[case["model"]], "both", 1024, rp=case["rp"], rkv=case["rkv"])
    assert round(got["n_star"] / 1024, case["digits"]) == pytest.approx(case["printed"])
    assert got["n_star"] == pytest.approx(ba.crossover(MODELS[case["model"]], case["rp"], case["rkv"]), rel=1e-6)


def test_library_crossover_batch_matches_printed_and_oracle():
    c = GOLD["crossover_batch_k"][0]
    m = MODELS[c["model"]]
    got = bc.crossover_batch(m, c["union_keep"], c["rkv"], c["batch"])
    assert round(got / 1024, c["digits"]) == pytest.approx(c["printed"])
    for keep, rkv, batch in [(0.92, 0.3, 4), (0.75, 0.5, 2), (0.996, 0.2, 8), (0.5, 0.3, 1)]:
        assert got_eq(bc.crossover_batch(m, keep, rkv, batch), ba.crossover_batch(m, keep, rkv, batch))
    # batch 1 with union_keep = rp is Equation 5's crossover
    assert got_eq(bc.crossover_batch(m, 0.5, 0.3, 1), ba.crossover(m, 0.5, 0.3))
    out = C.c_double()
    cfg = bc.config(m, 1)
    assert bc.bc_crossover_batch(C.byref(cfg), 0.0, 0.3, 4, C.byref(out)) == bc.BC_EINVAL
    assert bc.bc_crossover_batch(C.byref(cfg), 0.9, 1.0, 4, C.byref(out)) == bc.BC_EINVAL
    assert bc.bc_crossover_batch(C.byref(cfg), 0.9, 0.3, 0, C.byref(out)) == bc.BC_EINVAL


def got_eq(a, b):
    return a == pytest.approx(b, rel=1e-12)


def test_library_bound_and_ff_match_printed():
    m = MODELS["llama-3.1-8b"]
    assert round(bc.byte_account(m, "kv", 131072, rkv=0.3)["bound"], 2) == 1.60
    assert round(bc.byte_account(m, "both", 32768, rp=0.5, rkv=0.2)["bound"], 3) == 2.172
    assert round(bc.byte_account(m, "both", 0, rp=0.5, rkv=0.3)["n_star_ff"] / 1024, 1) == 60.0


@pytest.mark.parametrize("mode", ["dense", "act", "kv", "both", "snap"])
@pytest.mark.parametrize("n", [0, 15, 16, 2047, 8191, 32768, 131071])
@pytest.mark.parametrize("cfg", [TINY, LLAMA_8B], ids=["tiny", "8b"])
def test_library_implementation_bytes_match_oracle(cfg, mode, n):
    kw = dict(rp=0.5, rkv=0.3, sinks=1, recent=16)
    got = bc.byte_account(cfg, mode, n, **kw)
    ref = ba.implementation_bytes(cfg, mode, n, **kw)
    assert got["impl_weight_bytes"] == ref["weights"]
    assert got["impl_head_bytes"] == ref["head"]
    assert got["impl_kv_read_bytes"] == ref["kv_read"]
    assert got["impl_meta_read_bytes"] == ref["meta_read"]
    assert got["impl_kv_write_bytes"] == ref["kv_write"]
    assert got["impl_other_bytes"] == ref["other"]
    assert got["impl_total_bytes"] == ref["total"]


def test_byte_account_rejects_bad_ratios():
    c = _cfg(TINY)
    out = bc.bc_bytes()
    assert bc.bc_byte_account(C.byref(c), bc.BC_KV, 1.0, 0.0, 100, 1, 16, 16, C.byref(out)) == bc.BC_EINVAL
    assert bc.bc_byte_account(C.byref(c), bc.BC_ACT, 1.5, 1.0, 100, 1, 16, 16, C.byref(out)) == bc.BC_EINVAL
    assert bc.bc_byte_account(C.byref(c), bc.BC_KV, 1.0, 0.5, 100, 1, 0, 16, C.byref(out)) == bc.BC_EINVAL


@pytest.mark.parametrize("n", [20463, 20464, 20479, 40959, 81919])
@pytest.mark.parametrize("mode,rp,rkv", [("kv", 1.0, 0.3), ("both", 0.7, 0.3), ("snap", 1.0, 0.3),
                                         ("kv", 1.0, 0.7), ("both", 0.3, 0.1)])
def test_library_keep_counts_where_float_ratios_round_up(n, mode, rp, rkv):
    """At P a multiple of 10 (1280, 2560, 5120 pages) r*P is an integer; the
    library takes its ratios as doubles and keeps exactly the oracle's count
    (a float32 ratio would keep one more page)."""
    kw = dict(rp=rp, rkv=rkv, sinks=1, recent=16)
    got = bc.byte_account(LLAMA_8B, mode, n, **kw)
    ref = ba.implementation_bytes(LLAMA_8B, mode, n, **kw)
    assert got["impl_kv_read_bytes"] == ref["kv_read"]
    assert got["impl_total_bytes"] == ref["total"]
    if mode != "snap":
        P = -(-(n + 1) // 16)
        assert got["pages_kept"] == ba.page_keep(P, rkv, 1, 16)[0]


def test_batch_entries_validate_on_host():
    c = _cfg(TINY, 4096)
    assert bc.bc_batch_workspace_bytes(C.byref(c), 0) == 0
    assert bc.bc_batch_workspace_bytes(C.byref(c), 9) == 0
    w1 = bc.bc_batch_workspace_bytes(C.byref(c), 1)
    w4 = bc.bc_batch_workspace_bytes(C.byref(c), 4)
    assert 0 < w1 < w4
    bad = _cfg(dict(TINY, head_dim=96, hidden=768))
    assert bc.bc_batch_workspace_bytes(C.byref(bad), 2) == 0
    w = bc.bc_weights(*([C.c_void_p(256)] * 9))
    h = C.c_void_p()
    p = C.c_void_p(256)
    assert bc.bc_batch_create(C.byref(c), C.byref(w), 9, p, p, p, 1 << 40, None, C.byref(h)) == bc.BC_EINVAL
    assert bc.bc_batch_create(C.byref(c), C.byref(w), 2, None, p, p, 1 << 40, None, C.byref(h)) == bc.BC_EINVAL
    assert bc.bc_batch_create(C.byref(c), C.byref(w), 2, p, p, p, 16, None, C.byref(h)) == bc.BC_ENOMEM
    assert bc.bc_batch_create(C.byref(c), C.byref(w), 2, C.c_void_p(260), p, p, 1 << 40, None,
                              C.byref(h)) == bc.BC_EINVAL
    assert h.value is None
    toks = (C.c_int * 2)(1, 2)
    assert bc.bc_batch_step(None, toks, bc.BC_DENSE, 1.0, 1.0, 1, 16, 16, p) == bc.BC_EINVAL
