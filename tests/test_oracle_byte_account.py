"""Pins of the oracle's byte account to the values the ByteCross README prints."""
import json
import os

import pytest

from oracle import byte_account as ba
from synth import LLAMA_8B, TINY

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "byte_account.json")))
MODELS = {k: dict(v, page=16) for k, v in GOLD["models"].items()}


def _rounds_to(value, printed, digits):
    return round(value, digits) == pytest.approx(printed, abs=10 ** -(digits + 3))


@pytest.mark.parametrize("case", GOLD["crossover_k"], ids=lambda c: f"{c['model']}-{c['rp']}-{c['rkv']}")
def test_crossover_printed(case):
    n = ba.crossover(MODELS[case["model"]], case["rp"], case["rkv"]) / 1024
    assert _rounds_to(n, case["printed"], case["digits"]), n


@pytest.mark.parametrize("case", GOLD["crossover_ff_k"], ids=lambda c: c["model"])
def test_crossover_ff_printed(case):
    n = ba.crossover(MODELS[case["model"]], case["rp"], case["rkv"], ff_only=True) / 1024
    assert _rounds_to(n, case["printed"], case["digits"]), n


@pytest.mark.parametrize("case", GOLD["bound"], ids=lambda c: f"{c['n']}-{c['rp']}-{c['rkv']}")
def test_bound_printed(case):
    b = ba.bound(MODELS[case["model"]], case["n"], case["rp"], case["rkv"])
    assert _rounds_to(b, case["printed"], case["digits"]), b


def test_bound_needs_lm_head():
    """The printed 1.60x only comes out with the LM head inside B_total: a
    plausible slip (leaving it out) must fail this pin."""
    m = MODELS["llama-3.1-8b"]
    n, rkv = 131072, 0.3
    b_no_head = ba.weight_bytes(m) + n * ba.kv_bytes_per_token(m)
    wrong = b_no_head / (b_no_head - (1 - rkv) * n * ba.kv_bytes_per_token(m))
    assert round(wrong, 2) != 1.60
    assert round(ba.bound(m, n, rkv=rkv), 2) == 1.60


def test_crossover_batch_printed():
    c = GOLD["crossover_batch_k"][0]
    n = ba.crossover_batch(MODELS[c["model"]], c["union_keep"], c["rkv"], c["batch"]) / 1024
    assert _rounds_to(n, c["printed"], c["digits"]), n


def test_matched_crossover_printed():
    g = GOLD["matched_crossover_k"]
    proj = {float(k): v for k, v in g["proj"].items()}
    sel = {float(k): v for k, v in g["sel"].items()}
    for case in g["cases"]:
        n = ba.matched_crossover(MODELS[g["model"]], proj, sel, case["budget"]) / 1024
        assert _rounds_to(n, case["printed"], g["digits"]), (case, n)


def test_exact_token_counts():
    """The reconstructed crossovers are whole-token values for the 8B shape."""
    m = MODELS["llama-3.1-8b"]
    assert ba.params_per_layer(m) == 218103808
    assert ba.crossover(m, 0.5, 0.5) == pytest.approx(106496)
    assert ba.crossover(m, 0.5, 0.3, ff_only=True) == pytest.approx(61440)


def test_equal_savings_at_crossover():
    """Definition of Equation 5: at n* both branches save the same bytes."""
    for rp, rkv in ((0.7, 0.3), (0.5, 0.3), (0.5, 0.5)):
        n = ba.crossover(LLAMA_8B, rp, rkv)
        assert (1 - rp) * ba.weight_bytes(LLAMA_8B) == pytest.approx(
            (1 - rkv) * n * ba.kv_bytes_per_token(LLAMA_8B), rel=1e-12)


def test_implementation_bytes_dense_matches_paper_form():
    """Dense-mode implementation bytes equal W + H + (n+1)*kv_tok plus the
    small terms (norm gains, embedding row, logits, KV append)."""
    for cfg in (TINY, LLAMA_8B):
        for n in (0, 15, 16, 2047, 32768):
            imp = ba.implementation_bytes(cfg, "dense", n)
            assert imp["weights"] == ba.weight_bytes(cfg)
            assert imp["head"] == ba.head_bytes(cfg)
            assert imp["kv_read"] == (n + 1) * ba.kv_bytes_per_token(cfg)
            assert imp["meta_read"] == 0


def test_implementation_bytes_keep_one_is_dense():
    for mode in ("act", "kv", "both"):
        a = ba.implementation_bytes(TINY, mode, 2047, rp=1.0, rkv=1.0)
        b = ba.implementation_bytes(TINY, "dense", 2047)
        assert a["weights"] == b["weights"] and a["kv_read"] == b["kv_read"]


def test_implementation_bytes_brute_force_tiny():
    """KV bytes of a small selection, counted token by token."""
    cfg = dict(TINY, n_layers=1, n_kv_heads=1)
    n, rkv, sinks, recent = 100, 0.5, 1, 2        # 101 tokens -> 7 pages
    P = 7
    K = 4                                           # ceil(3.5)
    imp = ba.implementation_bytes(cfg, "kv", n, rkv=rkv, sinks=sinks, recent=recent)
    # pages 0, 5, 6 forced + one scored full page; page 6 holds 101-96 = 5 tokens
    tokens = 16 + 16 + 5 + 16
    assert imp["kv_read"] == tokens * 2 * cfg["head_dim"] * 2
    assert imp["meta_read"] == P * 2 * cfg["head_dim"] * 2
    assert ba.page_keep(P, rkv, sinks, recent) == (K, 3)
