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


# ---------------------------------------------------------------- exact, hand-counted implementation bytes
# The implementation form feeds every bytes-per-step, GB/s and fraction of
# peak the benchmark reports, so each of its branches is pinned to numbers
# counted by hand here (the arithmetic is spelled out in the comments), not
# recomputed from the function's own formula.

ONE_LAYER_8B = dict(LLAMA_8B, n_layers=1, n_kv_heads=1, vocab=1)   # q/k/v cols (32 + 2) * 128 = 4352


def test_keep_count_rounding_byte_account():
    """The byte account's keep count: ceil(r*n - 1e-9), at least 1 (ByteCross
    README, "Usage: The byte account"; the north-star's ceil(rp*d_in))."""
    assert ba.keep_count(0.7, 4096) == 2868          # 2867.2 -> 2868 (a floor would give 2867)
    assert ba.keep_count(0.7, 14336) == 10036        # 10035.2 -> 10036
    assert ba.keep_count(0.5, 4096) == 2048
    assert ba.keep_count(0.5, 14336) == 7168
    assert ba.keep_count(0.3, 10) == 3               # 0.3*10 = 3.0000000000000004 in binary64
    assert ba.keep_count(0.3, 1280) == 384           # the product lands on an integer: no extra row
    assert ba.keep_count(1e-9, 4096) == 1
    assert ba.keep_count(1.0, 4096) == 4096


def test_act_weight_bytes_rp07_hand_counted():
    # rows kept: 2868 of the 4096-wide inputs (q/k/v, o, gate/up), 10036 of the 14336-wide one (down)
    # q/k/v 2868*4352 = 12,481,536; o 2868*4096 = 11,747,328; gate/up 2868*28672 = 82,231,296;
    # down 10036*4096 = 41,107,456; sum 147,567,616 elements, 2 bytes each
    imp = ba.implementation_bytes(ONE_LAYER_8B, "act", 100, rp=0.7)
    assert imp["weights"] == 295_135_232
    assert imp["meta_read"] == 0
    assert imp["kv_read"] == 101 * 2 * 128 * 2            # dense KV: every token of the one kv head


def test_act_weight_bytes_rp05_hand_counted():
    # 2048*4352 = 8,912,896; 2048*4096 = 8,388,608; 2048*28672 = 58,720,256; 7168*4096 = 29,360,128
    imp = ba.implementation_bytes(ONE_LAYER_8B, "act", 100, rp=0.5)
    assert imp["weights"] == 210_763_776


def test_both_bytes_hand_counted():
    # weights as in the rp 0.5 case; n = 100 -> 101 tokens, P = 7 pages (page 6 holds 5 tokens);
    # rkv 0.5 -> K = ceil(3.5) = 4: sink page 0, recent pages 5 and 6, one scored full page
    cfg = dict(ONE_LAYER_8B)
    imp = ba.implementation_bytes(cfg, "both", 100, rp=0.5, rkv=0.5, sinks=1, recent=2)
    assert imp["weights"] == 210_763_776
    assert imp["kv_read"] == (16 + 16 + 16 + 5) * 2 * 128 * 2    # 53 tokens, keys and values, bf16
    assert imp["meta_read"] == 7 * 2 * 128 * 2                   # kmin and kmax of every page
    # append: k and v rows (2*128*2) plus the page's rewritten bounds (2*128*2); the slot is
    # 100 % 16 = 4, so the 4 earlier keys of the page are re-read to recompute them
    assert imp["kv_write"] == 1024
    assert imp["other"] == 4 * 128 * 2 + 2 * 4096 * 2 + 4096 * 2 + 4096 * 2 + 4 * 1


def test_snap_bytes_hand_counted():
    """The step right after a once-after-prefill selection made at n."""
    cfg = dict(TINY, n_layers=1, n_kv_heads=1)                 # head_dim 64
    row = 2 * 64 * 2                                            # one token's key and value, bf16
    # n = 112: the selection saw 112 tokens = 7 full pages and kept K = max(3, ceil(3.5)) = 4;
    # the step's token 112 opens page 7 (1 token), read on top of the 4 kept full pages
    imp = ba.implementation_bytes(cfg, "snap", 112, rkv=0.5, sinks=1, recent=2)
    assert imp["kv_read"] == (4 * 16 + 1) * row
    assert imp["meta_read"] == 0
    # n = 100: 7 pages at the selection (page 6 holds 4 tokens), the token lands in page 6:
    # no page is opened, the kept set {0, 5, 6, one full page} now holds 16 + 16 + 5 + 16 tokens
    imp = ba.implementation_bytes(cfg, "snap", 100, rkv=0.5, sinks=1, recent=2)
    assert imp["kv_read"] == (16 + 16 + 5 + 16) * row
    # n = 113: the selection saw 8 pages (page 7 holds 1 token) and kept K = max(3, ceil(4 - 1e-9)) = 4:
    # pages 0, 6, 7 and one scored full page; the token lands in page 7, which then holds 2 tokens
    imp = ba.implementation_bytes(cfg, "snap", 113, rkv=0.5, sinks=1, recent=2)
    assert imp["kv_read"] == (16 + 16 + 2 + 16) * row


def test_page_keep_float_sensitive_counts():
    """Products that land on an integer keep exactly that many pages:
    0.3 * 1280 = 384 (a ratio rounded to float32, 0.300000012, would give 385)."""
    assert ba.page_keep(1280, 0.3, 1, 16) == (384, 17)
    assert ba.page_keep(2560, 0.3, 1, 16) == (768, 17)
    assert ba.page_keep(1280, 0.7, 1, 16) == (896, 17)
