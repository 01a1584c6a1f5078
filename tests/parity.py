"""Shared parity helpers for the GPU tests: run the library and the oracle on
the same seeded inputs and compare them the way the tests state."""
from __future__ import annotations

import math

import numpy as np
import torch

import activation_kv_sparsity_b200 as bc
from oracle import decoder as od
from synth import bf16_bits

SITES = (("qkv", bc.BC_TRACE_XN, bc.BC_TRACE_SEL_QKV), ("o", bc.BC_TRACE_ATTN, bc.BC_TRACE_SEL_O),
         ("gu", bc.BC_TRACE_XN2, bc.BC_TRACE_SEL_GU), ("d", bc.BC_TRACE_H, bc.BC_TRACE_SEL_D))

# Floating-point tolerance of hidden states and logits: max relative error
# ||gpu - oracle||_inf / ||oracle||_inf.  bf16 weights and KV, fp32
# accumulation on the device against fp64 on the host.
REL_TOL = 1e-2
# Near-tie allowance of a selection: an index may differ from the oracle's own
# choice only if the oracle's score of it lies within this relative distance
# of the cut score.
TIE_TOL = 1e-3


def max_rel(got, ref):
    return float(np.abs(np.asarray(got, np.float64) - ref).max() / max(np.abs(ref).max(), 1e-30))


def to_host(t):
    return t.detach().cpu().numpy().astype(np.float64)


def gpu_traces(model: bc.Model, L: int, kvsel: bool):
    """All per-layer traces of the last step, on the host."""
    out = []
    for l in range(L):
        r = {}
        for name, kind in (("xn", bc.BC_TRACE_XN), ("attn", bc.BC_TRACE_ATTN), ("xn2", bc.BC_TRACE_XN2),
                           ("h", bc.BC_TRACE_H), ("x", bc.BC_TRACE_X), ("q", bc.BC_TRACE_Q)):
            r[name] = to_host(model.trace(l, kind))
        for site, _, skind in SITES:
            r["s_" + site] = model.trace(l, skind).cpu().numpy().astype(np.int64)
        if kvsel:
            r["page_scores"] = model.trace(l, bc.BC_TRACE_PAGE_SCORES).cpu().numpy().astype(np.float64)
            r["pages"] = model.trace(l, bc.BC_TRACE_PAGES).cpu().numpy().astype(np.int64)
        out.append(r)
    return out


def forced_from(tr, act: bool, kvsel: bool):
    forced = {}
    for l, r in enumerate(tr):
        if act:
            for site, _, _ in SITES:
                forced[(l, site)] = r["s_" + site]
        if kvsel:
            for h in range(r["pages"].shape[0]):
                forced[(l, "pages", h)] = r["pages"][h]
    return forced


def topk_of(score, k):
    """The k largest entries of score, ties to the lower index, ascending."""
    order = np.lexsort((np.arange(score.size), -score))
    return np.sort(order[:k])


def pages_of(score, rkv, sinks, recent):
    """Forced pages (the first `sinks`, the last `recent`) plus the best
    scored others up to K = clamp(ceil(rkv*P - 1e-9), |F|, P), ascending."""
    P = score.size
    forced = sorted(set(range(min(sinks, P))) | set(range(max(P - recent, 0), P)))
    K = max(len(forced), min(P, math.ceil(rkv * P - 1e-9)))
    fset = set(forced)
    free = np.array([p for p in range(P) if p not in fset], dtype=np.int64)
    chosen = free[np.lexsort((free, -score[free]))[:K - len(forced)]] if K > len(forced) else []
    return np.sort(np.concatenate([np.asarray(forced, dtype=np.int64), np.asarray(chosen, dtype=np.int64)]))


def check_selection_exact(tr, rp, rkv, sinks, recent, act, kvsel):
    """Every GPU set is exactly the selection its own pre-selection scores
    define (a property of the GPU's output checked here, in the test, on the
    GPU's own fp32 values; the oracle never sees them)."""
    for l, r in enumerate(tr):
        if act:
            for site, _, _ in SITES:
                score = np.abs({"qkv": r["xn"], "o": r["attn"], "gu": r["xn2"], "d": r["h"]}[site])
                k = max(1, min(score.size, math.ceil(rp * score.size - 1e-9)))
                np.testing.assert_array_equal(topk_of(score, k), r["s_" + site],
                                              err_msg=f"layer {l} site {site}")
        if kvsel:
            for h in range(r["pages"].shape[0]):
                np.testing.assert_array_equal(pages_of(r["page_scores"][h], rkv, sinks, recent),
                                              r["pages"][h], err_msg=f"layer {l} kv head {h}")


def check_selection_near(own, gpu_set, cut_from_scores, k):
    """Elements where the oracle's own choice differs from the GPU's must be
    near-ties: oracle score within TIE_TOL of the cut score."""
    diff = np.setxor1d(own, gpu_set)
    if diff.size == 0:
        return 0
    s = cut_from_scores
    cut = np.sort(s)[::-1][k - 1]
    bad = [int(e) for e in diff if abs(s[e] - cut) > TIE_TOL * max(abs(cut), 1e-6)]
    assert not bad, f"selection differs beyond near-ties at {bad[:10]} (cut {cut})"
    return diff.size


def compare_step(cfg, w_bits, cache, token, mode, rp, rkv, sinks, recent, logits_gpu, tr, layers=None):
    """Checks the GPU's sets (exact on its own scores), then runs the oracle
    over the whole step from its own inputs, told only the GPU's index sets
    (integers: where fp32 and fp64 scores straddle a cut, both choices are
    correct), and compares every set with the oracle's own choice (near-ties
    only), the hidden states of `layers` (default all) and the logits.
    Returns the oracle's logits and trace."""
    act = mode in ("act", "both")
    kvsel = mode in ("kv", "both")
    check_selection_exact(tr, rp, rkv, sinks, recent, act, kvsel)
    trace = {}
    ref = od.decode_step(cfg, w_bits, cache, token, mode, rp=rp, rkv=rkv, sinks=sinks, recent=recent,
                         forced=forced_from(tr, act, kvsel), trace=trace)
    for l, r in enumerate(tr):
        if layers is None or l in layers:
            e = max_rel(r["x"], trace[l]["x"])
            assert e < REL_TOL, f"layer {l} hidden rel err {e}"
        if act:
            for site, _, _ in SITES:
                own_scores = np.abs({"qkv": trace[l]["xn"], "o": trace[l]["attn"], "gu": trace[l]["xn2"],
                                     "d": trace[l]["h"]}[site])
                k = len(r["s_" + site])
                own = np.sort(np.lexsort((np.arange(own_scores.size), -own_scores))[:k])
                check_selection_near(own, r["s_" + site], own_scores, k)
        if kvsel:
            for h, sel in enumerate(r["pages"]):
                sc = trace[l]["page_scores"][h]
                own = od.page_select(sc, rkv, sinks, recent)
                forced = od.forced_pages(sc.size, sinks, recent)
                free = np.array([p for p in range(sc.size) if p not in forced])
                k_free = len(sel) - len(forced)
                if k_free > 0 and free.size:
                    sub = np.full(sc.size, -np.inf)
                    sub[free] = sc[free]
                    check_selection_near(np.setdiff1d(own, list(forced)), np.setdiff1d(sel, list(forced)),
                                         sub, k_free)
    e = max_rel(logits_gpu, ref)
    assert e < REL_TOL, f"logits rel err {e}"
    return ref, trace


def pool_from_tokens(k, v, Pmax):
    """Lays token-major bf16 keys/values [Hkv][n][hd] out as the library's
    pages [Hkv][Pmax][2][16][hd] (test-side input preparation)."""
    H, n, hd = k.shape
    pool = torch.zeros(H, Pmax, 2, 16, hd, dtype=torch.bfloat16, device=k.device)
    P = -(-n // 16)
    kp = torch.zeros(H, P * 16, hd, dtype=k.dtype, device=k.device)
    vp = torch.zeros_like(kp)
    kp[:, :n] = k
    vp[:, :n] = v
    pool[:, :P, 0] = kp.view(H, P, 16, hd)
    pool[:, :P, 1] = vp.view(H, P, 16, hd)
    return pool


def bits(t):
    return bf16_bits(t)
