"""Byte account of one batch-1 decode step (oracle side, fp64 host arithmetic).

Paper form.  The ByteCross README ("Overview"; "Usage: The byte account")
describes a step as re-reading the projection weights (fixed traffic) and the
KV cache (traffic growing with the context n).  The equations themselves are
not printed; the forms below reproduce every printed value:

* per-layer projection parameters
  P_l = d*Hq*hd + 2*d*Hkv*hd + Hq*hd*d + 3*d*d_ff      (q, k, v, o, gate, up, down)
* projection bytes W = 2*L*P_l, LM-head bytes H = 2*V*d, KV bytes per token
  kv_tok = 2*L*2*Hkv*hd (bf16 keys and values)
* Equation 5, byte crossover: (1-rp)*W = (1-rkv)*n*kv_tok, i.e.
  n* = (1-rp)*P_l / ((1-rkv)*2*Hkv*hd) tokens; ``ff_only`` keeps only the
  3*d*d_ff feed-forward term in P_l
* ideal speedup bound B/(B - dB), B = W + H + n*kv_tok,
  dB = (1-rp)*W + (1-rkv)*n*kv_tok.  The LM head must be part of B: only then
  does the README's "1.60x at 128K, KV keep 0.3" come out (1.5964; without it
  1.629)
* crossover_batch: a batch reads the union of selected weights once
  (fraction ``union_keep``) while each sequence saves its own KV bytes:
  n = (1-union_keep)*P_l / (batch*(1-rkv)*2*Hkv*hd)
* matched_crossover: each branch takes the lowest keep whose linearly
  interpolated perplexity increase stays within the budget (no extrapolation
  below the lowest listed keep), then the two savings are equated.

Implementation form.  The bytes this library's step must move in each mode,
enumerated layer by layer, head by head and page by page
(``implementation_bytes``): selected weight rows, the LM head, the KV tokens
of the selected pages, the page key-bound metadata, the KV append, norm
gains, the embedding row and the logits.  Readings of the pages it uses:
keep counts k = ceil(rp*d_in - 1e-9) per projection input; the page keep
count K = clamp(ceil(rkv*P - 1e-9), |forced|, P) with forced = sinks U recent.
"""
from __future__ import annotations

import math

BF16 = 2
F32 = 4


def _dims(cfg):
    d, f = cfg["hidden"], cfg["intermediate"]
    hq = cfg["n_heads"] * cfg["head_dim"]
    hkv = cfg["n_kv_heads"] * cfg["head_dim"]
    return d, f, hq, hkv


def params_per_layer(cfg, ff_only=False):
    """P_l, the seven projections' parameter count in one layer."""
    d, f, hq, hkv = _dims(cfg)
    ff = 3 * d * f
    if ff_only:
        return ff
    return d * hq + 2 * d * hkv + hq * d + ff


def weight_bytes(cfg):
    return BF16 * cfg["n_layers"] * params_per_layer(cfg)


def head_bytes(cfg):
    return BF16 * cfg["vocab"] * cfg["hidden"]


def kv_bytes_per_token(cfg):
    return BF16 * cfg["n_layers"] * 2 * cfg["n_kv_heads"] * cfg["head_dim"]


def crossover(cfg, rp, rkv, ff_only=False):
    """Equation 5 of the paper (ByteCross README, "Usage: The byte account"):
    context length, in tokens, at which both branches save the same bytes."""
    num = (1.0 - rp) * params_per_layer(cfg, ff_only)
    den = (1.0 - rkv) * 2 * cfg["n_kv_heads"] * cfg["head_dim"]
    return num / den


def dense_bytes(cfg, n):
    return weight_bytes(cfg) + head_bytes(cfg) + n * kv_bytes_per_token(cfg)


def saved_bytes(cfg, n, rp=1.0, rkv=1.0):
    return (1.0 - rp) * weight_bytes(cfg) + (1.0 - rkv) * n * kv_bytes_per_token(cfg)


def bound(cfg, n, rp=1.0, rkv=1.0):
    """Ideal speedup B_total / (B_total - dB) of a purely bandwidth-bound step
    (ByteCross README, "Quick start" and "Usage: The byte account")."""
    b = dense_bytes(cfg, n)
    return b / (b - saved_bytes(cfg, n, rp, rkv))


def crossover_batch(cfg, union_keep, rkv, batch):
    """Batch crossover (ByteCross README, "Usage: The byte account")."""
    num = (1.0 - union_keep) * params_per_layer(cfg)
    den = batch * (1.0 - rkv) * 2 * cfg["n_kv_heads"] * cfg["head_dim"]
    return num / den


def _lowest_keep(curve, budget):
    """Lowest keep ratio whose linearly interpolated increase is <= budget.
    ``curve`` maps keep -> increase; keeps are walked from high to low."""
    keeps = sorted(curve, reverse=True)
    best = None
    for i, kp in enumerate(keeps):
        if curve[kp] <= budget:
            best = kp
            continue
        # first keep over budget: interpolate between the previous keep and it
        if i > 0:
            hi, lo = keeps[i - 1], kp
            y0, y1 = curve[hi], curve[lo]
            best = hi - (hi - lo) * (budget - y0) / (y1 - y0)
        break
    return best


def matched_crossover(cfg, proj, sel, budget):
    """Crossover at equal perplexity increase (ByteCross README, "The
    quality-matched crossover")."""
    rp = _lowest_keep(proj, budget)
    rkv = _lowest_keep(sel, budget)
    return crossover(cfg, rp, rkv)


# ---------------------------------------------------------------- implementation form

def keep_count(ratio, n):
    """Number of kept items for a keep ratio: ceil(ratio*n - 1e-9), at least 1."""
    return max(1, min(n, math.ceil(ratio * n - 1e-9)))


def page_keep(P, rkv, sinks, recent):
    forced = set(range(min(sinks, P))) | set(range(max(P - recent, 0), P))
    K = max(len(forced), min(P, math.ceil(rkv * P - 1e-9)))
    return K, len(forced)


def implementation_bytes(cfg, mode, n, rp=1.0, rkv=1.0, sinks=1, recent=16):
    """Bytes one decode step moves at context n (n tokens cached; the step
    appends token n and attends over n+1), enumerated explicitly.

    mode: 'dense', 'act', 'kv', 'both', 'snap' (the pages a once-after-
    prefill selection made at context n kept, plus a page the step's token
    opens; no bounds are read) or 'masked' (the masked dense baseline: every
    KV byte is read, as in dense).  Returns a dict of byte counts.
    """
    act = mode in ("act", "both")
    kv = mode in ("kv", "both")
    snap = mode == "snap"
    L, d, f = cfg["n_layers"], cfg["hidden"], cfg["intermediate"]
    Hq, Hkv, hd, V, page = (cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"],
                            cfg["vocab"], cfg["page"])
    nqkv = (Hq + 2 * Hkv) * hd
    out = dict(weights=0, head=0, kv_read=0, meta_read=0, kv_write=0, other=0)
    n_tok = n + 1
    P = -(-n_tok // page)
    for _layer in range(L):
        for d_in, d_out in ((d, nqkv), (Hq * hd, d), (d, 2 * f), (f, d)):
            k = keep_count(rp, d_in) if act else d_in
            out["weights"] += BF16 * k * d_out
        for _h in range(Hkv):
            if kv:
                K, _ = page_keep(P, rkv, sinks, recent)
                # the forced recent pages include the last (partial) page
                pages = _selected_page_count_tokens(P, K, n_tok, page)
                out["meta_read"] += P * 2 * hd * BF16
            elif snap:
                P_sel = -(-max(n, 1) // page)
                K_sel, _ = page_keep(P_sel, rkv, sinks, recent)
                pages = _selected_page_count_tokens(P, K_sel + (P - P_sel), n_tok, page)
            else:
                pages = n_tok
            out["kv_read"] += pages * 2 * hd * BF16
            # append: the new k and v rows, the page's bounds rewritten, the
            # page's earlier keys re-read to recompute them
            slot = (n_tok - 1) % page
            out["kv_write"] += 2 * hd * BF16 + 2 * hd * BF16
            out["other"] += slot * hd * BF16
        out["other"] += 2 * d * BF16          # two RMSNorm gain vectors
    out["head"] = BF16 * V * d
    out["other"] += BF16 * d + BF16 * d + F32 * V   # embed row, final norm, logits
    out["total"] = sum(v for key, v in out.items())
    return out


def _selected_page_count_tokens(P, K, n_tok, page):
    """Tokens held by K selected pages when the last page (always selected,
    it is recent) holds the partial remainder."""
    last = n_tok - (P - 1) * page
    return (K - 1) * page + last
