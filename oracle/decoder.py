"""Plain fp64 decoder: one batch-1 decode step of a Llama-style GQA transformer
in the four modes ByteCross times (oracle side; test infrastructure only).

What the pages fix (ByteCross README, "Timing and quality on a GPU"): a step
runs in one of four modes -- dense, the projection branch (activation
sparsity on all seven projections), the KV selection, and both -- a keep
ratio of 1.0 disables a branch, and every mode reads its cache through the
same attention.  "What it does in one picture": the projection weights that
the activations of each token select are read at every step, and an
attention-scored selection keeps the sinks, part of the history and the
recent KV entries.  The projection branch is magnitude-based activation
sparsity in the manner of TEAL ("Training-Free Activation Sparsity in Large
Language Models", listed on the mlsanity paper page); the KV branch's scorer
is not spelled out, so the page key-bound of Quest (same list) is used.

Readings of what the pages leave open (each is a choice, stated once):

* activation select: per projection input, keep the k = ceil(rp*d_in - 1e-9)
  channels of largest |x|; ties go to the lower index.  q/k/v share one input
  and so one set, gate/up share one set: four sets per layer;
* pages of ``page`` tokens; page p holds tokens [p*page, (p+1)*page);
  per page and channel the min and max of its valid keys (post-rotation);
* page score s_p = max over the query heads h of the kv head's group of
  sum_c max(q_hc * kmin_pc, q_hc * kmax_pc), unscaled;
* page select: forced F = pages [0, sinks) U [P - recent, P);
  K = clamp(ceil(rkv*P - 1e-9), |F|, P); the other K - |F| pages are the
  best by (score descending, index ascending); the set is returned ascending;
* the new token's k and v are rounded to bf16 and appended before attention,
  which then covers n + 1 tokens; the last page is always recent;
* rotary embedding: rotate-half pairs (i, i + hd/2), inv_freq_i = theta^(-2i/hd),
  no frequency rescaling; cached keys are already rotated;
* RMSNorm x / sqrt(mean(x^2) + eps) * g; SwiGLU silu(gate) * up;
  the LM head is dense in every mode;
* once-after-prefill selection (the pages' own KV mode, SnapKV-style: an
  attention-scored choice made once after prefill, README "Timing and
  quality on a GPU"; SnapKV is listed on the mlsanity page): a window of
  observation queries per query head (the last prompt positions' queries,
  post-rotary; synthetic here) votes for the cached tokens with its softmax
  attention over the whole prefix (scale 1/sqrt(hd)); a page's score is the
  attention mass its valid tokens receive from all observation queries of
  the kv head's group; the same page rule as above keeps the sinks, the
  recent pages and the best scored others; the kept pages are frozen, and
  every decode step afterwards attends over them plus every page begun
  after the selection ("snap" mode, dense projections);
* masked dense baseline (README FAQ, "A KV method reports a speedup above
  its byte bound": a dense attention that masks the cache down to a KV
  method's pages): dense projections and softmax attention over all n + 1
  tokens with an additive mask, 0 on the tokens of the window's pages (the
  first ``sinks`` and the last ``recent`` pages) and -inf on every other
  token ("masked" mode).  Mathematically it is the KV window.

Arithmetic: fp64 throughout, on bf16 weights and KV widened exactly.
"""
from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------- bf16 helpers


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 to the nearest bf16 (ties to even), returned as bits.

    Works on the exact binary64 value: the bf16 grid is every float64 whose
    significand fits in 8 bits, so rounding is done on the float64 bits."""
    x = np.asarray(x, dtype=np.float64)
    bits = x.view(np.uint64)
    # bf16 keeps 7 fraction bits; float64 has 52 -> drop 45 bits with RNE
    drop = np.uint64(45)
    lsb = (bits >> drop) & np.uint64(1)
    rounded = (bits + (np.uint64(1) << (drop - np.uint64(1))) - np.uint64(1) + lsb) >> drop
    rounded = rounded << drop
    y = rounded.view(np.float64)
    # the float64 exponent range is wider than bf16's: re-express via float32
    # (exact, y has at most 8 significant bits) and take the top 16 bits
    f32 = y.astype(np.float32)
    out = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    return out


# ----------------------------------------------------------------- primitive steps


def rms_norm(x, g_bits, eps):
    """RMSNorm with gain g (bf16)."""
    return x / math.sqrt(float(np.mean(x * x)) + eps) * bf16_to_f64(g_bits)


def rope(heads: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """Rotate each head [H][hd] at position ``pos``; pairs (i, i + hd/2)."""
    hd = heads.shape[-1]
    half = hd // 2
    inv = theta ** (-(2.0 * np.arange(half)) / hd)
    ang = pos * inv
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = heads[..., :half], heads[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(x):
    return x / (1.0 + np.exp(-x))


def keep_count(ratio: float, n: int) -> int:
    return max(1, min(n, math.ceil(ratio * n - 1e-9)))


def channel_select(v: np.ndarray, rp: float, k: int | None = None) -> np.ndarray:
    """Indices of the k largest |v| (ties: lower index first), ascending;
    k = ceil(rp*d_in - 1e-9) unless given."""
    if k is None:
        k = keep_count(rp, v.shape[0])
    order = np.lexsort((np.arange(v.shape[0]), -np.abs(v)))
    return np.sort(order[:k])


def page_bounds(keys: np.ndarray, n_tok: int, page: int):
    """Channelwise min and max of the valid keys of every page.
    keys: [T >= n_tok][hd] float64 of one kv head.  Returns ([P][hd], [P][hd])."""
    P = -(-n_tok // page)
    kmin = np.empty((P, keys.shape[1]))
    kmax = np.empty((P, keys.shape[1]))
    for p in range(P):
        rows = keys[p * page:min((p + 1) * page, n_tok)]
        kmin[p] = rows.min(axis=0)
        kmax[p] = rows.max(axis=0)
    return kmin, kmax


def page_scores(q_group: np.ndarray, kmin: np.ndarray, kmax: np.ndarray):
    """Upper bound of the attention logit of each page, maximised over the
    group's query heads.  q_group [G][hd]; returns [P]."""
    lo = q_group[:, None, :] * kmin[None, :, :]
    hi = q_group[:, None, :] * kmax[None, :, :]
    return np.maximum(lo, hi).sum(axis=-1).max(axis=0)


def forced_pages(P: int, sinks: int, recent: int) -> set:
    return set(range(min(sinks, P))) | set(range(max(P - recent, 0), P))


def page_select(scores: np.ndarray, rkv: float, sinks: int, recent: int) -> np.ndarray:
    """Kept pages: the sinks and recent pages, then the best scored others."""
    P = scores.shape[0]
    F = forced_pages(P, sinks, recent)
    K = max(len(F), min(P, math.ceil(rkv * P - 1e-9)))
    rest = [p for p in range(P) if p not in F]
    rest.sort(key=lambda p: (-float(scores[p]), p))
    return np.array(sorted(F | set(rest[:K - len(F)])), dtype=np.int64)


def snap_scores(q_obs: np.ndarray, keys: np.ndarray, n_tok: int, page: int) -> np.ndarray:
    """Once-after-prefill page scores of one kv head: the softmax attention
    mass that the observation queries q_obs [Q][hd] put on each page's valid
    tokens (keys [>= n_tok][hd]), summed over the queries.  Returns [P]; the
    scores sum to Q."""
    s = q_obs @ keys[:n_tok].T / math.sqrt(q_obs.shape[-1])
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    mass = p.sum(axis=0)
    P = -(-n_tok // page)
    padded = np.zeros(P * page)
    padded[:n_tok] = mass
    return padded.reshape(P, page).sum(axis=1)


def snap_select(cfg, cache: "Cache", q_obs, rkv: float, sinks: int, recent: int):
    """The once-after-prefill selection over the cache's n tokens.  q_obs
    [L][W][Hq][hd] float64 (post-rotary).  Returns ({(layer, kv head):
    ascending kept pages}, {(layer, kv head): page scores}, P at selection)."""
    L, Hq, Hkv, hd = cfg["n_layers"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    G, page, n = Hq // Hkv, cfg["page"], cache.n
    kept, scores = {}, {}
    for l in range(L):
        for h in range(Hkv):
            qs = np.asarray(q_obs[l][:, h * G:(h + 1) * G], dtype=np.float64).reshape(-1, hd)
            sc = snap_scores(qs, bf16_to_f64(cache.k[l, h, :n]), n, page)
            scores[(l, h)] = sc
            kept[(l, h)] = page_select(sc, rkv, sinks, recent)
    return kept, scores, -(-n // page)


def attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray, tok: np.ndarray, bias=None):
    """Softmax attention of the G query heads q [G][hd] over the tokens
    ``tok`` of one kv head; scale 1/sqrt(hd); ``bias`` an optional additive
    mask over those tokens (0 or -inf).  Returns [G][hd]."""
    K = keys[tok]
    Vv = values[tok]
    s = q @ K.T / math.sqrt(q.shape[-1])
    if bias is not None:
        s = s + bias[None, :]
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ Vv) / p.sum(axis=1, keepdims=True)


def gemv_rows(xs: np.ndarray, w_bits: np.ndarray, rows: np.ndarray | None, chunk=2048):
    """y = sum_c xs[c] * W[c, :] over the listed rows of an input-channel-major
    bf16 matrix W [d_in][d_out] (all rows when ``rows`` is None)."""
    d_in, d_out = w_bits.shape
    if rows is None:
        rows = np.arange(d_in)
    y = np.zeros(d_out)
    for i in range(0, rows.shape[0], chunk):
        r = rows[i:i + chunk]
        y += xs[r] @ bf16_to_f64(w_bits[r])
    return y


# ----------------------------------------------------------------- the model


class Cache:
    """Token-major bf16 key/value store: [L][Hkv][capacity][hd] bit arrays."""

    def __init__(self, cfg, capacity):
        L, H, hd = cfg["n_layers"], cfg["n_kv_heads"], cfg["head_dim"]
        self.k = np.zeros((L, H, capacity, hd), dtype=np.uint16)
        self.v = np.zeros((L, H, capacity, hd), dtype=np.uint16)
        self.n = 0

    def extend(self, k_bits, v_bits):
        c = k_bits.shape[2]
        self.k[:, :, self.n:self.n + c] = k_bits
        self.v[:, :, self.n:self.n + c] = v_bits
        self.n += c


MODES = ("dense", "act", "kv", "both", "snap", "masked")


def decode_step(cfg, w, cache: Cache, token: int, mode: str, rp=1.0, rkv=1.0,
                sinks=1, recent=16, forced=None, kv_round=True, layers=None,
                x_in=None, trace=None, snap=None):
    """One decode step at position cache.n.  Appends the token's k, v.

    w: dict of bf16 bit arrays in the layouts of ``synth.make_weights``.
    forced: optional {(layer, site): index array} with site in
        'qkv', 'o', 'gu', 'd' (channel sets) and (layer, 'pages', h) page sets,
        used instead of this oracle's own selection.
    layers: optional range of layers to run (the rest are skipped and the
        logits are not computed); x_in: residual stream entering the first of
        them (default: the token's embedding row).
    snap: for mode 'snap', (kept pages per (layer, kv head), P at the
        selection) as returned by ``snap_select``.
    trace: optional dict that receives every intermediate per layer.
    Returns the logits [V] (or the residual stream when ``layers`` is given).
    """
    if mode not in MODES:
        raise ValueError(mode)
    act = mode in ("act", "both")
    kvsel = mode in ("kv", "both")
    forced = forced or {}
    L, d, f = cfg["n_layers"], cfg["hidden"], cfg["intermediate"]
    Hq, Hkv, hd = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    G, page, eps, theta = Hq // Hkv, cfg["page"], cfg["rms_eps"], cfg["rope_theta"]
    pos = cache.n
    n_tok = pos + 1
    P = -(-n_tok // page)
    run = range(L) if layers is None else layers
    x = bf16_to_f64(w["embed"][token]) if x_in is None else np.array(x_in, dtype=np.float64)

    def select(layer, site, v):
        if (layer, site) in forced:
            return np.asarray(forced[(layer, site)], dtype=np.int64)
        return channel_select(v, rp) if act else None

    for l in run:
        rec = {} if trace is not None else None
        # attention block
        xn = rms_norm(x, w["attn_norm"][l], eps)
        s_qkv = select(l, "qkv", xn)
        qkv = gemv_rows(xn, w["wqkv_t"][l], s_qkv)
        q = rope(qkv[:Hq * hd].reshape(Hq, hd), pos, theta)
        k = rope(qkv[Hq * hd:(Hq + Hkv) * hd].reshape(Hkv, hd), pos, theta)
        v = qkv[(Hq + Hkv) * hd:].reshape(Hkv, hd)
        if kv_round:
            cache.k[l, :, pos] = f64_to_bf16(k)
            cache.v[l, :, pos] = f64_to_bf16(v)
            k_new, v_new = None, None
        else:
            k_new, v_new = k, v
        attn = np.empty((Hq, hd))
        pages_l, scores_l = [], []
        for h in range(Hkv):
            keys = bf16_to_f64(cache.k[l, h, :n_tok])
            vals = bf16_to_f64(cache.v[l, h, :n_tok])
            if k_new is not None:
                keys[pos], vals[pos] = k_new[h], v_new[h]
            qg = q[h * G:(h + 1) * G]
            if mode == "snap":
                kept, p_snap = snap
                sel = np.array(sorted(set(int(p) for p in kept[(l, h)]) | set(range(p_snap, P))),
                               dtype=np.int64)
                tok = np.concatenate([np.arange(p * page, min((p + 1) * page, n_tok)) for p in sel])
                pages_l.append(sel)
            elif kvsel:
                kmin, kmax = page_bounds(keys, n_tok, page)
                sc = page_scores(qg, kmin, kmax)
                if (l, "pages", h) in forced:
                    sel = np.asarray(forced[(l, "pages", h)], dtype=np.int64)
                else:
                    sel = page_select(sc, rkv, sinks, recent)
                tok = np.concatenate([np.arange(p * page, min((p + 1) * page, n_tok))
                                      for p in sel])
                scores_l.append(sc)
                pages_l.append(sel)
            elif mode == "masked":
                tok = np.arange(n_tok)
                window = forced_pages(P, sinks, recent)
                bias = np.where(np.isin(tok // page, sorted(window)), 0.0, -np.inf)
                attn[h * G:(h + 1) * G] = attention(qg, keys, vals, tok, bias)
                continue
            else:
                tok = np.arange(n_tok)
            attn[h * G:(h + 1) * G] = attention(qg, keys, vals, tok)
        attn = attn.reshape(-1)
        s_o = select(l, "o", attn)
        x = x + gemv_rows(attn, w["wo_t"][l], s_o)
        # feed-forward block
        xn2 = rms_norm(x, w["mlp_norm"][l], eps)
        s_gu = select(l, "gu", xn2)
        gu = gemv_rows(xn2, w["wgu_t"][l], s_gu)
        hmid = silu(gu[:f]) * gu[f:]
        s_d = select(l, "d", hmid)
        x = x + gemv_rows(hmid, w["wd_t"][l], s_d)
        if rec is not None:
            rec.update(xn=xn, s_qkv=s_qkv, q=q, k=k, v=v, attn=attn, s_o=s_o,
                       xn2=xn2, s_gu=s_gu, h=hmid, s_d=s_d, x=x.copy(),
                       pages=pages_l, page_scores=scores_l)
            trace[l] = rec
    cache.n = n_tok
    if layers is not None:
        return x
    xf = rms_norm(x, w["final_norm"], eps)
    logits = np.empty(cfg["vocab"])
    for i in range(0, cfg["vocab"], 8192):
        logits[i:i + 8192] = bf16_to_f64(w["lm_head"][i:i + 8192]) @ xf
    if trace is not None:
        trace["final"] = dict(x=x, xf=xf)
    return logits
