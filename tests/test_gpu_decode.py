"""Decode-step parity on the GPU through the C ABI, against the fp64 oracle.

* tiny GQA decoder (2 layers, hidden 512, 8/2 heads, hd 64), 2048 cached
  tokens, 8 steps in each of the four modes at rp = rkv = 0.5, page 16,
  1 sink page, 8 recent pages;
* keep ratios of 1 reproduce dense bit for bit;
* the KV append (bulk and per step) and its page key bounds;
* planted-key retrieval of the page selection;
* the Llama-3.1-8B shape at 2K context in every mode, layer by layer.

Comparison rules (tests/parity.py): selected channel and page sets are
exact when the oracle ranks the GPU's own pre-selection scores; against the
oracle's own scores they may differ only at near-ties (1e-3 of the cut);
hidden states and logits within max relative error 1e-2.
"""
import numpy as np
import pytest
import torch

import activation_kv_sparsity_b200 as bc
from oracle import decoder as od
from parity import (REL_TOL, bits, check_selection_exact, check_selection_near, compare_step, pages_of,
                    gpu_traces, max_rel, to_host)
from synth import LLAMA_8B, TINY, kv_chunks, make_kv, make_weights, plant_keys, planted_positions, tokens

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
N_CTX = 2048
KW = dict(rp=0.5, rkv=0.5, sinks=1, recent=8)


@pytest.fixture(scope="module")
def tiny():
    cfg = TINY
    w_t = make_weights(cfg, seed=0)
    k, v = make_kv(cfg, N_CTX, seed=1)
    return dict(cfg=cfg, wb={n: bits(t) for n, t in w_t.items()}, wd={n: t.to(DEV) for n, t in w_t.items()},
                k=k, v=v)


def _model(t, max_ctx=N_CTX + 32):
    m = bc.Model(t["cfg"], t["wd"], max_ctx)
    m.append(t["k"].to(DEV), t["v"].to(DEV))
    return m


def _cache(t, cap=N_CTX + 32):
    c = od.Cache(t["cfg"], cap)
    c.extend(bits(t["k"]), bits(t["v"]))
    return c


@pytest.mark.parametrize("mode", ["dense", "act", "kv", "both"])
def test_tiny_eight_steps(tiny, mode):
    cfg = tiny["cfg"]
    m = _model(tiny)
    cache = _cache(tiny)
    logits = torch.empty(cfg["vocab"], device=DEV)
    for tok in tokens(8, cfg["vocab"], seed=3):
        m.step(tok, mode, logits, **KW)
        torch.cuda.synchronize()
        tr = gpu_traces(m, cfg["n_layers"], mode in ("kv", "both"))
        compare_step(cfg, tiny["wb"], cache, tok, mode, KW["rp"], KW["rkv"], KW["sinks"], KW["recent"],
                     to_host(logits), tr)
    assert len(m) == N_CTX + 8


def test_kv_window_baseline(tiny):
    """The KV window (the pages' window baseline: sinks and recent pages
    only, no scored pages) is the kv mode with a keep ratio small enough that
    K = |F|: every head keeps exactly the forced pages, and the step matches
    the oracle."""
    cfg = tiny["cfg"]
    kw = dict(rp=1.0, rkv=1e-6, sinks=1, recent=8)
    m = _model(tiny)
    cache = _cache(tiny)
    logits = torch.empty(cfg["vocab"], device=DEV)
    for tok in tokens(3, cfg["vocab"], seed=17):
        m.step(tok, "kv", logits, **kw)
        torch.cuda.synchronize()
        tr = gpu_traces(m, cfg["n_layers"], True)
        P = -(-len(m) // 16)
        want = np.array(sorted(od.forced_pages(P, kw["sinks"], kw["recent"])))
        for r in tr:
            for h in range(r["pages"].shape[0]):
                np.testing.assert_array_equal(r["pages"][h], want)
        compare_step(cfg, tiny["wb"], cache, tok, "kv", kw["rp"], kw["rkv"], kw["sinks"], kw["recent"],
                     to_host(logits), tr)


def test_masked_dense_baseline(tiny):
    """The masked dense baseline (every page read, an additive mask keeping
    the window's pages) matches the oracle's masked step, and the KV window
    computed from the window's pages alone, within fp32 rounding."""
    cfg = tiny["cfg"]
    kw = dict(sinks=1, recent=8)
    m = _model(tiny)
    cache = _cache(tiny)
    logits = torch.empty(cfg["vocab"], device=DEV)
    win = torch.empty(cfg["vocab"], device=DEV)
    for tok in tokens(3, cfg["vocab"], seed=19):
        n = len(m)
        m.step(tok, "kv", win, rkv=1e-6, **kw)
        m.reset(n)
        m.step(tok, "masked", logits, **kw)
        torch.cuda.synchronize()
        tr = gpu_traces(m, cfg["n_layers"], False)
        compare_step(cfg, tiny["wb"], cache, tok, "masked", 1.0, 1.0, kw["sinks"], kw["recent"],
                     to_host(logits), tr)
        assert max_rel(to_host(logits), to_host(win)) < 1e-5


def test_keep_one_is_dense_bit_for_bit(tiny):
    cfg = tiny["cfg"]
    m = _model(tiny)
    tok = 1234
    out = {}
    for mode in ("dense", "act", "kv", "both"):
        m.reset(N_CTX)
        logits = torch.empty(cfg["vocab"], device=DEV)
        m.step(tok, mode, logits, rp=1.0, rkv=1.0, sinks=1, recent=8)
        torch.cuda.synchronize()
        out[mode] = logits.clone()
    for mode in ("act", "kv", "both"):
        assert torch.equal(out[mode], out["dense"]), mode


def test_steps_are_deterministic(tiny):
    cfg = tiny["cfg"]
    m = _model(tiny)
    res = []
    for _ in range(2):
        m.reset(N_CTX)
        logits = torch.empty(cfg["vocab"], device=DEV)
        for tok in (5, 6, 7):
            m.step(tok, "both", logits, **KW)
        torch.cuda.synchronize()
        res.append(logits.clone())
    assert torch.equal(res[0], res[1])


@pytest.mark.parametrize("mode", ["dense", "act", "kv", "both"])
def test_graph_steps_equal_direct_steps(tiny, mode):
    """Steps replayed from a captured CUDA graph (nodes updated per step) give
    the same logits, bit for bit, as direct launches, across page boundaries
    (the page count and the attention grid change between steps)."""
    cfg = tiny["cfg"]
    start = N_CTX - 20                       # crosses positions 2032 and 2048 (page boundaries)
    outs = {}
    for graphs in (False, True):
        m = _model(tiny)
        m.set_graphs(graphs)
        m.reset(start)
        logits = torch.empty(cfg["vocab"], device=DEV)
        seq = []
        for tok in tokens(24, cfg["vocab"], seed=9):
            m.step(tok, mode, logits, **KW)
            seq.append(logits.clone())
        torch.cuda.synchronize()
        outs[graphs] = seq
        m.close()
    for i, (a, b) in enumerate(zip(outs[False], outs[True])):
        assert torch.equal(a, b), (mode, i)


@pytest.mark.parametrize("edge", [32768, 131072])
def test_graph_steps_across_page_select_variants(tiny, edge):
    """Across 2048 -> 2049 pages (32768 tokens) the one-CTA page select moves
    from 2 to 4 keys a thread, across 8192 -> 8193 pages (131072 tokens) to
    the cluster: a new graph is captured for the new variant and the steps
    still equal direct launches bit for bit, with exact page sets."""
    cfg = tiny["cfg"]
    n0 = edge - 12
    k, v = make_kv(cfg, n0, seed=5, device=DEV)
    outs = {}
    for graphs in (False, True):
        m = bc.Model(cfg, tiny["wd"], edge + 32)
        m.append(k, v)
        m.set_graphs(graphs)
        logits = torch.empty(cfg["vocab"], device=DEV)
        seq = []
        for tok in tokens(24, cfg["vocab"], seed=13):
            m.step(tok, "kv", logits, **KW)
            seq.append(logits.clone())
        torch.cuda.synchronize()
        tr = gpu_traces(m, cfg["n_layers"], True)
        check_selection_exact(tr, KW["rp"], KW["rkv"], KW["sinks"], KW["recent"], False, True)
        outs[graphs] = seq
        m.close()
    for i, (a, b) in enumerate(zip(outs[False], outs[True])):
        assert torch.equal(a, b), i


def _meta(m, cfg, max_ctx):
    Pmax = -(-max_ctx // 16)
    return m.meta_pool.view(torch.bfloat16).view(cfg["n_layers"], cfg["n_kv_heads"], Pmax, 2, cfg["head_dim"])


def _pool(m, cfg, max_ctx):
    Pmax = -(-max_ctx // 16)
    return m.kv_pool.view(torch.bfloat16).view(cfg["n_layers"], cfg["n_kv_heads"], Pmax, 2, 16, cfg["head_dim"])


def test_bulk_append_and_bounds(tiny):
    """Pages hold the appended tokens; page bounds equal the min/max of the
    valid keys exactly (min and max of bf16 values are exact)."""
    cfg = tiny["cfg"]
    max_ctx = N_CTX + 32
    m = bc.Model(cfg, tiny["wd"], max_ctx)
    k, v = tiny["k"], tiny["v"]
    # ragged appends across page boundaries
    for a, b in ((0, 5), (5, 16), (16, 1000), (1000, 2047), (2047, 2048)):
        m.append(k[:, :, a:b].to(DEV), v[:, :, a:b].to(DEV))
    torch.cuda.synchronize()
    assert len(m) == N_CTX
    pool, meta = _pool(m, cfg, max_ctx), _meta(m, cfg, max_ctx)
    P = N_CTX // 16
    got_k = pool[:, :, :P, 0].reshape(cfg["n_layers"], cfg["n_kv_heads"], N_CTX, -1)
    got_v = pool[:, :, :P, 1].reshape(cfg["n_layers"], cfg["n_kv_heads"], N_CTX, -1)
    assert torch.equal(got_k.cpu(), k) and torch.equal(got_v.cpu(), v)
    kb = bits(k)
    for l in range(cfg["n_layers"]):
        for h in range(cfg["n_kv_heads"]):
            kmin, kmax = od.page_bounds(od.bf16_to_f64(kb[l, h]), N_CTX, 16)
            np.testing.assert_array_equal(meta[l, h, :P, 0].float().cpu().numpy(), kmin)
            np.testing.assert_array_equal(meta[l, h, :P, 1].float().cpu().numpy(), kmax)
    # truncate into the middle of a page, append again: bounds cover valid keys only
    m.reset(1000)
    m.append(k[:, :, 1000:1003].to(DEV) * 0 + 7, v[:, :, 1000:1003].to(DEV))
    torch.cuda.synchronize()
    page = 1000 // 16
    rows = np.concatenate([od.bf16_to_f64(kb[0, 0, page * 16:1000]), np.full((3, cfg["head_dim"]), 7.0)])
    np.testing.assert_array_equal(meta[0, 0, page, 1].float().cpu().numpy(), rows.max(axis=0))
    np.testing.assert_array_equal(meta[0, 0, page, 0].float().cpu().numpy(), rows.min(axis=0))


def test_step_append_rotates_and_bounds(tiny):
    """The q/k/v epilogue writes bf16(rotate(k)) and bf16(v) at position n and
    refreshes that page's bounds from its valid keys."""
    cfg = tiny["cfg"]
    max_ctx = N_CTX + 32
    m = _model(tiny, max_ctx)
    logits = torch.empty(cfg["vocab"], device=DEV)
    n = N_CTX
    for step in range(3):
        m.step(11 + step, "dense", logits)
        torch.cuda.synchronize()
        pos = n + step
        pool, meta = _pool(m, cfg, max_ctx), _meta(m, cfg, max_ctx)
        hq, hkv, hd = cfg["n_heads"] * cfg["head_dim"], cfg["n_kv_heads"] * cfg["head_dim"], cfg["head_dim"]
        for l in range(cfg["n_layers"]):
            raw = to_host(m.trace(l, bc.BC_TRACE_QKV))
            k_rot = od.rope(raw[hq:hq + hkv].reshape(-1, hd), pos, cfg["rope_theta"])
            want_k = od.f64_to_bf16(k_rot).astype(np.int32)
            got_k = pool[l, :, pos // 16, 0, pos % 16].cpu().view(torch.int16).numpy().astype(np.int32) & 0xFFFF
            assert np.abs(got_k - want_k).max() <= 1          # at most one bf16 ulp (fp32 vs fp64 rotation)
            want_v = od.f64_to_bf16(raw[hq + hkv:].reshape(-1, hd)).astype(np.int32)
            got_v = pool[l, :, pos // 16, 1, pos % 16].cpu().view(torch.int16).numpy().astype(np.int32) & 0xFFFF
            assert np.abs(got_v - want_v).max() <= 1
            q_rot = od.rope(raw[:hq].reshape(-1, hd), pos, cfg["rope_theta"])
            assert max_rel(to_host(m.trace(l, bc.BC_TRACE_Q)).reshape(-1, hd), q_rot) < 1e-5
            keys = pool[l, :, pos // 16, 0, : pos % 16 + 1].float().cpu().numpy()
            np.testing.assert_array_equal(meta[l, :, pos // 16, 0].float().cpu().numpy(), keys.min(axis=1))
            np.testing.assert_array_equal(meta[l, :, pos // 16, 1].float().cpu().numpy(), keys.max(axis=1))


def test_planted_keys_are_retrieved(tiny):
    cfg = tiny["cfg"]
    sinks, recent, rkv = 1, 8, 0.3
    pos = planted_positions(N_CTX, 16, sinks, recent)
    k = plant_keys(tiny["k"].clone(), pos)
    m = bc.Model(cfg, tiny["wd"], N_CTX + 32)
    m.append(k.to(DEV), tiny["v"].to(DEV))
    logits = torch.empty(cfg["vocab"], device=DEV)
    m.step(77, "kv", logits, rkv=rkv, sinks=sinks, recent=recent)
    torch.cuda.synchronize()
    want = {p // 16 for p in pos}
    for l in range(cfg["n_layers"]):
        pages = m.trace(l, bc.BC_TRACE_PAGES).cpu().numpy()
        for h in range(cfg["n_kv_heads"]):
            assert want <= set(pages[h].tolist()), (l, h)


def test_capacity_and_argument_errors(tiny):
    cfg = tiny["cfg"]
    m = bc.Model(cfg, tiny["wd"], 40)
    k, v = tiny["k"][:, :, :40].to(DEV), tiny["v"][:, :, :40].to(DEV)
    m.append(k, v)
    logits = torch.empty(cfg["vocab"], device=DEV)
    with pytest.raises(bc.BCError) as e:
        m.step(1, "dense", logits)
    assert e.value.status == bc.BC_ECAPACITY
    with pytest.raises(bc.BCError) as e:
        m.append(k[:, :, :1], v[:, :, :1])
    assert e.value.status == bc.BC_ECAPACITY
    m.reset(30)
    for kw in (dict(rp=0.0), dict(rkv=1.5), dict(recent=0), dict(sinks=-1)):
        with pytest.raises(bc.BCError) as e:
            m.step(1, "both", logits, **kw)
        assert e.value.status == bc.BC_EINVAL
    with pytest.raises(bc.BCError):
        m.step(cfg["vocab"], "dense", logits)
    assert len(m) == 30
    m.step(1, "both", logits, rp=0.5, rkv=0.5, sinks=1, recent=1)   # still usable
    torch.cuda.synchronize()
    assert len(m) == 31


def test_host_buffer_step_matches_device_step(tiny):
    cfg = tiny["cfg"]
    m = _model(tiny)
    d = torch.empty(cfg["vocab"], device=DEV)
    m.step(9, "both", d, **KW)
    m.reset(N_CTX)
    h = torch.empty(cfg["vocab"], pin_memory=True)
    m.step_host(9, "both", h, **KW)
    assert torch.equal(d.cpu(), h)


# ------------------------------------------------------------------ Llama-3.1-8B shape

N8 = 2048


@pytest.fixture(scope="module")
def big():
    cfg = LLAMA_8B
    w = make_weights(cfg, seed=0, device=DEV)
    k, v = make_kv(cfg, N8, seed=1, device=DEV)
    wb = {n: bits(t) for n, t in w.items()}
    return dict(cfg=cfg, wd=w, wb=wb, k=k, v=v, kb=bits(k), vb=bits(v))


@pytest.mark.parametrize("mode", ["dense", "act", "kv", "both", "masked"])
def test_llama8b_shape_step(big, mode):
    """One step at the Llama-3.1-8B shape (2048 cached tokens): every set
    exact on the GPU's own scores and within near-ties of the oracle's own
    choice; the oracle runs all 32 layers from its own inputs (told only the
    index sets) and every layer's hidden state and the logits agree within
    1e-2."""
    cfg = big["cfg"]
    kw = dict(rp=0.5, rkv=0.3, sinks=1, recent=16)
    m = bc.Model(cfg, big["wd"], N8 + 16)
    m.append(big["k"], big["v"])
    logits = torch.empty(cfg["vocab"], device=DEV)
    tok = 4242
    m.step(tok, mode, logits, **kw)
    torch.cuda.synchronize()
    tr = gpu_traces(m, cfg["n_layers"], mode in ("kv", "both"))
    cache = od.Cache(cfg, N8 + 1)
    cache.extend(big["kb"], big["vb"])
    compare_step(cfg, big["wb"], cache, tok, mode, kw["rp"], kw["rkv"], kw["sinks"], kw["recent"],
                 to_host(logits), tr)
    m.close()


def test_llama8b_shape_snap_step(big):
    """The once-after-prefill selection and one snap step at the 8B shape:
    kept pages exact on the GPU's own scores and within near-ties of the
    oracle's own selection; the oracle runs all 32 layers from its own
    inputs, told only the kept page numbers, and every hidden state and the
    logits agree within 1e-2."""
    from synth import obs_queries
    cfg = big["cfg"]
    sel = dict(rkv=0.3, sinks=1, recent=16)
    m = bc.Model(cfg, big["wd"], N8 + 16)
    m.append(big["k"], big["v"])
    q_obs = obs_queries(cfg, 16, seed=11, device=DEV)
    m.snap_select(q_obs, **sel)
    logits = torch.empty(cfg["vocab"], device=DEV)
    tok = 4242
    m.step(tok, "snap", logits)
    torch.cuda.synchronize()
    cache = od.Cache(cfg, N8 + 1)
    cache.extend(big["kb"], big["vb"])
    own_kept, own_scores, P = od.snap_select(cfg, cache, q_obs.cpu().double().numpy(), **sel)
    forced_pages = od.forced_pages(P, sel["sinks"], sel["recent"])
    kept = {}
    for l in range(cfg["n_layers"]):
        sc = m.trace(l, bc.BC_TRACE_SNAP_SCORES).cpu().numpy().astype(np.float64)
        pg = m.trace(l, bc.BC_TRACE_SNAP_PAGES).cpu().numpy().astype(np.int64)
        for h in range(cfg["n_kv_heads"]):
            np.testing.assert_array_equal(pages_of(sc[h], **sel), pg[h], err_msg=f"layer {l} head {h}")
            free = np.array([p for p in range(P) if p not in forced_pages])
            sub = np.full(P, -np.inf)
            sub[free] = own_scores[(l, h)][free]
            check_selection_near(np.setdiff1d(own_kept[(l, h)], list(forced_pages)),
                                 np.setdiff1d(pg[h], list(forced_pages)), sub,
                                 len(pg[h]) - len(forced_pages))
            kept[(l, h)] = pg[h]
    tr = gpu_traces(m, cfg["n_layers"], False)
    trace = {}
    ref = od.decode_step(cfg, big["wb"], cache, tok, "snap", snap=(kept, P), trace=trace)
    for l in range(cfg["n_layers"]):
        assert max_rel(tr[l]["x"], trace[l]["x"]) < REL_TOL, l
    assert max_rel(to_host(logits), ref) < REL_TOL
    m.close()


def test_llama8b_shape_planted_retrieval():
    cfg = LLAMA_8B
    n, sinks, recent, rkv = 4096, 1, 16, 0.3
    w = make_weights(dict(cfg, n_layers=4), seed=0, device=DEV)
    c4 = dict(cfg, n_layers=4)
    pos = planted_positions(n, 16, sinks, recent)
    m = bc.Model(c4, w, n + 16)
    first = 0
    for k, v in kv_chunks(c4, n, seed=1, device=DEV):
        plant_keys(k, pos, first_token=first)
        m.append(k, v)
        first += k.shape[2]
    logits = torch.empty(cfg["vocab"], device=DEV)
    m.step(99, "both", logits, rp=0.5, rkv=rkv, sinks=sinks, recent=recent)
    torch.cuda.synchronize()
    want = {p // 16 for p in pos}
    for l in range(4):
        pages = m.trace(l, bc.BC_TRACE_PAGES).cpu().numpy()
        for h in range(cfg["n_kv_heads"]):
            assert want <= set(pages[h].tolist()), (l, h)
