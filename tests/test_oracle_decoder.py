"""Pins of the fp64 decoder oracle to things other than itself: library
routines (torch, Hugging Face's Llama), closed forms, invariants and brute
force on small inputs."""
import math

import numpy as np
import pytest
import torch

from oracle import decoder as od
from synth import TINY, bf16_bits, make_kv, make_weights, tokens

RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------- primitives

def test_bf16_widen_and_round():
    x32 = RNG.standard_normal(4096).astype(np.float32) * np.float32(3.0)
    x64 = x32.astype(np.float64)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = od.f64_to_bf16(x64)
    np.testing.assert_array_equal(got, ref)
    # widening is exact: bf16 -> f64 -> bf16 is the identity
    np.testing.assert_array_equal(od.f64_to_bf16(od.bf16_to_f64(ref)), ref)
    # ties to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    assert od.f64_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80
    assert od.f64_to_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82


def test_rms_norm_matches_torch():
    x = RNG.standard_normal(512)
    g = bf16_bits(torch.randn(512).to(torch.bfloat16))
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (512,),
                                       torch.from_numpy(od.bf16_to_f64(g)), eps=1e-5)
    np.testing.assert_allclose(od.rms_norm(x, g, 1e-5), ref.numpy(), rtol=1e-13)


def test_silu_matches_torch():
    x = RNG.standard_normal(1000) * 6
    np.testing.assert_allclose(od.silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(),
                               rtol=1e-13, atol=1e-300)


def test_rope_matches_hf_and_complex_form():
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    hd, H, pos, theta = 64, 3, 1234, 5e5
    x = RNG.standard_normal((H, hd))
    got = od.rope(x, pos, theta)
    # independent form: pair (i, i+hd/2) as a complex number times e^{i pos w_i}
    half = hd // 2
    w = 1.0 / theta ** (np.arange(0, hd, 2) / hd)
    z = (x[:, :half] + 1j * x[:, half:]) * np.exp(1j * pos * w)
    np.testing.assert_allclose(got, np.concatenate([z.real, z.imag], axis=1), rtol=1e-12, atol=1e-12)
    # Hugging Face's own rotation
    ang = torch.from_numpy(np.concatenate([pos * w, pos * w]))
    cos, sin = ang.cos()[None, None], ang.sin()[None, None]      # [batch, seq, hd]
    t = torch.from_numpy(x)[None, :, None, :]                    # [batch, heads, seq, hd]
    q2, _ = apply_rotary_pos_emb(t, t, cos, sin)
    np.testing.assert_allclose(got, q2[0, :, 0].numpy(), rtol=1e-12, atol=1e-12)
    # relative-position property and position 0 = identity
    q, k = RNG.standard_normal(hd), RNG.standard_normal(hd)
    a = od.rope(q[None], 700, theta)[0] @ od.rope(k[None], 500, theta)[0]
    b = od.rope(q[None], 200, theta)[0] @ k
    assert a == pytest.approx(b, rel=1e-10)
    np.testing.assert_array_equal(od.rope(x, 0, theta), x)


def _brute_topk(score, k):
    n = len(score)
    keep = []
    for c in range(n):
        better = sum(1 for j in range(n) if score[j] > score[c] or (score[j] == score[c] and j < c))
        if better < k:
            keep.append(c)
    return np.array(keep)


@pytest.mark.parametrize("n,rp", [(37, 0.5), (64, 0.7), (100, 0.3), (50, 1.0), (10, 0.01)])
def test_channel_select_brute_force(n, rp):
    v = np.round(RNG.standard_normal(n) * 3) / 2          # many ties on purpose
    got = od.channel_select(v, rp)
    k = math.ceil(rp * n - 1e-9)
    assert len(got) == max(1, k)
    np.testing.assert_array_equal(got, _brute_topk(np.abs(v), max(1, k)))
    # threshold property
    rest = np.setdiff1d(np.arange(n), got)
    if len(rest):
        assert np.abs(v[got]).min() >= np.abs(v[rest]).max()


def test_keep_count_rounding():
    assert od.keep_count(0.7, 14336) == 10036
    assert od.keep_count(0.5, 14336) == 7168
    assert od.keep_count(0.7, 4096) == 2868
    assert od.keep_count(0.3, 10) == 3          # 0.3*10 is 3.0000000000000004


def test_page_bound_is_an_upper_bound():
    hd, n_tok, page = 16, 77, 8
    keys = RNG.standard_normal((n_tok, hd))
    q = RNG.standard_normal((4, hd))
    kmin, kmax = od.page_bounds(keys, n_tok, page)
    s = od.page_scores(q, kmin, kmax)
    for p in range(len(s)):
        rows = keys[p * page:min((p + 1) * page, n_tok)]
        assert s[p] >= (q @ rows.T).max() - 1e-12
    # a one-token page: the bound is the exact logit
    kmin1, kmax1 = od.page_bounds(keys[:1], 1, page)
    assert od.page_scores(q, kmin1, kmax1)[0] == pytest.approx((q @ keys[0]).max(), rel=1e-13)


def test_page_bound_worked_example():
    q = np.array([[1.0, -2.0]])
    keys = np.array([[0.5, 1.0], [-1.0, 3.0]])
    kmin, kmax = od.page_bounds(keys, 2, 4)
    np.testing.assert_array_equal(kmin, [[-1.0, 1.0]])
    np.testing.assert_array_equal(kmax, [[0.5, 3.0]])
    # max(1*-1, 1*0.5) + max(-2*1, -2*3) = 0.5 + -2 = -1.5
    assert od.page_scores(q, kmin, kmax)[0] == -1.5


@pytest.mark.parametrize("P,rkv,sinks,recent", [(13, 0.5, 1, 2), (9, 0.3, 1, 8), (30, 0.3, 2, 3),
                                                 (5, 1.0, 1, 1), (4, 0.1, 2, 3), (1, 0.5, 1, 16)])
def test_page_select_brute_force(P, rkv, sinks, recent):
    scores = np.round(RNG.standard_normal(P) * 2)        # ties on purpose
    got = od.page_select(scores, rkv, sinks, recent)
    forced = sorted(set(range(min(sinks, P))) | set(range(max(P - recent, 0), P)))
    K = max(len(forced), min(P, math.ceil(rkv * P - 1e-9)))
    assert len(got) == K
    assert set(forced) <= set(got)
    free = [p for p in range(P) if p not in forced]
    want = [free[i] for i in _brute_topk(scores[free], K - len(forced))] if K > len(forced) else []
    assert sorted(set(forced) | set(want)) == list(got)


def test_attention_matches_sdpa():
    G, hd, T = 4, 32, 53
    q = RNG.standard_normal((G, hd))
    k = RNG.standard_normal((T, hd)) * 2
    v = RNG.standard_normal((T, hd))
    tok = np.array(sorted(RNG.choice(T, 29, replace=False)))
    got = od.attention(q, k, v, tok)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(k[tok])[None, None].expand(1, G, -1, -1),
        torch.from_numpy(v[tok])[None, None].expand(1, G, -1, -1))
    np.testing.assert_allclose(got, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-13)


def test_attention_with_additive_mask_matches_sdpa_boolean_mask():
    """The masked dense baseline's attention: an additive 0/-inf bias over
    every token equals SDPA with a boolean mask, and attention over the kept
    tokens alone."""
    G, hd, T = 4, 32, 80
    q = RNG.standard_normal((G, hd))
    k = RNG.standard_normal((T, hd)) * 2
    v = RNG.standard_normal((T, hd))
    keep = np.zeros(T, dtype=bool)
    keep[:16] = True
    keep[48:] = True
    bias = np.where(keep, 0.0, -np.inf)
    got = od.attention(q, k, v, np.arange(T), bias)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(k)[None, None].expand(1, G, -1, -1),
        torch.from_numpy(v)[None, None].expand(1, G, -1, -1), attn_mask=torch.from_numpy(keep)[None, None, None])
    np.testing.assert_allclose(got, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(got, od.attention(q, k, v, np.flatnonzero(keep)), rtol=1e-12, atol=1e-13)


def test_gemv_rows_matches_dense_and_masked():
    w = bf16_bits(torch.randn(40, 24).to(torch.bfloat16))
    x = RNG.standard_normal(40)
    rows = np.array([1, 5, 6, 30])
    xm = np.zeros(40)
    xm[rows] = x[rows]
    np.testing.assert_allclose(od.gemv_rows(x, w, rows), xm @ od.bf16_to_f64(w), rtol=1e-13)
    np.testing.assert_allclose(od.gemv_rows(x, w, None), x @ od.bf16_to_f64(w), rtol=1e-13)


# ----------------------------------------------------------------- whole decoder vs HF Llama (fp64)

N_CTX = 300


@pytest.fixture(scope="module")
def tiny():
    cfg = TINY
    w_t = make_weights(cfg, seed=0)
    k, v = make_kv(cfg, N_CTX, seed=1)
    w = {name: bf16_bits(t) for name, t in w_t.items()}
    return cfg, w_t, w, bf16_bits(k), bf16_bits(v)


def _hf_model(cfg, w_t):
    from transformers import LlamaConfig, LlamaForCausalLM
    hc = LlamaConfig(vocab_size=cfg["vocab"], hidden_size=cfg["hidden"],
                     intermediate_size=cfg["intermediate"], num_hidden_layers=cfg["n_layers"],
                     num_attention_heads=cfg["n_heads"], num_key_value_heads=cfg["n_kv_heads"],
                     head_dim=cfg["head_dim"], rms_norm_eps=cfg["rms_eps"],
                     rope_theta=cfg["rope_theta"], max_position_embeddings=65536,
                     tie_word_embeddings=False, attention_bias=False, mlp_bias=False)
    hc._attn_implementation = "eager"
    m = LlamaForCausalLM(hc).to(torch.float64).eval()
    Hq, Hkv, hd, f = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["intermediate"]
    d64 = {k: t.to(torch.float64) for k, t in w_t.items()}
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(d64["embed"])
        m.lm_head.weight.copy_(d64["lm_head"])
        m.model.norm.weight.copy_(d64["final_norm"])
        for l, layer in enumerate(m.model.layers):
            qkv = d64["wqkv_t"][l]
            layer.self_attn.q_proj.weight.copy_(qkv[:, :Hq * hd].T)
            layer.self_attn.k_proj.weight.copy_(qkv[:, Hq * hd:(Hq + Hkv) * hd].T)
            layer.self_attn.v_proj.weight.copy_(qkv[:, (Hq + Hkv) * hd:].T)
            layer.self_attn.o_proj.weight.copy_(d64["wo_t"][l].T)
            layer.mlp.gate_proj.weight.copy_(d64["wgu_t"][l][:, :f].T)
            layer.mlp.up_proj.weight.copy_(d64["wgu_t"][l][:, f:].T)
            layer.mlp.down_proj.weight.copy_(d64["wd_t"][l].T)
            layer.input_layernorm.weight.copy_(d64["attn_norm"][l])
            layer.post_attention_layernorm.weight.copy_(d64["mlp_norm"][l])
    return m


def _hf_step(m, cfg, kbits, vbits, n, token, hooks=()):
    from transformers.cache_utils import DynamicCache
    c = DynamicCache(config=m.config)
    for l in range(cfg["n_layers"]):
        c.update(torch.from_numpy(od.bf16_to_f64(kbits[l, :, :n]))[None],
                 torch.from_numpy(od.bf16_to_f64(vbits[l, :, :n]))[None], l)
    handles = [h() for h in hooks]
    try:
        with torch.no_grad():
            out = m(input_ids=torch.tensor([[token]]), past_key_values=c,
                    position_ids=torch.tensor([[n]]), cache_position=torch.tensor([n]), use_cache=True)
    finally:
        for h in handles:
            h.remove()
    return out.logits[0, 0].numpy()


def _close_to_hf(got, ref):
    """Hugging Face's Llama keeps its RMSNorm statistics and rotary angles in
    fp32 even for an fp64 model, so it agrees with a pure fp64 decoder to
    about 2e-6 of the largest logit; a wrong term, sign, index or operand
    moves the logits by O(1)."""
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


def _oracle(cfg, w, kbits, vbits, n, token, mode, **kw):
    cache = od.Cache(cfg, n + 4)
    cache.extend(kbits[:, :, :n], vbits[:, :, :n])
    trace = {}
    logits = od.decode_step(cfg, w, cache, token, mode, trace=trace, **kw)
    return logits, trace


def test_dense_decoder_matches_hf_llama(tiny):
    cfg, w_t, w, kb, vb = tiny
    m = _hf_model(cfg, w_t)
    tok = tokens(1, cfg["vocab"], seed=5)[0]
    ref = _hf_step(m, cfg, kb, vb, N_CTX, tok)
    got, _ = _oracle(cfg, w, kb, vb, N_CTX, tok, "dense", kv_round=False)
    _close_to_hf(got, ref)


def test_act_mode_matches_hf_with_masked_inputs(tiny):
    """The projection branch equals the dense model whose every projection
    input keeps only its top-k |x| channels (torch.topk) and zeroes the rest."""
    cfg, w_t, w, kb, vb = tiny
    m = _hf_model(cfg, w_t)
    rp = 0.5
    tok = tokens(2, cfg["vocab"], seed=5)[1]

    def mask_hook(mod, args):
        x = args[0]
        k = math.ceil(rp * x.shape[-1] - 1e-9)
        idx = torch.topk(x.abs(), k, dim=-1).indices
        keep = torch.zeros_like(x).scatter_(-1, idx, 1.0)
        return (x * keep,)

    mods = []
    for layer in m.model.layers:
        mods += [layer.self_attn.q_proj, layer.self_attn.k_proj, layer.self_attn.v_proj,
                 layer.self_attn.o_proj, layer.mlp.gate_proj, layer.mlp.up_proj, layer.mlp.down_proj]
    hooks = [(lambda mod=mod: mod.register_forward_pre_hook(mask_hook)) for mod in mods]
    ref = _hf_step(m, cfg, kb, vb, N_CTX, tok, hooks)
    got, _ = _oracle(cfg, w, kb, vb, N_CTX, tok, "act", rp=rp, kv_round=False)
    _close_to_hf(got, ref)
    dense, _ = _oracle(cfg, w, kb, vb, N_CTX, tok, "dense", kv_round=False)
    assert np.abs(dense - got).max() > 1e-3 * np.abs(dense).max()   # the branch does something


def test_kv_mode_matches_hf_with_head_masks(tiny):
    """The KV branch equals the dense model whose attention of each head is
    masked to the tokens of its kv head's selected pages."""
    cfg, w_t, w, kb, vb = tiny
    m = _hf_model(cfg, w_t)
    tok = tokens(3, cfg["vocab"], seed=5)[2]
    kw = dict(rkv=0.4, sinks=1, recent=2, kv_round=False)
    got, trace = _oracle(cfg, w, kb, vb, N_CTX, tok, "kv", **kw)
    n_tok, page, G = N_CTX + 1, cfg["page"], cfg["n_heads"] // cfg["n_kv_heads"]

    def layer_hook(l):
        mask = torch.full((1, cfg["n_heads"], 1, n_tok), float("-inf"), dtype=torch.float64)
        for h, sel in enumerate(trace[l]["pages"]):
            for p in sel:
                mask[0, h * G:(h + 1) * G, 0, p * page:min((p + 1) * page, n_tok)] = 0.0

        def hook(mod, args, kwargs):
            kwargs["attention_mask"] = mask
            return args, kwargs
        return hook

    hooks = [(lambda l=l, layer=layer: layer.self_attn.register_forward_pre_hook(layer_hook(l), with_kwargs=True))
             for l, layer in enumerate(m.model.layers)]
    ref = _hf_step(m, cfg, kb, vb, N_CTX, tok, hooks)
    _close_to_hf(got, ref)
    assert all(len(s) < -(-n_tok // page) for s in trace[0]["pages"])


def test_keep_one_reproduces_dense_exactly(tiny):
    cfg, _, w, kb, vb = tiny
    tok = tokens(4, cfg["vocab"], seed=5)[3]
    dense, _ = _oracle(cfg, w, kb, vb, N_CTX, tok, "dense")
    for mode in ("act", "kv", "both"):
        got, _ = _oracle(cfg, w, kb, vb, N_CTX, tok, mode, rp=1.0, rkv=1.0, sinks=1, recent=2)
        np.testing.assert_array_equal(got, dense)


def test_both_composes_the_branches(tiny):
    """'both' selects channels exactly as 'act' does on the same inputs and
    pages exactly as 'kv' does once the channel sets are fixed."""
    cfg, _, w, kb, vb = tiny
    tok = tokens(5, cfg["vocab"], seed=5)[4]
    kw = dict(rp=0.5, rkv=0.4, sinks=1, recent=2)
    both, tb = _oracle(cfg, w, kb, vb, N_CTX, tok, "both", **kw)
    forced = {}
    for l in range(cfg["n_layers"]):
        for site in ("qkv", "o", "gu", "d"):
            forced[(l, site)] = tb[l]["s_" + site]
    kv_forced, tk = _oracle(cfg, w, kb, vb, N_CTX, tok, "kv", forced=forced, **kw)
    np.testing.assert_array_equal(both, kv_forced)
    for l in range(cfg["n_layers"]):
        for a, b in zip(tb[l]["pages"], tk[l]["pages"]):
            np.testing.assert_array_equal(a, b)


def test_masked_dense_baseline_is_the_window(tiny):
    """The masked dense baseline computes the KV window (sinks and recent
    pages): it matches the kv mode with a keep ratio that leaves K = |F|."""
    cfg, _, w, kb, vb = tiny
    tok = tokens(6, cfg["vocab"], seed=5)[5]
    kw = dict(sinks=1, recent=2)
    masked, _ = _oracle(cfg, w, kb, vb, N_CTX, tok, "masked", **kw)
    window, tw = _oracle(cfg, w, kb, vb, N_CTX, tok, "kv", rkv=1e-6, **kw)
    P = -(-(N_CTX + 1) // 16)
    for l in range(cfg["n_layers"]):
        for sel in tw[l]["pages"]:
            assert set(sel.tolist()) == od.forced_pages(P, 1, 2)
    assert np.abs(masked - window).max() <= 1e-12 * np.abs(window).max()
    dense, _ = _oracle(cfg, w, kb, vb, N_CTX, tok, "dense")
    assert np.abs(masked - dense).max() > 1e-3 * np.abs(dense).max()


def test_appended_kv_is_rounded_to_bf16(tiny):
    cfg, _, w, kb, vb = tiny
    cache = od.Cache(cfg, N_CTX + 2)
    cache.extend(kb[:, :, :N_CTX], vb[:, :, :N_CTX])
    trace = {}
    od.decode_step(cfg, w, cache, 7, "dense", trace=trace)
    np.testing.assert_array_equal(cache.k[0, :, N_CTX], od.f64_to_bf16(trace[0]["k"]))
    assert cache.n == N_CTX + 1


# ----------------------------------------------------------------- once-after-prefill selection

def test_snap_scores_match_sdpa_page_masses():
    """Page scores are the attention mass per page: SDPA with one-hot page
    indicators as values gives each query's mass per page directly; a
    ragged last page counts only its valid tokens."""
    Q, hd, n, page = 12, 32, 77, 16
    q = RNG.standard_normal((Q, hd))
    k = RNG.standard_normal((n + 5, hd)) * 1.5
    got = od.snap_scores(q, k, n, page)
    P = -(-n // page)
    onehot = np.zeros((n, P))
    onehot[np.arange(n), np.arange(n) // page] = 1.0
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k[:n])[None, None],
        torch.from_numpy(onehot)[None, None])[0, 0].numpy().sum(axis=0)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)
    assert got.shape == (P,) and abs(got.sum() - Q) < 1e-12


def test_snap_scores_follow_a_planted_key():
    """A key aligned with every observation query draws almost all the
    mass to its page."""
    Q, hd, n, page = 8, 64, 160, 16
    u = RNG.standard_normal(hd)
    u /= np.linalg.norm(u)
    q = np.outer(np.ones(Q), u) * 4.0 + 0.01 * RNG.standard_normal((Q, hd))
    k = RNG.standard_normal((n, hd)) * 0.1
    k[83] = 40.0 * u                              # logit 4 * 40 / 8 = 20 above the rest
    sc = od.snap_scores(q, k, n, page)
    assert int(np.argmax(sc)) == 83 // page and sc[83 // page] > 0.99 * Q


def test_snap_select_keeps_forced_and_best(tiny):
    cfg, _, w, kb, vb = tiny
    cache = od.Cache(cfg, N_CTX + 4)
    cache.extend(kb[:, :, :N_CTX], vb[:, :, :N_CTX])
    rng = np.random.default_rng(3)
    q_obs = rng.standard_normal((cfg["n_layers"], 4, cfg["n_heads"], cfg["head_dim"]))
    kept, scores, P = od.snap_select(cfg, cache, q_obs, 0.3, 1, 2)
    assert P == -(-N_CTX // cfg["page"])
    for (l, h), sel in kept.items():
        F = od.forced_pages(P, 1, 2)
        assert F <= set(sel.tolist())
        K = max(len(F), math.ceil(0.3 * P - 1e-9))
        assert len(sel) == K
        rest = [p for p in range(P) if p not in F]
        best = sorted(rest, key=lambda p: (-scores[(l, h)][p], p))[:K - len(F)]
        assert set(best) == set(sel.tolist()) - F


def test_snap_mode_all_pages_is_dense_and_forced_only_is_the_window(tiny):
    """Keeping every page reproduces dense exactly; keeping only the forced
    pages, at a step inside the last selected page, is the kv mode's window
    (K = |F|) exactly."""
    cfg, _, w, kb, vb = tiny
    tok = tokens(6, cfg["vocab"], seed=5)[5]
    n = N_CTX - 3                                   # the step stays inside the last page
    P = -(-n // cfg["page"])
    everything = {(l, h): np.arange(P) for l in range(cfg["n_layers"]) for h in range(cfg["n_kv_heads"])}
    dense, _ = _oracle(cfg, w, kb, vb, n, tok, "dense")
    snap, _ = _oracle(cfg, w, kb, vb, n, tok, "snap", snap=(everything, P))
    np.testing.assert_array_equal(snap, dense)
    F = np.array(sorted(od.forced_pages(P, 1, 2)))
    only_forced = {key: F for key in everything}
    snap_f, ts = _oracle(cfg, w, kb, vb, n, tok, "snap", snap=(only_forced, P))
    window, tw = _oracle(cfg, w, kb, vb, n, tok, "kv", rkv=1e-6, sinks=1, recent=2)
    np.testing.assert_array_equal(snap_f, window)
    for l in range(cfg["n_layers"]):
        for a, b in zip(ts[l]["pages"], tw[l]["pages"]):
            np.testing.assert_array_equal(a, b)


def test_snap_mode_takes_pages_begun_after_the_selection(tiny):
    """A step that opens a new page attends over the frozen pages plus the
    new one."""
    cfg, _, w, kb, vb = tiny
    n = 18 * cfg["page"]                            # the step's token opens page 18
    P = n // cfg["page"]
    frozen = {(l, h): np.array([0, 5, P - 1]) for l in range(cfg["n_layers"]) for h in range(cfg["n_kv_heads"])}
    _, tr = _oracle(cfg, w, kb, vb, n, tokens(2, cfg["vocab"], seed=9)[1], "snap", snap=(frozen, P))
    for l in range(cfg["n_layers"]):
        for sel in tr[l]["pages"]:
            np.testing.assert_array_equal(sel, [0, 5, P - 1, P])
