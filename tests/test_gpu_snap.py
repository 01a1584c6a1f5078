"""Once-after-prefill page selection (the pages' own KV mode) on the GPU
through the C ABI, against the fp64 oracle.

* page scores (attention mass of the observation queries per page) within
  1e-4 of the number of observation queries, and the kept pages exact when
  the oracle ranks the GPU's own scores;
* snap decode steps over the frozen pages plus every page begun after the
  selection match the oracle (max relative error 1e-2), across a page
  boundary, through direct launches and graphs alike (bit-identical);
* a snap step without a valid selection is refused.
"""
import numpy as np
import pytest
import torch

import activation_kv_sparsity_b200 as bc
from oracle import decoder as od
from parity import REL_TOL, bits, max_rel, to_host
from synth import LLAMA_8B, TINY, make_kv, make_weights, obs_queries, tokens

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
SEL = dict(rkv=0.3, sinks=1, recent=4)


@pytest.fixture(scope="module")
def tiny():
    cfg = TINY
    w_t = make_weights(cfg, seed=0)
    return dict(cfg=cfg, wb={n: bits(t) for n, t in w_t.items()}, wd={n: t.to(DEV) for n, t in w_t.items()})


def _snap_traces(m, cfg):
    scores, pages = {}, {}
    for l in range(cfg["n_layers"]):
        sc = m.trace(l, bc.BC_TRACE_SNAP_SCORES).cpu().numpy().astype(np.float64)
        pg = m.trace(l, bc.BC_TRACE_SNAP_PAGES).cpu().numpy().astype(np.int64)
        for h in range(cfg["n_kv_heads"]):
            scores[(l, h)], pages[(l, h)] = sc[h], pg[h]
    return scores, pages


def _check_selection(cfg, cache, q_obs, gpu_scores, gpu_pages, n_obs):
    G = cfg["n_heads"] // cfg["n_kv_heads"]
    _, ref_scores, _ = od.snap_select(cfg, cache, q_obs.double().numpy(), SEL["rkv"], SEL["sinks"], SEL["recent"])
    for key, ref in ref_scores.items():
        err = np.abs(gpu_scores[key] - ref).max()
        assert err < 1e-4 * n_obs * G, (key, err)
        np.testing.assert_array_equal(od.page_select(gpu_scores[key], SEL["rkv"], SEL["sinks"], SEL["recent"]),
                                      gpu_pages[key], err_msg=str(key))


@pytest.mark.parametrize("n,n_obs", [(2048, 4), (777, 16), (40, 1)])
def test_snap_scores_and_pages(tiny, n, n_obs):
    cfg = tiny["cfg"]
    k, v = make_kv(cfg, n, seed=1)
    m = bc.Model(cfg, tiny["wd"], n + 64)
    m.append(k.to(DEV), v.to(DEV))
    q_obs = obs_queries(cfg, n_obs, seed=11)
    m.snap_select(q_obs.to(DEV), **SEL)
    torch.cuda.synchronize()
    scores, pages = _snap_traces(m, cfg)
    cache = od.Cache(cfg, n + 64)
    cache.extend(bits(k), bits(v))
    _check_selection(cfg, cache, q_obs, scores, pages, n_obs)
    P = -(-n // 16)
    for sc in scores.values():
        assert sc.shape == (P,) and abs(sc.sum() - n_obs * cfg["n_heads"] // cfg["n_kv_heads"]) < 1e-3
    m.close()


def _snap_model(t, n, n_obs=8):
    cfg = t["cfg"]
    k, v = make_kv(cfg, n, seed=1)
    m = bc.Model(cfg, t["wd"], n + 64)
    m.append(k.to(DEV), v.to(DEV))
    m.snap_select(obs_queries(cfg, n_obs, seed=12).to(DEV), **SEL)
    torch.cuda.synchronize()
    return m, k, v


def test_snap_steps_match_oracle(tiny):
    """Ten steps from 6 tokens before a page boundary: the oracle makes its
    own selection from the same observation queries (its scores leave a
    margin of 0.4% at every cut, far above the scorer's rounding, so the
    GPU's kept pages must equal it) and attends over those pages plus the
    page the steps open."""
    cfg = tiny["cfg"]
    n = 2048 - 6
    m, k, v = _snap_model(tiny, n)
    _, gpu_kept = _snap_traces(m, cfg)
    cache = od.Cache(cfg, n + 64)
    cache.extend(bits(k), bits(v))
    kept, _, P_snap = od.snap_select(cfg, cache, obs_queries(cfg, 8, seed=12).double().numpy(),
                                     SEL["rkv"], SEL["sinks"], SEL["recent"])
    for key, pages in kept.items():
        assert gpu_kept[key].tolist() == pages.tolist(), key
    logits = torch.empty(cfg["vocab"], device=DEV)
    for i, tok in enumerate(tokens(10, cfg["vocab"], seed=4)):
        m.step(tok, "snap", logits, **SEL)
        torch.cuda.synchronize()
        ref = od.decode_step(cfg, tiny["wb"], cache, tok, "snap", snap=(kept, P_snap))
        assert max_rel(to_host(logits), ref) < REL_TOL, i
    m.close()


def test_snap_graph_steps_equal_direct_steps(tiny):
    cfg = tiny["cfg"]
    outs = {}
    for graphs in (False, True):
        m, _, _ = _snap_model(tiny, 2048 - 6)
        m.set_graphs(graphs)
        logits = torch.empty(cfg["vocab"], device=DEV)
        seq = []
        for tok in tokens(12, cfg["vocab"], seed=4):
            m.step(tok, "snap", logits, **SEL)
            seq.append(logits.clone())
        torch.cuda.synchronize()
        outs[graphs] = seq
        m.close()
    for i, (a, b) in enumerate(zip(outs[False], outs[True])):
        assert torch.equal(a, b), i


def test_snap_step_needs_a_selection(tiny):
    cfg = tiny["cfg"]
    k, v = make_kv(cfg, 64, seed=1)
    m = bc.Model(cfg, tiny["wd"], 256)
    m.append(k.to(DEV), v.to(DEV))
    logits = torch.empty(cfg["vocab"], device=DEV)
    with pytest.raises(RuntimeError):
        m.step(3, "snap", logits)
    m.snap_select(obs_queries(cfg, 2, device=DEV), **SEL)
    m.step(3, "snap", logits)
    m.reset(60)
    with pytest.raises(RuntimeError):
        m.step(3, "snap", logits)
    m.close()


def test_llama8b_shape_snap_scores():
    """The Llama-3.1-8B shape at 4K context, 16 observation positions (64
    queries per kv head): scores and kept pages of layers 0 and 31."""
    cfg = dict(LLAMA_8B, n_layers=2)
    n = 4096
    w = make_weights(cfg, seed=0, device=DEV)
    k, v = make_kv(cfg, n, seed=1, device=DEV)
    m = bc.Model(cfg, w, n + 16)
    m.append(k, v)
    q_obs = obs_queries(cfg, 16, seed=11, device=DEV)
    m.snap_select(q_obs, **SEL)
    torch.cuda.synchronize()
    scores, pages = _snap_traces(m, cfg)
    cache = od.Cache(cfg, n + 16)
    cache.extend(bits(k), bits(v))
    _check_selection(cfg, cache, q_obs.cpu(), scores, pages, 16)
    m.close()


@pytest.mark.parametrize("n,n_obs", [(4096 + 16 * 37 + 5, 16), (40000 + 3, 16), (2560 + 7, 3), (3000, 32)])
def test_llama8b_shape_snap_tensor_core_path(n, n_obs):
    """The 8B layer shape (two layers) against the oracle where the scorer
    runs on tcgen05 (head_dim 128, n_obs*G <= 64): a ragged last page and
    tile, chunks of many tiles (40K tokens: both ring stages and both
    accumulators reused), few queries (12 of the 64 rows); and one shape
    beyond 64 queries, which stays on the mma.sync scorer."""
    cfg = dict(LLAMA_8B, n_layers=2)
    w = make_weights(cfg, seed=0, device=DEV)
    k, v = make_kv(cfg, n, seed=1, device=DEV)
    m = bc.Model(cfg, w, n + 16)
    m.append(k, v)
    q_obs = obs_queries(cfg, n_obs, seed=11, device=DEV)
    m.snap_select(q_obs, **SEL)
    torch.cuda.synchronize()
    scores, pages = _snap_traces(m, cfg)
    cache = od.Cache(cfg, n + 16)
    cache.extend(bits(k), bits(v))
    _check_selection(cfg, cache, q_obs.cpu(), scores, pages, n_obs)
    P = (n + 15) // 16
    G = cfg["n_heads"] // cfg["n_kv_heads"]
    for sc in scores.values():
        assert sc.shape == (P,) and abs(sc.sum() - n_obs * G) < 1e-3 * n_obs * G
    m.close()
