"""The batched decode step (bc_batch_*) on the GPU, against the fp64 oracle's
batch-1 step of each sequence.

A batch of sequences, each with its own synthetic cache and tokens, decodes in
lock step: every sequence keeps its own channels and pages, the projections
read the union of the batch's kept rows once.  For every sequence the test
checks what the batch-1 tests check (tests/parity.py): the GPU's sets are
exact on its own pre-selection scores, the oracle -- run from that
sequence's own inputs and told only its index sets -- agrees with every
layer's hidden state and the logits within 1e-2, and the sets differ from
the oracle's own choice only at near-ties.
"""
import pytest
import torch

import activation_kv_sparsity_b200 as bc
from oracle import decoder as od
from parity import bits, compare_step, gpu_traces, max_rel, to_host
from synth import LLAMA_8B, TINY, kv_chunks, make_weights, tokens

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
N_CTX = 2048


def _draw_caches(cfg, B, n, seed0=1):
    """One synthetic cache per sequence: [B][L][Hkv][n][hd] bf16 on the device."""
    ks, vs = [], []
    for b in range(B):
        k, v = zip(*kv_chunks(cfg, n, seed=seed0 + b, device=DEV))
        ks.append(torch.cat(k, dim=2))
        vs.append(torch.cat(v, dim=2))
    return torch.stack(ks), torch.stack(vs)


@pytest.fixture(scope="module")
def tiny3():
    cfg, B = TINY, 3
    w = make_weights(cfg, seed=0, device=DEV)
    k, v = _draw_caches(cfg, B, N_CTX)
    return dict(cfg=cfg, B=B, wd=w, wb={n: bits(t) for n, t in w.items()}, k=k, v=v)


def _oracle_caches(t, cap):
    caches = []
    for b in range(t["B"]):
        c = od.Cache(t["cfg"], cap)
        c.extend(bits(t["k"][b]), bits(t["v"][b]))
        caches.append(c)
    return caches


@pytest.mark.parametrize("mode", ["dense", "act", "kv", "both"])
def test_batch_steps_match_the_oracle_per_sequence(tiny3, mode):
    t, cfg, B = tiny3, tiny3["cfg"], tiny3["B"]
    kw = dict(rp=0.5, rkv=0.5, sinks=1, recent=8)
    bt = bc.Batch(cfg, t["wd"], B, N_CTX + 16)
    bt.append(t["k"], t["v"])
    caches = _oracle_caches(t, N_CTX + 16)
    logits = torch.empty(B, cfg["vocab"], device=DEV)
    toks = [tokens(4, cfg["vocab"], seed=30 + b) for b in range(B)]
    for i in range(4):
        bt.step([toks[b][i] for b in range(B)], mode, logits, **kw)
        torch.cuda.synchronize()
        for b in range(B):
            tr = gpu_traces(bt.seq(b), cfg["n_layers"], mode in ("kv", "both"))
            compare_step(cfg, t["wb"], caches[b], toks[b][i], mode, kw["rp"], kw["rkv"], kw["sinks"],
                         kw["recent"], to_host(logits[b]), tr)
    assert len(bt) == N_CTX + 4
    bt.close()


def test_identical_sequences_give_identical_logits(tiny3):
    """Each sequence's arithmetic is independent of its neighbours: copies of
    one sequence in a batch come out bit for bit the same."""
    t, cfg = tiny3, tiny3["cfg"]
    B = 4
    bt = bc.Batch(cfg, t["wd"], B, N_CTX + 8)
    bt.append(t["k"][:1].expand(B, -1, -1, -1, -1), t["v"][:1].expand(B, -1, -1, -1, -1))
    logits = torch.empty(B, cfg["vocab"], device=DEV)
    for mode in ("dense", "both"):
        bt.reset(N_CTX)
        bt.step([77] * B, mode, logits, rp=0.5, rkv=0.5, sinks=1, recent=8)
        torch.cuda.synchronize()
        for b in range(1, B):
            assert torch.equal(logits[b], logits[0]), (mode, b)
    bt.close()


def test_batch_graph_steps_equal_direct_steps(tiny3):
    """Steps replayed from the captured graph equal direct launches bit for
    bit, across page boundaries (page counts and the attention grid change)."""
    t, cfg, B = tiny3, tiny3["cfg"], tiny3["B"]
    outs = {}
    for graphs in (False, True):
        bt = bc.Batch(cfg, t["wd"], B, N_CTX + 32)
        bt.append(t["k"], t["v"])
        bt.set_graphs(graphs)
        bt.reset(N_CTX - 20)
        logits = torch.empty(B, cfg["vocab"], device=DEV)
        seq = []
        for i, tok in enumerate(tokens(24, cfg["vocab"], seed=41)):
            bt.step([tok, tok + 1, tok + 2], "both", logits, rp=0.5, rkv=0.5, sinks=1, recent=8)
            seq.append(logits.clone())
        torch.cuda.synchronize()
        outs[graphs] = seq
        bt.close()
    for i, (a, b) in enumerate(zip(outs[False], outs[True])):
        assert torch.equal(a, b), i


def test_batch_of_one_matches_the_batch1_step(tiny3):
    """A batch of one sequence computes the batch-1 step (different kernels,
    so equal up to fp32 summation order)."""
    t, cfg = tiny3, tiny3["cfg"]
    kw = dict(rp=0.5, rkv=0.5, sinks=1, recent=8)
    bt = bc.Batch(cfg, t["wd"], 1, N_CTX + 8)
    bt.append(t["k"][:1], t["v"][:1])
    m = bc.Model(cfg, t["wd"], N_CTX + 8)
    m.append(t["k"][0], t["v"][0])
    lb = torch.empty(1, cfg["vocab"], device=DEV)
    lm = torch.empty(cfg["vocab"], device=DEV)
    for mode in ("dense",):            # no selection: nothing can straddle a near-tie
        bt.reset(N_CTX)
        m.reset(N_CTX)
        bt.step([123], mode, lb, **kw)
        m.step(123, mode, lm, **kw)
        torch.cuda.synchronize()
        assert max_rel(to_host(lb[0]), to_host(lm)) < 1e-4, mode
    bt.close()
    m.close()


def test_batch_rejects_bad_arguments(tiny3):
    t, cfg = tiny3, tiny3["cfg"]
    bt = bc.Batch(cfg, t["wd"], 2, 64)
    logits = torch.empty(2, cfg["vocab"], device=DEV)
    for mode, kw in (("snap", {}), ("masked", {}), ("both", dict(rp=0.0)), ("kv", dict(recent=0))):
        with pytest.raises(bc.BCError) as e:
            bt.step([1, 2], mode, logits, **kw)
        assert e.value.status == bc.BC_EINVAL
    with pytest.raises(bc.BCError) as e:
        bt.step([1, cfg["vocab"]], "dense", logits)
    assert e.value.status == bc.BC_EINVAL
    bt.close()


def test_llama8b_layer_shape_batch():
    """Two layers of the Llama-3.1-8B shape, a batch of 2 at 4096 tokens in
    mode both (rp 0.5, rkv 0.3): each sequence against the oracle."""
    cfg = dict(LLAMA_8B, n_layers=2)
    B, n = 2, 4096
    kw = dict(rp=0.5, rkv=0.3, sinks=1, recent=16)
    w = make_weights(cfg, seed=0, device=DEV)
    wb = {name: bits(x) for name, x in w.items()}
    k, v = _draw_caches(cfg, B, n)
    bt = bc.Batch(cfg, w, B, n + 8)
    bt.append(k, v)
    logits = torch.empty(B, cfg["vocab"], device=DEV)
    toks = [4242, 17]
    bt.step(toks, "both", logits, **kw)
    torch.cuda.synchronize()
    for b in range(B):
        cache = od.Cache(cfg, n + 1)
        cache.extend(bits(k[b]), bits(v[b]))
        tr = gpu_traces(bt.seq(b), cfg["n_layers"], True)
        compare_step(cfg, wb, cache, toks[b], "both", kw["rp"], kw["rkv"], kw["sinks"], kw["recent"],
                     to_host(logits[b]), tr)
    bt.close()


@pytest.mark.parametrize("mode", ["dense", "both"])
def test_batch_of_eight_on_the_tensor_core_projection(mode):
    """Eight sequences (the projections run on the tensor-core kernel from
    seven on): every sequence against the oracle's batch-1 step, two steps."""
    cfg, B = TINY, 8
    w = make_weights(cfg, seed=0, device=DEV)
    k, v = _draw_caches(cfg, B, 600, seed0=40)
    t = dict(cfg=cfg, B=B, wd=w, wb={n: bits(x) for n, x in w.items()}, k=k, v=v)
    kw = dict(rp=0.5, rkv=0.5, sinks=1, recent=8)
    bt = bc.Batch(cfg, w, B, 600 + 8)
    bt.append(k, v)
    caches = _oracle_caches(t, 600 + 8)
    logits = torch.empty(B, cfg["vocab"], device=DEV)
    toks = [tokens(2, cfg["vocab"], seed=60 + b) for b in range(B)]
    for i in range(2):
        bt.step([toks[b][i] for b in range(B)], mode, logits, **kw)
        torch.cuda.synchronize()
        for b in range(B):
            tr = gpu_traces(bt.seq(b), cfg["n_layers"], mode in ("kv", "both"))
            compare_step(cfg, t["wb"], caches[b], toks[b][i], mode, kw["rp"], kw["rkv"], kw["sinks"],
                         kw["recent"], to_host(logits[b]), tr)
    bt.close()
