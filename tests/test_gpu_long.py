"""Decode-step parity at the context lengths the KV branch takes in the
benchmark, on the Llama-3.1-8B layer shape (hd 128, 8 kv heads, groups of 4,
hidden 4096, intermediate 14336, vocab 128256) with two layers.

At these lengths the page scorer makes several rounds per CTA with the next
round's bounds in flight, and the page select takes each of its variants:
the one-CTA select with 4 keys a thread (2049-4096 pages), with 8 keys a
thread (4097-8192 pages), and the 8-CTA cluster (8193 pages and more).  Each
case compares with the fp64 oracle:

* every page score, element by element, within 1e-4 of the head's score
  scale (the GPU scores its fp32 queries, the oracle its fp64 ones);
* the page sets: exact on the GPU's own scores, and against the oracle's own
  scores different only at near-ties (tests/parity.py);
* the channel sets the same way (act and both modes);
* each layer's hidden state and the logits within max relative error 1e-2.

Keep counts are ceil(r*n - 1e-9) in double on both sides; the 1280-page case
(0.3 * 1280 = 384 exactly) pins that the library keeps 384 pages, not 385.
"""
import numpy as np
import pytest
import torch

import activation_kv_sparsity_b200 as bc
from oracle import decoder as od
from parity import bits, compare_step, gpu_traces, to_host
from synth import LLAMA_8B, kv_chunks, make_weights

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
CFG2 = dict(LLAMA_8B, n_layers=2)
N_MAX = 131088                       # 8194 pages once the step's token lands: the cluster select
SCORE_TOL = 1e-4

# (mode, rp, rkv, cached tokens): what each case exercises
CASES = [
    ("kv", 1.0, 0.3, 20479),         # P = 1280: K = 0.3 * 1280 = 384 exactly
    ("kv", 1.0, 0.3, 32768),         # P = 2049: one-CTA select, 4 keys a thread
    ("both", 0.7, 0.3, 32768),       # rp 0.7: 2868 of 4096 and 10036 of 14336 rows
    ("kv", 1.0, 0.5, 65536),         # P = 4097: one-CTA select, 8 keys a thread
    ("kv", 1.0, 0.3, N_MAX),         # P = 8194: the 8-CTA cluster select
    ("both", 0.5, 0.3, N_MAX),
    ("act", 0.7, 1.0, 4096),
]


@pytest.fixture(scope="module")
def long_ctx():
    w = make_weights(CFG2, seed=0, device=DEV)
    ks, vs = [], []
    for k, v in kv_chunks(CFG2, N_MAX, seed=1, device=DEV):
        ks.append(k)
        vs.append(v)
    kd, vd = torch.cat(ks, dim=2), torch.cat(vs, dim=2)
    del ks, vs
    m = bc.Model(CFG2, w, N_MAX + 16)
    m.append(kd, vd)
    torch.cuda.synchronize()
    yield dict(m=m, wd=w, wb={n: bits(t) for n, t in w.items()}, kd=kd, vd=vd, kb=bits(kd), vb=bits(vd))
    m.close()


def _restore(t, n):
    """Put the pristine synthetic tokens back from the page the step wrote on."""
    p0 = (n // 16) * 16
    t["m"].reset(p0)
    t["m"].append(t["kd"][:, :, p0:], t["vd"][:, :, p0:])


@pytest.mark.parametrize("mode,rp,rkv,n", CASES, ids=[f"{c[0]}-{c[1]}-{c[2]}-{c[3]}" for c in CASES])
def test_long_context_step_matches_oracle(long_ctx, mode, rp, rkv, n):
    t = long_ctx
    m = t["m"]
    sinks, recent = 1, 16
    kvsel = mode in ("kv", "both")
    m.reset(n)
    logits = torch.empty(CFG2["vocab"], device=DEV)
    tok = 31337
    m.step(tok, mode, logits, rp=rp, rkv=rkv, sinks=sinks, recent=recent)
    torch.cuda.synchronize()
    tr = gpu_traces(m, CFG2["n_layers"], kvsel)
    _restore(t, n)
    cache = od.Cache(CFG2, n + 1)
    cache.extend(t["kb"][:, :, :n], t["vb"][:, :, :n])
    _, trace = compare_step(CFG2, t["wb"], cache, tok, mode, rp, rkv, sinks, recent, to_host(logits), tr)
    P = -(-(n + 1) // 16)
    if kvsel:
        K = max(1 + recent, int(np.ceil(rkv * P - 1e-9)))
        for l in range(CFG2["n_layers"]):
            assert tr[l]["page_scores"].shape == (CFG2["n_kv_heads"], P)
            assert tr[l]["pages"].shape == (CFG2["n_kv_heads"], K)
            for h in range(CFG2["n_kv_heads"]):
                ref = trace[l]["page_scores"][h]
                err = np.abs(tr[l]["page_scores"][h] - ref).max() / np.abs(ref).max()
                assert err < SCORE_TOL, (l, h, err)
        if n == 20479:
            assert K == 384
    if mode in ("act", "both"):
        want = {"qkv": 2868, "o": 2868, "gu": 2868, "d": 10036} if rp == 0.7 else None
        if want:
            for site, k in want.items():
                assert len(tr[0]["s_" + site]) == k, site
