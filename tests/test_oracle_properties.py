"""Property-based pins of the oracle (hypothesis): invariants the pages and
the mathematics fix at any size, so that a slip in an index, a sign or a
term fails for some drawn input."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import batch as ob
from oracle import byte_account as ba
from oracle import decoder as od
from synth import LLAMA_8B, TINY

MODELS = [TINY, LLAMA_8B]
ratio = st.floats(min_value=0.01, max_value=1.0, allow_nan=False)


@settings(max_examples=60, deadline=None)
@given(m=st.sampled_from(MODELS), mode=st.sampled_from(["dense", "act", "kv", "both", "snap"]),
       n=st.integers(min_value=0, max_value=200000), rp=ratio, rkv=ratio)
def test_implementation_bytes_never_exceed_dense_and_grow_with_context(m, mode, n, rp, rkv):
    kw = dict(rp=rp, rkv=rkv, sinks=1, recent=16)
    b = ba.implementation_bytes(m, mode, n, **kw)
    d = ba.implementation_bytes(m, "dense", n, **kw)
    # the weights and the KV a sparse step reads are at most the dense step's
    assert b["weights"] <= d["weights"] and b["kv_read"] <= d["kv_read"]
    assert b["total"] == sum(b[k] for k in ("weights", "head", "kv_read", "meta_read", "kv_write", "other"))
    assert ba.implementation_bytes(m, mode, n + 16, **kw)["kv_read"] >= b["kv_read"]


@settings(max_examples=60, deadline=None)
@given(m=st.sampled_from(MODELS), n=st.integers(min_value=0, max_value=1 << 20), rp=ratio, rkv=ratio)
def test_bound_is_at_least_one_and_composition_saves_most(m, n, rp, rkv):
    both = ba.bound(m, n, rp, rkv)
    assert both >= ba.bound(m, n, rp, 1.0) >= 1.0
    assert both >= ba.bound(m, n, 1.0, rkv) >= 1.0
    # saved bytes add across the branches
    s = ba.saved_bytes(m, n, rp, rkv)
    assert abs(s - ba.saved_bytes(m, n, rp, 1.0) - ba.saved_bytes(m, n, 1.0, rkv)) <= 1e-6 * max(s, 1.0)


@settings(max_examples=60, deadline=None)
@given(m=st.sampled_from(MODELS), u=st.floats(min_value=0.01, max_value=0.99),
       rkv=st.floats(min_value=0.01, max_value=0.99), batch=st.integers(min_value=1, max_value=64))
def test_crossover_batch_scales_inversely_with_batch_and_meets_equation5(m, u, rkv, batch):
    n, n1 = ba.crossover_batch(m, u, rkv, batch), ba.crossover_batch(m, u, rkv, 1)
    assert n1 > 0 and abs(n * batch - n1) <= 1e-9 * n1
    # one sequence keeping a fraction u is Equation 5 with rp = u
    assert abs(ba.crossover_batch(m, u, rkv, 1) - ba.crossover(m, u, rkv)) <= 1e-9 * ba.crossover(m, u, rkv)


@settings(max_examples=40, deadline=None)
@given(seed=st.integers(min_value=0, max_value=2 ** 31 - 1), B=st.integers(min_value=1, max_value=6),
       d_in=st.integers(min_value=1, max_value=40), d_out=st.integers(min_value=1, max_value=12))
def test_batched_projection_is_linear_and_the_union_only_grows(seed, B, d_in, d_out):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((d_in, d_out)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    X = rng.standard_normal((B, d_in))
    sels = [np.sort(rng.choice(d_in, size=int(rng.integers(1, d_in + 1)), replace=False)) for _ in range(B)]
    y = ob.gemv_batch(W, X, sels)
    a = float(rng.uniform(-2, 2))
    np.testing.assert_allclose(ob.gemv_batch(W, a * X, sels), a * y, rtol=1e-12, atol=1e-12)
    # every row of y is the batch-1 projection of its own input over its own set
    for b in range(B):
        np.testing.assert_allclose(y[b], od.gemv_rows(X[b], W, sels[b]), rtol=1e-12, atol=1e-12)
    keeps = [ob.union_keep(sels[:j], d_in) for j in range(1, B + 1)]
    assert all(x <= y_ for x, y_ in zip(keeps, keeps[1:]))
    assert keeps[-1] <= 1.0 and keeps[0] == len(sels[0]) / d_in
