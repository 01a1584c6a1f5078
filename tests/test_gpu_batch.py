"""Batched projection over the union of the sequences' kept channels, through
the C ABI, against the oracle on the same seeded inputs: every output within
the GEMV's summation tolerance, the union size exact, and the edge cases the
op has (one sequence, all channels, one channel, identical sequences,
duplicate and out-of-range list entries)."""
import numpy as np
import pytest
import torch

import activation_kv_sparsity_b200 as bc
from oracle import batch as ob
from oracle import decoder as od
from parity import bits
from synth import batch_activations

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _weights(d_in, d_out, seed):
    g = torch.Generator()
    g.manual_seed(seed)
    return (torch.randn(d_in, d_out, generator=g) * 0.02).to(torch.bfloat16)


def _run(W, X, sels, k, idx_rows=None):
    """The library's batched GEMV; idx_rows overrides the list given to it."""
    d_in, d_out = W.shape
    B = X.shape[0]
    rows = sels if idx_rows is None else idx_rows
    idx = None if rows is None else torch.tensor(np.asarray(rows, dtype=np.int32)).to(DEV)
    y = torch.full((B, d_out), float("nan"), device=DEV)
    nu = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    scratch = torch.full((bc.bc_gemv_batch_scratch_bytes(d_in, d_out, B),), 0xFF, dtype=torch.uint8, device=DEV)
    bc.gemv_batch(W.to(DEV), X.to(DEV), idx, y, scratch, nu)
    torch.cuda.synchronize()
    return y.cpu().double().numpy(), int(nu.item())


def _check(y, W, X, sels):
    """Element-wise bound: |err| <= 1e-5 * sum |x_b[c] W[c, j]| over S_b (fp32
    accumulation of bf16 products against fp64)."""
    wb = bits(W)
    X64 = X.double().numpy()
    ref = ob.gemv_batch(wb, X64, sels)
    for b, s in enumerate(sels):
        s = np.asarray(s, dtype=np.int64)
        mag = np.abs(X64[b, s]) @ np.abs(od.bf16_to_f64(wb[s]))
        err = np.abs(y[b] - ref[b])
        assert (err <= 1e-5 * mag + 1e-30).all(), (b, float((err / (mag + 1e-30)).max()))


@pytest.mark.parametrize("d_in,d_out,B,k", [
    (40, 256, 1, 40), (300, 512, 3, 77), (512, 768, 2, 256), (1792, 512, 8, 900),
    (4096, 6144, 4, 2048), (4096, 28672, 4, 2048), (14336, 4096, 8, 7168), (4096, 4096, 5, 1),
    (4096, 4096, 7, 4096), (16384, 256, 6, 3000)])
def test_batched_gemv_matches_oracle(d_in, d_out, B, k):
    W = _weights(d_in, d_out, d_in + 13 * d_out + B)
    X = batch_activations(B, d_in, seed=d_in + B)
    sels = [od.channel_select(X[b].double().numpy(), 1.0, k=k) for b in range(B)]
    y, nu = _run(W, X, sels, k)
    assert nu == ob.union_channels(sels, d_in).shape[0]
    _check(y, W, X, sels)


def test_all_channels_without_a_list():
    d_in, d_out, B = 1000, 1024, 3
    W = _weights(d_in, d_out, 1)
    X = batch_activations(B, d_in, seed=2)
    sels = [np.arange(d_in)] * B
    y, nu = _run_none(W, X)
    assert nu == d_in
    _check(y, W, X, sels)


def _run_none(W, X):
    d_in, d_out = W.shape
    B = X.shape[0]
    y = torch.full((B, d_out), float("nan"), device=DEV)
    nu = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    scratch = torch.empty(bc.bc_gemv_batch_scratch_bytes(d_in, d_out, B), dtype=torch.uint8, device=DEV)
    bc.gemv_batch(W.to(DEV), X.to(DEV), None, y, scratch, nu)
    torch.cuda.synchronize()
    return y.cpu().double().numpy(), int(nu.item())


def test_identical_sequences_give_identical_rows():
    d_in, d_out, B = 4096, 2048, 4
    W = _weights(d_in, d_out, 3)
    x = batch_activations(1, d_in, seed=4)
    X = x.repeat(B, 1)
    s = od.channel_select(x[0].double().numpy(), 0.5)
    y, nu = _run(W, X, [s] * B, s.shape[0])
    assert nu == s.shape[0]
    for b in range(1, B):
        assert np.array_equal(y[0], y[b])
    _check(y, W, X, [s] * B)


def test_duplicates_and_out_of_range_entries_are_ignored():
    d_in, d_out, B, k = 600, 512, 3, 50
    W = _weights(d_in, d_out, 5)
    X = batch_activations(B, d_in, seed=6)
    rng = np.random.default_rng(7)
    sels = [np.sort(rng.choice(d_in, size=k - 10, replace=False)) for _ in range(B)]
    given = []
    for s in sels:
        extra = np.concatenate([s[:5], [-1, d_in, d_in + 7, -100, 2 ** 30]])
        given.append(rng.permutation(np.concatenate([s, extra])))
    y, nu = _run(W, X, sels, k, idx_rows=np.stack(given))
    assert nu == ob.union_channels(sels, d_in).shape[0]
    _check(y, W, X, sels)


def test_batched_gemv_is_deterministic_and_reuses_scratch():
    d_in, d_out, B, k = 4096, 4096, 8, 2048
    W = _weights(d_in, d_out, 8).to(DEV)
    X = batch_activations(B, d_in, seed=9).to(DEV)
    idx = torch.stack([torch.sort(torch.topk(X[b].abs(), k).indices)[0] for b in range(B)]).to(torch.int32)
    scratch = torch.empty(bc.bc_gemv_batch_scratch_bytes(d_in, d_out, B), dtype=torch.uint8, device=DEV)
    ys = []
    for _ in range(3):
        y = torch.empty(B, d_out, device=DEV)
        bc.gemv_batch(W, X, idx, y, scratch)
        ys.append(y)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


def test_library_select_then_batched_gemv_matches_oracle_chain():
    # the chain of a batched projection site: each sequence's exact top-k of
    # |x_b| by the library, then the union GEMV; against the oracle's top-k
    # and batched projection of the same inputs
    d_in, d_out, B = 4096, 6144, 4
    k = od.keep_count(0.5, d_in)
    W = _weights(d_in, d_out, 10)
    X = batch_activations(B, d_in, seed=11)
    Xd = X.to(DEV)
    idx = torch.empty(B, k, dtype=torch.int32, device=DEV)
    for b in range(B):
        bc.select_topk(Xd[b], k, idx[b])
    y = torch.empty(B, d_out, device=DEV)
    nu = torch.empty(1, dtype=torch.int32, device=DEV)
    scratch = torch.empty(bc.bc_gemv_batch_scratch_bytes(d_in, d_out, B), dtype=torch.uint8, device=DEV)
    bc.gemv_batch(W.to(DEV), Xd, idx, y, scratch, nu)
    torch.cuda.synchronize()
    sels = [od.channel_select(X[b].double().numpy(), 0.5) for b in range(B)]
    for b in range(B):
        assert idx[b].cpu().numpy().tolist() == sels[b].tolist()
    assert int(nu.item()) == ob.union_channels(sels, d_in).shape[0]
    _check(y.cpu().double().numpy(), W, X, sels)
