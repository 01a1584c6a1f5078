"""Pins of the oracle's batched projection over the union of kept channels
(ByteCross README, "Usage: The byte account", crossover_batch): brute force on
tiny inputs, closed forms and invariants that a dropped term, a wrong index
or a transposed operand would break."""
import itertools

import numpy as np

from oracle import batch as ob
from oracle.decoder import bf16_to_f64, channel_select
from synth import BATCH_SHARED, batch_activations


def _bits(a):
    """bf16 bit patterns of a float array (truncation: exact for the small
    integers and halves used below)."""
    return (np.asarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_brute_force_tiny():
    rng = np.random.default_rng(0)
    d_in, d_out, B = 5, 3, 3
    W = rng.integers(-4, 5, size=(d_in, d_out)).astype(np.float64) / 2
    X = rng.integers(-3, 4, size=(B, d_in)).astype(np.float64)
    sels = [[0, 2], [1, 2, 4], [3]]
    y = ob.gemv_batch(_bits(W), X, sels)
    for b in range(B):
        for j in range(d_out):
            want = 0.0
            for c in range(d_in):
                if c in sels[b]:
                    want += X[b][c] * W[c][j]
            assert y[b, j] == want
    assert ob.union_channels(sels, d_in).tolist() == [0, 1, 2, 3, 4]
    assert ob.union_bytes(sels, d_in, d_out) == 5 * d_out * 2


def test_identity_weights_mask_each_sequence():
    # W = I: y_b is x_b with the channels outside S_b zeroed
    n, B = 16, 4
    rng = np.random.default_rng(1)
    X = rng.standard_normal((B, n)).round(2)
    sels = [np.sort(rng.choice(n, size=5 + b, replace=False)) for b in range(B)]
    y = ob.gemv_batch(_bits(np.eye(n)), X, sels)
    for b in range(B):
        want = np.zeros(n)
        want[sels[b]] = X[b, sels[b]]
        np.testing.assert_array_equal(y[b], want)


def test_a_sequence_ignores_channels_only_others_kept():
    # x_0 is large on channel 1, which only sequence 1 keeps
    W = np.ones((3, 2))
    X = np.array([[1.0, 100.0, 2.0], [0.0, 1.0, 0.0]])
    y = ob.gemv_batch(_bits(W), X, [[0, 2], [1]])
    np.testing.assert_array_equal(y, [[3.0, 3.0], [1.0, 1.0]])


def test_identical_sequences():
    rng = np.random.default_rng(2)
    W = rng.standard_normal((32, 8))
    x = rng.standard_normal(32)
    s = channel_select(x, 0.5)
    y = ob.gemv_batch(_bits(W), np.stack([x, x, x]), [s, s, s])
    assert np.array_equal(y[0], y[1]) and np.array_equal(y[1], y[2])
    assert ob.union_channels([s, s, s], 32).tolist() == s.tolist()
    assert ob.union_keep([s, s, s], 32) == 0.5


def test_disjoint_partition_sums_to_dense():
    # S_b = {c : c mod B == b} partitions the channels: the union is all of
    # them and, with one shared x, the rows of y sum to the dense product
    rng = np.random.default_rng(3)
    d_in, d_out, B = 24, 6, 4
    W = rng.standard_normal((d_in, d_out))
    wb = _bits(W)
    x = rng.standard_normal(d_in)
    sels = [np.arange(b, d_in, B) for b in range(B)]
    y = ob.gemv_batch(wb, np.stack([x] * B), sels)
    np.testing.assert_allclose(y.sum(axis=0), x @ bf16_to_f64(wb), rtol=1e-12, atol=1e-12)
    assert ob.union_keep(sels, d_in) == 1.0
    assert sum(len(s) for s in sels) == ob.union_channels(sels, d_in).shape[0]


def test_union_is_brute_force_union():
    rng = np.random.default_rng(4)
    for _ in range(20):
        d_in = int(rng.integers(1, 40))
        B = int(rng.integers(1, 6))
        sels = [np.sort(rng.choice(d_in, size=int(rng.integers(1, d_in + 1)), replace=False))
                for _ in range(B)]
        want = sorted(set(itertools.chain.from_iterable(s.tolist() for s in sels)))
        assert ob.union_channels(sels, d_in).tolist() == want


def test_union_keep_of_independent_halves():
    # with no shared component the kept sets are close to independent halves:
    # the union covers about 1 - 2^-B of the channels
    d = 4096
    for B in (2, 4):
        keeps = []
        for seed in range(8):
            X = batch_activations(B, d, shared=0.0, seed=100 + seed).double().numpy()
            keeps.append(ob.union_keep([channel_select(X[b], 0.5) for b in range(B)], d))
        assert abs(np.mean(keeps) - (1 - 0.5 ** B)) < 0.01, (B, np.mean(keeps))


def test_batch_recipe_overlap():
    # the synthetic batch's shared component gives the README's union of
    # about 92% at four sequences (rp 0.5)
    d = 4096
    keeps = []
    for seed in range(8):
        X = batch_activations(4, d, seed=200 + seed).double().numpy()
        keeps.append(ob.union_keep([channel_select(X[b], 0.5) for b in range(4)], d))
    assert BATCH_SHARED > 0
    assert abs(np.mean(keeps) - 0.92) < 0.01, np.mean(keeps)
