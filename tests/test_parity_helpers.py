"""The GPU tests check each GPU selection against its own fp32 scores with
test-side restatements of the selection rules (the oracle never receives a
GPU value).  Here those restatements are checked against the oracle's
definitions on small inputs with many ties."""
import numpy as np

import parity as pa
from oracle import decoder as od


def test_topk_and_page_rules_match_the_oracle():
    rng = np.random.default_rng(0)
    for _ in range(400):
        P = int(rng.integers(1, 70))
        sc = rng.integers(0, 5, P).astype(float)            # many ties
        rkv = float(rng.uniform(0.005, 1.0))
        sinks, recent = int(rng.integers(0, 4)), int(rng.integers(1, 6))
        assert pa.pages_of(sc, rkv, sinks, recent).tolist() == od.page_select(sc, rkv, sinks, recent).tolist()
        k = int(rng.integers(1, P + 1))
        assert pa.topk_of(sc, k).tolist() == od.channel_select(sc, 1.0, k=k).tolist()
