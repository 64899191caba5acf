"""The benchmark's NVLink model of the relay: its per-round and direct egress
per GPU equal the bytes the oracle's relay schedule sends from each GPU, on
random plans (CPU only)."""
import os
import sys

import numpy as np
import pytest

import oracle
from moe_expert_load_ue_b200 import inputs

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


@pytest.mark.parametrize("seed", range(12))
def test_model_egress_matches_oracle_schedule(seed):
    rng = np.random.default_rng(70 + seed)
    N = int(rng.choice([8, 16, 64]))
    H, R = int(rng.integers(1, 4)), int(rng.integers(1, 3))
    E = N * H
    w = inputs.TINY.with_(E=E, N=N, R=R)
    p = (rng.permutation(E) + 1.0) ** -1.5
    load = rng.multinomial(50000, p / p.sum()).astype(np.int32)
    se = oracle.plan(load, N, R)["slot_expert"]
    G = int(rng.choice([g for g in (2, 4, 8, 16) if N % g == 0]))
    nb = int(rng.choice([16, 96, 4000]))
    m = bench.nvlink_model(se, w, G, nb, 770.0)
    W = np.zeros((se.size, nb), np.uint8)
    for k in range(oracle.relay_rounds(G)):
        assert np.array_equal(m["relay_egress"][k], oracle.sync_relay(W, nb, E, N, R, se, G, k)), k
    assert np.array_equal(m["direct_egress"], oracle.sync_relay(W, nb, E, N, R, se, G, -1))
