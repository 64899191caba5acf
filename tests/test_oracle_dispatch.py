"""Pins for the oracle's dispatch layout (CPU only).

Token dispatch receives the physical routing of routing expansion and groups
the (t, k) assignments by physical slot.  The checks use hand-worked layouts
(tests/golden/dispatch_cases.json), numpy's stable argsort as an independent
library restatement, the plan's slot quotas (segment lengths) and the
structural properties of a stable grouping.
"""
import json
import os

import numpy as np
import pytest

import oracle
from moe_expert_load_ue_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dispatch_cases.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def _dyadic_gates(L):
    # distinct, exactly representable values: a dropped or shuffled gate is visible
    return ((np.arange(L) % 4096) + 1).astype(np.float32) / 8192.0


@pytest.mark.parametrize("case", _golden(), ids=lambda c: c["name"])
def test_dispatch_hand_cases(case):
    ids = np.array(case["ids"], np.int32).reshape(-1, case["K"])
    out = oracle.rebalance(ids, case["E"], case["N"], case["R"])
    if "phys" in case:
        assert out["phys"].ravel().tolist() == case["phys"]
    if "slot_quota" in case:
        assert out["plan"]["slot_quota"].tolist() == case["slot_quota"]
    S = out["plan"]["slot_quota"].shape[0]
    gates = _dyadic_gates(ids.size)
    slot_off, src, gout = oracle.dispatch(out["phys"], S, gates)
    assert slot_off.tolist() == case["slot_off"]
    assert src.tolist() == case["src_index"]
    assert np.array_equal(gout, gates[np.array(case["src_index"], np.int64)])


def dispatch_by_argsort(phys, S):
    """Library restatement: a stable argsort of the valid assignments by slot,
    and the segment starts from searchsorted."""
    flat = phys.ravel()
    idx = np.nonzero(flat >= 0)[0]
    order = idx[np.argsort(flat[idx], kind="stable")]
    starts = np.searchsorted(flat[order], np.arange(S + 1), side="left")
    return starts.astype(np.int32), order.astype(np.int32)


@pytest.mark.parametrize("w", [inputs.TINY, inputs.CLASS_106B.with_(tokens_per_rank=512),
                               inputs.CLASS_671B.with_(tokens_per_rank=256),
                               inputs.EXTREME.with_(tokens_per_rank=64)], ids=lambda w: w.name)
def test_dispatch_matches_stable_argsort_and_quotas(w):
    ids = inputs.topk_ids(w, 2)
    out = oracle.rebalance(ids, w.E, w.N, w.R)
    phys, pl = out["phys"], out["plan"]
    gates = inputs.gates(ids, w, 2)
    slot_off, src, gout = oracle.dispatch(phys, w.S, gates)
    ref_off, ref_src = dispatch_by_argsort(phys, w.S)
    assert np.array_equal(slot_off, ref_off)
    assert np.array_equal(src, ref_src)
    # segment lengths are the plan's slot quotas (every id is valid here)
    assert np.array_equal(np.diff(slot_off), pl["slot_quota"])
    # every segment holds only its own slot, in increasing flat index
    flat = phys.ravel()
    for s in range(w.S):
        seg = src[slot_off[s]:slot_off[s + 1]]
        assert (flat[seg] == s).all()
        assert (np.diff(seg) > 0).all()
    # a permutation of all assignments; gates carried bit for bit
    assert np.array_equal(np.sort(src), np.arange(ids.size))
    assert np.array_equal(gout.view(np.uint32), gates.ravel()[src].view(np.uint32))


def test_dispatch_drops_bad_ids():
    rng = np.random.default_rng(11)
    E, N, R = 12, 3, 1
    ids = rng.integers(-3, E + 3, size=(42, 4)).astype(np.int32)
    out = oracle.rebalance(ids, E, N, R)
    S = N * (E // N + R)
    slot_off, src, gout = oracle.dispatch(out["phys"], S)
    valid = ((ids >= 0) & (ids < E)).ravel()
    assert gout is None
    assert slot_off[S] == valid.sum()
    assert np.array_equal(np.sort(src), np.nonzero(valid)[0])
    ref_off, ref_src = dispatch_by_argsort(out["phys"], S)
    assert np.array_equal(slot_off, ref_off) and np.array_equal(src, ref_src)


def test_dispatch_empty_and_single_slot():
    slot_off, src, _ = oracle.dispatch(np.zeros((0, 8), np.int32), 5)
    assert slot_off.tolist() == [0] * 6 and src.size == 0
    phys = np.full((3, 2), 2, np.int32)
    slot_off, src, _ = oracle.dispatch(phys, 4)
    assert slot_off.tolist() == [0, 0, 0, 6, 6] and src.tolist() == list(range(6))


def test_dispatch_rejects_out_of_range_slots():
    with pytest.raises(oracle.OracleError):
        oracle.dispatch(np.array([0, 4], np.int32), 4)
    with pytest.raises(oracle.OracleError):
        oracle.dispatch(np.array([0, -2], np.int32), 4)
