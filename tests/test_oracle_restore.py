"""Pins of the oracle's weight restore (CPU only).

Reading ("How dots-infra/ultraep works", summary paragraph: weights are
restored during backward): the layers share the redundant slots; before a
layer's expert backward its slots must hold the layer's forward replicas again.
restore(target plan, held plan) copies, into every redundant slot the target
fills with expert e and that does not hold e already, e's home slot.

Pinned by properties of a stack of layers sharing the slots, on tagged bytes
(every byte names its slot and offset): after restoring a layer, every slot
its plan fills is byte-identical to the state right after that layer's
forward sync (the sync is pinned by its own byte map); nothing else changed;
a slot the caller says holds the expert already is not written (a canary in it
survives); the copy count is the number of filled slots whose expert differs;
restoring the plan the slots hold copies nothing; with the holder unknown the
restore equals a full sync; and one hand-worked case.
"""
import numpy as np
import pytest

import oracle


def _tagged_slots(S, B):
    s = np.arange(S, dtype=np.uint32)[:, None]
    x = np.arange(B, dtype=np.uint32)[None, :]
    return ((s * 2654435761 + x * 40503 + (x >> 8)) & 0xFF).astype(np.uint8)


def _plans(E, N, R, n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        p = rng.permutation(E) + 1.0
        ld = rng.multinomial(4000, (p ** -1.4) / (p ** -1.4).sum()).astype(np.int32)
        out.append(oracle.plan(ld, N, R)["slot_expert"])
    return out


@pytest.mark.parametrize("E,N,R", [(16, 4, 1), (16, 4, 2), (12, 6, 3)])
def test_restore_layer_stack(E, N, R):
    H, HR = E // N, E // N + R
    S, B = N * HR, 384
    red = (np.arange(S) % HR) >= H
    layers = _plans(E, N, R, 6, seed=E + R)
    W = _tagged_slots(S, B)
    homes = W[~red].copy()
    # forward: each layer's sync; the slots then hold that layer's replicas
    after_fwd, held = [], np.full(S, -1, np.int32)
    for se in layers:
        oracle.sync(W, B, E, N, R, se)
        after_fwd.append(W.copy())
        held = np.where(red & (se >= 0), se, held)
    # backward, last layer first: restore each layer's replicas from what the slots hold
    for li in reversed(range(len(layers))):
        se = layers[li]
        filled = red & (se >= 0)
        changed = filled & (se != held)
        before = W.copy()
        n = oracle.sync_restore(W, B, E, N, R, se, held)
        assert n == int(changed.sum())
        assert np.array_equal(W[filled], after_fwd[li][filled])    # the layer's forward replicas are back
        assert np.array_equal(W[~filled], before[~filled])         # nothing else changed
        assert np.array_equal(W[~red], homes)
        held = np.where(filled, se, held)


def test_restore_skips_slots_that_hold_the_expert():
    E, N, R = 8, 4, 2
    H, HR = E // N, E // N + R
    S, B = N * HR, 128
    a, b = _plans(E, N, R, 2, seed=3)
    red = (np.arange(S) % HR) >= H
    same = red & (a >= 0) & (a == b)
    assert same.any()
    W = _tagged_slots(S, B)
    W[same] = 0xA5              # canary: the caller says these already hold their expert
    n = oracle.sync_restore(W, B, E, N, R, a, b)
    assert (W[same] == 0xA5).all()
    assert n == int((red & (a >= 0) & (a != b)).sum())


def test_restore_same_plan_copies_nothing_and_unknown_holder_is_full_sync():
    E, N, R = 8, 4, 1
    (se,) = _plans(E, N, R, 1, seed=5)
    S, B = N * (E // N + R), 256
    W = _tagged_slots(S, B)
    before = W.copy()
    assert oracle.sync_restore(W, B, E, N, R, se, se) == 0
    assert np.array_equal(W, before)
    full = W.copy()
    oracle.sync(full, B, E, N, R, se)
    n = oracle.sync_restore(W, B, E, N, R, se, None)
    assert n == int(((np.arange(S) % (E // N + R) >= E // N) & (se >= 0)).sum()) > 0
    assert np.array_equal(W, full)


def test_restore_hand_case():
    # E = 4, N = 2, R = 1: slots 0, 1 (rank 0 homes e0, e1), 2 (rank 0's
    # redundant slot), 3, 4 (rank 1 homes e2, e3), 5 (rank 1's redundant slot).
    # Layer A replicated e0 on rank 1 (slot 5) and nothing on rank 0; the slots
    # now hold layer B's replicas: e3 in slot 2, e0 in slot 5.  Restoring A:
    # slot 5 holds e0 already (not copied), slot 2 is empty under A (untouched).
    # Restoring B from A's state: slot 2 gets e3's home (slot 4), slot 5 keeps e0.
    E, N, R, B = 4, 2, 1, 32
    A = np.array([0, 1, -1, 2, 3, 0], np.int32)
    Bp = np.array([0, 1, 3, 2, 3, 0], np.int32)
    W = _tagged_slots(6, B)
    W[2] = W[4]
    W[5] = W[0]
    before = W.copy()
    assert oracle.sync_restore(W, B, E, N, R, A, Bp) == 0
    assert np.array_equal(W, before)
    W[2] = 0x11                                     # slot 2 now holds something else (layer A left it)
    assert oracle.sync_restore(W, B, E, N, R, Bp, A) == 1
    assert np.array_equal(W[2], W[4]) and np.array_equal(W[5], W[0])
    assert np.array_equal(np.delete(W, 2, axis=0), np.delete(before, 2, axis=0))
