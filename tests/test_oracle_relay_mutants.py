"""The relay pins catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle's relay code (the copy
is compiled into a temporary library; the oracle itself is untouched) and
checks that the hand-worked schedules or the reach-the-single-GPU-sync
property reject it:
  - the all-gather round taking the parts from the home instead of the
    consumers (the slots still end right: only the egress pins see it);
  - parts rounded down instead of up (the tail of each slot is never copied);
  - the home GPU's own replicas left unfilled;
  - consumers numbered in reverse (a part is taken from a GPU that does not
    hold it).
"""
import ctypes
import json
import os
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "ue_oracle.c")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "relay_cases.json")

MUTANTS = {
    "all-gather from the home": ("src = first[j]; lo = j * q;", "src = home; lo = j * q;"),
    "parts rounded down": ("16 * ((nbytes + 16 * (int64_t)f - 1) / (16 * (int64_t)f))",
                           "16 * (nbytes / (16 * (int64_t)f))"),
    "home replicas unfilled": ("if (round > 0) break;", "break;"),
    "consumers reversed": ("if (cons[j] == g) i = j;", "if (cons[j] == g) i = f - 1 - j;"),
}


def _build(tmp_path, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, old
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(lib), str(src)], check=True,
                   capture_output=True)
    L = ctypes.CDLL(str(lib))
    vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.ue_oracle_sync_relay.argtypes = [vp, i64, i64, ci, ci, ci, vp, ci, ci, ci, vp]
    L.ue_oracle_sync_relay.restype = ci
    return L


def _relay(L, W, nb, E, N, R, se, G, rd):
    eg = np.zeros(G, np.int64)
    se = np.ascontiguousarray(se, np.int32)
    assert L.ue_oracle_sync_relay(W.ctypes.data, W.shape[1], nb, E, N, R, se.ctypes.data, G, rd, -1,
                                  eg.ctypes.data) == 0
    return eg


def _passes_pins(L):
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    rng = np.random.default_rng(0)
    for c in cases:
        se = np.array(c["slot_expert"], np.int32)
        W = rng.integers(0, 256, size=(se.size, c["nbytes"]), dtype=np.uint8)
        full = W.copy()
        oracle.sync(full, c["nbytes"], c["E"], c["N"], c["R"], se)
        for rd in c["rounds"]:
            if _relay(L, W, c["nbytes"], c["E"], c["N"], c["R"], se, c["G"], rd["round"]).tolist() != rd["egress"]:
                return False
        if not np.array_equal(W, full):
            return False
    for seed in range(20):
        r = np.random.default_rng(500 + seed)
        N = int(r.choice([4, 8, 16])); H = int(r.integers(1, 3)); R = int(r.integers(1, 3)); E = N * H
        p = (r.permutation(E) + 1.0) ** -1.5
        se = oracle.plan(r.multinomial(5000, p / p.sum()).astype(np.int32), N, R)["slot_expert"]
        G = int(r.choice([g for g in (2, 4, 8) if N % g == 0]))
        W = r.integers(0, 256, size=(se.size, 160), dtype=np.uint8)
        full = W.copy()
        oracle.sync(full, 160, E, N, R, se)
        for k in range(oracle.relay_rounds(G)):
            _relay(L, W, 160, E, N, R, se, G, k)
        if not np.array_equal(W, full):
            return False
    return True


def test_unchanged_copy_passes(tmp_path):
    assert _passes_pins(_build(tmp_path, "if (round > 0) break;", "if (round > 0) break;"))


@pytest.mark.parametrize("name", list(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    assert not _passes_pins(_build(tmp_path, *MUTANTS[name])), name
