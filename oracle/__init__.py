"""CPU oracle for the balancer's hot path (TEST INFRASTRUCTURE ONLY).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and it shares no code
with them.  The arithmetic lives in ``ue_oracle.c`` (plain single-threaded C);
this module only marshals numpy arrays into it.

Pinning status (what fixes each function other than itself; the tests under
``tests/test_oracle_*.py`` check every item):
  load          numpy.bincount of the ids; brute-force per-rank counting;
                sum = T*K; balls-in-bins expectation of the busiest rank at s=0.
  expert_load   brute-force counting of occurrences before each rank's tokens.
  plan          hand-worked examples (tests/golden/plan_cases.json); invariants
                (conservation, <= R replicas per rank, redundant quotas >= 1,
                loads <= Q unless slots ran out); optimality max load = Q when
                slots do not run out (Q is a lower bound for any plan); the
                brute-force optimum over all replica placements with an
                integer max-flow on tiny inputs.
  reroute       numpy stable argsort + searchsorted; per-slot counts equal
                quotas; every phys slot holds the token's expert.
  dispatch      hand-worked layouts (tests/golden/dispatch_cases.json); numpy
                stable argsort of the slots; segment lengths equal the plan's
                slot quotas; every segment holds only its slot, in increasing
                flat index; gates carried bit for bit.
  sync          byte-map conservation: every byte of every filled redundant
                slot comes from the right home byte exactly once, other slots
                untouched.
  sync_delta    byte map over a microbatch sequence: after a sync under the
                previous plan, the incremental sync leaves exactly the state a
                full sync gives; slots whose expert is unchanged are untouched;
                the copied-slot count equals a numpy count.
  sync_restore  replay of a stack of layers sharing the redundant slots
                (forward syncs, backward restores in reverse) on tagged bytes:
                after each restore every redundant slot the layer's plan fills
                holds its expert's home bytes and nothing else changed; the
                copy count equals a numpy count; restoring the plan the slots
                hold copies nothing; an unknown holder is a full sync.
  sync_relay    after the relay rounds (or the one direct round) the state
                equals the single-GPU sync on tagged bytes, so a pull from a
                GPU that had not yet received its part shows; the home sends
                each byte once (its egress per expert is the slot size, not f
                times it); relay and direct receive the same bytes per GPU;
                hand-worked schedules (tests/golden/relay_cases.json).
  grad_reduce   exact closed-form sums on dyadic values; zero gradients
                leave the master unchanged; numpy float32 reference order.

None of these pins comes from the UltraEP pages themselves, which print no
worked example, table or value for any step: parity against the pages is
"unpinned by the pages" for all five steps and the dispatch layout; the pins
above are the mathematics and hand-worked cases of the stated rule.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ue_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libue_oracle.so")
_lock = threading.Lock()
_lib = None

P_I32 = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile ue_oracle.c into oracle/libue_oracle.so with gcc (no fast-math, no FMA)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _open(path: str) -> ctypes.CDLL:
    """Load a compiled oracle library and declare its signatures."""
    lib = ctypes.CDLL(path)
    vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.ue_oracle_load.argtypes = [vp, i64, ci, ci, ci, vp, vp]
    lib.ue_oracle_expert_load.argtypes = [vp, ci, ci, vp, vp]
    lib.ue_oracle_plan.argtypes = [ci, ci, ci, vp] + [vp] * 9
    lib.ue_oracle_plan_ex.argtypes = [ci, ci, ci, vp, ci] + [vp] * 9
    lib.ue_oracle_reroute.argtypes = [vp, i64, ci, ci, vp, vp, vp, vp, vp]
    lib.ue_oracle_dispatch.argtypes = [vp, i64, ci, vp, vp, vp, vp]
    lib.ue_oracle_sync.argtypes = [vp, i64, i64, ci, ci, ci, vp]
    lib.ue_oracle_sync_delta.argtypes = [vp, i64, i64, ci, ci, ci, vp, vp, vp]
    lib.ue_oracle_sync_restore.argtypes = [vp, i64, i64, ci, ci, ci, vp, vp, vp]
    lib.ue_oracle_grad_reduce.argtypes = [vp, i64, vp, ci, i64, i64, ci, ci, ci, vp, vp]
    lib.ue_oracle_relay_rounds.argtypes = [ci]
    lib.ue_oracle_sync_relay.argtypes = [vp, i64, i64, ci, ci, ci, vp, ci, ci, ci, vp]
    for f in ("ue_oracle_load", "ue_oracle_expert_load", "ue_oracle_plan", "ue_oracle_plan_ex",
              "ue_oracle_reroute", "ue_oracle_dispatch", "ue_oracle_sync",
              "ue_oracle_sync_delta", "ue_oracle_sync_restore", "ue_oracle_grad_reduce", "ue_oracle_relay_rounds",
              "ue_oracle_sync_relay"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


def _get():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _open(build())
    return _lib


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise OracleError(f"{what} failed with code {rc}")


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def load(ids: np.ndarray, E: int, N: int):
    """Step 1: per-source-rank histogram counts[N][E] and per-rank bad-id counts."""
    ids = _c(ids, np.int32)
    T, K = ids.shape
    counts = np.empty((N, E), np.int32)
    bad = np.empty(N, np.int32)
    _check(_get().ue_oracle_load(_p(ids), T, K, E, N, _p(counts), _p(bad)), "load")
    return counts, bad


def expert_load(counts: np.ndarray):
    """load[e] = column sums of counts; rank_off[r][e] = exclusive column prefix."""
    counts = _c(counts, np.int32)
    N, E = counts.shape
    ld = np.empty(E, np.int32)
    off = np.empty((N, E), np.int32)
    _check(_get().ue_oracle_expert_load(_p(counts), N, E, _p(ld), _p(off)), "expert_load")
    return ld, off


PLAN_FIELDS = ("slot_expert", "slot_quota", "rep_off", "rep_slot", "rep_cum", "rep_experts",
               "rank_load_before", "rank_load_after", "info")


REQUEUE, SPREAD = 1, 2     # plan variants (bit flags), see ue_oracle.c


def plan(load_e: np.ndarray, N: int, R: int, variant: int = 0) -> dict:
    """Step 2: the quota-driven plan (see ue_oracle.c for the exact rule and
    the variants: REQUEUE re-queues partly placed experts, SPREAD spreads the
    remainder of stuck experts over their replicas)."""
    load_e = _c(load_e, np.int32)
    E = load_e.shape[0]
    if E % N:
        raise OracleError("E must be a multiple of N")
    H = E // N
    S = N * (H + R)
    out = {
        "slot_expert": np.empty(S, np.int32), "slot_quota": np.empty(S, np.int32),
        "rep_off": np.empty(E + 1, np.int32), "rep_slot": np.empty(E + N * R, np.int32),
        "rep_cum": np.empty(E + N * R, np.int32), "rep_experts": np.empty(E, np.int32),
        "rank_load_before": np.empty(N, np.int32), "rank_load_after": np.empty(N, np.int32),
        "info": np.empty(8, np.int32),
    }
    rc = _get().ue_oracle_plan_ex(E, N, R, _p(load_e), int(variant), *[_p(out[f]) for f in PLAN_FIELDS])
    _check(rc, "plan")
    return out


def reroute(ids: np.ndarray, E: int, pl: dict) -> np.ndarray:
    """Step 3: physical slot of every (t, k)."""
    ids = _c(ids, np.int32)
    T, K = ids.shape
    phys = np.empty_like(ids)
    rc = _get().ue_oracle_reroute(_p(ids), T, K, E, _p(_c(pl["rep_off"], np.int32)),
                                  _p(_c(pl["rep_slot"], np.int32)), _p(_c(pl["rep_cum"], np.int32)),
                                  _p(_c(pl["slot_quota"], np.int32)), _p(phys))
    _check(rc, "reroute")
    return phys


def dispatch(phys: np.ndarray, S: int, gates: np.ndarray | None = None):
    """Dispatch layout of the physical routing: (slot_off [S+1], src_index, gates_out).

    src_index (and gates_out, None without gates) hold the slot_off[S] valid
    assignments grouped by slot, in increasing flat index within a slot."""
    phys = _c(phys, np.int32).ravel()
    L = phys.shape[0]
    slot_off = np.empty(S + 1, np.int32)
    src = np.empty(L, np.int32)
    g = None if gates is None else _c(gates, np.float32).ravel()
    if g is not None and g.shape[0] != L:
        raise OracleError("gates must have one value per assignment")
    gout = None if g is None else np.empty(L, np.float32)
    _check(_get().ue_oracle_dispatch(_p(phys), L, S, _p(g), _p(slot_off), _p(src), _p(gout)), "dispatch")
    n = int(slot_off[S])
    return slot_off, src[:n], (None if gout is None else gout[:n])


def sync(W: np.ndarray, nbytes: int, E: int, N: int, R: int, slot_expert: np.ndarray) -> None:
    """Step 4, in place on W viewed as bytes [S][slot_stride]."""
    if not (W.flags.c_contiguous and W.ndim == 2):
        raise OracleError("W must be a C-contiguous [S][stride] array")
    stride = W.shape[1] * W.itemsize
    rc = _get().ue_oracle_sync(_p(W), stride, nbytes, E, N, R, _p(_c(slot_expert, np.int32)))
    _check(rc, "sync")


def sync_delta(W: np.ndarray, nbytes: int, E: int, N: int, R: int, slot_expert: np.ndarray,
               prev_slot_expert: np.ndarray | None) -> int:
    """Step 4, incremental: copies only filled redundant slots whose expert
    differs from the previous plan's (all of them when prev is None); returns
    the number of slots copied."""
    if not (W.flags.c_contiguous and W.ndim == 2):
        raise OracleError("W must be a C-contiguous [S][stride] array")
    stride = W.shape[1] * W.itemsize
    n = ctypes.c_int64(0)
    prev = None if prev_slot_expert is None else _c(prev_slot_expert, np.int32)
    rc = _get().ue_oracle_sync_delta(_p(W), stride, nbytes, E, N, R, _p(_c(slot_expert, np.int32)), _p(prev),
                                     ctypes.byref(n))
    _check(rc, "sync_delta")
    return int(n.value)


def sync_restore(W: np.ndarray, nbytes: int, E: int, N: int, R: int, target_slot_expert: np.ndarray,
                 held_slot_expert: np.ndarray | None) -> int:
    """Weight restore in backward, in place on W viewed as bytes [S][slot_stride]:
    every redundant slot the target plan fills with expert e and that does not
    hold e already (held_slot_expert[s] != e; all of them when held is None)
    receives e's home slot.  Returns the number of slots copied."""
    if not (W.flags.c_contiguous and W.ndim == 2):
        raise OracleError("W must be a C-contiguous [S][stride] array")
    stride = W.shape[1] * W.itemsize
    n = ctypes.c_int64(0)
    held = None if held_slot_expert is None else _c(held_slot_expert, np.int32)
    rc = _get().ue_oracle_sync_restore(_p(W), stride, nbytes, E, N, R, _p(_c(target_slot_expert, np.int32)),
                                       _p(held), ctypes.byref(n))
    _check(rc, "sync_restore")
    return int(n.value)


def relay_rounds(G: int) -> int:
    """Relay rounds after which every holder of an expert has it: 1 when G <= 2, else 2."""
    return int(_get().ue_oracle_relay_rounds(G))


def sync_relay(W: np.ndarray, nbytes: int, E: int, N: int, R: int, slot_expert: np.ndarray,
               G: int, round: int, dst_gpu: int = -1) -> np.ndarray:
    """Step 4 over G GPUs: relay round 0 (scatter of the parts from the home
    slot) or 1 (all-gather of the parts among the consumer GPUs), or the direct
    form (round = -1), in place on W viewed as bytes [S][slot_stride], writing
    only destinations on GPU dst_gpu (all when -1).  Returns the bytes each GPU
    sent to other GPUs in this round."""
    if not (W.flags.c_contiguous and W.ndim == 2):
        raise OracleError("W must be a C-contiguous [S][stride] array")
    stride = W.shape[1] * W.itemsize
    egress = np.zeros(max(G, 1), np.int64)
    rc = _get().ue_oracle_sync_relay(_p(W), stride, nbytes, E, N, R, _p(_c(slot_expert, np.int32)), G, round,
                                     dst_gpu, _p(egress))
    _check(rc, "sync_relay")
    return egress


def grad_reduce(master: np.ndarray, grads: np.ndarray, n: int, E: int, N: int, R: int,
                pl: dict) -> None:
    """Step 5, in place on master (float32 [E][mstride]); grads float32 or bf16 bits (uint16)."""
    if master.dtype != np.float32 or not master.flags.c_contiguous:
        raise OracleError("master must be C-contiguous float32")
    if not grads.flags.c_contiguous:
        raise OracleError("grads must be C-contiguous")
    is_bf16 = 1 if grads.dtype == np.uint16 else 0
    if not is_bf16 and grads.dtype != np.float32:
        raise OracleError("grads must be float32 or bf16 bits (uint16)")
    rc = _get().ue_oracle_grad_reduce(_p(master), master.shape[1], _p(grads), is_bf16,
                                      grads.shape[1], n, E, N, R,
                                      _p(_c(pl["rep_off"], np.int32)), _p(_c(pl["rep_slot"], np.int32)))
    _check(rc, "grad_reduce")


def rebalance(ids: np.ndarray, E: int, N: int, R: int, variant: int = 0):
    """Steps 1-3 chained: counts, expert loads, rank offsets, plan, phys."""
    counts, bad = load(ids, E, N)
    ld, off = expert_load(counts)
    pl = plan(ld, N, R, variant)
    phys = reroute(ids, E, pl)
    return {"counts": counts, "bad": bad, "load": ld, "rank_off": off, "plan": pl, "phys": phys}
