"""The C ABI: libue.so builds for sm_100a, loads without a GPU, exports every
entry point declared in include/ue.h, and refuses bad arguments on the host
before any launch (no GPU needed for any of this)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from moe_expert_load_ue_b200 import build, ue

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ue.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return ue.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^\s*(?:const\s+char\s*\*\s*|ue_status\s+|int32_t\s+)(ue_\w+)\s*\(", text, flags=re.M))


def test_exports_match_header(L):
    decl = declared_functions()
    assert decl == set(ue.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", ue.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    missing = decl - exported
    assert not missing, missing
    for name in decl:
        getattr(L, name)


def test_library_is_sm100a_only():
    # nvcc gencode flags: the library carries code for sm_100a and nothing else
    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1


def test_status_strings(L):
    assert L.ue_status_string(0) == b"UE_OK"
    assert L.ue_status_string(1) == b"UE_ERR_INVALID_ARG"
    assert L.ue_status_string(4) == b"UE_ERR_DEVICE"


def test_plan_sizes(L):
    s = ue.plan_sizes(ue.Config(E=256, N=64, R=1))
    assert s == {"slot_expert": 320, "slot_quota": 320, "rep_off": 257, "rep_slot": 320, "rep_cum": 320,
                 "rep_experts": 256, "load": 256, "rank_off": 64 * 256, "rank_load_before": 64,
                 "rank_load_after": 64, "info": 8}


@pytest.mark.parametrize("cfg,msg", [
    (dict(E=10, N=3, R=1), "multiple of N"),
    (dict(E=0, N=1, R=1), "E=0"),
    (dict(E=2048, N=2, R=1), "E=2048"),
    (dict(E=8, N=2, R=-1), "R=-1"),
    (dict(E=1024, N=1024, R=5), "N*R"),
])
def test_plan_sizes_refuses(L, cfg, msg):
    sizes = (ctypes.c_int64 * 11)()
    st = L.ue_plan_sizes(ctypes.byref(ue.UeConfig(cfg["E"], cfg["N"], cfg["R"], 8, 0)), sizes)
    assert st == ue.UE_ERR_INVALID_ARG
    assert msg in L.ue_last_error().decode()


class _HostPlan:
    """Host arrays standing in for plan buffers: refused calls must not touch them."""

    def __init__(self, n=64):
        self.arrays = [np.full(n, 7, np.int32) for _ in ue.PLAN_FIELDS]
        self.c = ue.UePlanBuffers(*[a.ctypes.data for a in self.arrays])

    def untouched(self):
        return all((a == 7).all() for a in self.arrays)


FAKE_CTX = ctypes.c_void_p(0x10)   # never dereferenced: every case below fails validation first


@pytest.mark.parametrize("bad", ["E_not_multiple", "T_not_multiple", "K_zero", "misaligned_ids", "null_counts",
                                 "TK_overflow"])
def test_load_refusals_leave_outputs_untouched(L, bad):
    cfg = dict(E=16, N=4, R=1, K=8, T=64)
    ids = np.zeros(64 * 8 + 4, np.int32)
    counts = np.full(4 * 16, 7, np.int32)
    ids_p, counts_p = ids.ctypes.data, counts.ctypes.data
    if bad == "E_not_multiple":
        cfg["E"] = 18
    elif bad == "T_not_multiple":
        cfg["T"] = 66
    elif bad == "K_zero":
        cfg["K"] = 0
    elif bad == "misaligned_ids":
        ids_p += 4
    elif bad == "null_counts":
        counts_p = None
    elif bad == "TK_overflow":
        cfg["T"] = 1 << 30
    c = ue.UeConfig(cfg["E"], cfg["N"], cfg["R"], cfg["K"], cfg["T"])
    st = L.ue_load(FAKE_CTX, ctypes.byref(c), ids_p, counts_p, None, None)
    assert st == ue.UE_ERR_INVALID_ARG, L.ue_last_error()
    assert (counts == 7).all()


def test_plan_and_reroute_refusals(L):
    hp = _HostPlan()
    counts = np.zeros(64, np.int32)
    c = ue.UeConfig(16, 3, 1, 8, 48)                      # E % N != 0
    assert L.ue_plan(FAKE_CTX, ctypes.byref(c), counts.ctypes.data, ctypes.byref(hp.c), None) == 1
    c = ue.UeConfig(16, 4, 1, 8, 64)
    nullp = ue.UePlanBuffers(*([hp.arrays[0].ctypes.data] * 10 + [None]))
    assert L.ue_plan(FAKE_CTX, ctypes.byref(c), counts.ctypes.data, ctypes.byref(nullp), None) == 1
    assert "plan array 10" in L.ue_last_error().decode()
    phys = np.full(512, 7, np.int32)
    assert L.ue_reroute(FAKE_CTX, ctypes.byref(c), None, ctypes.byref(hp.c), phys.ctypes.data, None) == 1
    assert L.ue_rebalance(FAKE_CTX, ctypes.byref(c), None, counts.ctypes.data, None, ctypes.byref(hp.c),
                          phys.ctypes.data, None) == 1
    assert hp.untouched() and (phys == 7).all()


def test_sync_and_grad_refusals(L):
    hp = _HostPlan()
    c = ue.UeConfig(16, 4, 1, 8, 64)
    w = np.zeros(1024, np.uint8)
    assert L.ue_sync(FAKE_CTX, ctypes.byref(c), w.ctypes.data, 24, ctypes.byref(hp.c), None) == 1   # not % 16
    assert L.ue_sync(FAKE_CTX, ctypes.byref(c), w.ctypes.data + 8, 32, ctypes.byref(hp.c), None) == 1
    m = np.zeros(64, np.float32)
    g = np.zeros(64, np.float32)
    assert L.ue_grad_reduce(FAKE_CTX, ctypes.byref(c), m.ctypes.data, g.ctypes.data, 2, 8,
                            ctypes.byref(hp.c), None) == 1          # bad dtype
    assert L.ue_grad_reduce(FAKE_CTX, ctypes.byref(c), m.ctypes.data, g.ctypes.data, 0, 12,
                            ctypes.byref(hp.c), None) == 1          # P % 8
    assert hp.untouched() and (w == 0).all()


def test_null_context_refused(L):
    c = ue.UeConfig(16, 4, 1, 8, 64)
    ids = np.zeros(64 * 8, np.int32)
    counts = np.full(64, 7, np.int32)
    assert L.ue_load(None, ctypes.byref(c), ids.ctypes.data, counts.ctypes.data, None, None) == 1
    assert "context" in L.ue_last_error().decode()
    assert (counts == 7).all()


def test_dispatch_refusals(L):
    hp = _HostPlan()
    c = ue.UeConfig(16, 4, 1, 8, 64)
    ids = np.zeros(64 * 8 + 4, np.int32)
    ids_p = ids.ctypes.data + (-ids.ctypes.data % 16)
    phys = np.full(512, 7, np.int32)
    slot_off = np.full(21, 7, np.int32)
    src = np.full(512, 7, np.int32)
    gates = np.zeros(512, np.float32)
    counts = np.zeros(64, np.int32)

    def call(d, ids_ptr=ids_p, rebalance=False):
        if rebalance:
            return L.ue_rebalance_dispatch(FAKE_CTX, ctypes.byref(c), ids_ptr, counts.ctypes.data, None,
                                           ctypes.byref(hp.c), phys.ctypes.data, d, None)
        return L.ue_dispatch(FAKE_CTX, ctypes.byref(c), ids_ptr, ctypes.byref(hp.c), phys.ctypes.data, d, None)

    assert call(None) == 1 and "dispatch buffers" in L.ue_last_error().decode()
    d = ue.UeDispatchBuffers(None, None, src.ctypes.data, None)
    assert call(ctypes.byref(d)) == 1 and "slot_off" in L.ue_last_error().decode()
    d = ue.UeDispatchBuffers(gates.ctypes.data, slot_off.ctypes.data, src.ctypes.data, None)
    assert call(ctypes.byref(d)) == 1 and "gates_out" in L.ue_last_error().decode()
    d = ue.UeDispatchBuffers(None, slot_off.ctypes.data, None, None)
    assert call(ctypes.byref(d), rebalance=True) == 1 and "src_index" in L.ue_last_error().decode()
    d = ue.UeDispatchBuffers(None, slot_off.ctypes.data, src.ctypes.data, None)
    assert call(ctypes.byref(d), ids_ptr=ids_p + 4) == 1 and "aligned" in L.ue_last_error().decode()
    assert hp.untouched() and (phys == 7).all() and (slot_off == 7).all() and (src == 7).all()


def test_sync_delta_refusals(L):
    hp = _HostPlan()
    c = ue.UeConfig(16, 4, 1, 8, 64)
    w = np.zeros(1024, np.uint8)
    prev = np.zeros(20, np.int32)
    assert L.ue_sync_delta(FAKE_CTX, ctypes.byref(c), w.ctypes.data, 24, ctypes.byref(hp.c),
                           prev.ctypes.data, None) == 1
    assert L.ue_sync_delta(FAKE_CTX, ctypes.byref(c), None, 32, ctypes.byref(hp.c), None, None) == 1
    assert hp.untouched() and (w == 0).all()


def test_plan_variant_refused(L):
    hp = _HostPlan()
    counts = np.zeros(64, np.int32)
    c = ue.UeConfig(16, 4, 1, 8, 64)
    assert L.ue_plan_ex(FAKE_CTX, ctypes.byref(c), counts.ctypes.data, ctypes.byref(hp.c), 4, None) == 1
    assert "variant" in L.ue_last_error().decode()
    phys = np.full(512, 7, np.int32)
    ids = np.zeros(64 * 8 + 4, np.int32)
    ids_p = ids.ctypes.data + (-ids.ctypes.data % 16)
    assert L.ue_rebalance_ex(FAKE_CTX, ctypes.byref(c), ids_p, counts.ctypes.data, None, ctypes.byref(hp.c),
                             phys.ctypes.data, -1, None) == 1
    assert hp.untouched() and (phys == 7).all()


def test_relay_rounds(L):
    assert [L.ue_relay_rounds(G) for G in (1, 2, 3, 4, 8, 72, 128)] == [1, 1, 2, 2, 2, 2, 2]
    assert L.ue_relay_rounds(0) == -1 and L.ue_relay_rounds(129) == -1


def test_shard_refusals(L):
    hp = _HostPlan()
    c = ue.UeConfig(16, 4, 1, 8, 64)
    ids = np.zeros(64 * 8 + 4, np.int32)
    ids_p = ids.ctypes.data + (-ids.ctypes.data % 16)
    counts = np.full(64, 7, np.int32)
    phys = np.full(512, 7, np.int32)

    def load(G, g, ip=ids_p):
        return L.ue_load_shard(FAKE_CTX, ctypes.byref(c), ctypes.byref(ue.UeShard(G, g)), ip, counts.ctypes.data,
                               None, None)

    for G, g, msg in ((0, 0, "G=0"), (129, 0, "G=129"), (3, 0, "multiple of G"), (2, 2, "g=2"), (2, -1, "g=-1")):
        assert load(G, g) == 1 and msg in L.ue_last_error().decode(), (G, g)
    assert load(2, 1, ids_p + 4) == 1 and "aligned" in L.ue_last_error().decode()
    assert L.ue_load_shard(FAKE_CTX, ctypes.byref(c), None, ids_p, counts.ctypes.data, None, None) == 1
    assert L.ue_reroute_shard(FAKE_CTX, ctypes.byref(c), ctypes.byref(ue.UeShard(2, 0)), ids_p, ctypes.byref(hp.c),
                              None, None) == 1 and "phys_local" in L.ue_last_error().decode()

    w = np.zeros(4096, np.uint8)
    base = w.ctypes.data + (-w.ctypes.data % 16)
    ok = (ctypes.c_void_p * 2)(base, base + 1024)

    def sync(tab, rd, nbytes=64, G=2):
        return L.ue_sync_shard(FAKE_CTX, ctypes.byref(c), ctypes.byref(ue.UeShard(G, 0)), tab, nbytes,
                               ctypes.byref(hp.c), rd, None)

    assert sync(None, 0) == 1 and "slot_bases" in L.ue_last_error().decode()
    assert sync((ctypes.c_void_p * 2)(base, base + 8), 0) == 1 and "slot_bases[1]" in L.ue_last_error().decode()
    assert sync((ctypes.c_void_p * 2)(base, None), 0) == 1
    assert sync(ok, 0, nbytes=40) == 1 and "slot_bytes" in L.ue_last_error().decode()
    assert sync(ok, 1) == 1 and "round=1" in L.ue_last_error().decode()       # G = 2: one round
    assert sync(ok, -2) == 1 and "round=-2" in L.ue_last_error().decode()
    four = (ctypes.c_void_p * 4)(base, base + 1024, base + 2048, base + 3072)
    assert sync(four, 2, G=4) == 1 and "round=2" in L.ue_last_error().decode()

    m = np.zeros(64, np.float32)

    def grad(mp, tab, dt=0, P=8):
        return L.ue_grad_reduce_shard(FAKE_CTX, ctypes.byref(c), ctypes.byref(ue.UeShard(2, 1)), mp, tab, dt, P,
                                      ctypes.byref(hp.c), None)

    mp = m.ctypes.data + (-m.ctypes.data % 16)
    assert grad(mp, ok, dt=2) == 1 and "grad_dtype" in L.ue_last_error().decode()
    assert grad(mp, ok, P=12) == 1 and "P=12" in L.ue_last_error().decode()
    assert grad(mp + 4, ok) == 1 and "master_local" in L.ue_last_error().decode()
    assert grad(mp, None) == 1 and "grad_bases" in L.ue_last_error().decode()
    assert hp.untouched() and (counts == 7).all() and (phys == 7).all() and (w == 0).all()


def test_header_is_plain_c(tmp_path):
    # the boundary is a C ABI: ue.h compiles as C99 and as C++ without CUDA headers
    src = tmp_path / "use.c"
    src.write_text('#include <string.h>\n'
                   '#include "ue.h"\n'
                   'int probe(ue_ctx *ctx, const ue_config *cfg, const ue_shard *sh, void *const *bases)\n'
                   '{\n'
                   '    ue_plan_buffers plan;\n'
                   '    ue_dispatch_buffers disp;\n'
                   '    memset(&plan, 0, sizeof plan);\n'
                   '    memset(&disp, 0, sizeof disp);\n'
                   '    (void)disp;\n'
                   '    return (int)ue_sync_shard(ctx, cfg, sh, bases, 16, &plan, ue_relay_rounds(sh->G) - 1, 0);\n'
                   '}\n')
    inc = os.path.join(ROOT, "include")
    for cc, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        args = [cc, std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", inc, "-c", str(src),
                "-o", str(tmp_path / f"use_{cc}.o")]
        if cc == "g++":
            args[args.index(str(src))] = "-xc++"
            args.insert(args.index("-xc++") + 1, str(src))
        subprocess.run(args, check=True, capture_output=True, text=True)


def test_set_wait_limit_refuses_without_context(L):
    assert L.ue_ctx_set_wait_limit(None, 2_000_000_000, 0) == ue.UE_ERR_INVALID_ARG
    assert "context" in L.ue_last_error().decode()
