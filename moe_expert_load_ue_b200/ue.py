"""Thin Python binding of libue.so (argument marshalling only).

Every function here forwards torch CUDA tensors (device pointers), sizes and
the current CUDA stream to the C ABI declared in include/ue.h; every step of
the balancer runs in the library's sm_100a kernels.  There is no CPU path:
if libue.so is missing or the device is not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libue.so")

UE_OK, UE_ERR_INVALID_ARG, UE_ERR_CUDA, UE_ERR_UNSUPPORTED, UE_ERR_DEVICE = range(5)
UE_PLAN_REQUEUE, UE_PLAN_SPREAD = 1, 2      # plan variant bits (include/ue.h)
UE_WAIT_STALL_ONCE = 1                      # ue_ctx_set_wait_limit flag (include/ue.h)

PLAN_FIELDS = ("slot_expert", "slot_quota", "rep_off", "rep_slot", "rep_cum", "rep_experts",
               "load", "rank_off", "rank_load_before", "rank_load_after", "info")

# Entry points declared in include/ue.h (checked against the header by the tests).
EXPORTS = ("ue_plan_sizes", "ue_ctx_create", "ue_ctx_destroy", "ue_ctx_device_error", "ue_ctx_set_wait_limit",
           "ue_load",
           "ue_plan", "ue_plan_ex", "ue_reroute", "ue_reroute_static", "ue_rebalance", "ue_rebalance_ex", "ue_dispatch", "ue_rebalance_dispatch", "ue_sync", "ue_sync_delta", "ue_sync_restore",
           "ue_grad_reduce", "ue_load_shard", "ue_reroute_shard", "ue_relay_rounds", "ue_sync_shard",
           "ue_grad_reduce_shard", "ue_status_string", "ue_last_error")


class UeConfig(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int32), ("N", ctypes.c_int32), ("R", ctypes.c_int32),
                ("K", ctypes.c_int32), ("T", ctypes.c_int64)]


class UePlanBuffers(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in PLAN_FIELDS]


class UeDispatchBuffers(ctypes.Structure):
    _fields_ = [("gates", ctypes.c_void_p), ("slot_off", ctypes.c_void_p), ("src_index", ctypes.c_void_p),
                ("gates_out", ctypes.c_void_p)]


class UeShard(ctypes.Structure):
    _fields_ = [("G", ctypes.c_int32), ("g", ctypes.c_int32)]


class UeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {_status_name(status)}: {detail}")


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load libue.so (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with "
                                  "`python -m moe_expert_load_ue_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            cfgp, planp = ctypes.POINTER(UeConfig), ctypes.POINTER(UePlanBuffers)
            dispp = ctypes.POINTER(UeDispatchBuffers)
            shardp, vpp = ctypes.POINTER(UeShard), ctypes.POINTER(ctypes.c_void_p)
            sig = {
                "ue_plan_sizes": [cfgp, ctypes.POINTER(ctypes.c_int64)],
                "ue_ctx_create": [ci, ctypes.POINTER(vp)],
                "ue_ctx_destroy": [vp],
                "ue_ctx_device_error": [vp, ctypes.POINTER(ctypes.c_int32), vp],
                "ue_ctx_set_wait_limit": [vp, ctypes.c_int64, ctypes.c_int32],
                "ue_load": [vp, cfgp, vp, vp, vp, vp],
                "ue_plan": [vp, cfgp, vp, planp, vp],
                "ue_plan_ex": [vp, cfgp, vp, planp, ci, vp],
                "ue_reroute": [vp, cfgp, vp, planp, vp, vp],
                "ue_reroute_static": [cfgp, vp, planp, vp, vp],
                "ue_rebalance": [vp, cfgp, vp, vp, vp, planp, vp, vp],
                "ue_rebalance_ex": [vp, cfgp, vp, vp, vp, planp, vp, ci, vp],
                "ue_dispatch": [vp, cfgp, vp, planp, vp, dispp, vp],
                "ue_rebalance_dispatch": [vp, cfgp, vp, vp, vp, planp, vp, dispp, vp],
                "ue_sync": [vp, cfgp, vp, i64, planp, vp],
                "ue_sync_delta": [vp, cfgp, vp, i64, planp, vp, vp],
                "ue_sync_restore": [vp, cfgp, vp, i64, planp, vp, vp],
                "ue_grad_reduce": [vp, cfgp, vp, vp, ci, i64, planp, vp],
                "ue_load_shard": [vp, cfgp, shardp, vp, vp, vp, vp],
                "ue_reroute_shard": [vp, cfgp, shardp, vp, planp, vp, vp],
                "ue_relay_rounds": [ctypes.c_int32],
                "ue_sync_shard": [vp, cfgp, shardp, vpp, i64, planp, ctypes.c_int32, vp],
                "ue_grad_reduce_shard": [vp, cfgp, shardp, vp, vpp, ci, i64, planp, vp],
            }
            for name, args in sig.items():
                fn = getattr(L, name)
                fn.argtypes = args
                fn.restype = ci
            L.ue_status_string.argtypes = [ci]
            L.ue_status_string.restype = ctypes.c_char_p
            L.ue_last_error.argtypes = []
            L.ue_last_error.restype = ctypes.c_char_p
            _lib = L
    return _lib


def _status_name(s: int) -> str:
    try:
        return lib().ue_status_string(s).decode()
    except Exception:  # pragma: no cover
        return str(s)


def _check(status: int, where: str) -> None:
    if status != UE_OK:
        raise UeError(status, where, lib().ue_last_error().decode())


@dataclasses.dataclass(frozen=True)
class Config:
    E: int
    N: int
    R: int
    K: int = 8
    T: int = 0

    @property
    def H(self) -> int:
        return self.E // self.N

    @property
    def S(self) -> int:
        return self.N * (self.H + self.R)

    def c(self) -> UeConfig:
        return UeConfig(self.E, self.N, self.R, self.K, self.T)


def plan_sizes(cfg: Config) -> dict:
    sizes = (ctypes.c_int64 * 11)()
    _check(lib().ue_plan_sizes(ctypes.byref(cfg.c()), sizes), "ue_plan_sizes")
    return dict(zip(PLAN_FIELDS, list(sizes)))


class Plan:
    """Device buffers of one placement plan: the 11 int32 arrays of
    ue_plan_buffers as views of one contiguous buffer (each view 16-byte
    aligned), so that the whole plan moves to or from the host in one copy
    (`buffer`)."""

    def __init__(self, cfg: Config, device="cuda"):
        self.cfg = cfg
        sizes = plan_sizes(cfg)
        offs, o = {}, 0
        for f in PLAN_FIELDS:
            offs[f] = o
            o += (sizes[f] + 3) // 4 * 4
        self.buffer = torch.empty(o, dtype=torch.int32, device=device)
        self.tensors = {f: self.buffer[offs[f]:offs[f] + sizes[f]] for f in PLAN_FIELDS}
        self.tensors["rank_off"] = self.tensors["rank_off"].view(cfg.N, cfg.E)
        self._c = UePlanBuffers(*[self.tensors[f].data_ptr() for f in PLAN_FIELDS])

    def __getitem__(self, k):
        return self.tensors[k]

    def ref(self):
        return ctypes.byref(self._c)

    def to_host(self) -> dict:
        return {k: v.cpu().numpy() for k, v in self.tensors.items()}

    def nbytes(self) -> int:
        """Bytes of the whole plan buffer (the 11 arrays and their alignment padding)."""
        return self.buffer.numel() * 4


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


class Context:
    """ue_ctx for one CUDA device."""

    def __init__(self, device: int | None = None):
        if device is None:
            device = torch.cuda.current_device()
        self.device = device
        h = ctypes.c_void_p()
        _check(lib().ue_ctx_create(device, ctypes.byref(h)), "ue_ctx_create")
        self._h = h

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h:
            _check(lib().ue_ctx_destroy(self._h), "ue_ctx_destroy")
            self._h = ctypes.c_void_p()

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass

    def set_wait_limit(self, limit_ns: int, flags: int = 0) -> None:
        _check(lib().ue_ctx_set_wait_limit(self._h, int(limit_ns), int(flags)), "ue_ctx_set_wait_limit")

    def device_error(self, stream=None) -> int:
        w = ctypes.c_int32(0)
        _check(lib().ue_ctx_device_error(self._h, ctypes.byref(w), _stream(stream)), "ue_ctx_device_error")
        return w.value


# ---- the five steps, under the C ABI's names ---------------------------------

def ue_load(ctx: Context, cfg: Config, ids: torch.Tensor, counts: torch.Tensor,
            bad: torch.Tensor | None = None, stream=None) -> None:
    _check(lib().ue_load(ctx.handle, ctypes.byref(cfg.c()), _ptr(ids), _ptr(counts), _ptr(bad),
                         _stream(stream)), "ue_load")


def ue_plan(ctx: Context, cfg: Config, counts: torch.Tensor, plan: Plan, stream=None) -> None:
    _check(lib().ue_plan(ctx.handle, ctypes.byref(cfg.c()), _ptr(counts), plan.ref(), _stream(stream)),
           "ue_plan")


def ue_plan_ex(ctx: Context, cfg: Config, counts: torch.Tensor, plan: Plan, variant: int, stream=None) -> None:
    _check(lib().ue_plan_ex(ctx.handle, ctypes.byref(cfg.c()), _ptr(counts), plan.ref(), int(variant),
                            _stream(stream)), "ue_plan_ex")


def ue_reroute(ctx: Context, cfg: Config, ids: torch.Tensor, plan: Plan, phys: torch.Tensor,
               stream=None) -> None:
    _check(lib().ue_reroute(ctx.handle, ctypes.byref(cfg.c()), _ptr(ids), plan.ref(), _ptr(phys),
                            _stream(stream)), "ue_reroute")


def ue_reroute_static(cfg: Config, ids: torch.Tensor, plan: Plan, phys: torch.Tensor, stream=None) -> None:
    """ue_reroute without a context (no device allocation by the library), on the current device."""
    _check(lib().ue_reroute_static(ctypes.byref(cfg.c()), _ptr(ids), plan.ref(), _ptr(phys), _stream(stream)),
           "ue_reroute_static")


def ue_rebalance(ctx: Context, cfg: Config, ids: torch.Tensor, counts: torch.Tensor,
                 bad: torch.Tensor | None, plan: Plan, phys: torch.Tensor, stream=None) -> None:
    _check(lib().ue_rebalance(ctx.handle, ctypes.byref(cfg.c()), _ptr(ids), _ptr(counts), _ptr(bad),
                              plan.ref(), _ptr(phys), _stream(stream)), "ue_rebalance")


class Dispatch:
    """Device buffers of one dispatch layout: slot_off [S+1], src_index [T*K]
    and, when gates are carried, gates_out [T*K] (torch tensors)."""

    def __init__(self, cfg: Config, with_gates: bool = True, device="cuda"):
        L = cfg.T * cfg.K
        self.slot_off = torch.empty(cfg.S + 1, dtype=torch.int32, device=device)
        self.src_index = torch.empty(L, dtype=torch.int32, device=device)
        self.gates_out = torch.empty(L, dtype=torch.float32, device=device) if with_gates else None

    def buffers(self, gates: torch.Tensor | None) -> UeDispatchBuffers:
        if gates is not None and self.gates_out is None:
            raise ValueError("this Dispatch was made without a gates_out buffer")
        return UeDispatchBuffers(_ptr(gates), _ptr(self.slot_off), _ptr(self.src_index),
                                 _ptr(self.gates_out) if gates is not None else None)

    def nbytes(self, with_gates: bool = True) -> int:
        n = (self.slot_off.numel() + self.src_index.numel()) * 4
        return n + (self.gates_out.numel() * 4 if with_gates and self.gates_out is not None else 0)


def ue_dispatch(ctx: Context, cfg: Config, ids: torch.Tensor, plan: Plan, phys: torch.Tensor,
                disp: Dispatch, gates: torch.Tensor | None = None, stream=None) -> None:
    b = disp.buffers(gates)
    _check(lib().ue_dispatch(ctx.handle, ctypes.byref(cfg.c()), _ptr(ids), plan.ref(), _ptr(phys),
                             ctypes.byref(b), _stream(stream)), "ue_dispatch")


def ue_rebalance_dispatch(ctx: Context, cfg: Config, ids: torch.Tensor, counts: torch.Tensor,
                          bad: torch.Tensor | None, plan: Plan, phys: torch.Tensor, disp: Dispatch,
                          gates: torch.Tensor | None = None, stream=None) -> None:
    b = disp.buffers(gates)
    _check(lib().ue_rebalance_dispatch(ctx.handle, ctypes.byref(cfg.c()), _ptr(ids), _ptr(counts), _ptr(bad),
                                       plan.ref(), _ptr(phys), ctypes.byref(b), _stream(stream)),
           "ue_rebalance_dispatch")


def ue_rebalance_ex(ctx: Context, cfg: Config, ids: torch.Tensor, counts: torch.Tensor,
                    bad: torch.Tensor | None, plan: Plan, phys: torch.Tensor, variant: int, stream=None) -> None:
    _check(lib().ue_rebalance_ex(ctx.handle, ctypes.byref(cfg.c()), _ptr(ids), _ptr(counts), _ptr(bad),
                                 plan.ref(), _ptr(phys), int(variant), _stream(stream)), "ue_rebalance_ex")


def ue_sync(ctx: Context, cfg: Config, weights: torch.Tensor, slot_bytes: int, plan: Plan,
            stream=None) -> None:
    _check(lib().ue_sync(ctx.handle, ctypes.byref(cfg.c()), _ptr(weights), int(slot_bytes), plan.ref(),
                         _stream(stream)), "ue_sync")


def ue_sync_delta(ctx: Context, cfg: Config, weights: torch.Tensor, slot_bytes: int, plan: Plan,
                  prev_slot_expert: torch.Tensor | None, stream=None) -> None:
    _check(lib().ue_sync_delta(ctx.handle, ctypes.byref(cfg.c()), _ptr(weights), int(slot_bytes), plan.ref(),
                               _ptr(prev_slot_expert), _stream(stream)), "ue_sync_delta")


def ue_sync_restore(ctx: Context, cfg: Config, weights: torch.Tensor, slot_bytes: int, plan: Plan,
                    held_slot_expert: torch.Tensor | None, stream=None) -> None:
    _check(lib().ue_sync_restore(ctx.handle, ctypes.byref(cfg.c()), _ptr(weights), int(slot_bytes), plan.ref(),
                                 _ptr(held_slot_expert), _stream(stream)), "ue_sync_restore")


def ue_grad_reduce(ctx: Context, cfg: Config, master: torch.Tensor, grads: torch.Tensor, P: int,
                   plan: Plan, stream=None) -> None:
    if grads.dtype == torch.bfloat16:
        dt = 1
    elif grads.dtype == torch.float32:
        dt = 0
    else:
        raise TypeError("replica grads must be float32 or bfloat16")
    _check(lib().ue_grad_reduce(ctx.handle, ctypes.byref(cfg.c()), _ptr(master), _ptr(grads), dt, int(P),
                                plan.ref(), _stream(stream)), "ue_grad_reduce")


# ---- across the GPUs of one NVLink domain ------------------------------------

def _grad_dtype(grads_dtype) -> int:
    if grads_dtype == torch.bfloat16:
        return 1
    if grads_dtype == torch.float32:
        return 0
    raise TypeError("replica grads must be float32 or bfloat16")


def _peer_table(bases) -> ctypes.Array:
    """Host array of device pointers from tensors or integer addresses."""
    ptrs = [b if isinstance(b, int) else b.data_ptr() for b in bases]
    return (ctypes.c_void_p * len(ptrs))(*ptrs)


def ue_relay_rounds(G: int) -> int:
    return int(lib().ue_relay_rounds(int(G)))


def ue_load_shard(ctx: Context, cfg: Config, G: int, g: int, ids_local: torch.Tensor, counts: torch.Tensor,
                  bad: torch.Tensor | None = None, stream=None) -> None:
    _check(lib().ue_load_shard(ctx.handle, ctypes.byref(cfg.c()), ctypes.byref(UeShard(G, g)), _ptr(ids_local),
                               _ptr(counts), _ptr(bad), _stream(stream)), "ue_load_shard")


def ue_reroute_shard(ctx: Context, cfg: Config, G: int, g: int, ids_local: torch.Tensor, plan: Plan,
                     phys_local: torch.Tensor, stream=None) -> None:
    _check(lib().ue_reroute_shard(ctx.handle, ctypes.byref(cfg.c()), ctypes.byref(UeShard(G, g)), _ptr(ids_local),
                                  plan.ref(), _ptr(phys_local), _stream(stream)), "ue_reroute_shard")


def ue_sync_shard(ctx: Context, cfg: Config, G: int, g: int, slot_bases, slot_bytes: int, plan: Plan,
                  round: int, stream=None) -> None:
    """slot_bases: G tensors or device addresses, GPU h's slots as mapped on this GPU."""
    t = _peer_table(slot_bases)
    _check(lib().ue_sync_shard(ctx.handle, ctypes.byref(cfg.c()), ctypes.byref(UeShard(G, g)), t, int(slot_bytes),
                               plan.ref(), int(round), _stream(stream)), "ue_sync_shard")


def ue_grad_reduce_shard(ctx: Context, cfg: Config, G: int, g: int, master_local: torch.Tensor, grad_bases,
                         grads_dtype, P: int, plan: Plan, stream=None) -> None:
    """grad_bases: G tensors or device addresses (GPU h's replica-gradient rows);
    grads_dtype: torch.float32 or torch.bfloat16."""
    t = None if grad_bases is None else _peer_table(grad_bases)
    _check(lib().ue_grad_reduce_shard(ctx.handle, ctypes.byref(cfg.c()), ctypes.byref(UeShard(G, g)),
                                      _ptr(master_local), t, _grad_dtype(grads_dtype), int(P), plan.ref(),
                                      _stream(stream)), "ue_grad_reduce_shard")
