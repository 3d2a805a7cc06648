"""Thin Python binding of libmoe_b200.so (argument marshalling only).

Every function has the name of the C entry point it calls and takes torch
tensors (device tensors for device pointers) or None for a NULL pointer.  All
computation happens in the library's CUDA kernels; nothing here falls back to
another implementation: a missing library raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import synth

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_b200.so")

MOE_OK, MOE_EINVAL, MOE_EUNSUPPORTED, MOE_ECUDA, MOE_ETIMEOUT, MOE_EDEVICE, MOE_EWORKSPACE = range(7)
MOE_FLAG_KEEP_LOGITS, MOE_FLAG_RANDOM_SECOND, MOE_FLAG_UNFUSED, MOE_FLAG_PACKED_WEIGHTS, MOE_FLAG_TRAINING = \
    1, 2, 4, 8, 16
MOE_FLAG_PACKED_ROUTER = 32
MOE_N_STAGE_EVENTS = 8
STAGES = ("router", "slots", "dispatch", "ffn_gemm1", "ffn_gemm2", "combine", "aux")
MOE_N_BWD_STAGE_EVENTS = 10
BWD_STAGES = ("combine_bwd", "dgrad_dh", "wgrad_w2", "dact_dz", "wgrad_w1", "router_bwd", "dgrad_dx", "dispatch_bwd",
              "router_wgrad")


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {code} ({strerror(code)})")


class moe_cfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("F", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("act", ctypes.c_int32),
                ("score", ctypes.c_int32), ("renorm", ctypes.c_int32), ("cap_mode", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("cf_num", ctypes.c_int64), ("cf_den", ctypes.c_int64),
                ("min_capacity", ctypes.c_int64), ("aux_alpha", ctypes.c_float), ("flags", ctypes.c_int32),
                ("z_coef", ctypes.c_float), ("drop_policy", ctypes.c_int32)]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w1", "w3", "w2", "sw1", "sw3", "sw2")]


class moe_weight_grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dw1", "dw3", "dw2", "dsw1", "dsw3", "dsw2")]


class moe_ws_views(ctypes.Structure):
    _fields_ = [("ids", ctypes.c_void_p), ("gates", ctypes.c_void_p), ("slot", ctypes.c_void_p),
                ("expert_count", ctypes.c_void_p), ("kept_count", ctypes.c_void_p),
                ("expert_offset", ctypes.c_void_p), ("row_token", ctypes.c_void_p), ("logits", ctypes.c_void_p),
                ("xbuf", ctypes.c_void_p), ("hbuf", ctypes.c_void_p), ("ybuf", ctypes.c_void_p),
                ("rows_max", ctypes.c_int64), ("dgate", ctypes.c_void_p), ("dlogits", ctypes.c_void_p),
                ("dyrow", ctypes.c_void_p), ("dh", ctypes.c_void_p), ("dz", ctypes.c_void_p),
                ("dxrow", ctypes.c_void_p)]


_lib = None
P, I64P, SZP = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_size_t)
CFGP = ctypes.POINTER(moe_cfg)
_SIGS = {
    "moe_capacity": [CFGP, I64P],
    "moe_rows_max": [CFGP, I64P],
    "moe_workspace_size": [CFGP, SZP],
    "moe_workspace_views": [CFGP, P, ctypes.POINTER(moe_ws_views)],
    "moe_route": [CFGP, P, P, P, P, P, P, P, P, P],
    "moe_route_from_logits": [CFGP, P, P, P, P, P, P],
    "moe_assign_slots": [CFGP, P, P, P, P, P, P, P, P, P],
    "moe_assign_slots_static": [CFGP, P, P, P, P, P, P, P],
    "moe_dispatch": [CFGP, P, P, P, P, P, P],
    "moe_expert_ffn": [CFGP, P, P, P, ctypes.POINTER(moe_weights), P, P, P],
    "moe_combine": [CFGP, P, P, P, P, P, P, P],
    "moe_aux_loss": [CFGP, P, P, P],
    "moe_layer_fwd": [CFGP, P, P, P, P, ctypes.POINTER(moe_weights), P, P, P, P, ctypes.c_size_t, P, P],
    "moe_activation_eval": [ctypes.c_int, P, P, P, ctypes.c_int64, P],
    "moe_layer_bwd": [CFGP, P, P, ctypes.POINTER(moe_weights), P, ctypes.c_float, ctypes.c_float, P, P,
                      ctypes.POINTER(moe_weight_grads), P, ctypes.c_size_t, P, P],
    "moe_sync_status": [P, P],
    "moe_packed_weight_bytes": [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, SZP],
    "moe_pack_weight": [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P],
    "moe_clear_status": [P, P],
    "moe_selftest_bounded_wait": [ctypes.c_int64, ctypes.c_int64, P, P, P],
    "moe_router_planes_bytes": [ctypes.c_int32, ctypes.c_int32, SZP],
    "moe_pack_router_weight": [P, ctypes.c_int32, ctypes.c_int32, P, P],
}


def load():
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m expert_dispatch_router_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        lib.moe_strerror.argtypes = [ctypes.c_int]
        lib.moe_strerror.restype = ctypes.c_char_p
        lib.moe_version.argtypes = []
        lib.moe_version.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def strerror(code: int) -> str:
    return load().moe_strerror(int(code)).decode()


def _check(code: int, where: str):
    if code != MOE_OK:
        raise MoeError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_cfg(shape: synth.LayerShape, flags: int = 0, **override) -> moe_cfg:
    s = shape.replace(**override) if override else shape
    return moe_cfg(T=s.T, H=s.H, F=s.F, E=s.E, k=s.k, n_shared=s.n_shared, act=s.act, score=s.score,
                   renorm=s.renorm, cap_mode=s.cap_mode, dtype=s.dtype, cf_num=s.cf_num, cf_den=s.cf_den,
                   min_capacity=s.min_capacity, aux_alpha=s.aux_alpha,
                   flags=flags | (MOE_FLAG_RANDOM_SECOND if s.random_second else 0), z_coef=s.z_coef,
                   drop_policy=s.drop_policy)


def make_weights(inp: dict) -> moe_weights:
    """Device pointers of the expert matrices; the struct keeps the tensors alive."""
    names = ("w1", "w3", "w2", "sw1", "sw3", "sw2")
    w = moe_weights(*(_ptr(inp.get(n)) for n in names))
    w._keep = [inp.get(n) for n in names]
    return w


# ------------------------------------------------------------------ sizing
def moe_capacity(cfg: moe_cfg) -> int:
    v = ctypes.c_int64()
    _check(load().moe_capacity(ctypes.byref(cfg), ctypes.byref(v)), "moe_capacity")
    return v.value


def moe_rows_max(cfg: moe_cfg) -> int:
    v = ctypes.c_int64()
    _check(load().moe_rows_max(ctypes.byref(cfg), ctypes.byref(v)), "moe_rows_max")
    return v.value


def moe_workspace_size(cfg: moe_cfg) -> int:
    v = ctypes.c_size_t()
    _check(load().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(v)), "moe_workspace_size")
    return v.value


def moe_workspace_views(cfg: moe_cfg, ws: torch.Tensor) -> moe_ws_views:
    v = moe_ws_views()
    _check(load().moe_workspace_views(ctypes.byref(cfg), _ptr(ws), ctypes.byref(v)), "moe_workspace_views")
    return v


# ------------------------------------------------------------------ stages
def moe_route(cfg, x, wg, logit_add, uniform, ids, gates, logits_out, ws, stream=None):
    _check(load().moe_route(ctypes.byref(cfg), _ptr(x), _ptr(wg), _ptr(logit_add), _ptr(uniform), _ptr(ids),
                            _ptr(gates), _ptr(logits_out), _ptr(ws), _stream(stream)), "moe_route")


def moe_route_from_logits(cfg, logits, uniform, ids, gates, ws, stream=None):
    _check(load().moe_route_from_logits(ctypes.byref(cfg), _ptr(logits), _ptr(uniform), _ptr(ids), _ptr(gates),
                                        _ptr(ws), _stream(stream)), "moe_route_from_logits")


def moe_assign_slots(cfg, ids, gates, slot, expert_count, kept_count, expert_offset, row_token, ws, stream=None):
    _check(load().moe_assign_slots(ctypes.byref(cfg), _ptr(ids), _ptr(gates), _ptr(slot), _ptr(expert_count),
                                   _ptr(kept_count), _ptr(expert_offset), _ptr(row_token), _ptr(ws),
                                   _stream(stream)), "moe_assign_slots")


def moe_assign_slots_static(cfg, ids, slot, expert_count, kept_count, expert_offset, row_token, stream=None):
    _check(load().moe_assign_slots_static(ctypes.byref(cfg), _ptr(ids), _ptr(slot), _ptr(expert_count),
                                          _ptr(kept_count), _ptr(expert_offset), _ptr(row_token), _stream(stream)),
           "moe_assign_slots_static")


def moe_dispatch(cfg, x, ids, slot, expert_offset, xbuf, stream=None):
    _check(load().moe_dispatch(ctypes.byref(cfg), _ptr(x), _ptr(ids), _ptr(slot), _ptr(expert_offset), _ptr(xbuf),
                               _stream(stream)), "moe_dispatch")


def moe_expert_ffn(cfg, xbuf, x, expert_offset, weights: moe_weights, ybuf, ws, stream=None):
    _check(load().moe_expert_ffn(ctypes.byref(cfg), _ptr(xbuf), _ptr(x), _ptr(expert_offset), ctypes.byref(weights),
                                 _ptr(ybuf), _ptr(ws), _stream(stream)), "moe_expert_ffn")


def moe_combine(cfg, ybuf, ids, slot, gates, expert_offset, y, stream=None):
    _check(load().moe_combine(ctypes.byref(cfg), _ptr(ybuf), _ptr(ids), _ptr(slot), _ptr(gates),
                              _ptr(expert_offset), _ptr(y), _stream(stream)), "moe_combine")


def moe_aux_loss(cfg, ws, aux, stream=None):
    _check(load().moe_aux_loss(ctypes.byref(cfg), _ptr(ws), _ptr(aux), _stream(stream)), "moe_aux_loss")


def moe_layer_fwd(cfg, x, wg, logit_add, uniform, weights: moe_weights, y, aux, expert_count, ws,
                  stage_events=None, stream=None):
    ev = None
    if stage_events is not None:
        arr = (ctypes.c_void_p * MOE_N_STAGE_EVENTS)(*[e.cuda_event for e in stage_events])
        ev = ctypes.cast(arr, ctypes.c_void_p)
    _check(load().moe_layer_fwd(ctypes.byref(cfg), _ptr(x), _ptr(wg), _ptr(logit_add), _ptr(uniform),
                                ctypes.byref(weights),
                                _ptr(y), _ptr(aux), _ptr(expert_count), _ptr(ws), ws.numel() * ws.element_size(),
                                ev, _stream(stream)), "moe_layer_fwd")


def moe_layer_bwd(cfg, x, wg, weights: moe_weights, dy, d_aux, d_z, dx, dwg, grads: moe_weight_grads, ws,
                  stage_events=None, stream=None):
    ev = None
    if stage_events is not None:
        arr = (ctypes.c_void_p * MOE_N_BWD_STAGE_EVENTS)(*[e.cuda_event for e in stage_events])
        ev = ctypes.cast(arr, ctypes.c_void_p)
    _check(load().moe_layer_bwd(ctypes.byref(cfg), _ptr(x), _ptr(wg), ctypes.byref(weights), _ptr(dy), float(d_aux),
                                float(d_z), _ptr(dx), _ptr(dwg), ctypes.byref(grads), _ptr(ws),
                                ws.numel() * ws.element_size(), ev, _stream(stream)), "moe_layer_bwd")


def make_weight_grads(g: dict) -> moe_weight_grads:
    """Device pointers of the weight-gradient outputs; the struct keeps the tensors alive."""
    names = ("dw1", "dw3", "dw2", "dsw1", "dsw3", "dsw2")
    w = moe_weight_grads(*(_ptr(g.get(n)) for n in names))
    w._keep = [g.get(n) for n in names]
    return w


def moe_activation_eval(act, z, u, out, stream=None):
    _check(load().moe_activation_eval(int(act), _ptr(z), _ptr(u), _ptr(out), z.numel(), _stream(stream)),
           "moe_activation_eval")


def moe_packed_weight_bytes(G: int, N: int, K: int) -> int:
    v = ctypes.c_size_t()
    _check(load().moe_packed_weight_bytes(G, N, K, ctypes.byref(v)), "moe_packed_weight_bytes")
    return v.value


def moe_pack_weight(w, packed, stream=None):
    G, N, K = w.shape
    _check(load().moe_pack_weight(_ptr(w), G, N, K, _ptr(packed), _stream(stream)), "moe_pack_weight")


def pack_weights(inp: dict, stream=None) -> dict:
    """Packed copies (moe_pack_weight) of every expert matrix in `inp`; the
    result replaces w1/w3/w2/sw1/sw3/sw2 for a layer run with
    MOE_FLAG_PACKED_WEIGHTS."""
    out = dict(inp)
    for n in ("w1", "w3", "w2", "sw1", "sw3", "sw2"):
        w = inp.get(n)
        if w is None:
            continue
        G, N, K = w.shape
        buf = torch.empty(moe_packed_weight_bytes(G, N, K) // 2, dtype=torch.bfloat16, device=w.device)
        moe_pack_weight(w, buf, stream)
        out[n] = buf
    return out


def moe_router_planes_bytes(E: int, H: int) -> int:
    v = ctypes.c_size_t()
    _check(load().moe_router_planes_bytes(E, H, ctypes.byref(v)), "moe_router_planes_bytes")
    return v.value


def moe_pack_router_weight(wg, planes, stream=None):
    E, H = wg.shape
    _check(load().moe_pack_router_weight(_ptr(wg), E, H, _ptr(planes), _stream(stream)), "moe_pack_router_weight")


def pack_router(wg, stream=None):
    """The three bf16 planes of the fp32 router weight (moe_pack_router_weight),
    to pass as wg with MOE_FLAG_PACKED_ROUTER."""
    E, H = wg.shape
    buf = torch.empty(moe_router_planes_bytes(E, H) // 2, dtype=torch.bfloat16, device=wg.device)
    moe_pack_router_weight(wg, buf, stream)
    return buf


def moe_selftest_bounded_wait(limit_cycles, abort_after_cycles, waited, ws, stream=None):
    """One kernel whose bounded mbarrier wait nothing satisfies (see the header)."""
    _check(load().moe_selftest_bounded_wait(int(limit_cycles), int(abort_after_cycles), _ptr(waited), _ptr(ws),
                                            _stream(stream)), "moe_selftest_bounded_wait")


def moe_sync_status(ws, stream=None) -> int:
    return load().moe_sync_status(_ptr(ws), _stream(stream))


def moe_clear_status(ws, stream=None):
    _check(load().moe_clear_status(_ptr(ws), _stream(stream)), "moe_clear_status")


# ------------------------------------------------------------------ helpers
def alloc_workspace(cfg: moe_cfg, device="cuda") -> torch.Tensor:
    """A zeroed workspace of moe_workspace_size bytes (allocated by torch)."""
    return torch.zeros(moe_workspace_size(cfg), dtype=torch.uint8, device=device)


def view_tensor(ptr: int, shape, dtype, like: torch.Tensor) -> torch.Tensor:
    """A torch view of `shape` over device memory inside `like`'s storage."""
    base = like.data_ptr()
    nbytes = like.numel() * like.element_size()
    off = int(ptr) - base
    n = 1
    for s in shape:
        n *= int(s)
    esz = torch.empty((), dtype=dtype).element_size()
    if off < 0 or off + n * esz > nbytes or off % esz:
        raise ValueError("view outside the workspace")
    return like.view(torch.uint8)[off:off + n * esz].view(dtype).view(*shape)


def workspace_tensors(cfg: moe_cfg, ws: torch.Tensor) -> dict:
    """Torch views of the intermediates moe_layer_fwd leaves in `ws`."""
    v = moe_workspace_views(cfg, ws)
    T, k, E, R = cfg.T, cfg.k, cfg.E, v.rows_max
    edt = torch.bfloat16 if cfg.dtype == synth.DTYPE_BF16 else torch.float32
    out = dict(ids=view_tensor(v.ids, (T, k), torch.int32, ws),
               gates=view_tensor(v.gates, (T, k), torch.float32, ws),
               slot=view_tensor(v.slot, (T, k), torch.int32, ws),
               expert_count=view_tensor(v.expert_count, (E,), torch.int32, ws),
               kept_count=view_tensor(v.kept_count, (E,), torch.int32, ws),
               expert_offset=view_tensor(v.expert_offset, (E + 2,), torch.int32, ws),
               row_token=view_tensor(v.row_token, (R,), torch.int32, ws),
               xbuf=view_tensor(v.xbuf, (R, cfg.H), edt, ws),
               hbuf=view_tensor(v.hbuf, (R, cfg.F), edt, ws),
               ybuf=view_tensor(v.ybuf, (R, cfg.H), edt, ws), rows_max=R)
    if v.logits:
        out["logits"] = view_tensor(v.logits, (T, E), torch.float32, ws)
    if v.dgate:
        dzw = 2 * ((cfg.F + 63) // 64 * 64) if cfg.act == synth.ACT_SWIGLU else cfg.F
        out.update(dgate=view_tensor(v.dgate, (T, k), torch.float32, ws),
                   dlogits=view_tensor(v.dlogits, (T, E), torch.float32, ws),
                   dyrow=view_tensor(v.dyrow, (R, cfg.H), edt, ws), dh=view_tensor(v.dh, (R, cfg.F), edt, ws),
                   dz=view_tensor(v.dz, (R, dzw), edt, ws), dxrow=view_tensor(v.dxrow, (R, cfg.H), edt, ws))
    return out
