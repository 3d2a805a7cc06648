"""Expert parallelism: one MoE FFN layer with its routed experts spread over
the ranks of a process group.

Method: "Expert-parallel MoE training" explainer, expert-parallel section (each
rank holds E / world experts; a dispatch all-to-all with variable splits sends
every token row to the rank that owns its expert, the experts run locally, and
a combine all-to-all returns the rows, which are then weighted by their gates
and summed); InferenceX "WideEP" note (EP = 8: 256 routed experts, 32 per GPU,
plus a shared expert).  Capacity is per rank, from the rank's own tokens, as in
the explainer's capacity section (the drop decision is taken before the
all-to-all).

Per forward, on every rank (T_local tokens, experts rank * E_l .. + E_l):
  1. route its tokens, assign slots over all E experts and dispatch them into
     the 128-row-padded per-expert row layout (the single-GPU stages);
  2. exchange the kept counts of the experts each rank owns (one all_to_all of
     E_l ints per pair of ranks), then send the padded row blocks of rank d's
     experts to rank d (all_to_all with variable splits);
  3. run its E_l experts over each source rank's block of rows;
  4. send the rows back the same way (the inverse all_to_all) and combine its
     tokens' rows with their gates, plus its replica of the shared expert.
The aux loss is each rank's own (f and P over its tokens).  Host-side splits
need the counts on the host: one device-to-host copy of E_l ints per source.

The arithmetic stays in the local stages (`LocalOps`): `CudaOps` runs this
library's kernels through the C ABI; the collectives are torch.distributed's.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

ROW_PAD = 128


def round_up(n: int, m: int = ROW_PAD) -> int:
    return -(-int(n) // m) * m


def owner_split(E: int, world: int) -> int:
    """Experts per rank (the experts must divide evenly over the ranks)."""
    if E % world:
        raise ValueError(f"{E} experts do not divide over {world} ranks")
    return E // world


def block_offsets(kept) -> list:
    """Offsets of 128-row-padded blocks holding `kept` rows each (len + 1 entries)."""
    off = [0]
    for v in kept:
        off.append(off[-1] + round_up(int(v)))
    return off


class LocalOps:
    """The single-device stages the expert-parallel layer calls.

    route_dispatch(x, wg, logit_add) -> dict with
        ids, gates, slot [T, k]; kept [E] (host ints); offsets [E + 2] (host
        ints, 128-padded blocks, the shared block at offsets[E]); xbuf [>= offsets[E], H]
        (the dispatched rows in that layout); aux (scalar tensor).
    expert_ffn(rows, kept_local, expert_base) -> rows' outputs: `rows` holds
        len(kept_local) padded blocks (block i: kept_local[i] token rows of
        expert expert_base + i, then padding); returns the same layout.
    shared_ffn(x) -> [T, H] the shared expert's rows, or None without one.
    combine(expert_rows, shared_rows, route) -> y [T, H]: expert_rows in the
        local layout of `route` (offsets), gate-weighted sum in choice order,
        plus the shared row.
    """

    def route_dispatch(self, x, wg, logit_add):
        raise NotImplementedError

    def expert_ffn(self, rows, kept_local, expert_base):
        raise NotImplementedError

    def shared_ffn(self, x):
        raise NotImplementedError

    def combine(self, expert_rows, shared_rows, route):
        raise NotImplementedError


def _all_to_all_rows(out: torch.Tensor, inp: torch.Tensor, out_splits, in_splits, group, world: int):
    """all_to_all of row blocks (variable row counts per peer)."""
    if world == 1:
        out.copy_(inp)
        return
    dist.all_to_all_single(out, inp, output_split_sizes=list(out_splits), input_split_sizes=list(in_splits),
                           group=group)


def ep_layer_forward(x: torch.Tensor, wg: torch.Tensor, logit_add: Optional[torch.Tensor], ops: LocalOps, E: int,
                     group=None):
    """One expert-parallel forward on this rank's tokens.  Returns (y, aux)."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    E_l = owner_split(E, world)
    H = x.shape[1]
    r = ops.route_dispatch(x, wg, logit_add)
    off, kept = r["offsets"], r["kept"]
    # 1. what each destination receives: the padded blocks of its experts
    send_rows = [off[(d + 1) * E_l] - off[d * E_l] for d in range(world)]
    kept_t = torch.tensor([int(v) for v in kept[:E]], dtype=torch.int64, device=x.device)
    recv_kept = torch.empty(world * E_l, dtype=torch.int64, device=x.device)
    if world == 1:
        recv_kept.copy_(kept_t)
    else:
        dist.all_to_all_single(recv_kept, kept_t, group=group)
    recv_kept = recv_kept.view(world, E_l).tolist()
    recv_rows = [block_offsets(rk)[-1] for rk in recv_kept]
    # 2. dispatch all-to-all: rows of rank d's experts go to rank d
    send = r["xbuf"][: off[E]]
    recv = torch.empty((sum(recv_rows), H), dtype=x.dtype, device=x.device)
    _all_to_all_rows(recv, send, recv_rows, send_rows, group, world)
    # 3. this rank's experts over every source's block
    out = torch.empty_like(recv)
    base = 0
    for s in range(world):
        n = recv_rows[s]
        if n:
            out[base:base + n] = ops.expert_ffn(recv[base:base + n], recv_kept[s], rank * E_l)
        base += n
    # 4. combine all-to-all: the rows return to their source, in their layout
    back = torch.empty((off[E], H), dtype=x.dtype, device=x.device)
    _all_to_all_rows(back, out, send_rows, recv_rows, group, world)
    y = ops.combine(back, ops.shared_ffn(x), r)
    return y, r["aux"]


class CudaOps(LocalOps):
    """The local stages on this library's CUDA kernels (C ABI).

    shape: the layer (synth.LayerShape-like: T is this rank's token count, E
    all experts); weights: this rank's experts only ({"w1", "w2", "w3"} with
    E / world experts each) plus the shared expert's ("sw1", "sw2", "sw3").
    """

    def __init__(self, shape, weights: dict):
        from expert_dispatch_router_b200 import binding as B
        self.B = B
        self.shape = shape
        self.w = weights
        B.load()

    def route_dispatch(self, x, wg, logit_add):
        B, s = self.B, self.shape
        cfg = B.make_cfg(s.replace(T=x.shape[0]))
        ws = B.alloc_workspace(cfg, device=x.device)
        T, k, E, H = x.shape[0], s.k, s.E, s.H
        R = B.moe_rows_max(cfg)
        ids = torch.empty((T, k), dtype=torch.int32, device=x.device)
        gates = torch.empty((T, k), dtype=torch.float32, device=x.device)
        slot = torch.empty_like(ids)
        cnt = torch.empty(E, dtype=torch.int32, device=x.device)
        kept = torch.empty(E, dtype=torch.int32, device=x.device)
        off = torch.empty(E + 2, dtype=torch.int32, device=x.device)
        rt = torch.empty(max(R, 1), dtype=torch.int32, device=x.device)
        xbuf = torch.empty((max(R, 1), H), dtype=x.dtype, device=x.device)
        aux = torch.full((2,), float("nan"), dtype=torch.float32, device=x.device)
        B.moe_route(cfg, x, wg, logit_add, None, ids, gates, None, ws)
        B.moe_assign_slots(cfg, ids, gates, slot, cnt, kept, off, rt, ws)
        B.moe_dispatch(cfg, x, ids, slot, off, xbuf)
        B.moe_aux_loss(cfg, ws, aux)
        st = B.moe_sync_status(ws)
        if st != B.MOE_OK:
            raise RuntimeError(f"device status {B.strerror(st)}")
        return dict(ids=ids, gates=gates, slot=slot, kept=kept.tolist(), offsets=off.tolist(), off_dev=off,
                    xbuf=xbuf, aux=aux[0], cfg=cfg)

    def _group_cfg(self, rows: int, groups: int):
        # a layer view whose row bound covers `rows` rows in `groups` padded blocks
        return self.B.make_cfg(self.shape.replace(T=max(rows, 1), k=1, E=groups, n_shared=0,
                                                  cap_mode=1, zipf_skew=0.0))

    def expert_ffn(self, rows, kept_local, expert_base):
        B = self.B
        G = len(kept_local)
        cfg = self._group_cfg(rows.shape[0], G)
        R = B.moe_rows_max(cfg)
        H = rows.shape[1]
        src = torch.zeros((R, H), dtype=rows.dtype, device=rows.device)
        src[: rows.shape[0]] = rows
        off = block_offsets(kept_local)
        off_t = torch.tensor(off + [off[-1]], dtype=torch.int32, device=rows.device)
        ybuf = torch.empty((R, H), dtype=rows.dtype, device=rows.device)
        ws = B.alloc_workspace(cfg, device=rows.device)
        w = {n: self.w[n] for n in ("w1", "w2", "w3")}
        B.moe_expert_ffn(cfg, src, None, off_t, B.make_weights(dict(w, sw1=None, sw2=None, sw3=None)), ybuf, ws)
        st = B.moe_sync_status(ws)
        if st != B.MOE_OK:
            raise RuntimeError(f"device status {B.strerror(st)}")
        return ybuf[: rows.shape[0]]

    def shared_ffn(self, x):
        if not self.shape.n_shared:
            return None
        B = self.B
        T, H = x.shape
        # the shared expert as a layer of one group over every token
        cfg = self._group_cfg(T, 1)
        R = B.moe_rows_max(cfg)
        src = torch.zeros((R, H), dtype=x.dtype, device=x.device)
        src[:T] = x
        off_t = torch.tensor([0, round_up(T), round_up(T)], dtype=torch.int32, device=x.device)
        ybuf = torch.empty((R, H), dtype=x.dtype, device=x.device)
        ws = B.alloc_workspace(cfg, device=x.device)
        w = dict(w1=self.w["sw1"], w2=self.w["sw2"], w3=self.w.get("sw3"), sw1=None, sw2=None, sw3=None)
        B.moe_expert_ffn(cfg, src, None, off_t, B.make_weights(w), ybuf, ws)
        st = B.moe_sync_status(ws)
        if st != B.MOE_OK:
            raise RuntimeError(f"device status {B.strerror(st)}")
        return ybuf[:T]

    def combine(self, expert_rows, shared_rows, route):
        B, cfg = self.B, route["cfg"]
        T, H = route["ids"].shape[0], self.shape.H
        R = B.moe_rows_max(cfg)
        off = route["offsets"]
        ybuf = torch.zeros((max(R, 1), H), dtype=expert_rows.dtype, device=expert_rows.device)
        ybuf[: off[self.shape.E]] = expert_rows
        if shared_rows is not None:
            ybuf[off[self.shape.E]: off[self.shape.E] + T] = shared_rows
        y = torch.empty((T, H), dtype=expert_rows.dtype, device=expert_rows.device)
        B.moe_combine(cfg, ybuf, route["ids"], route["slot"], route["gates"], route["off_dev"], y)
        torch.cuda.synchronize()
        return y
