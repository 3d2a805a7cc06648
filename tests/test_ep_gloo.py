"""Expert parallelism on CPU: gloo ranks (world size 2 and 4), each holding the
weights of E / world experts, run the layer over their own tokens through the
two all-to-alls of ep_layer_forward.  The local stages are written with the
oracle (test infrastructure: the product stages run the CUDA kernels); the
checker is the oracle's single-process layer on each rank's own tokens with
every expert, which the exchange must reproduce: a row sent to the wrong rank
meets the wrong expert's weights."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.moe_oracle as O
from expert_dispatch_router_b200 import ep, synth


class OracleOps(ep.LocalOps):
    """ep.LocalOps on the oracle, holding only this rank's experts' weights."""

    def __init__(self, shape, w_local, shared, expert_base):
        self.shape, self.w, self.shared, self.base = shape, w_local, shared, expert_base

    def route_dispatch(self, x, wg, logit_add):
        s = self.shape.replace(T=x.shape[0])
        layer = O.OracleLayer.from_mapping(s.as_dict())
        x64 = x.numpy()
        lg = O.router_logits(x64, wg.numpy(), None if logit_add is None else logit_add.numpy()).astype(np.float32)
        probs, selected, ids, gates = O.route_and_dispatch(layer, lg)
        slot, count, kept = O.assign_slots(ids, s.E, O.layer_capacity(layer))
        off = O.row_layout(kept, s.T, s.n_shared)
        rt = O.row_tokens(ids, slot, off, s.n_shared)
        xbuf = np.zeros((int(off[-1]), s.H))
        live = rt[: off[s.E]] >= 0
        xbuf[: off[s.E]][live] = x64[rt[: off[s.E]][live]]
        return dict(ids=ids, gates=gates, slot=slot, kept=[int(v) for v in kept], offsets=[int(v) for v in off],
                    xbuf=torch.from_numpy(xbuf), aux=torch.tensor(O.aux_loss(probs, selected, s.E, s.aux_alpha), dtype=torch.float64))

    def expert_ffn(self, rows, kept_local, expert_base):
        assert expert_base == self.base
        out = torch.zeros_like(rows)
        off = ep.block_offsets(kept_local)
        for i, n in enumerate(kept_local):
            if n:
                w1, w2, w3 = (None if m is None else m[i] for m in (self.w["w1"], self.w["w2"], self.w["w3"]))
                out[off[i]:off[i] + n] = torch.from_numpy(
                    O.expert_ffn(rows[off[i]:off[i] + n].numpy(), w1, w2, self.shape.act, w3))
        return out

    def shared_ffn(self, x):
        if not self.shape.n_shared:
            return None
        sw1, sw2, sw3 = self.shared
        return torch.from_numpy(O.expert_ffn(x.numpy(), sw1[0], sw2[0], self.shape.act,
                                             None if sw3 is None else sw3[0]))

    def combine(self, expert_rows, shared_rows, route):
        ids, slot, gates, off = route["ids"], route["slot"], route["gates"], route["offsets"]
        T, k = ids.shape
        y = np.zeros((T, self.shape.H))
        rows = expert_rows.numpy()
        for t in range(T):
            for r in range(k):
                if slot[t, r] >= 0:
                    y[t] += gates[t, r] * rows[off[ids[t, r]] + slot[t, r]]
        if shared_rows is not None:
            y += shared_rows.numpy()
        return torch.from_numpy(y)


SHAPES = {
    "capacity_top2": synth.GSHARD_TOP2.replace(name="ep_cap", T=0, H=32, F=48, E=8, k=2, cf_num=5, cf_den=4),
    "dropless_swiglu_shared": synth.WIDEEP_DROPLESS.replace(name="ep_wide", T=0, H=24, F=40, E=8, k=3),
}
TOKENS = (37, 60, 45, 29)          # a different token count on every rank


def _worker(rank, world, port, name, errq, plant=False):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        base = SHAPES[name]
        T_all = sum(TOKENS[:world])
        full = synth.make_inputs(base.replace(T=T_all), seed=3)
        d = lambda t: None if t is None else t.to(torch.float64)
        t0 = sum(TOKENS[:rank])
        T = TOKENS[rank]
        x = d(full["x"])[t0:t0 + T].contiguous()
        add = None if full["logit_add"] is None else full["logit_add"][t0:t0 + T].to(torch.float64).contiguous()
        E_l = base.E // world
        holder = (rank + 1) % world if plant else rank       # planted: the neighbour's experts
        own = slice(holder * E_l, (holder + 1) * E_l)
        w_local = {n: None if full[n] is None else d(full[n])[own].numpy() for n in ("w1", "w2", "w3")}
        shared = [None if full[n] is None else d(full[n]).numpy() for n in ("sw1", "sw2", "sw3")]
        ops = OracleOps(base.replace(T=T), w_local, shared, rank * E_l)
        y, aux = ep.ep_layer_forward(x, d(full["wg"]), add, ops, base.E)
        # the checker: this rank's tokens through the single-process oracle, every expert
        layer = O.OracleLayer.from_mapping(base.replace(T=T).as_dict())
        W = [None if full[n] is None else d(full[n]).numpy() for n in ("w1", "w2", "w3", "sw1", "sw2", "sw3")]
        ref = O.layer_forward(layer, x.numpy(), d(full["wg"]).numpy(), *W,
                              logit_add=None if add is None else add.numpy())
        if plant:
            assert not np.allclose(y.numpy(), ref["y"], rtol=1e-6, atol=1e-9), "a misplaced expert went unnoticed"
        else:
            np.testing.assert_allclose(y.numpy(), ref["y"], rtol=1e-10, atol=1e-14)
            assert abs(float(aux) - ref["aux"]) <= 1e-12 * abs(ref["aux"]) + 1e-15
        dist.barrier()
        dist.destroy_process_group()
    except Exception as exc:       # reported to the parent process
        errq.put(f"rank {rank}: {type(exc).__name__}: {exc}")
        raise


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _run(world, name, plant=False):
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, errq, plant)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not alive, "a rank did not finish"
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("name", list(SHAPES))
def test_expert_parallel_matches_single_process_oracle(world, name):
    _run(world, name)


def test_misplaced_experts_are_caught():
    """Planted mistake: every rank holds its neighbour's experts (as if the
    dispatch all-to-all delivered rows to the wrong rank); the checker fails."""
    _run(2, "capacity_top2", plant=True)


def test_block_offsets_and_owner_split():
    assert ep.block_offsets([0, 1, 128, 129]) == [0, 0, 128, 256, 512]
    assert ep.owner_split(256, 8) == 32
    with pytest.raises(ValueError):
        ep.owner_split(10, 4)
