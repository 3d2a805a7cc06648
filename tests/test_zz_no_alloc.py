"""moe_assign_slots_static: slot assignment for callers that cannot allocate
device memory (they hold only their inputs and outputs), through the C ABI.
Its outputs must equal moe_assign_slots' bit for bit, on two calls in a row,
since both calls share the library's fixed scratch array.  Kept in a file of
its own that pytest collects last."""
import numpy as np
import pytest
import torch

from expert_dispatch_router_b200 import binding as B
from expert_dispatch_router_b200 import build as build_mod
from expert_dispatch_router_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build_mod.build()
    B.load()


def _outputs(cfg, R):
    T, k, E = cfg.T, cfg.k, cfg.E
    return dict(slot=torch.full((T, k), -9, dtype=torch.int32, device="cuda"),
                count=torch.full((E,), -9, dtype=torch.int32, device="cuda"),
                kept=torch.full((E,), -9, dtype=torch.int32, device="cuda"),
                off=torch.full((E + 2,), -9, dtype=torch.int32, device="cuda"),
                rt=torch.full((max(R, 1),), -9, dtype=torch.int32, device="cuda"))


def _ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    w = rng.dirichlet(np.ones(E) * 0.4)
    return torch.from_numpy(np.stack([rng.choice(E, k, replace=False, p=w) for _ in range(T)])
                            .astype(np.int32)).cuda()


CASES = [
    synth.SWITCH_TOP1,                                                    # capacity, k=1, one expert overflows
    synth.DS_HIGHK,                                                       # capacity, k=4
    synth.WIDEEP_DROPLESS,                                                # dropless + shared block, k=8
    synth.GSHARD_TOP2.replace(T=777, E=9),                                # ragged
]


@pytest.mark.parametrize("shape", CASES, ids=[c.name for c in CASES])
def test_static_scratch_matches_workspace_version(shape):
    cfg = B.make_cfg(shape)
    R = B.moe_rows_max(cfg)
    ws = B.alloc_workspace(cfg)
    for call, seed in enumerate((11, 12)):                 # two calls in a row, different routings
        ids = _ids(shape.T, shape.E, shape.k, seed)
        ref, got = _outputs(cfg, R), _outputs(cfg, R)
        B.moe_assign_slots(cfg, ids, None, ref["slot"], ref["count"], ref["kept"], ref["off"], ref["rt"], ws)
        B.moe_assign_slots_static(cfg, ids, got["slot"], got["count"], got["kept"], got["off"], got["rt"])
        torch.cuda.synchronize()
        assert B.moe_sync_status(ws) == B.MOE_OK
        used = int(ref["off"][-1])
        for n in ("slot", "count", "kept", "off"):
            assert torch.equal(got[n], ref[n]), (call, n)
        assert torch.equal(got["rt"][:used], ref["rt"][:used]), call


def test_static_scratch_rejects_oversize():
    shape = synth.WIDEEP_DROPLESS.replace(E=1024, T=200000, k=8)     # E * ceil(T*k/256) > scratch
    cfg = B.make_cfg(shape)
    with pytest.raises(B.MoeError) as ei:
        B.moe_assign_slots_static(cfg, None, None, None, None, None, None)
    assert ei.value.code == B.MOE_EINVAL or ei.value.code == B.MOE_EUNSUPPORTED
    dummy = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.moe_assign_slots_static(cfg, dummy, dummy, dummy, dummy, dummy, dummy)
    assert ei.value.code == B.MOE_EUNSUPPORTED
