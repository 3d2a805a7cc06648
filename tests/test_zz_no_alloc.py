"""moe_assign_slots_static: slot assignment for callers that cannot allocate
device memory (they hold only their inputs and outputs), through the C ABI.
Its outputs must equal moe_assign_slots' bit for bit and the oracle's slots,
counts, offsets and row tokens, on two calls in a row, since both calls share
the library's fixed scratch array.  Kept in a file of its own that pytest
collects last."""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
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


def _ids_np(T, E, k, seed):
    rng = np.random.default_rng(seed)
    w = rng.dirichlet(np.ones(E) * 0.4)
    return np.stack([rng.choice(E, k, replace=False, p=w) for _ in range(T)]).astype(np.int32)


def _both(shape, ids_np):
    """(workspace version, static version, status of the workspace version)."""
    cfg = B.make_cfg(shape)
    R = B.moe_rows_max(cfg)
    ws = B.alloc_workspace(cfg)
    ids = torch.from_numpy(ids_np).cuda()
    ref, got = _outputs(cfg, R), _outputs(cfg, R)
    B.moe_assign_slots(cfg, ids, None, ref["slot"], ref["count"], ref["kept"], ref["off"], ref["rt"], ws)
    B.moe_assign_slots_static(cfg, ids, got["slot"], got["count"], got["kept"], got["off"], got["rt"])
    torch.cuda.synchronize()
    return ref, got, B.moe_sync_status(ws)


def _assert_equal(ref, got, what):
    used = int(ref["off"][-1])
    for n in ("slot", "count", "kept", "off"):
        assert torch.equal(got[n], ref[n]), (what, n)
    assert torch.equal(got["rt"][:used], ref["rt"][:used]), what


def _assert_oracle(shape, ids_np, got):
    C = None if shape.cap_mode == synth.CAP_DROPLESS else O.capacity(shape.T, shape.E, shape.k, shape.cf_num,
                                                                        shape.cf_den)
    rs, rc, rk = O.assign_slots(ids_np, shape.E, C)
    roff = O.row_layout(rk, shape.T, shape.n_shared)
    np.testing.assert_array_equal(got["slot"].cpu().numpy(), rs)
    np.testing.assert_array_equal(got["count"].cpu().numpy(), rc)
    np.testing.assert_array_equal(got["kept"].cpu().numpy(), rk)
    np.testing.assert_array_equal(got["off"].cpu().numpy(), roff)
    np.testing.assert_array_equal(got["rt"].cpu().numpy()[:roff[-1]], O.row_tokens(ids_np, rs, roff, shape.n_shared))


CASES = [
    synth.SWITCH_TOP1,                                                    # capacity, k=1, one expert overflows
    synth.DS_HIGHK,                                                       # capacity, k=4
    synth.WIDEEP_DROPLESS,                                                # dropless + shared block, k=8
    synth.GSHARD_TOP2.replace(T=777, E=9),                                # ragged
]


@pytest.mark.parametrize("shape", CASES, ids=[c.name for c in CASES])
def test_static_scratch_matches_workspace_version(shape):
    for call, seed in enumerate((11, 12)):                 # two calls in a row, different routings
        ids_np = _ids_np(shape.T, shape.E, shape.k, seed)
        ref, got, st = _both(shape, ids_np)
        assert st == B.MOE_OK
        _assert_equal(ref, got, call)
        _assert_oracle(shape, ids_np, got)


def test_static_scratch_bad_and_undispatched_ids():
    """-1 (a choice that is not dispatched) takes no slot; an id outside [0, E)
    gets slot -1 and the workspace version reports MOE_EDEVICE.  Everything else
    matches the workspace version."""
    shape = synth.GSHARD_TOP2.replace(T=500, E=7)
    ids_np = _ids_np(shape.T, shape.E, shape.k, 3)
    ids_np[10, 1] = -1
    ids_np[20, 0] = -1
    ref, got, st = _both(shape, ids_np)
    assert st == B.MOE_OK
    _assert_equal(ref, got, "undispatched")
    _assert_oracle(shape, ids_np, got)
    bad = ids_np.copy()
    bad[30, 0] = shape.E + 3
    bad[40, 1] = -5
    ref, got, st = _both(shape, bad)
    assert st == B.MOE_EDEVICE
    assert int(got["slot"][30, 0]) == -1 and int(got["slot"][40, 1]) == -1
    _assert_equal(ref, got, "bad ids")


def test_static_scratch_limit_is_exact():
    """The scratch holds E * ceil(T*k/256) <= 262080 chunk counts: 260 * 1008 is
    accepted and exact, 137 * 1913 = 262081 is refused before any launch."""
    at = synth.LayerShape("at_limit", T=258000, H=8, F=8, E=260, k=1, cap_mode=synth.CAP_DROPLESS)
    assert at.E * -(-at.T * at.k // 256) == 262080
    rng = np.random.default_rng(1)
    ids_np = rng.integers(0, at.E, size=(at.T, 1)).astype(np.int32)
    ref, got, st = _both(at, ids_np)
    assert st == B.MOE_OK
    _assert_equal(ref, got, "at the limit")
    over = synth.LayerShape("over_limit", T=489500, H=8, F=8, E=137, k=1, cap_mode=synth.CAP_DROPLESS)
    assert over.E * -(-over.T * over.k // 256) == 262081
    cfg = B.make_cfg(over)
    B.moe_rows_max(cfg)                                    # the configuration itself is valid
    dummy = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.moe_assign_slots_static(cfg, dummy, dummy, dummy, dummy, dummy, dummy)
    assert ei.value.code == B.MOE_EUNSUPPORTED
