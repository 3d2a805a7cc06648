"""Failure detection without a GPU fault: a bounded in-kernel wait that nothing
satisfies gives up, reports MOE_ETIMEOUT through the workspace status word and
returns, and the context stays usable (the next layer call is correct)."""
import time

import pytest
import torch

from expert_dispatch_router_b200 import binding as B
from expert_dispatch_router_b200 import build as build_mod
from expert_dispatch_router_b200 import synth
from tests.parity_utils import check_layer, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build_mod.build()
    B.load()


def _run(limit, abort_after):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    waited = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    t0 = time.perf_counter()
    B.moe_selftest_bounded_wait(limit, abort_after, waited, ws)
    st = B.moe_sync_status(ws)
    return st, int(waited.item()), time.perf_counter() - t0


def test_wait_runs_out_and_reports_timeout():
    limit = 2_000_000                      # about a millisecond of SM clock
    st, waited, wall = _run(limit, -1)
    assert st == B.MOE_ETIMEOUT
    assert limit <= waited < 4 * limit     # it waited the limit, then gave up
    assert wall < 5.0
    # the status word was cleared by the read, and the context still works
    shape = synth.WIDEEP_DROPLESS.replace(name="after_timeout", T=300, H=264, F=136, E=16, k=4)
    inp = synth.make_inputs(shape, seed=1, device="cuda")
    check_layer(shape, inp, run_layer(shape, inp))


def test_abort_flag_ends_the_wait_early():
    limit, abort_after = 200_000_000, 1_000_000
    st, waited, _ = _run(limit, abort_after)
    assert st == B.MOE_ETIMEOUT
    assert abort_after <= waited < limit // 10


def test_selftest_rejects_bad_arguments():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.moe_selftest_bounded_wait(-1, -1, waited, ws)
    assert ei.value.code == B.MOE_EINVAL
    with pytest.raises(B.MoeError) as ei:
        B.moe_selftest_bounded_wait(10 ** 12, -1, waited, ws)
    assert ei.value.code == B.MOE_EINVAL
