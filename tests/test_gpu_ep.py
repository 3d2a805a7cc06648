"""The expert-parallel layer's CUDA local stages (ep.CudaOps) on one GPU: with
one rank every expert is local and the two all-to-alls are copies, so the
result must match the single-GPU layer run unfused within the bf16 rule."""
import numpy as np
import pytest
import torch

from expert_dispatch_router_b200 import binding as B
from expert_dispatch_router_b200 import build as build_mod
from expert_dispatch_router_b200 import ep, synth
from tests.parity_utils import assert_bf16_close, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build_mod.build()
    B.load()


@pytest.mark.parametrize("shape", [
    synth.GSHARD_TOP2.replace(name="ep1_cap", T=500, H=136, F=200, E=8, k=2),
    synth.WIDEEP_DROPLESS.replace(name="ep1_wide", T=300, H=264, F=136, E=16, k=4),
], ids=["capacity_top2", "dropless_swiglu_shared"])
def test_single_rank_matches_layer(shape):
    inp = synth.make_inputs(shape, seed=2, device="cuda")
    ref = run_layer(shape, inp, unfused=True)
    w = {n: inp[n] for n in ("w1", "w2", "w3", "sw1", "sw2", "sw3")}
    y, aux = ep.ep_layer_forward(inp["x"], inp["wg"], inp["logit_add"], ep.CudaOps(shape, w), shape.E)
    assert_bf16_close(y.double().cpu().numpy(), ref["y"].double().cpu().numpy(), shape.name, literal=False)
    assert abs(float(aux) - float(ref["aux"][0])) <= 1e-5 * abs(float(ref["aux"][0]))
