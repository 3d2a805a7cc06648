"""The tensor-core router: the three-plane split of the fp32 router weight
(moe_pack_router_weight) is exact, precomputed planes give bitwise the same
layer, and both router paths (routing fused into the logits kernel for
E <= 256, a separate routing kernel for wider E) match the oracle."""
import numpy as np
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


@pytest.mark.parametrize("E,H", [(64, 768), (256, 136), (7, 8), (300, 72)])
def test_router_planes_sum_exactly_to_the_weight(E, H):
    g = torch.Generator(device="cuda")
    g.manual_seed(E + H)
    wg = torch.randn((E, H), generator=g, device="cuda") * 0.05
    wg[0, :4] = torch.tensor([0.0, -0.0, 1e-30, 3.0e38], device="cuda")     # zero, subnormal-range, huge
    planes = B.pack_router(wg)
    Hp = -(-H // 64) * 64
    assert planes.numel() * 2 == B.moe_router_planes_bytes(E, H) == E * 3 * Hp * 2
    pl = planes.view(E, 3, Hp).double().cpu()
    want = wg.double().cpu()
    got = pl[:, 0, :H] + pl[:, 1, :H] + pl[:, 2, :H]
    # hi + mid + lo recovers every fp32 value exactly (the sum of three bf16 is
    # exact in fp64); hi is the bf16 rounding of w
    assert torch.equal(got, want)
    assert torch.equal(pl[:, 0, :H], wg.to(torch.bfloat16).double().cpu())
    assert (pl[:, :, H:] == 0).all()


CASES = {
    "switch_small": synth.SWITCH_TOP1.replace(name="switch_small", T=1000, H=200, F=392, E=16),
    "wideep_small": synth.WIDEEP_DROPLESS.replace(name="wideep_small", T=300, H=264, F=136, E=16, k=4),
    "e256_ragged": synth.GSHARD_TOP2.replace(name="e256_ragged", T=333, H=136, F=72, E=256, k=8, renorm=0),
    "wide_e300": synth.GSHARD_TOP2.replace(name="wide_e300", T=400, H=72, F=136, E=300, k=2),
    "sigmoid_zloss": synth.SWITCH_TOP1.replace(name="sigmoid_zloss", T=517, H=96, F=136, E=32, k=2,
                                               score=synth.SCORE_SIGMOID_TOPK, z_coef=1e-3, bias_row0=0.0),
    # H >= 2048: the router runs on pairs of SMs (256 tokens per pair tile; T
    # not a multiple of 256 leaves the last pair's odd CTA without tokens)
    "pair_e256_k8_skew": synth.WIDEEP_DROPLESS.replace(name="pair_e256_k8_skew", T=777, H=2048, F=72, E=256, k=8,
                                                       n_shared=0),
    "pair_e200_sigmoid_zloss": synth.SWITCH_TOP1.replace(name="pair_e200_sigmoid_zloss", T=300, H=2112, F=72,
                                                         E=200, k=2, score=synth.SCORE_SIGMOID_TOPK, z_coef=1e-3,
                                                         bias_row0=0.0),
    "pair_e16_k12": synth.GSHARD_TOP2.replace(name="pair_e16_k12", T=513, H=2048, F=72, E=16, k=12),
    # fewer than 256 tokens: the one-SM router (128-token tiles, routing from TMEM)
    "onesm_e64_k2": synth.GSHARD_TOP2.replace(name="onesm_e64_k2", T=200, H=200, F=72, E=64, k=2),
    "onesm_e256_k8_skew": synth.WIDEEP_DROPLESS.replace(name="onesm_e256_k8_skew", T=255, H=136, F=72, E=256,
                                                        k=8, n_shared=0),
    "onesm_e12_k4_zloss": synth.DS_HIGHK.replace(name="onesm_e12_k4_zloss", T=129, H=64, F=72, z_coef=1e-3),
}


@pytest.mark.parametrize("name", list(CASES))
def test_router_paths_match_oracle(name):
    shape = CASES[name]
    inp = synth.make_inputs(shape, seed=5, device="cuda")
    check_layer(shape, inp, run_layer(shape, inp))


@pytest.mark.parametrize("name", list(CASES))
def test_packed_router_is_bitwise_the_same(name):
    shape = CASES[name]
    inp = synth.make_inputs(shape, seed=6, device="cuda")
    a = run_layer(shape, inp)
    snap = {n: a[n].clone() for n in ("logits", "ids", "gates", "slot", "y", "aux")}
    b = run_layer(shape, inp, packed_router=True)
    for n, v in snap.items():
        assert torch.equal(v.contiguous().view(torch.uint8), b[n].contiguous().view(torch.uint8)), n


def test_packed_router_rejects_fp32_layers_and_bad_args():
    shape = synth.SWITCH_TINY_F32
    with pytest.raises(B.MoeError) as ei:
        B.moe_workspace_size(B.make_cfg(shape, flags=B.MOE_FLAG_PACKED_ROUTER))
    assert ei.value.code == B.MOE_EINVAL
    wg = torch.zeros((4, 12), device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.pack_router(wg)                                  # H % 8 != 0
    assert ei.value.code == B.MOE_EUNSUPPORTED


@pytest.mark.parametrize("shape", [
    synth.GSHARD_TOP2.replace(name="ties_k2", T=300, H=72, F=72, E=32, k=2),
    synth.GSHARD_TOP2.replace(name="ties_k12_renorm", T=300, H=72, F=72, E=64, k=12),
    synth.GSHARD_TOP2.replace(name="ties_k3_softmax", T=257, H=136, F=72, E=200, k=3, renorm=0),
    synth.GSHARD_TOP2.replace(name="ties_onesm_k4", T=250, H=72, F=72, E=48, k=4),
], ids=lambda s: s.name)
def test_fused_router_exact_ties_and_wide_k(shape):
    """The fused router ranks each token's experts by (larger logit, then smaller
    index), the oracle's order: every third token has x = 0, so all its logits
    are exactly 0 and it must take experts 0 .. k-1 with equal gates.  k = 12
    runs the 16-wide selection; E = 200 leaves ragged column ranges."""
    inp = synth.make_inputs(shape, seed=4, device="cuda")
    inp["x"][::3] = 0
    out = run_layer(shape, inp)
    check_layer(shape, inp, out)
    k = shape.k
    ids = out["ids"][::3].cpu()
    assert (ids == torch.arange(k, dtype=ids.dtype)).all()
    gates = out["gates"][::3].cpu()
    want = 1.0 / k if shape.renorm else 1.0 / shape.E
    assert torch.allclose(gates, torch.full_like(gates, want), rtol=1e-6, atol=0)
