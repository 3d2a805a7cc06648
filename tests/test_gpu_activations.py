"""The expert-FFN epilogue's activation functions against fp64 references,
within the error bounds of the methods they use (GPU, through the C ABI)."""
import numpy as np
import pytest
import torch
from scipy.special import erf

from expert_dispatch_router_b200 import binding as B
from expert_dispatch_router_b200 import build as build_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build_mod.build()
    B.load()


def _grid():
    rng = np.random.default_rng(0)
    z = np.concatenate([np.linspace(-12, 12, 200001), rng.standard_normal(100000) * 3,
                        np.array([0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0])]).astype(np.float32)
    return z


def _eval(act, z, u=None):
    zt = torch.from_numpy(z).cuda()
    ut = None if u is None else torch.from_numpy(u).cuda()
    out = torch.empty_like(zt)
    B.moe_activation_eval(act, zt, ut, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def test_gelu_within_as7126_bound():
    z = _grid()
    got = _eval(1, z)
    z64 = z.astype(np.float64)
    ref = 0.5 * z64 * (1.0 + erf(z64 / np.sqrt(2.0)))
    # erf error: 1.5e-7 from the method (Abramowitz & Stegun 7.1.26) plus about
    # 2.5e-7 from evaluating 1 - poly*exp(-x^2) in fp32 (a few ulp of values <= 1);
    # GELU scales it by 0.5|z|, plus a few fp32 roundings of the result
    bound = 0.5 * np.abs(z64) * 4e-7 + 4 * 2.0 ** -24 * np.abs(ref) + 1e-38
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{int(bad.sum())} points, worst z={z[np.argmax(np.abs(got - ref) - bound)]}"


def test_silu_and_relu():
    z = _grid()
    u = np.random.default_rng(1).standard_normal(z.shape).astype(np.float32)
    got = _eval(2, z, u)
    z64, u64 = z.astype(np.float64), u.astype(np.float64)
    ref = z64 / (1.0 + np.exp(-z64)) * u64
    assert (np.abs(got - ref) <= 1e-5 * np.abs(ref) + 1e-38).all()
    got = _eval(0, z)
    assert (got == np.maximum(z64, 0.0)).all()
