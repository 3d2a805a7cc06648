"""The C-ABI library builds, loads without a GPU, exports every symbol that
include/moe_b200.h declares, and its host-only entry points (sizing,
validation) behave.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import oracle.moe_oracle as O
from expert_dispatch_router_b200 import binding as B
from expert_dispatch_router_b200 import build as build_mod
from expert_dispatch_router_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert lib.moe_version().startswith(b"moe_b200")
    # nothing but the C ABI is exported
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert {n for n in exported if n.startswith("moe_")} == set(names)


@pytest.mark.parametrize("shape", list(synth.WORKLOADS.values()), ids=list(synth.WORKLOADS))
def test_capacity_matches_oracle(lib, shape):
    cfg = B.make_cfg(shape)
    want = -1 if shape.cap_mode == synth.CAP_DROPLESS else O.capacity(shape.T, shape.E, shape.k, shape.cf_num,
                                                                       shape.cf_den, shape.min_capacity)
    assert B.moe_capacity(cfg) == want


def test_capacity_variants(lib):
    for cf, want in [((1, 1), 10923), ((1, 2), 5462), ((1, 4), 2731), ((2, 1), 21846)]:
        cfg = B.make_cfg(synth.DS_HIGHK, cf_num=cf[0], cf_den=cf[1])
        assert B.moe_capacity(cfg) == want
    cfg = B.make_cfg(synth.SWITCH_TOP1, T=10, E=8, k=1, cf_num=1, cf_den=1, min_capacity=4)
    assert B.moe_capacity(cfg) == 4


def _rows_brute(shape, counts):
    C = None if shape.cap_mode == synth.CAP_DROPLESS else O.capacity(shape.T, shape.E, shape.k, shape.cf_num,
                                                                      shape.cf_den, shape.min_capacity)
    kept = [c if C is None else min(c, C) for c in counts]
    return int(O.row_layout(kept, shape.T, shape.n_shared)[-1])


def test_rows_max_bounds_every_routing(lib):
    import numpy as np
    rng = np.random.default_rng(0)
    for shape in synth.WORKLOADS.values():
        bound = B.moe_rows_max(B.make_cfg(shape))
        assert bound % 128 == 0
        A = shape.T * shape.k
        # adversarial count vectors: balanced, one hot expert, random
        cands = [[A // shape.E + (1 if e < A % shape.E else 0) for e in range(shape.E)],
                 [A] + [0] * (shape.E - 1)]
        for _ in range(20):
            cands.append(list(rng.multinomial(A, rng.dirichlet(np.ones(shape.E) * 0.3))))
        for counts in cands:
            assert _rows_brute(shape, counts) <= bound


def test_workspace_is_not_dense_mask_sized(lib):
    shape = synth.DS_HIGHK
    ws = B.moe_workspace_size(B.make_cfg(shape))
    C = B.moe_capacity(B.make_cfg(shape))
    dense = O.dense_mask_bytes(shape.T, shape.E, C)
    assert dense == 34360786944
    # the workspace holds the three row buffers plus O(T*k) metadata, far below the mask
    assert ws < dense / 40


def test_validation_errors(lib):
    bad = [dict(k=0), dict(k=13), dict(E=0), dict(E=2000), dict(H=100), dict(F=12), dict(n_shared=2), dict(act=7),
           dict(score=3), dict(renorm=2), dict(cap_mode=5), dict(dtype=9), dict(cf_num=0), dict(cf_den=-1),
           dict(T=-1), dict(min_capacity=-3)]
    for kw in bad:
        cfg = B.make_cfg(synth.DS_HIGHK, **kw)
        with pytest.raises(B.MoeError) as ei:
            B.moe_workspace_size(cfg)
        assert ei.value.code in (B.MOE_EINVAL, B.MOE_EUNSUPPORTED), kw
    with pytest.raises(B.MoeError):
        B.moe_capacity(B.make_cfg(synth.DS_HIGHK, T=1 << 30))      # T*k beyond 2^31
    # null configuration and null outputs are rejected before any CUDA call
    assert lib.moe_capacity(None, None) == B.MOE_EINVAL
    assert lib.moe_route(None, None, None, None, None, None, None, None, None, None) == B.MOE_EINVAL
    cfg = B.make_cfg(synth.SWITCH_TINY_F32)
    assert lib.moe_layer_fwd(ctypes.byref(cfg), None, None, None, None, None, None, None, None, None, 0, None, None) \
        == B.MOE_EINVAL
    w = B.moe_weights()
    assert lib.moe_expert_ffn(ctypes.byref(cfg), None, None, None, ctypes.byref(w), None, None, None) == B.MOE_EINVAL
    for code in range(7):
        assert B.strerror(code)


def test_empty_batch_sizes(lib):
    cfg = B.make_cfg(synth.SWITCH_TOP1, T=0)
    assert B.moe_rows_max(cfg) == 0
    assert B.moe_workspace_size(cfg) > 0


def test_router_variant_validation(lib):
    """Sigmoid scores, the z-loss coefficient and the random-second flag are
    validated on the host before any launch."""
    g = synth.GSHARD_TOP2
    assert B.moe_workspace_size(B.make_cfg(g.replace(score=synth.SCORE_SIGMOID_TOPK, z_coef=1e-3))) > 0
    for kw in (dict(score=3), dict(z_coef=-1e-3), dict(z_coef=float("nan")), dict(z_coef=float("inf"))):
        with pytest.raises(B.MoeError) as ei:
            B.moe_workspace_size(B.make_cfg(g, **kw))
        assert ei.value.code == B.MOE_EINVAL, kw
    with pytest.raises(B.MoeError) as ei:
        B.moe_workspace_size(B.make_cfg(g, flags=64))
    assert ei.value.code == B.MOE_EINVAL
    # the flag needs the draws (k >= 2, T > 0); dummy device pointers are never touched
    cfg = B.make_cfg(g.replace(random_second=1))
    assert cfg.flags & B.MOE_FLAG_RANDOM_SECOND
    d = ctypes.c_void_p(256)
    assert lib.moe_route(ctypes.byref(cfg), d, d, None, None, d, d, None, d, None) == B.MOE_EINVAL
    assert lib.moe_route_from_logits(ctypes.byref(cfg), d, None, d, d, d, None) == B.MOE_EINVAL
    # the z-loss partials add T/BT floats to the workspace, nothing that scales with E
    a = B.moe_workspace_size(B.make_cfg(g))
    b = B.moe_workspace_size(B.make_cfg(g, z_coef=1e-3))
    assert a == b


def test_packed_weight_sizes(lib):
    assert B.moe_packed_weight_bytes(64, 3072, 768) == 64 * 24 * 12 * 16384
    assert B.moe_packed_weight_bytes(1, 1, 8) == 16384
    for args, code in [((0, 8, 8), B.MOE_EINVAL), ((1, 8, 12), B.MOE_EUNSUPPORTED), ((1, -1, 8), B.MOE_EINVAL)]:
        with pytest.raises(B.MoeError) as ei:
            B.moe_packed_weight_bytes(*args)
        assert ei.value.code == code
    # packed weights are a bf16 feature
    with pytest.raises(B.MoeError):
        B.moe_workspace_size(B.make_cfg(synth.SWITCH_TINY_F32, flags=B.MOE_FLAG_PACKED_WEIGHTS))


def test_backward_validation(lib):
    """moe_layer_bwd rejects bad calls on the host, before any CUDA call (dummy
    device pointers are never touched)."""
    d = ctypes.c_void_p(256)
    P = ctypes.c_void_p

    def call(shape, flags, grads=None, ws_bytes=None):
        cfg = B.make_cfg(shape, flags=flags)
        w = B.moe_weights(*([256] * 6))
        g = grads if grads is not None else B.moe_weight_grads(*([256] * 6))
        nbytes = ws_bytes if ws_bytes is not None else B.moe_workspace_size(cfg)
        return lib.moe_layer_bwd(ctypes.byref(cfg), d, d, ctypes.byref(w), d, ctypes.c_float(1.0),
                                 ctypes.c_float(1.0), d, d, ctypes.byref(g), d, ctypes.c_size_t(nbytes), None, None)

    small = synth.SWITCH_TOP1.replace(T=300, H=64, F=128, E=8)
    # the backward runs on bf16 layers only
    assert call(synth.SWITCH_TINY_F32, B.MOE_FLAG_TRAINING) == B.MOE_EUNSUPPORTED
    # it needs the workspace of a forward with MOE_FLAG_TRAINING
    assert call(small, 0) == B.MOE_EINVAL
    # every weight gradient the layer has must be given
    assert call(small, B.MOE_FLAG_TRAINING, grads=B.moe_weight_grads(0, 0, 256, 0, 0, 0)) == B.MOE_EINVAL
    sw = small.replace(act=synth.ACT_SWIGLU)
    assert call(sw, B.MOE_FLAG_TRAINING, grads=B.moe_weight_grads(256, 0, 256, 0, 0, 0)) == B.MOE_EINVAL
    shared = small.replace(n_shared=1)
    assert call(shared, B.MOE_FLAG_TRAINING, grads=B.moe_weight_grads(256, 0, 256, 0, 0, 0)) == B.MOE_EINVAL
    # a workspace sized without the backward's buffers is too small
    assert call(small, B.MOE_FLAG_TRAINING, ws_bytes=B.moe_workspace_size(B.make_cfg(small))) == B.MOE_EWORKSPACE


@pytest.mark.parametrize("shape", [s for s in synth.WORKLOADS.values() if s.dtype == synth.DTYPE_BF16],
                         ids=[n for n, s in synth.WORKLOADS.items() if s.dtype == synth.DTYPE_BF16])
def test_training_workspace(lib, shape):
    """MOE_FLAG_TRAINING adds the backward's buffers to the workspace (dgate,
    dlogits, dyrow, dh, dz, dxrow), each at its documented size, and exposes
    them in the views; without the flag the views are NULL."""
    import torch
    plain = B.make_cfg(shape)
    tr = B.make_cfg(shape, flags=B.MOE_FLAG_TRAINING)
    rows = B.moe_rows_max(tr)
    T, H, F, E, k = shape.T, shape.H, shape.F, shape.E, shape.k
    dzw = 2 * ((F + 63) // 64 * 64) if shape.act == synth.ACT_SWIGLU else F
    need = T * k * 4 + T * E * 4 + rows * (2 * H + F + dzw) * 2
    extra = B.moe_workspace_size(tr) - B.moe_workspace_size(plain)
    assert extra >= need
    fake = torch.empty(16, dtype=torch.uint8)         # views are host arithmetic on the base address only
    v0 = B.moe_workspace_views(plain, fake)
    assert not (v0.dgate or v0.dlogits or v0.dyrow or v0.dh or v0.dz or v0.dxrow)
    v = B.moe_workspace_views(tr, fake)
    base = fake.data_ptr()
    size = B.moe_workspace_size(tr)
    spans = sorted([(v.dgate, T * k * 4), (v.dlogits, T * E * 4), (v.dyrow, rows * H * 2), (v.dh, rows * F * 2),
                    (v.dz, rows * dzw * 2), (v.dxrow, rows * H * 2)])
    for (a, n), (b, _) in zip(spans, spans[1:]):
        assert a + n <= b, "training buffers overlap"
    assert all(base <= a and a + n <= base + size for a, n in spans)
    assert all(a % 256 == base % 256 for a, _ in spans)
