"""Host logic of bench.py that needs no GPU: the per-step kernel counts behind
`gpu_launches` (checked against the kernel sequences of the committed ncu
launch lists), workload overrides, and the roofline bound selection."""
import pytest

import bench
from expert_dispatch_router_b200 import synth


def test_forward_launch_counts():
    # Switch top-1: router (pre-split planes; the logits kernel routes too), 3 slot
    # kernels, GEMM1 with the dispatch, GEMM2 with the combine
    assert bench.launches_per_step(synth.SWITCH_TOP1) == 6
    # the router weight split on every call adds one launch
    assert bench.launches_per_step(synth.SWITCH_TOP1, packed_router=False) == 7
    # T*k > 256*E: dispatch kernel, token-tile prefix, two SM-pair contractions,
    # combine kernel
    assert bench.launches_per_step(synth.GSHARD_TOP2) == 1 + 3 + 1 + 1 + 2 + 1
    # fp32 router in one launch; the fp32 layer is never fused
    assert bench.launches_per_step(synth.SWITCH_TINY_F32) == 1 + 3 + 1 + 2 + 1
    # the "probs" drop policy adds the per-expert select
    assert bench.launches_per_step(synth.DS_HIGHK.replace(drop_policy=1)) == 1 + 4 + 1 + 1 + 2 + 1
    # wider than 256 experts: a separate routing kernel after the logits (top-2 on the
    # gather path: the combine runs as its own kernel)
    assert bench.launches_per_step(synth.GSHARD_TOP2.replace(E=300, T=100)) == 2 + 3 + 2 + 1


def test_training_launch_counts():
    # Switch top-1 (the forward with MOE_FLAG_TRAINING: router split + logits/routing,
    # 3 slot kernels, dispatch, zeroing of padding rows, 2 GEMMs, combine; then 11
    # backward launches with dh and dz fused)
    assert bench.train_launches_per_step(synth.SWITCH_TOP1) == 10 + 11
    # GShard top-2: T*k > 256*E (SM-pair forward, + the pair prefix) and H > 512, so
    # dh and dz are two kernels
    assert bench.train_launches_per_step(synth.GSHARD_TOP2) == 11 + 12
    # DeepSpeed k=4: H <= 512 fuses them again
    assert bench.train_launches_per_step(synth.DS_HIGHK) == 11 + 11


def test_workload_overrides():
    class A:
        workload = synth.DS_HIGHK.name
        set = ["drop_policy=1", "cf_den=4"]
    s = bench.workload_shape(A)
    assert s.drop_policy == 1 and s.cf_den == 4 and s.name.endswith("+drop_policy=1+cf_den=4")
    A.set = ["T=5"]
    with pytest.raises(SystemExit):
        bench.workload_shape(A)


def test_roofline_bound_selection():
    peaks = dict(bench.FALLBACK_PEAKS, _source="fallback")
    shape = synth.SWITCH_TOP1
    work = bench.stage_work(shape, kept=4422, experts_used=64)
    r = bench.roofline("ffn_gemm2", work, 0.08, peaks, shape.name)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["frac"] == pytest.approx(work["ffn_gemm2"]["bytes"] / 0.08e-3 / 1e9 / peaks["hbm_gbs"])
    bw = bench.bwd_stage_work(shape, kept=4422, experts_used=64)
    # the router terms of the backward run on the FFMA pipes
    r = bench.roofline("router_wgrad", bw, 0.04, peaks, shape.name)
    assert r["bound"] == "alu" and r["unit"] == "TFLOP/s"
    # a compute-heavy layer is bound by the tensor peak; the sustained one in long steps
    g = synth.GSHARD_TOP2
    wg = bench.stage_work(g, kept=32768, experts_used=32)
    r1 = bench.roofline("ffn_gemm1", wg, 0.3, peaks, g.name)
    r2 = bench.roofline("ffn_gemm1", wg, 0.3, peaks, g.name, sustained=True)
    assert r1["bound"] == "tensor" and r2["peak"] == peaks["bf16_tflops_sustained"] < r1["peak"]


def test_oracle_sample_choice_and_extrapolation():
    import torch
    # the WideEP layer's experts would take ~90 GB in float64: it is timed by sample
    assert bench.oracle_weights_fp64_bytes(synth.WIDEEP_DROPLESS) > bench.ORACLE_FULL_LAYER_BYTES
    assert bench.oracle_weights_fp64_bytes(synth.SWITCH_TOP1) < bench.ORACLE_FULL_LAYER_BYTES
    shape = synth.WIDEEP_DROPLESS.replace(name="tiny", T=96, H=32, F=24, E=8, k=2)
    inp = synth.make_inputs(shape, seed=0)
    host = bench.host_inputs(inp)
    sec, what = bench.oracle_extrapolated_time(shape, host, kept_rows=shape.T * shape.k, n_route=48, n_experts=2,
                                               n_shared_tok=16)
    assert sec > 0 and "extrapolated" in what and "48 of 96" in what
    assert torch.is_tensor(inp["x"])
