#!/usr/bin/env python
"""Benchmark of the single-GPU MoE FFN forward pass (router -> slots -> dispatch
-> grouped expert FFN -> combine -> aux loss) through the C ABI, and with
--pass train of one training step (the forward with MOE_FLAG_TRAINING, then
moe_layer_bwd).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                  [--set FIELD=VALUE ...] [--pass forward|train] [--unpacked] [--no-cpu-baseline]

--set overrides one routing option of the workload (score, renorm, z_coef,
random_second, drop_policy, cf_num, cf_den); the workload name then carries the
overrides, e.g. deepspeed_k4_T32768_H512_E12+drop_policy=1.

One step = one moe_layer_fwd call over one batch of T synthetic tokens already
resident in HBM.  L2 is flushed before every step, outside the timed events:
a 320 MiB write, then a 320 MiB read of another buffer, so no dirty lines of
the flush are written back inside the step.  Each rank of a multi-GPU launch (torchrun) runs an
independent replica on its own batch: the layer has no exchange step on one
device, so there is no data-path collective; the host-side barrier and the
max-over-ranks timing reduction are plumbing.

Prints one JSON line (rank 0).  `value` = tokens/s over all ranks, device-timed
with CUDA events; `e2e` = the same metric with the step's inputs copied from
pinned host memory and the result read back inside the timed region (the
training step: x and dy in, the loss terms out).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s on 1 B200; dispatch/combine HBM GB/s; expert GEMM TC util %"
DEFAULT_WORKLOAD = "wideep_dropless_T16384_H7168_E256_k8"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
SETTABLE = {"score": int, "renorm": int, "z_coef": float, "random_second": int, "drop_policy": int,
            "cf_num": int, "cf_den": int}


def router_launches(shape, packed_router: bool) -> int:
    """bf16 x: the weight split (none with pre-split planes), the tensor-core
    logits kernel (which also routes for E <= 256), and for wider E the routing
    kernel; fp32 x: one FFMA router kernel."""
    if shape.dtype != 1:
        return 1
    return (0 if packed_router else 1) + 1 + (0 if shape.E <= 256 else 1)


def launches_per_step(shape, packed_router: bool = True) -> int:
    """Kernels one moe_layer_fwd call launches: the router (router_launches);
    slots 3 (count; scan, with the offsets and aux loss in its last CTA; rank),
    plus the per-expert select of the "probs" policy; dispatch 1 (0 when fused into the first expert contraction: bf16
    with T*k <= 256*E); expert FFN 2, plus the pair-tile prefix when the
    contractions run on SM pairs (bf16 with T*k > 256*E); combine 1 (0 when
    fused into the second: top-1 without a shared expert on the gather path)."""
    router = router_launches(shape, packed_router)
    slots = 3 + (1 if shape.drop_policy == 1 and shape.cap_mode == 0 else 0)
    fused, fused_combine = fused_stages(shape)
    dispatch = 0 if fused else 1
    ffn = 2 + (1 if shape.dtype == 1 and not fused else 0)
    combine = 0 if fused_combine else 1
    return router + slots + dispatch + ffn + combine


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the short runs of the other workloads (and the cf sweep) reported beside the headline")
    ap.add_argument("--unpacked", action="store_true",
                    help="read expert weights in the linear-layer layout instead of packed blocks")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE")
    ap.add_argument("--pass", dest="pass_", default="forward", choices=["forward", "train"],
                    help="train: one step is moe_layer_fwd (MOE_FLAG_TRAINING) followed by moe_layer_bwd")
    return ap.parse_args()


def workload_shape(args):
    """The named workload with the --set overrides applied."""
    from expert_dispatch_router_b200 import synth
    shape = synth.WORKLOADS[args.workload]
    over = {}
    for item in args.set:
        key, _, val = item.partition("=")
        if key not in SETTABLE:
            raise SystemExit(f"--set: unknown field {key!r} (one of {sorted(SETTABLE)})")
        over[key] = SETTABLE[key](val)
    if over:
        tag = "+".join(f"{k}={v}" for k, v in over.items())
        shape = shape.replace(name=f"{shape.name}+{tag}", **over)
    return shape


# ------------------------------------------------------------------ plumbing
def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """Largest per-rank value (timing is reported as the slowest rank's)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base: int, rank: int) -> int:
    """Each replica draws its own batch (and its own weights) from seed base + rank."""
    return base + rank


def job_tokens_per_s(T: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes T tokens per step; the step
    time is the slowest rank's."""
    return world * T / (ms_per_step / 1e3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


class ClockSampler:
    """SM clocks and throttle reasons sampled in the background: through NVML
    every 2 ms (read-only queries), else nvidia-smi every 100 ms."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.samples = []
        self.proc = None
        self._stop = threading.Event()
        try:
            pr = torch.cuda.get_device_properties(device_index)
            sel = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        except Exception:
            sel = str(device_index)
        try:
            import pynvml as N
            N.nvmlInit()
            h = N.nvmlDeviceGetHandleByPciBusId(sel) if ":" in sel else N.nvmlDeviceGetHandleByIndex(device_index)
            mx = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
            bits = (N.nvmlClocksEventReasonHwSlowdown, N.nvmlClocksEventReasonHwThermalSlowdown,
                    N.nvmlClocksEventReasonSwThermalSlowdown, N.nvmlClocksEventReasonSwPowerCap)

            def poll():
                while not self._stop.is_set():
                    try:
                        sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                        r = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                    except Exception:
                        break
                    flags = ",".join("Active" if r & b else "Not Active" for b in bits)
                    self.samples.append((time.time(), f"{sm}, {mx}, 0, {flags}"))
                    time.sleep(0.002)
                try:
                    N.nvmlShutdown()
                except Exception:
                    pass

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def wait_first(self, timeout=5.0):
        t0 = time.time()
        while not self.samples and time.time() - t0 < timeout:
            time.sleep(0.02)

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        elif getattr(self, "thread", None) is not None:
            self.thread.join(timeout=2)

    def summary(self, t0, t1):
        rows = [s for (t, s) in self.samples if t0 <= t <= t1] or [s for (_, s) in self.samples]
        in_region = any(t0 <= t <= t1 for (t, _) in self.samples)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "in_timed_region": in_region}


def traffic_from_profiles(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(p):
        return None
    src = os.path.join(ROOT, "expert_dispatch_router_b200", "csrc", kernel_source(kernel, workload))
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:12]
    for line in open(p):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 4 and cells[0] == workload and cells[1] == kernel and cells[2] == sha:
            try:
                return float(cells[3])
            except ValueError:
                return None
    return None


def kernel_source(stage: str, workload: str = None) -> str:
    """The source file of the kernel a stage runs: the expert contractions of
    bf16 layers with T*k > 256*E run on SM pairs (grouped_gemm_tn.cu); the bf16
    router's logits GEMM (with the routing in its epilogue) runs on SM pairs in
    router_pair.cu for E <= 256 and T >= 256, else in grouped_gemm.cu."""
    from expert_dispatch_router_b200 import synth
    shape = synth.WORKLOADS.get(workload) if workload else None
    bf16 = shape is not None and shape.dtype == 1
    if stage in ("ffn_gemm1", "ffn_gemm2") and bf16 and shape.T * shape.k > 256 * shape.E:
        return "grouped_gemm_tn.cu"
    if stage == "router" and bf16:
        pair = shape.E <= 256 and shape.T >= 256
        return "router_pair.cu" if pair else "grouped_gemm.cu"
    return {"router": "router.cu", "dispatch": "permute.cu", "combine": "permute.cu",
            "ffn_gemm1": "grouped_gemm.cu", "ffn_gemm2": "grouped_gemm.cu",
            "combine_bwd": "backward.cu", "dispatch_bwd": "backward.cu", "router_wgrad": "backward.cu",
            "router_bwd": "router.cu", "dgrad_dh": "grouped_gemm_bwd.cu", "wgrad_w2": "grouped_gemm_bwd.cu",
            "dact_dz": "grouped_gemm_bwd.cu", "wgrad_w1": "grouped_gemm_bwd.cu", "dh_dz": "grouped_gemm_bwd.cu",
            "dgrad_dx": "grouped_gemm_bwd.cu"}.get(stage, "moe_abi.cu")


# kernels whose arithmetic runs on the fp32 FMA pipes, not the tensor cores
SIMT_STAGES = ("dispatch_bwd", "router_wgrad")


# ------------------------------------------------------------------ algorithmic work
def stage_work(shape, kept: int, experts_used: int):
    """Algorithmic bytes and flops of one launch of each kernel (padding rows and
    unused capacity count as waste, not work).  Where the top-1 combine runs
    inside the second contraction, that launch writes y (zero rows for dropped
    tokens) instead of the routed rows."""
    b = 2 if shape.dtype == 1 else 4
    T, H, F, E, k = shape.T, shape.H, shape.F, shape.E, shape.k
    sh = shape.n_shared
    rows = kept + sh * T
    nm1 = 2 if shape.act == 2 else 1
    wexp = experts_used + sh
    add = T * E * 4 if shape.zipf_skew else 0
    _, fused_combine = fused_stages(shape)
    g2_out = T * H * b + T * k * 8 if fused_combine else rows * H * b
    return {
        "router": {"flops": 2.0 * T * H * E, "bytes": T * H * b + E * H * 4 + T * k * 8 + add},
        "dispatch": {"flops": 0.0, "bytes": T * H * b + kept * H * b + T * k * 8},
        "ffn_gemm1": {"flops": 2.0 * rows * H * F * nm1,
                      "bytes": wexp * nm1 * F * H * b + rows * H * b + rows * F * b},
        "ffn_gemm2": {"flops": 2.0 * rows * F * H, "bytes": wexp * H * F * b + rows * F * b + g2_out},
        "combine": {"flops": 0.0, "bytes": kept * H * b + sh * T * H * b + T * H * b + T * k * 12},
    }


def roofline(stage: str, work: dict, ms: float, peaks: dict, workload: str, bf16: bool = True, sustained=False):
    """Bound = whichever of HBM bytes / tensor or ALU flops takes longer at peak.
    The router runs on the tensor cores for bf16 activations (fp32 FFMA otherwise).
    `sustained` selects the power-capped tensor peak for kernels inside long steps."""
    hbm = peaks["hbm_gbs"]
    tc = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) if sustained else peaks["bf16_tflops"]
    alu = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12   # fp32 FFMA TFLOP/s at max clock
    w = work[stage]
    s = ms / 1e3
    t_hbm = w["bytes"] / (hbm * 1e9)
    if (stage == "router" and not bf16) or stage in SIMT_STAGES:
        cpeak, cbound = alu, "alu"
    else:
        cpeak, cbound = tc, "tensor"
    t_cmp = w["flops"] / (cpeak * 1e12) if w["flops"] else 0.0
    if t_cmp > t_hbm:
        ach = w["flops"] / s / 1e12
        out = {"bound": cbound, "achieved": ach, "peak": cpeak, "unit": "TFLOP/s", "frac": ach / cpeak}
        out["peak_source"] = (f"{peaks['_source']} bf16 {'sustained' if sustained else 'burst'}" if cbound == "tensor"
                              else "148 SM x 128 FP32 lanes x 2 x max SM clock (derived)")
    else:
        ach = w["bytes"] / s / 1e9
        out = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
               "peak_source": f"{peaks['_source']} HBM copy"}
    out.update(kernel=stage, algorithmic_bytes=w["bytes"], algorithmic_flops=w["flops"], ms_per_launch=ms,
               traffic=traffic_from_profiles(workload, stage))
    return out


def train_launches_per_step(shape) -> int:
    """Kernels of one training step: the forward with MOE_FLAG_TRAINING (always
    unfused, plus the zeroing of xbuf's padding rows; the router weight is
    split on each call, since the backward takes it in fp32), then moe_layer_bwd:
    combine backward and the zeroing of dyrow's padding rows, five expert
    contractions (four when T*k <= 256*E or H <= 512: dh and dz in one; with
    T*k > 256*E the forward contractions run on SM pairs after a pair-tile
    prefix kernel), the router
    backward (the aux coefficients, then dlogits), the dispatch backward and
    dWg (partial sums, then their reduction)."""
    router = router_launches(shape, packed_router=False)
    slots = 3 + (1 if shape.drop_policy == 1 and shape.cap_mode == 0 else 0)
    pairs = 1 if shape.T * shape.k > 256 * shape.E else 0        # pair-tile prefix of the SM-pair GEMMs
    fwd = router + slots + 1 + 1 + 2 + pairs + 1
    fused = shape.T * shape.k <= 256 * shape.E or shape.H <= 512    # dh and dz in one kernel
    bwd = 2 + (4 if fused else 5) + 2 + 1 + 2
    return fwd + bwd


def bwd_stage_work(shape, kept: int, experts_used: int):
    """Algorithmic bytes and flops of each kernel of moe_layer_bwd.  The dz
    stage recomputes the first contraction (counted: it is the kernel's work);
    weight gradients are written in fp32."""
    b = 2
    T, H, F, E, k = shape.T, shape.H, shape.F, shape.E, shape.k
    sh = shape.n_shared
    rows = kept + sh * T
    nm1 = 2 if shape.act == 2 else 1
    wexp = experts_used + sh
    return {
        "combine_bwd": {"flops": 0.0, "bytes": T * H * b + 2 * kept * H * b + sh * T * H * b + T * k * 16},
        "dgrad_dh": {"flops": 2.0 * rows * H * F, "bytes": wexp * H * F * b + rows * H * b + rows * F * b},
        "wgrad_w2": {"flops": 2.0 * rows * H * F, "bytes": rows * H * b + rows * F * b + wexp * H * F * 4},
        "dact_dz": {"flops": 2.0 * rows * H * F * nm1,
                    "bytes": wexp * nm1 * F * H * b + rows * H * b + rows * F * b + rows * F * nm1 * b},
        "wgrad_w1": {"flops": 2.0 * rows * H * F * nm1, "bytes": rows * F * nm1 * b + rows * H * b + wexp * nm1 * F * H * 4},
        "router_bwd": {"flops": 0.0, "bytes": 2 * T * E * 4 + T * k * 8},
        "dgrad_dx": {"flops": 2.0 * rows * F * nm1 * H, "bytes": wexp * nm1 * F * H * b + rows * F * nm1 * b + rows * H * b},
        # dh and dz in one kernel: both contractions, no dh round trip
        "dh_dz": {"flops": 2.0 * rows * H * F * (1 + nm1),
                  "bytes": wexp * H * F * b + wexp * nm1 * F * H * b + 2 * rows * H * b + rows * F * nm1 * b},
        "dispatch_bwd": {"flops": 2.0 * T * E * H,
                         "bytes": kept * H * b + sh * T * H * b + T * H * b + T * E * 4 + E * H * 4 + T * k * 8},
        "router_wgrad": {"flops": 2.0 * T * E * H, "bytes": T * E * 4 + T * H * b + E * H * 4},
    }


# ------------------------------------------------------------------ CPU oracle timing
def oracle_sample_time(shape, inp_cpu: dict, tokens: int):
    """Run the CPU oracle on the first `tokens` tokens as a layer of its own."""
    import numpy as np
    import oracle.moe_oracle as O
    sub = shape.replace(T=tokens)
    layer = O.OracleLayer.from_mapping(sub.as_dict())
    d = lambda t: None if t is None else t
    x = inp_cpu["x"][:tokens]
    add = None if inp_cpu["logit_add"] is None else inp_cpu["logit_add"][:tokens]
    uni = None if inp_cpu.get("uniform") is None else inp_cpu["uniform"][:tokens]
    t0 = time.perf_counter()
    O.layer_forward(layer, x, inp_cpu["wg"], inp_cpu["w1"], inp_cpu["w2"], d(inp_cpu["w3"]), d(inp_cpu["sw1"]),
                    d(inp_cpu["sw2"]), d(inp_cpu["sw3"]), logit_add=add, uniform=uni)
    return time.perf_counter() - t0


def host_inputs(inp: dict):
    """float64 numpy copies for the oracle; expert weights copied lazily."""
    import torch

    class Lazy:
        def __init__(self, w):
            self.w = w

        def __getitem__(self, e):
            return self.w[e].to("cpu", torch.float64).numpy()

    d = lambda t: None if t is None else t.to("cpu", torch.float64).numpy()
    return {"x": d(inp["x"]), "wg": d(inp["wg"]), "w1": Lazy(inp["w1"]), "w2": Lazy(inp["w2"]),
            "w3": None if inp["w3"] is None else Lazy(inp["w3"]), "sw1": d(inp["sw1"]), "sw2": d(inp["sw2"]),
            "sw3": d(inp["sw3"]), "logit_add": None if inp["logit_add"] is None else inp["logit_add"].cpu().numpy(),
            "uniform": None if inp.get("uniform") is None else inp["uniform"].cpu().numpy()}


def oracle_train_sample_time(shape, inp_cpu: dict, dy, tokens: int):
    """The oracle's forward and backward on the first `tokens` tokens as a layer of its own."""
    import oracle.moe_oracle as O
    import oracle.moe_oracle_bwd as OB
    sub = shape.replace(T=tokens)
    layer = O.OracleLayer.from_mapping(sub.as_dict())
    add = None if inp_cpu["logit_add"] is None else inp_cpu["logit_add"][:tokens]
    uni = None if inp_cpu.get("uniform") is None else inp_cpu["uniform"][:tokens]
    t0 = time.perf_counter()
    OB.layer_backward(layer, inp_cpu["x"][:tokens], inp_cpu["wg"], inp_cpu["w1"], inp_cpu["w2"], inp_cpu["w3"],
                      inp_cpu["sw1"], inp_cpu["sw2"], inp_cpu["sw3"], dy=dy[:tokens], logit_add=add, uniform=uni)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_weights_fp64_bytes(shape) -> int:
    nm = 3 if shape.act == 2 else 2
    return (shape.E + shape.n_shared) * nm * shape.H * shape.F * 8


# Layers whose expert weights would take more than this in float64 on the host
# are timed by the extrapolated sample below instead of the whole layer.
ORACLE_FULL_LAYER_BYTES = 4 << 30


def oracle_extrapolated_time(shape, host: dict, kept_rows: int, n_route: int, n_experts: int, n_shared_tok: int):
    """The oracle's time for one whole layer, from a bounded sample.

    Routing (logits, softmax, top-k, gates, slots, row layout, aux loss) runs on
    the first n_route tokens as a batch of its own and is scaled by T / n_route
    (every step is linear in T).  The expert FFN with the gated sum runs on
    every row that the first n_experts experts (in id order among those chosen)
    receive from that batch, plus the shared expert on n_shared_tok tokens; its
    time per row is scaled to the layer's kept rows (+ T shared rows).  Weights
    are widened to float64 before the clock starts.  Returns (seconds per
    layer, description)."""
    import numpy as np
    import oracle.moe_oracle as O
    T = shape.T
    sub = shape.replace(T=n_route)
    layer = O.OracleLayer.from_mapping(sub.as_dict())
    x = host["x"][:n_route]
    add = None if host["logit_add"] is None else host["logit_add"][:n_route]
    uni = None if host.get("uniform") is None else host["uniform"][:n_route]
    t0 = time.perf_counter()
    logits = O.router_logits(x, host["wg"], add).astype(np.float32)
    probs, selected, ids, gates = O.route_and_dispatch(layer, logits, uni)
    slot, count, kept = O.assign_slots(ids, shape.E, O.layer_capacity(layer))
    off = O.row_layout(kept, n_route, shape.n_shared)
    O.row_tokens(ids, slot, off, shape.n_shared)
    O.aux_loss(probs, selected, shape.E, shape.aux_alpha)
    t_route = time.perf_counter() - t0
    experts = [int(e) for e in np.unique(ids[ids >= 0])][:n_experts]
    w = {e: (host["w1"][e], host["w2"][e], None if host["w3"] is None else host["w3"][e]) for e in experts}
    y = np.zeros((n_route, shape.H))
    rows = 0
    t0 = time.perf_counter()
    for e in experts:
        tt, rr = np.nonzero((ids == e) & (slot >= 0))
        Ye = O.expert_ffn(x[tt], w[e][0], w[e][1], shape.act, w[e][2])
        for j in range(len(tt)):
            y[tt[j]] += gates[tt[j], rr[j]] * Ye[j]
        rows += len(tt)
    if shape.n_shared:
        ts = np.arange(n_shared_tok)
        y[ts] += O.expert_ffn(x[ts], host["sw1"][0], host["sw2"][0], shape.act,
                              None if host["sw3"] is None else host["sw3"][0])
        rows += n_shared_tok
    t_ffn = time.perf_counter() - t0
    total_rows = kept_rows + shape.n_shared * T
    sec = t_route * T / n_route + t_ffn / max(rows, 1) * total_rows
    what = (f"extrapolated: the oracle's routing, slots and aux loss on the first {n_route} of {T} tokens "
            f"({t_route:.1f} s, scaled by T), and its expert FFN with the gated sum on the {rows} rows of "
            f"{len(experts)} routed expert(s) and {n_shared_tok if shape.n_shared else 0} shared-expert tokens "
            f"({t_ffn:.1f} s, scaled per row to {total_rows} kept + shared rows)")
    return sec, what


def cpu_baseline(shape, inp, kept_rows, budget_s=15.0):
    host = host_inputs(inp)
    if oracle_weights_fp64_bytes(shape) > ORACLE_FULL_LAYER_BYTES:
        sec, what = oracle_extrapolated_time(shape, host, kept_rows, n_route=min(shape.T, 2048), n_experts=2,
                                             n_shared_tok=min(shape.T, 256))
        return {"value": shape.T / sec, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                "sample": what}
    n = min(shape.T, 256)
    t = oracle_sample_time(shape, host, n)
    while t < budget_s / 3 and n < shape.T:
        n = min(shape.T, max(n * 2, int(n * budget_s / max(t, 1e-3) * 0.8)))
        t = oracle_sample_time(shape, host, n)
    return {"value": n / t, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"the oracle's whole layer on the first {n} of {shape.T} tokens as a batch of its own "
                      f"({t:.1f} s, capacity recomputed for that batch)"}


# ------------------------------------------------------------------ arms
def run_reference(args, world, rank):
    if rank != 0:
        return
    import torch
    from expert_dispatch_router_b200 import synth
    shape = workload_shape(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = synth.make_inputs(shape, seed=args.seed, device=dev)
    host = host_inputs(inp)
    budget = max(0.05, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    run = lambda m: oracle_sample_time(shape, host, m)
    what = "the oracle's whole layer"
    if args.pass_ == "train":
        gen = torch.Generator(device=dev)
        gen.manual_seed(args.seed + 1000)
        dyh = torch.randn((shape.T, shape.H), generator=gen, device=dev).to(torch.bfloat16).to(
            "cpu", torch.float64).numpy()
        run = lambda m: oracle_train_sample_time(shape, host, dyh, m)
        what = "the oracle's forward and backward"
    if args.pass_ != "train" and oracle_weights_fp64_bytes(shape) > ORACLE_FULL_LAYER_BYTES:
        # one step = one extrapolated estimate of the whole layer (see
        # oracle_extrapolated_time); kept rows from the oracle's own routing of all T
        import numpy as np
        import oracle.moe_oracle as O
        layer = O.OracleLayer.from_mapping(shape.as_dict())
        lg = O.router_logits(host["x"], host["wg"], host["logit_add"]).astype(np.float32)
        _, _, ids_all, _ = O.route_and_dispatch(layer, lg, host.get("uniform"))
        _, _, kept_all = O.assign_slots(ids_all, shape.E, O.layer_capacity(layer))
        kept_rows = int(kept_all.sum())
        n_route = min(shape.T, max(64, int(2048 * min(1.0, budget / 6.0))))
        est = lambda: oracle_extrapolated_time(shape, host, kept_rows, n_route, 1, min(shape.T, 64))
        for _ in range(args.warmup):
            est()
        outs = [est() for _ in range(args.steps)]
        ms = 1e3 * sum(o[0] for o in outs) / len(outs)
        value = shape.T / (ms / 1e3)
        n = shape.T
        sample = outs[-1][1]
    else:
        n = 16
        t = run(n)
        while t < budget * 0.5 and n < shape.T:
            n = min(shape.T, n * 2)
            t = run(n)
        for _ in range(args.warmup):
            run(n)
        times = [run(n) for _ in range(args.steps)]
        ms = 1e3 * sum(times) / len(times)
        value = n / (ms / 1e3)
        sample = f"{what} on the first {n} of {shape.T} tokens per step"
    print(json.dumps({"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1,
                      "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                      "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                      "config": {"workload": shape.name, "tokens_per_step": n,
                                 "pass": "forward+backward" if args.pass_ == "train" else "forward"},
                      "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                       "sample": sample},
                      "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
          flush=True)


class LayerRun:
    """One layer configuration set up on the device: inputs, packed weights,
    workspace and outputs, plus the L2 flush buffers."""

    def __init__(self, B, shape, seed, packed, dev, stream):
        import torch
        from expert_dispatch_router_b200 import synth
        self.B, self.shape, self.stream = B, shape, stream
        self.inp = synth.make_inputs(shape, seed=seed, device="cuda")
        self.packed = packed and shape.dtype == 1
        # expert weights and the router weight's bf16 planes prepared once
        self.cfg = B.make_cfg(shape, flags=(B.MOE_FLAG_PACKED_WEIGHTS | B.MOE_FLAG_PACKED_ROUTER) if self.packed
                              else 0)
        self.ws = B.alloc_workspace(self.cfg)
        self.edt = self.inp["x"].dtype
        self.y = torch.empty((shape.T, shape.H), dtype=self.edt, device=dev)
        self.aux = torch.empty(2, dtype=torch.float32, device=dev)
        # expert weights packed once into 16 KB TMA blocks (weight preprocessing,
        # outside every timed region), as a serving engine stores them
        wsrc = B.pack_weights(self.inp) if self.packed else self.inp
        self.wg = B.pack_router(self.inp["wg"]) if self.packed else self.inp["wg"]
        torch.cuda.synchronize()
        self.wts = B.make_weights(wsrc)
        self._wsrc = wsrc
        # L2 flush between steps (outside the timed events): write one 320 MiB
        # buffer, then read another, so the timed step starts with an L2 that holds
        # no data of the step and no dirty lines whose write-back would land inside it.
        self.flush_w = torch.empty(320 * 2**20 // 4, dtype=torch.float32, device=dev)
        self.flush_r = torch.ones(320 * 2**20 // 4, dtype=torch.float32, device=dev)
        self.flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2(self):
        import torch
        self.flush_w.zero_()
        torch.sum(self.flush_r, dim=0, out=self.flush_sink)

    def call(self, events=None):
        i = self.inp
        self.B.moe_layer_fwd(self.cfg, i["x"], self.wg, i["logit_add"], i["uniform"], self.wts, self.y, self.aux,
                             None, self.ws, stage_events=events, stream=self.stream)

    def check_status(self, when):
        st = self.B.moe_sync_status(self.ws, self.stream)
        if st != self.B.MOE_OK:
            raise RuntimeError(f"device status {when}: {self.B.strerror(st)}")

    def counts(self):
        wt = self.B.workspace_tensors(self.cfg, self.ws)
        return (int(wt["kept_count"].sum().item()), int((wt["kept_count"] > 0).sum().item()),
                int(wt["expert_offset"][-1].item()))

    def time_steps(self, steps):
        """Each step bracketed by two events around the layer call alone (L2
        flushed before each, outside the events).  Returns per-step ms."""
        import torch
        ends = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e in [x for pair in ends for x in pair]:
            e.record(self.stream)            # torch creates the CUDA event at its first record
        torch.cuda.synchronize()
        for i in range(steps):
            self.flush_l2()
            ends[i][0].record(self.stream)
            self.call()
            ends[i][1].record(self.stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ends]

    def time_stages(self, steps):
        """The same steps with the layer's per-stage events (each costs ~1-2 us of
        GPU time, so their sum runs a little above the plain steps)."""
        import torch
        B = self.B
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(B.MOE_N_STAGE_EVENTS)] for _ in range(steps)]
        for e in [x for row in evs for x in row]:
            e.record(self.stream)
        torch.cuda.synchronize()
        for i in range(steps):
            self.flush_l2()
            self.call(evs[i])
        torch.cuda.synchronize()
        stage_ms = {name: sum(e[j].elapsed_time(e[j + 1]) for e in evs) / steps for j, name in enumerate(B.STAGES)}
        total = sum(e[0].elapsed_time(e[-1]) for e in evs) / steps
        return stage_ms, total


def fused_stages(shape):
    """(dispatch fused into GEMM1, combine fused into GEMM2) for this layer: bf16
    layers with T*k <= 256*E gather x inside GEMM1 and, top-1 without a shared
    expert, scatter gate * row inside GEMM2; larger bf16 layers run their
    contractions on SM pairs between the dispatch and combine kernels."""
    fused = shape.dtype == 1 and shape.T * shape.k <= 256 * shape.E
    return fused, fused and shape.k == 1 and shape.n_shared == 0


def stage_report(shape, stage_ms, kept, experts_used, peaks, long_step):
    """Per-stage roofline records of the single-launch kernels, and the expert
    contractions' combined TFLOP/s (fraction of the burst and sustained peaks)."""
    work = stage_work(shape, kept, experts_used)
    fused, fused_combine = fused_stages(shape)
    single = ["router", "ffn_gemm1", "ffn_gemm2"] + ([] if fused else ["dispatch"]) \
        + ([] if fused_combine else ["combine"])
    bf16 = shape.dtype == 1
    per_stage = {s_: roofline(s_, work, stage_ms[s_], peaks, shape.name, bf16, long_step) for s_ in single}
    gemm_flops = work["ffn_gemm1"]["flops"] + work["ffn_gemm2"]["flops"]
    gemm_ms = stage_ms["ffn_gemm1"] + stage_ms["ffn_gemm2"]
    gemm_tf = gemm_flops / (gemm_ms / 1e3) / 1e12
    gemm = {"tflops": gemm_tf, "frac_of_burst": gemm_tf / peaks["bf16_tflops"],
            "frac_of_sustained": gemm_tf / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
            "ms": gemm_ms, "algorithmic_flops": gemm_flops}
    return work, single, per_stage, gemm


def other_workloads(B, args, peaks, dev, stream):
    """Short runs of every other layer workload (and the DeepSpeed k=4 capacity
    sweep, with a cf = 2.0 point where E*C far exceeds the kept rows) on this
    GPU: tokens/s, stage times, dispatch/combine GB/s and the contractions'
    TFLOP/s, each from its own timed loop of about a quarter second."""
    import torch
    from expert_dispatch_router_b200 import synth
    cases = [synth.SWITCH_TINY_F32, synth.SWITCH_TOP1, synth.GSHARD_TOP2]
    for num, den in ((2, 1), (1, 1), (1, 2), (1, 4)):
        cases.append(synth.DS_HIGHK.replace(name=f"{synth.DS_HIGHK.name}_cf{num / den:g}", cf_num=num, cf_den=den))
    out = {}
    for shape in cases:
        run = LayerRun(B, shape, args.seed, not args.unpacked, dev, stream)
        for _ in range(3):
            run.flush_l2()
            run.call()
        run.check_status("after warm-up")
        est = statistics.median(run.time_steps(5))
        steps = int(min(2000, max(20, 250.0 / max(est, 1e-3))))
        per_step = run.time_steps(steps)
        stage_ms, _ = run.time_stages(min(steps, 200))
        run.check_status("after the timed region")
        kept, used, rows = run.counts()
        C = B.moe_capacity(run.cfg)
        ms = sum(per_step) / steps
        _, _, per_stage, gemm = stage_report(shape, stage_ms, kept, used, peaks, False)
        out[shape.name] = {
            "T": shape.T, "H": shape.H, "F": shape.F, "E": shape.E, "k": shape.k,
            "cf": shape.cf_num / shape.cf_den if shape.cap_mode == 0 else None, "capacity": C,
            "E_times_C": shape.E * C if C is not None and C >= 0 else None, "kept_assignments": kept,
            "rows_used": rows, "steps": steps, "ms_per_step": ms, "tokens_per_s": shape.T / (ms / 1e3),
            "stages_ms": stage_ms,
            "dispatch_gbs": per_stage["dispatch"]["achieved"] if "dispatch" in per_stage else None,
            "combine_gbs": per_stage["combine"]["achieved"] if "combine" in per_stage else None,
            "frac": {s_: v["frac"] for s_, v in per_stage.items()},
            "expert_gemm": {k_: gemm[k_] for k_ in ("tflops", "frac_of_burst", "frac_of_sustained")},
            "fused": dict(zip(("dispatch_into_gemm1", "combine_into_gemm2"), fused_stages(shape))),
        }
        del run
        torch.cuda.empty_cache()
    return out


def run_ours(args, world, rank, local):
    import torch
    from expert_dispatch_router_b200 import binding as B

    B.load()                                     # raises if the CUDA library is missing
    shape = workload_shape(args)
    peaks = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    run = LayerRun(B, shape, replica_seed(args.seed, rank), not args.unpacked, dev, stream)
    inp, packed = run.inp, run.packed
    T, H = shape.T, shape.H
    edt = run.edt
    cfg, ws, wts = run.cfg, run.ws, run.wts

    for _ in range(max(args.warmup, 3)):
        run.flush_l2()
        run.call()
    run.check_status("after warm-up")
    kept, experts_used, rows_used = run.counts()

    # Timed region 1 (the headline): each step bracketed by two events, the layer
    # call alone between them.  Timed region 2 (the breakdown): the same steps
    # with the layer's per-stage events.
    n_stage_steps = min(args.steps, 300)
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.wait_first()
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    per_step = run.time_steps(args.steps)
    t1 = time.time()
    barrier(world)
    stage_ms, stage_sum_ms = run.time_stages(n_stage_steps)
    barrier(world)
    clocks = None
    if sampler:
        sampler.stop()
        clocks = sampler.summary(t0, t1)
    run.check_status("after the timed region")

    ms_local = sum(per_step) / args.steps
    ms = max_over_ranks(ms_local, world)
    value = job_tokens_per_s(T, world, ms)

    # The timed region is short (args.steps layer calls, a fraction of a second at
    # the default), so kernels are measured against the burst peaks; the expert
    # contractions' fraction of the sustained (power-capped) peak is printed beside.
    work, single, per_stage, gemm = stage_report(shape, stage_ms, kept, experts_used, peaks, False)
    fused, fused_combine = fused_stages(shape)
    dom = max(single, key=lambda s_: stage_ms[s_])
    roof = per_stage[dom]
    tc_util = 100.0 * gemm["frac_of_burst"]

    # end to end: every step copies its inputs from pinned host memory and reads
    # its result back.  Steps are pipelined over two buffer sets and three
    # streams (host->device copies, the layer, device->host copies), as a caller
    # streaming batches would run them: step i+1's inputs and step i-1's result
    # cross PCIe while step i computes.
    aux_n = 2 if shape.z_coef else 1
    x_host = inp["x"].cpu().pin_memory()
    add_host = None if inp["logit_add"] is None else inp["logit_add"].cpu().pin_memory()
    uni_host = None if inp["uniform"] is None else inp["uniform"].cpu().pin_memory()
    h2d = x_host.numel() * x_host.element_size() + (0 if add_host is None else add_host.numel() * 4) \
        + (0 if uni_host is None else uni_host.numel() * 4)
    d2h = T * H * x_host.element_size() + 4 * aux_n
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    bufs = []
    for _ in range(2):
        b = {"x": torch.empty_like(inp["x"]),
             "add": None if add_host is None else torch.empty_like(inp["logit_add"]),
             "uni": None if uni_host is None else torch.empty_like(inp["uniform"]),
             "y": torch.empty((T, H), dtype=edt, device=dev), "aux": torch.empty(2, dtype=torch.float32, device=dev),
             "y_host": torch.empty((T, H), dtype=edt).pin_memory(),
             "aux_host": torch.empty(aux_n, dtype=torch.float32).pin_memory()}
        for name in ("loaded", "computed", "drained"):
            b[name] = torch.cuda.Event()
            b[name].record(stream)          # created (and complete) before first use
        bufs.append(b)

    def e2e_step(i):
        b = bufs[i % 2]
        s_in.wait_event(b["computed"])      # the layer that read these inputs is done
        with torch.cuda.stream(s_in):
            b["x"].copy_(x_host, non_blocking=True)
            if add_host is not None:
                b["add"].copy_(add_host, non_blocking=True)
            if uni_host is not None:
                b["uni"].copy_(uni_host, non_blocking=True)
        b["loaded"].record(s_in)
        stream.wait_event(b["loaded"])
        stream.wait_event(b["drained"])     # this y buffer has been read back
        B.moe_layer_fwd(cfg, b["x"], run.wg, b["add"], b["uni"], wts, b["y"], b["aux"], None, ws, stream=stream)
        b["computed"].record(stream)
        s_out.wait_event(b["computed"])
        with torch.cuda.stream(s_out):
            b["y_host"].copy_(b["y"], non_blocking=True)
            b["aux_host"].copy_(b["aux"][:aux_n], non_blocking=True)
        b["drained"].record(s_out)

    for i in range(max(args.warmup, 3)):
        e2e_step(i)
    e2e_steps = args.steps
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ea.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    eb.record(s_out)                        # after the last read-back
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(ea.elapsed_time(eb) / e2e_steps, world)
    C = B.moe_capacity(cfg)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(shape, inp, kept)
    others = None
    if rank == 0 and world == 1 and not args.no_other_workloads and args.workload == DEFAULT_WORKLOAD \
            and not args.set:
        del bufs, x_host, run, wts
        inp = None
        torch.cuda.empty_cache()
        others = other_workloads(B, args, peaks, dev, stream)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if shape.dtype == 1 else "f32", "data": "synthetic",
            "config": {"workload": shape.name, "T": T, "H": H, "F": shape.F, "E": shape.E, "k": shape.k,
                       "n_shared": shape.n_shared, "act": ["relu", "gelu", "swiglu"][shape.act],
                       "capacity": C, "kept_assignments": kept, "rows_used": rows_used,
                       "l2": "flushed before every step (320 MiB write + 320 MiB read, outside the timed events)",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "weights": "packed once before timing (moe_pack_weight, moe_pack_router_weight)" if packed
                       else "linear-layer layout, router weight split on every call"},
            "stages_ms": stage_ms,
            "stages_note": f"second timed pass of {n_stage_steps} steps with per-stage events "
                           f"({stage_sum_ms:.4f} ms per step including the events' own cost)",
            "dispatch_gbs": per_stage["dispatch"]["achieved"] if "dispatch" in per_stage else None,
            "combine_gbs": per_stage["combine"]["achieved"] if "combine" in per_stage else None,
            "fused": {"dispatch_into_gemm1": fused, "combine_into_gemm2": fused_combine},
            "expert_gemm_tc_util_pct": tc_util,
            "expert_gemm": gemm,
            "roofline": {k_: roof[k_] for k_ in ("bound", "achieved", "peak", "unit", "frac", "traffic", "peak_source")},
            "roofline_detail": {s_: {k_: v[k_] for k_ in ("bound", "achieved", "unit", "frac", "ms_per_launch")}
                                for s_, v in per_stage.items()},
            "dominant_kernel": dom,
            "e2e": {"value": job_tokens_per_s(T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "pipelining": "2 buffer sets; copy-in, layer, copy-out streams"},
            "gpu_launches": launches_per_step(shape, packed) * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "other_workloads": others,
        }
        print(json.dumps(line), flush=True)


def run_train(args, world, rank, local):
    """One step = moe_layer_fwd with MOE_FLAG_TRAINING, then moe_layer_bwd with
    a synthetic upstream gradient dy (and d_aux = d_z = 1)."""
    import torch
    from expert_dispatch_router_b200 import binding as B
    from expert_dispatch_router_b200 import synth

    B.load()                                     # raises if the CUDA library is missing
    shape = workload_shape(args)
    if shape.dtype != 1:
        raise SystemExit("--pass train: the backward runs on bf16 layers only")
    peaks = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = synth.make_inputs(shape, seed=replica_seed(args.seed, rank), device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(replica_seed(args.seed, rank) + 1000)
    T, H, F, E = shape.T, shape.H, shape.F, shape.E
    dy = torch.randn((T, H), generator=gen, device=dev).to(torch.bfloat16)
    packed = not args.unpacked
    cfg = B.make_cfg(shape, flags=B.MOE_FLAG_TRAINING | (B.MOE_FLAG_PACKED_WEIGHTS if packed else 0))
    ws = B.alloc_workspace(cfg)
    wsrc = B.pack_weights(inp) if packed else inp
    torch.cuda.synchronize()
    wts = B.make_weights(wsrc)
    sw = shape.act == synth.ACT_SWIGLU
    g = dict(dw1=torch.empty((E, F, H), device=dev), dw2=torch.empty((E, H, F), device=dev),
             dw3=torch.empty((E, F, H), device=dev) if sw else None)
    if shape.n_shared:
        g.update(dsw1=torch.empty((1, F, H), device=dev), dsw2=torch.empty((1, H, F), device=dev),
                 dsw3=torch.empty((1, F, H), device=dev) if sw else None)
    grads = B.make_weight_grads(g)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    aux = torch.empty(2, dtype=torch.float32, device=dev)
    dx = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    dwg = torch.empty((E, H), dtype=torch.float32, device=dev)
    flush_w = torch.empty(320 * 2**20 // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(320 * 2**20 // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=flush_sink)

    def layer(x, d, add, uni, fev=None, bev=None):
        B.moe_layer_fwd(cfg, x, inp["wg"], add, uni, wts, y, aux, None, ws, stage_events=fev, stream=stream)
        B.moe_layer_bwd(cfg, x, inp["wg"], wts, d, 1.0, 1.0, dx, dwg, grads, ws, stage_events=bev, stream=stream)

    for _ in range(max(args.warmup, 3)):
        flush_l2()
        layer(inp["x"], dy, inp["logit_add"], inp["uniform"])
    st = B.moe_sync_status(ws, stream)
    if st != B.MOE_OK:
        raise RuntimeError(f"device status after warm-up: {B.strerror(st)}")
    wt = B.workspace_tensors(cfg, ws)
    kept = int(wt["kept_count"].sum().item())
    experts_used = int((wt["kept_count"] > 0).sum().item())

    n_stage_steps = min(args.steps, 200)
    ends = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    fevs = [[torch.cuda.Event(enable_timing=True) for _ in range(B.MOE_N_STAGE_EVENTS)] for _ in range(n_stage_steps)]
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(B.MOE_N_BWD_STAGE_EVENTS)]
            for _ in range(n_stage_steps)]
    for e in [x for pair in ends for x in pair] + [x for row in fevs + bevs for x in row]:
        e.record(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.wait_first()
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    for i in range(args.steps):
        flush_l2()
        ends[i][0].record(stream)
        layer(inp["x"], dy, inp["logit_add"], inp["uniform"])
        ends[i][1].record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    for i in range(n_stage_steps):
        flush_l2()
        layer(inp["x"], dy, inp["logit_add"], inp["uniform"], fevs[i], bevs[i])
    torch.cuda.synchronize()
    barrier(world)
    clocks = None
    if sampler:
        sampler.stop()
        clocks = sampler.summary(t0, t1)
    st = B.moe_sync_status(ws, stream)
    if st != B.MOE_OK:
        raise RuntimeError(f"device status after the timed region: {B.strerror(st)}")
    ms_local = sum(a.elapsed_time(b) for a, b in ends) / args.steps
    ms = max_over_ranks(ms_local, world)
    value = job_tokens_per_s(T, world, ms)
    fwd_ms = sum(e[0].elapsed_time(e[-1]) for e in fevs) / n_stage_steps
    stage_ms = {name: sum(e[j].elapsed_time(e[j + 1]) for e in bevs) / n_stage_steps
                for j, name in enumerate(B.BWD_STAGES)}
    # T*k <= 256*E or H <= 512: dh and dz come from one kernel, in the dh interval (dz's is empty)
    bwd_fused = T * shape.k <= 256 * E or H <= 512
    if bwd_fused:
        stage_ms["dh_dz"] = stage_ms.pop("dgrad_dh") + stage_ms.pop("dact_dz")
    dh_names = ["dh_dz"] if bwd_fused else ["dgrad_dh", "dact_dz"]
    bwd_names = ["combine_bwd"] + dh_names + ["wgrad_w2", "wgrad_w1", "router_bwd", "dgrad_dx", "dispatch_bwd",
                                              "router_wgrad"]
    bwd_ms = sum(e[0].elapsed_time(e[-1]) for e in bevs) / n_stage_steps
    work = bwd_stage_work(shape, kept, experts_used)
    long_step = ms_local > 5.0
    per_stage = {s_: roofline(s_, work, stage_ms[s_], peaks, shape.name, True, long_step) for s_ in bwd_names}
    dom = max(bwd_names, key=lambda s_: stage_ms[s_])
    roof = per_stage[dom]

    # end to end: x and dy copied in from pinned host memory, the loss terms
    # (aux, and the z-loss when on) read back, serially within each step
    aux_n = 2 if shape.z_coef else 1
    x_host = inp["x"].cpu().pin_memory()
    dy_host = dy.cpu().pin_memory()
    add_host = None if inp["logit_add"] is None else inp["logit_add"].cpu().pin_memory()
    uni_host = None if inp["uniform"] is None else inp["uniform"].cpu().pin_memory()
    xd, dyd = torch.empty_like(inp["x"]), torch.empty_like(dy)
    addd = None if add_host is None else torch.empty_like(inp["logit_add"])
    unid = None if uni_host is None else torch.empty_like(inp["uniform"])
    aux_host = torch.empty(aux_n, dtype=torch.float32).pin_memory()
    h2d = 2 * T * H * 2 + (0 if add_host is None else add_host.numel() * 4) + (0 if uni_host is None else T * 4)

    def e2e_step():
        xd.copy_(x_host, non_blocking=True)
        dyd.copy_(dy_host, non_blocking=True)
        if addd is not None:
            addd.copy_(add_host, non_blocking=True)
        if unid is not None:
            unid.copy_(uni_host, non_blocking=True)
        layer(xd, dyd, addd, unid)
        aux_host.copy_(aux[:aux_n], non_blocking=True)

    for _ in range(max(args.warmup, 3)):
        e2e_step()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ea.record(stream)
    for _ in range(args.steps):
        e2e_step()
    eb.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(ea.elapsed_time(eb) / args.steps, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = host_inputs(inp)
        dyh = dy.to("cpu", torch.float64).numpy()
        n = min(T, 128)
        t = oracle_train_sample_time(shape, host, dyh, n)
        while t < 5.0 and n < T:
            n = min(T, max(n * 2, int(n * 15.0 / max(t, 1e-3) * 0.8)))
            t = oracle_train_sample_time(shape, host, dyh, n)
        cpu = {"value": n / t, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"the oracle's forward and backward on the first {n} of {T} tokens as a batch of its own "
                         f"({t:.1f} s, capacity recomputed for that batch)"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": shape.name, "pass": "forward+backward (moe_layer_fwd TRAINING + moe_layer_bwd)",
                       "T": T, "H": H, "F": F, "E": E, "k": shape.k, "n_shared": shape.n_shared,
                       "act": ["relu", "gelu", "swiglu"][shape.act], "kept_assignments": kept,
                       "l2": "flushed before every step (320 MiB write + 320 MiB read, outside the timed events)",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "weights": "packed once before timing (moe_pack_weight)" if packed else "linear-layer layout"},
            "forward_ms": fwd_ms, "backward_ms": bwd_ms, "backward_stages_ms": stage_ms,
            "backward_dh_dz_fused": bwd_fused,
            "stages_note": f"second timed pass of {n_stage_steps} steps with per-stage events",
            "roofline": {k_: roof[k_] for k_ in ("bound", "achieved", "peak", "unit", "frac", "traffic", "peak_source")},
            "roofline_detail": {s_: {k_: v[k_] for k_ in ("bound", "achieved", "unit", "frac", "ms_per_launch")}
                                for s_, v in per_stage.items()},
            "dominant_kernel": dom,
            "e2e": {"value": job_tokens_per_s(T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": 4 * aux_n, "pipelining": "none (copies serial with the step)"},
            "gpu_launches": train_launches_per_step(shape) * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.pass_ == "train":
            run_train(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
