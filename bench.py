"""Benchmark of the ISA attention forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl isa|reference]
                    [--config 480p] [--no-cpu-baseline] [--no-e2e]

A step is one pass of the whole ISA forward (pre-selection, sharpness and
routing, full attention for routed queries, Taylor attention for the rest)
over one batch of the 480p-latent workload (B=1, H=24, d=128, 20280 source +
20280 context tokens, block 128, keep 0.25, rho 0.2; seeded synthetic bf16
inputs).  q, k, v (747 MB) are larger than the 126 MB L2, so no flush is
needed between steps.  Timing: CUDA events on the launching stream around
exactly K steps after W warm-up steps, barrier + synchronize on both sides,
max over ranks.  With N > 1 (torchrun), every rank runs its own replica of
the workload (heads are independent units: no collective on the data path).

--impl reference times the float64 CPU oracle on the host cores instead
(rank 0 only): each timed step runs one whole head of the workload
(`ms_per_step` is that sample's time); `value` scales it to all B*H heads.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import CONFIGS, bf16_bits_to_f64, head_inputs, make_inputs, to_torch_bf16  # noqa: E402

METRIC = "ISA attn fwd latency (ms), eff. TFLOP/s vs in-house dense kernel, 1×B200"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def counts(cfg):
    """Static per-head sizes of the ISA reading (block layout, kept / routed counts)."""
    import math

    nSB = -(-cfg.N_src // cfg.block)
    nCB = -(-cfg.N_ctx // cfg.block)
    def guarded(frac, n):  # ceil(frac*n - min(1e-6*n, 0.5)) in [0, n], as the library counts
        return int(min(max(math.ceil(frac * n - min(1e-6 * n, 0.5)), 0), n))

    n_keep = guarded(cfg.keep, nCB)
    n_route = guarded(cfg.rho, cfg.N)
    return nSB, nCB, n_keep, n_route


# DRAM bytes (read + write) of one routed full-attention stage at the 480p
# workload -- whole-wave launch, key-split launch and combine -- summed from
# ncu captures of one kernel each (dram__bytes_read.sum +
# dram__bytes_write.sum, one pass).
# They hold only for the kernel sources they were taken on: on any other
# source, or another workload, the report's traffic is null.
FULL_TRAFFIC = {
    "config": "480p",
    # whole-wave launch (read + write), key-split launch (read + write), combine
    "bytes": 394_021_632 + 40_587_008 + 14_961_152 + 1_536 + 18_468_096 + 0,
    "sources": {
        "sparse_attention_context_b200/csrc/flash2.cu": "a69fddf185ddeebee261af69fe5febba3d64c92f11b0083ef6b52262ff9f90aa",
        "sparse_attention_context_b200/csrc/gather.cuh": "842e9958e7de511bd130413934b8da2dfcbd8ed14cef6f38ff09d728b527b34a",
        "sparse_attention_context_b200/csrc/tc_ptx.cuh": "1026ba5d3e08b740b9d4aa8f4fc7e2bd31b8c482744693570e460f8679e5be71",
    },
}


def full_traffic(args):
    """The captured stage traffic if it applies to this run, else None."""
    import hashlib

    if args.config != FULL_TRAFFIC["config"] or args.heads or args.rho is not None or args.keep is not None:
        return None
    if getattr(args, "shard", "replicas") == "heads" and int(os.environ.get("WORLD_SIZE", "1")) > 1:
        return None  # a slice of the heads per rank: not the captured launch
    root = os.path.dirname(os.path.abspath(__file__))
    for rel, digest in FULL_TRAFFIC["sources"].items():
        with open(os.path.join(root, rel), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != digest:
                return None
    return FULL_TRAFFIC["bytes"]


def full_stage_launches(cfg, n_keep, n_route, nsm):
    """Kernel launches of the routed full-attention stage: one launch for the
    whole waves of 256-row items; when a partial last wave remains, its items
    run split along the key tiles over the SMs (a second launch) and a combine
    kernel merges the pieces (a third).  Mirrors the launcher's rule."""
    if n_route <= 0:
        return 0
    nSB = -(-cfg.N_src // cfg.block)
    items = cfg.B * cfg.H * (-(-n_route // 256))
    rem = items % nsm
    if rem == 0:
        return 1
    pieces = min(nsm // rem, (nSB + n_keep) // 4)
    return 3 if pieces >= 2 else 1


def work_model(cfg, kept_tokens_mean):
    """Executed FLOPs and algorithmic bytes of one step (all heads)."""
    nSB, nCB, n_keep, n_route = counts(cfg)
    BH, N, d = cfg.B * cfg.H, cfg.N, cfg.d
    nK = nSB + n_keep
    T = kept_tokens_mean
    return dict(
        dense_flops=4.0 * BH * N * N * d,
        full_flops=4.0 * BH * d * n_route * T,
        taylor_flops=4.0 * BH * d * (N - n_route) * nK,
        sharp_flops=2.0 * 2.0 * BH * d * N * nK,
        # fused sharpness + Taylor pass over every query: hi + lo logits and PV
        fused_flops=6.0 * BH * d * N * nK,
        # algorithmic bytes of the full-attention kernel: routed Q rows and O
        # rows once, K and V of the kept tokens once per head (L2 reuse)
        full_bytes=BH * (2 * n_route * d * 2 + 2 * T * d * 2),
    )


class ClockSampler:
    """Reads SM clocks and clock-event (throttle) reasons through NVML every
    few milliseconds while the timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, torch_device, period_s=0.002):
        self.dev = torch_device
        self.period = period_s
        self.sm, self.mx, self.reasons, self.err = [], None, set(), None
        self._stop = threading.Event()
        self.h = None

    def _handle(self):
        import pynvml as nv
        import torch

        nv.nvmlInit()
        p = torch.cuda.get_device_properties(self.dev)
        try:
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv, nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv, nv.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def _run(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                self.sm.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, attr in self.REASONS.items():
                    if r & getattr(nv, attr):
                        self.reasons.add(name)
            except Exception as e:  # keep timing even if NVML misbehaves
                self.err = repr(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        try:
            self.nv, self.h = self._handle()
            self.mx = self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception as e:
            self.err = repr(e)
            self.h = None
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.h is not None:
            self.t.join(timeout=2)

    def summary(self):
        if not self.sm:
            return {"sm_mhz": None, "sm_max_mhz": self.mx, "reasons": sorted(self.reasons), "samples": 0,
                    "source": "nvml", "error": self.err}
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": self.mx, "reasons": sorted(self.reasons),
                "samples": len(self.sm), "source": "nvml"}


def cpu_oracle_ms_per_step(cfg, heads, seed=0):
    """Wall time of the float64 oracle on `heads` of the workload, scaled to a
    whole step (all B*H heads).  Returns (ms_per_step, seconds_measured)."""
    import oracle  # the CPU baseline leg is the one place bench.py runs the oracle

    t_total = 0.0
    for h in heads:
        q, k, v = (bf16_bits_to_f64(x) for x in head_inputs(cfg, 0, h, seed))
        t0 = time.perf_counter()
        oracle.isa_head(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
        t_total += time.perf_counter() - t0
    return 1e3 * t_total / len(heads) * cfg.B * cfg.H, t_total


def dist_env():
    """(world size, rank, local rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x, device):
    """Max of a per-rank float over all ranks of the default process group
    (the value itself on one rank).  Timing only: never on the data path."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(rank):
    """Each rank's replica of the workload draws its own inputs (weak scaling:
    every (b, h) of every replica is an independent unit)."""
    return rank


def run_reference(args, cfg):
    """The reference arm: the float64 oracle on the host cores.  A whole
    480p step takes about half a minute of host time, so each timed step is
    a bounded sample, one whole head of the workload (heads are independent
    units).  `ms_per_step` is the wall time of that sample per timed step
    (what the clock around the run sees); `value` is the whole-step time
    it stands for, the per-head time x B*H, and `value_basis` says so."""
    _, rank, _ = dist_env()
    if rank != 0:
        return
    cores = len(os.sched_getaffinity(0))
    nh = cfg.B * cfg.H
    for s in range(args.warmup):
        cpu_oracle_ms_per_step(cfg, [s % nh])
    per, sample_ms = [], []
    for s in range(args.steps):
        ms, secs = cpu_oracle_ms_per_step(cfg, [(args.warmup + s) % nh])
        per.append(ms)
        sample_ms.append(1e3 * secs)
    v = float(np.mean(per))
    basis = f"one head of {nh} per timed step; value = mean per-head time x {nh}"
    rec = {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "ms", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(float(np.mean(sample_ms)), 3),
           "value_basis": basis, "higher_is_better": False,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config_dict(cfg, args.gpus),
           "cpu_baseline": {"value": round(v, 3), "unit": "ms", "cores": cores, "kind": "oracle",
                            "sample": f"1 of {nh} heads per step, scaled x{nh}"},
           "e2e": {"value": round(v, 3), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(rec), flush=True)


def run_sweep(args):
    """Latency of the ISA forward over the keep x rho grid of the sweep
    workload (B=1, H=24, d=128, 32768 + 32768 tokens, block 128) beside the
    in-house dense kernel; one JSON line per grid point.  The oracle error of
    every grid point is checked by tests/test_gpu_sweep.py."""
    import torch

    from sparse_attention_context_b200 import api

    cfg = CONFIGS["sweep"]
    if args.heads:
        cfg = cfg.replace(H=args.heads)
    q, k, v = (to_torch_bf16(b).cuda() for b in make_inputs(cfg, seed=0))
    stream = torch.cuda.current_stream()

    def timed(fn, warm, n):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    dws = api.dense_workspace(cfg.d)
    dout = torch.empty_like(q)
    dense_ms = timed(lambda: api.isa_dense_attn_fwd(q, k, v, out=dout, ws=dws), 1, 2)
    del dout
    dense_flops = 4.0 * cfg.B * cfg.H * cfg.N * cfg.N * cfg.d
    out = torch.empty_like(q)
    for keep in (0.1, 0.25, 0.5, 1.0):
        for rho in (0.0, 0.1, 0.2, 0.5, 1.0):
            shape = api.make_shape(q, cfg.N_src, cfg.block, keep, rho)
            ws = api.new_workspace(shape)
            ms = timed(lambda: api.isa_forward(q, k, v, cfg.N_src, cfg.block, keep, rho, ws=ws, out=out),
                       max(args.warmup, 1), max(args.steps, 1))
            assert api.isa_read_device_status(ws) == 0
            print(json.dumps({"sweep": cfg.name, "H": cfg.H, "keep": keep, "rho": rho, "ms": round(ms, 4),
                              "dense_ms": round(dense_ms, 3), "isa_over_dense": round(ms / dense_ms, 4),
                              "eff_tflops": round(dense_flops / (ms * 1e-3) / 1e12, 1)}), flush=True)
            del ws


def run_block_grouping(args):
    """The block-granular grouping variant on the 480p latent workload beside
    the per-token grouping: latency of both forwards (CUDA events), the
    stage split of the block variant, and the approximation error of each
    against full attention for every query over the same kept tokens
    (rho = 1), Sum|o - o_full| / Sum|o_full|.  One JSON line.  Oracle parity
    of the variant is checked by tests/test_gpu_block_route.py."""
    import torch

    from sparse_attention_context_b200 import api

    cfg = CONFIGS[args.config]
    if args.heads:
        cfg = cfg.replace(H=args.heads)
    if args.rho is not None:
        cfg = cfg.replace(rho=args.rho)
    if args.keep is not None:
        cfg = cfg.replace(keep=args.keep)
    q, k, v = (to_torch_bf16(b).cuda() for b in make_inputs(cfg, seed=0))
    stream = torch.cuda.current_stream()
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    out_t, out_b = torch.empty_like(q), torch.empty_like(q)

    def timed(fn, warm, n):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    W, K = max(args.warmup, 3), max(args.steps, 1)
    ms_tok = timed(lambda: api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws, out=out_t), W, K)
    ms_blk = timed(lambda: api.isa_forward_blocks(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws,
                                                  out=out_b), W, K)
    # stage split of the block variant
    kept = torch.empty((cfg.B, cfg.H, api.isa_n_keep(shape)), dtype=torch.int32, device=q.device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    acc = np.zeros(3)
    for i in range(W + K):
        ev[0].record(stream)
        api.isa_preselect_ctx(q, k, v, shape, ws, kept=kept, want_saliency=False)
        ev[1].record(stream)
        _, rows, _, _ = api.isa_route_blocks_taylor_fwd(q, kept, shape, ws, out_b, want_scores=False,
                                                        want_sharpness=False)
        ev[2].record(stream)
        api.isa_full_attn_rows_fwd(q, k, v, kept, rows, shape, ws, out_b)
        ev[3].record(stream)
        torch.cuda.synchronize()
        if i >= W:
            acc += [ev[j].elapsed_time(ev[j + 1]) for j in range(3)]
    acc /= K
    assert api.isa_read_device_status(ws) == 0
    ref = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, 1.0)  # every query on full attention
    torch.cuda.synchronize()
    ref_abs = ref.float().abs().sum().item()

    def err(o):
        d = (o.float() - ref.float()).abs()
        return {"mean_rel": round(d.sum().item() / ref_abs, 6), "max_abs": round(d.max().item(), 5)}

    nrb = api.isa_n_route_blocks(shape)
    print(json.dumps({
        "variant": "block-granular query grouping", "config": config_dict(cfg, 1),
        "token_grouping_ms": round(ms_tok, 4), "block_grouping_ms": round(ms_blk, 4),
        "block_stage_ms": {"preselect": round(acc[0], 4), "sharpness_taylor_route_blocks": round(acc[1], 4),
                           "full_attn_rows": round(acc[2], 4)},
        "routed_queries": {"token": api.isa_n_route(shape), "block_rows": nrb * cfg.block, "blocks": nrb},
        "error_vs_full_over_kept": {"token": err(out_t), "block": err(out_b)},
        "steps": K, "warmup": W}), flush=True)


def run_taylor1(args):
    """The first-order Taylor variant of stage 4 on the 480p latent workload
    beside the 0-th order forward: latency of both forwards (CUDA events),
    the stage split of the first-order forward, the executed TFLOP/s of its
    first-order stage against the measured bf16 peak, and the approximation
    error of each against full attention for every query over the same
    kept tokens (rho = 1).  One JSON line.  Oracle parity of the variant is
    checked by tests/test_gpu_taylor1.py."""
    import torch

    from sparse_attention_context_b200 import api

    cfg = CONFIGS[args.config]
    if args.heads:
        cfg = cfg.replace(H=args.heads)
    if args.rho is not None:
        cfg = cfg.replace(rho=args.rho)
    if args.keep is not None:
        cfg = cfg.replace(keep=args.keep)
    q, k, v = (to_torch_bf16(b).cuda() for b in make_inputs(cfg, seed=0))
    stream = torch.cuda.current_stream()
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    cws = api.taylor1_workspace(shape)
    out0, out1 = torch.empty_like(q), torch.empty_like(q)
    W, K = max(args.warmup, 3), max(args.steps, 1)

    def timed(fn):
        for _ in range(W):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K

    ms0 = timed(lambda: api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws, out=out0))
    ms1 = timed(lambda: api.isa_forward_taylor1(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws, cws=cws,
                                                out=out1))
    nSB, nCB, n_keep, n_route = counts(cfg)
    kept = torch.empty((cfg.B, cfg.H, n_keep), dtype=torch.int32, device=q.device)
    routed = torch.empty((cfg.B, cfg.H, n_route), dtype=torch.int32, device=q.device)
    taylor = torch.empty((cfg.B, cfg.H, cfg.N - n_route), dtype=torch.int32, device=q.device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    acc = np.zeros(4)
    for it in range(W + K):
        ev[0].record(stream)
        api.isa_preselect_ctx(q, k, v, shape, ws, kept=kept, want_saliency=False)
        ev[1].record(stream)
        api.isa_route_taylor_fwd(q, kept, shape, ws, out1, routed=routed, taylor=taylor, want_sharpness=False)
        ev[2].record(stream)
        api.isa_full_attn_fwd(q, k, v, kept, routed, shape, ws, out1)
        ev[3].record(stream)
        api.isa_taylor1_attn_fwd(q, k, v, kept, taylor, shape, ws, cws, out1)
        ev[4].record(stream)
        torch.cuda.synchronize()
        if it >= W:
            acc += [ev[j].elapsed_time(ev[j + 1]) for j in range(4)]
    acc /= K
    assert api.isa_read_device_status(ws) == 0
    ref = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, 1.0)  # every query on full attention
    torch.cuda.synchronize()
    ref_abs = ref.float().abs().sum().item()

    def err(o, rows=None):
        d = (o.float() - ref.float()).abs()
        return {"mean_rel": round(d.sum().item() / ref_abs, 6), "max_abs": round(d.max().item(), 5)}

    BH, d, nK = cfg.B * cfg.H, cfg.d, nSB + n_keep
    t1_flops = BH * (cfg.N - n_route) * nK * (4.0 * d + 2.0 * d * d) + BH * nK * 2.0 * d * d * cfg.block
    pk, pk_kind = peaks()
    ach = t1_flops / (acc[3] * 1e-3) / 1e12
    print(json.dumps({
        "variant": "first-order Taylor stage 4", "config": config_dict(cfg, 1),
        "taylor0_forward_ms": round(ms0, 4), "taylor1_forward_ms": round(ms1, 4),
        "taylor1_stage_ms": {"preselect": round(acc[0], 4), "sharpness_taylor0_route": round(acc[1], 4),
                             "full_attn": round(acc[2], 4), "first_order_taylor": round(acc[3], 4)},
        "first_order_stage_roofline": {"bound": "tensor", "executed_tflop": round(t1_flops / 1e12, 3),
                                       "achieved": round(ach, 1), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                                       "frac": round(ach / pk["bf16_tflops"], 4),
                                       "peak_kind": f"{pk_kind} burst bf16"},
        "error_vs_full_over_kept": {"taylor0": err(out0), "taylor1": err(out1)},
        "steps": K, "warmup": W}), flush=True)


def run_dit_layer(args):
    """A DiT self-attention layer (QKV projection, attention, output
    projection; random bf16 weights, C = H*d channels) on the 480p latent
    shape, with the ISA forward and with the in-house dense kernel as its
    attention: layer latency and its parts (CUDA events).  One JSON line."""
    import torch

    from sparse_attention_context_b200 import api
    from sparse_attention_context_b200.dit_layer import attention_layer, merge_heads, random_weights, split_heads

    cfg = CONFIGS[args.config]
    if args.heads:
        cfg = cfg.replace(H=args.heads)
    H, N, d = cfg.H, cfg.N, cfg.d
    C = H * d
    g = torch.Generator(device="cpu").manual_seed(0)
    x = torch.randn(N, C, generator=g).to(device="cuda", dtype=torch.bfloat16)
    w_qkv, w_o = random_weights(C)
    stream = torch.cuda.current_stream()
    shape = api.make_shape(torch.empty((1, H, N, d), device="meta"), cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape)
    dws = api.dense_workspace(d)
    W, K = max(args.warmup, 3), max(args.steps, 1)

    def timed(fn, k=K):
        for _ in range(W):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / k

    kw = dict(H=H, N_src=cfg.N_src, block=cfg.block, keep=cfg.keep, rho=cfg.rho)
    isa_ms = timed(lambda: attention_layer(x, w_qkv, w_o, attention="isa", ws=ws, **kw))
    dense_ms = timed(lambda: attention_layer(x, w_qkv, w_o, attention="dense", dense_ws=dws, **kw), max(2, K // 4))
    qkv_ms = timed(lambda: split_heads(x @ w_qkv.t(), H))
    q, k, v = split_heads(x @ w_qkv.t(), H)
    attn_ms = timed(lambda: api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws))
    o = api.isa_forward(q, k, v, cfg.N_src, cfg.block, cfg.keep, cfg.rho, ws=ws)
    out_ms = timed(lambda: merge_heads(o) @ w_o.t())
    dense_attn_ms = timed(lambda: api.isa_dense_attn_fwd(q, k, v, ws=dws), max(2, K // 4))
    assert api.isa_read_device_status(ws) == 0
    proj_flop = 2.0 * N * C * 3 * C + 2.0 * N * C * C
    print(json.dumps({
        "variant": "DiT self-attention layer", "config": config_dict(cfg, 1),
        "channels": C, "weights": "random bf16 (std 1/sqrt(C))", "input": "x ~ N(0, 1) bf16, seed 0",
        "layer_isa_ms": round(isa_ms, 4), "layer_dense_ms": round(dense_ms, 4),
        "layer_isa_over_dense": round(isa_ms / dense_ms, 4),
        "attention_isa_ms": round(attn_ms, 4), "attention_dense_ms": round(dense_attn_ms, 4),
        "qkv_projection_ms": round(qkv_ms, 4), "out_projection_ms": round(out_ms, 4),
        "projection_tflops": round(proj_flop / ((qkv_ms + out_ms) * 1e-3) / 1e12, 1),
        "steps": K, "warmup": W}), flush=True)


def config_dict(cfg, n, shard="replicas"):
    if n <= 1:
        par = "single GPU"
    elif shard == "heads":
        par = f"heads sharded x{n}"
    else:
        par = f"replicas x{n}"
    return {"workload": f"ISA fwd {cfg.name}-latent: B={cfg.B} H={cfg.H} d={cfg.d} N_src={cfg.N_src} "
                        f"N_ctx={cfg.N_ctx} block={cfg.block} keep={cfg.keep} rho={cfg.rho}",
            "B": cfg.B, "H": cfg.H, "d": cfg.d, "N_src": cfg.N_src, "N_ctx": cfg.N_ctx, "block": cfg.block,
            "keep": cfg.keep, "rho": cfg.rho, "parallelism": par,
            "l2": l2_note(cfg)}


def l2_note(cfg):
    mb = 3 * cfg.B * cfg.H * cfg.N * cfg.d * 2 / 1e6
    if mb > 126:
        return f"inputs ({mb:.0f} MB) larger than the 126 MB L2, no flush"
    return f"inputs ({mb:.1f} MB) fit in the 126 MB L2 and stay there between steps (warm, no flush)"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="isa", choices=["isa", "reference"])
    ap.add_argument("--config", default="480p")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--heads", type=int, default=None, help="override H (small profiling captures)")
    ap.add_argument("--rho", type=float, default=None, help="override rho (profiling captures)")
    ap.add_argument("--keep", type=float, default=None, help="override keep (profiling captures)")
    ap.add_argument("--sweep", action="store_true", help="keep x rho latency grid of the sweep workload")
    ap.add_argument("--grouping", default="token", choices=["token", "block"],
                    help="block: time the block-granular query grouping variant beside the per-token one")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: one replica of the workload per rank (weak scaling, default) or the heads of one "
                         "problem split over the ranks (strong scaling)")
    ap.add_argument("--gather", action="store_true",
                    help="with --shard heads: also time the all-gather of the output heads onto every rank")
    ap.add_argument("--dit-layer", action="store_true",
                    help="time a DiT self-attention layer (projections + ISA) beside the same layer with dense attention")
    ap.add_argument("--taylor-order", type=int, default=0, choices=[0, 1],
                    help="1: time the first-order Taylor variant of stage 4 beside the 0-th order forward")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.grouping == "block":
        run_block_grouping(args)
        return
    if args.taylor_order == 1:
        run_taylor1(args)
        return
    if args.dit_layer:
        run_dit_layer(args)
        return
    cfg = CONFIGS[args.config]
    if args.heads:
        cfg = cfg.replace(H=args.heads)
    if args.rho is not None:
        cfg = cfg.replace(rho=args.rho)
    if args.keep is not None:
        cfg = cfg.replace(keep=args.keep)
    if args.impl == "reference":
        run_reference(args, cfg)
        return

    import torch
    import torch.distributed as dist

    from sparse_attention_context_b200 import api

    world, rank, local = dist_env()
    if world > 1:
        import datetime

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    cfg_job = cfg  # the problem the report names
    if args.shard == "heads":
        # one problem, its heads split over the ranks: every rank draws its own
        # heads of the same seeded problem (per-head generator streams)
        from sparse_attention_context_b200.sharding import shard_heads

        h0, h1 = shard_heads(cfg.H, world, rank)
        if h1 <= h0:
            raise SystemExit(f"--shard heads: {cfg.H} heads cannot be split over {world} ranks")
        bits = make_inputs(cfg, seed=0, heads=range(h0, h1))
        cfg = cfg.replace(H=h1 - h0)
    else:
        bits = make_inputs(cfg, seed=replica_seed(rank))
    q, k, v = (to_torch_bf16(b).to(dev) for b in bits)
    shape = api.make_shape(q, cfg.N_src, cfg.block, cfg.keep, cfg.rho)
    ws = api.new_workspace(shape, dev)
    nSB, nCB, n_keep, n_route = counts(cfg)
    B, H, N = cfg.B, cfg.H, cfg.N
    kept = torch.empty((B, H, n_keep), dtype=torch.int32, device=dev)
    routed = torch.empty((B, H, n_route), dtype=torch.int32, device=dev)
    taylor = torch.empty((B, H, N - n_route), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()

    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    def step(i=None):
        # the isa_forward sequence, one ABI call per stage so that each is event-timed
        e = stage_ev[i] if i is not None else None
        if e: e[0].record(stream)
        api.isa_preselect_ctx(q, k, v, shape, ws, kept=kept, want_saliency=False)
        if e: e[1].record(stream)
        api.isa_route_taylor_fwd(q, kept, shape, ws, out, routed=routed, taylor=taylor, want_sharpness=False)
        if e: e[2].record(stream)
        api.isa_full_attn_fwd(q, k, v, kept, routed, shape, ws, out)
        if e: e[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert api.isa_read_device_status(ws) == 0
    # kept token count (for the work model), from the kept set of this input
    kept_h = kept.cpu().numpy().reshape(B * H, n_keep)
    tok = []
    for row in kept_h:
        ctx = sum(min(cfg.block, cfg.N_ctx - c * cfg.block) for c in row)
        tok.append(cfg.N_src + ctx)
    T_mean = float(np.mean(tok))
    wm = work_model(cfg, T_mean)

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        # wait by polling (sleep releases the GIL) so the sampler thread runs
        # while the GPU works; a blocking synchronize here starves it
        while not t1.query():
            time.sleep(2e-4)
        torch.cuda.synchronize()
    barrier()
    ms = t0.elapsed_time(t1) / args.steps
    stage_ms = np.array([[stage_ev[i][j].elapsed_time(stage_ev[i][j + 1]) for j in range(3)]
                         for i in range(args.steps)]).mean(axis=0)
    ms_max = max_over_ranks(ms, dev)
    assert api.isa_read_device_status(ws) == 0

    # the same step captured once in a CUDA graph and replayed (the launch
    # sequence without host calls between kernels); reported beside `value`
    graph_ms = None
    if not args.no_graph:
        gs = torch.cuda.Stream()
        gs.wait_stream(stream)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            api.isa_preselect_ctx(q, k, v, shape, ws, kept=kept, want_saliency=False, stream=gs)
            api.isa_route_taylor_fwd(q, kept, shape, ws, out, routed=routed, taylor=taylor, want_sharpness=False,
                                     stream=gs)
            api.isa_full_attn_fwd(q, k, v, kept, routed, shape, ws, out, stream=gs)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        graph_ms = max_over_ranks(g0.elapsed_time(g1) / args.steps, dev)
        assert api.isa_read_device_status(ws) == 0
        del graph

    # in-house dense kernel on the same inputs (the baseline the metric names)
    dense_ms = None
    if not args.no_dense:
        dws = api.dense_workspace(cfg.d, dev)
        dout = torch.empty_like(q)
        nd = max(2, min(args.steps, 5))
        for _ in range(2):
            api.isa_dense_attn_fwd(q, k, v, out=dout, ws=dws)
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for _ in range(nd):
            api.isa_dense_attn_fwd(q, k, v, out=dout, ws=dws)
        d1.record(stream)
        torch.cuda.synchronize()
        dense_ms = max_over_ranks(d0.elapsed_time(d1) / nd, dev)
        assert api.isa_read_device_status(dws) == 0
        del dout

    # end to end through the public API with host buffers: the C entry point
    # isa_forward_host (copies in, forward, copy out, pipelined over head
    # slices), every step a whole call that returns once the output is in
    # pinned host memory
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (to_torch_bf16(b).pin_memory() for b in bits)
        hout = torch.empty(q.shape, dtype=q.dtype).pin_memory()
        staging = torch.empty(api.host_staging_size(shape), dtype=torch.uint8, device=dev)
        for _ in range(2):
            api.isa_forward(hq, hk, hv, cfg.N_src, cfg.block, cfg.keep, cfg.rho, out=hout, staging=staging)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ne = args.steps
        e0.record(stream)
        for _ in range(ne):
            api.isa_forward(hq, hk, hv, cfg.N_src, cfg.block, cfg.keep, cfg.rho, out=hout, staging=staging)
        e1.record(stream)
        torch.cuda.synchronize()
        assert api.isa_read_device_status(staging) == 0
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / ne, dev)
        e2e = {"value": round(e2e_ms, 3), "unit": "ms", "h2d_bytes_per_step": 3 * q.numel() * 2,
               "d2h_bytes_per_step": q.numel() * 2, "steps": ne,
               "path": "isa_forward_host (C ABI), pinned host buffers, default head slices"}

    gather_ms = None
    if args.shard == "heads" and args.gather and world > 1:
        from sparse_attention_context_b200.sharding import gather_heads

        full = gather_heads(out)
        assert full.shape[1] == cfg_job.H
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            gather_heads(out)
        g1.record(stream)
        torch.cuda.synchronize()
        gather_ms = max_over_ranks(g0.elapsed_time(g1) / args.steps, dev)
        del full

    pk, pk_kind = peaks()
    full_ms = float(stage_ms[2])
    ach = wm["full_flops"] / (full_ms * 1e-3) / 1e12
    roof = {"kernel": "routed full attention (attn2_kernel<128,128,FULL>)", "bound": "tensor",
            "achieved": round(ach, 1), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(ach / pk["bf16_tflops"], 4), "peak_kind": f"{pk_kind} burst bf16",
            "frac_of_sustained": round(ach / pk["bf16_tflops_sustained"], 4),
            "traffic": full_traffic(args), "algorithmic_bytes": int(wm["full_bytes"]),
            "kernel_ms": round(full_ms, 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # bounded sample: whole heads until ~10 s of CPU work (at most all heads)
        heads, secs, per_head = [], 0.0, []
        while secs < 10.0 and len(heads) < cfg.H:
            h = (len(heads) * 7) % cfg.H
            _, s1 = cpu_oracle_ms_per_step(cfg, [h])
            heads.append(h)
            per_head.append(s1)
            secs += s1
        cms = 1e3 * float(np.mean(per_head)) * cfg.B * cfg.H
        cpu = {"value": round(cms, 1), "unit": "ms", "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"{len(heads)} of {cfg.B * cfg.H} heads ({secs:.1f} s of CPU work), "
                         f"scaled x{cfg.B * cfg.H / len(heads):g}"}

    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    # pre-selection: pooling, saliency, selection, and the value means of the
    # kept context blocks; sharpness + Taylor: operand build, fused pass, route
    launches_per_step = 3 + (1 if n_keep > 0 else 0) + 3 + full_stage_launches(cfg, n_keep, n_route, nsm)
    if rank == 0:
        rec = {"metric": METRIC, "value": round(ms_max, 4), "unit": "ms", "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "higher_is_better": False,
               "scaling": "strong" if args.shard == "heads" else "weak", "vs_baseline": None, "dtype": "bf16",
               "data": "synthetic", "config": config_dict(cfg_job, world, args.shard),
               "eff_tflops": round(work_model(cfg_job, T_mean)["dense_flops"] / (ms_max * 1e-3) / 1e12, 1),
               "dense_ms": None if dense_ms is None else round(dense_ms, 4),
               "isa_over_dense": None if dense_ms is None else round(ms_max / dense_ms, 4),
               "dense_tflops": None if dense_ms is None else round(wm["dense_flops"] / (dense_ms * 1e-3) / 1e12, 1),
               "stage_ms": {"preselect": round(float(stage_ms[0]), 4),
                            "sharpness_taylor_route": round(float(stage_ms[1]), 4),
                            "full_attn": round(float(stage_ms[2]), 4)},
               "executed_tflop": round((wm["full_flops"] + wm["fused_flops"]) / 1e12, 4),
               "graph_ms": None if graph_ms is None else round(graph_ms, 4),
               "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
               "gpu_launches": launches_per_step * args.steps, "clocks": clk.summary()}
        if gather_ms is not None:
            rec["gather_ms"] = round(gather_ms, 4)
        print(json.dumps(rec), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
