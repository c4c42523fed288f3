#!/usr/bin/env python3
"""BitLinear forward throughput on B200: one JSON line on rank 0.

A step is one pass of the per-token hot path over one batch of synthetic
input: for every layer of the workload, the forward on weights packed
beforehand (per-token INT8 quantization, ternary x INT8 product,
dequantization: steps 4-6), through the C ABI of libbitlinear.so.  Weight
preparation (absmean, ternarize + pack: steps 1-3) is offline -- done once per
weight matrix, not per token -- and is timed on its own as a secondary section
(``--phase all`` puts it back into every step).

Timing: W untimed warm-up steps; then exactly K steps captured into one CUDA
graph with CUDA events at its two ends, replayed once untimed and once timed
between barrier + synchronize on both sides; the device time is the max over
ranks.  The packed weights are rotated over enough copies to exceed 4x L2 (the
fp32 latent weights of ``--phase all`` exceed L2 on their own).  Multi-GPU:
one process per GPU (torchrun), every rank runs its own independent replica of
the workload (weak scaling).

``--impl reference`` times the CPU oracle instead (rank 0 only), each step a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "BitLinear GB/s (decode GEMV) & INT8 TOPS (prefill) vs roofline, 1×B200"
FALLBACK_HBM_GBS = 6650.0

# workload name -> layers (N, K), tokens M, packed format, activation dtype
WORKLOADS = {
    "3b_decode": dict(desc="3B-shaped decode GEMV: M=1, up K=3200->N=8640 and down K=8640->N=3200, "
                           "fp32 latent W N(0,0.02), bf16 x N(0,1), 2-bit pack, bf16 y",
                      layers=[(8640, 3200), (3200, 8640)], M=1, fmt=0, sigma=0.02, seed=2),
    "3b_decode_t5": dict(desc="3B-shaped decode GEMV, base-3 (5 trits/byte) pack",
                         layers=[(8640, 3200), (3200, 8640)], M=1, fmt=1, sigma=0.02, seed=2),
    "70b_decode": dict(desc="70B-shaped layer decode: M=1, K=8192->N=28672 and K=28672->N=8192, "
                            "fp32 latent W N(0,0.01), bf16 x, 2-bit pack",
                       layers=[(28672, 8192), (8192, 28672)], M=1, fmt=0, sigma=0.01, seed=5),
    "70b_decode_t5": dict(desc="70B-shaped layer decode, base-3 pack",
                          layers=[(28672, 8192), (8192, 28672)], M=1, fmt=1, sigma=0.01, seed=5),
}


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

KERNEL_SOURCE = {"absmean_kernel": "bl_weights.cu", "ternarize_flat_kernel": "bl_weights.cu",
                 "binarize_pack_kernel": "bl_weights.cu",
                 "ternarize_pack_kernel": "bl_weights.cu", "gemv_i2_kernel": "bl_gemv.cu", "gemv1_i2_kernel": "bl_gemv1.cu", "gemv1_t5_kernel": "bl_gemv1.cu", "gemv1_b1_kernel": "bl_gemv1.cu",
                 "gemv_kernel": "bl_gemv.cu", "gemv_t5_kernel": "bl_gemv.cu", "gemv_i2_mt_kernel": "bl_gemv.cu", "act_quant_row_kernel": "bl_acts.cu",
                 "act_quant_kernel": "bl_acts.cu", "ln_quant_kernel": "bl_acts.cu", "ln_quant_reg_kernel": "bl_acts.cu", "gemm_i2_2sm_kernel": "bl_gemm_sm100.cu",
                 "gemm_i2_kernel": "bl_gemm_sm100.cu", "b1_to_i2_kernel": "bl_gemm_sm100.cu",
                 "t5_to_i2_kernel": "bl_gemm_sm100.cu", "splitk_reduce_kernel": "bl_gemm_sm100.cu",
                 "pack_kernel": "bl_weights.cu",
                 "backward_dx_tile_kernel": "bl_backward.cu", "backward_dx_reduce_kernel": "bl_backward.cu",
                 "backward_dw_kernel": "bl_backward.cu", "backward_dw1_kernel": "bl_backward.cu"}


def csrc_digest(kernel: str | None = None) -> str:
    """Digest of the sources a kernel is built from (its .cu file and the
    shared headers), or of every source when no kernel is named."""
    csrc = os.path.join(ROOT, "bitlinear_b1_fwd_b200", "csrc")
    if kernel is None:
        files = sorted(glob.glob(os.path.join(csrc, "*")))
    else:
        files = sorted([os.path.join(csrc, KERNEL_SOURCE[kernel])] + glob.glob(os.path.join(csrc, "*.cuh")) +
                       glob.glob(os.path.join(csrc, "*.h")))
    h = hashlib.sha256()
    for p in files:
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode() + f.read())
    return h.hexdigest()[:16]


FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0  # nominal dense ratio: 4.5 PFLOP/s int8 : 2.25 bf16


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_int8_peak():
    """int8 dense peak = the measured bf16 burst peak x the nominal int8 : bf16 ratio."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]) * INT8_PER_BF16, "measured bf16 burst x 2"
    except Exception:
        return FALLBACK_BF16_TFLOPS * INT8_PER_BF16, "fallback bf16 x 2"


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    digest = csrc_digest(kernel)
    for p in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        kv = {}
        with open(p) as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    kv[k.strip()] = v.strip().strip("`")
        if kv.get("kernel") == kernel and kv.get("workload") == workload and kv.get("csrc_sha256") == digest:
            try:
                return int(kv["dram_bytes_per_launch"])
            except (KeyError, ValueError):
                return None
    return None


def nvml_handle_of(nv, props, device_index: int):
    """NVML handle of the CUDA device with properties `props`.  NVML numbers
    every GPU of the machine in PCI order and ignores CUDA_VISIBLE_DEVICES,
    while CUDA numbers the visible GPUs in its own order, so the device is
    found by its PCI location; the CUDA index is the fallback."""
    try:
        want = (int(props.pci_domain_id), int(props.pci_bus_id), int(props.pci_device_id))
        count = nv.nvmlDeviceGetCount()
    except Exception:
        return nv.nvmlDeviceGetHandleByIndex(device_index)
    for i in range(count):
        try:  # a GPU this process may not query is skipped
            h = nv.nvmlDeviceGetHandleByIndex(i)
            pi = nv.nvmlDeviceGetPciInfo(h)
            if (int(pi.domain), int(pi.bus), int(pi.device)) == want:
                return h
        except Exception:
            continue
    return nv.nvmlDeviceGetHandleByIndex(device_index)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running (every
    0.2 ms: the timed graphs of short workloads last about a millisecond)."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.0002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop, self._t = period_s, threading.Event(), None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                props = torch.cuda.get_device_properties(device_index)
            except Exception:
                props = None
            self.h = nvml_handle_of(pynvml, props, device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# multi-rank plumbing (one process per GPU; weak scaling over replicas)
# ----------------------------------------------------------------------------

def rank_seed_offset(rank: int) -> int:
    """Each rank draws its own replica of the workload."""
    return 10000 * rank


def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's time (all ranks take part; identity for one rank)."""
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(step_bytes: int, world: int, ms_per_step: float) -> float:
    """Aggregate GB/s: the bytes every rank processed in one step over the step time."""
    return step_bytes * world / (ms_per_step * 1e-3) / 1e9


# ----------------------------------------------------------------------------
# algorithmic bytes per launch (the unit of work of each kernel)
# ----------------------------------------------------------------------------

def layer_bytes(N, K, M, rb, w_es=4, x_es=2, y_es=2):
    absmean = N * K * w_es + 4
    ternarize = N * K * w_es + N * rb + 4
    forward = N * rb + M * K * x_es + M * N * y_es + 4 * M + 4
    return dict(absmean=absmean, ternarize_pack=ternarize, forward=forward)


# ----------------------------------------------------------------------------
# CPU oracle timing (the baseline and the reference arm)
# ----------------------------------------------------------------------------

def oracle_layer_inputs(wl, phase, rows_frac=1.0):
    """Seeded inputs of the workload's layers (the first rows_frac of each
    layer's weight rows); for ``phase == "forward"`` the weights are also
    quantized and packed here, outside any timed region (offline work)."""
    import oracle
    from bitlinear_b1_fwd_b200 import synth
    out = []
    for i, (N, K) in enumerate(wl["layers"]):
        n = max(1, int(N * rows_frac))
        W = synth.normal_f32(1000 + wl["seed"] + 100 * i, (N, K), wl["sigma"])[:n]
        x = synth.to_bf16_bits(synth.normal_f32(2000 + wl["seed"] + 100 * i, (wl["M"], K)))
        L = dict(W=W, x=x)
        if phase == "forward":
            L["g"] = oracle.gamma(W)
            L["packed"] = oracle.pack(oracle.ternarize(W, L["g"]), wl["fmt"])
        out.append(L)
    return out


def oracle_step(orc, wl, inputs, phase):
    """One oracle pass over the inputs; returns the algorithmic bytes processed."""
    total = 0
    for L in inputs:
        n, K = L["W"].shape
        rb = orc.packed_row_bytes(K, wl["fmt"])
        b = layer_bytes(n, K, wl["M"], rb)
        if phase == "all":
            g = orc.gamma(L["W"])
            packed = orc.pack(orc.ternarize(L["W"], g), wl["fmt"])
        else:
            g, packed = L["g"], L["packed"]
        orc.forward(packed, wl["fmt"], g, n, K, L["x"], ydt=orc.BF16)
        total += b["forward"] + (b["absmean"] + b["ternarize_pack"] if phase == "all" else 0)
    return total


def host_cpu():
    """The host's logical core count and CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


def time_oracle(wl, phase, budget_s, min_steps=1, rows_frac=1.0):
    import oracle
    oracle.build()
    inputs = oracle_layer_inputs(wl, phase, rows_frac)
    steps, nbytes, t0 = 0, 0, time.perf_counter()
    while steps < min_steps or time.perf_counter() - t0 < budget_s:
        nbytes += oracle_step(oracle, wl, inputs, phase)
        steps += 1
    dt = time.perf_counter() - t0
    return nbytes / dt / 1e9, steps, dt


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def graph_ms(stream, steps, body, sampler=None, world=1):
    """Device time (ms) of ``steps`` calls of ``body(i)`` captured into one CUDA
    graph, with CUDA events only at its two ends (events between the kernels
    would add their own cost to every launch).  One untimed replay first; the
    timed replay is bracketed by barrier + synchronize on both sides."""
    import contextlib
    import torch
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        e0.record(stream)
        for i in range(steps):
            body(i)
        e1.record(stream)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with (sampler if sampler is not None else contextlib.nullcontext()):
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = e0.elapsed_time(e1)
    del g
    return ms


def run_gpu(args, wl, rank, world, local_rank):
    import numpy as np
    import torch

    from bitlinear_b1_fwd_b200 import binding as B
    from bitlinear_b1_fwd_b200 import build as libbuild
    from bitlinear_b1_fwd_b200 import synth

    if rank == 0:
        libbuild.build()
    if world > 1:
        torch.distributed.barrier()
    B.lib()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    fmt, M = wl["fmt"], wl["M"]
    rank_seed = rank_seed_offset(rank)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    # every layer's tokens and outputs sit in one device buffer each (and one
    # pinned host buffer each), at 256-byte offsets, so the end-to-end step
    # moves them with one copy each way
    def offsets(sizes):
        offs, o = [], 0
        for n in sizes:
            offs.append(o)
            o += -(-n // 128) * 128  # bf16 elements: 256-byte steps
        return offs, o
    x_offs, x_tot = offsets([M * K for (_, K) in wl["layers"]])
    y_offs, y_tot = offsets([M * N for (N, _) in wl["layers"]])
    xs_dev = torch.zeros(x_tot, dtype=torch.bfloat16, device=dev)
    ys_dev = torch.zeros(y_tot, dtype=torch.bfloat16, device=dev)
    xs_host = torch.zeros(x_tot, dtype=torch.bfloat16).pin_memory()
    ys_host = torch.zeros(y_tot, dtype=torch.bfloat16).pin_memory()
    layers = []
    for i, (N, K) in enumerate(wl["layers"]):
        Wh = synth.normal_f32(1000 + wl["seed"] + 100 * i + rank_seed, (N, K), wl["sigma"])
        xh = synth.to_bf16_bits(synth.normal_f32(2000 + wl["seed"] + 100 * i + rank_seed, (M, K)))
        rb = B.bitlinear_packed_row_bytes(K, fmt)
        L = dict(N=N, K=K, rb=rb)
        L["W"] = torch.from_numpy(Wh).to(dev)
        L["x_host"] = xs_host[x_offs[i]:x_offs[i] + M * K].view(M, K)
        L["x_host"].copy_(torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).view(M, K))
        L["x"] = xs_dev[x_offs[i]:x_offs[i] + M * K].view(M, K)
        L["x"].copy_(L["x_host"])
        if args.phase == "all":  # the step copies the latent weights from the host too
            L["W_host"] = torch.from_numpy(Wh).pin_memory()
        L["gamma"] = torch.empty(1, dtype=torch.float32, device=dev)
        L["ws"] = torch.zeros(B.bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
        L["packed"] = torch.empty((N, rb), dtype=torch.uint8, device=dev)
        L["scale"] = torch.empty(M, dtype=torch.float32, device=dev)
        L["y"] = ys_dev[y_offs[i]:y_offs[i] + M * N].view(M, N)
        L["y_host"] = ys_host[y_offs[i]:y_offs[i] + M * N].view(M, N)
        L["fws"] = torch.zeros(B.bitlinear_forward_workspace_bytes(M, N, K, fmt, B.BL_BF16),
                               dtype=torch.uint8, device=dev)
        L["bytes"] = layer_bytes(N, K, M, rb)
        layers.append(L)
        del Wh

    stream = torch.cuda.Stream(device=dev)
    eps = 1e-5

    # weight preparation once (offline work), then copies of the packed
    # weights rotated so that consecutive steps read more than 4x L2
    with torch.cuda.stream(stream):
        for L in layers:
            B.bitlinear_quantize_weights(L["W"], eps, fmt, L["packed"], None, L["gamma"], L["ws"], stream)
    stream.synchronize()
    packed_bytes = sum(L["N"] * L["rb"] for L in layers)
    rot = max(2, -(-4 * l2 // packed_bytes))
    for L in layers:
        L["copies"] = [L["packed"]] + [L["packed"].clone() for _ in range(rot - 1)]

    ops = ["absmean", "ternarize_pack", "forward"] if args.phase == "all" else ["forward"]

    def run_op(op, L, i):
        if op == "absmean":
            B.bitlinear_absmean(L["W"], L["gamma"], L["ws"], stream)
        elif op == "ternarize_pack":
            B.bitlinear_ternarize_pack(L["W"], L["gamma"], eps, fmt, L["packed"], None, stream)
        else:
            packed = L["packed"] if args.phase == "all" else L["copies"][i % rot]
            B.bitlinear_forward(packed, fmt, L["gamma"], L["N"], L["K"], L["x"], L["scale"], L["y"],
                                L["fws"], stream)

    def step(i):
        for L in layers:
            for op in ops:
                run_op(op, L, i)

    # warm-up (eager), then the K timed steps as one graph
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    sampler = ClockSampler(local_rank)
    ms = graph_ms(stream, args.steps, step, sampler=sampler, world=world)
    for L in layers:
        st = B.bitlinear_device_status(L["fws"], stream)
        if st != B.BL_OK:
            raise RuntimeError(f"device status {B.status_string(st)}")

    # each op's average launch duration: a graph of K steps of that call alone
    # over every layer in turn (the inputs of consecutive launches together
    # exceed L2), timed at its two ends; the offline weight preparation is
    # timed this way in every run
    per_op_ms = {}
    for op in ("absmean", "ternarize_pack", "forward"):
        if op == "forward" and ops == ["forward"]:
            per_op_ms[op] = ms / (args.steps * len(layers))
            continue
        t = graph_ms(stream, args.steps, lambda i, op=op: [run_op(op, L, i) for L in layers])
        per_op_ms[op] = t / (args.steps * len(layers))
    step_bytes = sum(sum(L["bytes"][op] for op in ops) for L in layers)

    ms_max = max_over_ranks(ms, world, dev)

    # ---- end to end through the public API: each step copies its token(s)
    # (and, for --phase all, the latent weights) from pinned host memory and
    # reads y back ----
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    h2d = sum(L["W_host"].numel() * 4 for L in layers) if args.phase == "all" else 0
    h2d += xs_host.numel() * 2
    d2h = ys_host.numel() * 2
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e2e_steps):
            if args.phase == "all":
                for L in layers:
                    L["W"].copy_(L["W_host"], non_blocking=True)
            xs_dev.copy_(xs_host, non_blocking=True)  # every layer's tokens, one copy
            step(i)
            ys_host.copy_(ys_dev, non_blocking=True)  # every layer's outputs, one copy
        e1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)

    prefill = run_prefill(args, dev, stream, rank_seed, l2) if args.prefill else None
    decode = run_decode(args, dev, stream, rank_seed, l2) if args.decode else None
    sweep = run_sweep(args, dev, stream, l2) if args.sweep else None
    backward = run_backward(args, dev, stream, rank_seed, l2) if args.decode else None
    res = dict(prefill=prefill, decode=decode, sweep=sweep, backward=backward, ms_total=ms_max, per_op_ms=per_op_ms,
               step_bytes=step_bytes, layers=layers, ops=ops,
               clocks=sampler.summary(), e2e_ms=e2e_ms, e2e_steps=e2e_steps, h2d=h2d, d2h=d2h,
               rot=rot, l2=l2, launches_per_step=len(layers) * len(ops))
    return res


def run_prefill(args, dev, stream, rank_seed, l2):
    """3B prefill layer (M=4096, K=3200 -> N=8640, 2-bit): per-token INT8
    quantization and the tensor-core product timed separately (CUDA events in
    one graph), inputs rotated over copies that together exceed L2."""
    import numpy as np
    import torch

    from bitlinear_b1_fwd_b200 import binding as B
    from bitlinear_b1_fwd_b200 import synth

    M, K, N = 4096, 3200, 8640
    Wh, xh = synth.prefill_3b_inputs()
    if rank_seed:
        Wh = synth.normal_f32(1003 + rank_seed, (N, K), 0.02)
    rb = B.bitlinear_packed_row_bytes(K, 0)
    W = torch.from_numpy(Wh).to(dev)
    x0 = torch.from_numpy(xh.view(np.int16)).to(dev).view(torch.bfloat16)
    gamma = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.zeros(B.bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
    packed0 = torch.empty((N, rb), dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        B.bitlinear_quantize_weights(W, 1e-5, 0, packed0, None, gamma, ws, stream)
    stream.synchronize()
    del W
    per_copy = M * K * 2 + M * K + N * rb + M * N * 2
    rot = max(2, -(-2 * l2 // per_copy))
    xs = [x0] + [x0.clone() for _ in range(rot - 1)]
    pk = [packed0] + [packed0.clone() for _ in range(rot - 1)]
    xq = [torch.empty((M, K), dtype=torch.int8, device=dev) for _ in range(rot)]
    sc = [torch.empty(M, dtype=torch.float32, device=dev) for _ in range(rot)]
    ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(rot)]
    fws = torch.zeros(B.bitlinear_forward_workspace_bytes(M, N, K, 0, B.BL_I8), dtype=torch.uint8, device=dev)

    def act(i):
        r = i % rot
        B.bitlinear_quantize_acts(xs[r], xq[r], sc[r], stream)

    def gemm(i):
        r = i % rot
        B.bitlinear_forward(pk[r], 0, gamma, N, K, xq[r], sc[r], ys[r], fws, stream)

    # pre-norm variant of step 4: LayerNorm of each token, then INT8 (seeded N(1, 0.1) / N(0, 0.1) parameters)
    ln_w = torch.from_numpy(synth.normal_f32(95, (K,), 0.1) + np.float32(1.0)).to(dev)
    ln_b = torch.from_numpy(synth.normal_f32(96, (K,), 0.1)).to(dev)

    def lnq(i):
        r = i % rot
        B.bitlinear_layernorm_quantize_acts(xs[r], ln_w, ln_b, 1e-5, xq[r], sc[r], None, stream)

    steps = max(1, args.prefill_steps)
    with torch.cuda.stream(stream):
        for i in range(3):
            lnq(i)
            act(i)
            gemm(i)
    stream.synchronize()
    # each call timed as a graph of `steps` launches of it alone (rotating inputs)
    ln_ms = graph_ms(stream, steps, lnq) / steps
    act_ms = graph_ms(stream, steps, act) / steps
    gemm_ms = graph_ms(stream, steps, gemm) / steps
    st = B.bitlinear_device_status(fws, stream)
    if st != B.BL_OK:
        raise RuntimeError(f"prefill device status {B.status_string(st)}")
    ops = 2.0 * M * N * K
    return dict(M=M, K=K, N=N, act_ms=act_ms, gemm_ms=gemm_ms, ops=ops, rot=rot, steps=steps,
                act_bytes=M * K * 2 + M * K + 4 * M, ln_ms=ln_ms, ln_bytes=M * K * 2 + 2 * K * 4 + M * K + 4 * M)


DECODE_SHAPES = {"3b": ("3b_decode", "3B decode: M=1, K=3200->N=8640 and K=8640->N=3200"),
                 "70b": ("70b_decode", "70B decode: M=1, K=8192->N=28672 and K=28672->N=8192")}


def run_decode(args, dev, stream, rank_seed, l2):
    """Decode GEMV alone (steps 4-6, M=1) on weights packed beforehand, for the
    3B and 70B layer shapes, 2-bit, base-3 and 1-bit (the 1-bit BitNet variant,
    weights from bitlinear_binarize_weights): a graph of ``decode_steps``
    forward calls per layer over packed copies rotated so that consecutive reads
    exceed 4x L2, timed at its two ends.  Per layer: average launch duration,
    GB/s of algorithmic bytes and the fraction of the HBM peak."""
    import numpy as np
    import torch

    from bitlinear_b1_fwd_b200 import binding as B
    from bitlinear_b1_fwd_b200 import synth

    out = {}
    for key, (wname, desc) in DECODE_SHAPES.items():
        wl = WORKLOADS[wname]
        for fmt in (0, 1, 2):
            rows = []
            for i, (N, K) in enumerate(wl["layers"]):
                Wh = synth.normal_f32(1000 + wl["seed"] + 100 * i + rank_seed, (N, K), wl["sigma"])
                xh = synth.to_bf16_bits(synth.normal_f32(2000 + wl["seed"] + 100 * i + rank_seed, (1, K)))
                rb = B.bitlinear_packed_row_bytes(K, fmt)
                W = torch.from_numpy(Wh).to(dev)
                del Wh
                gamma = torch.empty(1, dtype=torch.float32, device=dev)
                p0 = torch.empty((N, rb), dtype=torch.uint8, device=dev)
                if fmt == B.BL_PACK_B1:
                    ws = torch.zeros(B.bitlinear_binarize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
                    alpha = torch.empty(1, dtype=torch.float32, device=dev)
                    with torch.cuda.stream(stream):
                        B.bitlinear_binarize_weights(W, p0, None, gamma, alpha, ws, stream)
                else:
                    ws = torch.zeros(B.bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
                    with torch.cuda.stream(stream):
                        B.bitlinear_quantize_weights(W, 1e-5, fmt, p0, None, gamma, ws, stream)
                stream.synchronize()
                del W
                rot = max(2, -(-4 * l2 // (N * rb)))
                copies = [p0] + [p0.clone() for _ in range(rot - 1)]
                x = torch.from_numpy(xh.view(np.int16)).to(dev).view(torch.bfloat16)
                y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
                scale = torch.empty(1, dtype=torch.float32, device=dev)
                fws = torch.zeros(B.bitlinear_forward_workspace_bytes(1, N, K, fmt, B.BL_BF16), dtype=torch.uint8,
                                  device=dev)

                def fwd(j, copies=copies, gamma=gamma, N=N, K=K, x=x, scale=scale, y=y, fws=fws, fmt=fmt):
                    B.bitlinear_forward(copies[j % len(copies)], fmt, gamma, N, K, x, scale, y, fws, stream)

                with torch.cuda.stream(stream):
                    for j in range(3):
                        fwd(j)
                steps = max(1, args.decode_steps)
                us = graph_ms(stream, steps, fwd) / steps * 1e3
                st = B.bitlinear_device_status(fws, stream)
                if st != B.BL_OK:
                    raise RuntimeError(f"decode device status {B.status_string(st)}")
                nbytes = layer_bytes(N, K, 1, rb)["forward"]
                rows.append(dict(N=N, K=K, us=us, bytes=nbytes, rot=rot))
                del copies, p0
            out[f"{key}_{['2bit', 'base3', '1bit'][fmt]}"] = dict(desc=desc, rows=rows)
    return out


def run_backward(args, dev, stream, rank_seed, l2):
    """STE backward for one token on the 3B decode layers (2-bit): dx reads the
    packed weights (plus dy) and writes dx; dW reads dy and x_q and writes N K
    fp32.  Each call alone in a graph of back-to-back launches, packed copies
    and dW outputs rotated past 4x L2; GB/s of the algorithmic bytes."""
    import torch

    from bitlinear_b1_fwd_b200 import binding as B

    peak, kind = measured_peaks()
    wl = WORKLOADS["3b_decode"]
    g = torch.Generator(device=dev)
    out = []
    for i, (N, K) in enumerate(wl["layers"]):
        g.manual_seed(3000 + 100 * i + rank_seed)
        W = torch.randn(N, K, generator=g, device=dev) * wl["sigma"]
        rb = B.bitlinear_packed_row_bytes(K, 0)
        p0 = torch.empty((N, rb), dtype=torch.uint8, device=dev)
        gamma = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.zeros(B.bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
        with torch.cuda.stream(stream):
            B.bitlinear_quantize_weights(W, 1e-5, 0, p0, None, gamma, ws, stream)
        stream.synchronize()
        del W
        rot = max(2, -(-4 * l2 // (N * rb)))
        copies = [p0] + [p0.clone() for _ in range(rot - 1)]
        dy = (torch.randn(1, N, generator=g, device=dev) * 1e-3).to(torch.bfloat16)
        xq = torch.randint(-127, 128, (1, K), generator=g, device=dev, dtype=torch.int8)
        sc = torch.rand(1, generator=g, device=dev) + 0.5
        dx = torch.empty((1, K), dtype=torch.float32, device=dev)
        dws = torch.zeros(B.bitlinear_backward_dx_workspace_bytes(1, N, K, 0), dtype=torch.uint8, device=dev)
        rot_w = max(2, -(-4 * l2 // (N * K * 4)))
        dw = [torch.empty((N, K), dtype=torch.float32, device=dev) for _ in range(rot_w)]

        def f_dx(j, copies=copies, gamma=gamma, N=N, K=K, dy=dy, dx=dx, dws=dws):
            B.bitlinear_backward_dx(copies[j % len(copies)], 0, gamma, N, K, dy, dx, dws, stream)

        def f_dw(j, dy=dy, xq=xq, sc=sc, gamma=gamma, dw=dw):
            B.bitlinear_backward_dw(dy, xq, sc, gamma, dw[j % len(dw)], stream)

        steps = max(1, args.decode_steps // 4)
        res = {"N": N, "K": K}
        for name, fn, nbytes in (("dx", f_dx, N * rb + 2 * N + 4 * K + 4),
                                 ("dw", f_dw, 4 * N * K + 2 * N + K + 8)):
            with torch.cuda.stream(stream):
                for j in range(3):
                    fn(j)
            us = graph_ms(stream, steps, fn) / steps * 1e3
            res[name] = {"us": us, "bytes": nbytes, "GB_s": nbytes / (us * 1e-6) / 1e9,
                         "frac_of_hbm": nbytes / (us * 1e-6) / 1e9 / peak}
        if B.bitlinear_device_status(dws, stream) != B.BL_OK:
            raise RuntimeError("backward device status")
        out.append(res)
        del copies, p0, dw
    return {"workload": "3B decode layers, one bf16 gradient token, 2-bit weights", "peak": peak, "peak_kind": kind,
            "layers": out, "note": "fp64 sums in a fixed order, fp32 out; bytes: dx = packed + dy + dx, "
                                   "dw = N K fp32 + dy + x_q"}


def run_sweep(args, dev, stream, l2):
    """Config sweeps (opt-in): the 70B layers (2-bit) over M = 1, 2, 4, ..., 8192
    and the 3B block's six BitLinears (Q, K, V, O, up, down, each with its
    own per-token quantization) as one graph per block at M = 1, 16, 128, 1024,
    and the same block with Q, K and V as one grouped call on a shared input.
    Latent weights N(0, sigma) and bf16 tokens N(0, 1) are drawn on the device
    with a seeded generator (parity on the host-generated recipe is the tests'
    job); packed weights and tokens rotate over copies past 4x L2 where they
    fit.  Each point: a graph of back-to-back calls timed at its two ends."""
    import torch

    from bitlinear_b1_fwd_b200 import binding as B
    from bitlinear_b1_fwd_b200 import synth

    peak_gbs, _ = measured_peaks()
    peak_tops, _ = measured_int8_peak()
    g = torch.Generator(device=dev)

    def prep(N, K, sigma, seed):
        g.manual_seed(seed)
        W = torch.randn(N, K, generator=g, device=dev) * sigma
        rb = B.bitlinear_packed_row_bytes(K, 0)
        packed = torch.empty((N, rb), dtype=torch.uint8, device=dev)
        gamma = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.zeros(B.bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
        with torch.cuda.stream(stream):
            B.bitlinear_quantize_weights(W, 1e-5, 0, packed, None, gamma, ws, stream)
        stream.synchronize()
        return packed, gamma, rb

    def point(N, K, M, rb, us):
        nbytes = N * rb + M * K * 2 + M * N * 2 + 4 * M + 4
        ops = 2.0 * M * N * K
        gbs = nbytes / (us * 1e-6) / 1e9
        tops = ops / (us * 1e-6) / 1e12
        kern = gemv_kernel_name(0, [(N, K)], M) if M <= 4 else gemm_kernel_name(M)
        return {"M": M, "us": us, "GB_s": gbs, "frac_of_hbm": gbs / peak_gbs, "TOPS": tops,
                "frac_of_int8": tops / peak_tops, "kernel": kern}

    out = {"layer_70b": {}, "block_3b": [], "block_3b_fused_qkv": []}
    for li, c in enumerate(synth.LAYER_70B):
        N, K = c["N"], c["K"]
        p0, gamma, rb = prep(N, K, c["w_sigma"], 1005 + 100 * li)
        pk = [p0] + [p0.clone() for _ in range(max(0, -(-4 * l2 // (N * rb)) - 1))]
        pts = []
        for M in synth.LAYER_70B_M:
            xr = max(1, min(4, -(-4 * l2 // (M * K * 2))))
            g.manual_seed(2005 + 100 * li + M)
            xs = [torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16) for _ in range(xr)]
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            sc = torch.empty(M, dtype=torch.float32, device=dev)
            fws = torch.zeros(B.bitlinear_forward_workspace_bytes(M, N, K, 0, B.BL_BF16), dtype=torch.uint8,
                              device=dev)

            def fwd(j, M=M, xs=xs, y=y, sc=sc, fws=fws):
                B.bitlinear_forward(pk[j % len(pk)], 0, gamma, N, K, xs[j % len(xs)], sc, y, fws, stream)

            with torch.cuda.stream(stream):
                for j in range(3):
                    fwd(j)
            steps = 100 if M <= 16 else (30 if M <= 512 else 6)
            us = graph_ms(stream, steps, fwd) / steps * 1e3
            if B.bitlinear_device_status(fws, stream) != B.BL_OK:
                raise RuntimeError("sweep device status")
            pts.append(point(N, K, M, rb, us))
            del xs, y, fws
        out["layer_70b"][c["name"]] = {"N": N, "K": K, "points": pts}
        del pk, p0
    blk = [prep(c["N"], c["K"], 0.02, 1004 + 100 * i) for i, c in enumerate(synth.BLOCK_3B)]
    blk_bytes = sum(c["N"] * rb for c, (_, _, rb) in zip(synth.BLOCK_3B, blk))
    rot = max(1, -(-4 * l2 // blk_bytes))
    copies = [[p] + [p.clone() for _ in range(rot - 1)] for (p, _, _) in blk]
    for M in synth.BLOCK_3B_M:
        g.manual_seed(2004 + M)
        xs = [torch.randn(M, c["K"], generator=g, device=dev).to(torch.bfloat16) for c in synth.BLOCK_3B]
        ys = [torch.empty((M, c["N"]), dtype=torch.bfloat16, device=dev) for c in synth.BLOCK_3B]
        scs = [torch.empty(M, dtype=torch.float32, device=dev) for _ in synth.BLOCK_3B]
        fwss = [torch.zeros(B.bitlinear_forward_workspace_bytes(M, c["N"], c["K"], 0, B.BL_BF16),
                            dtype=torch.uint8, device=dev) for c in synth.BLOCK_3B]

        def block(j, M=M, xs=xs, ys=ys, scs=scs, fwss=fwss):
            for i, c in enumerate(synth.BLOCK_3B):
                B.bitlinear_forward(copies[i][j % rot], 0, blk[i][1], c["N"], c["K"], xs[i], scs[i], ys[i],
                                    fwss[i], stream)

        with torch.cuda.stream(stream):
            for j in range(3):
                block(j)
        steps = 50 if M <= 128 else 10
        us = graph_ms(stream, steps, block) / steps * 1e3
        nbytes = sum(c["N"] * rb + M * c["K"] * 2 + M * c["N"] * 2 + 4 * M + 4
                     for c, (_, _, rb) in zip(synth.BLOCK_3B, blk))
        ops = sum(2.0 * M * c["N"] * c["K"] for c in synth.BLOCK_3B)
        out["block_3b"].append({"M": M, "us_per_block": us, "GB_s": nbytes / (us * 1e-6) / 1e9,
                                "frac_of_hbm": nbytes / (us * 1e-6) / 1e9 / peak_gbs,
                                "TOPS": ops / (us * 1e-6) / 1e12,
                                "frac_of_int8": ops / (us * 1e-6) / 1e12 / peak_tops})
        # the same block with Q, K and V as one grouped call on one shared input
        qkv_rows = [c["N"] for c in synth.BLOCK_3B[:3]]
        qkv = [torch.cat([copies[i][r] for i in range(3)], dim=0) for r in range(rot)]
        qkv_g = torch.cat([blk[i][1] for i in range(3)])
        y_qkv = torch.empty((M, sum(qkv_rows)), dtype=torch.bfloat16, device=dev)
        ws_qkv = torch.zeros(B.bitlinear_forward_grouped_workspace_bytes(M, qkv_rows, synth.BLOCK_3B[0]["K"], 0,
                                                                         B.BL_BF16), dtype=torch.uint8, device=dev)

        def block_fused(j, M=M, xs=xs, ys=ys, scs=scs, fwss=fwss, y_qkv=y_qkv, ws_qkv=ws_qkv):
            B.bitlinear_forward_grouped(qkv[j % rot], 0, qkv_g, qkv_rows, synth.BLOCK_3B[0]["K"], xs[0], scs[0],
                                        y_qkv, ws_qkv, stream)
            for i, c in enumerate(synth.BLOCK_3B[3:], start=3):
                B.bitlinear_forward(copies[i][j % rot], 0, blk[i][1], c["N"], c["K"], xs[i], scs[i], ys[i],
                                    fwss[i], stream)

        with torch.cuda.stream(stream):
            for j in range(3):
                block_fused(j)
        us_f = graph_ms(stream, steps, block_fused) / steps * 1e3
        if B.bitlinear_device_status(ws_qkv, stream) != B.BL_OK:
            raise RuntimeError("fused block device status")
        nbytes_f = nbytes - 2 * M * synth.BLOCK_3B[0]["K"] * 2
        out["block_3b_fused_qkv"].append({"M": M, "us_per_block": us_f, "GB_s": nbytes_f / (us_f * 1e-6) / 1e9,
                                          "frac_of_hbm": nbytes_f / (us_f * 1e-6) / 1e9 / peak_gbs,
                                          "TOPS": ops / (us_f * 1e-6) / 1e12,
                                          "frac_of_int8": ops / (us_f * 1e-6) / 1e12 / peak_tops,
                                          "vs_separate": us / us_f})
        del xs, ys, scs, fwss, qkv, y_qkv, ws_qkv
    out["note"] = ("graphs of back-to-back forward calls timed at their two ends; bytes = packed weights + bf16 x + "
                   "bf16 y; TOPS = 2 M N K; fractions of the measured HBM copy rate and of the int8 peak")
    return out


def decode_summary(d):
    if d is None:
        return None
    peak, kind = measured_peaks()
    res = {}
    for name, v in d.items():
        rows = v["rows"]
        tot_b = sum(r["bytes"] for r in rows)
        tot_us = sum(r["us"] for r in rows)
        gbs = tot_b / (tot_us * 1e-6) / 1e9
        fmt = 1 if name.endswith("base3") else (2 if name.endswith("1bit") else 0)
        res[name] = {"workload": v["desc"] + [", 2-bit pack", ", base-3 pack", ", 1-bit weights (8 per byte)"][fmt],
                     "kernel": gemv_kernel_name(fmt, [(r["N"], r["K"]) for r in rows]), "GB_s": gbs, "frac_of_hbm": gbs / peak,
                     "per_layer": [{"N": r["N"], "K": r["K"], "us_per_launch": r["us"], "bytes_per_launch": r["bytes"],
                                    "GB_s": r["bytes"] / (r["us"] * 1e-6) / 1e9,
                                    "frac_of_hbm": r["bytes"] / (r["us"] * 1e-6) / 1e9 / peak} for r in rows],
                     "l2": f"packed copies rotated (>= 4x L2): {[r['rot'] for r in rows]}"}
    return {"peak": peak, "peak_kind": kind, "unit": "GB/s", "shapes": res,
            "launch_duration": "CUDA events at the two ends of a graph of back-to-back forward calls"}


def gemv1_fits(N, K, rb, t5=False, xwords=2, cps=None):
    """Mirror of the library's one-token kernel geometry (bf16 tokens by
    default): K % 16 == 0, at most 512 lanes per row, at most four 16-byte code
    chunks per thread, and the (table,) token region, row sums and a ring of 8
    or 6 stages within 110 KB of shared memory."""
    segs = rb // 16
    lpr = segs if segs < 32 else -(-segs // 32) * 32
    if K % 16 or segs < 1 or lpr > 512:
        return False
    grid = min(N, 148)
    rpc = -(-N // grid)
    R = min(512 // lpr, rpc)
    threads = -(-(R * lpr) // 32) * 32
    cps = cps or (5 if t5 else 4)  # 16-byte code chunks per segment (1-bit: 8)
    per = -(-(cps * segs) // threads)
    if per > 4 or (cps == 8 and per > 2):
        return False
    xreg = -(-max(K * xwords, rb * cps) // 16) * 16
    fixed = (32768 if t5 else 0) + xreg + 4 * rpc
    return any(fixed + 16 * st * threads <= 110 * 1024 for st in ((6,) if cps == 8 else (8, 6)))


def gemv_kernel_name(fmt, layers, M=1):
    """The decode kernel the forward dispatches to (M <= 4), '+'-joined when
    the layers take different ones: for one token the column-stationary
    one-token kernels where they fit (2-bit: gemv1_i2_kernel, base 3:
    gemv1_t5_kernel); for 2..4 tokens of 2-bit rows of at most 8192 bytes
    (and at most 1024 rows per CTA) the column-stationary multi-token kernel,
    else the lean 2-bit kernel for rows of at most 8192 packed bytes; for one
    token of base 3 that the one-token kernel does not take, the older
    column-stationary kernel for rows of at most 768 segments and at most 1024
    rows per CTA; else the general one."""
    def one(N, K):
        if fmt == 2:  # 1-bit: the one-token kernel where it fits, else the lean kernel's 1-bit form
            rb = ((K + 7) // 8 + 15) // 16 * 16
            if M == 1 and gemv1_fits(N, K, rb, cps=8):
                return "gemv1_b1_kernel"
            return "gemv_i2_kernel" if rb <= 4096 else "gemv_kernel"
        if fmt == 0:
            rb = ((K + 3) // 4 + 15) // 16 * 16
            if M == 1 and rb <= 8192 and gemv1_fits(N, K, rb):
                return "gemv1_i2_kernel"
            if 2 <= M <= 4 and rb <= 8192 and -(-N // min(N, 148)) <= 1024:
                return "gemv_i2_mt_kernel"
            return "gemv_i2_kernel" if rb <= 8192 else "gemv_kernel"
        rb = ((K + 4) // 5 + 15) // 16 * 16
        if M == 1 and gemv1_fits(N, K, rb, t5=True):
            return "gemv1_t5_kernel"
        if M == 1 and rb // 16 <= 768 and -(-N // min(N, 148)) <= 1024:
            return "gemv_t5_kernel"
        return "gemv_kernel"
    names = []
    for (N, K) in layers:
        n = one(N, K)
        if n not in names:
            names.append(n)
    return "+".join(names)


def gemm_kernel_name(M):
    """The tensor-core kernel the forward dispatches to for M tokens (M > 4)."""
    return "gemm_i2_2sm_kernel" if M > 128 else "gemm_i2_kernel"


def prefill_summary(p):
    if p is None:
        return None
    peak, kind = measured_int8_peak()
    tops = p["ops"] / (p["gemm_ms"] * 1e-3) / 1e12
    fwd_tops = p["ops"] / ((p["gemm_ms"] + p["act_ms"]) * 1e-3) / 1e12
    hbm, hkind = measured_peaks()
    act_gbs = p["act_bytes"] / (p["act_ms"] * 1e-3) / 1e9
    return {"workload": f"3B prefill: M={p['M']} tokens, K={p['K']} -> N={p['N']}, 2-bit, bf16 x with "
                        "16 outlier channels x30, bf16 y",
            "value": tops, "unit": "TOPS (int8)", "forward_TOPS_incl_act_quant": fwd_tops,
            "gemm_us": p["gemm_ms"] * 1e3, "act_quant_us": p["act_ms"] * 1e3,
            "act_quant_GB_s": act_gbs, "act_quant_frac_of_hbm": act_gbs / hbm,
            "layernorm_act_quant": {"kernel": "ln_quant_reg_kernel" if p["K"] % 2 == 0 and p["K"] <= 4096
                                    else "ln_quant_kernel", "us": p["ln_ms"] * 1e3,
                                    "GB_s": p["ln_bytes"] / (p["ln_ms"] * 1e-3) / 1e9,
                                    "frac_of_hbm": p["ln_bytes"] / (p["ln_ms"] * 1e-3) / 1e9 / hbm},
            "roofline": {"bound": "tensor", "kernel": gemm_kernel_name(p["M"]), "achieved": tops, "peak": peak,
                         "peak_kind": kind, "unit": "TOPS", "frac": tops / peak,
                         "traffic": profiled_traffic(gemm_kernel_name(p["M"]), "3b_prefill")},
            "steps": p["steps"], "l2": f"inputs rotated over {p['rot']} copies (> 2x L2)"}


# Small standalone cases for ncu captures: one call repeated a few times on one
# shape, with seeded N(0, sigma) latent weights and N(0, 1) bf16 tokens drawn on
# the device.  Launch order: the weight preparation (absmean, ternarize + pack)
# once, then three forwards; a "quantize" case runs the preparation three times.
PROFILE_CASES = {
    "quantize_3b_up": dict(N=8640, K=3200, fmt=0, M=1, sigma=0.02, op="quantize"),
    "decode_3b_up": dict(N=8640, K=3200, fmt=0, M=1, sigma=0.02, op="forward"),
    "decode_70b_up": dict(N=28672, K=8192, fmt=0, M=1, sigma=0.01, op="forward"),
    "decode_70b_down": dict(N=8192, K=28672, fmt=0, M=1, sigma=0.01, op="forward"),
    "decode_70b_up_t5": dict(N=28672, K=8192, fmt=1, M=1, sigma=0.01, op="forward"),
    "prefill_3b": dict(N=8640, K=3200, fmt=0, M=4096, sigma=0.02, op="forward"),
    "batch16_70b_up": dict(N=28672, K=8192, fmt=0, M=16, sigma=0.01, op="forward"),
    "lnquant_3b_prefill": dict(N=8640, K=3200, fmt=0, M=4096, sigma=0.02, op="lnquant"),
    "batch16_70b_down": dict(N=8192, K=28672, fmt=0, M=16, sigma=0.01, op="forward"),
    "binarize_3b_up": dict(N=8640, K=3200, fmt=2, M=1, sigma=0.02, op="quantize"),
    "decode_70b_up_1bit": dict(N=28672, K=8192, fmt=2, M=1, sigma=0.01, op="forward"),
    "backward_3b_up": dict(N=8640, K=3200, fmt=0, M=1, sigma=0.02, op="backward"),
    "batch4_70b_up": dict(N=28672, K=8192, fmt=0, M=4, sigma=0.01, op="forward"),
    "batch2_70b_up_t5": dict(N=28672, K=8192, fmt=1, M=2, sigma=0.01, op="forward"),
    "batch16_70b_up_t5": dict(N=28672, K=8192, fmt=1, M=16, sigma=0.01, op="forward"),
    "batch16_70b_up_1bit": dict(N=28672, K=8192, fmt=2, M=16, sigma=0.01, op="forward"),
    "backward_3b_down": dict(N=3200, K=8640, fmt=0, M=1, sigma=0.02, op="backward"),
    "backward_3b_up_m8": dict(N=8640, K=3200, fmt=0, M=8, sigma=0.02, op="backward"),
    "decode_70b_down_t5": dict(N=8192, K=28672, fmt=1, M=1, sigma=0.01, op="forward"),
    "decode_70b_down_1bit": dict(N=8192, K=28672, fmt=2, M=1, sigma=0.01, op="forward"),
    "lnquant_70b_down": dict(N=8192, K=28672, fmt=0, M=256, sigma=0.01, op="lnquant"),
    "pack_3b_up": dict(N=8640, K=3200, fmt=0, M=1, sigma=0.02, op="pack"),
    "actquant_16x40000": dict(N=16, K=40000, fmt=0, M=16, sigma=0.02, op="actquant"),
    "quantize_3b_up_t5": dict(N=8640, K=3200, fmt=1, M=1, sigma=0.02, op="quantize"),
}


def run_profile_case(name):
    import torch

    from bitlinear_b1_fwd_b200 import binding as B
    from bitlinear_b1_fwd_b200 import build as libbuild

    c = PROFILE_CASES[name]
    libbuild.build()
    dev = torch.device("cuda", 0)
    N, K, M, fmt = c["N"], c["K"], c["M"], c["fmt"]
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    W = torch.randn(N, K, generator=g, device=dev) * c["sigma"]
    x = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
    packed = torch.empty((N, B.bitlinear_packed_row_bytes(K, fmt)), dtype=torch.uint8, device=dev)
    gamma = torch.empty(1, dtype=torch.float32, device=dev)
    if fmt == B.BL_PACK_B1:  # the 1-bit variant: beta (in gamma's place) and alpha
        alpha = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.zeros(B.bitlinear_binarize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
        for _ in range(3 if c["op"] == "quantize" else 1):
            B.bitlinear_binarize_weights(W, packed, None, gamma, alpha, ws)
    else:
        ws = torch.zeros(B.bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
        for _ in range(3 if c["op"] == "quantize" else 1):
            B.bitlinear_quantize_weights(W, 1e-5, fmt, packed, None, gamma, ws)
    status = [B.bitlinear_device_status(ws)]
    if c["op"] == "pack":  # A3 alone: int8 codes -> packed rows
        codes = torch.empty((N, K), dtype=torch.int8, device=dev)
        B.bitlinear_quantize_weights(W, 1e-5, fmt, packed, codes, gamma, ws)
        for _ in range(3):
            B.bitlinear_pack(codes, fmt, packed, ws)
        status.append(B.bitlinear_device_status(ws))
    if c["op"] == "actquant":  # A4 alone on rows longer than the one-CTA-per-token kernels take
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sc = torch.empty(M, dtype=torch.float32, device=dev)
        for _ in range(3):
            B.bitlinear_quantize_acts(x, xq, sc)
    if c["op"] == "lnquant":
        ln_w = torch.randn(K, generator=g, device=dev) * 0.1 + 1.0
        ln_b = torch.randn(K, generator=g, device=dev) * 0.1
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sc = torch.empty(M, dtype=torch.float32, device=dev)
        for _ in range(3):
            B.bitlinear_layernorm_quantize_acts(x, ln_w, ln_b, 1e-5, xq, sc)
    if c["op"] == "forward":
        scale = torch.empty(M, dtype=torch.float32, device=dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        fws = torch.zeros(B.bitlinear_forward_workspace_bytes(M, N, K, fmt, B.BL_BF16), dtype=torch.uint8, device=dev)
        for _ in range(3):
            B.bitlinear_forward(packed, fmt, gamma, N, K, x, scale, y, fws)
        status.append(B.bitlinear_device_status(fws))
    if c["op"] == "backward":  # STE backward for M tokens: dx from the packed weights, dW from x_q
        dy = (torch.randn(M, N, generator=g, device=dev) * 1e-3).to(torch.bfloat16)
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sc = torch.empty(M, dtype=torch.float32, device=dev)
        B.bitlinear_quantize_acts(x, xq, sc)
        dx = torch.empty((M, K), dtype=torch.float32, device=dev)
        dw = torch.empty((N, K), dtype=torch.float32, device=dev)
        bws = torch.zeros(B.bitlinear_backward_dx_workspace_bytes(M, N, K, fmt), dtype=torch.uint8, device=dev)
        for _ in range(3):
            B.bitlinear_backward_dx(packed, fmt, gamma, N, K, dy, dx, bws)
            B.bitlinear_backward_dw(dy, xq, sc, gamma, dw)
        status.append(B.bitlinear_device_status(bws))
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, **c, "status": status}))
    if any(status):
        sys.exit(1)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="3b_decode")
    ap.add_argument("--phase", choices=["forward", "all"], default="forward")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--prefill", action=argparse.BooleanOptionalAction, default=True,
                    help="also time the 3B prefill layer (INT8 TOPS of the tensor-core product)")
    ap.add_argument("--prefill-steps", type=int, default=20)
    ap.add_argument("--decode", action=argparse.BooleanOptionalAction, default=True,
                    help="also time the decode GEMV alone on packed 3B and 70B layers (2-bit and base-3)")
    ap.add_argument("--decode-steps", type=int, default=200)
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of oracle time for the cpu_baseline sample (0 = skip)")
    ap.add_argument("--sweep", action=argparse.BooleanOptionalAction, default=False,
                    help="also time the 70B layers over M = 1..8192 and the 3B block at M = 1, 16, 128, 1024")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES), default=None,
                    help="run one small standalone case (for ncu captures) and exit")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case)
        return
    wl = WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    # one config dict, printed unchanged by both arms
    config = {"workload": args.workload, "desc": wl["desc"], "phase": args.phase, "M": wl["M"],
              "layers_NK": wl["layers"], "pack": ["2-bit", "base-3"][wl["fmt"]],
              "parallelism": f"replicas x{args.gpus}"}

    if args.impl == "reference":
        if rank != 0:
            return
        # per-step sample of the oracle sized so the whole run stays within ~2 minutes
        import oracle
        oracle.build()
        probe_frac = 0.02
        v, s, dt = time_oracle(wl, args.phase, 0.0, min_steps=1, rows_frac=probe_frac)
        per_step_full = dt / s / probe_frac
        budget = 120.0 / max(1, args.steps + args.warmup)
        frac = min(1.0, max(1e-4, budget / per_step_full))
        inputs = oracle_layer_inputs(wl, args.phase, frac)
        for _ in range(args.warmup):
            oracle_step(oracle, wl, inputs, args.phase)
        t0 = time.perf_counter()
        nbytes = sum(oracle_step(oracle, wl, inputs, args.phase) for _ in range(args.steps))
        dt = time.perf_counter() - t0
        val = nbytes / dt / 1e9
        what = "the forward on weights packed beforehand" if args.phase == "forward" else "all steps of the path"
        sample = f"first {frac:.4%} of each layer's weight rows per step, {what}"
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64+i32",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": val, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
                             **host_cpu()},
            "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    import torch
    if world > 1:
        torch.distributed.init_process_group("nccl", device_id=torch.device("cuda", local_rank),
                                             timeout=__import__("datetime").timedelta(seconds=120))
    res = run_gpu(args, wl, rank, world, local_rank)

    if rank == 0:
        ms = res["ms_total"] / args.steps
        value = whole_job_gbs(res["step_bytes"], world, ms)
        peak, peak_kind = measured_peaks()
        nl = len(res["layers"])

        def stage(op):
            per_launch = res["per_op_ms"][op]
            nb = sum(L["bytes"][op] for L in res["layers"])
            return {"us_per_launch": per_launch * 1e3, "bytes_per_step": nb,
                    "GB_s": nb / (per_launch * nl * 1e-3) / 1e9,
                    "frac_of_hbm": nb / (per_launch * nl * 1e-3) / 1e9 / peak}

        stages = {op: stage(op) for op in res["ops"]}
        flat = wl["fmt"] == 0 and all(K % 64 == 0 for (_, K) in wl["layers"])
        names = {"absmean": "absmean_kernel",
                 "ternarize_pack": "ternarize_flat_kernel" if flat else "ternarize_pack_kernel",
                 "forward": gemv_kernel_name(wl["fmt"], wl["layers"], wl["M"])}
        # the roofline is the forward's (the per-token kernel the metric names);
        # with --phase all, the step's dominant kernel
        dom = "forward" if args.phase == "forward" else max(stages, key=lambda o: stages[o]["us_per_launch"])
        avg_launch_ms = res["per_op_ms"][dom]
        bytes_per_launch = stages[dom]["bytes_per_step"] / nl
        achieved = bytes_per_launch / (avg_launch_ms * 1e-3) / 1e9
        kernel_name = names[dom]
        traffic = profiled_traffic(kernel_name, args.workload)
        weight_prep = {op: dict(stage(op), kernel=names[op]) for op in ("absmean", "ternarize_pack")} \
            if args.phase == "forward" else None
        if weight_prep is not None:
            for op in weight_prep:
                nb = sum(L["bytes"][op] for L in res["layers"])
                weight_prep[op]["bytes_per_step"] = nb
        cpu = None
        if args.cpu_budget > 0 and world == 1:
            v, s, dt = time_oracle(wl, args.phase, args.cpu_budget)
            what = "forwards on weights packed beforehand" if args.phase == "forward" else "full oracle steps"
            cpu = {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                   "sample": f"{s} {what} of the same workload ({dt:.1f} s, 1 thread)", **host_cpu()}
        e2e_value = whole_job_gbs(res["step_bytes"], world, res["e2e_ms"])
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "i8xternary->i32 (fp32 scales, fp64 gamma)",
            "data": "synthetic (seeded N(0,sigma) latent weights, N(0,1) bf16 activations)",
            "config": config,
            "l2": (f"packed weights rotated over {res['rot']} copies (>= 4x L2)" if args.phase == "forward" else
                   "inputs larger than L2 (fp32 latent weights "
                   f"{sum(L['N'] * L['K'] * 4 for L in res['layers']) / 1e6:.0f} MB per step)"),
            "kernels_per_step": res["launches_per_step"],
            "roofline": {"bound": "hbm", "kernel": kernel_name, "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic, "bytes_per_launch": bytes_per_launch,
                         "launch_duration": ("CUDA events at the two ends of the graph of K steps "
                                             "(K x layers back-to-back forward launches)"
                                             if args.phase == "forward" else
                                             "CUDA events at the two ends of a graph of K steps of this "
                                             "call alone over every layer")},
            "stages": stages,
            "weight_prep": weight_prep,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": res["h2d"],
                    "d2h_bytes_per_step": res["d2h"], "steps": res["e2e_steps"]},
            "prefill": prefill_summary(res["prefill"]),
            "decode_gemv": decode_summary(res["decode"]),
            "backward": res.get("backward"),
            "sweep": res["sweep"],
            "gpu_launches": res["launches_per_step"] * args.steps,
            "clocks": res["clocks"],
        }
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
