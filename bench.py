#!/usr/bin/env python
"""Benchmark of the DSFQ W4A4 linear (libw4a4) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Workload (default, c5_full_stack): the full-depth linear stack of a VGGT-style
1024-wide transformer at 64 frames (M = 87936 tokens): 48 blocks x the four
linears (QKV 1024->3072, proj 1024->1024, fc1 1024->4096 with the GELU on its
output, fc2 4096->1024), fresh seeded weights per layer and a fresh seeded
heavy-tailed activation batch for every layer that reads the block's input
(fc2 reads its block's GELU(fc1) output).  One "step" = every layer once:
rotate + smooth + per-token int4 quantize (kernel 1), integer GEMM on the
tensor cores + dequant/bias epilogue (kernel 2).  Weight preparation is
offline and untimed.  Other workloads (--workload): the single linear, the
frame-attention QKV at 8 frames, the MLP pair, the global-attention block and
the 3DTurboQuant KV-cache codec.

Metric: W4A4 linear throughput in TOPS (2*M*N*K integer ops per layer, summed
over the step), with tokens/s alongside; roofline fractions of the GEMM
against the int8 tensor peak and of the quantize kernel against HBM bandwidth.

Under torchrun each rank runs an independent replica on its own GPU (token
batches are independent: weak scaling, no data-path collective); the timed
region is bracketed by barrier + synchronize and the max over ranks is used.

--impl reference times the CPU oracle (the only reference this build has: the
pages hold no code) on a bounded sample of the same workload, on the host
cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from w4a4_post_quantized_b200 import synth  # noqa: E402

WORKLOADS = {
    "c2_frame_qkv": dict(frames=8, K=1024, N=3072,
                         desc="VGGT frame-attention QKV linear, 8 frames: M=10992, K=1024, N=3072"),
    "c1_single_linear": dict(frames=1, K=1024, N=1024,
                             desc="single linear, 1 frame: M=1374, K=1024, N=1024"),
    "c3_fc2": dict(frames=8, K=4096, N=1024,
                   desc="VGGT MLP fc2 (GELU on input), 8 frames: M=10992, K=4096, N=1024", gelu=True),
}
# Multi-layer workloads: the four linears of a transformer block (fc2 takes
# fc1's output through GELU, applied by fc1's GEMM epilogue; the other layers
# take synthetic activations, since attention and normalisation sit between
# them), repeated over `blocks` blocks with fresh weights per layer.
STACKS = {
    "c3_mlp_pair": dict(frames=8, blocks=1, layers=[("fc1", 1024, 4096), ("fc2", 4096, 1024)],
                        desc="VGGT MLP pair, 8 frames: fc1 1024->4096, GELU, fc2 4096->1024, M=10992"),
    "c4_global_block": dict(frames=32, blocks=1,
                            layers=[("qkv", 1024, 3072), ("proj", 1024, 1024), ("fc1", 1024, 4096),
                                    ("fc2", 4096, 1024)],
                            desc="global-attention block's four linears, 32 frames: M=43968"),
    "c5_full_stack": dict(frames=64, blocks=48,
                          layers=[("qkv", 1024, 3072), ("proj", 1024, 1024), ("fc1", 1024, 4096),
                                  ("fc2", 4096, 1024)],
                          desc="48 blocks x the four linears, 64 frames: M=87936"),
}
METRIC = "W4A4 linear TOPS & tokens/s on VGGT shapes, % of INT8 TC peak / HBM BW"
NSETS = 4          # input/output buffer sets rotated so no step finds its inputs in L2
INT8_PER_BF16 = 2.0  # nominal dense int8 : bf16 tensor throughput ratio (4.5 / 2.25 POPS)
TF32_PER_BF16 = 1.1 / 2.25  # nominal dense tf32 : bf16 tensor throughput ratio


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained"),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def profile_traffic(kernel_file: str, key: str):
    """Per-launch DRAM bytes from the committed ncu summary, or None when the
    kernel source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(key)
    if not d:
        return None
    src = os.path.join(ROOT, "w4a4_post_quantized_b200", "csrc", kernel_file)
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return d["bytes_per_launch"] if d.get("source_sha") == h else None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                rows.append((float(f[0]), float(f[1]), f[3:7]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, x: float) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    # the process group's own device: CUDA under NCCL, the host under gloo
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_sample(wl, rows_per_step: int, seed: int = 0):
    """Prepare (untimed) and return a closure that runs the oracle's hot path
    (rotate, smooth, quantize, integer GEMM, dequantize) on `rows_per_step`
    rows of the workload."""
    import oracle
    K, N = wl["K"], wl["N"]
    M = wl["frames"] * synth.FRAME_TOKENS
    X = synth.activations(M, K, seed=seed)
    W = synth.weights(N, K, seed=seed + 1)
    b = synth.bias(N, seed=seed + 2)
    pw = oracle.prepare_weights(W, b, X[:synth.calibration_rows(M)])
    rows = np.concatenate([synth.special_rows(min(M, rows_per_step)),
                           np.arange(5, M, max(1, M // rows_per_step))])[:rows_per_step]
    Xs = X[np.sort(rows)]
    gelu = wl.get("gelu", False)

    def run():
        return oracle.linear(Xs, pw, gelu=gelu)[0]
    return run, len(Xs), oracle.max_threads()


def run_reference(args, wl, world, rank):
    if rank != 0:
        return
    # each step is the oracle on a bounded row sample, sized so that the whole
    # run (warm-up + timed steps) takes about two minutes of CPU time
    K, N = wl["K"], wl["N"]
    probe, r0, _ = cpu_oracle_sample(wl, args.cpu_rows)
    t = time.perf_counter()
    probe()
    per_row = (time.perf_counter() - t) / r0
    rows = int(min(args.cpu_rows, max(16, 120.0 / max(1, args.steps + args.warmup) / per_row)))
    run, r, cores = cpu_oracle_sample(wl, rows)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = (time.perf_counter() - t0) / args.steps
    tops = 2.0 * r * N * K / dt / 1e12
    sample = f"{r} of {wl['frames'] * synth.FRAME_TOKENS} token rows per step (special tokens included)"
    line = {
        "impl": "reference", "metric": METRIC, "value": tops, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64/int64",
        "data": "synthetic", "tokens_per_s": r / dt,
        "config": {"workload": wl["desc"], "M_sampled": r, "N": N, "K": K},
        "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, wl, world, rank, local):
    import torch
    from w4a4_post_quantized_b200 import w4a4
    K, N = wl["K"], wl["N"]
    gelu = wl.get("gelu", False)
    flags = w4a4.W4A4_FLAG_GELU if gelu else 0
    M = wl["frames"] * synth.FRAME_TOKENS
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    def bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

    # ------------------------------------------------------------ inputs (untimed)
    seed = 1000 * rank
    W = bf16(synth.weights(N, K, seed=seed + 1))
    b = bf16(synth.bias(N, seed=seed + 2))
    Xs = [bf16(synth.activations(M, K, seed=seed + 10 + i)) for i in range(NSETS)]
    pw = w4a4.w4a4_prepare_weights(W, b, Xs[0][:synth.calibration_rows(M)])
    Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(NSETS)]
    # the workspace of the fused call's fastest route: int4 codes one per byte
    # (operand order of the expanded weights), then the steps
    wsb = w4a4.w4a4_workspace_bytes(M, K)
    WSs = [torch.empty(wsb, dtype=torch.uint8, device=dev) for _ in range(NSETS)]
    st_off = ((M * K + 255) // 256) * 256
    QX = [ws[:M * K].view(M, K) for ws in WSs]
    ST = [ws[st_off:st_off + 4 * M].view(torch.float32) for ws in WSs]
    unp = w4a4.W4A4_FLAG_UNPACKED
    torch.cuda.synchronize()

    def step(i):
        w4a4.w4a4_linear_fused(Xs[i % NSETS], pw, Y=Ys[i % NSETS], workspace=WSs[i % NSETS], flags=flags)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    w4a4.w4a4_clear_device_status()

    # ---------------------------------------------------------------- timed region
    # each step is the call a user makes, w4a4_linear_fused: the quantize
    # kernel and the GEMM back to back on one stream (each may start its setup
    # while the previous kernel finishes; see the programmatic launch in csrc)
    evq = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        torch.cuda.nvtx.range_push("timed")
        for i in range(args.steps):
            step(i)
        torch.cuda.nvtx.range_pop()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        # each kernel alone, launched back to back over the same rotating
        # buffers (consecutive launches overlap their setup as in a step):
        # the per-launch durations the rooflines use
        n_iso = max(3, min(args.steps, 500))
        iso = {}
        for name, fn in (("quant", lambda j: w4a4.w4a4_quantize_act(Xs[j], pw.inv_smooth, flags | unp,
                                                                     qx=QX[j], scale_tok=ST[j])),
                         ("gemm", lambda j: w4a4.w4a4_linear_ex(QX[j], ST[j], pw, flags=unp, Y=Ys[j]))):
            for i in range(3):  # warm-up launches of this kernel alone
                fn(i % NSETS)
            k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            k0.record(stream)
            for i in range(n_iso):
                fn(i % NSETS)
            k1.record(stream)
            torch.cuda.synchronize()
            iso[name] = max_over_ranks(world, k0.elapsed_time(k1)) / n_iso
        # attribution pass (not part of `value`): the same steps with an event
        # between the two kernels, for each kernel's duration.  An event between
        # them keeps the GEMM from overlapping the quantize kernel's tail, so
        # these durations are slightly longer than the kernels' share of a step.
        for i in range(args.steps):
            j = i % NSETS
            e0, e1, e2 = evq[i]
            e0.record(stream)
            w4a4.w4a4_quantize_act(Xs[j], pw.inv_smooth, flags | unp, qx=QX[j], scale_tok=ST[j])
            e1.record(stream)
            w4a4.w4a4_linear_ex(QX[j], ST[j], pw, flags=unp, Y=Ys[j])
            e2.record(stream)
        torch.cuda.synchronize()
    status = w4a4.w4a4_get_device_status()
    elapsed_ms = max_over_ranks(world, t0.elapsed_time(t1))
    q_step_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evq)
    g_step_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evq)
    q_ms, g_ms = iso["quant"], iso["gemm"]
    ms_step = elapsed_ms / args.steps
    ops = 2.0 * M * N * K
    value = world * ops * args.steps / (elapsed_ms * 1e-3) / 1e12

    # ------------------------------------------------------------- end to end
    # the C-ABI host-buffer call a user with host tensors makes: every step
    # copies its X from pinned host memory and its Y back, in row chunks whose
    # copies in, kernels and copies out overlap on three streams
    Xh = [torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    for x, src in zip(Xh, Xs):
        x.copy_(src.cpu())
    Yh = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    chunk = args.e2e_chunk
    pipe = w4a4.HostPipe()
    hws = torch.empty(w4a4.w4a4_host_workspace_bytes(chunk, K, N), dtype=torch.uint8, device=dev)

    def host_step(i):
        w4a4.w4a4_linear_fused_host(Xh[i % 2], pw, Y_host=Yh[i % 2], chunk_rows=chunk, workspace=hws,
                                    pipe=pipe, flags=flags)
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    for i in range(3):
        host_step(i)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a0.record(stream)
    for i in range(e2e_steps):
        host_step(i)
    a1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    pipe.close()
    e2e_ms = max_over_ranks(world, a0.elapsed_time(a1)) / e2e_steps
    e2e_value = world * ops / (e2e_ms * 1e-3) / 1e12

    # ------------------------------------------------- DSFQ overhead (M7) and bytes (M2)
    # the same fused call with the rotation and smoothing skipped (plain
    # per-token / per-channel int4, weights prepared the same way), timed over
    # the same rotating buffers; the pages put DSFQ's extra latency at 0.2 %
    n7 = max(3, min(args.steps, 400))
    pw_plain = w4a4.w4a4_prepare_weights(W, b, Xs[0][:synth.calibration_rows(M)],
                                         flags=w4a4.W4A4_FLAG_PLAIN)
    m7 = {}
    for mode, p, fl in (("dsfq", pw, flags), ("plain", pw_plain, flags | w4a4.W4A4_FLAG_PLAIN)):
        for i in range(3):
            w4a4.w4a4_linear_fused(Xs[i % NSETS], p, Y=Ys[i % NSETS], workspace=WSs[i % NSETS], flags=fl)
        barrier(world)
        torch.cuda.synchronize()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for i in range(n7):
            w4a4.w4a4_linear_fused(Xs[i % NSETS], p, Y=Ys[i % NSETS], workspace=WSs[i % NSETS], flags=fl)
        b1.record(stream)
        torch.cuda.synchronize()
        m7[mode] = max_over_ranks(world, b0.elapsed_time(b1)) / n7 * 1e3
    # quantization quality of both modes on the first frame of the batch (the
    # heavy-tailed special-token rows included): SQNR of Y against the
    # unquantized product of the same bf16 inputs, computed in fp64 by torch
    rows = synth.calibration_rows(M)
    xr = Xs[0][:rows]
    if gelu:  # the layer's input is GELU(x) in bf16
        xr = torch.nn.functional.gelu(xr.float()).to(torch.bfloat16)
    ref = (xr.double() @ W.double().t() + b.double())
    sq = {}
    for mode, p, fl in (("dsfq", pw, flags), ("plain", pw_plain, flags | w4a4.W4A4_FLAG_PLAIN)):
        y = w4a4.w4a4_linear_fused(Xs[0][:rows], p, flags=fl).double()
        sq[mode] = float(10.0 * torch.log10((ref ** 2).sum() / ((y - ref) ** 2).sum()))
    torch.cuda.synchronize()
    dsfq_overhead = {"dsfq_us_per_step": m7["dsfq"], "plain_us_per_step": m7["plain"],
                     "overhead_pct": 100.0 * (m7["dsfq"] - m7["plain"]) / m7["plain"],
                     "steps": n7, "pages_figure_pct": 0.2,
                     "sqnr_db": sq, "sqnr_rows": rows}
    # ------------------------------------------------------- W8A8 (8-bit codes)
    # the setting the pages report beside W4A4, on the same inputs: 8-bit
    # codes need no widening in the GEMM, so the isolated GEMM times of the
    # two settings bracket what the 4-bit codes cost there (the 8-bit GEMM
    # also reads twice the activation bytes and uses 128 x 256 tiles)
    i8 = w4a4.W4A4_FLAG_INT8
    pw8 = w4a4.w4a4_prepare_weights(W, b, Xs[0][:synth.calibration_rows(M)], flags=i8)
    fl8 = flags | i8
    t8 = {}
    for name, fn in (("step", lambda j: w4a4.w4a4_linear_fused(Xs[j], pw8, Y=Ys[j], workspace=WSs[j], flags=fl8)),
                     ("quant", lambda j: w4a4.w4a4_quantize_act(Xs[j], pw8.inv_smooth, fl8, qx=QX[j],
                                                                 scale_tok=ST[j])),
                     ("gemm", lambda j: w4a4.w4a4_linear(QX[j], ST[j], pw8, Y=Ys[j]))):
        for i in range(3):
            fn(i % NSETS)
        barrier(world)
        torch.cuda.synchronize()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for i in range(n7):
            fn(i % NSETS)
        b1.record(stream)
        torch.cuda.synchronize()
        t8[name] = max_over_ranks(world, b0.elapsed_time(b1)) / n7 * 1e3
    y8 = w4a4.w4a4_linear_fused(Xs[0][:rows], pw8, flags=fl8).double()
    sq8 = float(10.0 * torch.log10((ref ** 2).sum() / ((y8 - ref) ** 2).sum()))
    torch.cuda.synchronize()
    w8a8 = {"us_per_step": t8["step"], "tops": ops / (t8["step"] * 1e-6) / 1e12,
            "quantize_us": t8["quant"], "gemm_us": t8["gemm"],
            "gemm_tops": ops / (t8["gemm"] * 1e-6) / 1e12,
            "quantize_gbs": (2.0 * M * K + M * K + 4.0 * M) / (t8["quant"] * 1e-6) / 1e9,
            "w4a4_gemm_us": g_ms * 1e3, "w4a4_quantize_us": q_ms * 1e3,
            "sqnr_db": sq8, "sqnr_db_w4a4": sq["dsfq"], "sqnr_rows": rows,
            "timing": f"CUDA events around {n7} back-to-back launches each (step = w4a4_linear_fused)"}
    # ------------------------------------- the packed route (codes two per byte)
    # the fused call with the smallest workspace it accepts: packed int4 codes,
    # which the GEMM widens on every tile (once per output tile); the one-per-
    # byte route above is what the fused call takes with the full workspace
    wsp = w4a4.w4a4_workspace_bytes_min(M, K, flags)
    QP = [ws[:M * K // 2].view(M, K // 2) for ws in WSs]
    STP = [ws[((M * K // 2 + 255) // 256) * 256:][:4 * M].view(torch.float32) for ws in WSs]
    tp = {}
    for name, fn in (("step", lambda j: w4a4.w4a4_linear_fused(Xs[j], pw, Y=Ys[j], workspace=WSs[j][:wsp],
                                                                 flags=flags)),
                     ("quant", lambda j: w4a4.w4a4_quantize_act(Xs[j], pw.inv_smooth, flags, qx=QP[j],
                                                                 scale_tok=STP[j])),
                     ("gemm", lambda j: w4a4.w4a4_linear(QP[j], STP[j], pw, Y=Ys[j]))):
        for i in range(3):
            fn(i % NSETS)
        barrier(world)
        torch.cuda.synchronize()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for i in range(n7):
            fn(i % NSETS)
        b1.record(stream)
        torch.cuda.synchronize()
        tp[name] = max_over_ranks(world, b0.elapsed_time(b1)) / n7 * 1e3
    packed_route = {"us_per_step": tp["step"], "tops": ops / (tp["step"] * 1e-6) / 1e12,
                    "quantize_us": tp["quant"], "gemm_us": tp["gemm"],
                    "gemm_tops": ops / (tp["gemm"] * 1e-6) / 1e12,
                    "workspace_bytes": wsp, "workspace_bytes_fast_route": wsb,
                    "what": "w4a4_linear_fused with its minimum workspace: int4 codes two per byte, "
                            "widened by the GEMM on every tile"}
    weight_bytes = {"packed_int4": N * K // 2 + 12 * N + 4 * K, "bf16": 2 * N * K + 2 * N,
                    "expanded_int8_copy": N * K + 4 * N,
                    "ratio_bf16_over_packed": (2 * N * K + 2 * N) / (N * K // 2 + 12 * N + 4 * K)}

    # ------------------------------------------------------------- roofline
    peaks = load_peaks()
    int8_peak = peaks["bf16"] * INT8_PER_BF16
    gemm_tops = ops / (g_ms * 1e-3) / 1e12
    q_bytes = 2.0 * M * K + M * K / 2 + 4.0 * M
    q_gbs = q_bytes / (q_ms * 1e-3) / 1e9
    roofline = {"bound": "tensor", "kernel": "w4a4_gemm_kernel", "achieved": gemm_tops,
                "peak": int8_peak, "unit": "TOPS", "frac": gemm_tops / int8_peak,
                "traffic": profile_traffic("gemm.cu", f"gemm_{args.workload}"),
                "peak_note": f"int8 = {INT8_PER_BF16:g} x {peaks['src']} bf16 burst {peaks['bf16']} TFLOP/s",
                "ms_per_launch": g_ms, "algorithmic_ops_per_launch": ops,
                "ms_per_launch_in_step": g_step_ms,
                "timing": f"CUDA events around {n_iso} back-to-back launches of this kernel alone; "
                          "ms_per_launch_in_step: events between the two kernels of a step"}
    q_kernel = "quant_tc_kernel" if not gelu else "quantize_rows_kernel"
    roofline_q = {"bound": "hbm", "kernel": q_kernel, "achieved": q_gbs,
                  "peak": peaks["hbm"], "unit": "GB/s", "frac": q_gbs / peaks["hbm"],
                  "traffic": profile_traffic("quant_tc.cu" if not gelu else "quant.cu",
                                             f"quant_{args.workload}"),
                  "ms_per_launch": q_ms, "algorithmic_bytes_per_launch": q_bytes,
                  "ms_per_launch_in_step": q_step_ms}

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s4xs4->s32 (bf16 in/out, fp32 transform)", "data": "synthetic",
        "tokens_per_s": world * M * args.steps / (elapsed_ms * 1e-3),
        "config": {"workload": wl["desc"], "M": M, "N": N, "K": K, "per_rank_batch": M,
                   "parallelism": f"dp{world} (independent replicas)",
                   "l2": f"inputs/outputs rotated over {NSETS} buffer sets (~{(2*M*K+2*M*N+M*K//2)*NSETS/1e6:.0f} MB > L2)"},
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": "TOPS", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": 2 * M * K, "d2h_bytes_per_step": 2 * M * N,
                "api": f"w4a4_linear_fused_host (C ABI, pinned host X/Y, {chunk}-row chunks, "
                       "copies in / kernels / copies out overlapped)"},
        "gpu_launches": 2 * args.steps,
        "roofline": roofline,
        "roofline_quantize": roofline_q,
        "dsfq_overhead": dsfq_overhead,
        "w8a8": w8a8,
        "packed_route": packed_route,
        "weight_bytes": weight_bytes,
        "device_status": status,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        # the oracle on the whole batch (all M rows), repeated until about 10 s
        # of CPU work has been timed (at most 8 passes)
        run, r, cores = cpu_oracle_sample(wl, M)
        passes, t_total = 0, 0.0
        while passes < 8 and t_total < 10.0:
            t = time.perf_counter()
            run()
            t_total += time.perf_counter() - t
            passes += 1
        dt = t_total / passes
        line["cpu_baseline"] = {"value": 2.0 * r * N * K / dt / 1e12, "unit": "TOPS", "cores": cores,
                                "kind": "oracle",
                                "sample": f"all {r} token rows of one batch, {passes} passes, "
                                          f"{dt:.2f} s per pass"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def stack_layers(st):
    """(block, name, K, N) of every layer of a multi-layer workload, in order."""
    return [(b, name, K, N) for b in range(st["blocks"]) for (name, K, N) in st["layers"]]


def stack_ops(st, M):
    return sum(2.0 * M * N * K for (_, _, K, N) in stack_layers(st))


def stack_oracle_sample(st, rows: int, seed: int = 0):
    """Prepare (untimed) the oracle's weights for one block's layer shapes and
    return a closure that runs the oracle's hot path on `rows` token rows of
    each (special-token rows first, then a regular stride of patch tokens;
    fc2's input through the GELU, as the block's MLP feeds it).  One block
    stands for every block of the stack: they share the four layer shapes."""
    import oracle
    M = st["frames"] * synth.FRAME_TOKENS
    sel = np.concatenate([synth.special_rows(M), np.arange(5, M, max(1, M // rows))])[:rows]
    cases = []
    for j, (name, K, N) in enumerate(st["layers"]):
        W = synth.weights(N, K, seed=seed + 10 * j + 1)
        b = synth.bias(N, seed=seed + 10 * j + 2)
        Xc = synth.activations(synth.calibration_rows(M), K, seed=seed + 10 * j + 3)
        gelu = name == "fc2"
        pw = oracle.prepare_weights(W, b, oracle.gelu_bf16(Xc) if gelu else Xc)
        # the sampled rows of a full-size batch, drawn directly (the generator's
        # special rows sit at the frame starts, so sel's first rows are those)
        X = synth.activations(len(sel), K, seed=seed + 10 * j + 4)
        cases.append((X, pw, gelu))

    def run():
        for X, pw, gelu in cases:
            oracle.linear(X, pw, gelu=gelu)
    return run, len(sel), oracle.max_threads()


def time_stack_oracle(st, rows: int, budget_s: float, max_passes: int = 8):
    """The oracle's per-token rate on the stack: one block's four layer shapes
    on `rows` rows per pass, repeated until about budget_s of CPU time; the
    stack's time per token is 48 blocks' worth of that block's."""
    run, r, cores = stack_oracle_sample(st, rows)
    passes, t_total = 0, 0.0
    while passes < max_passes and (passes == 0 or t_total < budget_s):
        t = time.perf_counter()
        run()
        t_total += time.perf_counter() - t
        passes += 1
    t_block = t_total / passes
    M = st["frames"] * synth.FRAME_TOKENS
    sec_per_token = t_block * st["blocks"] / r
    tops = stack_ops(st, M) / M / sec_per_token / 1e12
    return tops, 1.0 / sec_per_token, r, passes, t_block, cores


def run_stack_reference(args, st, world, rank):
    """The reference arm on a multi-layer workload: the CPU oracle on a
    bounded row sample of one block's four layer shapes per step (the stack's
    rate is 48 blocks of that), sized so the whole run takes a few minutes."""
    if rank != 0:
        return
    run, r0, _ = stack_oracle_sample(st, 64)
    t = time.perf_counter()
    run()
    per_row = (time.perf_counter() - t) / r0
    rows = int(min(args.cpu_rows * 2, max(32, 150.0 / max(1, args.steps + args.warmup) / per_row)))
    run, r, cores = stack_oracle_sample(st, rows)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    t_block = (time.perf_counter() - t0) / args.steps
    M = st["frames"] * synth.FRAME_TOKENS
    sec_per_token = t_block * st["blocks"] / r
    tops = stack_ops(st, M) / M / sec_per_token / 1e12
    sample = (f"{r} of {M} token rows (special tokens included) through one block's four layer "
              f"shapes per step; the stack's rate is {st['blocks']} blocks of it (sampled, per-token rate)")
    line = {
        "impl": "reference", "metric": METRIC, "value": tops, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_block * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64/int64",
        "data": "synthetic", "tokens_per_s": 1.0 / sec_per_token,
        "config": {"workload": st["desc"], "M": M, "blocks": st["blocks"], "M_sampled": r,
                   "layers": [f"{n} {K}->{N}" for (n, K, N) in st["layers"]]},
        "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def int8_ceiling(dev, stream):
    """Dense int8 tensor-core throughput measured on this GPU by a library
    GEMM (cuBLASLt through torch._int_mm, 8192^3, s8 x s8 -> s32): the
    measured ceiling the GEMM's roofline fraction is also reported against.
    None when the library call is not available here."""
    import torch
    try:
        n = 8192
        a = torch.randint(-8, 8, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-8, 8, (n, n), dtype=torch.int8, device=dev).t()
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 20
        e0.record(stream)
        for _ in range(reps):
            torch._int_mm(a, b)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        del a, b
        return {"tops": 2.0 * n ** 3 / (ms * 1e-3) / 1e12, "ms": ms,
                "how": "torch._int_mm (cuBLASLt) s8 x s8 -> s32, 8192^3, 20 back-to-back calls"}
    except Exception as e:  # noqa: BLE001
        return {"tops": None, "why": f"{type(e).__name__}: {e}"[:200]}


def run_stack(args, st, world, rank, local):
    """A block (or stack of blocks) of quantized linears: one step = every
    layer once, in order, on one batch of M tokens."""
    import torch
    from w4a4_post_quantized_b200 import w4a4
    M = st["frames"] * synth.FRAME_TOKENS
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    layers = stack_layers(st)
    C = synth.calibration_rows(M)
    GOUT, UNP = w4a4.W4A4_FLAG_GELU_OUT, w4a4.W4A4_FLAG_UNPACKED

    # ------------------------------------------------------------ inputs (untimed)
    # every layer that reads the block's input stream (qkv, proj, fc1) gets a
    # fresh seeded heavy-tailed activation batch of its own, drawn on the
    # device; fc2 reads GELU(fc1's output) of its block (the MLP's own data
    # flow; fc1's GEMM epilogue applies the GELU).  Weights: fresh seeded
    # normal(0, 0.02^2) per layer, bias normal(0, 0.01^2), prepared untimed.
    seed0 = 100000 * rank
    X = {i: synth.activations_device(M, K, seed0 + i, dev)
         for i, (_, name, K, _) in enumerate(layers) if name != "fc2"}
    Ys = {name: torch.empty((M, N), dtype=torch.bfloat16, device=dev) for (name, K, N) in st["layers"]}
    pws = []
    for i, (b, name, K, N) in enumerate(layers):
        W = synth.weights_device(N, K, seed0 + 7 * i + 1, dev)
        bias = synth.bias_device(N, seed0 + 7 * i + 2, dev)
        if name == "fc2":   # calibration: the block's fc1 output (with its GELU) on the first frame
            Xc = w4a4.w4a4_linear_fused(X[i - 1][:C], pws[i - 1], flags=GOUT)
        else:
            Xc = X[i][:C]
        pws.append(w4a4.w4a4_prepare_weights(W, bias, Xc))
        del W, bias, Xc
    ws = torch.empty(max(w4a4.w4a4_workspace_bytes(M, K) for (_, _, K, _) in layers), dtype=torch.uint8,
                     device=dev)
    torch.cuda.synchronize()
    ops_step = stack_ops(st, M)

    def layer_input(i, name):
        return Ys["fc1"] if name == "fc2" else X[i]

    def run_layer(i, b, name, K, N):
        w4a4.w4a4_linear_fused(layer_input(i, name), pws[i], Y=Ys[name], workspace=ws,
                               flags=GOUT if name == "fc1" else 0)

    def step():
        for i, (b, name, K, N) in enumerate(layers):
            run_layer(i, b, name, K, N)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    w4a4.w4a4_clear_device_status()

    # ---------------------------------------------------------------- timed region
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        torch.cuda.nvtx.range_push("timed")
        for _ in range(args.steps):
            step()
        torch.cuda.nvtx.range_pop()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        # attribution step (not part of `value`): the same work as a step, the
        # fused call's two kernels launched separately (the quantize kernel's
        # one-per-byte codes into the workspace, then the GEMM) with CUDA
        # events on the launching stream around each, for every layer
        ws_q = ws[:M * 4096]
        st_off = ((M * 4096 + 255) // 256) * 256
        ws_s = ws[st_off:st_off + 4 * M].view(torch.float32)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in layers]
        for i, (b, name, K, N) in enumerate(layers):
            q = ws_q[:M * K].view(M, K)
            ev[i][0].record(stream)
            w4a4.w4a4_quantize_act(layer_input(i, name), pws[i].inv_smooth, UNP, qx=q, scale_tok=ws_s)
            ev[i][1].record(stream)
            w4a4.w4a4_linear_ex(q, ws_s, pws[i], flags=UNP | (GOUT if name == "fc1" else 0), Y=Ys[name])
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    status = w4a4.w4a4_get_device_status()
    elapsed_ms = max_over_ranks(world, t0.elapsed_time(t1))
    ms_step = elapsed_ms / args.steps
    value = world * ops_step * args.steps / (elapsed_ms * 1e-3) / 1e12
    q_ms = [e[0].elapsed_time(e[1]) for e in ev]
    g_ms = [e[1].elapsed_time(e[2]) for e in ev]
    # algorithmic bytes of the quantizer: X in, 4-bit codes out (half a byte
    # each), the steps; the fused call's route stores the codes one per byte
    # (M K bytes instead of M K / 2: the GEMM then reads them without widening)
    q_bytes = [2.5 * M * K + 4.0 * M for (_, _, K, _) in layers]
    q_moved = [3.0 * M * K + 4.0 * M for (_, _, K, _) in layers]
    g_ops = [2.0 * M * N * K for (_, _, K, N) in layers]
    peaks = load_peaks()
    int8_peak_burst = peaks["bf16"] * INT8_PER_BF16
    int8_peak = (peaks["bf16_sus"] or peaks["bf16"]) * INT8_PER_BF16   # kernels timed inside a long step
    per = {name: {"quantize_ms": 0.0, "gemm_ms": 0.0, "count": 0} for (name, _, _) in st["layers"]}
    for (b, name, K, N), tq_, tg_ in zip(layers, q_ms, g_ms):
        per[name]["quantize_ms"] += tq_
        per[name]["gemm_ms"] += tg_
        per[name]["count"] += 1

    # each kernel alone, per layer shape (block 0's weights and inputs): 10
    # back-to-back launches between CUDA events
    n_iso = 10
    per_layer = {}
    for i, (b, name, K, N) in enumerate(layers[:len(st["layers"])]):
        x = layer_input(i, name)
        gfl = UNP | (GOUT if name == "fc1" else 0)
        q = ws_q[:M * K].view(M, K)
        Yk = Ys[name]
        times = []
        for fn in (lambda: w4a4.w4a4_quantize_act(x, pws[i].inv_smooth, UNP, qx=q, scale_tok=ws_s),
                   lambda: w4a4.w4a4_linear_ex(q, ws_s, pws[i], flags=gfl, Y=Yk)):
            fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n_iso):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(max_over_ranks(world, e0.elapsed_time(e1)) / n_iso)
        tq_ms, tg_ms = times
        gtops = 2.0 * M * N * K / (tg_ms * 1e-3) / 1e12
        c = per[name]["count"]
        per_layer[name] = {
            "K": K, "N": N, "layers": c,
            "in_step_quantize_us": per[name]["quantize_ms"] / c * 1e3,
            "in_step_gemm_us": per[name]["gemm_ms"] / c * 1e3,
            "alone_quantize_us": tq_ms * 1e3, "alone_quantize_gbs": (2.5 * M * K + 4 * M) / (tq_ms * 1e-3) / 1e9,
            "alone_quantize_gbs_moved": (3.0 * M * K + 4 * M) / (tq_ms * 1e-3) / 1e9,
            "alone_gemm_us": tg_ms * 1e3, "alone_gemm_tops": gtops,
            "alone_gemm_frac_burst": gtops / int8_peak_burst}
    # M7 (the pages' +0.2 % for DSFQ over plain quantization): the fused call per
    # layer shape with the rotation and smoothing skipped (weights of the same
    # layers prepared plain), 10 calls each, summed over the stack's layers
    m7 = {"dsfq": 0.0, "plain": 0.0}
    for i, (b, name, K, N) in enumerate(layers[:len(st["layers"])]):
        x = layer_input(i, name)
        W = synth.weights_device(N, K, seed0 + 7 * i + 1, dev)
        bias = synth.bias_device(N, seed0 + 7 * i + 2, dev)
        pplain = w4a4.w4a4_prepare_weights(W, bias, None, flags=w4a4.W4A4_FLAG_PLAIN)
        for mode, p, fl in (("dsfq", pws[i], 0), ("plain", pplain, w4a4.W4A4_FLAG_PLAIN)):
            fl |= GOUT if name == "fc1" else 0
            fn = lambda: w4a4.w4a4_linear_fused(x, p, Y=Ys[name], workspace=ws, flags=fl)
            fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n_iso):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            m7[mode] += st["blocks"] * max_over_ranks(world, e0.elapsed_time(e1)) / n_iso
        del W, bias, pplain
    ceiling = int8_ceiling(dev, stream)

    # ------------------------------------------------------------- end to end
    # through the C ABI's host-buffer call: the stack's input comes from pinned
    # host memory into the first layer (w4a4_linear_fused_host, X on the host,
    # Y left on the device) and the last layer's output goes back to pinned host
    # memory (X on the device, Y on the host); the layers between run on the
    # device.  Copies overlap those two layers' kernels chunk by chunk.
    chunk = args.e2e_chunk
    Xh = torch.empty((M, layers[0][2]), dtype=torch.bfloat16, pin_memory=True)
    Xh.copy_(X[0].cpu())
    last = len(layers) - 1
    Yh = torch.empty((M, layers[last][3]), dtype=torch.bfloat16, pin_memory=True)
    pipe = w4a4.HostPipe()
    hws = torch.empty(max(w4a4.w4a4_host_workspace_bytes(chunk, K, N) for (_, _, K, N) in layers),
                      dtype=torch.uint8, device=dev)

    def host_step():
        for i, (b, name, K, N) in enumerate(layers):
            fl = GOUT if name == "fc1" else 0
            if i == 0:
                w4a4.w4a4_linear_fused_host(Xh, pws[i], Y_host=Ys[name], chunk_rows=chunk, workspace=hws,
                                            pipe=pipe, flags=fl | w4a4.W4A4_FLAG_Y_DEVICE)
            elif i == last:
                w4a4.w4a4_linear_fused_host(layer_input(i, name), pws[i], Y_host=Yh, chunk_rows=chunk,
                                            workspace=hws, pipe=pipe, flags=fl | w4a4.W4A4_FLAG_X_DEVICE)
            else:
                run_layer(i, b, name, K, N)
    n_e2e = max(3, min(args.steps, args.e2e_steps))
    host_step()
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a0.record(stream)
    for _ in range(n_e2e):
        host_step()
    a1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    pipe.close()
    e2e_ms = max_over_ranks(world, a0.elapsed_time(a1)) / n_e2e

    # ------------------------------------------------------------- roofline
    g_total_ms, q_total_ms = sum(g_ms), sum(q_ms)
    g_ach = sum(g_ops) / (g_total_ms * 1e-3) / 1e12
    q_ach = sum(q_bytes) / (q_total_ms * 1e-3) / 1e9
    nominal_int8 = 4500.0
    roofline = {
        "bound": "tensor", "kernel": "w4a4_gemm_kernel", "achieved": g_ach, "peak": int8_peak,
        "unit": "TOPS", "frac": g_ach / int8_peak,
        "traffic": profile_traffic("gemm.cu", f"gemm_{args.workload}"),
        "peak_note": f"int8 = {INT8_PER_BF16:g} x {peaks['src']} sustained bf16 {peaks['bf16_sus']} TFLOP/s "
                     "(the kernel runs inside a 66 ms step under the power cap)",
        "frac_of_nominal_4500": g_ach / nominal_int8,
        "frac_of_measured_int8_ceiling": (g_ach / ceiling["tops"]) if ceiling.get("tops") else None,
        "measured_int8_ceiling": ceiling,
        "ms_per_launch": g_total_ms / len(layers), "launches_per_step": len(layers),
        "algorithmic_ops_per_launch": sum(g_ops) / len(layers),
        "timing": "CUDA events on the launching stream around each GEMM launch of one step "
                  "(time-weighted: sum of ops / sum of launch durations)"}
    roofline_q = {
        "bound": "hbm", "kernel": "quant_tc_kernel", "achieved": q_ach, "peak": peaks["hbm"],
        "unit": "GB/s", "frac": q_ach / peaks["hbm"],
        "traffic": profile_traffic("quant_tc.cu", f"quant_{args.workload}"),
        "ms_per_launch": q_total_ms / len(layers), "algorithmic_bytes_per_launch": sum(q_bytes) / len(layers),
        "bytes_moved_per_launch": sum(q_moved) / len(layers),
        "achieved_moved": sum(q_moved) / (q_total_ms * 1e-3) / 1e9,
        "bytes_note": "algorithmic = 2 M K (X) + M K / 2 (4-bit codes) + 4 M (steps); moved: the codes "
                      "go one per byte on the fused call's route (3 M K + 4 M)"}
    # the same kernel launched alone (per layer shape, back to back), weighted
    # by the step's layers: in the step each launch also pays for the write-back
    # of the GEMM output that the previous launch left dirty in L2
    q_alone_ms = sum(per_layer[name]["alone_quantize_us"] * 1e-3 for (_, name, _, _) in layers)
    roofline_q.update({
        "achieved_alone": sum(q_bytes) / (q_alone_ms * 1e-3) / 1e9,
        "frac_alone": sum(q_bytes) / (q_alone_ms * 1e-3) / 1e9 / peaks["hbm"],
        "frac_alone_moved": sum(q_moved) / (q_alone_ms * 1e-3) / 1e9 / peaks["hbm"],
        "timing": "frac: CUDA events around each quantize launch of one step (time-weighted); "
                  "frac_alone: each layer shape's kernel alone, 10 back-to-back launches"})
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s4xs4->s32 (bf16 in/out, fp32 transform)",
        "data": "synthetic (seeded heavy-tailed activations, a fresh batch per layer; seeded normal weights "
                "per layer; drawn on the device)",
        "tokens_per_s": world * M * args.steps / (elapsed_ms * 1e-3),
        "config": {"workload": st["desc"], "M": M, "blocks": st["blocks"],
                   "layers": [f"{n} {K}->{N}" for (n, K, N) in st["layers"]],
                   "parallelism": f"dp{world} (independent replicas)",
                   "l2": "every layer reads its own input batch (>= 180 MB, larger than L2)"},
        "clocks": clk.summary(),
        "e2e": {"value": world * ops_step / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": 2 * M * layers[0][2], "d2h_bytes_per_step": 2 * M * layers[last][3],
                "api": f"w4a4_linear_fused_host (C ABI) for the first layer (X from pinned host memory) and "
                       f"the last (Y to pinned host memory), {chunk}-row chunks; w4a4_linear_fused between"},
        "gpu_launches": 2 * len(layers) * args.steps,
        "roofline": roofline,
        "roofline_quantize": roofline_q,
        "per_layer": per_layer,
        "dsfq_overhead": {"dsfq_ms_per_step": m7["dsfq"], "plain_ms_per_step": m7["plain"],
                          "overhead_pct": 100.0 * (m7["dsfq"] - m7["plain"]) / m7["plain"],
                          "pages_figure_pct": 0.2,
                          "how": f"fused call per layer shape, {n_iso} calls each, x {st['blocks']} blocks"},
        "device_status": status,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        tops, tps, r, passes, t_block, cores = time_stack_oracle(st, 1024, budget_s=10.0)
        line["cpu_baseline"] = {
            "value": tops, "unit": "TOPS", "cores": cores, "kind": "oracle", "tokens_per_s": tps,
            "sample": f"sampled, per-token rate: {r} token rows (special tokens included) through one "
                      f"block's four layer shapes, {passes} passes, {t_block:.2f} s per pass; the stack is "
                      f"{st['blocks']} blocks of it"}
    if rank == 0:
        print(json.dumps(line), flush=True)


TQ_WORKLOAD = "kv_turboquant"
TQ_METRIC = "3DTurboQuant KV-cache codec GB/s (encode + decode, algorithmic bytes), % of HBM BW"


def tq_bytes(n: int, d: int):
    """Algorithmic bytes of one encode and one decode of n vectors (fp32 in and
    out, 4-bit codes + fp32 norm)."""
    packed = n * (d // 2 + 4)
    return n * 4 * d + packed, packed + n * 4 * d


TQ_PI_SEED = 77   # seed of the Gaussian matrix whose QR factor is the rotation


def tq_oracle_sample(rows: int, seed: int = 0):
    """The oracle's encode + decode with the page's rotation (Q of a Gaussian
    matrix) on `rows` KV vectors (untimed setup)."""
    from oracle import turboquant as tq
    d = synth.KV_DIM
    X = synth.kv_vectors(rows, d, seed=seed + 10)
    P = tq.rotation_qr(synth.gaussian_matrix(d, seed=TQ_PI_SEED))
    c, t = tq.lloyd_max(d, 4)

    def run():
        codes, gamma, _ = tq.encode(X, P, t)
        return tq.decode(codes, gamma, P, c)
    import oracle
    return run, rows, oracle.max_threads()


def run_tq(args, world, rank, local):
    """The 3DTurboQuant KV-cache codec on the page's DUSt3R case: 24576 vectors
    of d = 1024 (100.7 MB of fp32), b = 4; a step encodes and decodes one batch
    with the page's rotation (the Q factor of a Gaussian matrix, a dense
    product on the tensor cores).  The signed-Hadamard fast variant is timed
    beside it."""
    import torch
    from w4a4_post_quantized_b200 import w4a4
    n, d = synth.KV_VECTORS, synth.KV_DIM
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    c, t = w4a4.tq_codebook(d, 4)
    cd, td = torch.from_numpy(c).to(dev), torch.from_numpy(t).to(dev)
    seed = 1000 * rank
    # the rotation: QR on the host, once (untimed, like weight preparation)
    hi, lo, thi, tlo = [torch.from_numpy(a).to(dev)
                        for a in w4a4.tq_rotation_qr(synth.gaussian_matrix(d, seed=TQ_PI_SEED))]
    sg = torch.from_numpy(synth.random_signs(d, seed=seed + 2)).to(dev)
    Xs = [torch.from_numpy(synth.kv_vectors(n, d, seed=seed + 10 + i)).to(dev) for i in range(NSETS)]
    Cs = [torch.empty((n, d // 2), dtype=torch.uint8, device=dev) for _ in range(NSETS)]
    Ns = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(NSETS)]
    Ys = [torch.empty((n, d), dtype=torch.float32, device=dev) for _ in range(NSETS)]
    enc = lambda j: w4a4.tq_encode_dense(Xs[j], hi, lo, td, codes=Cs[j], norms=Ns[j])
    dec = lambda j: w4a4.tq_decode_dense(Cs[j], Ns[j], thi, tlo, cd, Y=Ys[j])
    fenc = lambda j: w4a4.tq_encode(Xs[j], sg, td, codes=Cs[j], norms=Ns[j])
    fdec = lambda j: w4a4.tq_decode(Cs[j], Ns[j], sg, cd, Y=Ys[j])

    def step(i):
        enc(i % NSETS)
        dec(i % NSETS)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    w4a4.w4a4_clear_device_status()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        torch.cuda.nvtx.range_push("timed")
        for i in range(args.steps):
            step(i)
        torch.cuda.nvtx.range_pop()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        iso = {}
        n_iso = max(3, min(args.steps, 200))
        for name, fn in (("encode", enc), ("decode", dec), ("fast_encode", fenc), ("fast_decode", fdec)):
            for i in range(3):
                fn(i % NSETS)
            k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            k0.record(stream)
            for i in range(n_iso):
                fn(i % NSETS)
            k1.record(stream)
            torch.cuda.synchronize()
            iso[name] = max_over_ranks(world, k0.elapsed_time(k1)) / n_iso
    status = w4a4.w4a4_get_device_status()
    elapsed_ms = max_over_ranks(world, t0.elapsed_time(t1))
    ms_step = elapsed_ms / args.steps
    be, bd = tq_bytes(n, d)
    value = world * (be + bd) * args.steps / (elapsed_ms * 1e-3) / 1e9
    # reconstruction quality of batch 0 against the page's bound, both variants
    bound = math.sqrt(3.0) * math.pi / 2.0 * 4.0 ** -4
    X64 = Xs[0].double()
    quality = {}
    for name, (e_, d_) in (("page_rotation", (enc, dec)), ("fast_variant", (fenc, fdec))):
        e_(0)
        d_(0)
        torch.cuda.synchronize()
        rel = (((X64 - Ys[0].double()) ** 2).sum(1) / (X64 ** 2).sum(1))
        quality[name] = {"mse_rel_mean": float(rel.mean()), "mse_rel_max": float(rel.max())}
    quality.update({"page_bound": bound, "compression_vs_fp32": (4 * n * d) / (n * (d // 2) + 4 * n)})
    # end to end: X from pinned host memory, encode + decode, Y back to pinned host memory
    Xh = Xs[0].cpu().pin_memory()
    Yh = torch.empty((n, d), dtype=torch.float32, pin_memory=True)
    Xd, Yd = torch.empty_like(Xs[0]), torch.empty_like(Ys[0])

    def host_step():
        Xd.copy_(Xh, non_blocking=True)
        w4a4.tq_encode_dense(Xd, hi, lo, td, codes=Cs[0], norms=Ns[0])
        w4a4.tq_decode_dense(Cs[0], Ns[0], thi, tlo, cd, Y=Yd)
        Yh.copy_(Yd, non_blocking=True)
    for _ in range(3):
        host_step()
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    a0.record(stream)
    for _ in range(e2e_steps):
        host_step()
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, a0.elapsed_time(a1)) / e2e_steps
    peaks = load_peaks()
    # the dense codec is a contraction: 2 n d^2 flops per kernel (the method's
    # product), run as three tf32 products for fp32-level accuracy; its peak is
    # the tf32 rate = the measured bf16 burst x the nominal tf32 : bf16 ratio
    tf32_peak = peaks["bf16"] * TF32_PER_BF16
    kern = "encode" if iso["encode"] >= iso["decode"] else "decode"
    kms = iso[kern]
    flops = 2.0 * n * d * d
    ach = flops / (kms * 1e-3) / 1e12
    line = {
        "metric": TQ_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 in/out, u4 codes, tf32x3 products", "data": "synthetic",
        "vectors_per_s": world * n * args.steps / (elapsed_ms * 1e-3),
        "config": {"workload": "3DTurboQuant DUSt3R KV cache: 24576 x 1024 fp32 (100.7 MB), b = 4, "
                               "the page's rotation (Q of a seeded Gaussian matrix)",
                   "n": n, "d": d, "bits": 4, "per_rank_batch": n,
                   "parallelism": f"dp{world} (independent replicas)",
                   "l2": f"inputs/outputs rotated over {NSETS} buffer sets (~{(8 * n * d + n * d // 2) * NSETS / 1e6:.0f} MB > L2)"},
        "clocks": clk.summary(),
        "e2e": {"value": world * (be + bd) / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": 4 * n * d, "d2h_bytes_per_step": 4 * n * d,
                "api": "tq_encode_dense + tq_decode_dense (C ABI) with X copied from and Y copied to pinned host memory"},
        "gpu_launches": 2 * args.steps,
        "roofline": {"bound": "tensor", "kernel": f"tq_dense_kernel ({kern})", "achieved": ach,
                     "peak": tf32_peak, "unit": "TFLOP/s", "frac": ach / tf32_peak,
                     "traffic": None, "ms_per_launch": kms, "algorithmic_flops_per_launch": flops,
                     "executed_tflops_3_terms": 3 * ach,
                     "peak_note": f"tf32 = {TF32_PER_BF16:.3f} x {peaks['src']} bf16 burst {peaks['bf16']} TFLOP/s "
                                  "(nominal 1.1 : 2.25 PFLOP/s)",
                     "encode_ms": iso["encode"], "decode_ms": iso["decode"],
                     "timing": f"CUDA events around {n_iso} back-to-back launches of each kernel alone"},
        "fast_variant": {
            "what": "tq_encode / tq_decode: Pi = H diag(s) / sqrt(d) (signed Hadamard, not the page's matrix), "
                    "HBM-bound", "encode_ms": iso["fast_encode"], "decode_ms": iso["fast_decode"],
            "encode_gbs": be / (iso["fast_encode"] * 1e-3) / 1e9,
            "decode_gbs": bd / (iso["fast_decode"] * 1e-3) / 1e9,
            "encode_frac_hbm": be / (iso["fast_encode"] * 1e-3) / 1e9 / peaks["hbm"],
            "decode_frac_hbm": bd / (iso["fast_decode"] * 1e-3) / 1e9 / peaks["hbm"]},
        "quality": quality,
        "device_status": status,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        run, r, cores = tq_oracle_sample(256)
        passes, tt = 0, 0.0
        while passes < 2000 and tt < 10.0:  # about 10 s of CPU work
            t_ = time.perf_counter()
            run()
            tt += time.perf_counter() - t_
            passes += 1
        dt = tt / passes
        eb, db = tq_bytes(r, d)
        line["cpu_baseline"] = {"value": (eb + db) / dt / 1e9, "unit": "GB/s", "cores": cores,
                                "kind": "oracle", "sample": f"{r} of {n} vectors per pass, {passes} passes, "
                                                            f"{dt:.2f} s per pass"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_tq_reference(args, world, rank):
    if rank != 0:
        return
    d = synth.KV_DIM
    probe, r0, _ = tq_oracle_sample(64)
    t_ = time.perf_counter()
    probe()
    per_vec = (time.perf_counter() - t_) / r0
    rows = int(min(1024, max(16, 120.0 / max(1, args.steps + args.warmup) / per_vec)))
    run, r, cores = tq_oracle_sample(rows)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = (time.perf_counter() - t0) / args.steps
    eb, db = tq_bytes(r, d)
    gbs = (eb + db) / dt / 1e9
    line = {"impl": "reference", "metric": TQ_METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "3DTurboQuant DUSt3R KV cache: 24576 x 1024 fp32 (100.7 MB), b = 4, "
                                   "the page's rotation (Q of a seeded Gaussian matrix)",
                       "n": synth.KV_VECTORS, "d": d, "bits": 4, "n_sampled": r},
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"{r} of {synth.KV_VECTORS} vectors per step"},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 20 for the multi-layer workloads, 2000 otherwise)")
    ap.add_argument("--warmup", type=int, default=None, help="warm-up steps (default: 3 / 20)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(STACKS) + [TQ_WORKLOAD],
                    default="c5_full_stack")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--e2e-chunk", type=int, default=1408, help="row chunk of the host-buffer call")
    ap.add_argument("--cpu-rows", type=int, default=512)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    multi = args.workload in STACKS
    if args.steps is None:
        args.steps = 20 if multi else 2000
    if args.warmup is None:
        args.warmup = 3 if multi else 20
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.workload == TQ_WORKLOAD:
        if args.impl == "reference":
            run_tq_reference(args, world, rank)
            return
        world, rank, local = dist_setup()
        try:
            run_tq(args, world, rank, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    if args.workload in STACKS:
        if args.impl == "reference":
            run_stack_reference(args, STACKS[args.workload], world, rank)
            return
        world, rank, local = dist_setup()
        try:
            run_stack(args, STACKS[args.workload], world, rank, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, wl, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
