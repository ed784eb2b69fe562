#!/usr/bin/env python
"""Benchmark of the factorised binary low-rank linear, y = s1 * (U (V^T (s2 * x))).

Default workload (one "step"): the seven linears of a Llama-2-7B-shaped block
(q/k/v/o 4096x4096 r=1664, gate/up 11008x4096 r=2432, down 4096x11008 r=2432) at decode
batch 1, each layer with its own seeded input, all through the C ABI
(nq_lowrank_linear_fwd) on one stream, the whole run captured in CUDA graphs.
Metric: packed-weight HBM GB/s = (packed sign bytes of the seven layers) x steps / time.
The weights rotate over enough seeded copies (> 2x the 126 MB L2) that every step
streams its signs from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (independent replicas, one per GPU)

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead
(rank 0 only) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from binary_rank_linear_02_b200 import synth  # noqa: E402

METRIC = "packed-weight HBM GB/s (decode) & TFLOP/s (prefill), binary low-rank linear"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def packed_bytes(m, n, r):
    return r * (m + n) // 8


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks during the timed region

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="nq_clocks_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # wait (up to 3 s) for the first sample, so the timed region is covered
        t0 = time.time()
        while time.time() - t0 < 3.0:
            self.fh.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons, n = [], [], set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                n += 1
                for name, flag in zip(names, parts[5:9]):
                    if flag.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": n}


# ------------------------------------------------------------------ the decode workload on the GPU

class DecodeWorkload:
    """Seven factorised linears per step, weights rotating over `copies` seeded sets."""

    def __init__(self, layers, batch, seed, device, min_bytes=2 * L2_BYTES):
        import torch

        from binary_rank_linear_02_b200 import nq

        self.nq = nq
        self.layers = layers
        self.batch = batch
        self.step_bytes = sum(packed_bytes(m, n, r) for _, m, n, r in layers)
        self.copies = max(1, -(-min_bytes // self.step_bytes))
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
        self.sets = []
        for c in range(self.copies):
            per = []
            for li, (name, m, n, r) in enumerate(layers):
                Upk = torch.randint(-(1 << 31), 1 << 31, (m, r // 32), dtype=torch.int64, device=device,
                                    generator=gen).to(torch.int32)
                Vpk = torch.randint(-(1 << 31), 1 << 31, (r, n // 32), dtype=torch.int64, device=device,
                                    generator=gen).to(torch.int32)
                s1 = torch.from_numpy(synth.scales_f16(m, seed, c, li, "s1").view(np.int16)).to(device)
                s2 = torch.from_numpy(synth.scales_f16(n, seed, c, li, "s2").view(np.int16)).to(device)
                per.append((Upk, Vpk, s1, s2))
            self.sets.append(per)
        self.x = [torch.from_numpy(synth.activations_bf16(batch, n, seed, li, "x").view(np.int16)).to(device)
                  for li, (_, m, n, r) in enumerate(layers)]
        self.y = [torch.empty((batch, m), dtype=torch.float32, device=device) for (_, m, n, r) in layers]
        for (_, m, n, r) in layers:
            nq.workspace_reserve(m, n, r, batch)
        # one grouped descriptor array per weight copy (kept alive for graph replays)
        self.descs = [nq.make_descs([(self.x[li], *per[li][:2], *per[li][2:], self.y[li], m, n, r)
                                     for li, (_, m, n, r) in enumerate(layers)]) for per in self.sets]
        self.grouped = True

    def step(self, i, stream_handle, layer_filter=None):
        """One pass over the layers: one grouped call, or one call per layer."""
        per = self.sets[i % self.copies]
        if self.grouped and layer_filter is None:
            arr = self.descs[i % self.copies]
            st = self.nq.lib().nq_lowrank_linear_fwd_grouped(ctypes.addressof(arr), len(self.layers), self.batch,
                                                               stream_handle)
            if st != 0:
                raise RuntimeError(f"nq_lowrank_linear_fwd_grouped: {self.nq.nq_status_string(st)}")
            return
        fwd = self.nq.lib().nq_lowrank_linear_fwd
        for li, (name, m, n, r) in enumerate(self.layers):
            if layer_filter is not None and li != layer_filter:
                continue
            Upk, Vpk, s1, s2 = per[li]
            st = fwd(self.x[li].data_ptr(), Upk.data_ptr(), Vpk.data_ptr(), s1.data_ptr(), s2.data_ptr(),
                     m, n, r, self.batch, self.y[li].data_ptr(), stream_handle)
            if st != 0:
                raise RuntimeError(f"nq_lowrank_linear_fwd: {self.nq.nq_status_string(st)}")


def backward_workload(layers, batch, seed, device):
    """The input gradient of the same layers, one grouped call per step: each layer's
    forward packings are transposed on the device (nq_transpose_signs) and the grouped
    forward call runs with the factors' roles exchanged (U' = V, V' = U, s1' = s2,
    s2' = s1, m' = n, n' = m), which is what nq_lowrank_linear_bwd_input does per layer."""
    import torch

    work = DecodeWorkload(layers, batch, seed, device)
    nq = work.nq
    work.dy = [torch.from_numpy(synth.activations_bf16(batch, m, seed, li, "dy").view(np.int16)).to(device)
               for li, (_, m, n, r) in enumerate(layers)]
    work.dx = [torch.empty((batch, n), dtype=torch.float32, device=device) for (_, m, n, r) in layers]
    work.transposed = []  # kept alive for graph replays
    descs = []
    for per in work.sets:
        entries = []
        for li, (_, m, n, r) in enumerate(layers):
            Upk, Vpk, s1, s2 = per[li]
            UpkT = nq.transpose_signs(Upk, m, r)
            VpkT = nq.transpose_signs(Vpk, r, n)
            work.transposed += [UpkT, VpkT]
            entries.append((work.dy[li], VpkT, UpkT, s2, s1, work.dx[li], n, m, r))
        descs.append(nq.make_descs(entries))
    for (_, m, n, r) in layers:
        nq.workspace_reserve(n, m, r, batch)
    torch.cuda.synchronize()
    work.descs = descs
    return work


def aggregate(ms_local: float, units_local: float, dist=None, device=None):
    """Whole-job numbers of independent replicas: (max time over ranks, units of all ranks).

    Each rank timed its own K steps on its own device; the job took as long as the slowest
    rank, and did the work of all of them.  Works over NCCL (device tensors) or gloo.
    """
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return ms_local, units_local
    import torch

    t = torch.tensor([ms_local, units_local], dtype=torch.float64, device=device)
    ms = t[:1].clone()
    units = t[1:].clone()
    dist.all_reduce(ms, op=dist.ReduceOp.MAX)
    dist.all_reduce(units, op=dist.ReduceOp.SUM)
    return float(ms.item()), float(units.item())


def capture(fn, stream):
    import torch

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        fn(torch.cuda.current_stream().cuda_stream)
    return g


def timed_graphs(work, steps, warmup, stream, layer_filter=None, dist=None):
    """Capture graphs covering `steps` steps (rotating copies) and time them with events."""
    import torch

    full = capture(lambda h: [work.step(i, h, layer_filter) for i in range(work.copies)], stream)
    rem = steps % work.copies
    part = capture(lambda h: [work.step(i, h, layer_filter) for i in range(rem)], stream) if rem else None
    reps = steps // work.copies
    for _ in range(max(1, -(-warmup // work.copies))):
        full.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(reps):
            full.replay()
        if part is not None:
            part.replay()
        end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    if dist is not None:
        dist.barrier()
    del full, part
    return ms


def run_ours(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
        dist = tdist
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from binary_rank_linear_02_b200 import nq

    peaks = load_peaks()
    if args.workload == "prefill":
        return run_prefill_only(args, device, peaks)
    if args.workload == "chain7b":
        return run_chain_only(args, device, peaks)
    layers = synth.LLAMA2_70B_LAYERS if args.workload == "decode70b" else synth.LLAMA2_7B_LAYERS
    model = "llama2-70b" if args.workload == "decode70b" else "llama2-7b"
    batch = args.batch
    work = DecodeWorkload(layers, batch, seed=1234 + rank, device=device)
    stream = torch.cuda.Stream(device)
    # first calls outside capture (kernel attributes, workspace)
    with torch.cuda.stream(stream):
        work.step(0, stream.cuda_stream)
    torch.cuda.synchronize()

    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local)
    sampler.start()
    ms = timed_graphs(work, args.steps, args.warmup, stream, dist=dist)
    clocks = sampler.stop()
    ms_max, total_bytes = aggregate(ms, float(work.step_bytes * args.steps), dist, device)
    value = total_bytes / (ms_max * 1e-3) / 1e9
    tokens_per_s = batch * args.steps * world / (ms_max * 1e-3)

    # roofline: the kernels of the headline step (the stage-1 and stage-2 kernels of one
    # grouped call, timed live above), against the measured HBM copy bandwidth
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if os.path.exists(tpath) and batch == 1 and args.workload == "decode7b":
        import hashlib

        with open(tpath) as f:
            rec = json.load(f)
        with open(os.path.join(ROOT, rec["kernel_source"])) as f:
            code = f.read()
        # the source with comments and white space removed: counters are only valid for the
        # kernel code they were taken from
        code = re.sub(r"/\*.*?\*/", "", code, flags=re.S)
        code = "".join(re.sub(r"//[^\n]*", "", code).split())
        if hashlib.sha256(code.encode()).hexdigest()[:16] == rec["kernel_code_sha256_16"]:
            traffic = rec["dram_bytes_per_step_b1"]
    achieved = value / world
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                "kernel": f"stage1_kernel + stage2_kernel of one grouped call ({work.step_bytes} packed bytes "
                          "per launch pair), per-GPU",
                "peak_source": peaks["source"]}

    # the largest layer (gate) alone, back to back over its own rotating copies
    gate = [l for l in layers if l[0] == "gate"][0]
    _, gm, gn, gr = gate
    gwork = DecodeWorkload([gate], batch, seed=777 + rank, device=device)
    with torch.cuda.stream(stream):
        gwork.step(0, stream.cuda_stream)
    torch.cuda.synchronize()
    r_steps = max(gwork.copies * 10, 500)
    ms_gate = timed_graphs(gwork, r_steps, args.warmup, stream)
    del gwork
    gate_gbs = packed_bytes(gm, gn, gr) * r_steps / (ms_gate * 1e-3) / 1e9

    # end to end through the public API with host buffers (pinned), synchronous per call
    e2e = run_e2e(work, stream, min(args.steps, 100), device)

    # secondary: the same step as seven separate nq_lowrank_linear_fwd calls; batch 8
    secondary = {"decode_%s_gate_alone_b%d_gbs" % (model, batch): round(gate_gbs, 1)}
    if args.secondary and world == 1:
        work.grouped = False
        ms1 = timed_graphs(work, args.steps, args.warmup, stream)
        work.grouped = True
        secondary["decode_b%d_per_layer_calls_gbs" % batch] = round(work.step_bytes * args.steps / (ms1 * 1e-3) / 1e9, 1)
    if args.secondary and batch == 1 and world == 1 and args.workload == "decode7b":
        for b70 in (1, 4):  # the Llama-2-70B-shaped block, batch 1 and 4
            w70 = DecodeWorkload(synth.LLAMA2_70B_LAYERS, b70, seed=70 + b70, device=device)
            with torch.cuda.stream(stream):
                w70.step(0, stream.cuda_stream)
            torch.cuda.synchronize()
            st70 = max(w70.copies, min(args.steps, 400) // w70.copies * w70.copies)
            ms70 = timed_graphs(w70, st70, args.warmup, stream)
            secondary["decode70b_b%d_gbs" % b70] = round(w70.step_bytes * st70 / (ms70 * 1e-3) / 1e9, 1)
            secondary["decode70b_b%d_tokens_per_s" % b70] = round(b70 * st70 / (ms70 * 1e-3), 1)
            del w70
        w8 = DecodeWorkload(layers, 8, seed=99, device=device)
        with torch.cuda.stream(stream):
            w8.step(0, stream.cuda_stream)
        torch.cuda.synchronize()
        ms8 = timed_graphs(w8, args.steps, args.warmup, stream)
        secondary["decode_b8_gbs"] = round(w8.step_bytes * args.steps / (ms8 * 1e-3) / 1e9, 1)
        secondary["decode_b8_tokens_per_s"] = round(8 * args.steps / (ms8 * 1e-3), 1)
        del w8
        # 16 tokens in one grouped call of the block (the decode kernels over two token chunks)
        w16 = DecodeWorkload(layers, 16, seed=116, device=device)
        with torch.cuda.stream(stream):
            w16.step(0, stream.cuda_stream)
        torch.cuda.synchronize()
        ms16 = timed_graphs(w16, args.steps, args.warmup, stream)
        secondary["grouped_b16_us_per_call"] = round(ms16 * 1e3 / args.steps, 2)
        secondary["grouped_b16_tokens_per_s"] = round(16 * args.steps / (ms16 * 1e-3), 1)
        del w16
        # the input gradient dx = W^T dy of the same block (backward of the layers)
        for bb in (1, 8):
            wb = backward_workload(layers, bb, seed=123 + bb, device=device)
            with torch.cuda.stream(stream):
                wb.step(0, stream.cuda_stream)
            torch.cuda.synchronize()
            msb = timed_graphs(wb, args.steps, args.warmup, stream)
            secondary["backward_input_b%d_gbs" % bb] = round(wb.step_bytes * args.steps / (msb * 1e-3) / 1e9, 1)
            del wb

    if args.secondary and world == 1:
        secondary["prefill_11008x4096_r2432"] = run_prefill_sweep(device, stream, args.warmup, peaks)
    if args.secondary and world == 1 and batch == 1 and args.workload == "decode7b":
        secondary["chain_llama2-7b_32_blocks_b1"] = run_chain(device, stream, args.warmup, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(layers, batch, budget_s=args.cpu_seconds)

    launches = args.steps * 2  # stage-1 and stage-2 kernels of one grouped call per step
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in; int8x2-limb tensor-core products, int32/fp32 acc",
            "data": "synthetic",
            "config": {"workload": f"{model}-shaped decode, batch {batch}: 7 factorised linears per step "
                                   f"({', '.join(f'{nm} {m}x{n} r{r}' for nm, m, n, r in layers)}), "
                                   "one nq_lowrank_linear_fwd_grouped call per step",
                       "batch": batch, "packed_bytes_per_step": work.step_bytes,
                       "l2": f"weights rotate over {work.copies} seeded copies "
                             f"({work.copies * work.step_bytes / 1e6:.0f} MB > 2x L2)",
                       "graphs": "CUDA graphs of the C-ABI calls", "parallelism": f"replicas x{world}"},
            "tokens_per_s": round(tokens_per_s, 1),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    del work
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_prefill_sweep(device, stream, warmup, peaks, calls=20, batches=synth.PREFILL_BATCHES):
    """Config-4 sweep: the 11008x4096 r=2432 layer at token batches 16..4096 (tcgen05 path)."""
    import torch

    from binary_rank_linear_02_b200 import nq

    _, m, n, r = synth.PREFILL_SHAPE
    gen = torch.Generator(device=device)
    gen.manual_seed(4242)
    Upk = torch.randint(-(1 << 31), 1 << 31, (m, r // 32), dtype=torch.int64, device=device, generator=gen).to(torch.int32)
    Vpk = torch.randint(-(1 << 31), 1 << 31, (r, n // 32), dtype=torch.int64, device=device, generator=gen).to(torch.int32)
    s1 = torch.from_numpy(synth.scales_f16(m, 4242, "s1").view(np.int16)).to(device)
    s2 = torch.from_numpy(synth.scales_f16(n, 4242, "s2").view(np.int16)).to(device)
    out = {}
    for b in batches:
        x = torch.from_numpy(synth.activations_bf16(b, n, 4242, b).view(np.int16)).to(device)
        y = torch.empty((b, m), dtype=torch.float32, device=device)
        nq.workspace_reserve(m, n, r, b)
        fwd = nq.lib().nq_lowrank_linear_fwd

        def one(h):
            st = fwd(x.data_ptr(), Upk.data_ptr(), Vpk.data_ptr(), s1.data_ptr(), s2.data_ptr(), m, n, r, b,
                     y.data_ptr(), h)
            if st != 0:
                raise RuntimeError(nq.nq_status_string(st))

        with torch.cuda.stream(stream):
            one(stream.cuda_stream)
        torch.cuda.synchronize()
        g = capture(lambda h: [one(h) for _ in range(calls)], stream)
        for _ in range(max(1, warmup // calls)):
            g.replay()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(reps):
                g.replay()
            end.record(stream)
        torch.cuda.synchronize()
        nq.device_status(stream.cuda_stream)
        ms = start.elapsed_time(end) / (reps * calls)
        flops = 2.0 * b * r * (m + n)
        tf = flops / (ms * 1e-3) / 1e12
        out[str(b)] = {"tflops": round(tf, 1), "us_per_call": round(ms * 1e3, 2),
                       "frac_of_bf16_burst": round(tf / peaks["bf16_tflops"], 4),
                       "tokens_per_s": round(b / (ms * 1e-3), 1)}
        del g, x, y
    return out


def run_chain(device, stream, warmup, peaks, passes=20, batch=1, nblocks=synth.CHAIN_7B_BLOCKS):
    """The decode chain: 32 Llama-2-7B-shaped blocks x 7 factorised linears at batch 1, per
    block two grouped forward calls, one cast and one RMS normalisation (6 kernels).  659 MB
    of packed weights per pass (> 5x L2), so every pass streams its weights from HBM."""
    import torch

    from binary_rank_linear_02_b200 import chain

    gen = torch.Generator(device=device)
    gen.manual_seed(5150)
    blocks = []
    for b in range(nblocks):
        w = {}
        for li, (name, m, n, r) in enumerate(synth.LLAMA2_7B_LAYERS):
            Upk = torch.randint(-(1 << 31), 1 << 31, (m, r // 32), dtype=torch.int64, device=device,
                                generator=gen).to(torch.int32)
            Vpk = torch.randint(-(1 << 31), 1 << 31, (r, n // 32), dtype=torch.int64, device=device,
                                generator=gen).to(torch.int32)
            s1 = torch.from_numpy(synth.scales_f16(m, 5150, b, li, "s1").view(np.int16)).to(device)
            s2 = torch.from_numpy(synth.scales_f16(n, 5150, b, li, "s2").view(np.int16)).to(device)
            w[name] = (Upk, Vpk, s1, s2, m, n, r)
        blocks.append(w)
    ch = chain.DecodeChain(blocks, batch)
    h0 = torch.from_numpy(synth.activations_bf16(batch, ch.d, 5150, "h0").view(np.int16)).to(device)
    ch.h[0].copy_(h0)
    with torch.cuda.stream(stream):
        ch.run(stream=stream.cuda_stream)
    torch.cuda.synchronize()
    g = capture(lambda h: ch.run(stream=h), stream)
    for _ in range(max(3, warmup // 10)):
        g.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(passes):
            g.replay()
        end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / passes
    pb = ch.packed_bytes()
    gbs = pb / (ms * 1e-3) / 1e9
    out = {"tokens_per_s": round(batch / (ms * 1e-3), 1), "us_per_pass": round(ms * 1e3, 1),
           "packed_gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
           "packed_bytes_per_pass": pb, "blocks": nblocks, "batch": batch,
           "kernels_per_pass": nblocks * chain.DecodeChain.launches_per_step_per_block,
           "roofline_tokens_per_s": round(batch * peaks["hbm_gbs"] * 1e9 / pb, 1)}
    del g, ch, blocks
    return out


def run_chain_only(args, device, peaks):
    """--workload chain7b: the decode chain alone, one JSON line (tokens/s of the chain)."""
    import torch

    stream = torch.cuda.Stream(device)
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    c = run_chain(device, stream, args.warmup, peaks, passes=max(1, args.steps), batch=args.batch)
    clocks = sampler.stop()
    line = {"metric": METRIC, "value": c["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(c["us_per_pass"] / 1e3, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 in; int8x2-limb tensor-core products, int32/fp32 acc", "data": "synthetic",
            "config": {"workload": f"decode chain: {c['blocks']} llama2-7b-shaped blocks x 7 factorised linears, "
                                   f"batch {c['batch']}, per-block RMS re-normalisation",
                       "l2": "659 MB of packed weights per pass (> 5x L2)", "graphs": "one CUDA graph per pass"},
            "roofline": {"bound": "hbm", "achieved": c["packed_gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": c["frac_of_hbm"], "traffic": None, "peak_source": peaks["source"]},
            "gpu_launches": c["kernels_per_pass"] * max(1, args.steps), "clocks": clocks, "chain": c}
    print(json.dumps(line), flush=True)


def run_prefill_only(args, device, peaks):
    """--workload prefill: the config-4 sweep alone (or one batch), one JSON line, TFLOP/s."""
    import torch

    stream = torch.cuda.Stream(device)
    sweep = run_prefill_sweep(device, stream, args.warmup, peaks, calls=max(1, args.steps),
                              batches=(args.prefill_batch,) if args.prefill_batch else synth.PREFILL_BATCHES)
    top = str(max(int(b) for b in sweep))
    line = {"metric": METRIC, "value": sweep[top]["tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp16 tcgen05 operands, fp32 accumulate", "data": "synthetic",
            "config": {"workload": f"prefill 11008x4096 r=2432, token batch {top}"}, "prefill": sweep}
    print(json.dumps(line), flush=True)


def run_e2e(work, stream, steps, device):
    """End to end through the public API: one nq_lowrank_linear_fwd_grouped call per step
    with every layer's x and y in pinned host memory (the call copies x in, runs the launch
    pair, copies y out and synchronises); wall clock around the steps.  Also the same with
    seven nq_lowrank_linear_fwd calls per step (one copy-in, launch pair, copy-out and sync
    each)."""
    import torch

    nq = work.nq
    xs = [x.cpu().pin_memory() for x in work.x]
    ys = [torch.empty(y.shape, dtype=torch.float32).pin_memory() for y in work.y]
    h = stream.cuda_stream
    descs = [nq.make_descs([(xs[li], *per[li][:2], *per[li][2:], ys[li], m, n, r)
                            for li, (_, m, n, r) in enumerate(work.layers)]) for per in work.sets]
    grouped = nq.lib().nq_lowrank_linear_fwd_grouped
    fwd = nq.lib().nq_lowrank_linear_fwd

    def one_grouped(i):
        st = grouped(ctypes.addressof(descs[i % work.copies]), len(work.layers), work.batch, h)
        if st != 0:
            raise RuntimeError(nq.nq_status_string(st))

    def one_per_layer(i):
        per = work.sets[i % work.copies]
        for li, (name, m, n, r) in enumerate(work.layers):
            Upk, Vpk, s1, s2 = per[li]
            st = fwd(xs[li].data_ptr(), Upk.data_ptr(), Vpk.data_ptr(), s1.data_ptr(), s2.data_ptr(), m, n, r,
                     work.batch, ys[li].data_ptr(), h)
            if st != 0:
                raise RuntimeError(nq.nq_status_string(st))

    def timed(fn):
        # warm-up: every weight copy's call twice, so that the timed calls run in the steady
        # state of a decode loop (the library replays a synchronising call it has seen before
        # from a CUDA graph captured at its second occurrence)
        for i in range(max(3, 2 * work.copies + 1)):
            fn(i)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for i in range(steps):
            fn(i)
        torch.cuda.synchronize()
        return time.perf_counter() - t0

    dt = timed(one_grouped)
    dt_layers = timed(one_per_layer)
    h2d = sum(x.numel() * 2 for x in xs)
    d2h = sum(y.numel() * 4 for y in ys)
    return {"value": round(work.step_bytes * steps / dt / 1e9, 2), "unit": "GB/s", "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "us_per_step": round(dt / steps * 1e6, 2),
            "per_layer_calls_gbs": round(work.step_bytes * steps / dt_layers / 1e9, 2),
            "how": "one nq_lowrank_linear_fwd_grouped call per step with pinned host x and y (x gathered "
                   "in, launch pair, y written to host, stream sync inside the call; repeated calls replayed "
                   "from the library's captured CUDA graph), warm-up 2 calls per weight copy, wall clock"}


# ------------------------------------------------------------------ the oracle on the host

def run_cpu_baseline(layers, batch, budget_s):
    import oracle

    o = oracle.default()
    data = []
    for li, (name, m, n, r) in enumerate(layers):
        Upk = synth.random_words(m, r // 32, 5, li, "U")
        Vpk = synth.random_words(r, n // 32, 5, li, "V")
        data.append((Upk, Vpk, synth.scales_f16(m, 5, li), synth.scales_f16(n, 6, li),
                     synth.activations_bf16(batch, n, 5, li), m, n, r))
    step_bytes = sum(packed_bytes(m, n, r) for _, m, n, r in layers)
    steps = 0
    t0 = time.perf_counter()
    while True:
        for (Upk, Vpk, s1, s2, x, m, n, r) in data:
            o.lowrank_linear_fwd(x, Upk, Vpk, s1, s2, m, n, r)
        steps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(step_bytes * steps / dt / 1e9, 4), "unit": "GB/s", "cores": o.num_threads(),
            "kind": "oracle",
            "sample": f"{steps} step(s) of the 7-layer batch-{batch} workload on the fp64 C oracle ({dt:.1f} s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cpu = run_cpu_baseline(synth.LLAMA2_7B_LAYERS, args.batch, budget_s=args.cpu_seconds)
    steps_done = int(cpu["sample"].split()[0])
    value = cpu["value"]
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "impl": "reference",
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"llama2-7b-shaped decode, batch {args.batch}: 7 factorised linears per step",
                       "batch": args.batch, "steps_sampled": steps_done},
            "cpu_baseline": cpu, "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                                          "d2h_bytes_per_step": 0},
            "vs_baseline": None}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", dest="secondary", action="store_false")
    ap.add_argument("--workload", choices=["decode7b", "decode70b", "prefill", "chain7b"], default="decode7b")
    ap.add_argument("--prefill-batch", type=int, default=0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
