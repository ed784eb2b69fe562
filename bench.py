#!/usr/bin/env python
"""Benchmark of the factorised binary low-rank linear, y = s1 * (U (V^T (s2 * x))).

Default workload (one "step"): the seven linears of a Llama-2-70B-shaped block
(q/o 8192x8192 r=2432, k/v 1024x8192 r=384, gate/up 28672x8192 r=3840, down 8192x28672
r=3840) at decode batch 1, each layer with its own seeded input, in one grouped call
through the C ABI (nq_lowrank_linear_fwd_grouped), captured in CUDA graphs.
Metric: packed-weight HBM GB/s = (packed sign bytes of the seven layers) x steps / time.
The weights rotate over enough seeded copies (> 2x the 126 MB L2) that every step
streams its signs from HBM.  The K-step region is timed `--repeats` times (CUDA events,
synchronised on both sides) and the median is reported.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode70b|decode7b|prefill|chain7b|admm|backward]
    torchrun --nproc-per-node N bench.py --gpus N ...   (independent replicas, one per GPU)

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead
(rank 0 only) on a bounded sample of the same workload, with the same ``config``.
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


DECODE_WORKLOADS = {
    "decode70b": ("llama2-70b", synth.LLAMA2_70B_LAYERS),
    "decode7b": ("llama2-7b", synth.LLAMA2_7B_LAYERS),
}


def weight_copies(layers, min_bytes=2 * L2_BYTES):
    """Seeded weight copies a decode step rotates over, so that the copies' packed signs
    exceed `min_bytes` (every step then streams its weights from HBM, not L2)."""
    step = sum(packed_bytes(m, n, r) for _, m, n, r in layers)
    return max(1, -(-min_bytes // step))


def decode_config(model, layers, batch):
    """The `config` of a decode line, the same for the GPU arm and the oracle arm."""
    step = sum(packed_bytes(m, n, r) for _, m, n, r in layers)
    copies = weight_copies(layers)
    return {"workload": f"{model}-shaped decode, batch {batch}: 7 factorised linears per step "
                        f"({', '.join(f'{nm} {m}x{n} r{r}' for nm, m, n, r in layers)}), "
                        "one nq_lowrank_linear_fwd_grouped call per step",
            "batch": batch, "packed_bytes_per_step": step,
            "l2": f"inputs larger than L2: weights rotate over {copies} seeded copies "
                  f"({copies * step / 1e6:.0f} MB > 2x the 126 MB L2)"}


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
        self.copies = weight_copies(layers, min_bytes)
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


def timed_graphs(work, steps, warmup, stream, layer_filter=None, dist=None, repeats=1):
    """Capture graphs covering `steps` steps (rotating copies), then time the `steps`-step
    region `repeats` times with CUDA events on the launching stream, each bracketed by a
    synchronisation (and a barrier across ranks).  Returns (median ms, all ms)."""
    import torch

    full = capture(lambda h: [work.step(i, h, layer_filter) for i in range(work.copies)], stream)
    rem = steps % work.copies
    part = capture(lambda h: [work.step(i, h, layer_filter) for i in range(rem)], stream) if rem else None
    reps = steps // work.copies
    for _ in range(max(1, -(-warmup // work.copies))):
        full.replay()
    times = []
    for _ in range(repeats):
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
        times.append(start.elapsed_time(end))
        if dist is not None:
            dist.barrier()
    del full, part
    return statistics.median(times), times


def traffic_record(workload, batch):
    """DRAM bytes per decode step from an ncu capture recorded in profiles/decode_traffic.json,
    or None when there is none for this workload or the decode kernels' code has changed
    since it was taken (the record holds a hash of the source without comments)."""
    import hashlib

    tpath = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(tpath):
        return None
    with open(tpath) as f:
        recs = json.load(f)
    for rec in recs.get("records", []):
        if rec.get("workload_key") != f"{workload}-b{batch}":
            continue
        with open(os.path.join(ROOT, rec["kernel_source"])) as f:
            code = f.read()
        code = re.sub(r"/\*.*?\*/", "", code, flags=re.S)
        code = "".join(re.sub(r"//[^\n]*", "", code).split())
        if hashlib.sha256(code.encode()).hexdigest()[:16] == rec["kernel_code_sha256_16"]:
            return rec["dram_bytes_per_step"]
    return None


def decode_line_numbers(work, ms, steps, peaks):
    gbs = work.step_bytes * steps / (ms * 1e-3) / 1e9
    return {"gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
            "us_per_step": round(ms * 1e3 / steps, 2),
            "tokens_per_s": round(work.batch * steps / (ms * 1e-3), 1)}


def run_secondary_decode(name, layers, batch, steps, warmup, stream, device, peaks, seed, repeats=3):
    import torch

    w = DecodeWorkload(layers, batch, seed=seed, device=device)
    with torch.cuda.stream(stream):
        w.step(0, stream.cuda_stream)
    torch.cuda.synchronize()
    st = max(w.copies, steps // w.copies * w.copies)
    ms, _ = timed_graphs(w, st, warmup, stream, repeats=repeats)
    out = decode_line_numbers(w, ms, st, peaks)
    out["steps"] = st
    del w
    return out


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
    from binary_rank_linear_02_b200 import nq  # noqa: F401  (fails loudly without libnq.so)

    peaks = load_peaks()
    if args.workload == "prefill":
        return run_prefill_only(args, device, peaks)
    if args.workload == "chain7b":
        return run_chain_only(args, device, peaks)
    if args.workload == "admm":
        return run_admm_only(args, device, peaks)
    if args.workload == "backward":
        return run_backward_only(args, device, peaks)
    model, layers = DECODE_WORKLOADS[args.workload]
    batch = args.batch
    work = DecodeWorkload(layers, batch, seed=1234 + rank, device=device)
    stream = torch.cuda.Stream(device)
    # first calls outside capture (kernel attributes, workspace)
    with torch.cuda.stream(stream):
        work.step(0, stream.cuda_stream)
    torch.cuda.synchronize()

    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local)
    sampler.start()
    ms, all_ms = timed_graphs(work, args.steps, args.warmup, stream, dist=dist, repeats=args.repeats)
    clocks = sampler.stop()
    ms_max, total_bytes = aggregate(ms, float(work.step_bytes * args.steps), dist, device)
    value = total_bytes / (ms_max * 1e-3) / 1e9
    tokens_per_s = batch * args.steps * world / (ms_max * 1e-3)

    # roofline: the decode kernels of the headline step (stage 1 + stage 2 of one grouped
    # call, timed live above), against the measured HBM copy bandwidth
    achieved = value / world
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic_record(args.workload, batch),
                "algorithmic_bytes_per_launch": work.step_bytes,
                "kernel": f"stage1_kernel + stage2_kernel of one grouped call ({work.step_bytes} packed bytes "
                          "per launch pair), per GPU",
                "peak_source": peaks["source"]}

    # end to end through the public API with host buffers (pinned), synchronous per call
    e2e = run_e2e(work, stream, min(args.steps, 100), device)

    secondary = {}
    prefill_roofline = prefill_cpu = None
    if args.secondary and world == 1:
        # the largest layer (gate) alone, back to back over its own rotating copies
        gate = [l for l in layers if l[0] == "gate"][0]
        secondary[f"decode_{model}_gate_alone_b{batch}"] = run_secondary_decode(
            "gate", [gate], batch, max(500, args.steps), args.warmup, stream, device, peaks, seed=777)
        work.grouped = False
        ms1, _ = timed_graphs(work, args.steps, args.warmup, stream, repeats=3)
        work.grouped = True
        secondary[f"decode_{model}_b{batch}_per_layer_calls"] = decode_line_numbers(work, ms1, args.steps, peaks)
        others = [("decode70b", 4), ("decode7b", 1), ("decode7b", 8)]
        if args.workload != "decode70b" or batch != 1:
            others = [("decode70b", 1)] + others
        for wl, b in others:
            if wl == args.workload and b == batch:
                continue
            m2, l2 = DECODE_WORKLOADS[wl]
            secondary[f"decode_{m2}_b{b}"] = run_secondary_decode(wl, l2, b, min(args.steps, 400), args.warmup,
                                                                   stream, device, peaks, seed=70 + b)
        # 16 tokens in one grouped call of the 7B block (the decode kernels over two token chunks)
        g16 = run_secondary_decode("decode7b", synth.LLAMA2_7B_LAYERS, 16, min(args.steps, 400), args.warmup,
                                   stream, device, peaks, seed=116)
        secondary["grouped_llama2-7b_b16"] = g16
        # the input gradient dx = W^T dy of the 7B block (backward of the layers)
        for bb in (1, 8):
            wb = backward_workload(synth.LLAMA2_7B_LAYERS, bb, seed=123 + bb, device=device)
            with torch.cuda.stream(stream):
                wb.step(0, stream.cuda_stream)
            torch.cuda.synchronize()
            msb, _ = timed_graphs(wb, args.steps, args.warmup, stream, repeats=3)
            secondary[f"backward_input_llama2-7b_b{bb}"] = decode_line_numbers(wb, msb, args.steps, peaks)
            del wb
        sweep = run_prefill_sweep(device, stream, args.warmup, peaks)
        secondary["prefill_11008x4096_r2432"] = sweep
        prefill_roofline = prefill_roofline_of(sweep, peaks)
        secondary["chain_llama2-7b_32_blocks_b1"] = run_chain(device, stream, args.warmup, peaks)
        secondary["envelope_llama2-7b_q_l2_b1"] = run_envelope(device, stream, peaks)
        secondary["admm_init_llama2-7b_q"] = run_admm(device, stream, peaks)
        secondary["backward_11008x4096_r2432"] = run_backward_calibration(device, stream, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(layers, batch, budget_s=args.cpu_seconds)
        if args.secondary:
            prefill_cpu = run_cpu_baseline_prefill(budget_s=max(3.0, args.cpu_seconds / 2))
            if prefill_roofline is not None:
                prefill_roofline["cpu_baseline"] = prefill_cpu
            if "admm_init_llama2-7b_q" in secondary:
                secondary["admm_init_llama2-7b_q"]["cpu_baseline"] = run_cpu_baseline_admm()

    launches = args.steps * 2  # stage-1 and stage-2 kernels of one grouped call per step
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in; int8x2-limb tensor-core products, int32/fp32 acc",
            "data": "synthetic",
            "config": decode_config(model, layers, batch),
            "parallelism": f"independent replicas x{world} (no data-path collective)",
            "timing": {"repeats": args.repeats, "reported": "median of the repeats",
                       "ms_per_repeat": [round(t, 4) for t in all_ms],
                       "method": "CUDA events on the launching stream around exactly `steps` steps, "
                                 "synchronised on both sides, CUDA graphs of the C-ABI calls"},
            "tokens_per_s": round(tokens_per_s, 1),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "gpu_launches_all_repeats": launches * args.repeats, "clocks": clocks,
            "prefill_roofline": prefill_roofline,
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    del work
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def prefill_roofline_of(sweep, peaks):
    """The prefill half of the metric: config-4 sweep against the bf16 dense burst peak (the
    two GEMMs are timed back to back in isolation), reported at the largest batch with the
    fraction at every batch."""
    top = str(max(int(b) for b in sweep))
    tf = sweep[top]["tflops"]
    return {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(tf / peaks["bf16_tflops"], 4), "traffic": None,
            "kernel": f"prescale_kernel + two tcgen05 GEMM kernels of one nq_lowrank_linear_fwd call, "
                      f"11008x4096 r=2432 layer, {top} tokens (2*b*r*(m+n) flops per call)",
            "frac_per_batch": {b: v["frac_of_bf16_burst"] for b, v in sweep.items()},
            "peak_source": peaks["source"] + " (burst)"}


def run_prefill_sweep(device, stream, warmup, peaks, calls=20, batches=synth.PREFILL_BATCHES, repeats=5):
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
        times = []
        for _ in range(repeats):
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                start.record(stream)
                g.replay()
                end.record(stream)
            torch.cuda.synchronize()
            times.append(start.elapsed_time(end) / calls)
        nq.device_status(stream.cuda_stream)
        ms = statistics.median(times)
        flops = 2.0 * b * r * (m + n)
        tf = flops / (ms * 1e-3) / 1e12
        out[str(b)] = {"tflops": round(tf, 1), "us_per_call": round(ms * 1e3, 2),
                       "frac_of_bf16_burst": round(tf / peaks["bf16_tflops"], 4),
                       "tokens_per_s": round(b / (ms * 1e-3), 1)}
        del g, x, y
    return out


def run_chain(device, stream, warmup, peaks, passes=20, batch=1, nblocks=synth.CHAIN_7B_BLOCKS, repeats=3):
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
    times = []
    for _ in range(repeats):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(passes):
                g.replay()
            end.record(stream)
        torch.cuda.synchronize()
        times.append(start.elapsed_time(end) / passes)
    ms = statistics.median(times)
    pb = ch.packed_bytes()
    gbs = pb / (ms * 1e-3) / 1e9
    out = {"tokens_per_s": round(batch / (ms * 1e-3), 1), "us_per_pass": round(ms * 1e3, 1),
           "packed_gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
           "packed_bytes_per_pass": pb, "blocks": nblocks, "batch": batch,
           "kernels_per_pass": nblocks * chain.DecodeChain.launches_per_step_per_block,
           "roofline_tokens_per_s": round(batch * peaks["hbm_gbs"] * 1e9 / pb, 1)}
    del g, ch, blocks
    return out


def run_backward_calibration(device, stream, peaks, batches=(1024, 4096), reps=5):
    """The refinement step's gradients of one layer (the 11008x4096 r=2432 gate shape) at
    calibration batch sizes: nq_lowrank_linear_bwd_factors (rank vectors by the prefill
    GEMMs, sums over the tokens on the tensor cores) and nq_lowrank_linear_bwd_scales.
    Algorithmic flops: factors 4 b r (m + n) (t, u and the two outer products), scales
    4 b r (m + n) (two factorised evaluations) plus 2 b (m + n)."""
    import torch

    from binary_rank_linear_02_b200 import nq

    _, m, n, r = synth.PREFILL_SHAPE
    gen = torch.Generator(device=device)
    gen.manual_seed(777)
    Upk = torch.randint(-(1 << 31), 1 << 31, (m, r // 32), dtype=torch.int64, device=device, generator=gen).to(torch.int32)
    Vpk = torch.randint(-(1 << 31), 1 << 31, (r, n // 32), dtype=torch.int64, device=device, generator=gen).to(torch.int32)
    UpkT = nq.transpose_signs(Upk, m, r)
    VpkT = nq.transpose_signs(Vpk, r, n)
    s1 = torch.from_numpy(synth.scales_f16(m, 777, "s1").view(np.int16)).to(device)
    s2 = torch.from_numpy(synth.scales_f16(n, 777, "s2").view(np.int16)).to(device)
    out = {}
    for b in batches:
        x = torch.from_numpy(synth.activations_bf16(b, n, 777, b).view(np.int16)).to(device)
        dy = torch.from_numpy(synth.activations_bf16(b, m, 778, b).view(np.int16)).to(device)
        for name, fn in (("factors", lambda: nq.lowrank_linear_bwd_factors(x, dy, Vpk, UpkT, s1, s2, m, n, r,
                                                                           stream=stream.cuda_stream)),
                         ("scales", lambda: nq.lowrank_linear_bwd_scales(x, dy, Upk, Vpk, UpkT, VpkT, s1, s2, m, n, r,
                                                                         stream=stream.cuda_stream))):
            with torch.cuda.stream(stream):
                fn()
            torch.cuda.synchronize()
            times = []
            for _ in range(reps):
                start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    start.record(stream)
                    fn()
                    end.record(stream)
                torch.cuda.synchronize()
                times.append(start.elapsed_time(end))
            ms = statistics.median(times)
            fl = 4.0 * b * r * (m + n) + (2.0 * b * (m + n) if name == "scales" else 0.0)
            tf = fl / (ms * 1e-3) / 1e12
            out[f"{name}_b{b}"] = {"us_per_call": round(ms * 1e3, 1), "tflops": round(tf, 1),
                                   "frac_of_bf16_burst": round(tf / peaks["bf16_tflops"], 4)}
        del x, dy
    return out


FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # SMs x fp32 lanes x 2 flops (FMA) x max clock


def admm_flops_per_iteration(m, n, r):
    """Algorithmic flops of one ADMM iteration (both half-steps): the W products 2 x 2mnr,
    the Gram matrices 2 x 2r^2 (m or n), the two triangular solves of each side 2 x 2r^2
    (n or m), two Cholesky factorisations 2 x r^3/3."""
    return 4.0 * m * n * r + 4.0 * r * r * (m + n) + 2.0 * r ** 3 / 3.0


def run_admm(device, stream, peaks, iters=40, shape=(4096, 4096, 1664), repeats=3):
    """The LB-ADMM initialiser on a synthetic Llama-2-7B attention-shaped weight: the whole
    nq_admm_factorize call by wall clock (start, iterations, balancing, packing, error; host
    allocation included), and the iterations by CUDA events on the call's stream around
    nq_admm_iterate calls of `iters` iterations from one start (median of `repeats`)."""
    import torch

    from binary_rank_linear_02_b200 import nq

    m, n, r = shape
    W = torch.from_numpy(synth.weights_bf16(m, n, 8080).view(np.int16)).to(device)
    Om = torch.from_numpy(synth.gaussian_f32(n, r, 8080, "omega")).to(device)

    def one(k):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        out = nq.admm_factorize(W, m, n, r, Om, iters=k, stream=stream.cuda_stream)
        torch.cuda.synchronize()
        return time.perf_counter() - t0, out[4]

    one(2)  # warm-up (module load, first allocations)
    runs = [one(iters) for _ in range(repeats)]
    t_full = statistics.median([t for t, _ in runs])
    err = runs[0][1]
    st = nq.admm_init(W, m, n, r, Om, 1, stream=stream.cuda_stream)
    nq.admm_iterate(W, st, 2, stream=stream.cuda_stream)
    times = []
    for _ in range(repeats):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        nq.admm_iterate(W, st, iters, stream=stream.cuda_stream)
        end.record(stream)
        torch.cuda.synchronize()
        times.append(start.elapsed_time(end) / 1e3)
    per_it = statistics.median(times) / iters
    fl = admm_flops_per_iteration(m, n, r)
    tf = fl / per_it / 1e12
    return {"shape": f"{m}x{n} r={r}", "iters": iters, "seconds_per_call": round(t_full, 4),
            "ms_per_iteration": round(per_it * 1e3, 3), "gflop_per_iteration": round(fl / 1e9, 1),
            "tflops": round(tf, 2), "rel_err": round(err, 5),
            "roofline": {"bound": "alu", "achieved": round(tf, 2), "peak": round(FP32_ALU_TFLOPS, 1),
                         "unit": "TFLOP/s", "frac": round(tf / FP32_ALU_TFLOPS, 4),
                         "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flops x 1965 MHz"},
            "timing": "iterations: CUDA events on the launching stream around nq_admm_iterate calls "
                      "(median); seconds_per_call: wall clock around the whole synchronising call"}


def run_envelope(device, stream, peaks, steps=200, batch=1, l=2, shape=(4096, 4096, 1664)):
    """The rank-l envelope forward on the Llama-2-7B q shape, back to back over rotating
    weight copies, against the plain forward on the same copies."""
    import torch

    from binary_rank_linear_02_b200 import nq

    m, n, r = shape
    pb = packed_bytes(m, n, r)
    copies = max(1, -(-2 * L2_BYTES // pb))
    gen = torch.Generator(device=device)
    gen.manual_seed(9090)
    sets = [(torch.randint(-(1 << 31), 1 << 31, (m, r // 32), dtype=torch.int64, device=device, generator=gen).to(torch.int32),
             torch.randint(-(1 << 31), 1 << 31, (r, n // 32), dtype=torch.int64, device=device, generator=gen).to(torch.int32))
            for _ in range(copies)]
    a = torch.from_numpy(np.stack([synth.scales_f16(m, 9090, "a", q) for q in range(l)]).view(np.int16)).to(device)
    b = torch.from_numpy(np.stack([synth.scales_f16(n, 9090, "b", q) for q in range(l)]).view(np.int16)).to(device)
    x = torch.from_numpy(synth.activations_bf16(batch, n, 9090).view(np.int16)).to(device)
    y = torch.empty((batch, m), dtype=torch.float32, device=device)
    env, fwd = nq.lib().nq_lowrank_linear_fwd_envelope, nq.lib().nq_lowrank_linear_fwd

    def step_env(i, h):
        U, V = sets[i % copies]
        st = env(x.data_ptr(), U.data_ptr(), V.data_ptr(), a.data_ptr(), b.data_ptr(), l, m, n, r, batch, y.data_ptr(), h)
        if st != 0:
            raise RuntimeError(nq.nq_status_string(st))

    def step_fwd(i, h):
        U, V = sets[i % copies]
        st = fwd(x.data_ptr(), U.data_ptr(), V.data_ptr(), a.data_ptr(), b.data_ptr(), m, n, r, batch, y.data_ptr(), h)
        if st != 0:
            raise RuntimeError(nq.nq_status_string(st))

    out = {"shape": f"{m}x{n} r={r}", "l": l, "batch": batch, "packed_bytes": pb}
    for name, fn in (("envelope", step_env), ("plain", step_fwd)):
        with torch.cuda.stream(stream):
            fn(0, stream.cuda_stream)
        torch.cuda.synchronize()
        g = capture(lambda h: [fn(i, h) for i in range(steps)], stream)
        g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(3):
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                start.record(stream)
                g.replay()
                end.record(stream)
            torch.cuda.synchronize()
            times.append(start.elapsed_time(end) / steps)
        ms = statistics.median(times)
        gbs = pb / (ms * 1e-3) / 1e9
        out[name] = {"us_per_call": round(ms * 1e3, 2), "packed_gbs": round(gbs, 1),
                     "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4)}
        del g
    return out


def run_chain_only(args, device, peaks):
    """--workload chain7b: the decode chain alone, one JSON line (tokens/s of the chain)."""
    import torch

    stream = torch.cuda.Stream(device)
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    c = run_chain(device, stream, args.warmup, peaks, passes=max(1, args.steps), batch=args.batch,
                  repeats=args.repeats)
    clocks = sampler.stop()
    cpu = None if args.no_cpu_baseline else run_cpu_baseline_chain(budget_s=args.cpu_seconds)
    line = {"metric": METRIC, "value": c["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(c["us_per_pass"] / 1e3, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 in; int8x2-limb tensor-core products, int32/fp32 acc", "data": "synthetic",
            "config": chain_config(args.batch),
            "timing": {"repeats": args.repeats, "reported": "median of the repeats", "graphs": "one CUDA graph per pass"},
            "roofline": {"bound": "hbm", "achieved": c["packed_gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": c["frac_of_hbm"], "traffic": None, "peak_source": peaks["source"],
                         "algorithmic_bytes_per_launch": c["packed_bytes_per_pass"],
                         "kernel": "every decode kernel of one chain pass"},
            "cpu_baseline": cpu,
            "gpu_launches": c["kernels_per_pass"] * max(1, args.steps), "clocks": clocks, "chain": c}
    print(json.dumps(line), flush=True)


def run_admm_only(args, device, peaks):
    """--workload admm: the LB-ADMM initialiser alone on the 4096x4096 r=1664 problem
    (--admm-iters iterations per call), one JSON line, TFLOP/s of its iterations."""
    import torch

    stream = torch.cuda.Stream(device)
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    a = run_admm(device, stream, peaks, iters=args.admm_iters, repeats=args.repeats)
    clocks = sampler.stop()
    cpu = None if args.no_cpu_baseline else run_cpu_baseline_admm()
    line = {"metric": METRIC, "value": a["tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.admm_iters,
            "warmup": 1, "ms_per_step": a["ms_per_iteration"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32 (W read as bf16)", "data": "synthetic",
            "config": {"workload": f"LB-ADMM initialiser, {a['shape']}, {args.admm_iters} iterations per call"},
            "roofline": a["roofline"], "cpu_baseline": cpu, "clocks": clocks, "admm": a}
    print(json.dumps(line), flush=True)


def run_backward_only(args, device, peaks):
    """--workload backward: the refinement step's factor and scale gradients of the
    11008x4096 r=2432 layer alone (--backward-batch tokens, else 1024 and 4096), one JSON line,
    TFLOP/s of the factor gradients at the largest batch."""
    import torch

    stream = torch.cuda.Stream(device)
    batches = (args.backward_batch,) if args.backward_batch else (1024, 4096)
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    b = run_backward_calibration(device, stream, peaks, batches=batches, reps=max(3, args.repeats))
    clocks = sampler.stop()
    top = max(batches)
    f = b[f"factors_b{top}"]
    line = {"metric": METRIC, "value": f["tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": 1, "warmup": 1,
            "ms_per_step": round(f["us_per_call"] / 1e3, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 operands (t, u split into two bf16 parts), fp32 accumulate",
            "data": "synthetic",
            "config": {"workload": f"factor and scale gradients, 11008x4096 r=2432 layer, {top} tokens"},
            "roofline": {"bound": "tensor", "achieved": f["tflops"], "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": f["frac_of_bf16_burst"], "traffic": None,
                         "kernel": "nq_lowrank_linear_bwd_factors (4 b r (m + n) flops per call)",
                         "peak_source": peaks["source"] + " (burst)"},
            "cpu_baseline": None, "clocks": clocks, "backward": b}
    print(json.dumps(line), flush=True)


def run_prefill_only(args, device, peaks):
    """--workload prefill: the config-4 sweep alone (or one batch), one JSON line, TFLOP/s."""
    import torch

    stream = torch.cuda.Stream(device)
    batches = (args.prefill_batch,) if args.prefill_batch else synth.PREFILL_BATCHES
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    sweep = run_prefill_sweep(device, stream, args.warmup, peaks, calls=max(1, args.steps), batches=batches,
                              repeats=args.repeats)
    clocks = sampler.stop()
    top = str(max(int(b) for b in sweep))
    cpu = None if args.no_cpu_baseline else run_cpu_baseline_prefill(budget_s=args.cpu_seconds)
    line = {"metric": METRIC, "value": sweep[top]["tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(sweep[top]["us_per_call"] / 1e3, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp16 tcgen05 operands, fp32 accumulate", "data": "synthetic",
            "config": prefill_config(batches),
            "timing": {"repeats": args.repeats, "reported": "median of the repeats"},
            "roofline": prefill_roofline_of(sweep, peaks), "cpu_baseline": cpu,
            "gpu_launches": 3 * max(1, args.steps), "clocks": clocks, "prefill": sweep}
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
    """The oracle on the host cores over the decode workload: whole steps (the seven
    layers), rotating over the same number of seeded weight copies as the GPU arm, until
    `budget_s` seconds have passed."""
    import oracle

    o = oracle.default()
    copies = weight_copies(layers)
    data = []
    for c in range(copies):
        per = []
        for li, (name, m, n, r) in enumerate(layers):
            per.append((synth.random_words(m, r // 32, 5, c, li, "U"), synth.random_words(r, n // 32, 5, c, li, "V"),
                        synth.scales_f16(m, 5, c, li), synth.scales_f16(n, 6, c, li),
                        synth.activations_bf16(batch, n, 5, li), m, n, r))
        data.append(per)
    step_bytes = sum(packed_bytes(m, n, r) for _, m, n, r in layers)
    steps = 0
    t0 = time.perf_counter()
    while True:
        for (Upk, Vpk, s1, s2, x, m, n, r) in data[steps % copies]:
            o.lowrank_linear_fwd(x, Upk, Vpk, s1, s2, m, n, r)
        steps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(step_bytes * steps / dt / 1e9, 4), "unit": "GB/s", "cores": o.num_threads(),
            "kind": "oracle", "steps": steps, "seconds": round(dt, 2),
            "sample": f"{steps} step(s) of the 7-layer batch-{batch} workload ({copies} rotating weight copies) "
                      f"on the fp64 C oracle ({dt:.1f} s)"}


def run_cpu_baseline_prefill(budget_s, batch=16):
    """The oracle on the host cores over the prefill layer (11008x4096, r=2432): calls of
    `batch` tokens until `budget_s` seconds have passed; TFLOP/s over 2*b*r*(m+n)."""
    import oracle

    o = oracle.default()
    _, m, n, r = synth.PREFILL_SHAPE
    Upk = synth.random_words(m, r // 32, 9, "U")
    Vpk = synth.random_words(r, n // 32, 9, "V")
    s1, s2 = synth.scales_f16(m, 9, "s1"), synth.scales_f16(n, 9, "s2")
    x = synth.activations_bf16(batch, n, 9)
    calls = 0
    t0 = time.perf_counter()
    while True:
        o.lowrank_linear_fwd(x, Upk, Vpk, s1, s2, m, n, r)
        calls += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    flops = 2.0 * batch * r * (m + n) * calls
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": o.num_threads(), "kind": "oracle",
            "sample": f"{calls} call(s) of {batch} tokens on the 11008x4096 r=2432 layer, fp64 C oracle ({dt:.1f} s)"}


def run_cpu_baseline_chain(budget_s, nblocks=synth.CHAIN_7B_BLOCKS):
    """The oracle's decode chain on the host cores: blocks of the 32-block chain (seeded
    weights as the GPU arm draws them) one after another until `budget_s` seconds have
    passed; tokens/s scaled to the whole chain."""
    import oracle

    o = oracle.default()
    w = synth.chain_weights(1, synth.LLAMA2_7B_LAYERS, 5150)[0]
    h = synth.activations_bf16(1, 4096, 5150, "h0")
    done = 0
    t0 = time.perf_counter()
    while True:
        h = o.chain_block(h, w)["h_next"]
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(done / nblocks / dt, 4), "unit": "tokens/s", "cores": o.num_threads(), "kind": "oracle",
            "sample": f"{done} Llama-2-7B-shaped block(s) of the {nblocks}-block chain, batch 1, fp64 C oracle "
                      f"({dt:.1f} s)"}


def run_cpu_baseline_admm(shape=(4096, 4096, 1664), iters=2):
    """The oracle's ADMM iterations on the host cores (numpy fp64) for the same shape: the
    start, then `iters` iterations timed; TFLOP/s over the same algorithmic flops."""
    import oracle.admm as adm

    m, n, r = shape
    W = adm.decode_bf16(synth.weights_bf16(m, n, 8080))
    Om = synth.gaussian_f32(n, r, 8080, "omega").astype(np.float64)
    st = adm.start_state(*adm.power_iteration_init(W, Om, 1))
    t0 = time.perf_counter()
    for k in range(iters):
        st = adm.admm_step(W, st, 0.2 * 1.05 ** k)
    dt = (time.perf_counter() - t0) / iters
    import os as _os

    return {"value": round(admm_flops_per_iteration(m, n, r) / dt / 1e12, 4), "unit": "TFLOP/s",
            "cores": _os.cpu_count(), "kind": "oracle", "seconds_per_iteration": round(dt, 3),
            "sample": f"{iters} ADMM iteration(s) of the {m}x{n} r={r} problem on the numpy fp64 oracle"}


def run_cpu_baseline_backward(budget_s=10.0):
    """The oracle's factor gradients of the 11008x4096 r=2432 layer on the host cores (fp64 C),
    for growing token samples until the time budget; TFLOP/s over the same 4 b r (m + n)
    algorithmic flops as the GPU arm."""
    import oracle as orc

    _, m, n, r = synth.PREFILL_SHAPE
    U = synth.signs(m, r, 777, "U")
    V = synth.signs(n, r, 777, "V")
    Upk, Vpk = orc.pack_signs(U), orc.pack_signs(np.ascontiguousarray(V.T))  # V^T: r x n/32 words
    s1 = synth.scales_f16(m, 777, "s1")
    s2 = synth.scales_f16(n, 777, "s2")
    b, spent, calls, toks = 1, 0.0, 0, 0
    while spent < budget_s and b <= 64:
        x = synth.activations_bf16(b, n, 777, b)
        dy = synth.activations_bf16(b, m, 778, b)
        t0 = time.perf_counter()
        orc.lowrank_linear_bwd_factors(x, dy, Upk, Vpk, s1, s2, m, n, r)
        spent += time.perf_counter() - t0
        calls += 1
        toks += b
        b *= 2
    import os as _os

    return {"value": round(4.0 * toks * r * (m + n) / spent / 1e12, 6), "unit": "TFLOP/s", "cores": _os.cpu_count(),
            "kind": "oracle", "seconds": round(spent, 2),
            "sample": f"{calls} call(s), {toks} tokens in all, of the factor gradients of the {m}x{n} r={r} layer "
                      f"on the fp64 C oracle ({spent:.1f} s)"}


def prefill_config(batches):
    _, m, n, r = synth.PREFILL_SHAPE
    return {"workload": f"prefill {m}x{n} r={r}, token batch {max(batches)} "
                        f"(sweep {', '.join(str(b) for b in batches)})",
            "batches": list(batches)}


def chain_config(batch=1, nblocks=synth.CHAIN_7B_BLOCKS):
    return {"workload": f"decode chain: {nblocks} llama2-7b-shaped blocks x 7 factorised linears, "
                        f"batch {batch}, per-block RMS re-normalisation",
            "l2": "inputs larger than L2: 659 MB of packed weights per pass (> 5x L2)"}


def run_reference(args):
    """The oracle arm: the CPU oracle as it stands, on the host cores, over a bounded sample
    of this arm's workload, with the same config, metric and unit as the GPU arm."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if args.workload == "prefill":
        batches = (args.prefill_batch,) if args.prefill_batch else synth.PREFILL_BATCHES
        cpu = run_cpu_baseline_prefill(budget_s=args.cpu_seconds)
        config = prefill_config(batches)
    elif args.workload == "chain7b":
        cpu = run_cpu_baseline_chain(budget_s=args.cpu_seconds)
        config = chain_config(args.batch)
    elif args.workload == "admm":
        cpu = run_cpu_baseline_admm()
        config = {"workload": f"LB-ADMM initialiser, 4096x4096 r=1664, {args.admm_iters} iterations per call"}
    elif args.workload == "backward":
        cpu = run_cpu_baseline_backward(budget_s=args.cpu_seconds)
        top = args.backward_batch if args.backward_batch else 4096
        config = {"workload": f"factor and scale gradients, 11008x4096 r=2432 layer, {top} tokens"}
    else:
        model, layers = DECODE_WORKLOADS[args.workload]
        cpu = run_cpu_baseline(layers, args.batch, budget_s=args.cpu_seconds)
        config = decode_config(model, layers, args.batch)
    value = cpu["value"]
    line = {"metric": METRIC, "value": value, "unit": cpu["unit"], "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "impl": "reference",
            "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": cpu, "e2e": {"value": value, "unit": cpu["unit"], "h2d_bytes_per_step": 0,
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
    ap.add_argument("--workload", choices=["decode70b", "decode7b", "prefill", "chain7b", "admm", "backward"],
                    default="decode70b")
    ap.add_argument("--backward-batch", type=int, default=0,
                    help="--workload backward: one token batch instead of 1024 and 4096")
    ap.add_argument("--admm-iters", type=int, default=40)
    ap.add_argument("--repeats", type=int, default=5)
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
