"""Benchmark of the sparse-MoE FFN layer on B200: tokens/s of one layer forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one whole layer forward (router -> top-k -> permutation -> gather -> expert up +
SwiGLU -> expert down -> combine) over one batch of T synthetic tokens already resident in
HBM.  Each step uses a different seeded batch, and L2 is flushed (256 MiB write) between
steps outside the timed intervals.  Times come from CUDA events the library records on its
launch stream around each kernel stage (moe_forward_profiled), summed over the K timed
steps, max over ranks.  N > 1 runs N independent replicas (one per GPU, no data-path
collective): value = all ranks' tokens / the slowest rank's time.

`--impl reference` times the CPU oracle (plain C, fp64) on the host cores instead, on a
bounded sample of each step's batch; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s on 1 B200; achieved HBM GB/s / tensor-pipe % of peak"
DEFAULT_WORKLOAD = "prefill_t8192"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
THROTTLE_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                 0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
                 0x100: "display_clock_setting"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------ clocks sampler
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.reader.join(timeout=2)
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 5:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
                bits = int(parts[4], 16)
            except ValueError:
                continue
            for b, name in THROTTLE_BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        sm.sort()
        med = sm[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------ roofline model
def algorithmic(w, counts, T):
    """Algorithmic bytes / flops of each stage for one forward (touched experts only)."""
    import numpy as np

    touched = int((np.asarray(counts) > 0).sum()) + w.n_shared
    es = 2 if w.dtype == "bf16" else 4
    Tk = T * w.k
    P = Tk + w.n_shared * T
    d, f, E = w.d, w.f, w.E
    up_bytes = touched * 2 * f * d * es + (Tk + w.n_shared * T) * d * es + P * f * es
    down_bytes = touched * d * f * es + P * f * es + P * d * 4  # y rows are fp32
    up_flops = 2.0 * P * 2 * f * d
    down_flops = 2.0 * P * d * f
    layer_bytes = touched * 3 * f * d * es + E * d * es + 2 * T * d * es
    layer_flops = up_flops + down_flops + 2.0 * T * d * E
    return dict(touched=touched, up_bytes=up_bytes, down_bytes=down_bytes, up_flops=up_flops,
                down_flops=down_flops, layer_bytes=layer_bytes, layer_flops=layer_flops)


def kernel_roofline(algo, key, dur_s, peaks):
    """Roofline of the dominant expert GEMM launch: its algorithmic bytes or flops per launch
    (mean over the timed batches) over its event-timed duration, against the bound its own
    flop/byte ratio puts it under (ridge of the burst peaks)."""
    import numpy as np

    bytes_per = float(np.mean([a[f"{key}_bytes"] for a in algo]))
    flops_per = float(np.mean([a[f"{key}_flops"] for a in algo]))
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops_per / bytes_per > ridge:
        achieved = flops_per / dur_s / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        achieved = bytes_per / dur_s / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    roof["frac"] = round(achieved / roof["peak"], 4)
    roof["algorithmic_bytes_per_launch"] = int(bytes_per)
    roof["algorithmic_flops_per_launch"] = int(flops_per)
    return roof


def tensor_peak_regime(peaks, gemm_mhz):
    """Which measured bf16 peak's clock regime the expert GEMMs ran in: "sustained" (the GEMM
    loop held at the 1 kW cap) when the GEMMs' own effective clock is within 10 % of that
    loop's median SM clock, else "burst".  Returns (TFLOP/s of that regime, regime, note)."""
    sus = peaks.get("bf16_tflops_sustained")
    med = (peaks.get("clocks_under_load") or {}).get("sm_mhz_median")
    if sus and med and gemm_mhz and abs(gemm_mhz - med) <= 0.1 * med:
        return sus, "sustained", (f"expert GEMMs measured at {gemm_mhz:.0f} MHz inside their "
                                  f"CTAs; the sustained GEMM loop's median clock {med:.0f} MHz")
    note = f"expert GEMMs measured at {gemm_mhz:.0f} MHz" if gemm_mhz else "GEMM clock unmeasured"
    return peaks["bf16_tflops"], "burst", note


def layer_roofline(layer_bytes, layer_flops, step_s, peaks, gemm_mhz=None):
    """The whole forward against the burst bf16 peak when it is tensor-bound (layer flops per
    algorithmic byte above the ridge of the burst peaks), else None.  Beside it: the fraction
    of the peak whose clock regime the GEMMs were measured in (gemm_mhz), with the evidence."""
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if layer_flops / layer_bytes <= ridge:
        return None
    peak_rg, regime, note = tensor_peak_regime(peaks, gemm_mhz)
    achieved = layer_flops / step_s / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
            "clock_regime": regime, "frac_of_clock_regime_peak": round(achieved / peak_rg, 4),
            "clock_regime_evidence": note,
            "scope": "layer", "algorithmic_flops_per_step": int(layer_flops),
            "algorithmic_bytes_per_step": int(layer_bytes)}


def kernel_source_sha():
    """sha256 (first 16 hex) of every kernel and launch source of the library: a committed
    DRAM capture counts only while the code it measured is unchanged."""
    csrc = os.path.join(ROOT, "sparse_moe_layer_warp_b200", "csrc")
    h = hashlib.sha256()
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh")):
            h.update(fn.encode())
            h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source; otherwise None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    ent = d.get(f"{kernel}/{workload}")
    if not ent or ent.get("source_sha") != kernel_source_sha():
        return None
    return ent.get("dram_bytes_per_launch")


# ------------------------------------------------------------------------ multi-rank
def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's time: every rank contributes, every rank gets the max."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time (weak scaling:
    every replica runs the same per-GPU workload)."""
    return world * steps * tokens_per_rank_step / (max_ms / 1e3)


# ------------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from sparse_moe_layer_warp_b200 import (MOE_OPTION_GEMM_CLOCK, MOE_PROFILE_STAGES,
                                            PROFILE_STAGE_NAMES, MoELayer,
                                            moe_forward_launch_count,
                                            moe_forward, moe_forward_profiled, synth)

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    T = w.T
    inp = synth.make_inputs(w, device=dev)
    layer = MoELayer(inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down, top_k=w.k,
                     max_tokens=T, n_shared=w.n_shared, routed_scale=w.routed_scale)
    nb = args.steps + args.warmup
    batches = [synth.make_x(w, T, device=dev, seed=1000 * (rank + 1) + i) for i in range(nb)]
    out = torch.empty_like(batches[0])
    ws = layer.workspace(T)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    # routing statistics of every timed batch (outside the timed region) for the roofline
    algo = []
    for i in range(args.warmup, nb):
        r = layer.route(x=batches[i])
        algo.append(algorithmic(w, r["counts"].cpu().numpy(), T))
    st = torch.cuda.current_stream()

    for i in range(args.warmup):
        flush.zero_()
        moe_forward(layer.handle, batches[i], T, out, ws)
    torch.cuda.synchronize()

    # timed region 1 (the headline value): the plain public call, one event pair per step
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    # timed region 2 (per-kernel durations for the roofline): the same steps through
    # moe_forward_profiled, which records events between its kernels on the launch stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(MOE_PROFILE_STAGES + 1)]
           for _ in range(args.steps)]
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(visible.split(",")[local_rank] if visible else local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(st)
        moe_forward(layer.handle, batches[args.warmup + i], T, out, ws)
        ev[i][1].record(st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        moe_forward_profiled(layer.handle, batches[args.warmup + i], T, out, ws, evs[i], st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    stage_ms = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(MOE_PROFILE_STAGES)]
                         for i in range(args.steps)])
    step_ms = np.array([ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)])
    total_ms = max_over_ranks(float(step_ms.sum()), world, dev)
    profiled_ms = float(np.array([evs[i][0].elapsed_time(evs[i][-1]) for i in range(args.steps)]).mean())
    status = layer.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    # the clock the expert GEMMs actually ran at (SM cycles over %globaltimer inside every
    # CTA, MOE_OPTION_GEMM_CLOCK), outside the timed region, with the same flushed steps:
    # under the 1 kW cap it sits well below the sampled clock of the lines above
    layer.set_option(MOE_OPTION_GEMM_CLOCK, 1)
    layer.gemm_clock_mhz()
    for i in range(min(args.steps, 10)):
        flush.zero_()
        moe_forward(layer.handle, batches[args.warmup + i], T, out, ws)
    gemm_mhz_pair = layer.gemm_clock_mhz()
    layer.set_option(MOE_OPTION_GEMM_CLOCK, 0)
    clocks["gemm_effective_mhz"] = {"up": round(gemm_mhz_pair[0], 1),
                                    "down": round(gemm_mhz_pair[1], 1)}

    # end to end through the public API, serial (the bench line's e2e): per step, outside
    # the events the L2 flush as in the device-timed region; inside them the copy of that
    # step's x from pinned host memory, the forward and the copy of its out back to pinned
    # host memory, one after another on the launch stream.
    hx = [b.cpu().pin_memory() for b in batches]
    hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    dxb = [torch.empty_like(batches[0]) for _ in range(2)]
    outb = [torch.empty_like(out) for _ in range(2)]
    evs_e2e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]

    def serial_step(i, evp=None):
        flush.zero_()
        if evp:
            evp[0].record(st)
        dxb[0].copy_(hx[i], non_blocking=True)
        moe_forward(layer.handle, dxb[0], T, outb[0], ws)
        hout[0].copy_(outb[0], non_blocking=True)
        if evp:
            evp[1].record(st)

    for i in range(args.warmup):
        serial_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    for i in range(args.steps):
        serial_step(args.warmup + i, evs_e2e[i])
    torch.cuda.synchronize()
    e2e_serial_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs_e2e), world, dev)
    if world > 1:
        dist.barrier()

    # end to end, pipelined (reported beside it): two device buffers and two copy streams,
    # step i's copies run while step i-1 (out) and step i+1 (in) compute, as a serving loop
    # would overlap them; each forward waits for its own input copy, each output copy for
    # its own forward, and no buffer is reused before the copy that reads it has finished.
    # Steps run back to back with no L2 flush between them.
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # input copy of buffer j done
    ev_fwd = [torch.cuda.Event() for _ in range(2)]   # forward on buffer j done
    ev_out = [torch.cuda.Event() for _ in range(2)]   # output copy of buffer j done

    def e2e_steps(first, n):
        for i in range(first, first + n):
            j = i % 2
            if i - first >= 2:  # buffer j is free once step i-2's forward and copy are done
                s_in.wait_event(ev_fwd[j])
                st.wait_event(ev_out[j])
            with torch.cuda.stream(s_in):
                dxb[j].copy_(hx[i], non_blocking=True)
                ev_in[j].record(s_in)
            st.wait_event(ev_in[j])
            moe_forward(layer.handle, dxb[j], T, outb[j], ws)
            ev_fwd[j].record(st)
            s_out.wait_event(ev_fwd[j])
            with torch.cuda.stream(s_out):
                hout[j].copy_(outb[j], non_blocking=True)
                ev_out[j].record(s_out)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps(0, args.warmup)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0.record(st)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    e2e_steps(args.warmup, args.steps)
    for j in range(2):
        st.wait_event(ev_out[j])
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if world > 1:
        dist.barrier()

    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    mean_stage = stage_ms.mean(axis=0)
    names = list(PROFILE_STAGE_NAMES)
    up_i, down_i = names.index("expert_up_swiglu"), names.index("expert_down")
    dom = up_i if mean_stage[up_i] >= mean_stage[down_i] else down_i
    dom_name = "grouped_gemm_up" if dom == up_i else "grouped_gemm_down"
    key = "up" if dom == up_i else "down"
    layer_bytes = float(np.mean([a["layer_bytes"] for a in algo]))
    layer_flops = float(np.mean([a["layer_flops"] for a in algo]))
    step_s = total_ms / args.steps / 1e3
    kern = kernel_roofline(algo, key, mean_stage[dom] / 1e3, peaks)
    kern["traffic"] = ncu_traffic(dom_name, args.workload)
    kern["kernel"] = dom_name
    kern["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback"
    # the roofline of the whole forward when the workload is tensor-bound (its flops per
    # algorithmic byte above the ridge of the burst peaks): one forward's flops over the
    # plain step time against the burst bf16 peak, and beside it against the peak of the
    # clock regime the GEMMs were measured in (their effective clock, above); otherwise the
    # dominant kernel's, which streams the weights at the HBM bound
    t_up, t_down = mean_stage[up_i], mean_stage[down_i]
    gemm_mhz = ((t_up * gemm_mhz_pair[0] + t_down * gemm_mhz_pair[1]) / (t_up + t_down)
                if (t_up + t_down) > 0 and min(gemm_mhz_pair) > 0 else None)
    roof = layer_roofline(layer_bytes, layer_flops, step_s, peaks, gemm_mhz)
    if roof is None:
        roof = kern
    else:
        roof["traffic"] = ncu_traffic("layer", args.workload)
        roof["kernel"] = "moe_forward (all kernels of one forward)"
        roof["peak_source"] = kern["peak_source"] + ", burst bf16"
    value = job_throughput(T, args.steps, world, total_ms)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded; a different x batch every step; random-init weights)",
        "config": {"workload": w.name, "tokens": T, "d_model": w.d, "n_experts": w.E,
                   "top_k": w.k, "d_ff": w.f, "n_shared": w.n_shared,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "flushed between timed steps (256 MiB write, outside the events)"},
        "roofline": roof,
        "kernel_roofline": kern,
        "layer_roofline": {"algorithmic_bytes": int(layer_bytes), "algorithmic_flops": int(layer_flops),
                           "hbm_frac": round(layer_bytes / step_s / 1e9 / peaks["hbm_gbs"], 4),
                           "tensor_frac": round(layer_flops / step_s / 1e12 / peaks["bf16_tflops"], 4),
                           # against the measured sustained bf16 rate (the GEMM loop under the
                           # 1 kW power cap): the regime of a long back-to-back step loop
                           "tensor_frac_sustained": round(
                               layer_flops / step_s / 1e12 /
                               peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), 4),
                           "touched_experts_mean": float(np.mean([a["touched"] for a in algo]))},
        "stages_ms": {n: round(float(v), 4) for n, v in zip(names, mean_stage)},
        "profiled_ms_per_step": round(profiled_ms, 4),
        "e2e": {"value": round(job_throughput(T, args.steps, world, e2e_serial_ms), 1),
                "unit": "tokens/s",
                "h2d_bytes_per_step": int(T * w.d * (2 if w.dtype == "bf16" else 4)),
                "d2h_bytes_per_step": int(T * w.d * (2 if w.dtype == "bf16" else 4)),
                "copies": "serial: per step copy x in (pinned host), forward, copy out back "
                          "(pinned host) on one stream; L2 flushed between steps outside the "
                          "events, as in the device-timed region"},
        "e2e_pipelined": {"value": round(job_throughput(T, args.steps, world, e2e_ms), 1),
                          "unit": "tokens/s",
                          "copies": "each step's in/out copies overlap the neighbouring "
                                    "steps' forwards (two device buffers, two copy streams); "
                                    "no L2 flush between steps"},
        # kernels of the timed region: every rank's forwards, as the library plans them
        "gpu_launches": int(world * args.steps * moe_forward_launch_count(layer.handle, T)),
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, inp, batches[args.warmup], budget_s=args.cpu_budget)
    return res


# ------------------------------------------------------------------------ oracle timing
def _host_weights(inp):
    from sparse_moe_layer_warp_b200 import synth

    cv = synth.to_numpy_bits
    return [cv(t) for t in (inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down)]


def cpu_baseline(w, inp, x_batch, budget_s=15.0, host=None):
    """The oracle, as it stands, on a bounded sample of one batch (tokens/s)."""
    import numpy as np

    from oracle import oracle_moe_forward, oracle_num_threads
    from sparse_moe_layer_warp_b200 import synth

    wr, b, wg, wu, wd = host if host is not None else _host_weights(inp)
    x = synth.to_numpy_bits(x_batch)
    cores = oracle_num_threads()
    n = min(x.shape[0], cores)
    done, t0 = 0, time.perf_counter()
    start = 0
    while True:
        toks = (np.arange(n) + start) % x.shape[0]
        oracle_moe_forward(x, wr, b, wg, wu, wd, k=w.k, n_shared=w.n_shared,
                           routed_scale=w.routed_scale, tokens=toks.astype(np.int32))
        done += n
        start += n
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": round(done / el, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} tokens of one {w.name} batch ({el:.1f} s of plain-C fp64 oracle, "
                      f"OpenMP over tokens)"}


def cpu_baseline_backward(w, inp, x_batch, dout_batch, idx, gates, budget_s=10.0):
    """The oracle's backward, as it stands (single-threaded, fp64), on tokens of one batch
    taken one at a time until the budget is spent (tokens/s)."""
    from oracle import oracle_moe_backward
    from sparse_moe_layer_warp_b200 import synth

    import numpy as np

    wr, _, wg, wu, wd = _host_weights(inp)
    x = synth.to_numpy_bits(x_batch)
    o = synth.to_numpy_bits(dout_batch)
    E = w.E
    done, el = 0, 0.0
    while el < budget_s:
        t = done % x.shape[0]
        # the token's own experts (and the shared one) only: the oracle's dense fp64
        # gradients of all experts would not fit in host memory at full size
        sel = np.concatenate([idx[t], np.arange(E, E + w.n_shared)]).astype(np.int64)
        args = (x[t:t + 1], o[t:t + 1], np.ascontiguousarray(wr[idx[t]]),
                np.ascontiguousarray(wg[sel]), np.ascontiguousarray(wu[sel]),
                np.ascontiguousarray(wd[sel]), np.arange(w.k, dtype=np.int32)[None],
                gates[t:t + 1])
        t0 = time.perf_counter()
        oracle_moe_backward(*args, w.routed_scale, w.n_shared)
        el += time.perf_counter() - t0
        done += 1
    return {"value": round(done / el, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} tokens of one {w.name} batch, one at a time ({el:.1f} s of the "
                      f"plain-C fp64 oracle backward, single-threaded, on each token's "
                      f"{w.k} + {w.n_shared} experts)"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import numpy as np
    import torch

    from oracle import oracle_moe_forward, oracle_num_threads, oracle_set_num_threads
    from sparse_moe_layer_warp_b200 import synth

    # rank 0 runs alone: every host core this process may use (torchrun sets
    # OMP_NUM_THREADS=1 for each of its processes)
    oracle_set_num_threads(len(os.sched_getaffinity(0)))
    w = synth.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = synth.make_inputs(w, device=dev)
    host = _host_weights(inp)
    wr, b, wg, wu, wd = host
    cores = oracle_num_threads()
    sample = min(w.T, max(1, cores))
    xs = [synth.to_numpy_bits(synth.make_x(w, w.T, device=dev, seed=1000 + i))
          for i in range(args.steps + args.warmup)]

    def step(i):
        toks = np.arange(sample, dtype=np.int32)
        oracle_moe_forward(xs[i], wr, b, wg, wu, wd, k=w.k, n_shared=w.n_shared,
                           routed_scale=w.routed_scale, tokens=toks)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    value = args.steps * sample / el
    desc = (f"{sample} of the {w.T} tokens of each step's {w.name} batch, plain-C fp64 oracle, "
            f"OpenMP over tokens")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "tokens": w.T, "d_model": w.d, "n_experts": w.E,
                       "top_k": w.k, "d_ff": w.f, "n_shared": w.n_shared,
                       "parallelism": "rank 0 only (host cores)",
                       "l2": "not applicable (host oracle)"},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------- backward arm
# fp32 CUDA-core peak of the backward kernels: 148 SMs x 128 FP32 lanes x 2 flop (FMA) x
# the 1965 MHz maximum SM clock
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_backward(args, rank, world, local_rank):
    """Times moe_backward (gradients of <forward(x), dout>) on the workload: a separate
    measurement, not the forward's headline line."""
    import numpy as np
    import torch
    import torch.distributed as dist

    from sparse_moe_layer_warp_b200 import MoELayer, synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    T = w.T
    inp = synth.make_inputs(w, device=dev)
    layer = MoELayer(inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down, top_k=w.k,
                     max_tokens=T, n_shared=w.n_shared, routed_scale=w.routed_scale)
    nb = args.steps + args.warmup
    xs = [synth.make_x(w, T, device=dev, seed=1000 * (rank + 1) + i) for i in range(nb)]
    douts = [synth.make_x(w, T, device=dev, seed=5000 * (rank + 1) + i) for i in range(nb)]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    touched = []
    for i in range(args.warmup, nb):
        touched.append(int((layer.route(x=xs[i])["counts"] > 0).sum().item()) + w.n_shared)
    # --saved: each step's pre-activations kept by a training forward (moe_forward_save) of
    # its x, run before the timed region; the timed call then skips their recompute
    saved = [None] * nb
    if args.saved:
        for i in range(nb):
            saved[i] = layer.forward_save(xs[i])[1]
    # weight-gradient buffers allocated once; every step accumulates into them
    grads = layer.backward(xs[0], douts[0], saved=saved[0])
    for i in range(args.warmup):
        flush.zero_()
        layer.backward(xs[i], douts[i], grads=grads, saved=saved[i], overwrite=args.overwrite)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(visible.split(",")[local_rank] if visible else local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(st)
        layer.backward(xs[args.warmup + i], douts[args.warmup + i], grads=grads,
                       saved=saved[args.warmup + i], overwrite=args.overwrite)
        ev[i][1].record(st)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    step_ms = np.array([a.elapsed_time(b) for a, b in ev])
    total_ms = max_over_ranks(float(step_ms.sum()), world, dev)
    if layer.device_status() != 0:
        raise RuntimeError("device status after the timed region")
    if rank != 0:
        return None
    P = T * w.k + w.n_shared * T
    es = 2 if w.dtype == "bf16" else 4
    tm = float(np.mean(touched))
    peaks, src = load_peaks()
    step_s = total_ms / args.steps / 1e3
    if w.dtype == "bf16":
        # tensor cores: recompute a and b (4 P f d), dh (2), rows of dx (4), three weight
        # gradients (6): 16 P f d flops; the router adds 4 T k d.  Weights of the touched
        # experts read five times (gate and up twice, down once); their three fp32 weight
        # gradients and the router's read and written (they accumulate).
        flops = 16.0 * P * w.f * w.d + 4.0 * T * w.k * w.d
        nbytes = tm * 5 * w.f * w.d * es + tm * 3 * w.f * w.d * 8 + w.E * w.d * 8
        label = "tcgen05 grouped GEMMs"
        if args.saved:
            # a and b kept by the training forward: no recompute (12 P f d flops, weights read
            # three times), the kept fp32 a, b read once
            flops = 12.0 * P * w.f * w.d + 4.0 * T * w.k * w.d
            nbytes = (tm * 3 * w.f * w.d * es + tm * 3 * w.f * w.d * 8 + w.E * w.d * 8
                      + 8.0 * P * w.f)
            label += ", pre-activations kept by the training forward"
        if args.overwrite:
            # gradients written, not read: every expert's (zeros for the untouched ones)
            G = w.E + w.n_shared
            nbytes += G * 3 * w.f * w.d * 4 - tm * 3 * w.f * w.d * 8 - w.E * w.d * 4
            label += ", weight gradients overwritten"
        peak_c = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        peak_name = f"bf16 dense, sustained ({src})"
        unit_c, kind = "TFLOP/s", "tensor"
    else:
        # CUDA cores: recompute a and b, unscaled outputs, dh, rows of dx (two products),
        # three weight gradients: 18 P f d flops; weights read six times
        flops = 18.0 * P * w.f * w.d + 4.0 * T * w.k * w.d
        nbytes = tm * 6 * w.f * w.d * es + tm * 3 * w.f * w.d * 8 + w.E * w.d * 8
        peak_c, peak_name = FP32_ALU_TFLOPS, "fp32 FFMA: 148 SMs x 128 lanes x 2 x 1965 MHz"
        unit_c, kind = "TFLOP/s", "alu"
        label = "fp32 CUDA-core kernels"
    comp = flops / step_s / 1e12
    hbm = nbytes / step_s / 1e9
    ridge = peak_c * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops / nbytes > ridge:
        roof = {"bound": kind, "achieved": round(comp, 2), "peak": round(peak_c, 1),
                "unit": unit_c, "frac": round(comp / peak_c, 4)}
    else:
        roof = {"bound": "hbm", "achieved": round(hbm, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(hbm / peaks["hbm_gbs"], 4)}
    roof.update({"traffic": None, "kernel": "moe_backward (all kernels)",
                 "algorithmic_flops_per_step": int(flops), "algorithmic_bytes_per_step": int(nbytes),
                 "peak_source": f"{peak_name}; HBM {src}"})
    return {
        "metric": f"MoE-layer backward tokens/s on 1 B200 ({label})",
        "pass": "backward",
        "value": round(job_throughput(T, args.steps, world, total_ms), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded; fresh x and dout every step; random-init weights)",
        "config": {"workload": w.name, "tokens": T, "d_model": w.d, "n_experts": w.E,
                   "top_k": w.k, "d_ff": w.f, "n_shared": w.n_shared,
                   "l2": "flushed between timed steps (256 MiB write, outside the events)"},
        "roofline": roof, "clocks": clocks,
    } | ({} if args.no_cpu_baseline else {"cpu_baseline": cpu_baseline_backward(
        w, inp, xs[args.warmup], douts[args.warmup], *_routing_np(layer, xs[args.warmup]),
        budget_s=min(args.cpu_budget, 10.0))})


def run_ep_rank(args, rank, world, local_rank):
    """One rank's device work in the expert-parallel layer (--ep-ranks R, emulated on this
    GPU: no exchange is timed).  The global batch is R x T tokens (T = the workload's tokens
    per rank); rank 0 holds EP group 0 (experts [0, E/R) and the shared expert).
    allgather: its partial forward of all R x T tokens in its experts plus the shared expert
    on its own T tokens, and the rounding of its T output rows.  alltoall: its partial forward
    of the tokens the other ranks would send it (every token of the global batch with a slot
    in its experts), and the per-token combine of its own T tokens' returned rows (taken as
    the rows it computed itself) with its shared expert."""
    import numpy as np
    import torch

    from sparse_moe_layer_warp_b200 import synth
    from sparse_moe_layer_warp_b200.expert_parallel import LibraryOps, expert_range

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    R, T = args.ep_ranks, w.T
    inp = synth.make_inputs(w, device=dev, T=1)
    e0, e1 = expert_range(w.E, 0, R)
    sl = lambda t: torch.cat([t[e0:e1], t[w.E:]]).contiguous()  # noqa: E731
    ops = LibraryOps(inp.w_router, inp.bias, sl(inp.w_gate), sl(inp.w_up), sl(inp.w_down),
                     n_experts=w.E, top_k=w.k, max_tokens=T, rank=0, world=R,
                     n_shared=w.n_shared, routed_scale=w.routed_scale)
    del inp
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    nb = args.steps + args.warmup
    steps = []
    for i in range(nb):
        xg = synth.make_x(w, R * T, device=dev, seed=2000 + i)
        idx, gates = ops.route(xg)
        if args.ep_mode == "allgather":
            steps.append((xg, idx, gates))
        else:  # the received tokens: every token with a slot in this rank's experts
            keep = ((idx >= e0) & (idx < e1)).any(dim=1).nonzero().squeeze(1)
            steps.append((xg[keep].contiguous(), idx[keep].contiguous(),
                          gates[keep].contiguous(), xg[:T].contiguous(), idx[:T].contiguous(),
                          gates[:T].contiguous()))
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()

    def one(s):
        if args.ep_mode == "allgather":
            xg, idx, gates = s
            part = ops.partial(xg, idx, gates, (e0, e1), (0, T))
            return ops.combine(None, None, None, part[:T].contiguous(), R, T)
        xr, ir, gr, xo, io, go = s
        part = ops.partial(xr, ir, gr, (e0, e1), (0, 0))
        shared = ops.partial(xo, io, go, (e0, e0), (0, T))
        return part, shared

    for i in range(args.warmup):
        flush.zero_()
        one(steps[i])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(st)
        one(steps[args.warmup + i])
        ev[i][1].record(st)
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    rows = float(np.mean([s[0].shape[0] for s in steps[args.warmup:]]))
    # bytes a rank must stream: its touched experts' weights once (plus the shared expert)
    touched = float(np.mean([
        int(torch.unique(s[1][((s[1] >= e0) & (s[1] < e1))]).numel()) for s in steps[args.warmup:]]))
    wbytes = (touched + w.n_shared) * 3 * w.d * w.f * 2
    # flops of the rank's expert work: its slots of the global batch and the shared expert
    # on its own tokens (3 products of d x f per row)
    slots = float(np.mean([int(((s[1] >= e0) & (s[1] < e1)).sum()) for s in steps[args.warmup:]]))
    flops = 2.0 * (slots + T * w.n_shared) * 3 * w.d * w.f
    peaks, src = load_peaks()
    return {"pass": f"ep rank (emulated, {args.ep_mode})", "ep_ranks": R, "workload": w.name,
            "tokens_per_rank": T, "rows_in_rank_partial": rows, "ms_per_step": round(ms, 4),
            "rank_touched_experts": touched,
            "rank_weight_bytes": int(wbytes),
            "rank_weight_stream_frac_of_hbm": round(wbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
            "rank_slots": slots, "rank_flops": int(flops),
            "rank_tensor_frac_burst": round(flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
            "note": "device steps of one rank only; the NCCL exchange is not timed (one GPU)"}


def _routing_np(layer, x):
    r = layer.route(x=x)
    return r["idx"].cpu().numpy(), r["gates"].cpu().numpy()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--overwrite", action="store_true",
                    help="with --pass backward: the weight gradients are set, not accumulated "
                         "(MOE_BACKWARD_OVERWRITE)")
    ap.add_argument("--saved", action="store_true",
                    help="with --pass backward: time moe_backward_saved on pre-activations "
                         "kept by a training forward (moe_forward_save) instead")
    ap.add_argument("--pass", dest="which", default="forward",
                    choices=["forward", "backward", "ep"],
                    help="backward: time moe_backward instead; ep: one rank's device work in "
                         "the expert-parallel layer (separate measurements)")
    ap.add_argument("--ep-ranks", type=int, default=8)
    ap.add_argument("--ep-mode", default="allgather", choices=["allgather", "alltoall"])
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        ap.error(f"WORLD_SIZE={world} but --gpus {args.gpus}")

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch.distributed as dist
    import datetime

    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=None)
    try:
        run = {"backward": run_backward, "ep": run_ep_rank}.get(args.which, run_ours)
        res = run(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
