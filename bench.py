#!/usr/bin/env python
"""Engram forward benchmark: tokens/s of engram_forward on B200.

One step = one engram_forward over one batch of the workload (hash + row
gather -> tcgen05 projection on CTA pairs + score partials -> gate -> gated
value + short conv + residual), inputs resident in HBM.  Default workload: the
largest one that fits one GPU, the HBM-scale table (B=16, T=4096, 32 heads x
2^22 rows x 64 bf16 = 17.2 GB of tables, H=4096, hc=4); --config selects the
others (model_bf16, large_table_bf16, decode_bf16, tiny_f32).

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events on
the launching stream; between steps, outside the events, L2 is flushed (a
256 MB write) and then drained (a 256 MB read of another buffer, so the
flush's dirty lines are written back before the next step starts instead of
during its first kernel); barrier + synchronize on both sides; the max over
ranks is reported.
Multi-GPU: one process per GPU, every rank runs its own replica of the
workload (the pass has no cross-sequence exchange), scaling "weak".

The headline loop records events only around each whole step, so the
library's kernels chain with programmatic dependent launch; a second loop of
K steps over the same inputs has the library record events at its stage
boundaries (engram_set_stage_events), which times the dominant kernel (the
projection) and the other stages.  The CPU baseline is
the float64 oracle on a bounded sample of the same workload on the host cores.

--impl reference runs that oracle as the reference arm (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np
import torch

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    """Peaks from MEASURED_PEAKS.json when it holds them (numbers under the
    keys of PEAKS_FALLBACK), else the machine's fallback figures, key by key."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"
    peaks, measured = dict(PEAKS_FALLBACK), []
    for k in PEAKS_FALLBACK:
        v = d.get(k) if isinstance(d, dict) else None
        if isinstance(v, (int, float)) and v > 0:
            peaks[k] = float(v)
            measured.append(k)
    if len(measured) == len(PEAKS_FALLBACK):
        return peaks, "measured"
    if not measured:
        return peaks, "fallback"
    return peaks, "measured (%s), else fallback" % ", ".join(measured)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        # nvidia-smi numbers GPUs physically; address this one by its UUID
        try:
            self.index = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [x for x in vis.split(",") if x.strip()]
            self.index = ids[device_index] if device_index < len(ids) else str(device_index)
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.index, "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    sm.append(float(parts[2]))
                    smax.append(float(parts[3]))
                except ValueError:
                    continue
                try:
                    pw.append(float(parts[4]))
                except ValueError:
                    pass
                for n, v in zip(names, parts[6:10]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(smax),
                "power_w": float(np.median(pw)) if pw else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- oracle (CPU)
def oracle_sample(w, tokens: int, nthreads: int, p=None):
    """Prepare the float64 oracle over the first `tokens` positions of
    sequence 0 of a workload of the same shapes and distributions (whole pass
    from ids, host cores).  Returns (n, run) where run() -> seconds.  For a
    workload whose tables are drawn on the device, p (its device Params) may
    be passed in to avoid drawing them again."""
    from hashed_gram_conditional_hash_b200 import workloads as W
    from oracle import engram_oracle as O
    n = max(1, min(tokens, w.B * w.seq_len))
    if W.gen_device_for(w, "cuda") == "cpu":
        # whole sequences of the workload's length (the last one cut to fit)
        T = min(n, w.seq_len)
        wp = w.replace(B=(n + T - 1) // T, T=T, decode_calls=0)
        n = wp.B * wp.T
        p = W.make_params(wp, "cpu")
        x = p.ids.numpy()
        if p.lookup is not None:
            x = O.compress_ids(x, p.lookup.numpy())

        def run():
            t0 = time.perf_counter()
            O.forward(x=x, orders=wp.orders, J=wp.heads_per_order, mult=p.mult, primes=p.primes,
                      row_offsets=p.offsets, pad_id=wp.pad_id, table=p.table, w_value=p.w_value,
                      w_key=p.w_key, norm_key=p.norm_key, norm_query=p.norm_query,
                      conv_w=p.conv_w, hidden=p.hidden, K=wp.conv_kernel, dil=wp.dil,
                      nthreads=nthreads)
            return time.perf_counter() - t0
        return n, run
    # tables drawn on the device: the oracle receives the rows it needs
    if p is None:
        p = W.make_params(w, "cuda")
    dev = p.table.device
    n = min(n, w.seq_len)
    pos = [(0, t) for t in range(n)]
    if w.decode_calls:
        hid = lambda b, t: p.hidden[torch.from_numpy(t).to(dev), torch.from_numpy(b).to(dev)].cpu()
    else:
        hid = lambda b, t: p.hidden[torch.from_numpy(b).to(dev), torch.from_numpy(t).to(dev)].cpu()
    x = p.ids.cpu().numpy()
    args = (p.w_value.cpu(), p.w_key.cpu(), p.norm_key.cpu(), p.norm_query.cpu(), p.conv_w.cpu())

    def run():
        t0 = time.perf_counter()
        O.forward_sampled(x, pos, w.orders, w.heads_per_order, p.mult, p.primes, p.offsets,
                          w.pad_id, lambda r: p.table[torch.from_numpy(r).to(dev)].cpu(), hid,
                          *args, K=w.conv_kernel, dil=w.dil, nthreads=nthreads)
        return time.perf_counter() - t0
    return n, run


def oracle_tokens_for(w, seconds: float, nthreads: int, p=None) -> int:
    """Sample size that takes about `seconds` of oracle time (calibrated)."""
    n, run = oracle_sample(w, 32, nthreads, p)
    run()
    dt = run()
    return int(max(8, n / max(dt, 1e-6) * seconds))


def cpu_baseline(w, budget_s: float, p=None):
    """The oracle on all host cores (the reported value) and on one core."""
    nthreads = os.cpu_count() or 1
    n, run = oracle_sample(w, oracle_tokens_for(w, budget_s, nthreads, p), nthreads, p)
    dt = run()
    n1, run1 = oracle_sample(w, oracle_tokens_for(w, budget_s / 4, 1, p), 1, p)
    dt1 = run1()
    return {"value": n / dt, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
            "single_thread_value": n1 / dt1,
            "sample": "%d positions (whole sequences) of a workload with the shapes and "
                      "distributions of %s, whole pass from ids, float64, %.1f s; one thread: %d "
                      "positions, %.1f s" % (n, w.name, dt, n1, dt1)}


# ---------------------------------------------------------------- GPU arm
def kernel_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    record (profiles/dram_traffic.json), only if the kernel's source file is
    unchanged since that capture; else None."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)["%s@%s" % (kernel, workload)]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != rec["source_sha1"]:
                return None
        return rec["dram_read_bytes"] + rec["dram_write_bytes"]
    except (OSError, KeyError, ValueError):
        return None


def algorithmic(w):
    """Per-token algorithmic bytes / flops of each stage (see the design notes)."""
    es = w.elem_bytes
    return {
        "proj_flops": 2.0 * w.E * w.hidden * (1 + w.hc_mult),
        # hash + gather kernel: ids in, the nh table rows read, e written
        "hash_bytes": 8.0 + 2.0 * w.E * es,
        "conv_bytes": float(w.hidden * es + 4 * w.hc_mult + w.hc_mult * w.hidden * es),
        "pass_bytes": float(8 + w.E * es + 2 * w.hc_mult * w.hidden * es),
    }


def pass_roofline(w, tokens_step, step_s, tc_peak_tflops, hbm_gbs):
    """The whole pass against its own roofline: the bytes the method must move
    (ids, gathered rows, hidden read, Y written, the weights once per step;
    in decode also the three V-ring taps read and the step's V row written)
    and the projection flops; t = max(bytes / HBM peak, flops / tensor peak),
    frac = t / the measured step time."""
    es = w.elem_bytes
    per_tok = 8 + w.E * es + 2 * w.hc_mult * w.hidden * es
    if w.decode_calls:
        per_tok += 4 * w.hidden * es
    weights = (1 + w.hc_mult) * w.hidden * w.E * es
    nbytes = per_tok * tokens_step + weights
    flops = algorithmic(w)["proj_flops"] * tokens_step
    t_hbm = nbytes / (hbm_gbs * 1e9)
    t_tc = flops / (tc_peak_tflops * 1e12)
    return {"bytes_per_step": nbytes, "flops_per_step": flops, "t_hbm_us": t_hbm * 1e6,
            "t_tensor_us": t_tc * 1e6, "bound": "tensor" if t_tc >= t_hbm else "hbm",
            "frac": max(t_hbm, t_tc) / step_s}


def max_over_ranks(t, world):
    """Element-wise max over ranks of a float64 tensor of per-rank timings
    (on the device of the process group's backend); identity for one rank."""
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t


def job_throughput(world, units_per_step_per_rank, steps, max_ms):
    """Whole-job units/s: every rank processes its own replica's units, timed
    by the slowest rank."""
    return world * units_per_step_per_rank * steps / (max_ms / 1e3)


def device_memory(w, p, ws, y):
    """Device memory of one replica, GB: tables, weights, this step's inputs and
    output, the forward workspace, and the library's static scratch (the array
    behind engram_forward_no_alloc, held by every GPU that loads libengram.so
    whether or not that entry point is called)."""
    from hashed_gram_conditional_hash_b200 import _lib as L
    nb = lambda t: t.numel() * t.element_size() if t is not None else 0
    weights = sum(nb(t) for t in (p.w_value, p.w_key, p.norm_key, p.norm_query, p.conv_w, p.lookup))
    return {"tables": round(nb(p.table) / 1e9, 3), "weights": round(weights / 1e9, 3),
            "inputs_outputs": round((nb(p.ids) + nb(p.hidden) + nb(y)) / 1e9, 3),
            "workspace": round(nb(ws) / 1e9, 3),
            "static_scratch": round(L.NO_ALLOC_SCRATCH_BYTES / 1e9, 3)}


class L2Flush:
    """Between timed steps: write 256 MB (twice L2), then read another 256 MB
    so that the written lines leave L2 now rather than during the next step's
    first kernel (whose stage time would otherwise include that write-back)."""

    def __init__(self, device):
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.src = torch.ones(32 << 20, dtype=torch.int64, device=device)
        self.out = torch.empty((), dtype=torch.int64, device=device)

    def __call__(self, i):
        self.buf.fill_(i & 0xff)
        torch.sum(self.src, dim=0, out=self.out)


def run_ours(args, rank, world, device):
    from hashed_gram_conditional_hash_b200 import EngramLayer
    from hashed_gram_conditional_hash_b200 import _lib as L
    from hashed_gram_conditional_hash_b200 import workloads as W

    w = W.CONFIGS[args.config]
    if w.decode_calls and args.decode_calls:
        w = w.replace(decode_calls=args.decode_calls)
    peaks, peak_kind = load_peaks()
    L.engram_set_overlap_chunks(args.overlap_chunks)
    L.engram_set_debug(args.debug_flags)
    p = W.make_params(w, device)
    layer = EngramLayer.from_params(p)
    engine = "tcgen05" if L.engram_projection_engine(layer.cfg) == L.ENGINE_TCGEN05 else "simt"
    # the dense tensor-core projection runs on CTA pairs
    kname = "proj_tc2_kernel" if engine == "tcgen05" else "proj_simt_kernel"
    stream = torch.cuda.current_stream()
    decode = bool(w.decode_calls)
    if decode:
        Bq, Tq = w.B, 1
        state = layer.new_state(w.B)
        steps_ids = p.ids.t().contiguous().view(w.decode_calls, w.B, 1)
        step_in = lambda i: (steps_ids[i % w.decode_calls],
                             p.hidden[i % w.decode_calls].view(w.B, 1, w.hc_mult, w.hidden))
    else:
        Bq, Tq = w.B, w.T
        state = None
        step_in = lambda i: (p.ids, p.hidden)
    ws = layer.workspace(Bq, Tq)
    y = torch.empty((Bq, Tq, w.hc_mult, w.hidden), dtype=w.torch_dtype, device=device)
    flush = L2Flush(device)
    st = torch.zeros(1, dtype=torch.int32, device=device)

    def step(i):
        ids, hid = step_in(i)
        layer.forward(ids, hid, y=y, ws=ws, state=state, dev_status=st)

    for i in range(args.warmup):
        step(i)
        flush(i)
    torch.cuda.synchronize()
    bits = L.engram_read_status(st)
    if bits:
        raise RuntimeError("device status 0x%x during warm-up" % bits)

    K = args.steps
    mk = lambda: torch.cuda.Event(enable_timing=True)
    # Loop 1 (the headline): events around each whole step only, so the
    # library's kernels follow one another with programmatic dependent launch.
    # Loop 2 (the stage times and the roofline): the library records events at
    # its stage boundaries, which also serialises those boundaries.
    ev_step = [(mk(), mk()) for _ in range(K)]
    ev = [{k: mk() for k in ("before_hash", "before_projection", "before_gate", "before_conv",
                             "after_conv")} for _ in range(K)]
    for e in ev:  # create the underlying events before handing them to the library
        for x in e.values():
            x.record(stream)
    torch.cuda.synchronize()

    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    n0 = L.engram_launch_count()
    for i in range(K):
        ev_step[i][0].record(stream)
        step(args.warmup + i)
        ev_step[i][1].record(stream)
        flush(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    launches = L.engram_launch_count() - n0
    torch.cuda.synchronize()
    for i in range(K):
        L.engram_set_stage_events(ev[i])
        step(args.warmup + K + i)
        L.engram_set_stage_events(None)
        flush(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop() if clocks else None
    bits = L.engram_read_status(st)
    if bits:
        raise RuntimeError("device status 0x%x during the timed steps" % bits)

    t_step = sum(a.elapsed_time(b) for a, b in ev_step)                                # ms
    t_proj = sum(e["before_projection"].elapsed_time(e["before_gate"]) for e in ev)
    t_hash = sum(e["before_hash"].elapsed_time(e["before_projection"]) for e in ev)
    t_gate = sum(e["before_gate"].elapsed_time(e["before_conv"]) for e in ev)
    t_conv = sum(e["before_conv"].elapsed_time(e["after_conv"]) for e in ev)
    times = torch.tensor([t_step, t_proj, t_hash, t_gate, t_conv], dtype=torch.float64, device=device)
    t_step, t_proj, t_hash, t_gate, t_conv = max_over_ranks(times, world).tolist()

    tokens_step = Bq * Tq
    value = job_throughput(world, tokens_step, K, t_step)
    a = algorithmic(w)
    proj_s = t_proj / K / 1e3
    proj_tflops = a["proj_flops"] * tokens_step / proj_s / 1e12
    # the burst peak for a step that runs at full clock, the sustained one when
    # the clocks sampled during the timed loops sat below it (power cap)
    sustained = bool(clk and clk.get("sm_mhz") and clk.get("sm_max_mhz")
                     and clk["sm_mhz"] < 0.97 * clk["sm_max_mhz"]) or "sw_power_cap" in (clk or {}).get("reasons", [])
    tc_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    stages = {
        "hash_gather": {"us": t_hash / K * 1e3, "bound": "hbm",
                 "achieved_gbs": a["hash_bytes"] * tokens_step / (t_hash / K / 1e3) / 1e9},
        "projection": {"us": t_proj / K * 1e3, "bound": "tensor", "engine": engine,
                       "achieved_tflops": proj_tflops},
        "gate": {"us": t_gate / K * 1e3},
        "conv": {"us": t_conv / K * 1e3, "bound": "hbm",
                 "achieved_gbs": a["conv_bytes"] * tokens_step / (t_conv / K / 1e3) / 1e9},
    }
    for s in ("hash_gather", "conv"):
        stages[s]["frac_of_measured_hbm"] = stages[s]["achieved_gbs"] / peaks["hbm_gbs"]
    result = {
        "metric": "Engram forward tokens/s on 1xB200 (engram_forward); % of HBM and bf16 tensor roofline",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": t_step / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded; shapes and distributions of the workload)",
        "config": {"workload": w.name, "B": w.B, "T": Tq, "tokens_per_step_per_gpu": tokens_step,
                   "orders": list(w.orders), "heads_per_order": w.heads_per_order,
                   "row_dim": w.row_dim, "hidden": w.hidden, "hc_mult": w.hc_mult,
                   "dilation": w.dil, "table_gb": round(W.table_bytes(w) / 1e9, 3),
                   "l2": "flushed (256 MB write) and drained (256 MB read) between timed steps",
                   "parallelism": "replicas x%d" % world, "projection_engine": engine,
                   "device_memory_gb": device_memory(w, p, ws, y),
                   "overlap_chunks": 1 if decode else min(w.B, 8, max(1, args.overlap_chunks or
                                                                        int(os.environ.get("ENGRAM_OVERLAP_CHUNKS", "1"))))},
        "roofline": {"bound": "tensor", "kernel": kname,
                     "achieved": proj_tflops, "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": proj_tflops / tc_peak, "peak_kind": "%s bf16 %s" % (peak_kind, "sustained" if sustained else "burst"),
                     "frac_of_burst": proj_tflops / peaks["bf16_tflops"],
                     "frac_of_sustained": proj_tflops / peaks["bf16_tflops_sustained"],
                     "traffic": kernel_traffic(kname, w.name),
                     "flops_per_launch": a["proj_flops"] * tokens_step},
        "pass_roofline": pass_roofline(w, tokens_step, t_step / K / 1e3, tc_peak, peaks["hbm_gbs"]),
        "stages": stages,
        "clocks": clk,
        "gpu_launches": int(launches),
    }
    return result, layer, p, w


def run_e2e(args, layer, p, w, device, world):
    """Same metric through the public API with host buffers: every step copies
    its inputs in from pinned host memory and its y back out, all inside the
    timed region.  As a serving loop would run it, the copies of the next and
    previous steps overlap the current step's forward: a copy-in stream, the
    compute stream and a copy-out stream with two device buffers each."""
    decode = bool(w.decode_calls)
    if decode:
        Bq, Tq = w.B, 1
        ids_h = p.ids[:, :1].contiguous().cpu().pin_memory()
        hid_h = p.hidden[0].view(w.B, 1, w.hc_mult, w.hidden).cpu().pin_memory()
        state = layer.new_state(w.B)
    else:
        Bq, Tq = w.B, w.T
        ids_h = p.ids.cpu().pin_memory()
        hid_h = p.hidden.cpu().pin_memory()
        state = None
    y_h = [torch.empty((Bq, Tq, w.hc_mult, w.hidden), dtype=w.torch_dtype).pin_memory() for _ in range(2)]
    ids_d = [torch.empty_like(ids_h, device=device) for _ in range(2)]
    hid_d = [torch.empty_like(hid_h, device=device) for _ in range(2)]
    y_d = [torch.empty_like(y_h[0], device=device) for _ in range(2)]
    ws = layer.workspace(Bq, Tq)
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    mk = lambda: torch.cuda.Event()
    ev_in, ev_out = [mk(), mk()], [mk(), mk()]
    free_in, free_out = [mk(), mk()], [mk(), mk()]   # buffer b may be refilled / overwritten
    for e in free_in + free_out:
        e.record(comp)

    def step(i):
        b = i & 1
        s_in.wait_event(free_in[b])                   # the forward two steps back is done with it
        with torch.cuda.stream(s_in):
            ids_d[b].copy_(ids_h, non_blocking=True)
            hid_d[b].copy_(hid_h, non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        comp.wait_event(free_out[b])                  # y buffer b has been copied out
        layer.forward(ids_d[b], hid_d[b], y=y_d[b], ws=ws, state=state)
        free_in[b].record(comp)
        ev_out[b].record(comp)
        s_out.wait_event(ev_out[b])
        with torch.cuda.stream(s_out):
            y_h[b].copy_(y_d[b], non_blocking=True)
            free_out[b].record(s_out)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    K = max(3, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0.record(comp)
    s_in.wait_event(e0)
    for i in range(K):
        step(i)
    comp.wait_event(free_out[(K - 1) & 1])        # the last y is on the host
    e1.record(comp)
    torch.cuda.synchronize()
    t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=device)
    ms = max_over_ranks(t, world).item()
    h2d = ids_h.numel() * 8 + hid_h.numel() * hid_h.element_size()
    d2h = y_h[0].numel() * y_h[0].element_size()
    value = job_throughput(world, Bq * Tq, K, ms)
    res = {"value": value, "unit": "tokens/s",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "overlap": "copies of neighbouring steps overlap the forward (3 streams, 2 buffers)"}
    link = host_link_rates(hid_h, hid_d[0], y_h[0], y_d[0], s_in, s_out)
    # with the copies of neighbouring steps overlapped, a step can go no faster
    # than its slower direction at the rates both directions reach together
    bound_s = max(h2d / (link["h2d_concurrent_gbs"] * 1e9), d2h / (link["d2h_concurrent_gbs"] * 1e9))
    link["bound_tokens_per_s"] = world * Bq * Tq / bound_s
    link["frac"] = value / link["bound_tokens_per_s"]
    res["host_link"] = link
    return res


def host_link_rates(src_h, dst_d, dst_h, src_d, s_in, s_out):
    """Pinned host <-> device copy rates with the step's own buffers: each
    direction alone, then both at once on two streams (median of 3, CUDA
    events on the copying streams)."""
    mk = lambda: torch.cuda.Event(enable_timing=True)

    def timed(pairs):
        out = []
        for _ in range(3):
            ev = []
            torch.cuda.synchronize()
            for stream, dst, src in pairs:
                a, b = mk(), mk()
                a.record(stream)
                with torch.cuda.stream(stream):
                    dst.copy_(src, non_blocking=True)
                b.record(stream)
                ev.append((a, b))
            torch.cuda.synchronize()
            out.append([a.elapsed_time(b) for a, b in ev])
        return [sorted(x[i] for x in out)[1] for i in range(len(pairs))]

    nb_in = src_h.numel() * src_h.element_size()
    nb_out = src_d.numel() * src_d.element_size()
    (t_in,) = timed([(s_in, dst_d, src_h)])
    (t_out,) = timed([(s_out, dst_h, src_d)])
    t_in2, t_out2 = timed([(s_in, dst_d, src_h), (s_out, dst_h, src_d)])
    return {"h2d_gbs": nb_in / t_in / 1e6, "d2h_gbs": nb_out / t_out / 1e6,
            "h2d_concurrent_gbs": nb_in / t_in2 / 1e6, "d2h_concurrent_gbs": nb_out / t_out2 / 1e6,
            "bytes": [int(nb_in), int(nb_out)]}


def run_offload(args, layer, p, w, device):
    """Tables resident in pinned host memory (explainer §4.4), prefill
    workloads: the same steps as the headline loop (L2 flushed between steps)
    with (a) the device-resident table, (b) the host-resident table read by
    the forward's gather over the host link, and (c) the pages' hash-ahead
    form: engram_gather_ids for step i+1 on a second stream (host table) while
    engram_forward_gathered runs step i, two row buffers."""
    from hashed_gram_conditional_hash_b200 import EngramLayer
    host_tab = p.table.cpu().pin_memory()
    hl = EngramLayer(orders=w.orders, heads_per_order=w.heads_per_order, row_dim=w.row_dim,
                     hidden=w.hidden, hc_mult=w.hc_mult, conv_kernel=w.conv_kernel,
                     dilation=w.dil, pad_id=w.pad_id, vocab=w.vocab, table=host_tab,
                     row_offsets=p.offsets, primes=p.primes, multipliers=p.mult,
                     w_value=p.w_value, w_key=p.w_key, norm_key=p.norm_key,
                     norm_query=p.norm_query, conv_w=p.conv_w, lookup=p.lookup,
                     rms_eps=w.rms_eps, gate_eps=w.gate_eps)
    B, T = w.B, w.T
    ws = layer.workspace(B, T)
    y = torch.empty((B, T, w.hc_mult, w.hidden), dtype=w.torch_dtype, device=device)
    e = [hl.gather_ids(p.ids) for _ in range(2)]
    flush = L2Flush(device)
    comp = torch.cuda.current_stream()
    side = torch.cuda.Stream(device=device)
    ready, free = [torch.cuda.Event(), torch.cuda.Event()], [torch.cuda.Event(), torch.cuda.Event()]
    for ev in free:
        ev.record(comp)
    K = max(3, min(args.steps, 200))

    def timed(step):
        for i in range(3):
            step(i)
            flush(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        side.wait_event(e0)
        for i in range(K):
            step(i)
            flush(i)
        comp.wait_stream(side)
        e1.record(comp)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K          # ms per step, flushes included

    def flush_ms():
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        for i in range(K):
            flush(i)
        e1.record(comp)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K

    def ahead(i):
        b = i & 1
        # rows of step i + 1 on the side stream (host table) ...
        side.wait_event(free[(i + 1) & 1])
        with torch.cuda.stream(side):
            hl.gather_ids(p.ids, e=e[(i + 1) & 1])
            ready[(i + 1) & 1].record(side)
        # ... while step i runs on rows gathered one step earlier
        if i > 0:                                  # (step 0's rows were gathered before the loop)
            comp.wait_event(ready[b])
        layer.forward_gathered(e[b], p.hidden, y=y, ws=ws)
        free[b].record(comp)

    # two Engram layers' rows of the same ids (own multipliers; the same
    # device table here): one batched launch vs two gathers
    from hashed_gram_conditional_hash_b200 import _lib as L
    l2 = EngramLayer(orders=w.orders, heads_per_order=w.heads_per_order, row_dim=w.row_dim,
                     hidden=w.hidden, hc_mult=w.hc_mult, conv_kernel=w.conv_kernel,
                     dilation=w.dil, pad_id=w.pad_id, vocab=w.vocab, table=p.table,
                     row_offsets=p.offsets, primes=p.primes, multipliers=p.mult[::-1].copy(),
                     w_value=p.w_value, w_key=p.w_key, norm_key=p.norm_key,
                     norm_query=p.norm_query, conv_w=p.conv_w, lookup=p.lookup,
                     rms_eps=w.rms_eps, gate_eps=w.gate_eps)
    e2 = [torch.empty_like(e[0]), torch.empty_like(e[0])]
    t_pair = timed(lambda i: (layer.gather_ids(p.ids, e=e2[0]), l2.gather_ids(p.ids, e=e2[1])))
    t_batched = timed(lambda i: L.engram_gather_ids_layers(layer.cfg, [layer.weights, l2.weights], p.ids, e2))

    f = flush_ms()
    t_dev = timed(lambda i: layer.forward(p.ids, p.hidden, y=y, ws=ws)) - f
    t_host = timed(lambda i: hl.forward(p.ids, p.hidden, y=y, ws=ws)) - f
    t_ahead = timed(ahead) - f
    tok = B * T
    rows_mb = tok * w.nh * w.row_dim * p.table.element_size() / 1e6
    from hashed_gram_conditional_hash_b200 import workloads as W
    return {"table_gb": round(W.table_bytes(w) / 1e9, 3), "rows_per_step_mb": round(rows_mb, 1),
            "device_table_tokens_per_s": tok / (t_dev / 1e3),
            "host_table_tokens_per_s": tok / (t_host / 1e3),
            "host_table_hash_ahead_tokens_per_s": tok / (t_ahead / 1e3),
            "cost_host_table": 1.0 - t_dev / t_host, "cost_hash_ahead": 1.0 - t_dev / t_ahead,
            "two_layer_gather_us": {"separate": (t_pair - f) * 1e3, "one_launch": (t_batched - f) * 1e3},
            "note": "step times exclude the L2 flush between steps; one Engram layer, no other "
                    "layers' compute to hide the host-link transfer behind"}


# Assumed NVLink 5 peer-copy rate per direction per GPU (a figure quoted for
# B200 HGX nodes; no run of this bench has had two GPUs to measure it).
PEER_COPY_GBS = 770.0


def run_sharded(args, layer, p, w, device):
    """The table sharded over R GPUs (explainer §4.4), on ONE GPU: the device
    steps of one rank's gather timed against the plain hash + gather of the
    same ids (L2 flushed between steps).  route = engram_shard_route (3
    kernels); serve = the rows one rank serves per step: every rank asks about
    N/R rows of each shard, so a rank serves about N rows of its shard in one
    launch (timed as the N local rows of this batch served from shard 0, the
    largest, of total/R rows); place = engram_shard_place.  The two
    all-to-alls cannot run on one GPU: their per-rank bytes are reported with
    the time they would take at an assumed peer-copy rate, as an estimate."""
    from hashed_gram_conditional_hash_b200 import _lib as L
    R = args.sharded
    B, T = w.B, w.T
    n = B * T * w.nh
    rb = w.row_dim * p.table.element_size()
    counts = torch.empty(R, dtype=torch.int64, device=device)
    req_rows = torch.empty(n, dtype=torch.int64, device=device)
    req_pos = torch.empty(n, dtype=torch.int32, device=device)
    ws = torch.empty(max(L.engram_shard_route_workspace_size(layer.cfg, B, T, R), 256), dtype=torch.uint8,
                     device=device)
    shard0 = p.table[0::R].contiguous()
    got = torch.empty((n, w.row_dim), dtype=p.table.dtype, device=device)
    e = torch.empty((B * T, w.nh * w.row_dim), dtype=p.table.dtype, device=device)
    L.engram_shard_route(layer.cfg, layer.weights, p.ids, R, counts, req_rows, req_pos, ws)
    flush = L2Flush(device)
    K = max(3, min(args.steps, 200))

    def timed(step):
        for i in range(3):
            step()
            flush(i)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(K):
            ev[i][0].record()
            step()
            ev[i][1].record()
            flush(i)
        torch.cuda.synchronize()
        return sorted(a.elapsed_time(b) * 1e3 for a, b in ev)[K // 2]     # median µs

    t_plain = timed(lambda: layer.gather_ids(p.ids, e=e))
    t_route = timed(lambda: L.engram_shard_route(layer.cfg, layer.weights, p.ids, R, counts, req_rows, req_pos, ws))
    t_serve = timed(lambda: L.engram_shard_serve(layer.cfg, shard0, req_rows, got))
    t_place = timed(lambda: L.engram_shard_place(layer.cfg, got, req_pos, e, n))

    def steps():
        L.engram_shard_route(layer.cfg, layer.weights, p.ids, R, counts, req_rows, req_pos, ws)
        L.engram_shard_serve(layer.cfg, shard0, req_rows, got)
        L.engram_shard_place(layer.cfg, got, req_pos, e, n)
    t_steps = timed(steps)
    remote = n * (R - 1) / R                       # requests of one rank that leave the GPU
    x_bytes = remote * (8 + rb)                    # local row ids out + rows back, per direction
    return {"shards": R, "requests_per_rank": n, "row_bytes": rb,
            "plain_hash_gather_us": t_plain, "route_us": t_route, "serve_us": t_serve, "place_us": t_place,
            "device_steps_us": t_steps,
            "exchange_bytes_per_rank_each_way": int(x_bytes),
            "exchange_us_estimated": x_bytes / (PEER_COPY_GBS * 1e3),
            "note": "one GPU: device steps measured (medians, L2 flushed and drained before each timed "
                    "launch; device_steps_us is the three back to back after one flush); the two "
                    "all-to-alls estimated from their bytes at an assumed %.0f GB/s per "
                    "direction, not measured" % PEER_COPY_GBS}


PROBE_OPS = {"write_v4": 0, "write_v8": 1, "write_v4_cs": 2, "write_bulk": 3, "read_v4": 4, "read_v8": 5,
             "copy_v4": 6, "copy_v8": 7}


def hbm_rates(device, table=None, n_rows=0):
    """HBM write-only, read-only and copy rates on 1 GiB buffers: this
    library's probe kernels (16- and 32-byte stores and loads, evict-first
    stores, bulk-copy-engine stores; libengram_probe.so) beside torch's fill,
    sum and copy; median of 20 launches by CUDA events.  They are the write and
    read sides of the roofline of kernels whose traffic is mostly one way."""
    import ctypes
    n = 1 << 30
    a = torch.empty(n, dtype=torch.uint8, device=device)
    b = torch.empty_like(a)
    out = torch.empty((), dtype=torch.int64, device=device)
    stream = torch.cuda.current_stream()

    def med_ms(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
        for e0, e1 in ev:
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        return sorted(x.elapsed_time(y) for x, y in ev)[10]

    a.fill_(1)
    res = {"bytes": n, "note": "1 GiB buffers, median of 20 launches; copy rates count bytes read + written"}
    res["torch_fill_gbs"] = n / med_ms(lambda: a.fill_(2)) / 1e6
    res["torch_sum_gbs"] = n / med_ms(lambda: torch.sum(a.view(torch.int64), dim=0, out=out)) / 1e6
    res["torch_copy_gbs"] = 2 * n / med_ms(lambda: b.copy_(a)) / 1e6
    from hashed_gram_conditional_hash_b200 import build as Bld
    lib = ctypes.CDLL(Bld.PROBE_LIB)
    lib.engram_probe_hbm.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                     ctypes.c_int, ctypes.c_void_p]
    for name, op in PROBE_OPS.items():
        best = None
        for blocks_per_sm in (2, 4, 8):
            blocks = blocks_per_sm * torch.cuda.get_device_properties(device).multi_processor_count
            if name == "write_bulk":
                blocks *= 4      # 32-thread blocks: one bulk-copy issuer each

            def run():
                rc = lib.engram_probe_hbm(op, b.data_ptr(), a.data_ptr(), n, blocks, stream.cuda_stream)
                if rc != 0:
                    raise RuntimeError("probe %s failed: %d" % (name, rc))
            ms = med_ms(run)
            rate = (2 if name.startswith("copy") else 1) * n / ms / 1e6
            if best is None or rate > best[0]:
                best = (rate, blocks)
        res[name + "_gbs"] = best[0]
        res[name + "_blocks"] = best[1]
    if table is not None and n_rows > 0:
        # random 128-byte rows out of the workload's own table, as many as one
        # step gathers: the access pattern of the hash+gather stage without
        # its hash (read + write bytes over time)
        lib.engram_probe_gather.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_size_t,
                                            ctypes.c_int, ctypes.c_void_p]
        out = torch.empty(n_rows * 128, dtype=torch.uint8, device=device)
        src_bytes = (table.numel() * table.element_size()) // 128 * 128
        best = None
        for blocks_per_sm in (4, 8, 16):
            blocks = blocks_per_sm * torch.cuda.get_device_properties(device).multi_processor_count

            def run():
                rc = lib.engram_probe_gather(out.data_ptr(), table.data_ptr(), out.numel(), src_bytes, blocks,
                                             stream.cuda_stream)
                if rc != 0:
                    raise RuntimeError("gather probe failed: %d" % rc)
            ms = med_ms(run)
            rate = 2 * out.numel() / ms / 1e6
            if best is None or rate > best[0]:
                best = (rate, blocks)
        res["gather_random_rows_gbs"], res["gather_random_rows_blocks"] = best
        res["gather_random_rows"] = {"rows": int(n_rows), "table_bytes": int(src_bytes)}
        del out
    # fp32 multiply-add rate, packed pairs against scalar (16 independent chains
    # per thread, 8 blocks of 256 per SM)
    lib.engram_probe_fma.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    fblocks = 8 * torch.cuda.get_device_properties(device).multi_processor_count
    fout = torch.empty(fblocks * 256, dtype=torch.float32, device=device)
    iters = 4096
    for name, packed in (("fma_packed_tflops", 1), ("fma_scalar_tflops", 0)):
        def run():
            rc = lib.engram_probe_fma(packed, fout.data_ptr(), fblocks, iters, stream.cuda_stream)
            if rc != 0:
                raise RuntimeError("fma probe failed: %d" % rc)
        res[name] = 2.0 * 16 * iters * fblocks * 256 / med_ms(run) / 1e9
    del fout
    res["write_only_gbs"] = max(res[k + "_gbs"] for k in ("write_v4", "write_v8", "write_v4_cs", "write_bulk"))
    res["read_only_gbs"] = max(res["read_v4_gbs"], res["read_v8_gbs"])
    res["copy_gbs"] = max(res["copy_v4_gbs"], res["copy_v8_gbs"])
    return res


def gemm_ref(args, w, device):
    """cuBLAS (torch.matmul) on the projection's own GEMM shape, without its
    epilogue: e [M, E] times the stacked value and key weights [E, H (1 + hc)],
    bf16 in, fp32 accumulate, bf16 out.  Same L2 protocol as the timed steps
    (flush and drain between launches); median of the launches by CUDA events.
    It is the practical tensor-core rate for this shape on this GPU, beside
    which the fused projection's rate can be read."""
    M = w.B * (1 if w.decode_calls else w.T)
    E = w.E
    N = w.hidden * (1 + w.hc_mult)
    g = torch.Generator(device=device).manual_seed(7)
    a = (torch.randn(M, E, device=device, generator=g) * 0.5).to(torch.bfloat16)
    b = (torch.randn(N, E, device=device, generator=g) * (E ** -0.5)).to(torch.bfloat16)
    c = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    flush = L2Flush(device)
    n = max(5, min(args.steps, 50))
    for i in range(3):
        torch.matmul(a, b.t(), out=c)
        flush(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i, (e0, e1) in enumerate(ev):
        e0.record()
        torch.matmul(a, b.t(), out=c)
        e1.record()
        flush(i)
    torch.cuda.synchronize()
    ms = sorted(x.elapsed_time(y) for x, y in ev)[n // 2]
    flops = 2.0 * M * E * N
    del a, b, c
    return {"M": M, "K": E, "N": N, "launches": n, "median_us": ms * 1e3,
            "tflops": flops / (ms / 1e3) / 1e12,
            "note": "torch.matmul (cuBLAS) bf16, no epilogue, L2 flushed between launches"}


def run_reference(args):
    """The reference arm: the float64 oracle on the host cores, K timed steps
    of a bounded sample each, sized so that warm-up + steps take ~2 minutes."""
    from hashed_gram_conditional_hash_b200 import workloads as W
    w = W.CONFIGS[args.config]
    nthreads = os.cpu_count() or 1
    per_step = min(args.ref_step_s, 120.0 / max(1, args.steps + args.warmup))
    # tables above 1 GiB are drawn on the GPU (plumbing only: the oracle runs
    # on the host cores and receives the table rows its sample needs)
    p = W.make_params(w, "cuda") if W.gen_device_for(w, "cuda") != "cpu" else None
    n, run = oracle_sample(w, oracle_tokens_for(w, per_step, nthreads, p), nthreads, p)
    for _ in range(args.warmup):
        run()
    tot = 0.0
    for _ in range(args.steps):
        tot += run()
    rate = n * args.steps / tot
    sample = ("per step: %d positions (whole sequences) of a workload with the shapes and "
              "distributions of %s, whole pass from ids, float64 oracle" % (n, w.name))
    return {
        "impl": "reference",
        "metric": "Engram forward tokens/s on 1xB200 (engram_forward); % of HBM and bf16 tensor roofline",
        "value": rate, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "B": w.B, "T": w.T if not w.decode_calls else 1},
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="hbm_table_bf16")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--ref-step-s", type=float, default=3.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--debug-flags", type=lambda x: int(x, 0), default=0,
                    help="library comparison knobs (ENGRAM_DEBUG_* of engram.h), e.g. 0x40")
    ap.add_argument("--overlap-chunks", type=int, default=0,
                    help="prefill in this many sequence chunks whose gate and conv overlap the next "
                         "chunk's projection (0: the library default)")
    ap.add_argument("--decode-calls", type=int, default=0,
                    help="decode workload: number of distinct calls drawn (default: all 256)")
    ap.add_argument("--offload", action="store_true",
                    help="also measure tables resident in pinned host memory (prefill workloads)")
    ap.add_argument("--hbm-rates", action="store_true",
                    help="also measure HBM write-only, read-only and copy rates (1 GiB torch kernels)")
    ap.add_argument("--gemm-ref", action="store_true",
                    help="also time cuBLAS on the projection's GEMM shape (no epilogue), for context")
    ap.add_argument("--sharded", type=int, default=0,
                    help="also time the device steps of a gather from a table sharded over this many GPUs")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    torch.cuda.set_device(local)
    device = "cuda:%d" % local
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device(device))
    try:
        res, layer, p, w = run_ours(args, rank, world, device)
        if not args.no_e2e:
            res["e2e"] = run_e2e(args, layer, p, w, device, world)
        if args.offload and not w.decode_calls:
            res["offload"] = run_offload(args, layer, p, w, device)
        if args.hbm_rates:
            tab = p.table if (p.table is not None and p.table.is_cuda and w.row_dim * p.table.element_size() == 128) else None
            res["hbm_rates"] = hbm_rates(device, tab, w.M * w.nh)
        if args.gemm_ref:
            res["gemm_ref"] = gemm_ref(args, w, device)
            res["gemm_ref"]["projection_over_cublas"] = \
                res["roofline"]["achieved"] / res["gemm_ref"]["tflops"]
        if args.sharded and not w.decode_calls:
            res["sharded"] = run_sharded(args, layer, p, w, device)
        from hashed_gram_conditional_hash_b200 import workloads as W
        # device-drawn tables are kept for the oracle's sample (it fetches its rows)
        keep = p if W.gen_device_for(w, device) != "cpu" else None
        del layer, p
        torch.cuda.empty_cache()
        if rank == 0 and not args.no_cpu_baseline and world == 1:
            res["cpu_baseline"] = cpu_baseline(w, args.cpu_budget_s, keep)
        del keep
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
