#!/usr/bin/env python
"""Benchmark of the decode/verify-step megakernel on synthetic workloads.

`python bench.py [--gpus N --steps K --warmup W --workload large]` runs one
full step (every layer of the QK-normed MoE stack) per timed iteration on
each GPU -- independent replicas under torchrun, no collective on the data
path -- and prints one JSON line.  The metric is the step's algorithmic HBM
bytes (distinct dense + expert weights + KV read/written + hidden in/out)
divided by the device-timed step time, summed over ranks; the line also
carries the step time, tokens/s, the fraction of the 8 TB/s and measured
copy bandwidth, step time / stream time, the end-to-end number through the
C ABI with host buffers, the roofline object, clocks, and (rank 0, N = 1)
the fp64 oracle timed on a bounded sample of the same workload.

`--impl reference` times the oracle alone (the CPU reference arm).
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE step µs, HBM GB/s vs 8 TB/s peak, step time ÷ weight+KV stream time"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_hash():
    h = hashlib.sha256()
    for name in ("msk_kernel.cu", "msk_device.cuh", "msk_internal.h"):
        with open(os.path.join(ROOT, "verify_step_megakernel_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else null)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t.get(workload)
        if e and e.get("kernel_hash") == kernel_hash():
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def workload_config(w):
    return {"workload": w.name, "layers": w.n_layers, "d_model": w.d_model, "q_heads": w.n_q_heads,
            "kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "experts": f"top{w.top_k} of {w.n_experts}",
            "expert_dim": w.expert_dim, "sliding_layers": sum(w.sliding), "window": w.window,
            "seqs": w.n_seqs, "tokens_per_seq": w.tokens_per_seq, "past_tokens": w.past,
            "weights": "NVFP4 (e2m1 + e4m3/16 + fp32 global)", "kv": "fp8 e4m3"}


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.path = tempfile.mktemp(suffix=".csv")
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9:
                try:
                    rows.append((float(p[1]), float(p[2]), p[5], p[6], p[7], p[8]))
                except ValueError:
                    pass
        os.unlink(self.path)
        if not rows:
            return None
        top = max(r[0] for r in rows)
        loaded = [r for r in rows if r[0] >= 0.5 * top] or rows
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in loaded:
            for n, v in zip(names, r[2:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": loaded[0][1],
                "reasons": sorted(reasons), "samples": len(loaded)}


def cpu_sample(w, threads=None, seq=0, n_layers=None, warm=True):
    """Time the oracle on one sequence of the workload (all its tokens), on
    its first n_layers layers (default all).  Returns (seconds, algorithmic
    bytes of the sample, threads).  warm: run once untimed first, so the
    timed call does not include generating the inputs."""
    import oracle
    import synth
    one = w.with_(n_seqs=1)
    if n_layers is not None and n_layers < w.n_layers:
        one = one.with_(n_layers=n_layers, sliding=list(w.sliding[:n_layers]))
    src = _oracle_source(one)
    hid = synth.host_hidden(w, 1, w.tokens_per_seq, seq0=seq)
    pos = [w.positions()[seq]]
    nt = threads or min(64, os.cpu_count() or 1)
    if warm:
        oracle.step(one, src.ptr, hid, pos, seq_ids=[seq], threads=nt)  # generates the inputs it needs
    t0 = time.perf_counter()
    ref = oracle.step(one, src.ptr, hid, pos, seq_ids=[seq], threads=nt)
    dt = time.perf_counter() - t0
    return dt, sample_bytes(one, ref["n_distinct"], 1), nt


_SOURCES = {}


def _oracle_source(w):
    """One lazily generated input source per workload shape, kept for the run
    (the generator caches what it has produced)."""
    import synth
    key = (w.name, w.n_layers)
    if key not in _SOURCES:
        _SOURCES[key] = synth.LazySource(w)
    return _SOURCES[key]


def sample_bytes(w, n_distinct, n_seqs):
    """Algorithmic bytes of n_seqs sequences of the workload given the
    distinct experts per layer (same definition as msk_query)."""
    nvb = lambda n: n // 2 + n // 16
    d, qd, kvd, f = w.d_model, w.n_q_heads * w.head_dim, w.n_kv_heads * w.head_dim, w.expert_dim
    T = n_seqs * w.tokens_per_seq
    b = 0
    for l in range(w.n_layers):
        b += nvb(qd * d) + 2 * nvb(kvd * d) + nvb(d * qd) + w.n_experts * d * 4
        b += int(n_distinct[l]) * 3 * nvb(d * f)
        lo = max(0, w.past - w.window + 1) if w.sliding[l] else 0
        b += n_seqs * w.n_kv_heads * (w.past + w.tokens_per_seq - lo) * 2 * w.head_dim
        b += T * 2 * kvd
    return b + T * d * 2 * 2


def run_reference(args, w):
    """The reference arm: the fp64 oracle, as it stands, on the host cores.
    Each step is a bounded sample of the workload -- one sequence, all its
    tokens, the first REF_LAYERS layers (one period of the sliding/full
    pattern of the largest workload) -- so the whole run ends in minutes."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    nl = min(w.n_layers, REF_LAYERS)
    sample = (f"fp64 oracle on 1 of {w.n_seqs} sequences x {w.tokens_per_seq} tokens, the first {nl} of "
              f"{w.n_layers} layers, per step")
    times, byts, nt = [], 0, 1
    cpu_sample(w, threads=args.cpu_threads, n_layers=nl)  # input generation, untimed
    for i in range(args.warmup + args.steps):
        dt, byts, nt = cpu_sample(w, threads=args.cpu_threads, n_layers=nl, warm=False)
        if i >= args.warmup:
            times.append(dt)
    t = statistics.mean(times)
    val = byts / t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": nt, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


REF_LAYERS = 4


def max_over_ranks(value, device="cpu"):
    """The largest of each rank's `value` (a float) over the default process
    group; the value itself when there is no group or one rank.  Every rank
    must call it, in the same order."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, units_per_rank, ms_max):
    """Whole-job throughput: the units all ranks processed per second, over
    the slowest rank's step time (replicas: each rank processes the same
    units per step)."""
    return world * units_per_rank / (ms_max * 1e-3)


def run_msk(args, w):
    import numpy as np
    import torch
    import torch.distributed as dist

    import synth.gpu as sg
    import verify_step_megakernel_b200 as msk
    from synth.engine import Engine

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    def barrier():
        if world > 1:
            dist.barrier()

    t_setup = time.perf_counter()
    eng = Engine(w, device=local, flags=msk.F_TC_EXPERTS if args.tc_experts else 0, tau=args.tau)
    eng.fill_past()
    hid = sg.hidden(w, local)
    pos = torch.tensor(w.positions(), dtype=torch.int32, device=dev)
    out = torch.empty((w.T, w.d_model), dtype=torch.int16, device=dev)
    stream = torch.cuda.Stream(dev)
    sptr = stream.cuda_stream
    msk.msk_set_debug(eng.h)
    setup_s = time.perf_counter() - t_setup

    def launch():
        msk.msk_step(eng.h, hid.data_ptr(), pos.data_ptr(), w.n_seqs, w.tokens_per_seq, eng.kv, out.data_ptr(), sptr)

    flush = None
    stats_probe = None
    if args.trace:
        return trace_step(args, w, eng, launch, stream, dev, rank)
    for _ in range(args.warmup):
        launch()
    stream.synchronize()
    st = msk.msk_step_status(eng.h)
    if st != 0:
        raise RuntimeError(f"warm-up step failed: {msk.STATUS.get(st)}")
    stats_probe = msk.msk_query(eng.h)
    bytes_step = int(stats_probe.algorithmic_bytes)
    l2_note = "inputs larger than L2 (%.1f GB per step), no flush" % (bytes_step / 1e9)
    if bytes_step < 4 * 126e6:
        flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        l2_note = "L2 flushed between timed steps (512 MB write)"

    uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    clocks = ClockSampler(uuid)
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            launch()
            ev[i][1].record(stream)
        t1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    st = msk.msk_step_status(eng.h)
    if st != 0:
        raise RuntimeError(f"timed step failed: {msk.STATUS.get(st)}")
    per = [a.elapsed_time(b) for a, b in ev]
    ms = statistics.mean(per)
    total_ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, dev)

    # end to end through the C ABI: pinned host input -> device, step, output -> host
    h_in_host = hid.cpu().pin_memory()
    pos_host = pos.cpu().pin_memory()
    out_host = torch.empty_like(out, device="cpu").pin_memory()
    hid_dev = torch.empty_like(hid)
    pos_dev = torch.empty_like(pos)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(args.steps):
            hid_dev.copy_(h_in_host, non_blocking=True)
            pos_dev.copy_(pos_host, non_blocking=True)
            msk.msk_step(eng.h, hid_dev.data_ptr(), pos_dev.data_ptr(), w.n_seqs, w.tokens_per_seq, eng.kv,
                         out.data_ptr(), sptr)
            out_host.copy_(out, non_blocking=True)
        e1.record(stream)
    stream.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_step_ms = max_over_ranks(e2e_ms / args.steps, dev)
    if msk.msk_step_status(eng.h) != 0:
        raise RuntimeError("e2e step failed")

    peak, peak_kind = measured_peak()
    achieved = bytes_step / (ms * 1e-3) / 1e9  # this rank's kernel, GB/s
    value = job_rate(world, bytes_step, ms_max) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 x f16 -> fp32 (NVFP4/fp8 storage)", "data": "synthetic",
        "config": dict(workload_config(w), parallelism=f"{world} independent replicas", l2=l2_note),
        "step_us": round(ms_max * 1e3, 2),
        "tokens_per_s": round(job_rate(world, w.T, ms_max), 1),
        "hbm_gbs_per_gpu": round(achieved, 1),
        "frac_of_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
        "step_over_stream_time": round((ms * 1e-3) / (bytes_step / (NOMINAL_HBM_GBS * 1e9)), 3),
        "algorithmic_bytes_per_step": bytes_step,
        "distinct_experts_per_layer": list(stats_probe.n_distinct[:w.n_layers]),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} copy bandwidth",
                     "traffic": ncu_traffic(w.name)},
        "e2e": {"value": round(job_rate(world, bytes_step, e2e_step_ms) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(hid.numel() * 2 + pos.numel() * 4),
                "d2h_bytes_per_step": int(out.numel() * 2), "ms_per_step": round(e2e_step_ms, 4)},
        "gpu_launches": world * args.steps,
        "timed_region_ms": round(total_ms, 3),
        "setup_s": round(setup_s, 1),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, sb, nt = cpu_sample(w, threads=args.cpu_threads)
        # one core, on the first layer of the same sequence (a bounded sample)
        dt1, sb1, _ = cpu_sample(w, threads=1, n_layers=1)
        line["cpu_baseline"] = {"value": round(sb / dt / 1e9, 4), "unit": "GB/s", "cores": nt, "kind": "oracle",
                                "sample": f"fp64 oracle on 1 of {w.n_seqs} sequences x {w.tokens_per_seq} tokens, "
                                          f"all {w.n_layers} layers ({sb / 1e9:.2f} GB algorithmic, {dt:.1f} s)",
                                "single_core": {"value": round(sb1 / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                                                "sample": f"the same sequence, first layer only "
                                                          f"({sb1 / 1e9:.3f} GB algorithmic, {dt1:.1f} s)"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    eng.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_sweep(args, w):
    """Step time of the workload's model over a range of batch shapes (S
    sequences x Tq draft tokens, S*Tq <= 64): one JSON line per shape, timed
    like the main line (warm-up, CUDA events per step, L2 flushed when the
    step's bytes would fit in it).  One handle serves all shapes with the
    same token limit per sequence; Tq = 8 needs a second one (at most 8
    sequences), built after the first is released."""
    import torch

    import synth.gpu as sg
    import verify_step_megakernel_b200 as msk
    from synth.engine import Engine

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    groups = [(4, [(1, 1), (2, 1), (4, 1), (8, 1), (16, 1), (1, 4), (4, 4), (16, 4)]), (8, [(1, 8), (4, 8), (8, 8)])]
    for tps, shapes in groups:
        max_s = min(64 // tps, max(s for s, _ in shapes))
        eng = Engine(w.with_(n_seqs=max_s, tokens_per_seq=tps), device=0)
        eng.fill_past()
        stream = torch.cuda.Stream(dev)
        msk.msk_set_debug(eng.h)
        for S, Tq in shapes:
            ws = w.with_(n_seqs=S, tokens_per_seq=Tq)
            hid = sg.hidden(ws, 0)
            pos = torch.tensor(ws.positions(), dtype=torch.int32, device=dev)
            out = torch.empty((ws.T, ws.d_model), dtype=torch.int16, device=dev)

            def launch():
                msk.msk_step(eng.h, hid.data_ptr(), pos.data_ptr(), S, Tq, eng.kv, out.data_ptr(),
                             stream.cuda_stream)

            for _ in range(args.warmup):
                launch()
            stream.synchronize()
            if msk.msk_step_status(eng.h) != 0:
                raise RuntimeError(f"sweep step {S}x{Tq} failed")
            stats = msk.msk_query(eng.h)
            nbytes = int(stats.algorithmic_bytes)
            flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if nbytes < 4 * 126e6 else None
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            torch.cuda.synchronize(dev)
            with torch.cuda.stream(stream):
                for i in range(args.steps):
                    if flush is not None:
                        flush.fill_(i & 0xFF)
                    ev[i][0].record(stream)
                    launch()
                    ev[i][1].record(stream)
            stream.synchronize()
            if msk.msk_step_status(eng.h) != 0:
                raise RuntimeError(f"sweep step {S}x{Tq} failed")
            ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
            nd = list(stats.n_distinct[:w.n_layers])
            print(json.dumps({"sweep": w.name, "n_seqs": S, "tokens_per_seq": Tq, "T": S * Tq,
                              "step_us": round(ms * 1e3, 1), "tokens_per_s": round(S * Tq / (ms * 1e-3), 1),
                              "algorithmic_bytes_per_step": nbytes, "hbm_gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                              "frac_of_measured": round(nbytes / (ms * 1e-3) / 1e9 / measured_peak()[0], 4),
                              "distinct_experts_per_layer_mean": round(sum(nd) / len(nd), 1),
                              "l2": "flushed" if flush is not None else "inputs larger than L2"}), flush=True)
            del flush
        eng.close()
        del eng
        torch.cuda.empty_cache()
    return 0


PHASES = ["in", "qkv", "qknorm", "attention", "attn_combine", "wo", "moe_norm", "router", "topk", "gate_up",
          "down", "combine"]


def trace_step(args, w, eng, launch, stream, dev, rank):
    """Per-phase device time of one step: %globaltimer stamps taken by CTA 0
    when it leaves each grid barrier (all CTAs have finished the phase)."""
    import torch
    import verify_step_megakernel_b200 as msk
    for _ in range(args.warmup):
        launch()
    trace = torch.zeros((w.n_layers, 16), dtype=torch.int64, device=dev)
    msk.msk_set_debug(eng.h, trace=trace.data_ptr())
    launch()
    stream.synchronize()
    msk.msk_set_debug(eng.h)
    distinct = list(msk.msk_query(eng.h).n_distinct[:w.n_layers])
    t = trace.cpu().numpy()
    order = [(0, 0)] + [(l, p) for l in range(w.n_layers) for p in (1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11)
                        if not (l == w.n_layers - 1 and p == 11)]
    # a phase folded into another (the attention combine at head dim 128) leaves no stamp
    order = [(l, p) for (l, p) in order if t[l, p] != 0]
    out = {PHASES[p]: 0.0 for p in range(len(PHASES))}
    prev = None
    for (l, p) in order:
        if prev is not None:
            out[PHASES[p]] += (t[l, p] - prev) / 1e3
        prev = t[l, p]
    total = (t[order[-1]] - t[0, 0]) / 1e3
    if rank == 0:
        print(json.dumps({"trace_us": {k: round(v, 1) for k, v in out.items()}, "total_us_after_in": round(total, 1),
                          "distinct_experts_per_layer": distinct,
                          "note": "each phase ends at its grid barrier; top-k ends when CTA 0 has its routing (no barrier), so gate_up starts there; down includes the encoding of the SwiGLU rows as e2m1 terms"}))
    eng.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="msk", choices=["msk", "reference"])
    ap.add_argument("--workload", default="large")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-threads", type=int, default=0)
    ap.add_argument("--trace", action="store_true", help="print a per-phase device-time breakdown instead")
    ap.add_argument("--tc-experts", action="store_true",
                    help="gate/up on the block-scaled tensor cores (MSK_F_TC_EXPERTS) instead of the default path")
    ap.add_argument("--tau", type=int, default=0,
                    help="expert_mma_min_tokens: units with at least this many tokens take the block-scaled path "
                         "(0 = never)")
    ap.add_argument("--sweep", action="store_true",
                    help="step time of the workload's model over batch shapes (one JSON line per shape)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    import synth
    w = synth.WORKLOADS.get(args.workload) or synth.PROFILE_WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.sweep:
        return run_sweep(args, w)
    return run_msk(args, w)


if __name__ == "__main__":
    sys.exit(main())
