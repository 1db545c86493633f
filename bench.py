#!/usr/bin/env python3
"""Benchmark of one MLA decode layer step over a paged latent KV cache.

A step is one pass of the whole path on one batch: append the new token of
every sequence, absorb the queries, split-KV decode, merge the splits, output
projection -- four C-ABI calls into libmla (the split merge runs inside the
output projection's first kernel).  Default workload: the
DeepSeek-V2-shaped decode, batch 32, context 2048, bf16 paged cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...     (N > 1; data parallel)

Prints ONE JSON line on rank 0.  ``value`` is decode tokens/s of the whole
job (all ranks), from CUDA-event times of the steps with inputs resident in
HBM; L2 is flushed before every step, outside the step's events.  ``e2e`` is
the same metric through the public API with host<->device copies inside the
timed region.  ``--impl reference`` times the fp64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode latent-cache GB/s & TFLOP/s vs B200 roofline; decode tokens/s"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "v2_b32_l2048"
WORKLOAD_TEXT = {
    "v2_b32_l2048": "DeepSeek-V2-shape single-layer decode: batch 32, context 2048 each, H=128, "
                    "d_model=5120, d_c=512, d_r=64, d_nope=d_v=128, bf16 paged cache (block 64), "
                    "fp32 accumulation",
    "v2_ragged64": "V2 dims, 64 sequences with history uniform in [1,8192], shuffled pages, "
                   "append at position len then decode",
    "v2_b4_l32k": "V2 dims, batch 4, context 32768, bf16 cache",
    "v2_b2_l128k_fp8": "V2 dims, batch 2, context 131072, e4m3 cache with per-token fp32 scale",
}
STAGES = ("append", "absorb", "decode_partial", "combine_out_proj")   # DecodeStep.stages()
# the sources that define each tensor-core stage's kernel (its device code, the
# PTX wrappers it uses and its launcher): a traffic figure taken by ncu is only
# reported while all of them are unchanged
KERNEL_FILES = {
    "decode_partial": ["mla_latent_kv_19_b200/csrc/decode_umma.cuh",
                       "mla_latent_kv_19_b200/csrc/sm100_ptx.cuh",
                       "mla_latent_kv_19_b200/csrc/umma_kernels.cu"],
    "combine_out_proj": ["mla_latent_kv_19_b200/csrc/gemm_umma.cuh",
                         "mla_latent_kv_19_b200/csrc/sm100_ptx.cuh",
                         "mla_latent_kv_19_b200/csrc/umma_kernels.cu"],
    "out_proj": ["mla_latent_kv_19_b200/csrc/gemm_umma.cuh",
                 "mla_latent_kv_19_b200/csrc/sm100_ptx.cuh",
                 "mla_latent_kv_19_b200/csrc/umma_kernels.cu"],
    "absorb": ["mla_latent_kv_19_b200/csrc/gemm_umma.cuh",
               "mla_latent_kv_19_b200/csrc/sm100_ptx.cuh",
               "mla_latent_kv_19_b200/csrc/umma_kernels.cu"],
}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def algorithmic(wl, S):
    """Algorithmic bytes and flops per launch of each stage (each byte the
    method must touch, once; implementation scratch not counted)."""
    d = wl.dims
    B, H, dc, dr, dn, dv, dm = wl.batch, d["num_heads"], d["d_c"], d["d_r"], d["d_nope"], d["d_v"], d["d_model"]
    D = dc + dr
    a = 4 if wl.act_dtype == "fp32" else 2
    row = D * (1 if wl.cache_dtype == "fp8_e4m3" else a) + (4 if wl.cache_dtype == "fp8_e4m3" else 0)
    tokens = int(wl.seq_lens.sum())
    out = {
        "append": dict(bytes=B * D * a + B * row, flops=0),
        "absorb": dict(bytes=H * dn * dc * a + B * H * (dn + dr) * a + B * H * D * a,
                       flops=2 * B * H * dn * dc),
        "decode_partial": dict(bytes=tokens * row + B * H * D * a + B * H * dc * a,
                               flops=2 * H * (D + dc) * tokens),
        # merge + output projection: the weights, o_lat and lse written, y written
        # (the split partials it reads are the decode's scratch, not counted)
        "combine_out_proj": dict(bytes=H * dv * dc * a + dm * H * dv * a + B * H * dc * a + B * H * 4 + B * dm * a,
                                 flops=2 * B * H * dv * dc + 2 * B * dm * H * dv),
    }
    return out, tokens


def source_hash(stage):
    h = hashlib.sha256()
    for f in KERNEL_FILES.get(stage, []):
        p = os.path.join(ROOT, f)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(stage, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of that kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{stage}:{workload}")
    if not d or d.get("source_hash") != source_hash(stage):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"mla_bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), active=parts[4],
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return None
        smax = max(r["smax"] for r in rows)
        loaded = [r for r in rows if r["sm"] > 0.5 * smax] or rows
        reasons = set()
        for r in rows:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                            ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[k].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r["sm"] for r in loaded])), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(rows)}


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(wl, seconds=12.0, max_seqs=None):
    """The fp64 oracle as it stands, on whole sequences of the workload until
    about ``seconds`` of CPU work; returns (tokens/s, sequences, seconds)."""
    import oracle
    n, t0 = 0, time.perf_counter()
    seqs = list(range(wl.batch))
    while True:
        b = seqs[n % len(seqs)]
        oracle.step_outputs(wl, [b])
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_seqs and n >= max_seqs):
            return n / el, n, el


def reference_arm(args, rank, world):
    """The oracle timed on the host cores, rank 0 only."""
    if rank != 0:
        return
    import workloads
    wl = workloads.make(args.workload)
    per = []
    for _ in range(args.warmup):
        time_oracle(wl, seconds=0.0, max_seqs=1)
    for _ in range(args.steps):
        v, n, el = time_oracle(wl, seconds=args.ref_seconds)
        per.append(el / n)
    sec_per_seq = float(np.mean(per))
    value = 1.0 / sec_per_seq
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec_per_seq * wl.batch * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": f"{args.workload}: {WORKLOAD_TEXT.get(args.workload, '')}"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"whole sequences of the workload (absorbed fp64 form: absorb, "
                                   f"decode, output projection), ~{args.ref_seconds:.0f} s per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--overlap", action="store_true",
                    help="launch each kernel as a programmatic dependent of the one before it")
    ap.add_argument("--ref-seconds", type=float, default=10.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    import torch
    from mla_latent_kv_19_b200 import dist

    if args.impl == "reference":
        rank, _, world = dist.env_world()
        reference_arm(args, rank, world)
        return

    rank, local, world = dist.init("nccl")
    import workloads
    from mla_latent_kv_19_b200 import mla_launch_count
    from mla_latent_kv_19_b200.step import DecodeStep, to_device

    base_seed = {"v2_b32_l2048": 1, "v2_ragged64": 2, "v2_b4_l32k": 3, "v2_b2_l128k_fp8": 4}.get(args.workload, 1)
    wl = workloads.make(args.workload, seed=dist.rank_seed(base_seed, rank))
    dev = torch.device("cuda", local)
    st = DecodeStep(wl, device=dev, num_splits=args.num_splits, overlap=args.overlap)
    stream = torch.cuda.current_stream(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    flush_sum = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2():
        # write a buffer of twice the L2 size, then read it back: the read evicts
        # the dirty lines the write left (their write-back happens here, not in
        # the next step) and leaves L2 holding clean lines no step uses
        flush.zero_()
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)

    # one eager step configures the kernels and counts this library's launches per
    # step.  Each timed step replays ONE CUDA graph of the whole step with timing
    # events at its two ends only (an event between two kernels would end the
    # overlap of the second's launch with the first); the per-stage breakdown
    # comes from a second graph of the same step with events between the stages,
    # replayed after it (with its own L2 flush)
    l0 = mla_launch_count()
    st.run(stream)
    torch.cuda.synchronize(dev)
    launches_per_step = mla_launch_count() - l0
    st.capture()
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    timed = torch.cuda.CUDAGraph()
    with torch.cuda.graph(timed):
        ev[0].record()
        st.run()
        ev[1].record()
    sev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(STAGES) + 1)]
    staged = torch.cuda.CUDAGraph()
    with torch.cuda.graph(staged):
        sev[0].record()
        for i, (_, fn) in enumerate(st.stages()):
            fn()
            sev[i + 1].record()
    torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        flush_l2()
        timed.replay()
        flush_l2()
        staged.replay()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    step_ms, stage_rows = [], []
    for k in range(args.steps):
        flush_l2()                         # L2 flush, outside the step's events
        timed.replay()
        torch.cuda.synchronize(dev)        # read this replay's events before the next one
        step_ms.append(ev[0].elapsed_time(ev[1]))
        flush_l2()
        staged.replay()
        torch.cuda.synchronize(dev)
        stage_rows.append([sev[i].elapsed_time(sev[i + 1]) for i in range(len(STAGES))])
    torch.cuda.synchronize(dev)
    dist.barrier()
    launches = launches_per_step * args.steps
    clk = clocks.stop()

    step_ms = np.array(step_ms)
    stage_ms = {s: float(np.mean([row[i] for row in stage_rows])) for i, s in enumerate(STAGES)}
    ms = float(np.mean(step_ms))
    ms_max = dist.max_over_ranks(ms)
    total_seqs = dist.sum_over_ranks(wl.batch)
    value = total_seqs / (ms_max / 1e3)

    # end to end through the public API: H2D of the step's inputs from pinned
    # memory, the step, D2H of the result, synchronised, wall clock
    host_in = {"q_nope": to_device(wl.q_nope, "cpu", pin=True), "q_pe": to_device(wl.q_pe, "cpu", pin=True),
               "new_pos": to_device(wl.new_pos.astype(np.int32), "cpu", pin=True)}
    if st.tiny:
        host_in["new_x"] = to_device(wl.new_x, "cpu", pin=True)
    else:
        host_in["new_c_kv"] = to_device(wl.new_c_kv, "cpu", pin=True)
        host_in["new_k_r"] = to_device(wl.new_k_r, "cpu", pin=True)
    y_host = torch.empty(st.y.shape, dtype=st.y.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = y_host.numel() * y_host.element_size()
    def e2e_calls():
        for name, t in host_in.items():
            getattr(st, name).copy_(t, non_blocking=True)
        st.run()
        y_host.copy_(st.y, non_blocking=True)

    # the copies and the step's calls in one CUDA graph (copies from and to pinned
    # host memory are graph nodes): one launch per step; if the capture is
    # refused, the copies are issued one by one around the step graph
    e2e_graph, e2e_mode = torch.cuda.CUDAGraph(), "one graph: H2D copies, the step, D2H copy"
    try:
        with torch.cuda.graph(e2e_graph):
            e2e_calls()
        torch.cuda.synchronize(dev)
    except RuntimeError:
        torch.cuda.synchronize(dev)
        e2e_graph, e2e_mode = None, "H2D copies, step graph replay, D2H copy, issued one by one"
    e2e_times = []
    for k in range(args.warmup + args.steps):
        flush_l2()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        if e2e_graph is not None:
            e2e_graph.replay()
        else:
            for name, t in host_in.items():
                getattr(st, name).copy_(t, non_blocking=True)
            st.replay()
            y_host.copy_(st.y, non_blocking=True)
        torch.cuda.synchronize(dev)
        if k >= args.warmup:
            e2e_times.append(time.perf_counter() - t0)
    e2e_s = dist.max_over_ranks(float(np.mean(e2e_times)))
    e2e_value = total_seqs / e2e_s

    alg, tokens = algorithmic(wl, st.num_splits)
    hbm, bf16, bf16_sus, peak_kind = measured_peaks()
    # the dominant kernel: the split-KV decode is the step's longest single
    # kernel (the other stages hold several kernels each; the committed launch
    # list has the per-kernel times)
    dom = "decode_partial"
    kernels = {}
    for s in STAGES:
        t = stage_ms[s] / 1e3
        kernels[s] = {"us": stage_ms[s] * 1e3, "GB/s": alg[s]["bytes"] / t / 1e9,
                      "TFLOP/s": alg[s]["flops"] / t / 1e12,
                      "hbm_frac": alg[s]["bytes"] / t / 1e9 / hbm}
    t_dom = stage_ms[dom] / 1e3
    roof = {"kernel": dom, "bound": "hbm", "achieved": alg[dom]["bytes"] / t_dom / 1e9, "peak": hbm,
            "unit": "GB/s", "frac": alg[dom]["bytes"] / t_dom / 1e9 / hbm,
            "traffic": ncu_traffic(dom, args.workload),
            "algorithmic_bytes_per_launch": alg[dom]["bytes"],
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback"}
    t_dec = stage_ms["decode_partial"] / 1e3
    dec = alg["decode_partial"]
    decode_roof_s = max(dec["bytes"] / (hbm * 1e9), dec["flops"] / (bf16 * 1e12))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.act_dtype == "bf16" else "fp32",
        "data": "synthetic (seeded: latents/queries N(0,1), weights N(0,1/sqrt(fan_in)))",
        "config": {"workload": f"{args.workload}: {WORKLOAD_TEXT.get(args.workload, '')}",
                   "batch_per_gpu": wl.batch, "tokens_per_gpu": tokens, "num_splits": st.num_splits,
                   "parallelism": f"data parallel over sequences, {world} rank(s), no collective on the path",
                   "launch_overlap": args.overlap,
                   "l2": "flushed before every step (write of 2x L2 size, then a read of it so that no dirty "
                         "line is left to write back), outside the step's events"},
        "decode": {"us": t_dec * 1e6, "latent_cache_GB/s": dec["bytes"] / t_dec / 1e9,
                   "TFLOP/s": dec["flops"] / t_dec / 1e12,
                   "roofline_frac": decode_roof_s / t_dec,
                   "roofline_us": decode_roof_s * 1e6},
        "kernels": kernels,
        "roofline": roof,
        "gpu_launches": int(launches),
        "graphs": "each timed step is one replay of a CUDA graph of the step's C-ABI calls (append on a "
                  "side stream beside the absorb" + ("; kernels launched as programmatic dependents of the "
                  "one before" if args.overlap else "") + "), timed by events at its two ends; the per-stage "
                  "times come from a second graph with events between the stages, replayed after it; e2e "
                  "replays a graph of the input copies, the step and the result copy (see e2e.how)",
        "clocks": clk,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_s * 1e3,
                "how": e2e_mode + "; wall clock from before the launch to after a synchronise, per step"},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, el = time_oracle(wl, seconds=args.ref_seconds)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                                "sample": f"{n} whole sequences of the same workload through the fp64 "
                                          f"oracle (absorbed form: absorb, decode, output projection), "
                                          f"{el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    st.close()
    dist.finish()


if __name__ == "__main__":
    main()
