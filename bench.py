"""Benchmark: exact attention on B200 through the library's C ABI, one JSON line on rank 0.

Headline step (default workload cfg2): one bf16 prefill, batch 4, 16 heads,
n_q = n_kv = 2048, d = 64, scale 1/8, run non-causal AND causal -- both
launches of the tcgen05 prefill kernel -- over inputs resident in HBM.
value = algorithmic TFLOP/s (2 matmuls x 2 FLOP per multiply-add, causal
halved).  L2 is flushed (256 MiB write) before every timed step; each step is
timed with CUDA events on the launching stream and the flush is excluded.

The line also carries:
  roofline     the prefill kernel's achieved TFLOP/s against the measured bf16 peak
  decode       the decode workload (64 x 32 heads, cache 16384, lengths U{1024..16384},
               d = 128) in GB/s of algorithmic bytes against the measured HBM copy rate
  e2e          the same step through the public API from pinned host buffers
               (host->device inputs and device->host outputs inside the timed region)
  cpu_baseline the CPU oracle on a bounded sample of rows of the same workload
  clocks       nvidia-smi SM clocks and throttle reasons sampled during the timed region

Multi-GPU: `torchrun --nproc-per-node N bench.py --gpus N`: every rank runs an
independent replica (attention over independent (batch, head) slices needs no
exchange), timing is the max over ranks, value is the work of all ranks over
that time (weak scaling).  `--impl reference` times the CPU oracle instead
(rank 0 only).
"""
import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PREFILL_SOURCES = ["memory_optimal_sdpa_b200/csrc/prefill_bf16.cuh", "memory_optimal_sdpa_b200/csrc/sm100.cuh"]
DECODE_SOURCES = ["memory_optimal_sdpa_b200/csrc/decode.cuh"]
BWD_SOURCES = ["memory_optimal_sdpa_b200/csrc/backward.cuh", "memory_optimal_sdpa_b200/csrc/sm100.cuh"]
GQA_SOURCES = ["memory_optimal_sdpa_b200/csrc/decode_gqa.cuh", "memory_optimal_sdpa_b200/csrc/decode.cuh",
               "memory_optimal_sdpa_b200/csrc/sm100.cuh"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def source_digest(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(summary, paths):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("source_digest") != source_digest(paths):
        return None
    try:
        return float(fields["dram_bytes_per_launch_full_workload"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi SM clocks, utilisation and throttle reasons, sampled every 100 ms while running.

    summary(t0, t1) reports the samples taken inside [t0, t1] (host wall clock; the timed
    region) when there are any, else the samples of the whole window during which the GPU
    was busy (utilisation > 0), and says which.
    """
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,utilization.gpu,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.samples = []  # (unix time, sm_mhz, max_mhz, util, reasons)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        import datetime
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx, util = float(parts[2]), float(parts[3]), float(parts[4])
            except ValueError:
                continue
            reasons = {n for n, f in zip(self.NAMES, parts[5:9]) if f.lower() in ("active", "1")}
            self.samples.append((ts, sm, mx, util, reasons))

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.25)  # let the last sample land
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self, t0=None, t1=None):
        inside = [x for x in self.samples if t0 is not None and t0 - 0.05 <= x[0] <= t1 + 0.05]
        chosen, where = inside, "timed region"
        if not chosen:
            chosen, where = [x for x in self.samples if x[3] > 0], "busy samples of the bench window"
        if not chosen:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "from": "none"}
        reasons = sorted(set().union(*(x[4] for x in chosen)))
        return {"sm_mhz": float(np.median([x[1] for x in chosen])), "sm_max_mhz": chosen[-1][2],
                "reasons": reasons, "samples": len(chosen), "from": where}


# ---------------------------------------------------------------------------------------------- distributed
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def aggregate(local_seconds, local_units, group=None):
    """Max of the timed seconds and sum of the work units over all ranks (plain host numbers)."""
    import torch
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return local_seconds, local_units
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([local_seconds], dtype=torch.float64, device=dev)
    u = torch.tensor([local_units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(u, op=dist.ReduceOp.SUM, group=group)
    return float(t.item()), float(u.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------------------------------------ oracle leg
def oracle_rate(w_list, seconds_target, seed=0):
    """CPU oracle on sampled rows of the workloads; returns (TFLOP/s, cores, description)."""
    import oracle
    import seeded_inputs as si
    from seeded_inputs import workloads as W
    threads = oracle.threads_available()
    host = W.prefill_host(w_list[0])
    qf, kf, vf = (W.as_f32(host[n]) for n in ("q", "k", "v"))
    w0 = w_list[0]

    def run(rows_per_head):
        # one call per workload over every (batch, head) slice, so all host threads have work
        flops = 0.0
        rows = si.sample_rows(w0.n_q, rows_per_head, seed)
        t0 = time.perf_counter()
        for w in w_list:
            oracle.sdpa_rows(qf, kf, vf, w.scale_f32, w.causal, rows=rows, threads=threads)
            # per row: scores (2 d_k FLOP per visible key) and the weighted sum (2 d_v per visible key)
            vis = (rows + 1 + (w.n_kv - w.n_q)).clip(0, w.n_kv) if w.causal else np.full(len(rows), w.n_kv)
            flops += float(vis.sum()) * 2 * (w.d + w.d) * w.batch * w.heads
        return flops, time.perf_counter() - t0

    f, t = run(8)
    per_row = t / (8 * w0.batch * w0.heads * len(w_list))
    rows = int(max(2, min(w0.n_q, seconds_target / max(per_row, 1e-9) / (w0.batch * w0.heads * len(w_list)))))
    f, t = run(rows)
    desc = "%d sampled query rows per head of each of %s (oracle, double precision)" % (
        rows, "+".join(w.name for w in w_list))
    return f / t / 1e12, threads, desc, t


# --------------------------------------------------------------------------------------------------- our arm
def cost_model(flops, nbytes, t_meas, peaks, standard_bytes=None):
    """The pages' execution-time model T = alpha F + beta M (MoA article, "memory bottleneck"), alpha and
    beta the reciprocals of this GPU's measured dense bf16 rate and HBM copy bandwidth, against the
    measured time; with the traffic of an implementation that writes and reads the score and
    probability matrices, the speedup the model predicts for avoiding them."""
    a = 1.0 / (peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]) * 1e12)
    b = 1.0 / (peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]) * 1e9)
    t_add = a * flops + b * nbytes
    out = {"alpha_s_per_flop": a, "beta_s_per_byte": b, "flop": float(flops), "bytes": float(nbytes),
           "predicted_ms": round(t_add * 1e3, 5), "roofline_ms": round(max(a * flops, b * nbytes) * 1e3, 5),
           "measured_ms": round(t_meas * 1e3, 5), "measured_over_predicted": round(t_meas / t_add, 3)}
    if standard_bytes is not None:
        t_std = a * flops + b * standard_bytes
        out.update({"standard_bytes": float(standard_bytes), "standard_predicted_ms": round(t_std * 1e3, 5),
                    "predicted_speedup_vs_standard": round(t_std / t_add, 2)})
    return out


def standard_bytes(w):
    """Traffic of the textbook implementation: the DNF's bytes plus the score matrix written and read
    in fp32 and the probabilities written and read in bf16 (12 bytes per query-key pair, every pair)."""
    return w.bytes() + w.batch * w.heads * w.n_q * w.n_kv * 12


def run_ours(args):
    import torch
    import torch.distributed as dist

    import memory_optimal_sdpa_b200 as sdpa
    import seeded_inputs as si
    from seeded_inputs import workloads as W

    rank, local_rank, world = dist_env()
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d: launch N>1 with torchrun" % (args.gpus, world))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    peaks, peak_kind = load_peaks()
    w_nc = W.CFG2 if args.workload == "cfg2" else getattr(W, args.workload.upper())
    works = [w_nc, w_nc.with_causal(True)] if args.workload == "cfg2" else [w_nc]

    # Inputs: generated on the host (seeded), copied once; resident in HBM for the device-timed region.
    host = W.prefill_host(w_nc)
    q, k, v = (W.to_torch(host[n], dev) for n in ("q", "k", "v"))
    outs = [(torch.empty_like(q), torch.empty((w_nc.batch, w_nc.heads, w_nc.n_q), dtype=torch.float32, device=dev))
            for _ in works]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call(w, qq, kk, vv, o, lse):
        if w.window is not None:
            sdpa.fwd_window(qq, kk, vv, w.window[0], w.window[1], scale=w.scale_f32, o=o, lse=lse, stream=stream)
        else:
            sdpa.fwd(qq, kk, vv, causal=w.causal, scale=w.scale_f32, o=o, lse=lse, stream=stream)

    def step(qq=q, kk=k, vv=v):
        for w, (o, lse) in zip(works, outs):
            call(w, qq, kk, vv, o, lse)

    clocks = ClockSampler(local_rank).__enter__()  # sampled from warm-up through the end-to-end loop
    time.sleep(0.3)
    for _ in range(args.warmup):
        step()
    if sdpa.get_last_device_error() != sdpa.SDPA_OK:
        raise SystemExit("device error during warm-up")

    # ---- device-timed region: K steps, L2 flushed before each (flush not timed)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in works]
          for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for s in range(args.steps):
        flush.zero_()
        for (a, b), w, (o, lse) in zip(ev[s], works, outs):
            a.record(stream)
            call(w, q, k, v, o, lse)
            b.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier()
    per_launch = np.array([[a.elapsed_time(b) for (a, b) in row] for row in ev]) / 1e3  # seconds [step, launch]
    local_t = float(per_launch.sum())
    step_flops = sum(w.flops() for w in works)
    t_max, units = aggregate(local_t, step_flops * args.steps)
    value = units / t_max / 1e12
    if sdpa.get_last_device_error() != sdpa.SDPA_OK:
        raise SystemExit("device error in the timed region")

    # roofline of the dominant kernel (the first launch of the step): algorithmic FLOPs / mean launch time
    peak_tf = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    dom = works[0]
    t_dom = float(per_launch[:, 0].mean())
    achieved = dom.flops() / t_dom / 1e12
    roof = {"kernel": "sdpa_fwd_bf16_kernel<%d,%d> (%s)" % (dom.d, int(dom.causal), dom.name), "bound": "tensor",
            "achieved": round(achieved, 2), "peak": peak_tf, "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4),
            "peak_kind": peak_kind + " burst bf16 (kernel timed alone)",
            "algorithmic_flop_per_launch": dom.flops(),
            "traffic": profiled_traffic("prefill_%s_dram.txt" % dom.name, PREFILL_SOURCES),
            "per_launch_ms": {w.name: round(float(per_launch[:, i].mean()) * 1e3, 4) for i, w in enumerate(works)},
            "per_launch_tflops": {w.name: round(w.flops() / float(per_launch[:, i].mean()) / 1e12, 1)
                                  for i, w in enumerate(works)}}

    # ---- end to end through the public API: pinned host inputs -> device -> pinned host outputs.
    # Every step copies all of its inputs in and all of its outputs out; the copies of neighbouring
    # steps run on their own streams (double-buffered device tensors), overlapping this step's kernels.
    hq, hk, hv = (torch.from_numpy(host[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in ("q", "k", "v"))
    dins = [tuple(torch.empty_like(x) for x in (q, k, v)) for _ in range(2)]
    douts = [[(torch.empty_like(o), torch.empty_like(l)) for o, l in outs] for _ in range(2)]
    houts = [[(torch.empty(o.shape, dtype=o.dtype).pin_memory(), torch.empty(l.shape, dtype=l.dtype).pin_memory())
              for o, l in outs] for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        """n pipelined steps; returns the device time from the first copy in to the last copy out."""
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_comp = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        t0.record(stream)
        s_in.wait_event(t0)
        for i in range(n + 2):
            if i < n:  # copy in step i (its buffer's previous step has finished reading it)
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_comp[i - 2])
                    for dst, src in zip(dins[i % 2], (hq, hk, hv)):
                        dst.copy_(src, non_blocking=True)
                    ev_in[i].record(s_in)
            j = i - 1
            if 0 <= j < n:  # compute step j (its output buffer has been copied out)
                stream.wait_event(ev_in[j])
                if j >= 2:
                    stream.wait_event(ev_out[j - 2])
                for w, (o, lse) in zip(works, douts[j % 2]):
                    call(w, *dins[j % 2], o, lse)
                ev_comp[j].record(stream)
            m = i - 2
            if 0 <= m < n:  # copy out step m
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[m])
                    for (o, l), (po, pl) in zip(douts[m % 2], houts[m % 2]):
                        po.copy_(o, non_blocking=True)
                        pl.copy_(l, non_blocking=True)
                    ev_out[m].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / 1e3

    e2e_run(3)
    barrier()
    e_local = e2e_run(args.steps)
    clocks.__exit__(None, None, None)
    e_max, e_units = aggregate(e_local, step_flops * args.steps)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = sum(po.numel() * po.element_size() + pl.numel() * pl.element_size() for po, pl in houts[0])
    e2e = {"value": round(e_units / e_max / 1e12, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h,
           "schedule": "steps pipelined: step i+1's inputs copied in and step i-1's outputs copied out "
                       "(pinned host memory, own streams) while step i computes"}
    del hq, hk, hv, houts, dins, douts

    # ---- backward pass on the same workload (its own sub-benchmark)
    backward = None if args.skip_backward else run_backward(args, sdpa, si, W, works, q, k, v, outs, stream, flush,
                                                             peaks, peak_kind)

    # ---- decode workload (HBM-bound), its own roofline
    decode = None if args.skip_decode else run_decode(args, sdpa, si, W, dev, stream, flush, peaks, peak_kind)
    decode_gqa = (None if args.skip_decode else
                  run_decode(args, sdpa, si, W, dev, stream, flush, peaks, peak_kind, grouped=True))

    line = {
        "metric": "attention fwd TFLOP/s (prefill) & decode HBM GB/s, as % of B200 roofline",
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t_max / args.steps * 1e3, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded SplitMix64/Box-Muller, bf16 RNE)",
        "config": {"workload": "cfg2: prefill bf16 batch 4 x 16 heads, n_q = n_kv = 2048, d_k = d_v = 64, scale 1/8, "
                               "non-causal + causal per step" if args.workload == "cfg2" else args.workload,
                   "global_batch": w_nc.batch * world, "seq_len": w_nc.n_q, "heads": w_nc.heads, "head_dim": w_nc.d,
                   "parallelism": "replicas x%d (independent heads, no collective)" % world,
                   "l2": "flushed before every timed step (256 MiB write, not timed)"},
        "roofline": roof,
        "cost_model": {w.name: cost_model(w.flops(), w.bytes(), float(per_launch[:, i].mean()), peaks, standard_bytes(w))
                       for i, w in enumerate(works)},
        "gpu_launches": args.steps * len(works),
        "e2e": e2e,
        "clocks": clocks.summary(t_wall0, t_wall1),
    }
    if backward is not None:
        line["backward"] = backward
    if decode is not None:
        line["decode"] = decode
    if decode_gqa is not None:
        line["decode_gqa"] = decode_gqa
    if rank == 0 and world == 1 and not args.skip_cpu:
        rate, cores, desc, secs = oracle_rate(works, args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(rate, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": round(secs, 2)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_backward(args, sdpa, si, W, works, q, k, v, outs, stream, flush, peaks, peak_kind):
    """dQ, dK, dV of each prefill workload of the step, from the forward's O and LSE.  Algorithmic
    FLOPs: 2.5x the forward's (five matrix products of the gradient); the kernels execute seven
    (S and dP are formed in both the dK/dV and the dQ kernel)."""
    import torch
    w0 = works[0]
    do = W.to_torch(si.fill_host((w0.batch, w0.heads, w0.n_q, w0.d), w0.seed, si.STREAM_DO), q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(sdpa.bwd_workspace_size(w0.batch, w0.heads, w0.n_q), dtype=torch.uint8, device=q.device)
    res = {}
    for w, (o, lse) in zip(works, outs):
        if w.window is not None:  # the backward pass takes full or causal attention
            continue
        call = lambda: sdpa.bwd(q, k, v, o, do, lse, causal=w.causal, scale=w.scale_f32, dq=dq, dk=dk, dv=dv,
                                workspace=ws, stream=stream)
        for _ in range(max(3, args.warmup)):
            call()
        torch.cuda.synchronize()
        times = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b) / 1e3)
        if sdpa.get_last_device_error() != sdpa.SDPA_OK:
            raise SystemExit("device error in backward")
        t = float(np.mean(times))
        flops = 2.5 * w.flops()
        peak = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
        res[w.name] = {"value": round(flops / t / 1e12, 1), "unit": "TFLOP/s", "ms": round(t * 1e3, 4),
                       "gpu_launches_per_call": 3,
                       "roofline": {"kernel": "sdpa_bwd_pre + sdpa_bwd_dkdv + sdpa_bwd_dq", "bound": "tensor",
                                    "achieved": round(flops / t / 1e12, 1), "peak": peak, "unit": "TFLOP/s",
                                    "frac": round(flops / t / 1e12 / peak, 4),
                                    "peak_kind": peak_kind + " burst bf16", "algorithmic_flop": flops,
                                    "executed_flop": 3.5 * w.flops(),
                                    "traffic": (profiled_traffic("backward_cfg2_dram.txt", BWD_SOURCES)
                                                if w.name == "cfg2" else None),
                                    "traffic_covers": "dK/dV and dQ kernels (ncu); not the preprocess kernel"}}
    del dq, dk, dv, ws, do
    return res


def run_decode(args, sdpa, si, W, dev, stream, flush, peaks, peak_kind, grouped=False):
    """Decode sub-benchmark: cfg5 (one key/value head per query head) or, grouped, cfg5g."""
    import torch
    w = W.CFG5G if grouped else W.CFG5
    if args.decode_batch != w.batch:  # same recipe, fewer sequences (e.g. to keep a profiler capture small)
        w = W.Decode("%s_b%d" % (w.name, args.decode_batch), args.decode_batch, w.heads, w.n_cap, w.d, w.len_lo,
                     w.len_hi, w.scale, w.seed, w.heads_kv)
    lens = w.lengths()
    tl = torch.from_numpy(lens).to(dev)
    shape = (w.batch, w.kv_heads, w.n_cap, w.d)
    kc = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    vc = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    si.fill_device_cache(kc, tl, w.seed, si.STREAM_K)
    si.fill_device_cache(vc, tl, w.seed, si.STREAM_V)
    q = W.to_torch(si.fill_host((w.batch, w.heads, w.d), w.seed, si.STREAM_Q), dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.batch, w.heads), dtype=torch.float32, device=dev)
    if grouped:
        ws = torch.empty(sdpa.decode_gqa_workspace_size(w.batch, w.heads, w.kv_heads, w.n_cap, w.d),
                         dtype=torch.uint8, device=dev)
        call = lambda: sdpa.decode_gqa(q, kc, vc, tl, scale=w.scale_f32, o=o, lse=lse, workspace=ws, stream=stream)
    else:
        ws = torch.empty(sdpa.decode_workspace_size(w.batch, w.heads, w.n_cap, w.d), dtype=torch.uint8, device=dev)
        call = lambda: sdpa.decode(q, kc, vc, tl, scale=w.scale_f32, o=o, lse=lse, workspace=ws, stream=stream)
    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) / 1e3)
    if sdpa.get_last_device_error() != sdpa.SDPA_OK:
        raise SystemExit("device error in decode")
    t = float(np.mean(times))
    gbs = w.bytes(lens) / t / 1e9
    peak = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    del kc, vc
    torch.cuda.empty_cache()
    heads = ("%d query heads over %d key/value heads" % (w.heads, w.kv_heads)) if grouped else "%d heads" % w.heads
    if grouped:
        kernel, prof, srcs = "sdpa_decode_gqa_kernel<16> + combine", "decode_cfg5g_dram.txt", GQA_SOURCES
    else:
        kernel, prof, srcs = "sdpa_decode_split_kernel + combine", "decode_cfg5_dram.txt", DECODE_SOURCES
    return {"workload": "%s: decode bf16 batch %d x %s, cache 16384, lengths U{1024..16384} (sum %d), d = 128"
                        % (w.name, w.batch, heads, int(lens.sum())),
            "value": round(gbs, 1), "unit": "GB/s", "ms": round(t * 1e3, 4), "gpu_launches_per_call": 2,
            "gflops": round(w.flops(lens) / t / 1e9, 1),
            "cost_model": cost_model(w.flops(lens), w.bytes(lens), t, peaks),
            "roofline": {"kernel": kernel, "bound": "hbm", "achieved": round(gbs, 1),
                         "peak": peak, "unit": "GB/s", "frac": round(gbs / peak, 4),
                         "peak_kind": peak_kind + " HBM copy",
                         "traffic": (None if args.decode_batch != 64 else profiled_traffic(prof, srcs)),
                         "algorithmic_bytes": w.bytes(lens)}}


# --------------------------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The CPU oracle as the reference arm: rank 0 only, K timed steps of a bounded sample of the workload."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    from seeded_inputs import workloads as W
    import oracle
    works = [W.CFG2, W.CFG2C]
    for _ in range(args.warmup):
        oracle_rate(works, 0.2)
    rates, secs = [], 0.0
    desc, cores = "", 1
    for _ in range(args.steps):
        rate, cores, desc, t = oracle_rate(works, args.cpu_seconds / max(args.steps, 1))
        rates.append(rate)
        secs += t
    value = float(np.mean(rates))
    line = {"impl": "reference", "metric": "attention fwd TFLOP/s (prefill) & decode HBM GB/s, as % of B200 roofline",
            "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs / args.steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded SplitMix64/Box-Muller, bf16 RNE)",
            "config": {"workload": "cfg2: prefill bf16 batch 4 x 16 heads, n_q = n_kv = 2048, d_k = d_v = 64, "
                                   "scale 1/8, non-causal + causal per step (bounded row sample per step)",
                       "global_batch": 4, "seq_len": 2048, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="cfg2", choices=["cfg2", "cfg3", "cfg4", "cfg3w"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU oracle sample budget")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-backward", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=64, help="sequences in the decode workload (default 64)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
