"""Benchmark: exact attention on B200 through the library's C ABI, one JSON line on rank 0.

Headline step (default workload cfg4, the largest single-GPU prefill): one bf16
prefill launch, batch 1, 8 heads, n_q = n_kv = 32768, d = 128, Q,K ~ N(0, 2.5^2),
V ~ N(0,1), scale 1/sqrt(128), non-causal, over inputs resident in HBM.
value = algorithmic TFLOP/s (two matmuls, 2 FLOP per multiply-add, causal
halved).  L2 is flushed (256 MiB write) before every timed launch; each launch
is timed with CUDA events on the launching stream and the flush is excluded.

The line also carries:
  roofline      the headline kernel's achieved TFLOP/s against the measured bf16 peak, and
                against the spec dense-bf16 figure
  prefill_legs  the other prefill workloads, each in its own timed loop (at least
                --leg-seconds of launches) with its own roofline: cfg2 (d = 64, 4 x 16 heads,
                n = 2048) non-causal and causal, cfg3 (d = 128 causal, 32 heads, n = 8192),
                cfg3w (cfg3 under a 512-key causal window)
  backward      dQ, dK, dV of cfg2, cfg2 causal and cfg3
  decode        the decode workload (64 x 32 heads, cache 16384, lengths U{1024..16384},
                d = 128) in GB/s of algorithmic bytes against the measured HBM copy rate;
                decode_gqa the same with 64 query heads over 8 key/value heads
  e2e           the headline step through the public API from pinned host buffers
                (host->device inputs and device->host outputs inside the timed region)
  cpu_baseline  the CPU oracle on a bounded sample of rows of the headline workload
  clocks        nvidia-smi SM clocks and throttle reasons sampled during the timed region

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
# B200 datasheet figures (dense bf16 tensor, HBM3e), the spec denominators reported beside the measured ones
SPEC = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}
PREFILL_SOURCES = ["memory_optimal_sdpa_b200/csrc/prefill_bf16.cuh", "memory_optimal_sdpa_b200/csrc/sm100.cuh"]
DECODE_SOURCES = ["memory_optimal_sdpa_b200/csrc/decode.cuh"]
BWD_SOURCES = ["memory_optimal_sdpa_b200/csrc/backward.cuh", "memory_optimal_sdpa_b200/csrc/backward_d64.cuh",
               "memory_optimal_sdpa_b200/csrc/sm100.cuh"]
GQA_SOURCES = ["memory_optimal_sdpa_b200/csrc/decode_gqa.cuh", "memory_optimal_sdpa_b200/csrc/decode.cuh",
               "memory_optimal_sdpa_b200/csrc/sm100.cuh"]
PREFILL_WORKLOADS = ["cfg4", "cfg3", "cfg2", "cfg2c", "cfg3w"]
METRIC = "attention fwd TFLOP/s (prefill) & decode HBM GB/s, as % of B200 roofline"
DESCRIBE = {
    "cfg2": "cfg2: prefill bf16 batch 4 x 16 heads, n_q = n_kv = 2048, d_k = d_v = 64, scale 1/8, non-causal",
    "cfg2c": "cfg2c: prefill bf16 batch 4 x 16 heads, n_q = n_kv = 2048, d_k = d_v = 64, scale 1/8, causal",
    "cfg3": "cfg3: prefill bf16 batch 1 x 32 heads, n_q = n_kv = 8192, d_k = d_v = 128, scale 1/sqrt(128), causal, "
            "V ~ U(-1,1)",
    "cfg4": "cfg4: prefill bf16 batch 1 x 8 heads, n_q = n_kv = 32768, d_k = d_v = 128, scale 1/sqrt(128), "
            "non-causal, Q,K ~ N(0, 2.5^2)",
    "cfg3w": "cfg3w: cfg3 under a causal local window of 512 keys (window_left 511, window_right 0)",
}


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
        return float(fields["dram_bytes_per_launch_full_workload"].split()[0])
    except (KeyError, ValueError, IndexError):
        return None


class ClockSampler:
    """nvidia-smi SM clocks, utilisation and throttle reasons, sampled every 20 ms while running.

    summary(t0, t1) reports the samples taken inside [t0, t1] (host wall clock; a timed region)
    when there are any, else the samples of the whole window during which the GPU was busy
    (utilisation > 0), and says which.
    """
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,utilization.gpu,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index, period_ms=20):
        self.index = index
        self.period_ms = period_ms
        self.proc = None
        self.samples = []  # (unix time, sm_mhz, max_mhz, util, reasons)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
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
            time.sleep(0.1)  # let the last sample land
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self, t0=None, t1=None):
        inside = [x for x in self.samples if t0 is not None and t0 - 0.01 <= x[0] <= t1 + 0.01]
        chosen, where = inside, "timed region"
        if not chosen:
            chosen, where = [x for x in self.samples if x[3] > 0], "busy samples of the bench window"
        if not chosen:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "from": "none"}
        reasons = sorted(set().union(*(x[4] for x in chosen)))
        return {"sm_mhz": float(np.median([x[1] for x in chosen])), "sm_max_mhz": chosen[-1][2],
                "sm_mhz_min": float(min(x[1] for x in chosen)), "reasons": reasons, "samples": len(chosen),
                "from": where, "period_ms": self.period_ms}


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
    """CPU oracle on sampled rows of the workloads; returns (TFLOP/s, cores, description, seconds)."""
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

    f, t = run(2)
    per_row = t / (2 * w0.batch * w0.heads * len(w_list))
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


def tensor_roofline(kernel, flops, nbytes, t, peaks, peak_kind, traffic, note):
    """Roofline object of a tensor-pipe-bound launch: algorithmic FLOPs / mean launch time against the
    measured burst bf16 peak (the kernel is timed alone) and against the spec dense-bf16 figure."""
    peak = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    a = flops / t / 1e12
    return {"kernel": kernel, "bound": "tensor", "achieved": round(a, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(a / peak, 4), "peak_kind": peak_kind + " burst bf16 (kernel timed alone)",
            "spec_peak": SPEC["bf16_tflops"], "spec_frac": round(a / SPEC["bf16_tflops"], 4),
            "sustained_peak": peaks.get("bf16_tflops_sustained"),
            "sustained_frac": (round(a / peaks["bf16_tflops_sustained"], 4) if peaks.get("bf16_tflops_sustained")
                               else None),
            "algorithmic_flop_per_launch": float(flops), "algorithmic_bytes_per_launch": float(nbytes),
            "traffic": traffic,
            "traffic_over_algorithmic_bytes": None if traffic is None else round(traffic / nbytes, 3),
            "traffic_source": note}


def hbm_roofline(kernel, nbytes, t, peaks, peak_kind, traffic):
    peak = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    g = nbytes / t / 1e9
    return {"kernel": kernel, "bound": "hbm", "achieved": round(g, 1), "peak": peak, "unit": "GB/s",
            "frac": round(g / peak, 4), "peak_kind": peak_kind + " HBM copy", "spec_peak": SPEC["hbm_gbs"],
            "spec_frac": round(g / SPEC["hbm_gbs"], 4), "traffic": traffic, "algorithmic_bytes": float(nbytes)}


def workload(name):
    from seeded_inputs import workloads as W
    return getattr(W, name.upper())


def kernel_name(w):
    mask = 2 if w.window is not None else int(w.causal)
    return "sdpa_fwd_bf16_kernel<%d,%d>" % (w.d, mask)


class PrefillInputs:
    """Seeded inputs of a prefill workload, resident on the device, and its output buffers."""

    def __init__(self, w, dev):
        import torch
        from seeded_inputs import workloads as W
        self.w = w
        self.host = W.prefill_host(w)
        self.q, self.k, self.v = (W.to_torch(self.host[n], dev) for n in ("q", "k", "v"))
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((w.batch, w.heads, w.n_q), dtype=torch.float32, device=dev)


def prefill_call(sdpa, w, q, k, v, o, lse, stream):
    if w.window is not None:
        sdpa.fwd_window(q, k, v, w.window[0], w.window[1], scale=w.scale_f32, o=o, lse=lse, stream=stream)
    else:
        sdpa.fwd(q, k, v, causal=w.causal, scale=w.scale_f32, o=o, lse=lse, stream=stream)


def timed_launches(call, n, flush, stream):
    """n launches, each preceded by an (untimed) L2 flush and bracketed by CUDA events on `stream`;
    returns the per-launch seconds."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    return np.array([a.elapsed_time(b) for a, b in ev]) / 1e3


def launches_for(call, flush, stream, seconds, minimum):
    """Launch count that fills about `seconds` of device time (at least `minimum`)."""
    t = float(np.median(timed_launches(call, 3, flush, stream)))
    return max(minimum, int(math.ceil(seconds / max(t, 1e-7))))


def run_e2e(sdpa, w, inp, stream, steps):
    """The headline step end to end through the public API: pinned host inputs -> device -> pinned host
    outputs.  Every step copies all of its inputs in and all of its outputs out; the copies of
    neighbouring steps run on their own streams (double-buffered device tensors), overlapping this
    step's kernel.  Returns (seconds for `steps` steps on this rank, h2d bytes, d2h bytes per step)."""
    import torch
    hq, hk, hv = (torch.from_numpy(inp.host[n].view(np.int16)).view(torch.bfloat16).pin_memory()
                  for n in ("q", "k", "v"))
    dins = [tuple(torch.empty_like(x) for x in (inp.q, inp.k, inp.v)) for _ in range(2)]
    douts = [(torch.empty_like(inp.o), torch.empty_like(inp.lse)) for _ in range(2)]
    houts = [(torch.empty(inp.o.shape, dtype=inp.o.dtype).pin_memory(),
              torch.empty(inp.lse.shape, dtype=inp.lse.dtype).pin_memory()) for _ in range(2)]
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
                o, lse = douts[j % 2]
                prefill_call(sdpa, w, *dins[j % 2], o, lse, stream)
                ev_comp[j].record(stream)
            m = i - 2
            if 0 <= m < n:  # copy out step m
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[m])
                    (o, l), (po, pl) = douts[m % 2], houts[m % 2]
                    po.copy_(o, non_blocking=True)
                    pl.copy_(l, non_blocking=True)
                    ev_out[m].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / 1e3

    e2e_run(3)
    barrier()
    t = e2e_run(steps)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = sum(x.numel() * x.element_size() for x in houts[0])
    return t, h2d, d2h


def run_prefill_leg(args, sdpa, name, dev, stream, flush, peaks, peak_kind, clocks):
    w = workload(name)
    inp = PrefillInputs(w, dev)
    call = lambda: prefill_call(sdpa, w, inp.q, inp.k, inp.v, inp.o, inp.lse, stream)
    for _ in range(args.warmup):
        call()
    n = launches_for(call, flush, stream, args.leg_seconds, args.steps)
    t0 = time.time()
    per = timed_launches(call, n, flush, stream)
    t1 = time.time()
    if sdpa.get_last_device_error() != sdpa.SDPA_OK:
        raise SystemExit("device error in prefill leg %s" % name)
    t = float(per.mean())
    traffic = profiled_traffic("prefill_%s_dram.txt" % name, PREFILL_SOURCES)
    return {"workload": DESCRIBE[name], "launches": n, "ms": round(t * 1e3, 4), "ms_min": round(float(per.min()) * 1e3, 4),
            "value": round(w.flops() / t / 1e12, 2), "unit": "TFLOP/s",
            "roofline": tensor_roofline(kernel_name(w) + " (%s)" % name, w.flops(), w.bytes(), t, peaks, peak_kind,
                                        traffic, "profiles/prefill_%s_dram.txt" % name),
            "cost_model": cost_model(w.flops(), w.bytes(), t, peaks, standard_bytes(w)),
            "clocks": clocks.summary(t0, t1)}


def run_backward(args, sdpa, si, W, name, dev, stream, flush, peaks, peak_kind, clocks):
    """dQ, dK, dV of a prefill workload from the forward's O and LSE.  Algorithmic FLOPs: 2.5x the
    forward's (five matrix products of the gradient).  At d = 64 the kernels execute exactly those
    (dQ is formed beside dK and dV and reduce-added in fp32); at d = 128 they execute 3.5x (S and dP
    are formed in both the dK/dV and the dQ kernel)."""
    import torch
    w = workload(name)
    inp = PrefillInputs(w, dev)
    prefill_call(sdpa, w, inp.q, inp.k, inp.v, inp.o, inp.lse, stream)
    do = W.to_torch(si.fill_host((w.batch, w.heads, w.n_q, w.d), w.seed, si.STREAM_DO), dev)
    dq, dk, dv = torch.empty_like(inp.q), torch.empty_like(inp.k), torch.empty_like(inp.v)
    ws = torch.empty(sdpa.bwd_workspace_size(w.batch, w.heads, w.n_q), dtype=torch.uint8, device=dev)
    call = lambda: sdpa.bwd(inp.q, inp.k, inp.v, inp.o, do, inp.lse, causal=w.causal, scale=w.scale_f32,
                            dq=dq, dk=dk, dv=dv, workspace=ws, stream=stream)
    for _ in range(args.warmup):
        call()
    n = launches_for(call, flush, stream, args.leg_seconds, args.steps)
    t0 = time.time()
    per = timed_launches(call, n, flush, stream)
    t1 = time.time()
    if sdpa.get_last_device_error() != sdpa.SDPA_OK:
        raise SystemExit("device error in backward %s" % name)
    t = float(per.mean())
    flops = 2.5 * w.flops()
    nbytes = 2 * w.bytes()  # Q, K, V, O, dO and LSE read; dQ, dK, dV written (dO is O's size)
    kernels = "sdpa_bwd_pre + " + ("sdpa_bwd_d64 + sdpa_bwd_dq_out" if w.d == 64 else "sdpa_bwd_dkdv + sdpa_bwd_dq")
    roof = tensor_roofline("%s (%s)" % (kernels, name), flops, nbytes, t, peaks,
                           peak_kind, profiled_traffic("backward_%s_dram.txt" % name, BWD_SOURCES),
                           "profiles/backward_%s_dram.txt (all three kernels of a call)" % name)
    roof["executed_flop"] = (2.5 if w.d == 64 else 3.5) * w.flops()
    return {"workload": DESCRIBE[name], "launches": n, "gpu_launches_per_call": 3, "ms": round(t * 1e3, 4),
            "value": round(flops / t / 1e12, 1), "unit": "TFLOP/s", "roofline": roof,
            "clocks": clocks.summary(t0, t1)}


def run_decode(args, sdpa, si, W, dev, stream, flush, peaks, peak_kind, clocks, grouped=False):
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
    for _ in range(args.warmup):
        call()
    n = launches_for(call, flush, stream, args.leg_seconds, args.steps)
    t0 = time.time()
    per = timed_launches(call, n, flush, stream)
    t1 = time.time()
    if sdpa.get_last_device_error() != sdpa.SDPA_OK:
        raise SystemExit("device error in decode")
    t = float(per.mean())
    gbs = w.bytes(lens) / t / 1e9
    del kc, vc
    torch.cuda.empty_cache()
    heads = ("%d query heads over %d key/value heads" % (w.heads, w.kv_heads)) if grouped else "%d heads" % w.heads
    if grouped:
        kernel, prof, srcs = "sdpa_decode_gqa_kernel<16> + combine", "decode_cfg5g_dram.txt", GQA_SOURCES
    else:
        kernel, prof, srcs = "sdpa_decode_split_kernel + combine", "decode_cfg5_dram.txt", DECODE_SOURCES
    traffic = None if args.decode_batch != 64 else profiled_traffic(prof, srcs)
    return {"workload": "%s: decode bf16 batch %d x %s, cache 16384, lengths U{1024..16384} (sum %d), d = 128"
                        % (w.name, w.batch, heads, int(lens.sum())),
            "launches": n, "value": round(gbs, 1), "unit": "GB/s", "ms": round(t * 1e3, 4),
            "gpu_launches_per_call": 2, "gflops": round(w.flops(lens) / t / 1e9, 1),
            "cost_model": cost_model(w.flops(lens), w.bytes(lens), t, peaks),
            "roofline": hbm_roofline(kernel, w.bytes(lens), t, peaks, peak_kind, traffic),
            "clocks": clocks.summary(t0, t1)}


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
    wh = workload(args.workload)
    inp = PrefillInputs(wh, dev)  # seeded on the host, copied once: resident in HBM for the timed region
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    call = lambda: prefill_call(sdpa, wh, inp.q, inp.k, inp.v, inp.o, inp.lse, stream)

    clocks = ClockSampler(local_rank).__enter__()  # sampled from warm-up through the last leg
    time.sleep(0.2)
    for _ in range(args.warmup):
        call()
    if sdpa.get_last_device_error() != sdpa.SDPA_OK:
        raise SystemExit("device error during warm-up")

    # ---- device-timed region: K steps (one launch each), L2 flushed before each (flush not timed)
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    per_launch = timed_launches(call, args.steps, flush, stream)
    t_wall1 = time.time()
    barrier()
    local_t = float(per_launch.sum())
    t_max, units = aggregate(local_t, wh.flops() * args.steps)
    value = units / t_max / 1e12
    if sdpa.get_last_device_error() != sdpa.SDPA_OK:
        raise SystemExit("device error in the timed region")
    t_dom = float(per_launch.mean())
    roof = tensor_roofline(kernel_name(wh) + " (%s)" % wh.name, wh.flops(), wh.bytes(), t_dom, peaks, peak_kind,
                           profiled_traffic("prefill_%s_dram.txt" % wh.name, PREFILL_SOURCES),
                           "profiles/prefill_%s_dram.txt" % wh.name)
    roof["per_launch_ms"] = round(t_dom * 1e3, 4)
    roof["per_launch_ms_min"] = round(float(per_launch.min()) * 1e3, 4)

    # ---- end to end through the public API
    e_local, h2d, d2h = run_e2e(sdpa, wh, inp, stream, args.steps)
    e_max, e_units = aggregate(e_local, wh.flops() * args.steps)
    e2e = {"value": round(e_units / e_max / 1e12, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h,
           "schedule": "steps pipelined: step i+1's inputs copied in and step i-1's outputs copied out "
                       "(pinned host memory, own streams) while step i computes"}
    del inp

    # ---- sub-benchmarks: the other prefill workloads, backward, decode (each its own timed loop)
    legs = {}
    if not args.skip_legs:
        for name in args.legs.split(","):
            if name and name != args.workload:
                legs[name] = run_prefill_leg(args, sdpa, name, dev, stream, flush, peaks, peak_kind, clocks)
    backward = {}
    if not args.skip_backward:
        for name in filter(None, args.backward_legs.split(",")):
            backward[name] = run_backward(args, sdpa, si, W, name, dev, stream, flush, peaks, peak_kind, clocks)
    dlegs = [] if args.skip_decode else args.decode_legs.split(",")
    decode = (run_decode(args, sdpa, si, W, dev, stream, flush, peaks, peak_kind, clocks) if "cfg5" in dlegs
              else None)
    decode_gqa = (run_decode(args, sdpa, si, W, dev, stream, flush, peaks, peak_kind, clocks, grouped=True)
                  if "cfg5g" in dlegs else None)
    clocks.__exit__(None, None, None)

    line = {
        "metric": METRIC,
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t_max / args.steps * 1e3, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded SplitMix64/Box-Muller, bf16 RNE)",
        "config": {"workload": DESCRIBE[wh.name], "global_batch": wh.batch * world, "seq_len": wh.n_q,
                   "heads": wh.heads, "head_dim": wh.d,
                   "parallelism": "replicas x%d (independent heads, no collective)" % world,
                   "l2": "flushed before every timed launch (256 MiB write, not timed); inputs also exceed L2"},
        "roofline": roof,
        "cost_model": cost_model(wh.flops(), wh.bytes(), t_dom, peaks, standard_bytes(wh)),
        "gpu_launches": args.steps,
        "e2e": e2e,
        "clocks": clocks.summary(t_wall0, t_wall1),
        "clocks_all_legs": clocks.summary(t_wall0, time.time()),
    }
    if legs:
        line["prefill_legs"] = legs
    if backward:
        line["backward"] = backward
    if decode is not None:
        line["decode"] = decode
    if decode_gqa is not None:
        line["decode_gqa"] = decode_gqa
    if rank == 0 and world == 1 and not args.skip_cpu:
        rate, cores, desc, secs = oracle_rate([wh], args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(rate, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": round(secs, 2)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The CPU oracle as the reference arm: rank 0 only, K timed steps of a bounded sample of the workload."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    wh = workload(args.workload)
    for _ in range(args.warmup):
        oracle_rate([wh], 0.2)
    rates, secs = [], 0.0
    desc, cores = "", 1
    for _ in range(args.steps):
        rate, cores, desc, t = oracle_rate([wh], args.cpu_seconds / max(args.steps, 1))
        rates.append(rate)
        secs += t
    value = float(np.mean(rates))
    line = {"impl": "reference", "metric": METRIC,
            "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs / args.steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded SplitMix64/Box-Muller, bf16 RNE)",
            "config": {"workload": DESCRIBE[wh.name] + " (bounded row sample per step)",
                       "global_batch": wh.batch, "seq_len": wh.n_q, "heads": wh.heads, "head_dim": wh.d,
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)  # ~0.14 s of the headline kernel: 7 clock samples
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="cfg4", choices=PREFILL_WORKLOADS, help="headline prefill workload")
    ap.add_argument("--leg-seconds", type=float, default=0.1,
                    help="device time each sub-benchmark's timed loop fills (at least --steps launches)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU oracle sample budget")
    ap.add_argument("--legs", default="cfg2,cfg2c,cfg3,cfg3w,cfg4",
                    help="prefill sub-benchmarks (comma list; the headline workload is skipped)")
    ap.add_argument("--backward-legs", default="cfg2,cfg2c,cfg3", help="backward sub-benchmarks (comma list)")
    ap.add_argument("--decode-legs", default="cfg5,cfg5g", help="decode sub-benchmarks (comma list of cfg5, cfg5g)")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-legs", action="store_true", help="no prefill sub-benchmarks")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-backward", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=64, help="sequences in the decode workload (default 64)")
    args = ap.parse_args(argv)
    for name in filter(None, args.legs.split(",") + args.backward_legs.split(",")):
        if name not in PREFILL_WORKLOADS:
            raise SystemExit("unknown workload %r (choose from %s)" % (name, ", ".join(PREFILL_WORKLOADS)))
    for name in filter(None, args.decode_legs.split(",")):
        if name not in ("cfg5", "cfg5g"):
            raise SystemExit("unknown decode workload %r (choose from cfg5, cfg5g)" % name)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
