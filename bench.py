#!/usr/bin/env python
"""Throughput of the AuT audio-encoder forward on B200 (one process per GPU).

One step = one full forward (plan upload, conv stem, 24 pre-LN layers with
window attention, final LN and projector) over one batch of synthetic log-mel
input resident in HBM.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload omni_16req]
  python bench.py --impl reference ...   # the CPU oracle, timed on the host cores

Timing: W untimed warm-up steps; then K steps, each bracketed by CUDA events on
the launching stream, with a 256 MiB buffer written between steps (L2 flush,
outside the events); barrier + synchronize around the timed region; the
device time is the max over ranks.  Weak scaling: with N ranks the job is N
copies of the workload's requests, cut at window boundaries and assigned to
the ranks by tokens (audio_encoder_aut_b200.shard); each rank encodes its
shard, weights replicated; no collective is on the data path (only the timing
maximum is reduced).  `--gpus N` outside a launcher starts the N processes
itself.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import aut_synth as S  # noqa: E402

METRIC = "encoded audio-seconds/s on 1 B200 (bf16); tokens/s and % of bf16 TC peak alongside"
UNIT = "audio-s/s"


# The roofline's kernel: gemm_tc_kernel over the layer GEMMs (qkv, o_proj, fc1,
# fc2; 4 launches per layer).  DRAM bytes (read + write) per launch, mean over
# layer 0's four launches of one omni_16req forward (every layer has the same
# shapes), from one ncu capture of the current kernel: dram__bytes_read.sum +
# dram__bytes_write.sum of 18.26 / 28.34 / 21.57 / 63.51 MB (the command and
# the table are in profiles/gemm_tc_kernel_dram_omni_16req.md).  Set to None
# whenever the kernel changes.
LAYER_GEMM_DRAM_BYTES_PER_LAUNCH = 32.920e6
LAYER_GEMMS = ("qkv", "o_proj", "fc1", "fc2")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["bf16_tflops"], d["bf16_tflops_sustained"], d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# ------------------------------------------------------------ FLOP credit ----
def _half(n):
    return (n + 1) // 2 if n > 0 else 0


def credited_flops(cfg, lens, cu):
    """Algorithmic FLOPs of one forward, valid positions only, by kernel kind:
    the stem per chunk (conv1, conv2, conv3 on the output positions the chunk's
    valid frames reach, conv_out on its kept tokens), 2 d (3 d), 2 d d, 2 d F,
    2 F d per token and layer for qkv, o_proj, fc1, fc2, 4 d len^2 per window
    and layer for attention, 2 d d and 2 d O per token for the projector."""
    C, d, F, O, L = (cfg.downsample_hidden_size, cfg.d_model, cfg.encoder_ffn_dim,
                     cfg.output_dim, cfg.encoder_layers)
    k = dict.fromkeys(["conv1", "conv2", "conv3", "conv_out"], 0)
    for n in lens:
        for s in range(0, n, 100):
            v = min(100, n - s)
            f1 = _half(v)
            f2 = _half(f1)
            f3 = _half(f2)
            k["conv1"] += 2 * C * 9 * 64 * f1
            k["conv2"] += 2 * C * 9 * C * 32 * f2
            k["conv3"] += 2 * C * 9 * C * 16 * f3
            k["conv_out"] += 2 * f3 * 16 * C * d
    T = cu[-1]
    k["qkv"] = L * 2 * T * 3 * d * d
    k["o_proj"] = L * 2 * T * d * d
    k["fc1"] = L * 2 * T * d * F
    k["fc2"] = L * 2 * T * F * d
    k["attention"] = L * 4 * d * sum((b - a) ** 2 for a, b in zip(cu[:-1], cu[1:]))
    k["proj1"] = 2 * T * d * d
    k["proj2"] = 2 * T * d * O
    return k


def layer_gemm_operand_bytes(cfg, T):
    """Mean bytes a layer GEMM must read once (A, W, and the fp32 residual of
    o_proj and fc2; outputs stay in L2): the algorithmic traffic per launch."""
    d, F = cfg.d_model, cfg.encoder_ffn_dim
    qkv = 2 * T * d + 2 * 3 * d * d
    o = 2 * T * d + 2 * d * d + 4 * T * d
    fc1 = 2 * T * d + 2 * F * d
    fc2 = 2 * T * F + 2 * d * F + 4 * T * d
    return (qkv + o + fc1 + fc2) / 4


def memory_kernel_bytes(cfg, T, n_chunks):
    """Algorithmic bytes per step of the kernels measured against HBM bandwidth:
    window attention reads q, k, v (6 d B) and writes O (2 d B) per token per
    layer; each layer LayerNorm reads 4 d B and writes 2 d B per token, the final
    one writes [hi | lo] (4 d B); conv1 reads the chunk's mel tile and writes its
    64 x 50 x C bf16 output."""
    d, L, C = cfg.d_model, cfg.encoder_layers, cfg.downsample_hidden_size
    return {"attention": L * 8 * d * T,
            "layernorm": 2 * L * 6 * d * T + 8 * d * T,
            "conv1": n_chunks * (64 * 50 * C * 2 + 128 * 100 * 2)}


# ---------------------------------------------------------------- clocks ----
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every 5 ms
    in a background thread while the timed region runs."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device):
        import threading
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml as N
            N.nvmlInit()
            h = None
            try:
                p = __import__("torch").cuda.get_device_properties(torch_device)
                h = N.nvmlDeviceGetHandleByPciBusId(
                    f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0")
            except Exception:
                h = N.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self.N, self.h = N, h
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
            get_r = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                N.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self._stop.is_set():
                    self.samples.append(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM))
                    r = get_r(h)
                    for bit, name in self.REASONS.items():
                        if r & bit:
                            self.reasons.add(name)
                    self._stop.wait(0.005)
            self.t = threading.Thread(target=loop, daemon=True)
            self.t.start()
        except Exception as e:  # no NVML: report that instead of clocks
            self.t = None
            self.error = str(e)

    def stop(self):
        if self.t is None:
            return {"error": getattr(self, "error", "nvml unavailable")}
        self._stop.set()
        self.t.join()
        sm = self.samples
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(sm) if sm else None, "reasons": sorted(self.reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- CPU oracle ----
def cpu_oracle_run(cfg, w, feats, lens):
    import oracle as O
    t0 = time.perf_counter()
    O.forward(cfg, w, feats, lens, dtype=np.float32)
    return time.perf_counter() - t0


def oracle_sample(workload, lens, seconds_wanted=30.0):
    """A bounded sample of the workload for the CPU oracle: its first requests
    until about `seconds_wanted` of audio (clipped to a whole number of windows)."""
    out, tot = [], 0
    for n in lens:
        take = min(n, int(seconds_wanted * 100) - tot)
        if take <= 0:
            break
        out.append(take)
        tot += take
    return out


def layout_counts(cfg, lens):
    """(total tokens, windows, chunks) of a batch, from the oracle's planner
    (the reference arm runs none of the library)."""
    import oracle as O
    lay = O.plan(cfg, lens)
    return lay.total_tokens, len(lay.cu_seqlens) - 1, len(lay.chunks)


def workload_config(args, world, lens, T, nW, nch, impl="ours"):
    """The `config` object of the JSON line (both arms)."""
    cfg = S.WORKLOADS[args.workload]
    c = {"workload": args.workload, "requests": len(lens), "frames": sum(lens),
         "audio_seconds": sum(lens) / 100.0, "total_tokens": T, "windows": nW,
         "chunks": nch, "d_model": cfg.d_model, "layers": cfg.encoder_layers}
    if impl == "reference":
        c.update(launch="numpy oracle on the host cores (no GPU)", l2="not applicable (CPU)",
                 parallelism="one process (rank 0)")
    else:
        c.update(l2="256 MiB buffer written between timed steps (outside the events)",
                 launch="CUDA graph of the whole forward" if args.graph else "eager",
                 parallelism=f"dp{world}: {world} copies of the workload's requests, "
                             "window-sharded across the ranks (LPT by tokens), "
                             "rows kept on the rank that computed them")
    return c


def reference_arm(args, rank, world):
    """The oracle as it stands, timed on the host cores; each step encodes one
    8 s window of the workload's first request."""
    if rank != 0:
        return
    cfg = S.WORKLOADS[args.workload]
    lens_all = S.request_lengths(args.workload)
    w = S.weights(cfg)
    lens = [min(lens_all[0], cfg.n_window_infer)]
    feats = S.features(lens)
    for _ in range(args.warmup):
        cpu_oracle_run(cfg, w, feats, lens)
    ts = [cpu_oracle_run(cfg, w, feats, lens) for _ in range(args.steps)]
    audio = sum(lens) / 100.0
    value = audio * len(ts) / sum(ts)
    cores = len(os.sched_getaffinity(0))
    sample = f"{lens[0]} frames (one attention window) of request 0 per step, numpy fp32"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(ts) / len(ts),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": workload_config(args, 1, lens_all, *layout_counts(cfg, lens_all),
                                      impl="reference"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm ----
def our_arm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from audio_encoder_aut_b200 import _lib as A
    from audio_encoder_aut_b200.encoder import Encoder

    from audio_encoder_aut_b200 import shard as SH

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = S.WORKLOADS[args.workload]
    base = S.request_lengths(args.workload)
    w = S.weights(cfg)
    enc = Encoder(cfg, w, local_rank)
    # The whole job: `world` copies of the workload's requests (copy i with its
    # own features), cut at window boundaries and assigned to the ranks by
    # tokens; this rank encodes its shard as one packed batch.  One rank: the
    # workload itself.
    glens = base * world
    shard = SH.assign(SH.pieces(glens, cfg.n_window_infer), world, enc.c)[rank]
    copies = sorted({p.request // len(base) for p in shard})
    feats_of = {i: S.features(base, seed=S.SEED_FEATURES + i) for i in copies}
    lens = [p.frames for p in shard]
    feats = np.zeros((len(shard), cfg.num_mel_bins, max(lens)), np.float32)
    for j, p in enumerate(shard):
        f = feats_of[p.request // len(base)][p.request % len(base)]
        feats[j, :, :p.frames] = f[:, p.frame0:p.frame0 + p.frames]
    tpr, cu, T, nW, nch = enc.plan(lens)
    audio_s = sum(lens) / 100.0
    job_audio_s = sum(glens) / 100.0
    fd = enc.features_to_device(feats)
    out = torch.empty((T, cfg.output_dim), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, k):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(k)]
        barrier()
        torch.cuda.synchronize()
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        barrier()
        return [a.elapsed_time(b) for a, b in evs]

    if args.graph:
        graph, _ = enc.capture(fd, lens, out=out)
        step = graph.replay
    else:
        step = lambda: enc.encode(fd, lens, out=out)  # noqa: E731
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert enc.check() == A.AUT_OK

    sampler = ClockSampler(dev)
    step_ms = timed(step, args.steps)
    clocks = sampler.stop()
    status = enc.check()
    total_ms = sum(step_ms)
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms = total_ms / args.steps
    job_T = torch.tensor([T], dtype=torch.int64, device=dev)
    if world > 1:
        dist.all_reduce(job_T)
    value = job_audio_s * args.steps / (total_ms / 1e3)
    tokens_s = int(job_T.item()) * args.steps / (total_ms / 1e3)
    kflops = credited_flops(cfg, lens, cu)
    flops = sum(kflops.values())
    pk, pk_sus, hbm, pk_src = peaks()

    # Per-kernel breakdown: the same forward captured as a graph with an event
    # node after every launch, replayed like the timed steps (L2 flushed first).
    # The first launch's time counts from an event recorded just before the replay.
    cap = 4096
    events = [torch.cuda.Event(enable_timing=True) for _ in range(cap + 1)]
    for e in events:  # torch creates the CUDA event on first record
        e.record(stream)
    torch.cuda.synchronize()
    ev_ptrs = (A.c_void_p * cap)(*[e.cuda_event for e in events[1:]])
    kinds = (A.c_int32 * cap)()
    trace = A.aut_trace(ev_ptrs, cap, 0, kinds)
    if args.graph:
        tgraph, _ = enc.capture(fd, lens, out=out, trace=trace)
        traced_step = tgraph.replay
    else:
        def traced_step():
            enc.encode(fd, lens, out=out, trace=trace)
        traced_step()
        torch.cuda.synchronize()
    launches = trace.count
    assert 0 < launches <= cap
    per_kind = {}
    n_trace = max(3, min(10, args.steps))
    for _ in range(n_trace):
        flush.zero_()
        events[0].record(stream)
        traced_step()
        torch.cuda.synchronize()
        for i in range(launches):
            k = A.KERNEL_KINDS[kinds[i]]
            per_kind.setdefault(k, []).append(events[i].elapsed_time(events[i + 1]))
    kind_ms = {k: sum(v) / n_trace for k, v in per_kind.items()}
    # The roofline's kernel: the layer GEMMs.  achieved = their credited FLOPs
    # per launch / their mean launch time (from the event-timed replay).
    gemm_launches = sum(len(per_kind[k]) for k in LAYER_GEMMS if k in per_kind) / n_trace
    gemm_ms = sum(kind_ms[k] for k in LAYER_GEMMS if k in kind_ms)
    gemm_avg_ms = gemm_ms / gemm_launches
    gemm_flops = sum(kflops[k] for k in LAYER_GEMMS)
    achieved = gemm_flops / gemm_launches / (gemm_avg_ms / 1e3) / 1e12
    per_kind_tflops = {k: {"tflops": round(kflops[k] / (kind_ms[k] / 1e3) / 1e12, 1),
                           "frac": round(kflops[k] / (kind_ms[k] / 1e3) / 1e12 / pk, 3)}
                       for k in kflops if k in kind_ms and kind_ms[k] > 0 and k in A.GEMM_KINDS}
    all_gemm = sum(kflops[k] for k in A.GEMM_KINDS if k in kflops)
    all_gemm_ms = sum(kind_ms[k] for k in A.GEMM_KINDS if k in kind_ms)
    # The other kernels against HBM bandwidth: algorithmic bytes / event-timed time.
    mem_bytes = memory_kernel_bytes(cfg, T, nch)
    memory_kernels = {k: {"gb_per_s": round(b / (kind_ms[k] / 1e3) / 1e9, 1),
                          "frac_hbm": round(b / (kind_ms[k] / 1e3) / 1e9 / hbm, 3),
                          "mb_per_step": round(b / 1e6, 2)}
                      for k, b in mem_bytes.items() if kind_ms.get(k, 0) > 0}

    # End to end through the public API: every step copies its features in from
    # pinned host memory and its fp32 result back out; the copies of steps
    # i - 1 and i + 1 overlap step i's compute (Encoder.encode_stream).
    h_feats = fd.cpu().pin_memory()
    h_outs = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    graphs, _ = enc.encode_stream([h_feats] * 3, lens, [h_outs[i % 2] for i in range(3)],
                                  before_each=flush.zero_)
    torch.cuda.synchronize()
    barrier()
    _, (e0, e1) = enc.encode_stream([h_feats] * args.steps, lens,
                                    [h_outs[i % 2] for i in range(args.steps)], graphs=graphs,
                                    before_each=flush.zero_)
    torch.cuda.synchronize()
    barrier()
    e2e_total = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_total], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_total = float(t.item())
    e2e_value = job_audio_s * args.steps / (e2e_total / 1e3)
    h_out = h_outs[0]
    del graphs

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = oracle_sample(args.workload, lens, args.cpu_sample_seconds)
        sfeats = S.features(sample, seed=S.SEED_FEATURES)
        dt = cpu_oracle_run(cfg, w, sfeats, sample)
        cpu = {"value": (sum(sample) / 100.0) / dt, "unit": UNIT,
               "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"first {len(sample)} request(s) of the workload cut to "
                         f"{sum(sample)} frames ({sum(sample) / 100:.0f} s audio), numpy fp32, "
                         f"{dt:.1f} s"}

    if rank == 0:
        q = sorted(step_ms)
        pct = lambda p: q[min(len(q) - 1, int(math.ceil(p / 100 * len(q))) - 1)]
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(args, world, glens, int(job_T.item()), nW, nch),
            "tokens_per_s": tokens_s,
            "tflops": flops / (ms / 1e3) / 1e12,
            "pct_bf16_peak": 100 * flops / (ms / 1e3) / 1e12 / pk,
            "pct_bf16_peak_sustained": 100 * flops / (ms / 1e3) / 1e12 / pk_sus,
            "step_ms_p50_p95_p99": [pct(50), pct(95), pct(99)],
            "credited_gflop_per_step": flops / 1e9,
            "roofline": {"bound": "tensor",
                         "kernel": "gemm_tc_kernel on the layer GEMMs (qkv, o_proj, fc1, fc2 "
                                   "x layers)",
                         "achieved": achieved, "peak": pk, "unit": "TFLOP/s",
                         "frac": achieved / pk, "peak_source": f"{pk_src} bf16 burst",
                         "peak_sustained": pk_sus, "launches_per_step": gemm_launches,
                         "avg_launch_ms": gemm_avg_ms,
                         "traffic": LAYER_GEMM_DRAM_BYTES_PER_LAUNCH,
                         "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + "
                                         "dram__bytes_write.sum, mean over layer 0's qkv, "
                                         "o_proj, fc1, fc2)",
                         "algorithmic_bytes_per_launch": layer_gemm_operand_bytes(cfg, T),
                         "per_gemm": per_kind_tflops,
                         "all_gemms_frac": all_gemm / (all_gemm_ms / 1e3) / 1e12 / pk,
                         "memory_kernels": memory_kernels,
                         "hbm_peak_gbs": hbm, "hbm_peak_source": pk_src},
            "kernel_ms_per_step": {k: round(v, 4) for k, v in sorted(kind_ms.items(), key=lambda x: -x[1])},
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": h_feats.numel() * h_feats.element_size(),
                    "d2h_bytes_per_step": h_out.numel() * h_out.element_size(),
                    "ms_per_step": e2e_total / args.steps,
                    "copies": "each step's host-to-device and device-to-host copies run on a "
                              "second stream, overlapping the neighbouring steps' compute; "
                              "the L2 flush before every step is inside the timed region"},
            "gpu_launches": launches * args.steps,
            "device_status": A.status_string(status),
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def sweep(args):
    """Throughput against the packed total: Omni-class batches of requests with
    log-uniform lengths on [0.5, 60] s, grown to each target token count; one
    JSON line per point (CUDA-graph replay, L2 flushed between steps)."""
    import numpy as np
    import torch
    from audio_encoder_aut_b200.encoder import Encoder

    cfg = S.WORKLOADS["omni_256req"]
    w = S.weights(cfg)
    enc = Encoder(cfg, w, 0)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    pk = peaks()[0]
    rng = np.random.default_rng(S.SEED_LENGTHS + 7)
    pool = [int(round(100 * np.exp(rng.uniform(np.log(0.5), np.log(60.0))))) for _ in range(4096)]
    for target in (1000, 2000, 4000, 8000, 16000, 32000, 64000, 100000, 128000, 200000):
        # Requests from the pool until the next one would pass the target, then
        # one request of exactly the missing k tokens: 100 floor(k / 13) +
        # 8 (k mod 13) frames gives 13 floor(k / 13) + (k mod 13) tokens.
        lens, T = [], 0
        while True:
            t_next = enc.plan(lens + [pool[len(lens)]])[2]
            if t_next > target:
                break
            lens.append(pool[len(lens)])
            T = t_next
        k = target - T
        if k > 0:
            lens.append(100 * (k // 13) + 8 * (k % 13))
        feats = S.features(lens, seed=S.SEED_FEATURES)
        fd = enc.features_to_device(feats)
        _, cu, T, nW, nch = enc.plan(lens)
        out = torch.empty((T, cfg.output_dim), dtype=torch.float32, device="cuda")
        graph, _ = enc.capture(fd, lens, out=out)
        for _ in range(3):
            graph.replay()
        ms = []
        for _ in range(5):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        t = sorted(ms)[len(ms) // 2]
        flops = sum(credited_flops(cfg, lens, cu).values())
        print(json.dumps({"sweep_tokens": T, "requests": len(lens), "audio_seconds": sum(lens) / 100,
                          "ms_per_step": t, "audio_s_per_s": sum(lens) / 100 / (t / 1e3),
                          "tokens_per_s": T / (t / 1e3), "tflops": flops / (t / 1e3) / 1e12,
                          "pct_bf16_peak": 100 * flops / (t / 1e3) / 1e12 / pk}), flush=True)
        del graph, out, fd
    assert enc.check() == 0


def _spawned_rank(rank, world, port, argv):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.argv = [sys.argv[0]] + list(argv)
    main()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="omni_16req", choices=sorted(S.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch the forward eagerly instead of replaying its CUDA graph")
    ap.add_argument("--cpu-sample-seconds", type=float, default=60.0)
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the bench line, one line per packed total of 1k-200k tokens")
    args = ap.parse_args()
    if args.sweep:
        sweep(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # Not under a launcher: start one process per GPU here.
        import socket
        import torch.multiprocessing as mp
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        mp.spawn(_spawned_rank, args=(args.gpus, port, sys.argv[1:]), nprocs=args.gpus, join=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        our_arm(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
