#!/usr/bin/env python
"""Throughput benchmark of the ASR audio-encoder forward pass on B200.

One step = one whole forward (log-mel, conv stem, 32-layer windowed tower,
head, SwiGLU adapter) over one batch of seeded synthetic audio, inputs
already resident in HBM.  The default workload is 16 clips x 30 s
(6240 tokens).  Metric: encoder audio-seconds per second (whole job, all
ranks) with TFLOP/s beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle on the host cores
  python bench.py --kernel gemm_fc1 ...  # one op of the workload's shape (for ncu captures)

Under torchrun (N > 1) every rank runs an independent replica of the
workload (clips are independent: weak scaling, no collective on the data
path); the reported time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# --------------------------------------------------------------- FLOP model
def conv_len(n, k=3, s=2, p=1):
    return (n + 2 * p - k) // s + 1


def flop_breakdown(g, n_samples, batch):
    """Algorithmic FLOPs of one forward (2 per multiply-add of every GEMM and
    convolution; attention 4 w^2 d per window per layer over the keys it
    visits).  Returns dict stage -> FLOPs."""
    d, F = g.d_model, n_samples // g.hop
    out = {}
    if g.stem == synth.STEM_CONV2D_CHUNKED:
        chunks = batch * (F // g.chunk_frames)
        C = g.conv_ch
        t1, f1 = conv_len(g.chunk_frames), conv_len(g.n_mels)
        t2, f2 = conv_len(t1), conv_len(f1)
        t3, f3 = conv_len(t2), conv_len(f2)
        out["conv1"] = 2 * chunks * t1 * f1 * C * 9
        out["gemm_conv"] = 2 * chunks * (t2 * f2 + t3 * f3) * C * 9 * C
        out["gemm_conv_out"] = 2 * chunks * t3 * f3 * C * d
        tc = (F // g.chunk_frames) * t3
    else:
        tc = conv_len(conv_len(F, s=1))
        out["gemm_conv"] = 2 * batch * (F * d * 3 * g.n_mels + tc * d * 3 * d)
    T = tc * batch
    L = g.n_layers
    out["gemm_qkv"] = 2 * T * d * 3 * d * L
    out["gemm_o"] = 2 * T * d * d * L
    out["gemm_fc1"] = 2 * T * d * g.d_ffn * L
    out["gemm_fc2"] = 2 * T * g.d_ffn * d * L
    w = g.window_tokens if g.window_tokens else tc
    att = 0
    for b in range(batch):
        pos = 0
        while pos < tc:
            s = min(w, tc - pos)
            att += 4 * s * s * d
            pos += s
    out["attention"] = att * L
    if g.proj1_out:
        out["gemm_head"] = 2 * T * (d * g.proj1_out + g.proj1_out * g.proj2_out)
    if g.adapter_hidden:
        out["gemm_adapter"] = 2 * T * (g.proj2_out * 2 * g.adapter_hidden + g.adapter_hidden * g.adapter_out)
    return out


# ------------------------------------------------------------ clock sampler
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        def reader():
            for line in self.proc.stdout:
                self.rows.append([c.strip() for c in line.split(",")])
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        def f(x):
            try:
                return float(x)
            except ValueError:
                return None
        load = [r for r in self.rows if len(r) >= 9 and (f(r[3]) or 0) >= 50]
        use = load if load else [r for r in self.rows if len(r) >= 9]
        if not use:
            return None
        sm = [f(r[0]) for r in use if f(r[0]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in use:
            for i, nm in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": f(use[0][1]),
                "power_w_max": max((f(r[2]) or 0) for r in use), "samples": len(self.rows),
                "samples_under_load": len(load), "reasons": sorted(reasons)}


class NvmlClockSampler:
    """SM clock, power and clock-event (throttle) reasons every ~2 ms through
    NVML, the library nvidia-smi reads, from a thread in this process; only
    the samples taken between mark_begin() and mark_end() (the timed loop)
    count.  The nvidia-smi sampler above polls every 100 ms, which leaves a
    sub-second timed region with one or two samples; this one sees the 1 kW
    power cap engage a few steps into it."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown"}

    def __init__(self, gpu_uuid):
        self.uuid = gpu_uuid
        self.samples = []
        self.window = [None, None]
        self.stop_flag = False
        self.thread = None
        self.max_mhz = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return False

        def poll():
            while not self.stop_flag:
                try:
                    self.samples.append((time.perf_counter(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                         pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                         pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
                except Exception:
                    return
                time.sleep(0.002)
        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        return True

    def mark_begin(self):
        self.window[0] = time.perf_counter()

    def mark_end(self):
        self.window[1] = time.perf_counter()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=2)
        t0, t1 = self.window
        use = [x for x in self.samples if t0 is not None and t1 is not None and t0 <= x[0] <= t1]
        if not use:
            return None
        sm = [x[1] for x in use]
        reasons = set()
        for x in use:
            for bit, nm in self.REASONS.items():
                if x[3] & bit:
                    reasons.add(nm)
        q = max(len(sm) // 4, 1)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "sm_mhz_min": min(sm),
                "sm_mhz_by_quarter": [statistics.median(sm[i * q:(i + 1) * q]) for i in range(4) if sm[i * q:(i + 1) * q]],
                "power_w_max": max(x[2] for x in use), "samples": len(use), "samples_under_load": len(use),
                "reasons": sorted(reasons), "source": "NVML, every ~2 ms over the timed loop"}


def power_capped(clocks):
    """The timed loop ran under the power cap: the cap was active and held
    the SM clock well below its maximum.  The lowest sample decides, not the
    median: NVML's clock readings trail the steps (in a 20-step run the step
    times slow from the sixth step on while most samples still read the
    maximum)."""
    if not clocks or "sw_power_cap" not in clocks.get("reasons", []):
        return False
    lo, hi = clocks.get("sm_mhz_min", clocks.get("sm_mhz")), clocks.get("sm_max_mhz")
    return bool(lo and hi and lo < 0.95 * hi)


# ------------------------------------------------------------ multi-GPU logic
def rank_clip_seeds(w, rank):
    """PCM seeds of the clips rank `rank` processes: every rank runs its own
    replica of the workload (weak scaling), with disjoint seeds."""
    return [w.pcm_seed_base + rank * w.batch + b for b in range(w.batch)]


def reduce_max(value, device=None):
    """Maximum of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(audio_s_per_rank, world, ms_max):
    """Whole-job audio-seconds per second: all ranks' audio over the slowest rank's time."""
    return audio_s_per_rank * world / (ms_max / 1000.0)


# ------------------------------------------------------- committed ncu summaries
GEMM_SOURCES = ["speech_recognition_audio_b200/csrc/gemm.cuh", "speech_recognition_audio_b200/csrc/gemm2.cuh",
                "speech_recognition_audio_b200/csrc/common.cuh", "speech_recognition_audio_b200/csrc/gemm.cu"]


def gemm_source_hash():
    import hashlib
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_traffic(name):
    """DRAM bytes per launch recorded in profiles/<name>.md, or None when the
    summary is missing or the GEMM sources changed since the capture."""
    p = os.path.join(ROOT, "profiles", name + ".md")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- `"):
                k, _, v = line.strip()[3:].partition("`:")
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha256") != gemm_source_hash():
        return None
    try:
        return int(float(vals["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- oracle arm
def oracle_sample(w, g, W, pcm0):
    """One bounded sample of the workload on the CPU oracle: the log-mel of a
    whole clip and the full encoder path of its first attention window."""
    import oracle
    t0 = time.perf_counter()
    if g.window_tokens:
        out = oracle.encode_clip(pcm0, W, g, windows=[0])
        tokens = out.shape[0]
        t_chunk = oracle.token_count(g, g.chunk_frames * g.hop)
        audio_s = tokens / t_chunk * g.chunk_frames * g.hop / synth.SAMPLE_RATE
    else:
        out = oracle.encode_clip(pcm0, W, g)
        audio_s = pcm0.shape[0] / synth.SAMPLE_RATE
    return audio_s, time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("internal_api") in ("openblas", "mkl", "blis")]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


METRIC = "encoder audio-seconds/s (TFLOP/s beside it)"


def bench_config(w, T):
    return {"workload": w.name, "batch_per_gpu": w.batch, "seconds_per_clip": w.seconds, "tokens_per_gpu": T * w.batch,
            "l2": "flushed between timed steps (256 MB write)",
            "timing": "CUDA events per step, mean of steps, max over ranks"}


def run_reference(args, w, g, rank):
    if rank != 0:
        return 0
    W = synth.make_weights(g, w.weight_seed)
    pcm0 = synth.pcm_clip(w.n_samples, w.pcm_seed_base, w.speech_like)
    for _ in range(args.warmup):
        oracle_sample(w, g, W, pcm0)
    secs, audio = [], 0.0
    for _ in range(args.steps):
        a, t = oracle_sample(w, g, W, pcm0)
        secs.append(t)
        audio = a
    ms = 1000.0 * statistics.mean(secs)
    value = audio / (ms / 1000.0)
    sample = (f"first attention window ({audio:.0f} s of audio) of clip 0 plus that clip's full log-mel"
              if g.window_tokens else "one whole clip")
    import oracle
    T = oracle.token_count(g, w.n_samples)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "audio-s/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(bench_config(w, T), l2="n/a (host CPU)",
                           timing="host wall clock (perf_counter) per sample, mean of steps"),
            "cpu_baseline": {"value": value, "unit": "audio-s/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "audio-s/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- one op
def run_kernel(args, w, g):
    """Times one op of the workload's shape (warmup + steps launches)."""
    import torch
    import speech_recognition_audio_b200 as sra
    T = sra.tokens(g, w.n_samples) * w.batch
    d, f = g.d_model, g.d_ffn
    gen = torch.Generator().manual_seed(7)
    dev = torch.device("cuda", 0)
    if args.kernel == "log_mel":
        pcm = torch.from_numpy(synth.pcm_batch(w)).to(dev)
        run = lambda: sra.log_mel(pcm, g.n_mels)
        flops, unit = 4 * pcm.numel() + 4 * w.batch * g.n_mels * (w.n_samples // g.hop), "bytes"
    elif args.kernel == "layer_norm":
        x = (torch.randn(T, d, generator=gen) * 3).to(dev)
        gam, bet = torch.ones(d, device=dev), torch.zeros(d, device=dev)
        run = lambda: sra.layer_norm(x, gam, bet)
        flops, unit = T * d * (4 + 2), "bytes"
    elif args.kernel == "attention":
        import ctypes
        qkv = (torch.randn(T, 3 * d, generator=gen)).to(torch.bfloat16).to(dev)
        cu_h = sra.windows(g, w.n_samples, w.batch)
        cu = torch.tensor(cu_h, dtype=torch.int32, device=dev)
        att = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
        aws = torch.zeros(256, dtype=torch.uint8, device=dev)
        mx = max(b - a for a, b in zip(cu_h[:-1], cu_h[1:]))
        st = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
        run = lambda: sra.lib.asr_op_attention(ctypes.c_void_p(qkv.data_ptr()), ctypes.c_void_p(cu.data_ptr()),
                                               len(cu_h) - 1, mx, T, g.n_heads, ctypes.c_void_p(att.data_ptr()),
                                               ctypes.c_void_p(aws.data_ptr()), 256, st)
        wt = g.window_tokens if g.window_tokens else T // w.batch
        tc = T // w.batch
        flops = sum(4 * min(wt, tc - a) ** 2 * d for a in range(0, tc, wt)) * w.batch
        unit = "flop"
    else:
        N, K, epi = {"gemm_fc1": (f, d, sra.EPI_BF16_GELU), "gemm_fc2": (d, f, sra.EPI_F32_RESID),
                     "gemm_qkv": (3 * d, d, sra.EPI_BF16), "gemm_o": (d, d, sra.EPI_F32_RESID)}[args.kernel]
        x = (torch.randn(T, K, generator=gen) * 0.5).to(torch.bfloat16).to(dev)
        wt = (torch.randn(N, K, generator=gen) * 0.02).to(torch.bfloat16).to(dev)
        b = torch.zeros(N, device=dev)
        out = torch.zeros(T, N, device=dev) if epi == sra.EPI_F32_RESID else None
        run = lambda: sra.linear(x, wt, b, epi, out=out)
        flops, unit = 2 * T * N * K, "flop"
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s_.record()
    for _ in range(args.steps):
        run()
    e_.record()
    torch.cuda.synchronize()
    ms = s_.elapsed_time(e_) / args.steps
    print(json.dumps({"kernel": args.kernel, "workload": w.name, "ms_per_launch": ms, "work_per_launch": flops,
                      "unit": unit, "rate": flops / (ms / 1000.0)}), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="moss_16x30s", choices=list(synth.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=3)
    ap.add_argument("--kernel", default=None, choices=["gemm_fc1", "gemm_fc2", "gemm_qkv", "gemm_o", "log_mel", "layer_norm",
                                                       "attention"],
                    help="run one op of the workload's shape through the C ABI (for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    w = synth.WORKLOADS[args.workload]
    g = synth.GEOMETRIES[w.geometry]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, w, g, rank)
    if args.kernel:
        return run_kernel(args, w, g)

    import torch
    import torch.distributed as dist
    import speech_recognition_audio_b200 as sra

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    W = synth.make_weights(g, w.weight_seed)
    enc = sra.Encoder(g, {k: v.to(dev) for k, v in W.items()})
    del W
    # every rank processes its own replica of the workload (different seeds)
    pcm_np = np.stack([synth.pcm_clip(w.n_samples, sd, w.speech_like) for sd in rank_clip_seeds(w, rank)])
    pcm = torch.from_numpy(pcm_np).to(dev)
    T = enc.tokens(w.n_samples)
    out = torch.empty((w.batch, T, enc.d_out), dtype=torch.float32, device=dev)
    ws = enc.workspace(w.n_samples, w.batch)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        enc.forward(pcm, out=out, workspace=ws)
    enc.sync_status()

    gpu_id = local
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    nvml = NvmlClockSampler(gpu_id)
    nvml.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    nvml.mark_begin()
    for i in range(args.steps):
        flush.zero_()                      # evict L2 between steps (outside the events)
        starts[i].record(stream)
        enc.forward(pcm, out=out, workspace=ws)
        ends[i].record(stream)
    torch.cuda.synchronize()
    nvml.mark_end()
    barrier()
    clocks = nvml.stop() or sampler.stop()
    if clocks is not None and clocks.get("source"):
        sampler.stop()
    enc.sync_status()
    launches_per_step = sra.lib.asr_enc_last_launches(enc.handle)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = reduce_max(statistics.mean(step_ms), dev)

    audio_per_step = w.batch * w.seconds * world
    value = job_throughput(w.batch * w.seconds, world, ms)
    fl = flop_breakdown(g, w.n_samples, w.batch)
    flops = sum(fl.values())
    tflops = flops * world / (ms / 1000.0) / 1e12
    peaks, peak_kind = load_peaks()

    # ---- per-kernel timing (events around each launch), same workload
    enc_prof = {}
    sra.lib.asr_enc_profile(enc.handle, 1)
    import ctypes
    for _ in range(args.profile_steps):
        flush.zero_()
        enc.forward(pcm, out=out, workspace=ws)
        names = (ctypes.c_char_p * 32)()
        tms = (ctypes.c_double * 32)()
        cnt = (ctypes.c_int * 32)()
        k = sra.lib.asr_enc_profile_read(enc.handle, 32, names, tms, cnt)
        for i in range(k):
            nm = names[i].decode()
            a = enc_prof.setdefault(nm, [0.0, 0])
            a[0] += tms[i]
            a[1] += cnt[i]
    sra.lib.asr_enc_profile(enc.handle, 0)
    per_step = {k: v[0] / args.profile_steps for k, v in enc_prof.items()}
    launches_prof = {k: v[1] // args.profile_steps for k, v in enc_prof.items()}
    gemm_keys = [k for k in per_step if k.startswith("gemm")]
    gemm_ms = sum(per_step[k] for k in gemm_keys)
    gemm_flops = sum(fl.get(k, 0) for k in gemm_keys)
    # The denominator follows the clock regime the work ran in.  The timed
    # steps and the profiled ones after them run back to back; a few steps in,
    # the 1 kW power cap engages and holds the SM clock well below its
    # maximum (about 1650 against 1965 MHz), the regime of the sustained
    # measurement, whose figure is then the peak; without the cap, the burst
    # figure.  The fraction of the other figure is reported beside.
    peak_burst = peaks.get("bf16_tflops", peaks.get("bf16_tflops_sustained"))
    peak_sus = peaks.get("bf16_tflops_sustained", peak_burst)
    capped = power_capped(clocks)
    regime = "sustained" if capped else "burst"
    peak_t = peak_sus if capped else peak_burst
    # Dominant kernel: the largest GEMM stage of the step (one shape, one kernel).
    top = max(gemm_keys, key=lambda k: per_step[k]) if gemm_keys else None
    roofline = None
    if top:
        n_l = max(launches_prof[top], 1)
        avg_ms = per_step[top] / n_l
        per_launch = fl.get(top, 0) / n_l
        achieved = per_launch / (avg_ms / 1000.0) / 1e12 if avg_ms else None
        roofline = {"bound": "tensor", "kernel": f"tcgen05 GEMM, stage {top}", "achieved": achieved, "peak": peak_t,
                    "unit": "TFLOP/s", "frac": (achieved / peak_t) if achieved else None,
                    "traffic": profile_traffic(f"{top}_{w.name}"),
                    "flops_per_launch": per_launch, "avg_launch_ms": avg_ms, "launches_per_step": n_l,
                    "peak_kind": f"{peak_kind} {regime} bf16 (MEASURED_PEAKS.json; power-capped clocks: {capped})",
                    "frac_of_burst": (achieved / peak_burst) if achieved and peak_burst else None,
                    "frac_of_sustained": (achieved / peak_sus) if achieved and peak_sus else None}
    engine = {"achieved": gemm_flops / (gemm_ms / 1000.0) / 1e12 if gemm_ms else None, "unit": "TFLOP/s",
              "ms_per_step": gemm_ms, "share_of_step": gemm_ms / sum(per_step.values()) if per_step else None}
    mel_ms = per_step.get("log_mel")
    mel_bytes = 4 * w.batch * w.n_samples + 4 * w.batch * g.n_mels * (w.n_samples // g.hop)
    mel_roof = None
    if mel_ms:
        a = mel_bytes / (mel_ms / 1000.0) / 1e9
        mel_roof = {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": a / peaks["hbm_gbs"], "bytes": mel_bytes, "ms": mel_ms}
    kernels = {k: {"ms": round(per_step[k], 4), "launches": launches_prof[k],
                   "tflops": (fl[k] / (per_step[k] / 1000.0) / 1e12) if k in fl and per_step[k] else None}
               for k in sorted(per_step, key=lambda x: -per_step[x])}

    # ---- end to end through the host-buffer ABI call (pinned host memory)
    pcm_host = torch.from_numpy(pcm_np).pin_memory()
    out_host = torch.empty((w.batch, T, enc.d_out), dtype=torch.float32).pin_memory()
    for _ in range(2):
        enc.forward_host(pcm_host, out_host=out_host, workspace=ws)
    e2e_steps = max(3, min(args.steps, 10))
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    barrier()
    for i in range(e2e_steps):
        flush.zero_()
        e_s[i].record(stream)
        enc.forward_host(pcm_host, out_host=out_host, workspace=ws)
        e_e[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(statistics.mean(s.elapsed_time(e) for s, e in zip(e_s, e_e)), dev)
    e2e = {"value": audio_per_step / (e2e_ms / 1000.0), "unit": "audio-s/s",
           "h2d_bytes_per_step": int(pcm_host.numel() * 4), "d2h_bytes_per_step": int(out_host.numel() * 4),
           "ms_per_step": e2e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        Wc = synth.make_weights(g, w.weight_seed)
        a, t = oracle_sample(w, g, Wc, pcm_np[0])
        sample = (f"first attention window ({a:.0f} s of audio) of clip 0 plus its full log-mel, one run"
                  if g.window_tokens else "one whole clip, one run")
        cpu = {"value": a / t, "unit": "audio-s/s", "cores": blas_threads(), "kind": "oracle", "sample": sample,
               "seconds": t}

    if world > 1:
        if dist.is_initialized():
            dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC,
        "value": value, "unit": "audio-s/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded sines + noise, random-init N(0,0.02) bf16 weights)",
        "config": bench_config(w, T),
        "tflops": tflops, "tflops_frac_of_measured_peak": tflops / peak_t, "tflops_peak_kind": regime,
        "tflops_frac_of_burst": tflops / peak_burst, "tflops_frac_of_sustained": tflops / peak_sus,
        "tflops_frac_of_spec_2250": tflops / 2250.0,
        "flops_per_step": flops,
        "e2e": e2e,
        "gpu_launches": int(launches_per_step * args.steps),
        "roofline": roofline,
        "gemm_engine": engine,
        "mel_roofline": mel_roof,
        "kernels_ms_per_step": kernels,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "step_ms_min_max": [min(step_ms), max(step_ms)],
        "step_ms": [round(t, 3) for t in step_ms],  # in timed order (the steps run back to back)
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
