#!/usr/bin/env python
"""Throughput of the BigVGAN waveform decode on B200: decoded audio-seconds per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one decode of the 10 s stereo workload (B=2 batch items, N=400 latents -> 2 x
320000 samples at 32 kHz, random-init weights, seeded N(0,1) latents) through the C ABI, with
the latents already in HBM.  Audio-seconds count every batch item: B * N / 40 per step.

Multi-GPU (torchrun, one process per GPU): independent replicas, each rank decoding its own
batch with no collective on the data path ("scaling": "weak"); ranks meet only at the barriers
around the timed region and in the max-over-ranks reduction of the timings.

Timing: W untimed warm-up decodes, then K decodes, each bracketed by CUDA events on the
launching stream; a 256 MiB buffer (> 126 MB L2) is rewritten between steps outside the events,
so every step starts with a cold L2.  `ms_per_step` is the median step (the mean is reported
beside it).  GPU clocks are sampled with nvidia-smi during the timed region.  The timed decodes
carry no other events: the per-launch kernel times of the dominant AMP stage (the roofline) and
the per-segment table come from untimed decodes afterwards, each with its own events.  `e2e`
repeats the measurement through mh3a_decode_host with pinned host buffers: the host->device copy
of the latents and the waveform's transfer to host memory are inside the timing (with a pinned
output buffer the decode's last kernel stores the waveform into host memory over the bus, so
`d2h_bytes_per_step` bytes cross it during that kernel rather than in a copy after it).

Two more workloads are reported as extra keys (the headline stays the 10 s stereo decode): the
single AMP stage x [2, 512, 2000] through mh3a_amp_stage (`amp_stage`), and the batched 20 s
decode B=16, N=800 with per-channel latent denormalisation (`batched_decode`).

`--impl reference` times the fp64 CPU oracle (the correctness reference) on the host cores
on a bounded sample of the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decoded audio-seconds/sec at 32 kHz on 1 B200; % of roofline per stage"

# Tile shape <MT, NT, KGT, EW, R> of the persistent GEMM per AMP width (as dispatched by the
# library), for labelling the roofline's kernel.
GEMM_TILE = {512: "1, 256, 4, 8, 1", 256: "1, 256, 4, 8, 1", 128: "2, 128, 4, 8, 1",
             64: "2, 64, 4, 16, 1", 32: "2, 32, 4, 8, 1", 16: "2, 16, 2, 8, 1", 8: "4, 16, 1, 16, 1"}
# DRAM bytes (read + write) per launch of that GEMM kernel on this workload, keyed by (channels,
# B * N), from one ncu capture (profiles/k_gemm_ps_stage1_B2_L10000.md); null when unmeasured
# or when the kernel changed after the capture.
GEMM_TRAFFIC = {(256, 800): 110.4e6}
GEMM_TRAFFIC_SRC = "profiles/k_gemm_ps_stage1_B2_L10000.md"
UNIT = "audio-s/s"
WORKLOAD = 3
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--precision", choices=["bf16x3", "fp32"], default="bf16x3")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every decode directly instead of replaying its CUDA graph")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the single-stage and batched-decode figures")
    ap.add_argument("--ref-sample-frames", type=int, default=200,
                    help="latent frames of one batch item per reference-arm step; the oracle's "
                         "fixed cost per batch item (its weight-norm folds) stays near 5 percent "
                         "of a step at 200 frames")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: the replicas' job ends when the last one does."""
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, audio_s_per_step: float, max_ms: float) -> float:
    """Whole-job audio-seconds per second: every rank decodes its own batch in every step."""
    return world * steps * audio_s_per_step / (max_ms / 1e3)


class Clocks:
    """nvidia-smi sampler of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(rows), "reasons": sorted(reasons)}


def cpu_baseline() -> dict:
    """The oracle as it stands, on the whole workload: both items, all 400 latent frames."""
    import oracle
    from bigvgan_waveform_decoder_b200 import synthetic as S

    arch, w, z = S.workload_inputs(WORKLOAD)
    B, _, N = z.shape
    t0 = time.perf_counter()
    oracle.decode(arch, w, z)
    dt = time.perf_counter() - t0
    audio_s = B * N / 40.0
    return {"value": audio_s / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"B={B} N={N} in full ({audio_s:g} audio-s), fp64 oracle, one decode, "
                      f"{dt:.1f} s wall"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from bigvgan_waveform_decoder_b200 import synthetic as S

    arch, w, z = S.workload_inputs(WORKLOAD)
    zs = z[:1, :, :args.ref_sample_frames].copy()
    audio_s = args.ref_sample_frames / 40.0
    for _ in range(args.warmup):
        oracle.decode(arch, w, zs)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.decode(arch, w, zs)
        times.append(time.perf_counter() - t0)
    med = statistics.median(times)
    value = audio_s / med
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * med,
        "ms_per_step_mean": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "decode B=2 N=400 (10 s stereo), sampled: 1 item x "
                               f"{args.ref_sample_frames} frames per step", "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"1 batch item x {args.ref_sample_frames} latent frames per "
                                   "step of the B=2 N=400 workload"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def timed_calls(fn, flush, steps: int, stream) -> list[float]:
    """CUDA-event time (ms) of each of `steps` calls of fn on `stream`, L2 flushed before each
    call outside its events."""
    import torch

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = []
    for k in range(steps):
        flush.fill_(float(k))
        ev0.record(stream)
        fn()
        ev1.record(stream)
        ev1.synchronize()
        out.append(ev0.elapsed_time(ev1))
    return out


def extra_amp_stage(Bd, PM, peaks, p_tc, p_fp32, flush, stream, dev, steps: int) -> dict:
    """The single-AMP-stage workload: x [2, 512, 2000] ~ N(0,1) and weights of seed 1, through
    mh3a_amp_stage (the kernels the decode runs for its first AMP stage)."""
    import torch
    from bigvgan_waveform_decoder_b200 import synthetic as S

    arch, w, xn = S.workload_inputs(1)
    B, C, L = xn.shape
    stage = S.WORKLOADS[1].stage
    dec = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=B,
                     max_frames=-(-L // (arch.rates[0])))
    x = torch.from_numpy(xn).to(dev)
    out = torch.empty_like(x)
    for _ in range(3):
        dec.amp_stage(x, stage, out)
    torch.cuda.synchronize()
    ms = timed_calls(lambda: dec.amp_stage(x, stage, out), flush, steps, stream)
    dec.check_device_error()
    dec.close()
    # x [2, 512, 2000] is exactly the decode's amp0 segment at B = 2, N = 400
    seg = [sg for sg in PM.segments(arch, B, L // arch.rates[0]) if sg.name == "amp0"][0]
    seg.tensor = True
    roof = PM.roofline_time(seg, p_tc, p_fp32, peaks["hbm_gbs"]) * 1e3
    med = statistics.median(ms)
    return {"workload": f"AMP stage {stage}, x [{B}, {C}, {L}] (seed {S.WORKLOADS[1].seed})",
            "ms": med, "conv_tflops": seg.conv_flops / (med * 1e-3) / 1e12, "roof_ms": roof,
            "frac": roof / med, "calls": steps, "statistic": "median call",
            "l2": "flushed between calls"}


PROFILER_ENV = ("NV_NSIGHT_INJECTION_TRANSPORT_TYPE", "NV_COMPUTE_PROFILER_PERFWORKS_DIR",
                "CUDA_INJECTION64_PATH")


def graphs_allowed() -> bool:
    """False when a profiler has injected itself into the CUDA runtime (Nsight Compute sets the
    first two variables in the program it starts; CUDA_INJECTION64_PATH is the runtime's own
    injection hook).  Under ncu, the replay of a captured decode -- kernels chained by
    programmatic dependent launch -- failed to launch, so a profiled run launches every decode
    directly: the same kernels, arguments and order."""
    return not any(os.environ.get(k) for k in PROFILER_ENV)


def extra_batched(arch_w, Bd, flush, stream, dev, steps: int) -> dict:
    """The batched 20 s decode: B=16, N=800, per-channel latent denormalisation, seed 4."""
    import torch
    from bigvgan_waveform_decoder_b200 import synthetic as S

    arch, w, z = arch_w
    B, _, N = z.shape
    dec = Bd.Decoder(arch, w, precision=Bd.MH3A_BF16X3, max_batch=B, max_frames=N)
    dec.set_graph_mode(graphs_allowed())
    x = torch.from_numpy(z).to(dev)
    out = torch.empty((B, 1, dec.hop * N), device=dev, dtype=torch.float32)
    for _ in range(2):
        dec.decode(x, out)
    torch.cuda.synchronize()
    ms = timed_calls(lambda: dec.decode(x, out), flush, steps, stream)
    dec.check_device_error()
    dec.close()
    med = statistics.median(ms)
    return {"workload": f"decode B={B} N={N} (20 s, denormalised latents, seed 4)",
            "value": B * N / 40.0 / (med * 1e-3), "unit": UNIT, "ms_per_step": med, "steps": steps,
            "l2": "inputs and every stage tensor larger than L2; flushed between steps"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from bigvgan_waveform_decoder_b200 import binding as Bd
    from bigvgan_waveform_decoder_b200 import perfmodel as PM
    from bigvgan_waveform_decoder_b200 import synthetic as S

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    wl = S.WORKLOADS[WORKLOAD]
    B, N = wl.B, wl.N
    arch, w, _ = S.workload_inputs(WORKLOAD)
    z = S.make_latents(B, N, arch.latent_channels, wl.seed + 1000 * rank)
    precision = Bd.MH3A_BF16X3 if args.precision == "bf16x3" else Bd.MH3A_FP32
    use_graph = not args.no_graph and graphs_allowed()
    dec = Bd.Decoder(arch, w, precision=precision, max_batch=B, max_frames=N)
    x = torch.from_numpy(z).to(dev)
    out = torch.empty((B, 1, dec.hop * N), device=dev, dtype=torch.float32)
    flush = torch.empty(FLUSH_BYTES // 4, device=dev, dtype=torch.float32)
    # A stream of our own: the legacy default stream cannot be captured, so decodes on it never
    # replay a graph.  torch's fills of the L2 flush buffer run on it too.
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    if use_graph:
        dec.set_graph_mode(True)   # the second warm-up decode captures, later ones replay
    audio_s = B * N / 40.0
    n_stages = len(arch.rates)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        flush.fill_(1.0)
        dec.decode(x, out)
    barrier()
    torch.cuda.synchronize()

    # ---- timed region: K decodes, nothing but the step events on the stream
    clocks = Clocks(local)
    clocks.start()
    launches0 = dec.launch_count()
    step_ms = timed_calls(lambda: dec.decode(x, out), flush, args.steps, stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    launches = dec.launch_count() - launches0
    clk = clocks.stop()
    dec.check_device_error()

    med_ms = max_over_ranks(statistics.median(step_ms), world, dev)
    value = job_throughput(world, 1, audio_s, med_ms)

    # ---- untimed decodes with events: the per-segment table, then per-launch kernel times of
    # the most expensive AMP stage (each event between two kernels costs a little overlap)
    n_seg = 5
    seg_sum = None
    dec.set_profiling(True)
    for k in range(n_seg):
        flush.fill_(float(k))
        dec.decode(x, out)
        seg = dec.segment_times()
        seg_sum = seg if seg_sum is None else [a + b for a, b in zip(seg_sum, seg)]
    dec.set_profiling(False)
    seg_ms = [t / n_seg for t in seg_sum]
    amp_ms = [seg_ms[3 + 2 * i] for i in range(n_stages)]
    kstage = max(range(n_stages), key=lambda i: amp_ms[i])
    kern = [0.0, 0.0]
    n_kern = 5
    if dec.stage_uses_tensor_cores(kstage):
        dec.set_kernel_profiling(kstage)
        for k in range(n_kern):
            flush.fill_(float(k))
            dec.decode(x, out)
            a_ms, g_ms = dec.stage_kernel_times(kstage)
            kern[0] += a_ms
            kern[1] += g_ms
        dec.set_kernel_profiling(-1)
    torch.cuda.synchronize()

    # ---- end to end through the host-buffer entry point (pinned host memory)
    zp = torch.from_numpy(z).pin_memory()
    yp = torch.empty((B, 1, dec.hop * N), dtype=torch.float32).pin_memory()
    for _ in range(args.warmup):
        dec.decode_host(zp, yp)
    barrier()
    e2e_ms = timed_calls(lambda: dec.decode_host(zp, yp), flush, args.steps, stream)
    e2e_value = job_throughput(world, 1, audio_s, max_over_ranks(statistics.median(e2e_ms), world, dev))

    # ---- per-segment roofline
    segs = PM.segments(arch, B, N)
    for i, sgm in enumerate(segs):
        sgm.tensor = dec.segment_uses_tensor_cores(i)
    peaks = PM.measured_peaks()
    p_fp32 = PM.fp32_peak_tflops(peaks["sm_max_mhz"])
    p_tc = peaks["bf16_tflops"] / 3.0
    stages = []
    for sgm, ms in zip(segs, seg_ms):
        roof = PM.roofline_time(sgm, p_tc, p_fp32, peaks["hbm_gbs"]) * 1e3
        stages.append({"segment": sgm.name, "ms": round(ms, 4), "roof_ms": round(roof, 4),
                       "frac": round(roof / ms, 4) if ms > 0 else None,
                       "tflops": round(sgm.flops / (ms * 1e-3) / 1e12, 2) if ms > 0 else None,
                       "pipe": "tensor" if sgm.tensor else "fp32"})
    sgm = segs[3 + 2 * kstage]
    C = arch.decoder_dim >> (kstage + 1)
    roofline = None
    roofline_act = None
    if kern[1] > 0:
        # the stage's GEMM kernel alone: algorithmic flops of one launch (3 residual blocks)
        # over its average launch duration
        gemm_launch_ms = kern[1] / n_kern / 6
        act_launch_ms = kern[0] / n_kern / 6
        achieved = sgm.conv_flops / 6 / (gemm_launch_ms * 1e-3) / 1e12
        traffic = GEMM_TRAFFIC.get((C, B * N))
        roofline = {"bound": "tensor", "achieved": achieved, "peak": p_tc, "unit": "TFLOP/s",
                    "frac": achieved / p_tc, "traffic": traffic,
                    "traffic_source": (f"{GEMM_TRAFFIC_SRC} (an earlier ncu capture of the same kernel "
                                       "build, not measured in this run)") if traffic else None,
                    "kernel": f"k_gemm_ps<{GEMM_TILE.get(C, '?')}> ({sgm.name} conv, 3 residual blocks per launch)",
                    "launch_ms": gemm_launch_ms, "launches_per_step": 6,
                    "flops_per_launch": sgm.conv_flops / 6,
                    "activation_kernel_ms_per_launch": act_launch_ms,
                    "timing": f"CUDA events around each launch, {n_kern} untimed decodes after the timed region",
                    "peak_basis": f"bf16 burst {peaks['bf16_tflops']} ({peaks['source']}) / 3 "
                                  "bf16 products per fp32 product"}
        # the same stage's activation kernel, the other half of every AMP layer: fp32 work
        # (56 flops per output; the 2 sines per output run on the SFU and are not counted)
        act_flops = sgm.act_flops / 6
        act_achieved = act_flops / (act_launch_ms * 1e-3) / 1e12
        roofline_act = {"bound": "alu", "achieved": act_achieved, "peak": p_fp32, "unit": "TFLOP/s",
                        "frac": act_achieved / p_fp32, "traffic": None,
                        "kernel": f"k_act_split ({sgm.name}, 3 residual blocks per launch)",
                        "launch_ms": act_launch_ms, "launches_per_step": 6,
                        "flops_per_launch": act_flops,
                        "peak_basis": f"148 SM x 128 fp32 lanes x 2 x {peaks['sm_max_mhz']} MHz"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": med_ms,
        "ms_per_step_mean": sum(step_ms) / len(step_ms), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16x3" if precision == Bd.MH3A_BF16X3 else "f32",
        "data": "synthetic",
        "config": {"workload": f"decode B={B} N={N} (10 s stereo, 2 x 320000 samples) per GPU",
                   "global_batch": B * world, "latent_frames": N, "replicas": world,
                   "weights": "random init, seed 3", "l2": "flushed between steps (256 MiB write)",
                   "statistic": "median step", "cuda_graph": use_graph},
        "roofline": roofline,
        "roofline_activation": roofline_act,
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": int(z.nbytes), "d2h_bytes_per_step": int(yp.numel() * 4),
                "d2h": "the last kernel stores the waveform into the pinned host buffer"},
        "gpu_launches": launches,
        "clocks": clk,
        "stages": stages,
        "stages_basis": f"segment events on {n_seg} untimed decodes after the timed region",
        "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16x3_tflops": p_tc, "fp32_tflops": p_fp32,
                  "source": peaks["source"]},
    }
    if rank == 0 and world == 1 and not args.no_extra:
        line["amp_stage"] = extra_amp_stage(Bd, PM, peaks, p_tc, p_fp32, flush, stream, dev,
                                            max(args.steps, 10))
    dec.close()
    if rank == 0 and world == 1 and not args.no_extra:
        line["batched_decode"] = extra_batched(S.workload_inputs(4), Bd, flush, stream, dev, 5)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
