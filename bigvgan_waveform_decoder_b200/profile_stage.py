"""Time one AMP stage (or one full decode) through the C ABI; the driver for ncu captures.

    python -m bigvgan_waveform_decoder_b200.profile_stage --stage 1 --B 2 --L 10000 [--iters 3]
    python -m bigvgan_waveform_decoder_b200.profile_stage --decode --B 2 --N 400

Prints one line per call with its CUDA-event time, and the per-segment times of the last
decode.  Random-init weights (seed 3) and N(0,1) inputs, as in the benchmark workloads.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import binding as Bd
from . import perfmodel as PM
from . import synthetic as S


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--stage", type=int, default=1)
    ap.add_argument("--B", type=int, default=2)
    ap.add_argument("--L", type=int, default=10000)
    ap.add_argument("--N", type=int, default=400)
    ap.add_argument("--decode", action="store_true")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=1)
    ap.add_argument("--precision", choices=["bf16x3", "fp32"], default="bf16x3")
    a = ap.parse_args()
    prec = Bd.MH3A_BF16X3 if a.precision == "bf16x3" else Bd.MH3A_FP32
    arch = S.Arch()
    w = S.workload_weights(3, arch)
    dev = torch.device("cuda:0")
    if a.decode:
        d = Bd.Decoder(arch, w, precision=prec, max_batch=a.B, max_frames=a.N)
        x = torch.from_numpy(S.make_latents(a.B, a.N, 32, 3)).to(dev)
        run = lambda: d.decode(x)  # noqa: E731
    else:
        C = arch.stage_channels(a.stage)
        L_cap = -(-a.L // int(np.prod(arch.rates[: a.stage + 1])))
        d = Bd.Decoder(arch, w, precision=prec, max_batch=a.B, max_frames=L_cap)
        x = torch.from_numpy(S.make_stage_input(a.B, C, a.L, 3)).to(dev)
        run = lambda: d.amp_stage(x, a.stage)  # noqa: E731
    d.set_profiling(a.decode)
    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(a.iters):
        e0.record()
        run()
        e1.record()
        e1.synchronize()
        print(f"call {i}: {e0.elapsed_time(e1):.3f} ms")
    d.check_device_error()
    if a.decode:
        segs = PM.segments(arch, a.B, a.N)
        print(json.dumps({s.name: round(t, 4) for s, t in zip(segs, d.segment_times())}))
    d.close()


if __name__ == "__main__":
    main()
