"""Seeded synthetic inputs: random-init weights of the decoder architecture and latents.

This module draws numbers and names tensors; it holds none of the decoder's arithmetic
(no weight norm, no filters, no convolutions).  Both the CUDA library's tests/bench and the
CPU oracle consume what it returns, so the two sides see identical inputs.

Recipe (the five workloads of the decode benchmark; the pages print no numeric example):
  * latents ~ N(0, 1), fp32, [B, 32, N];
  * every weight-normed kernel: v ~ N(0, 1), g = 1;
  * every bias ~ N(0, 0.01^2);
  * every SnakeBeta alpha, beta = 1 + U(-0.2, 0.2);
  * dec_in_proj.weight ~ N(0, 1) / sqrt(32) (plain 1x1 conv, not weight-normed);
  * the Kaiser-sinc filters are not drawn: each side builds them from their formula;
  * denormalised workload: latents_mean_c ~ U(-0.5, 0.5), latents_std_c ~ U(0.5, 1.5).
Tensors are drawn in one canonical order (create order, stage-major) from a single
numpy PCG64 generator seeded per workload.

Weight names follow the released checkpoint keys the MLX page's ``decode`` reads
(``dec_in_proj.*``, ``decoder.conv_pre.*``, ``decoder.ups.{i}.0.*``,
``decoder.resblocks.{3i+j}.*``, ``decoder.activation_post.act.*``, ``decoder.conv_post.*``);
inside a residual block the sub-keys ``convs1.{m}``, ``convs2.{m}`` and
``activations.{a}.act.{alpha,beta}`` (a = 2m before convs1.m, a = 2m+1 before convs2.m)
are this library's naming, since the pages do not print the block body.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from functools import lru_cache

import numpy as np


@dataclass(frozen=True)
class Arch:
    """Decoder architecture; defaults are the diffusers constructor defaults."""

    latent_channels: int = 32
    latent_dim: int = 2048
    decoder_dim: int = 1024
    rates: tuple = (5, 5, 2, 2, 2, 2, 2)
    kernels: tuple = (9, 9, 4, 4, 4, 4, 4)
    rb_kernels: tuple = (3, 7, 11)
    rb_dilations: tuple = ((1, 3, 5), (1, 3, 5), (1, 3, 5))
    conv_pre_kernel: int = 7
    conv_post_kernel: int = 7
    latents_mean: tuple | None = None
    latents_std: tuple | None = None

    @property
    def n_stages(self) -> int:
        return len(self.rates)

    @property
    def hop(self) -> int:
        return int(np.prod(self.rates))

    def stage_channels(self, i: int) -> int:
        """Channels after upsampling stage i (input of AMP stage i)."""
        return self.decoder_dim >> (i + 1)

    def stage_length(self, i: int, N: int) -> int:
        return N * int(np.prod(self.rates[: i + 1]))


def weight_specs(arch: Arch):
    """Canonical (name, shape, kind) list; kind in {v, g, bias, snake, in_w}."""
    specs = [
        ("dec_in_proj.weight", (arch.latent_dim, arch.latent_channels, 1), "in_w"),
        ("dec_in_proj.bias", (arch.latent_dim,), "bias"),
    ]
    D, C0 = arch.latent_dim, arch.decoder_dim
    kp = arch.conv_pre_kernel
    specs += [
        ("decoder.conv_pre.weight_v", (C0, D, kp), "v"),
        ("decoder.conv_pre.weight_g", (C0, 1, 1), "g"),
        ("decoder.conv_pre.bias", (C0,), "bias"),
    ]
    nrb = len(arch.rb_kernels)
    C = C0
    for i, (r, K) in enumerate(zip(arch.rates, arch.kernels)):
        Co = C // 2
        p = f"decoder.ups.{i}.0"
        specs += [
            (f"{p}.weight_v", (C, Co, K), "v"),
            (f"{p}.weight_g", (C, 1, 1), "g"),
            (f"{p}.bias", (Co,), "bias"),
        ]
        for j, k in enumerate(arch.rb_kernels):
            rb = f"decoder.resblocks.{i * nrb + j}"
            for m in range(len(arch.rb_dilations[j])):
                for conv in ("convs1", "convs2"):
                    q = f"{rb}.{conv}.{m}"
                    specs += [
                        (f"{q}.weight_v", (Co, Co, k), "v"),
                        (f"{q}.weight_g", (Co, 1, 1), "g"),
                        (f"{q}.bias", (Co,), "bias"),
                    ]
            for a in range(2 * len(arch.rb_dilations[j])):
                specs += [
                    (f"{rb}.activations.{a}.act.alpha", (Co,), "snake"),
                    (f"{rb}.activations.{a}.act.beta", (Co,), "snake"),
                ]
        C = Co
    specs += [
        ("decoder.activation_post.act.alpha", (C,), "snake"),
        ("decoder.activation_post.act.beta", (C,), "snake"),
        ("decoder.conv_post.weight_v", (1, C, arch.conv_post_kernel), "v"),
        ("decoder.conv_post.weight_g", (1, 1, 1), "g"),
        ("decoder.conv_post.bias", (1,), "bias"),
    ]
    return specs


def make_weights(arch: Arch, seed: int) -> dict:
    """Random-init weights drawn in canonical order from PCG64(seed)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    for name, shape, kind in weight_specs(arch):
        n = int(np.prod(shape))
        if kind == "v":
            a = rng.standard_normal(n, dtype=np.float32)
        elif kind == "g":
            a = np.ones(n, dtype=np.float32)
        elif kind == "bias":
            a = (0.01 * rng.standard_normal(n, dtype=np.float64)).astype(np.float32)
        elif kind == "snake":
            a = (1.0 + rng.uniform(-0.2, 0.2, n)).astype(np.float32)
        elif kind == "in_w":
            a = (rng.standard_normal(n, dtype=np.float64) / math.sqrt(shape[1])).astype(np.float32)
        else:  # pragma: no cover
            raise ValueError(kind)
        out[name] = a.reshape(shape)
    return out


def make_latents(B: int, N: int, channels: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed + 0x5EED))
    return rng.standard_normal((B, channels, N), dtype=np.float32)


def make_stage_input(B: int, C: int, L: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed + 0xA3F))
    return rng.standard_normal((B, C, L), dtype=np.float32)


def make_denorm(channels: int, seed: int):
    rng = np.random.Generator(np.random.PCG64(seed + 0xD0E))
    mean = rng.uniform(-0.5, 0.5, channels).astype(np.float32)
    std = rng.uniform(0.5, 1.5, channels).astype(np.float32)
    return tuple(float(x) for x in mean), tuple(float(x) for x in std)


@dataclass(frozen=True)
class Workload:
    """One of the five benchmark workloads."""

    name: str
    kind: str  # "decode" or "amp_stage"
    B: int
    N: int  # latent frames (decode) or samples (amp_stage)
    seed: int
    stage: int = -1
    channels: int = 0
    tensor_cores: bool = False
    denorm: bool = False
    note: str = field(default="")


WORKLOADS = {
    0: Workload("decode B=1 N=4", "decode", 1, 4, 0),
    1: Workload("AMP stage 0 x[2,512,2000]", "amp_stage", 2, 2000, 1, stage=0, channels=512),
    2: Workload("decode B=2 N=40 (1 s stereo)", "decode", 2, 40, 2),
    3: Workload("decode B=2 N=400 (10 s stereo)", "decode", 2, 400, 3, tensor_cores=True),
    4: Workload("decode B=16 N=800 (20 s, denormalised)", "decode", 16, 800, 4,
                tensor_cores=True, denorm=True),
}


def workload_arch(w: Workload) -> Arch:
    if w.denorm:
        mean, std = make_denorm(32, w.seed)
        return Arch(latents_mean=mean, latents_std=std)
    return Arch()


@lru_cache(maxsize=4)
def workload_weights(seed: int, arch: Arch = Arch()) -> dict:
    return make_weights(arch, seed)


def workload_inputs(index: int):
    """(arch, weights, input array) of workload `index`."""
    w = WORKLOADS[index]
    arch = workload_arch(w)
    weights = workload_weights(w.seed, Arch())
    if w.kind == "decode":
        x = make_latents(w.B, w.N, arch.latent_channels, w.seed)
    else:
        x = make_stage_input(w.B, w.channels, w.N, w.seed)
    return arch, weights, x
