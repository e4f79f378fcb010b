"""ctypes front end of the fp64 CPU oracle (TEST INFRASTRUCTURE ONLY).

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of bench.py
may import this package.  The product path (``bigvgan_waveform_decoder_b200``) never imports
it and shares no code with it.

The oracle follows the method as two web pages state it:
  * diffusers "AutoencoderKLMiniMaxH3Audio" API page (constructor defaults, ``decode``);
  * FastVideo "minimax_h3_audio_vae" MLX page (``MLXMiniMaxH3AudioVAE.decode``,
    ``kaiser_sinc_filter1d``).
Every function is pinned in tests/test_oracle_*.py against closed forms, brute-force
definitions or independent library routines (numpy, scipy, torch CPU fp64).
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, field

import numpy as np

from . import build as _build

_LIB = None


class _Tensor(C.Structure):
    _fields_ = [
        ("name", C.c_char_p),
        ("data", C.POINTER(C.c_float)),
        ("ndim", C.c_int),
        ("shape", C.c_longlong * 3),
    ]


class _Config(C.Structure):
    _fields_ = [
        ("latent_channels", C.c_int),
        ("latent_dim", C.c_int),
        ("decoder_dim", C.c_int),
        ("n_stages", C.c_int),
        ("rates", C.c_int * 8),
        ("kernels", C.c_int * 8),
        ("n_resblocks", C.c_int),
        ("rb_kernels", C.c_int * 4),
        ("n_dilations", C.c_int),
        ("rb_dilations", (C.c_int * 4) * 4),
        ("clamp", C.c_int),
        ("latents_mean", C.POINTER(C.c_float)),
        ("latents_std", C.POINTER(C.c_float)),
    ]


_D = C.POINTER(C.c_double)
_F = C.POINTER(C.c_float)


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = C.CDLL(path)
        L.orc_bessel_i0.restype = C.c_double
        L.orc_bessel_i0.argtypes = [C.c_double]
        L.orc_kaiser_sinc_filter.argtypes = [C.c_double, C.c_double, C.c_int, _D, _D, _D]
        L.orc_weight_norm.argtypes = [_F, _F, C.c_longlong, C.c_longlong, _D]
        L.orc_conv1d.argtypes = [_D, C.c_int, C.c_int, _D, C.c_int, C.c_int, _D, C.c_int,
                                 C.c_int, C.c_int, _D, C.c_int]
        L.orc_conv_transpose1d.argtypes = [_D, C.c_int, C.c_int, _D, C.c_int, C.c_int, _D,
                                           C.c_int, C.c_int, _D, C.c_int]
        L.orc_snake_beta.argtypes = [_D, C.c_longlong, C.c_double, C.c_double, _D]
        L.orc_upsample2.argtypes = [_D, C.c_int, _D, C.c_int, _D]
        L.orc_downsample2.argtypes = [_D, C.c_int, _D, C.c_int, _D]
        L.orc_activation1d.argtypes = [_D, C.c_int, C.c_double, C.c_double, _D, C.c_int, _D]
        L.orc_num_threads.argtypes = []
        L.orc_num_threads.restype = C.c_int
        L.orc_default_config.argtypes = [C.POINTER(_Config)]
        L.orc_decode.argtypes = [C.POINTER(_Config), C.POINTER(_Tensor), C.c_int, _F, C.c_int,
                                 C.c_int, _D]
        L.orc_decode.restype = C.c_int
        L.orc_amp_stage.argtypes = [C.POINTER(_Config), C.POINTER(_Tensor), C.c_int, C.c_int, _F,
                                    C.c_int, C.c_int, _D]
        L.orc_amp_stage.restype = C.c_int
        L.orc_amp_stage_f64.argtypes = [C.POINTER(_Config), C.POINTER(_Tensor), C.c_int, C.c_int,
                                        _D, C.c_int, C.c_int, _D]
        L.orc_amp_stage_f64.restype = C.c_int
        _LIB = L
    return _LIB


def _dp(a: np.ndarray):
    return a.ctypes.data_as(_D)


def _fp(a: np.ndarray):
    return a.ctypes.data_as(_F)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


# --------------------------------------------------------------------------------------------
# primitives
# --------------------------------------------------------------------------------------------

def bessel_i0(x: float) -> float:
    return lib().orc_bessel_i0(float(x))


def kaiser_sinc_filter(cutoff: float, half_width: float, K: int):
    """Return (taps fp64 [K], attenuation, beta)."""
    taps = np.zeros(K, dtype=np.float64)
    A = C.c_double()
    b = C.c_double()
    lib().orc_kaiser_sinc_filter(cutoff, half_width, K, _dp(taps), C.byref(A), C.byref(b))
    return taps, A.value, b.value


def weight_norm(v: np.ndarray, g: np.ndarray) -> np.ndarray:
    v = _f32(v)
    g = _f32(g).reshape(-1)
    out = np.zeros(v.shape, dtype=np.float64)
    lib().orc_weight_norm(_fp(v), _fp(g), v.shape[0], v.size // v.shape[0], _dp(out))
    return out


def conv1d(x, w, bias=None, stride=1, pad=0, dil=1) -> np.ndarray:
    x = _f64(x)
    w = _f64(w)
    Cin, Lin = x.shape
    Cout, Cin2, K = w.shape
    assert Cin2 == Cin
    Lout = (Lin + 2 * pad - dil * (K - 1) - 1) // stride + 1
    y = np.zeros((Cout, Lout), dtype=np.float64)
    b = _f64(bias) if bias is not None else None
    lib().orc_conv1d(_dp(x), Cin, Lin, _dp(w), Cout, K, _dp(b) if b is not None else None,
                     stride, pad, dil, _dp(y), Lout)
    return y


def conv_transpose1d(x, w, bias=None, stride=1, pad=0) -> np.ndarray:
    x = _f64(x)
    w = _f64(w)
    Cin, Lin = x.shape
    Cin2, Cout, K = w.shape
    assert Cin2 == Cin
    Lout = (Lin - 1) * stride - 2 * pad + K
    y = np.zeros((Cout, Lout), dtype=np.float64)
    b = _f64(bias) if bias is not None else None
    lib().orc_conv_transpose1d(_dp(x), Cin, Lin, _dp(w), Cout, K,
                               _dp(b) if b is not None else None, stride, pad, _dp(y), Lout)
    return y


def snake_beta(x, alpha: float, beta: float) -> np.ndarray:
    x = _f64(x)
    y = np.zeros_like(x)
    lib().orc_snake_beta(_dp(x), x.size, alpha, beta, _dp(y))
    return y


def upsample2(x, taps) -> np.ndarray:
    x = _f64(x)
    taps = _f64(taps)
    u = np.zeros(2 * x.size, dtype=np.float64)
    lib().orc_upsample2(_dp(x), x.size, _dp(taps), taps.size, _dp(u))
    return u


def downsample2(s, taps) -> np.ndarray:
    s = _f64(s)
    taps = _f64(taps)
    y = np.zeros(s.size // 2, dtype=np.float64)
    lib().orc_downsample2(_dp(s), s.size, _dp(taps), taps.size, _dp(y))
    return y


def activation1d(x, alpha: float, beta: float, taps) -> np.ndarray:
    x = _f64(x)
    taps = _f64(taps)
    y = np.zeros_like(x)
    lib().orc_activation1d(_dp(x), x.size, alpha, beta, _dp(taps), taps.size, _dp(y))
    return y


def act_taps() -> np.ndarray:
    """The activation filter as the oracle uses it: K=12, cutoff 0.25, half-width 0.3,
    rounded to fp32 (a stored fp32 buffer), returned widened to fp64."""
    t, _, _ = kaiser_sinc_filter(0.25, 0.3, 12)
    return t.astype(np.float32).astype(np.float64)


# --------------------------------------------------------------------------------------------
# decode / AMP stage
# --------------------------------------------------------------------------------------------

@dataclass
class Arch:
    latent_channels: int = 32
    latent_dim: int = 2048
    decoder_dim: int = 1024
    rates: tuple = (5, 5, 2, 2, 2, 2, 2)
    kernels: tuple = (9, 9, 4, 4, 4, 4, 4)
    rb_kernels: tuple = (3, 7, 11)
    rb_dilations: tuple = ((1, 3, 5), (1, 3, 5), (1, 3, 5))
    latents_mean: object = None
    latents_std: object = None
    clamp: bool = True
    _keep: list = field(default_factory=list, repr=False)

    @staticmethod
    def from_any(a) -> "Arch":
        if isinstance(a, Arch):
            return a
        out = Arch()
        for k in ("latent_channels", "latent_dim", "decoder_dim", "rates", "kernels",
                  "rb_kernels", "rb_dilations", "latents_mean", "latents_std"):
            if hasattr(a, k):
                setattr(out, k, getattr(a, k))
        return out

    def to_c(self) -> _Config:
        c = _Config()
        c.latent_channels = self.latent_channels
        c.latent_dim = self.latent_dim
        c.decoder_dim = self.decoder_dim
        c.n_stages = len(self.rates)
        for i, (r, k) in enumerate(zip(self.rates, self.kernels)):
            c.rates[i] = r
            c.kernels[i] = k
        c.n_resblocks = len(self.rb_kernels)
        for j, k in enumerate(self.rb_kernels):
            c.rb_kernels[j] = k
        c.n_dilations = len(self.rb_dilations[0])
        for j, ds in enumerate(self.rb_dilations):
            for m, d in enumerate(ds):
                c.rb_dilations[j][m] = d
        c.clamp = 1 if self.clamp else 0
        self._keep = []
        if self.latents_mean is not None:
            m = _f32(self.latents_mean)
            self._keep.append(m)
            c.latents_mean = _fp(m)
        if self.latents_std is not None:
            s = _f32(self.latents_std)
            self._keep.append(s)
            c.latents_std = _fp(s)
        return c


def _table(weights: dict):
    keep = []
    arr = (_Tensor * len(weights))()
    for i, (name, a) in enumerate(weights.items()):
        a = _f32(a)
        keep.append(a)
        nb = name.encode()
        keep.append(nb)
        arr[i].name = nb
        arr[i].data = _fp(a)
        arr[i].ndim = a.ndim
        for d in range(3):
            arr[i].shape[d] = a.shape[d] if d < a.ndim else 1
    return arr, keep


_ERR = {1: "invalid argument", 2: "missing weight", 3: "weight shape mismatch", 4: "alloc"}


def decode(arch, weights: dict, latents: np.ndarray, clamp: bool = True) -> np.ndarray:
    """fp64 decode of fp32 latents [B, 32, N] -> waveform [B, 1, hop*N] (fp64)."""
    a = Arch.from_any(arch)
    a.clamp = clamp
    cfg = a.to_c()
    tab, keep = _table(weights)
    z = _f32(latents)
    B, _, N = z.shape
    hop = int(np.prod(a.rates))
    out = np.zeros((B, 1, hop * N), dtype=np.float64)
    rc = lib().orc_decode(C.byref(cfg), tab, len(weights), _fp(z), B, N, _dp(out))
    if rc:
        raise RuntimeError(f"oracle decode failed: {_ERR.get(rc, rc)}")
    return out


def amp_stage(arch, weights: dict, stage: int, x: np.ndarray) -> np.ndarray:
    """fp64 AMP stage `stage` on x [B, C, L] (fp32 or fp64 input)."""
    a = Arch.from_any(arch)
    cfg = a.to_c()
    tab, keep = _table(weights)
    B, Cc, L = x.shape
    out = np.zeros((B, Cc, L), dtype=np.float64)
    if x.dtype == np.float64:
        xd = _f64(x)
        rc = lib().orc_amp_stage_f64(C.byref(cfg), tab, len(weights), stage, _dp(xd), B, L,
                                     _dp(out))
    else:
        xf = _f32(x)
        rc = lib().orc_amp_stage(C.byref(cfg), tab, len(weights), stage, _fp(xf), B, L, _dp(out))
    if rc:
        raise RuntimeError(f"oracle amp_stage failed: {_ERR.get(rc, rc)}")
    return out


def num_threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(lib().orc_num_threads())
