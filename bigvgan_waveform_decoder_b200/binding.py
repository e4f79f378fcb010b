"""Thin ctypes binding of the C ABI in include/mh3a.h (argument marshalling only).

Every step of the decode runs in the CUDA library ``libmh3a.so`` built in this package
directory; there is no fallback.  If the library is missing or cannot be loaded, every call
raises ``RuntimeError``.  PyTorch is used only for device memory and streams.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmh3a.so")

MH3A_FP32 = 0
MH3A_BF16X3 = 1
MH3A_FLAG_NO_CLAMP = 1
MAX_STAGES, MAX_RESBLOCKS, MAX_DILATIONS = 8, 4, 4

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "shape mismatch",
          4: "missing weight", 5: "allocation failed", 6: "CUDA error", 7: "unsupported request"}

EXPORTS = ("mh3a_default_config", "mh3a_config_from_json", "mh3a_create", "mh3a_create_with_allocator", "mh3a_create_from_safetensors",
           "mh3a_decode",
           "mh3a_decode_host",
           "mh3a_amp_stage", "mh3a_set_graph_mode", "mh3a_set_profiling", "mh3a_segment_times", "mh3a_launch_count",
           "mh3a_device_bytes", "mh3a_destroy", "mh3a_status_string", "mh3a_last_error",
           "mh3a_stage_uses_tensor_cores", "mh3a_segment_uses_tensor_cores",
           "mh3a_check_device_error")


class mh3a_config(C.Structure):
    _fields_ = [
        ("latent_channels", C.c_int),
        ("latent_dim", C.c_int),
        ("decoder_dim", C.c_int),
        ("n_stages", C.c_int),
        ("rates", C.c_int * MAX_STAGES),
        ("kernels", C.c_int * MAX_STAGES),
        ("n_resblocks", C.c_int),
        ("rb_kernels", C.c_int * MAX_RESBLOCKS),
        ("n_dilations", C.c_int),
        ("rb_dilations", (C.c_int * MAX_DILATIONS) * MAX_RESBLOCKS),
        ("sampling_rate", C.c_int),
        ("precision", C.c_int),
        ("flags", C.c_uint),
        ("latents_mean", C.POINTER(C.c_float)),
        ("latents_std", C.POINTER(C.c_float)),
        ("max_batch", C.c_int),
        ("max_frames", C.c_int),
    ]


class mh3a_tensor(C.Structure):
    _fields_ = [
        ("name", C.c_char_p),
        ("host_data", C.POINTER(C.c_float)),
        ("ndim", C.c_int),
        ("shape", C.c_longlong * 3),
    ]


ALLOC_FN = C.CFUNCTYPE(C.c_void_p, C.c_size_t, C.c_void_p)
RELEASE_FN = C.CFUNCTYPE(None, C.c_void_p, C.c_void_p)


class mh3a_allocator(C.Structure):
    _fields_ = [("alloc", ALLOC_FN), ("release", RELEASE_FN), ("user", C.c_void_p)]


class MH3AError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        msg = f"{what}: {STATUS.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


_lib = None


def load():
    """Load libmh3a.so (once).  Raises RuntimeError when it is absent: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                           "(run python -m bigvgan_waveform_decoder_b200.build)")
    L = C.CDLL(LIB_PATH)
    vp = C.c_void_p
    L.mh3a_default_config.argtypes = [C.POINTER(mh3a_config)]
    L.mh3a_default_config.restype = None
    L.mh3a_create.argtypes = [C.POINTER(mh3a_config), C.POINTER(mh3a_tensor), C.c_int, C.POINTER(vp)]
    L.mh3a_create.restype = C.c_int
    L.mh3a_create_with_allocator.argtypes = [C.POINTER(mh3a_config), C.POINTER(mh3a_tensor), C.c_int,
                                             C.POINTER(mh3a_allocator), C.POINTER(vp)]
    L.mh3a_create_with_allocator.restype = C.c_int
    L.mh3a_create_from_safetensors.argtypes = [C.POINTER(mh3a_config), C.c_char_p, C.POINTER(mh3a_allocator),
                                               C.POINTER(vp)]
    L.mh3a_create_from_safetensors.restype = C.c_int
    L.mh3a_config_from_json.argtypes = [C.c_char_p, C.POINTER(mh3a_config), C.POINTER(C.c_float),
                                        C.POINTER(C.c_float), C.c_int]
    L.mh3a_config_from_json.restype = C.c_int
    L.mh3a_decode.argtypes = [vp, vp, C.c_int, C.c_int, vp, vp]
    L.mh3a_decode.restype = C.c_int
    L.mh3a_decode_host.argtypes = [vp, vp, C.c_int, C.c_int, vp, vp]
    L.mh3a_decode_host.restype = C.c_int
    L.mh3a_amp_stage.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, vp, vp]
    L.mh3a_amp_stage.restype = C.c_int
    L.mh3a_set_graph_mode.argtypes = [vp, C.c_int]
    L.mh3a_set_graph_mode.restype = C.c_int
    L.mh3a_set_profiling.argtypes = [vp, C.c_int]
    L.mh3a_set_profiling.restype = C.c_int
    L.mh3a_set_kernel_profiling.argtypes = [vp, C.c_int]
    L.mh3a_set_kernel_profiling.restype = C.c_int
    L.mh3a_stage_kernel_times.argtypes = [vp, C.c_int, C.POINTER(C.c_float), C.POINTER(C.c_float)]
    L.mh3a_stage_kernel_times.restype = C.c_int
    L.mh3a_segment_times.argtypes = [vp, C.POINTER(C.c_float), C.c_int, C.POINTER(C.c_int)]
    L.mh3a_segment_times.restype = C.c_int
    L.mh3a_launch_count.argtypes = [vp]
    L.mh3a_launch_count.restype = C.c_longlong
    L.mh3a_stage_uses_tensor_cores.argtypes = [vp, C.c_int]
    L.mh3a_stage_uses_tensor_cores.restype = C.c_int
    L.mh3a_segment_uses_tensor_cores.argtypes = [vp, C.c_int]
    L.mh3a_segment_uses_tensor_cores.restype = C.c_int
    L.mh3a_check_device_error.argtypes = [vp]
    L.mh3a_check_device_error.restype = C.c_int
    L.mh3a_device_bytes.argtypes = [vp]
    L.mh3a_device_bytes.restype = C.c_longlong
    L.mh3a_destroy.argtypes = [vp]
    L.mh3a_destroy.restype = None
    L.mh3a_status_string.argtypes = [C.c_int]
    L.mh3a_status_string.restype = C.c_char_p
    L.mh3a_last_error.argtypes = []
    L.mh3a_last_error.restype = C.c_char_p
    _lib = L
    return L


def _check(st: int, what: str):
    if st != 0:
        detail = load().mh3a_last_error().decode() if st == 6 else ""
        raise MH3AError(st, what, detail)


def make_config(arch, precision: int = MH3A_BF16X3, max_batch: int = 2, max_frames: int = 400,
                no_clamp: bool = False):
    """mh3a_config from an architecture object with the fields of synthetic.Arch.
    Returns (config, keepalive)."""
    cfg = mh3a_config()
    load().mh3a_default_config(C.byref(cfg))
    cfg.latent_channels = arch.latent_channels
    cfg.latent_dim = arch.latent_dim
    cfg.decoder_dim = arch.decoder_dim
    cfg.n_stages = len(arch.rates)
    for i, (r, k) in enumerate(zip(arch.rates, arch.kernels)):
        cfg.rates[i] = r
        cfg.kernels[i] = k
    cfg.n_resblocks = len(arch.rb_kernels)
    for j, k in enumerate(arch.rb_kernels):
        cfg.rb_kernels[j] = k
    cfg.n_dilations = len(arch.rb_dilations[0])
    for j, ds in enumerate(arch.rb_dilations):
        for m, d in enumerate(ds):
            cfg.rb_dilations[j][m] = d
    cfg.precision = precision
    cfg.flags = MH3A_FLAG_NO_CLAMP if no_clamp else 0
    cfg.max_batch = max_batch
    cfg.max_frames = max_frames
    keep = []
    if getattr(arch, "latents_mean", None) is not None:
        m = np.ascontiguousarray(arch.latents_mean, dtype=np.float32)
        keep.append(m)
        cfg.latents_mean = m.ctypes.data_as(C.POINTER(C.c_float))
    if getattr(arch, "latents_std", None) is not None:
        s = np.ascontiguousarray(arch.latents_std, dtype=np.float32)
        keep.append(s)
        cfg.latents_std = s.ctypes.data_as(C.POINTER(C.c_float))
    return cfg, keep


class ComponentArch:
    """The architecture fields make_config reads, from a component's config.json."""

    def __init__(self, cfg: "mh3a_config", mean, std):
        n = cfg.n_stages
        self.latent_channels = cfg.latent_channels
        self.latent_dim = cfg.latent_dim
        self.decoder_dim = cfg.decoder_dim
        self.rates = tuple(cfg.rates[i] for i in range(n))
        self.kernels = tuple(cfg.kernels[i] for i in range(n))
        self.rb_kernels = tuple(cfg.rb_kernels[j] for j in range(cfg.n_resblocks))
        self.rb_dilations = tuple(tuple(cfg.rb_dilations[j][m] for m in range(cfg.n_dilations))
                                  for j in range(cfg.n_resblocks))
        self.sampling_rate = cfg.sampling_rate
        self.latents_mean = mean
        self.latents_std = std


def load_config(path) -> ComponentArch:
    """mh3a_config_from_json: the architecture (and latent statistics) of a config.json."""
    cfg = mh3a_config()
    cap = 4096
    mean = np.zeros(cap, np.float32)
    std = np.zeros(cap, np.float32)
    fp = C.POINTER(C.c_float)
    _check(load().mh3a_config_from_json(os.fsencode(path), C.byref(cfg), mean.ctypes.data_as(fp),
                                        std.ctypes.data_as(fp), cap), "mh3a_config_from_json")
    n = cfg.latent_channels
    return ComponentArch(cfg, mean[:n].copy() if cfg.latents_mean else None,
                         std[:n].copy() if cfg.latents_std else None)


def make_table(weights: dict):
    keep = []
    arr = (mh3a_tensor * len(weights))()
    for i, (name, a) in enumerate(weights.items()):
        a = np.ascontiguousarray(a, dtype=np.float32)
        nb = name.encode()
        keep += [a, nb]
        arr[i].name = nb
        arr[i].host_data = a.ctypes.data_as(C.POINTER(C.c_float))
        arr[i].ndim = a.ndim
        for d in range(3):
            arr[i].shape[d] = a.shape[d] if d < a.ndim else 1
    return arr, keep


def _stream_ptr(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


class Decoder:
    """Owns one mh3a handle on the current CUDA device."""

    def __init__(self, arch, weights, precision: int = MH3A_BF16X3, max_batch: int = 2,
                 max_frames: int = 400, no_clamp: bool = False, allocator=None):
        """weights: a dict name -> array (mh3a_create), or the path of a safetensors checkpoint
        (mh3a_create_from_safetensors).  allocator: optional (alloc(bytes) -> int device pointer
        or 0, release(ptr)) pair that provides the handle's device memory
        (mh3a_create_with_allocator); it is kept alive with the handle."""
        L = load()
        self.arch = arch
        self.hop = int(np.prod(arch.rates))
        self.latent_channels = arch.latent_channels
        cfg, keep = make_config(arch, precision, max_batch, max_frames, no_clamp)
        h = C.c_void_p()
        self._alloc = None
        if allocator is not None:
            alloc_py, release_py = allocator
            self._alloc = mh3a_allocator(ALLOC_FN(lambda n, user: alloc_py(int(n)) or None),
                                         RELEASE_FN(lambda ptr, user: release_py(int(ptr))), None)
        if isinstance(weights, (str, os.PathLike)):
            a = C.byref(self._alloc) if self._alloc is not None else None
            _check(L.mh3a_create_from_safetensors(C.byref(cfg), os.fsencode(weights), a, C.byref(h)),
                   "mh3a_create_from_safetensors")
        else:
            tab, keep2 = make_table(weights)
            if self._alloc is None:
                _check(L.mh3a_create(C.byref(cfg), tab, len(weights), C.byref(h)), "mh3a_create")
            else:
                _check(L.mh3a_create_with_allocator(C.byref(cfg), tab, len(weights), C.byref(self._alloc),
                                                    C.byref(h)), "mh3a_create_with_allocator")
            del keep2
        self._h = h
        del keep

    @classmethod
    def from_component_dir(cls, component_dir, **kw):
        """The released audio VAE component directory: config.json (mh3a_config_from_json; the
        defaults when absent) and diffusion_pytorch_model.safetensors
        (mh3a_create_from_safetensors), as the MLX page's `mlx_h3_audio_vae_from_dir` loads
        it."""
        d = os.fspath(component_dir)
        weights = os.path.join(d, "diffusion_pytorch_model.safetensors")
        if not os.path.exists(weights):
            raise FileNotFoundError(f"No audio VAE safetensors under {d}")
        conf = os.path.join(d, "config.json")
        if os.path.exists(conf):
            arch = load_config(conf)
        else:
            cfg = mh3a_config()
            load().mh3a_default_config(C.byref(cfg))
            arch = ComponentArch(cfg, None, None)
        return cls(arch, weights, **kw)

    @property
    def handle(self):
        return self._h

    def decode(self, latents, out=None, stream=None):
        """latents: CUDA float32 tensor [B, 32, N] -> CUDA float32 [B, 1, hop*N]."""
        import torch
        assert latents.is_cuda and latents.dtype == torch.float32 and latents.is_contiguous()
        B, _, N = latents.shape
        if out is None:
            out = torch.empty((B, 1, self.hop * N), device=latents.device, dtype=torch.float32)
        _check(load().mh3a_decode(self._h, latents.data_ptr(), B, N, out.data_ptr(),
                                  _stream_ptr(stream)), "mh3a_decode")
        return out

    def decode_host(self, latents, out, stream=None):
        """Host (ideally pinned) float32 tensors or arrays; blocks until `out` is filled."""
        B, _, N = latents.shape
        lp = latents.data_ptr() if hasattr(latents, "data_ptr") else latents.ctypes.data
        op = out.data_ptr() if hasattr(out, "data_ptr") else out.ctypes.data
        _check(load().mh3a_decode_host(self._h, lp, B, N, op, _stream_ptr(stream)),
               "mh3a_decode_host")
        return out

    def amp_stage(self, x, stage: int, out=None, stream=None):
        import torch
        assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
        B, _, Lx = x.shape
        if out is None:
            out = torch.empty_like(x)
        _check(load().mh3a_amp_stage(self._h, x.data_ptr(), B, Lx, stage, out.data_ptr(),
                                     _stream_ptr(stream)), "mh3a_amp_stage")
        return out

    def set_graph_mode(self, on: bool):
        """Replay each (B, N, input, output) decode from a CUDA graph captured on first use."""
        _check(load().mh3a_set_graph_mode(self._h, 1 if on else 0), "mh3a_set_graph_mode")

    def set_profiling(self, on: bool):
        _check(load().mh3a_set_profiling(self._h, 1 if on else 0), "mh3a_set_profiling")

    def set_kernel_profiling(self, stage: int):
        """Events around the activation and GEMM launches of one AMP stage (-1: none)."""
        _check(load().mh3a_set_kernel_profiling(self._h, stage), "mh3a_set_kernel_profiling")

    def stage_kernel_times(self, stage: int):
        """(activation ms, GEMM ms) summed over the AMP stage's six layers of the last decode."""
        a, g = C.c_float(), C.c_float()
        _check(load().mh3a_stage_kernel_times(self._h, stage, C.byref(a), C.byref(g)), "mh3a_stage_kernel_times")
        return a.value, g.value

    def segment_times(self):
        buf = (C.c_float * 64)()
        n = C.c_int()
        _check(load().mh3a_segment_times(self._h, buf, 64, C.byref(n)), "mh3a_segment_times")
        return [buf[i] for i in range(n.value)]

    def launch_count(self) -> int:
        return int(load().mh3a_launch_count(self._h))

    def stage_uses_tensor_cores(self, stage: int) -> bool:
        return load().mh3a_stage_uses_tensor_cores(self._h, stage) == 1

    def segment_uses_tensor_cores(self, segment: int) -> bool:
        return load().mh3a_segment_uses_tensor_cores(self._h, segment) == 1

    def check_device_error(self):
        """Raise if a tensor-core kernel of this handle timed out on a pipeline wait."""
        _check(load().mh3a_check_device_error(self._h), "device pipeline")

    def device_bytes(self) -> int:
        return int(load().mh3a_device_bytes(self._h))

    def close(self):
        if getattr(self, "_h", None):
            load().mh3a_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
