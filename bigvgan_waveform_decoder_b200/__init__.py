"""B200-native (sm_100a) BigVGAN waveform decoder of the MiniMax-H3 audio VAE.

Latents [B, 32, N] -> mono 32 kHz waveform [B, 1, 800 N] in [-1, 1], computed entirely by the
CUDA library libmh3a.so (C ABI in include/mh3a.h).  ``binding.Decoder`` is the Python front
end; ``synthetic`` draws the seeded random-init weights and latents used by tests and bench.
"""
from .binding import (MH3A_BF16X3, MH3A_FLAG_NO_CLAMP, MH3A_FP32, Decoder, MH3AError,  # noqa: F401
                      load)
