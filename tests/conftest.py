import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def small_arch():
    """A reduced architecture with the default rates, kernels and residual blocks but few
    channels, so that whole decodes run in well under a second on the oracle."""
    from bigvgan_waveform_decoder_b200.synthetic import Arch

    return Arch(latent_channels=4, latent_dim=32, decoder_dim=128)
