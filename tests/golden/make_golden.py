"""Write the stored fixtures under tests/golden/ from the oracle only.

    python tests/golden/make_golden.py

kaiser_sinc_k12_c0.25_hw0.3.txt -- the activation filter (FastVideo "minimax_h3_audio_vae"
page, kaiser_sinc_filter1d at cutoff 0.5/2, half-width 0.6/2, 12 taps) in fp64.  The test that
reads it also checks it against scipy.signal.firwin, so the fixture is pinned independently.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def main():
    taps, atten, beta = oracle.kaiser_sinc_filter(0.25, 0.3, 12)
    path = os.path.join(HERE, "kaiser_sinc_k12_c0.25_hw0.3.txt")
    header = (f"Kaiser-sinc low-pass, K=12, cutoff=0.25, half_width=0.3; "
              f"attenuation={atten:.17g} beta={beta:.17g}")
    np.savetxt(path, taps, fmt="%.17g", header=header)
    print(path)


if __name__ == "__main__":
    main()
