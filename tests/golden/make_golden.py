"""Writes tests/golden/single_layer_seed0.txt from the CPU oracle only.

The fixture pins the oracle's output on the 512x512 single-layer case (X [1,512] ~ N(0,1),
W [512,512] ~ N(0,0.02), seed 0, group 128) so that later edits to the oracle cannot change
it silently; the GPU tests compare the library's packed bytes against the same digests.
Run:  python tests/golden/make_golden.py
"""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from weight_only_int4_06_b200 import synth  # noqa: E402


def digests():
    X, W = synth.single_layer_case()
    packed, scales, zeros = oracle.quantize_pack(W)
    Y = oracle.gemm(X, packed, scales, zeros)
    return {
        "packed_sha256": hashlib.sha256(np.ascontiguousarray(packed, dtype="<u4").tobytes()).hexdigest(),
        "scales_sha256": hashlib.sha256(np.ascontiguousarray(scales, dtype="<f2").tobytes()).hexdigest(),
        "zeros_sha256": hashlib.sha256(np.ascontiguousarray(zeros, dtype="u1").tobytes()).hexdigest(),
        "Y_first8": " ".join(repr(float(v)) for v in Y[0, :8]),
    }


def main():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "single_layer_seed0.txt")
    with open(path, "w") as f:
        f.write("# Oracle output on the single-layer case (512x512, seed 0, group 128).\n")
        f.write("# Written by tests/golden/make_golden.py, which calls only oracle/ and the seeded generators.\n")
        for k, v in digests().items():
            f.write(f"{k} = {v}\n")


if __name__ == "__main__":
    main()
