"""Writes the oracle regression fixture for the toy layer (M=4, K=512,
N=256, seed 0).  Calls only ``oracle`` and ``synth``; never the CUDA path.

    python tests/golden/make_golden.py
"""

import hashlib
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402
import synth  # noqa: E402


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def toy():
    w = synth.weights(256, 512, synth.rng_for(0, 0, "weight"))
    c = O.convert_weight(w)
    bits, x, ch = synth.activations(4, 512, synth.rng_for(0, 0, "act"), 2)
    q, s_x, _ = O.quantize_activations(x)
    y = O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"])
    return {
        "config": "toy W4A8 linear: M=4, K=512, N=256, seed 0",
        "fit_rounds": int(c["fit_rounds"]),
        "codebook": [float(v) for v in c["cb"]],
        "sha256": {"packed": digest(c["packed"]), "s_rel": digest(c["s_rel"]),
                   "s_ch": digest(c["s_ch"]), "x_bf16": digest(bits),
                   "q": digest(q), "s_x": digest(s_x)},
        "s_x": [float(v) for v in s_x],
        "y_row0_first8": [float(v) for v in y[0, :8]],
        "y_norm": float(np.linalg.norm(y)),
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "toy_oracle.json"), "w") as f:
        json.dump(toy(), f, indent=1)
        f.write("\n")
