"""Write the oracle's regression fixture for the ``small`` workload.

The pages print no worked numerical example (neither the Quaff notes nor
the QQQ review gives input/output values for any step), so the stored
values here are written by this script, which calls only the CPU oracle
(and the seeded input generator).  Re-run it only when an oracle change is
justified by a passage of the pages; the test compares the oracle's current
output with this file so that an unintended change shows up.

    python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import oracle  # noqa: E402
from quantized_linear_layers_token_b200 import synth  # noqa: E402


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def compute() -> dict:
    out = {}
    for fmt, tag in [(synth.W4_PERCHANNEL, "w4pc"), (synth.W4_G128, "w4g128"),
                     (synth.W8_PERCHANNEL, "w8")]:
        L = synth.layer("small", 0)
        Xb = np.ascontiguousarray(L["X"]).view(np.uint16)
        Wb = np.ascontiguousarray(L["W"]).view(np.uint16)
        pk = oracle.pack_layer(Wb, L["O"], fmt)
        r = oracle.forward(Xb, Wb, pk, np.ones(len(L["O"]), np.float32), L["gamma"])
        # input gradient with the forward's scales (straight-through estimator)
        dY = np.ascontiguousarray(synth.grad_output(0, 0, L["M"], L["N"])).view(np.uint16)
        dX = oracle.backward_dx(dY, Wb, pk, r["s"])
        out[tag] = {
            "dX_00_01_10": [float(dX[0, 0]), float(dX[0, 1]), float(dX[1, 0])],
            "O": L["O"].tolist(),
            "s": [float(v) for v in r["s"]],
            "a_first4": [float(v) for v in r["a"][:4]],
            "y_00_01_10": [float(r["y"][0, 0]), float(r["y"][0, 1]), float(r["y"][1, 0])],
            "acc_00": int(r["acc"][0, 0]),
            "sha256": {
                "packed": digest(pk["packed"]), "B": digest(pk["B"]), "cscale": digest(pk["cscale"]),
                "Xq": digest(r["Xq"]), "a": digest(r["a"]), "XqO": digest(r["XqO"]),
                "acc": digest(r["acc"]), "s": digest(r["s"]), "dX": digest(dX),
            },
        }
    return out


if __name__ == "__main__":
    data = {"source": "CPU oracle on the seeded 'small' workload (M=16, K=N=512, 10 outlier "
                      "channels, gamma=0.9, one momentum step, s0=1), and its input gradient for "
                      "the seeded dY; the pages print no worked example, so these are regression "
                      "values, not the pages'.",
            "cases": compute()}
    with open(os.path.join(HERE, "small_oracle.json"), "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
    print("wrote", os.path.join(HERE, "small_oracle.json"))
