"""Writes tiny_forward.json from the oracle alone (inputs from the seeded generator)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import synth  # noqa: E402
from oracle import msa_oracle as O  # noqa: E402

SPEC = dict(seed=11, B=1, Hq=4, Hkv=2, d=16, lens=[300, 257, 40, 512], Lc=20, Tq=4,
            route_block=2, top_k=2)


def inputs(spec):
    B, Hq, Hkv, d, Lc, Tq = (spec[k] for k in ("B", "Hq", "Hkv", "d", "Lc", "Tq"))
    N = sum(spec["lens"])
    shapes = {"K": (Hkv, N, d), "V": (Hkv, N, d), "R": (Hkv, N, d), "Q": (B, Hq, Tq, d),
              "Qr": (B, Hkv, Tq, d), "LK": (B, Hkv, Lc, d), "LV": (B, Hkv, Lc, d)}
    ids = {"K": synth.T_K, "V": synth.T_V, "R": synth.T_R, "Q": synth.T_Q, "Qr": synth.T_QR,
           "LK": synth.T_LK, "LV": synth.T_LV}
    return {k: synth.normal_f32(spec["seed"], ids[k], 0, int(np.prod(s))).reshape(s).astype(np.float64)
            for k, s in shapes.items()}


def main():
    res = O.forward(inputs(SPEC), SPEC["lens"], SPEC["top_k"], SPEC["route_block"])
    out = {"spec": SPEC, "topk": res["topk"].tolist(),
           "doc_scores": np.round(res["doc_scores"], 12).tolist(),
           "out": np.round(res["out"], 12).tolist(),
           "K_r_head0_first4": np.round(res["K_r"][0, :4], 12).tolist()}
    with open(os.path.join(HERE, "tiny_forward.json"), "w") as f:
        json.dump(out, f)


if __name__ == "__main__":
    main()
