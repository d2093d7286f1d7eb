"""Writes cfg1_oracle.json: oracle outputs for the tiny fp32 workload (2 x 64 tokens,
64 -> 64, K = 8, sigma = 1e-2, gamma = 0.9 and 0).  Calls only ``oracle`` and ``workloads``;
the stored values guard the oracle against unintended changes.  Run from the repo root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import workloads  # noqa: E402


def compute():
    data = workloads.generate(1)
    L = data.layers[0]
    wl = data.wl
    out = {}
    for gamma in wl.gammas:
        res = oracle.dust_layer(L.x_f64, L.W_f64, L.u_f64, wl.K, wl.sigma, gamma,
                                data.cu_seqlens, wl.seed, layer_id=L.shape.layer_id)
        out[f"gamma={gamma}"] = {
            "dloss[0,:6]": (res["loss"][0, :6] - res["clean"][:6]).tolist(),
            "r[3,60:66]": res["r"][3, 60:66].tolist(),
            "g[127,:6]": res["g"][127, :6].tolist(),
            "G_W[5,:6]": res["G_W"][5, :6].tolist(),
            "|g|_F": float(np.linalg.norm(res["g"])),
            "|G_W|_F": float(np.linalg.norm(res["G_W"])),
        }
    return out


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "cfg1_oracle.json")
    with open(path, "w") as f:
        json.dump(compute(), f, indent=1)
    print("wrote", path)
