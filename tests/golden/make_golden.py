"""Writes the oracle regression fixtures in this folder.

Calls only the fp64 oracle (and the seeded input module for its inputs);
nothing here touches the CUDA library.  Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402
import synth        # noqa: E402


def tiny_workload_fixture(seed=0):
    """The tiny GQA-4 workload (T=512, r=32, tau=0.3), drawn on the CPU."""
    w = synth.workload(0)
    L = synth.make_layer(w, 0, seed, device="cpu")
    f64 = lambda t: t.double().numpy()
    D = O.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, r_k=w.r_k, r_v=w.r_v, T_cap=w.T, F_cap=w.T)
    cache = O.Cache.empty(D, f64(L["U_k"]), f64(L["U_v"]))
    e, _, _ = O.compress(cache, f64(L["K"]), f64(L["V"]), w.tau)
    out = O.decode_attn(cache, f64(L["q"]))
    n = int(cache.full_cnt[0, 0])
    return {
        "cite": "OjaKV repository README, Method Summary (StaticPCA basis, hybrid full-rank policy); "
                "inputs: the tiny GQA-4 workload drawn by synth.make_layer on the CPU",
        "workload": w.name, "seed": seed, "tau": w.tau,
        "full_idx": cache.full_idx[0, 0, :n].tolist(),
        "outlier_pos": L["outlier_pos"][0][0].tolist(),
        "err_first8": [float(x) for x in e[0, 0, :8]],
        "coef_k_bits_sum": int(O.bf16_bits(cache.coef_k[0, 0]).astype(np.int64).sum()),
        "out": [[float(x) for x in row] for row in out[0]],
    }


if __name__ == "__main__":
    fx = tiny_workload_fixture()
    with open(os.path.join(HERE, "tiny_workload_seed0.json"), "w") as f:
        json.dump(fx, f, indent=1)
        f.write("\n")
    print("full-rank tokens:", len(fx["full_idx"]), "outliers:", len(fx["outlier_pos"]))
