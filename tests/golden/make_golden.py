"""Writes tests/golden/tiny_128.json from the fp64 oracle alone.

The stored numbers are a regression fixture of the oracle on the smallest
seeded workload (B=1, H=1, N_Q=N_K=128, d=64, no mask, student = teacher +
0.1 noise).  Run ``python tests/golden/make_golden.py`` from the repository
root; it calls nothing but ``oracle`` and the seeded input generator.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from attention_kl_divergence_attn_b200 import inputs  # noqa: E402


def main():
    w = inputs.WORKLOADS["tiny_128"]
    qt, kt, qs, ks = inputs.make_inputs(w)
    kl, lt, ls = oracle.fwd(qt, kt, qs, ks, w.scale_t, w.scale_s, w.causal, nthreads=1)
    g = 1.0 / w.rows
    dqs, dks, dqt, dkt = oracle.bwd(qt, kt, qs, ks, w.scale_t, w.scale_s, w.causal, g=g, nthreads=1)
    out = {
        "workload": w.as_dict(),
        "g": g,
        "loss_mean": oracle.mean(kl),
        "kl_rows_0_8": kl.ravel()[:8].tolist(),
        "lse_t_rows_0_8": lt.ravel()[:8].tolist(),
        "lse_s_rows_0_8": ls.ravel()[:8].tolist(),
        "dq_s_row0": dqs.reshape(-1, w.d_s)[0].tolist(),
        "dk_s_row0": dks.reshape(-1, w.d_s)[0].tolist(),
        "norms": {"dq_s": float(np.linalg.norm(dqs)), "dk_s": float(np.linalg.norm(dks)),
                  "dq_t": float(np.linalg.norm(dqt)), "dk_t": float(np.linalg.norm(dkt))},
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_128.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
