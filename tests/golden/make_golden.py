"""Write the oracle regression fixtures in this folder.

The Flash-KMeans pages print no worked example, so every fixture here is an
oracle output: this script calls only ``oracle/`` (and the seeded input
generators) and must be re-run, with the change named in the commit message,
whenever the oracle's arithmetic is changed on purpose.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import workloads  # noqa: E402


def tiny_f32(N=512, K=16, n_centers=16, iters=2, seed=0):
    s = workloads.spec("tiny_f32", N=N, K=K, n_centers=n_centers)
    w = workloads.make(s, seed=seed)
    out = oracle.lloyd(w.X.double().numpy(), w.C0.double().numpy(), iters, "f32")
    return {
        "what": "tiny_f32 workload recipe at N=512, K=16: oracle Lloyd after 2 iterations",
        "N": N, "K": K, "n_centers": n_centers, "iters": iters, "seed": seed,
        "labels": out["labels"].tolist(), "counts": out["counts"].tolist(),
        "C": out["C"].tolist(),
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_f32_n512_k16.json"), "w") as f:
        json.dump(tiny_f32(), f)
    print("wrote tiny_f32_n512_k16.json")
