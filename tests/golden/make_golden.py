"""Writes the regression fixtures of this folder from the oracle alone (no CUDA code runs).

The pages print no worked example of the method, so no fixture here holds the pages' own values;
these record what the oracle computes on seeded inputs, so that a later change of the oracle's
arithmetic shows up as a diff of a committed file, and so that the GPU path can be checked
against stored values without running the oracle.

    python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import Oracle  # noqa: E402
from synth.workloads import WORKLOADS, Workload, full_inputs  # noqa: E402

# (workload, sampled query ids): early queries (fewer candidates than k), block-boundary queries, late queries
FIXTURES = [
    (WORKLOADS["tiny_prefill_1k"], [0, 1, 63, 64, 65, 127, 128, 255, 256, 511, 512, 700, 767, 768, 1000, 1023]),
    (Workload("golden_gqa_mh", 2, 300, 500, 64, 32, 5, 96, 4, 2, 64, n_idx_heads=2),
     [0, 37, 150, 299, 300, 333, 450, 599]),
]


def fixture_path(w) -> str:
    return os.path.join(HERE, f"oracle_{w.name}.txt")


def write(w, ids) -> str:
    out = Oracle().run(w, full_inputs(w), query_ids=np.array(ids, dtype=np.int64))
    lines = [f"# oracle outputs of workload {w.name} (seed {w.seed}) for the query ids below; written by",
             "# tests/golden/make_golden.py from the oracle alone",
             f"workload {w.name} {w.batch} {w.n_q} {w.n_kv} {w.d_idx} {w.block} {w.top_m} {w.top_k} "
             f"{w.n_heads} {w.n_kv_heads} {w.d_head} {w.n_idx_heads}"]
    for r, q in enumerate(ids):
        lines.append(f"query {q}")
        lines.append("blocks " + " ".join(str(int(x)) for x in out["block_idx"][r]))
        lines.append("tokens " + " ".join(str(int(x)) for x in out["token_idx"][r]))
        lines.append("lse " + " ".join(repr(float(x)) for x in out["lse"][r]))
        lines.append("o " + " ".join(repr(float(x)) for x in out["o"][r].reshape(-1)))
    path = fixture_path(w)
    with open(path, "w") as f:
        f.write("\n".join(lines) + "\n")
    return path


def read(path):
    """-> (workload fields, {query: {"blocks", "tokens", "lse", "o"}})"""
    fields, rows, cur = None, {}, None
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        if key == "workload":
            fields = vals
        elif key == "query":
            cur = int(vals[0])
            rows[cur] = {}
        elif key in ("blocks", "tokens"):
            rows[cur][key] = np.array([int(v) for v in vals], dtype=np.int32)
        else:
            rows[cur][key] = np.array([float(v) for v in vals], dtype=np.float64)
    return fields, rows


if __name__ == "__main__":
    for w, ids in FIXTURES:
        print("wrote", write(w, ids))
