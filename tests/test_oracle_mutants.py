"""Plant plausible mistakes in copies of the oracle and check that the pins catch each one.

Every mutant is a one-line textual change of ``oracle/hisa_oracle.c`` compiled
into a temporary library (the committed oracle is untouched).  The mutants
are memory-safe, so a mutant can only fail checks, never crash the process.
"""
import os
import tempfile

import pytest

import oracle
import oracle_checks as C

MUTANTS = [
    ("tie-break toward the higher index",
     "if (x->score < y->score) return 1;\n  return (x->index > y->index) - (x->index < y->index);",
     "if (x->score < y->score) return 1;\n  return (x->index < y->index) - (x->index > y->index);"),
    ("lowest scores kept instead of highest",
     "if (x->score > y->score) return -1;\n  if (x->score < y->score) return 1;",
     "if (x->score > y->score) return 1;\n  if (x->score < y->score) return -1;"),
    ("own block not forced",
     "for (int64_t r = 0; r < s - 2; ++r) sel[n++] = (int32_t)cand[r].index;\n    sel[n++] = (int32_t)c;",
     "for (int64_t r = 0; r < s - 1; ++r) sel[n++] = (int32_t)cand[r].index;"),
    ("first block not forced",
     "sel[n++] = 0;\n    for (int64_t r = 0; r < s - 2; ++r)",
     "for (int64_t r = 0; r < s - 1; ++r)"),
    ("pooling divides by B instead of the block's token count",
     "block_keys[j * d_idx + e] = sum / (double)cnt;",
     "block_keys[j * d_idx + e] = sum / (double)block;"),
    ("pooling drops the last token of each block",
     "for (int64_t t = t0; t < t0 + cnt; ++t) sum +=",
     "for (int64_t t = t0; t < t0 + cnt - 1; ++t) sum +="),
    ("causal bound excludes the query's own position",
     "if (t1 > p + 1) t1 = p + 1;",
     "if (t1 > p) t1 = p;"),
    ("own block taken from the previous position",
     "int64_t c = p / block; /* the query's own block */",
     "int64_t c = (p > 0 ? p - 1 : 0) / block; /* the query's own block */"),
    ("one token too few kept",
     "int64_t k_eff = n < top_k ? n : top_k;",
     "int64_t k_eff = n < top_k ? n : top_k - 1;"),
    ("dot product drops the last dimension",
     "for (int32_t e = 0; e < n; ++e) s += bf16_value(a[e]) * bf16_value(b[e]);",
     "for (int32_t e = 0; e < n - 1; ++e) s += bf16_value(a[e]) * bf16_value(b[e]);"),
    ("attention scale not applied",
     "w[r] = scale * dot_bf16_bf16(qh, kr, d_head);",
     "w[r] = dot_bf16_bf16(qh, kr, d_head);"),
    ("log-sum-exp missing the max",
     "lse[h] = mx + log(sum);",
     "lse[h] = log(sum);"),
    ("wrong query-head to kv-head map",
     "int32_t g = h / group;",
     "int32_t g = h % n_kv_heads;"),
    ("multi-head block score without the ReLU",
     "s += w[j] * relu(dot_bf16_f64(q + (int64_t)j * d_idx, key, d_idx));",
     "s += w[j] * dot_bf16_f64(q + (int64_t)j * d_idx, key, d_idx);"),
    ("multi-head token score ignores the head weights",
     "s += w[j] * relu(dot_bf16_bf16(q + (int64_t)j * d_idx, key, d_idx));",
     "s += relu(dot_bf16_bf16(q + (int64_t)j * d_idx, key, d_idx));"),
    ("multi-head token score reads head 0 for every head",
     "s += w[j] * relu(dot_bf16_bf16(q + (int64_t)j * d_idx, key, d_idx));",
     "s += w[j] * relu(dot_bf16_bf16(q, key, d_idx));"),
]


@pytest.mark.parametrize("name,orig,mut", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, orig, mut):
    src = open(oracle.SRC).read()
    assert src.count(orig) == 1, f"mutation site for '{name}' not found exactly once"
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "hisa_oracle.c")
        with open(path, "w") as f:
            f.write(src.replace(orig, mut))
        so = os.path.join(td, "libmutant.so")
        import subprocess

        subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", path, "-o", so, "-lm"],
                       check=True)
        O = oracle.Oracle(oracle.load(so))
        caught = []
        for check in C.ALL_CHECKS:
            try:
                check(O)
            except Exception:  # a failed assertion or a check that cannot even run
                caught.append(check.__name__)
        assert caught, f"no pin caught the mutant '{name}'"
