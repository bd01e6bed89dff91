"""The CPU oracle against closed forms, library routines, brute force and invariants."""
import numpy as np
import pytest

import oracle_checks as C
from synth.workloads import WORKLOADS, full_inputs


@pytest.mark.parametrize("check", C.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check, oracle_lib):
    check(oracle_lib)


def test_tiny_workload_invariants(oracle_lib):
    """The full tiny prefill workload: forced blocks, counts and the cost-model closed form."""
    w = WORKLOADS["tiny_prefill_1k"]
    inp = full_inputs(w)
    r = oracle_lib.run(w, inp, attention=False)
    for i in range(w.n_q):
        p = i
        c = p // w.block
        s = min(w.top_m, c + 1)
        sel = r["block_idx"][i]
        assert sel[0] == 0 and sel[s - 1] == c and np.all(sel[s:] == -1)
        assert r["n_cand"][i] == C._n_cand_closed_form(p, w.block, w.top_m, w.n_kv)
        tok = r["token_idx"][i]
        k_eff = min(w.top_k, int(r["n_cand"][i]))
        assert np.all(np.diff(tok[:k_eff]) > 0) and np.all(tok[k_eff:] == -1) and tok[k_eff - 1] <= p


def test_needle_recall_probe(oracle_lib):
    """Behavioural check of the recipe: the probe query's top-m finds the planted needle blocks."""
    from synth.workloads import k_idx_rows, needle_table, q_idx_rows

    w = WORKLOADS["prefill_8k"]
    k = k_idx_rows(w, 0, 0, w.n_kv)
    q = q_idx_rows(w, 0, w.n_q - 1, 1)[0]
    bk = oracle_lib.block_pool(k, w.block)
    sel, s = oracle_lib.block_topm(q, bk, w.block, w.n_kv - 1, w.top_m)
    needles = needle_table(w, 0)
    recall = np.isin(needles, sel[:s]).mean()
    assert recall >= 0.99, (recall, needles, sel)
