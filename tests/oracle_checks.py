"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each ``check_*`` takes an ``oracle.Oracle`` and raises AssertionError on a
mismatch.  They run against the real oracle (tests/test_oracle_pins.py) and
against deliberately broken builds of it (tests/test_oracle_mutants.py), which
shows that a plausible mistake in any step fails at least one of them.

Independent references used here: exact integer / rational arithmetic in
numpy int64 and ``fractions``, numpy ``lexsort`` for top-k, exhaustive subset
enumeration, PyTorch CPU fp64 ``scaled_dot_product_attention`` and
``logsumexp``, and closed forms of the candidate count.
"""
from __future__ import annotations

import itertools
import math
from fractions import Fraction

import numpy as np

from synth.workloads import int8_to_bf16_bits


def _ints(rng, shape, lo=-4, hi=4):
    return rng.integers(lo, hi + 1, size=shape).astype(np.int8)


def _bf(x_int8):
    return int8_to_bf16_bits(np.asarray(x_int8))


def _normal_bf16(rng, shape):
    x = rng.standard_normal(shape).astype(np.float32)
    u = x.view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def _bf16_to_f64(b):
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _order(scores_exact, idx):
    """Indices sorted by the selection order (score desc, index asc) via numpy lexsort."""
    scores_exact = np.asarray(scores_exact)
    idx = np.asarray(idx)
    return idx[np.lexsort((idx, -scores_exact))]


def _n_cand_closed_form(p, block, top_m, n_kv):
    c = p // block
    n_vis = c + 1
    s = min(top_m, n_vis)
    if s == n_vis:
        return p + 1
    return (s - 1) * block + (p % block) + 1


# ---------------------------------------------------------------- step 1: pooling

def check_pool_exact(O):
    """Block keys equal the exact rational mean of the integer keys (correctly rounded)."""
    rng = np.random.default_rng(11)
    for n_kv, d, block in [(200, 8, 16), (64, 4, 64), (100, 3, 7), (1, 5, 16), (37, 2, 1)]:
        k = _ints(rng, (n_kv, d))
        bk = O.block_pool(_bf(k), block)
        n_blk = -(-n_kv // block)
        assert bk.shape == (n_blk, d)
        for j in range(n_blk):
            rows = k[j * block:min(n_kv, (j + 1) * block)].astype(np.int64)
            cnt = rows.shape[0]
            for e in range(d):
                exact = Fraction(int(rows[:, e].sum()), cnt)
                assert bk[j, e] == float(exact), (n_kv, block, j, e, bk[j, e], exact)


# ---------------------------------------------------------------- steps 2-3: block top-m

def _block_case(rng, n_kv, d, block):
    k = _ints(rng, (n_kv, d))
    q = _ints(rng, (d,))
    return q, k


def check_block_scores_exact(O):
    """Scores of the selected blocks equal q . (S_j / cnt_j) computed exactly."""
    rng = np.random.default_rng(12)
    for n_kv, d, block, m in [(300, 8, 16, 5), (130, 4, 8, 3), (64, 6, 4, 8)]:
        q, k = _block_case(rng, n_kv, d, block)
        bk = O.block_pool(_bf(k), block)
        for p in range(0, n_kv, 7):
            sel, s, sc = O.block_topm(_bf(q), bk, block, p, m, scores=True)
            for r in range(s):
                j = sel[r]
                rows = k[j * block:min(n_kv, (j + 1) * block)].astype(np.int64)
                exact = Fraction(int(q.astype(np.int64) @ rows.sum(0)), rows.shape[0])
                assert abs(Fraction(sc[r]) - exact) <= Fraction(1, 2**40), (p, j, sc[r], exact)


def check_block_topm_invariants(O):
    """Forced blocks present, size s, ascending, distinct, visible, -1 tail, threshold property."""
    rng = np.random.default_rng(13)
    for n_kv, d, block, m in [(500, 8, 16, 6), (257, 4, 8, 2), (96, 4, 32, 3), (1000, 6, 10, 9)]:
        q, k = _block_case(rng, n_kv, d, block)
        k64 = k.astype(np.int64)
        bk = O.block_pool(_bf(k), block)
        for p in list(range(0, n_kv, 11)) + [n_kv - 1]:
            c = p // block
            sel, s = O.block_topm(_bf(q), bk, block, p, m)
            assert s == min(m, c + 1), (p, s)
            chosen = sel[:s]
            assert np.all(sel[s:] == -1)
            assert np.all(np.diff(chosen) > 0), chosen
            assert chosen[0] == 0 and chosen[-1] == c, (p, chosen)
            assert np.all((chosen >= 0) & (chosen <= c))
            if s < c + 1:
                mids = np.arange(1, c)
                # full blocks only among 1..c-1, so ranking by q.S equals ranking by q.S/B
                score = np.array([int(q.astype(np.int64) @ k64[j * block:(j + 1) * block].sum(0)) for j in mids])
                want = np.sort(_order(score, mids)[: s - 2])
                assert np.array_equal(chosen[1:-1], want), (p, chosen, want)


def check_block_topm_bruteforce(O):
    """Tiny cases: the chosen set is the unique subset (with the forced blocks) whose every
    member beats every non-member under (score desc, index asc)."""
    rng = np.random.default_rng(14)
    for trial in range(6):
        block, d = 4, 3
        n_kv = int(rng.integers(20, 48))
        q, k = _block_case(rng, n_kv, d, block)
        # few distinct values -> many ties
        k = (k // 3).astype(np.int8)
        bk = O.block_pool(_bf(k), block)
        m = int(rng.integers(2, 6))
        for p in range(n_kv):
            c = p // block
            sel, s = O.block_topm(_bf(q), bk, block, p, m)
            mids = list(range(1, c))
            if s == c + 1:
                assert list(sel[:s]) == list(range(c + 1))
                continue
            score = {j: Fraction(int(q.astype(np.int64) @ k[j * block:(j + 1) * block].astype(np.int64).sum(0)),
                                 block) for j in mids}
            key = lambda j: (score[j], -j)  # noqa: E731  larger is better
            winners = []
            for sub in itertools.combinations(mids, s - 2):
                rest = [j for j in mids if j not in sub]
                ok = True
                if sub and rest:
                    ok = min(key(j) for j in sub) > max(key(j) for j in rest)
                if ok:
                    winners.append(sub)
            assert len(winners) == 1, (p, winners)
            assert list(sel[:s]) == [0, *winners[0], c], (p, sel, winners)


# ---------------------------------------------------------------- steps 4-5: token top-k

def _flat_reference(q, k, p, top_k):
    scores = k[: p + 1].astype(np.int64) @ q.astype(np.int64)
    t = np.arange(p + 1)
    best = np.sort(_order(scores, t)[:top_k])
    out = np.full(top_k, -1, dtype=np.int64)
    out[: len(best)] = best
    return out, scores


def check_flat_topk_lexsort(O):
    """Flat top-k equals numpy lexsort top-k on exact integer scores; scores exact."""
    rng = np.random.default_rng(15)
    for n_kv, d, top_k in [(300, 8, 17), (64, 4, 64), (50, 3, 1), (129, 2, 200)]:
        k = (_ints(rng, (n_kv, d)) // 2).astype(np.int8)  # heavy ties
        q = _ints(rng, (d,))
        for p in range(0, n_kv, 5):
            tok, k_eff, sc = O.flat_topk(_bf(q), _bf(k), p, top_k, scores=True)
            want, scores = _flat_reference(q, k, p, top_k)
            assert k_eff == min(top_k, p + 1)
            assert np.array_equal(tok, want), (p, tok, want)
            valid = tok >= 0
            assert np.array_equal(sc[valid], scores[tok[valid]].astype(np.float64))


def check_token_topk_candidates(O):
    """Token top-k over the selected blocks equals lexsort top-k over exactly the candidate
    set {t in selected blocks, t <= p}; candidate count equals the closed form."""
    rng = np.random.default_rng(16)
    for n_kv, d, block, m, top_k in [(700, 8, 16, 5, 40), (300, 4, 32, 3, 500), (257, 6, 8, 4, 9)]:
        q, k = _block_case(rng, n_kv, d, block)
        k = (k // 2).astype(np.int8)
        bk = O.block_pool(_bf(k), block)
        for p in list(range(0, n_kv, 9)) + [n_kv - 1]:
            sel, s = O.block_topm(_bf(q), bk, block, p, m)
            tok, k_eff, n_cand = O.token_topk(_bf(q), _bf(k), block, p, sel, top_k)
            cand = np.array([t for j in sel[:s] for t in range(j * block, min((j + 1) * block, p + 1, n_kv))])
            assert n_cand == len(cand) == _n_cand_closed_form(p, block, m, n_kv), (p, n_cand, len(cand))
            scores = k[cand].astype(np.int64) @ q.astype(np.int64)
            want = np.sort(_order(scores, cand)[:top_k])
            assert k_eff == min(top_k, len(cand))
            assert np.array_equal(tok[:k_eff], want) and np.all(tok[k_eff:] == -1), (p, tok, want)


def check_degeneration(O):
    """With m >= number of visible blocks the two-level result equals the flat indexer's
    (the short-context degeneration the pages state)."""
    rng = np.random.default_rng(17)
    for n_kv, d, block, top_k in [(400, 8, 16, 30), (128, 4, 64, 128), (90, 5, 7, 12)]:
        q, k = _block_case(rng, n_kv, d, block)
        k = (k // 2).astype(np.int8)
        m = -(-n_kv // block)
        bk = O.block_pool(_bf(k), block)
        for p in range(0, n_kv, 3):
            sel, s = O.block_topm(_bf(q), bk, block, p, m)
            tok, _, _ = O.token_topk(_bf(q), _bf(k), block, p, sel, top_k)
            flat, _ = O.flat_topk(_bf(q), _bf(k), p, top_k)
            assert np.array_equal(tok, flat), p


def check_constructed_ranking(O):
    """Hand-constructed case with a known answer: q = e_0 and block j's keys all carry
    first coordinate v_j; the block ranking is the ranking of v_j, and the token ranking
    inside the kept blocks follows the per-token first coordinate."""
    block, d, n_blk = 4, 3, 9
    v = np.array([0, 3, -2, 4, 4, 1, -4, 2, 0], dtype=np.int64)  # block values
    k = np.zeros((n_blk * block, d), dtype=np.int8)
    for j in range(n_blk):
        k[j * block:(j + 1) * block, 0] = v[j]
    k[:, 1] = 1  # ignored by q
    q = np.array([1, 0, 0], dtype=np.int8)
    bk = O.block_pool(_bf(k), block)
    p = n_blk * block - 1  # own block 8
    # m = 4: forced {0, 8}; best two of blocks 1..7 by value: v3 = v4 = 4 (tie -> lower ids 3, 4)
    sel, s = O.block_topm(_bf(q), bk, block, p, 4)
    assert s == 4 and list(sel) == [0, 3, 4, 8], sel
    # m = 5: next best is block 1 (value 3)
    sel5, _ = O.block_topm(_bf(q), bk, block, p, 5)
    assert list(sel5) == [0, 1, 3, 4, 8], sel5
    # tokens: all tokens of blocks 3 and 4 score 4; top-6 of {0..3, 12..19, 32..35}
    tok, k_eff, n_cand = O.token_topk(_bf(q), _bf(k), block, p, sel, 6)
    assert n_cand == 16 and k_eff == 6
    assert list(tok) == [12, 13, 14, 15, 16, 17], tok
    # query at p = 9 (own block 2, value -2): m = 2 keeps {0, 2}; candidates 0..3, 8, 9
    sel2, s2 = O.block_topm(_bf(q), bk, block, 9, 2)
    assert list(sel2) == [0, 2] and s2 == 2
    tok2, k2, nc2 = O.token_topk(_bf(q), _bf(k), block, 9, sel2, 5)
    assert nc2 == 6 and k2 == 5 and list(tok2) == [0, 1, 2, 3, 8], tok2


# ---------------------------------------------------------------- step 6: attention

def _sdpa_dense(q, k, v, scale):
    import torch

    qt = torch.from_numpy(q).permute(1, 0, 2)[None]  # [1][H][n][d]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2)[None]
    if kt.shape[1] != qt.shape[1]:
        rep = qt.shape[1] // kt.shape[1]
        kt = kt.repeat_interleave(rep, dim=1)
        vt = vt.repeat_interleave(rep, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    s = (qt @ kt.transpose(-1, -2)) * scale
    n = s.shape[-1]
    s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o[0].permute(1, 0, 2).numpy(), lse[0].permute(1, 0).numpy()


def check_dense_equivalence(O):
    """k >= n_kv and m >= n_blk: the path equals dense causal softmax attention
    (PyTorch CPU fp64 SDPA) for every query, output and log-sum-exp."""
    from synth.workloads import Workload

    rng = np.random.default_rng(18)
    for n, d_idx, block, h, hkv, d in [(70, 4, 8, 2, 2, 16), (33, 3, 16, 4, 2, 8)]:
        w = Workload("t", 1, n, n, d_idx, block, -(-n // block), n, h, hkv, d)
        inp = {"q_idx": _bf(_ints(rng, (1, n, d_idx))), "k_idx": _bf(_ints(rng, (1, n, d_idx))),
               "q": _normal_bf16(rng, (1, n, h, d)), "k": _normal_bf16(rng, (1, n, hkv, d)),
               "v": _normal_bf16(rng, (1, n, hkv, d))}
        r = O.run(w, inp)
        for i in range(n):
            assert np.array_equal(r["token_idx"][i][: i + 1], np.arange(i + 1))
        scale = 1.0 / math.sqrt(d)
        o_ref, lse_ref = _sdpa_dense(_bf16_to_f64(inp["q"][0]), _bf16_to_f64(inp["k"][0]),
                                     _bf16_to_f64(inp["v"][0]), scale)
        assert np.max(np.abs(r["o"] - o_ref)) < 1e-10
        assert np.max(np.abs(r["lse"] - lse_ref)) < 1e-10


def check_attention_special_cases(O):
    """k = 1 gives the selected V row exactly; Q = 0 gives the mean of the selected V rows;
    permuting the index list leaves the result unchanged."""
    rng = np.random.default_rng(19)
    n, h, d = 50, 3, 16
    k = _normal_bf16(rng, (n, h, d))
    v = _normal_bf16(rng, (n, h, d))
    q = _normal_bf16(rng, (h, d))
    o, lse = O.sparse_attn(q, k, v, np.array([17], dtype=np.int32))
    assert np.array_equal(o, _bf16_to_f64(v[17]))
    qk = (_bf16_to_f64(q) * _bf16_to_f64(k[17])).sum(-1) / math.sqrt(d)
    assert np.max(np.abs(lse - qk)) < 1e-12
    sel = np.array([3, 9, 10, 31, 44, -1, -1], dtype=np.int32)
    o0, lse0 = O.sparse_attn(np.zeros_like(q), k, v, sel)
    assert np.max(np.abs(o0 - _bf16_to_f64(v[sel[:5]]).mean(0))) < 1e-12
    assert np.max(np.abs(lse0 - math.log(5))) < 1e-12
    o1, l1 = O.sparse_attn(q, k, v, sel)
    perm = sel.copy()
    perm[:5] = perm[:5][::-1]
    o2, l2 = O.sparse_attn(q, k, v, perm[[0, 5, 1, 2, 6, 3, 4]])
    assert np.max(np.abs(o1 - o2)) < 1e-12 and np.max(np.abs(l1 - l2)) < 1e-12
    # GQA mapping: head h reads kv head h // (H / H_kv)
    kk = _normal_bf16(rng, (n, 1, d))
    vv = _normal_bf16(rng, (n, 1, d))
    og, _ = O.sparse_attn(q, kk, vv, np.array([5], dtype=np.int32))
    for hh in range(h):
        assert np.array_equal(og[hh], _bf16_to_f64(vv[5, 0]))


# ---------------------------------------------------------------- the multi-head indexer score

def _mh_case(rng, n_kv, d, heads):
    q = _ints(rng, (heads, d))
    k = _ints(rng, (n_kv, d))
    w = rng.choice(np.array([-2.0, -1.0, 1.0, 2.0, 3.0]), size=heads)
    return q, k, w


def _mh_score_int(q, w, key_int):
    """sum_j w_j * max(0, q_j . key) in exact integer arithmetic (int64)."""
    dots = q.astype(np.int64) @ key_int.astype(np.int64)
    return sum(int(w[j]) * max(0, int(dots[j])) for j in range(len(w)))


def check_multihead_token_scores_bruteforce(O):
    """Token scores and top-k of the multi-head indexer equal a brute-force integer evaluation of
    sum_j w_j * ReLU(q_j . k) ranked by numpy lexsort."""
    rng = np.random.default_rng(31)
    for heads, n_kv, block, top_m, top_k in [(1, 90, 8, 4, 17), (3, 200, 16, 5, 40), (8, 130, 32, 3, 64)]:
        d = 16
        q, k, w = _mh_case(rng, n_kv, d, heads)
        p = n_kv - 1
        sel = np.arange(0, -(-n_kv // block), dtype=np.int32)  # every block: all tokens are candidates
        sel_m = np.full(len(sel), -1, dtype=np.int32)
        sel_m[: len(sel)] = sel
        tok, k_eff, _, sc = O.token_topk(_bf(q), _bf(k), block, p, sel_m, top_k, scores=True, w=w)
        exact = np.array([_mh_score_int(q, w, k[t]) for t in range(n_kv)])
        want = np.sort(_order(exact, np.arange(n_kv))[:top_k])
        assert k_eff == min(top_k, n_kv)
        assert np.array_equal(tok[:k_eff], want), (heads, tok[:k_eff], want)
        assert np.array_equal(sc[:k_eff], exact[tok[:k_eff]].astype(np.float64))


def check_multihead_block_scores_exact(O):
    """Block scores of the multi-head indexer equal sum_j w_j * ReLU(q_j . mean) in exact rational
    arithmetic, and the kept blocks are the forced pair plus the best m-2 by those scores."""
    rng = np.random.default_rng(37)
    for heads, n_kv, block, top_m in [(2, 300, 16, 6), (5, 257, 8, 9)]:
        d = 8
        q, k, w = _mh_case(rng, n_kv, d, heads)
        bk = O.block_pool(_bf(k), block)
        p = n_kv - 1
        c = p // block
        sel, s_, sc = O.block_topm(_bf(q), bk, block, p, top_m, scores=True, w=w)
        exact = []
        for j in range(c + 1):
            t0, t1 = j * block, min(n_kv, (j + 1) * block)
            mean = [Fraction(int(k[t0:t1, e].sum()), t1 - t0) for e in range(d)]
            sj = sum(Fraction(int(w[h])) * max(Fraction(0), sum(int(q[h, e]) * mean[e] for e in range(d)))
                     for h in range(heads))
            exact.append(sj)
        mid = _order(np.array([float(x) for x in exact[1:c]]), np.arange(1, c))[: s_ - 2]
        assert np.array_equal(sel[:s_], np.sort(np.concatenate([[0, c], mid]))), (sel, mid)
        for r in range(s_):
            assert sc[r] == float(exact[sel[r]])


def check_multihead_reduces_to_dot_product(O):
    """One head with weight 1 and non-negative inputs (so every dot product is >= 0 and the ReLU
    is the identity) selects exactly what the plain dot-product indexer selects."""
    rng = np.random.default_rng(41)
    n_kv, d, block, top_m, top_k = 400, 16, 16, 6, 50
    q = _ints(rng, (d,), 0, 4)
    k = _ints(rng, (n_kv, d), 0, 4)
    bk = O.block_pool(_bf(k), block)
    p = n_kv - 1
    sel_plain, _ = O.block_topm(_bf(q), bk, block, p, top_m)
    sel_mh, _ = O.block_topm(_bf(q[None]), bk, block, p, top_m, w=np.array([1.0]))
    assert np.array_equal(sel_plain, sel_mh)
    tok_plain, _, _ = O.token_topk(_bf(q), _bf(k), block, p, sel_plain, top_k)
    tok_mh, _, _ = O.token_topk(_bf(q[None]), _bf(k), block, p, sel_plain, top_k, w=np.array([1.0]))
    assert np.array_equal(tok_plain, tok_mh)


ALL_CHECKS = [
    check_pool_exact,
    check_block_scores_exact,
    check_block_topm_invariants,
    check_block_topm_bruteforce,
    check_flat_topk_lexsort,
    check_token_topk_candidates,
    check_degeneration,
    check_constructed_ranking,
    check_dense_equivalence,
    check_attention_special_cases,
    check_multihead_token_scores_bruteforce,
    check_multihead_block_scores_exact,
    check_multihead_reduces_to_dot_product,
]
