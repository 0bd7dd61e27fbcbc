"""Pins of the oracle's token-level label-channel base selector (the synthetic
Double-Sparsity-style selector) against things other than the oracle itself:
exact integer arithmetic done with Python ints, brute-force sorting, invariances
that hold when every sum is exact, and the degenerate budgets."""
import itertools

import numpy as np
import pytest

import oracle as O
import workloads as W


def _int_case(seed, T=60, G=2, r=5, lo=-6, hi=7):
    """Integer-valued fp16 queries and keys: every product and partial sum of a
    label score is a small integer, so fp32 holds it exactly."""
    rng = np.random.default_rng(seed)
    k = rng.integers(lo, hi, (T, 128)).astype(np.float16)
    q = rng.integers(lo, hi, (G, 128)).astype(np.float16)
    ch = rng.choice(128, r, replace=False)
    return q, k, ch


def _brute_scores(q, k, ch):
    return [sum(int(q[h, c]) * int(k[t, c]) for h in range(q.shape[0]) for c in ch)
            for t in range(k.shape[0])]


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_scores_and_selection_match_integer_brute_force(seed):
    q, k, ch = _int_case(seed)
    lab = O.label_cache(k, ch)
    assert lab.shape == (k.shape[0], len(ch))
    assert np.array_equal(lab, k[:, ch])
    s = O.label_scores(q, lab, ch)
    ref = _brute_scores(q, k, ch)
    assert s.dtype == np.float32 and [int(v) for v in s] == ref
    for budget in (1, 7, 30, 59):
        got = O.select_tokens(s, budget).tolist()
        want = sorted(sorted(range(len(ref)), key=lambda t: (-ref[t], t))[:budget])
        assert got == want, budget


def test_channel_order_and_head_order_do_not_change_exact_scores():
    q, k, ch = _int_case(4, G=4)
    base = O.label_scores(q, O.label_cache(k, ch), ch)
    for perm in itertools.islice(itertools.permutations(range(len(ch))), 0, 24, 5):
        c2 = ch[list(perm)]
        assert np.array_equal(O.label_scores(q, O.label_cache(k, c2), c2), base)
    assert np.array_equal(O.label_scores(q[::-1], O.label_cache(k, ch), ch), base)


def test_ties_go_to_the_lower_token_index():
    k = np.zeros((40, 128), np.float16)
    k[:, 3] = 1.0
    k[[5, 17, 33], 3] = 2.0
    q = np.zeros((1, 128), np.float16)
    q[0, 3] = 1.0
    s = O.label_scores(q, O.label_cache(k, [3]), [3])
    assert O.select_tokens(s, 3).tolist() == [5, 17, 33]
    assert O.select_tokens(s, 5).tolist() == [0, 1, 5, 17, 33]


def test_budget_at_least_length_keeps_every_token():
    q, k, ch = _int_case(5, T=23)
    s = O.label_scores(q, O.label_cache(k, ch), ch)
    assert O.select_tokens(s, 23).tolist() == list(range(23))
    assert O.select_tokens(s, 1000).tolist() == list(range(23))
    assert O.select_tokens(s[:0], 16).tolist() == []


def test_all_channels_rank_like_exact_dot_products():
    """With every channel a label channel the score is q . k summed in fp32;
    its ranking agrees with the exact fp64 ranking except between keys whose
    exact scores lie closer than the fp32 error bound."""
    rng = np.random.default_rng(9)
    k = rng.standard_normal((300, 128)).astype(np.float16)
    q = rng.standard_normal((1, 128)).astype(np.float16)
    ch = np.arange(128)
    s = O.label_scores(q, O.label_cache(k, ch), ch).astype(np.float64)
    exact = k.astype(np.float64) @ q[0].astype(np.float64)
    bound = 128 * 2.0 ** -24 * (np.abs(k.astype(np.float64)) @ np.abs(q[0].astype(np.float64)))
    assert np.all(np.abs(s - exact) <= bound + 1e-12)
    sel = set(O.select_tokens(s, 50).tolist())
    ex = set(np.sort(np.argsort(-exact, kind="stable")[:50]).tolist())
    theta = np.sort(exact)[-50]
    for t in sel ^ ex:
        assert abs(exact[t] - theta) <= 2 * bound.max()


def test_oracle_unit_with_label_selector():
    """Through the whole oracle: the candidates are the selected tokens, p = 1
    keeps all of them, and the attention runs over them."""
    w = W.random_small(61, B=2, Hq=4, Hk=2, N=500, budget_tokens=96, group_mode=1)
    x = O.SeqInputs.from_workload(w)
    ch = W.label_channels(w, r=8)
    assert len(ch) == 2 and all(len(c) == 8 and len(set(c)) == 8 for c in ch)
    for b in range(2):
        for hk in range(2):
            r = O.oracle_unit(x, b, hk, 96, 1.0, 1, label_channels=ch)
            k_seq = O.sequence_rows(x.k, x.page_table, b, hk, r["len"])
            toks = O.select_tokens(
                O.label_scores(x.q[b, 2 * hk:2 * hk + 2], k_seq[:, ch[hk]], ch[hk]), 96)
            assert r["pages"] is None and r["cand_tokens"].tolist() == toks.tolist()
            assert len(toks) == min(96, r["len"])
            assert r["sel_tokens"][2 * hk].tolist() == toks.tolist()


def test_label_channels_put_planted_outliers_first():
    w = W.llama2_mha(N=256, H=2, budget_tokens=64)
    ch = W.label_channels(w, r=16)
    planted = w.heavy["outlier_channels"]
    assert all(c[:4] == planted and len(set(c)) == 16 for c in ch)
