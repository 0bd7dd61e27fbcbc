"""Pins of the oracle's Quest page metadata, page bound and top-k selection:
brute force on tiny inputs, the bound's defining property (it is >= q.k of
every key in the page), the one-token closed form, and a scalar re-derivation
of the fixed fp32 summation order through struct rounding."""
import math
import struct

import numpy as np
import pytest

import oracle as O


def _f32(x: float) -> float:
    return struct.unpack("<f", struct.pack("<f", x))[0]


def test_page_meta_brute_force_partial_page():
    rng = np.random.default_rng(0)
    L = 53                                   # 3 full pages + 5 tokens
    k = rng.standard_normal((64, 128)).astype(np.float16)
    k[60:] = np.float16(100.0)               # beyond the length: must be ignored
    meta = O.page_meta(k, L)
    assert meta.shape == (4, 2, 128)
    for pg in range(4):
        rows = range(pg * 16, min(L, pg * 16 + 16))
        for j in range(128):
            vals = [float(k[t, j]) for t in rows]
            key = lambda v: (v, math.copysign(1.0, v))
            assert float(meta[pg, 0, j]) == min(vals, key=key)
            assert float(meta[pg, 1, j]) == max(vals, key=key)
    assert np.all(meta[3, 1] < 100)


def _scalar_score(qh, meta_page):
    """Fixed-order fp32 sum done one rounding at a time (fp64 op, then fp32)."""
    t = []
    for j in range(128):
        a = _f32(float(qh[j]) * float(meta_page[0, j]))
        b = _f32(float(qh[j]) * float(meta_page[1, j]))
        t.append(max(a, b))
    c = []
    for ch in range(16):
        s = t[8 * ch]
        for j in range(1, 8):
            s = _f32(s + t[8 * ch + j])
        c.append(s)
    a = [_f32(c[i] + c[i + 8]) for i in range(8)]
    b = [_f32(a[i] + a[i + 4]) for i in range(4)]
    d = [_f32(b[i] + b[i + 2]) for i in range(2)]
    return _f32(d[0] + d[1])


@pytest.mark.parametrize("G", [1, 4])
def test_scores_match_scalar_order(G):
    rng = np.random.default_rng(G)
    k = rng.standard_normal((16 * 12, 128)).astype(np.float16)
    q = rng.standard_normal((G, 128)).astype(np.float16)
    meta = O.page_meta(k, k.shape[0])
    sc = O.quest_page_scores(q, meta)
    for pg in range(meta.shape[0]):
        tot = None
        for h in range(G):
            s = _scalar_score(q[h], meta[pg])
            tot = s if tot is None else _f32(tot + s)
        assert np.float32(tot).tobytes() == sc[pg].tobytes()


def test_score_upper_bounds_every_key_and_one_token_closed_form():
    rng = np.random.default_rng(5)
    k = (rng.standard_normal((16 * 40 + 7, 128)) * 2).astype(np.float16)
    q = rng.standard_normal((3, 128)).astype(np.float16)
    L = k.shape[0]
    meta = O.page_meta(k, L)
    sc = O.quest_page_scores(q, meta).astype(np.float64)
    qk = (k.astype(np.float64) @ q.astype(np.float64).T).sum(1)     # group sum of q_h.k
    for pg in range(meta.shape[0]):
        rows = slice(pg * 16, min(L, pg * 16 + 16))
        exact = sum(math.fsum(max(float(q[h, j]) * float(meta[pg, 0, j]),
                                  float(q[h, j]) * float(meta[pg, 1, j])) for j in range(128))
                    for h in range(3))
        assert abs(sc[pg] - exact) <= 1e-5 * max(1.0, abs(exact))
        assert exact >= qk[rows].max() - 1e-9
    # the last page has 7 tokens; a single-token page's bound is q.k itself
    one = O.page_meta(k[:1], 1)
    s1 = O.quest_page_scores(q[:1], one)[0]
    assert abs(float(s1) - float(k[0].astype(np.float64) @ q[0].astype(np.float64))) < 1e-4


def test_select_pages_brute_force_ties_and_order():
    rng = np.random.default_rng(9)
    for trial in range(50):
        P = int(rng.integers(1, 40))
        sc = rng.integers(-3, 4, size=P).astype(np.float32)   # many ties
        budget = int(rng.integers(1, 48)) * 16 + int(rng.integers(0, 16))
        got = O.select_pages(sc, budget).tolist()
        kp = min(budget // 16, P)
        ranked = sorted(range(P), key=lambda i: (-float(sc[i]), i))
        assert got == sorted(ranked[:kp])
        assert got == sorted(got)
    # budget >= context keeps every page
    assert O.select_pages(np.zeros(5, np.float32), 5 * 16).tolist() == [0, 1, 2, 3, 4]
    assert O.select_pages(np.zeros(5, np.float32), 10 ** 6).tolist() == [0, 1, 2, 3, 4]


def test_negative_zero_score_ties_plain_zero():
    sc = np.array([0.0, -0.0, 1.0, -0.0], np.float32)
    assert O.select_pages(sc, 3 * 16).tolist() == [0, 1, 2]


def test_candidate_tokens_partial_last_page():
    assert O.candidate_tokens(np.array([0, 3]), 55).tolist() == list(range(16)) + list(range(48, 55))
    assert O.candidate_tokens(None, 5).tolist() == [0, 1, 2, 3, 4]
    assert O.candidate_tokens(np.array([], np.int64), 5).tolist() == []
