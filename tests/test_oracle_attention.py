"""Pins of the oracle's sparse attention stage: dense attention through a
library routine (torch scaled_dot_product_attention) when every token is kept,
closed forms for one and two tokens, and the empty selection."""
import math

import numpy as np
import torch

import oracle as O


def test_all_tokens_equals_library_sdpa():
    rng = np.random.default_rng(0)
    N = 777
    q = rng.standard_normal(128).astype(np.float16)
    k = rng.standard_normal((N, 128)).astype(np.float16)
    v = rng.standard_normal((N, 128)).astype(np.float16)
    out, lse = O.sparse_attention(q, k, v)
    qt = torch.from_numpy(q.astype(np.float32)).view(1, 1, 1, 128)
    kt = torch.from_numpy(k.astype(np.float32)).view(1, 1, N, 128)
    vt = torch.from_numpy(v.astype(np.float32)).view(1, 1, N, 128)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).view(128).numpy()
    np.testing.assert_allclose(out, ref, atol=2e-6)
    s = (kt.view(N, 128) @ qt.view(128)) / math.sqrt(128)
    assert abs(lse - float(torch.logsumexp(s.double(), 0))) < 1e-5


def test_one_and_two_token_closed_forms():
    rng = np.random.default_rng(1)
    q = rng.standard_normal(128).astype(np.float16)
    k = rng.standard_normal((2, 128)).astype(np.float16)
    v = rng.standard_normal((2, 128)).astype(np.float16)
    out, lse = O.sparse_attention(q, k[:1], v[:1])
    np.testing.assert_array_equal(out, v[0].astype(np.float64))
    s0 = math.fsum(float(a) * float(b) for a, b in zip(q, k[0])) / math.sqrt(128)
    assert abs(lse - s0) < 1e-12
    out2, lse2 = O.sparse_attention(q, k, v)
    s1 = math.fsum(float(a) * float(b) for a, b in zip(q, k[1])) / math.sqrt(128)
    a = 1.0 / (1.0 + math.exp(s1 - s0))
    np.testing.assert_allclose(out2, a * v[0].astype(np.float64) + (1 - a) * v[1].astype(np.float64),
                               atol=1e-12)
    assert abs(lse2 - (s0 + math.log1p(math.exp(s1 - s0)))) < 1e-12


def test_empty_selection():
    out, lse = O.sparse_attention(np.zeros(128, np.float16), np.zeros((0, 128), np.float16),
                                  np.zeros((0, 128), np.float16))
    assert np.all(out == 0) and lse == -math.inf
