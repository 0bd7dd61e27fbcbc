"""The oracle's end-to-end unit on small seeded workloads: layout independence
(the same sequences stored contiguously and as a shuffled page pool give the
same results), p = 1 reproducing dense attention over the candidate set, and the
candidate set obeying the page budget."""
import math

import numpy as np
import torch

import oracle as O
import workloads as W


def _to_paged(x: O.SeqInputs, seed: int) -> O.SeqInputs:
    rng = np.random.default_rng(seed)
    B, Hk = x.k.shape[0], x.k.shape[1]
    pages = [(int(L) + 15) // 16 for L in x.seq_lens]
    total = sum(pages)
    perm = rng.permutation(total)
    pool_k = np.zeros((total, Hk, 16, 128), np.float16)
    pool_v = np.zeros_like(pool_k)
    table = np.zeros((B, max(pages)), np.int64)
    off = 0
    for b in range(B):
        for pg in range(pages[b]):
            dst = perm[off + pg]
            table[b, pg] = dst
            seg_k = x.k[b, :, pg * 16:(pg + 1) * 16]
            pool_k[dst, :, :seg_k.shape[1]] = seg_k
            pool_v[dst, :, :seg_k.shape[1]] = x.v[b, :, pg * 16:(pg + 1) * 16]
        off += pages[b]
    return O.SeqInputs(x.q, pool_k, pool_v, x.seq_lens, table)


def test_layout_independence_and_budget():
    w = W.random_small(5, B=3, Hq=4, Hk=2, N=300, budget_tokens=96, group_mode=1)
    x = O.SeqInputs.from_workload(w)
    xp = _to_paged(x, 1)
    r1 = O.oracle_decode(x, w.budget_tokens, 0.85, 1)
    r2 = O.oracle_decode(xp, w.budget_tokens, 0.85, 1)
    for u in r1:
        np.testing.assert_array_equal(r1[u]["codes"], r2[u]["codes"])
        np.testing.assert_array_equal(r1[u]["meta"], r2[u]["meta"])
        np.testing.assert_array_equal(r1[u]["pages"], r2[u]["pages"])
        for h in r1[u]["sel_tokens"]:
            np.testing.assert_array_equal(r1[u]["sel_tokens"][h], r2[u]["sel_tokens"][h])
            np.testing.assert_array_equal(r1[u]["out"][h], r2[u]["out"][h])
        L = r1[u]["len"]
        assert len(r1[u]["pages"]) == min(96 // 16, (L + 15) // 16)
        assert len(r1[u]["cand_tokens"]) <= 96


def test_p1_is_dense_attention_over_candidates():
    w = W.random_small(6, B=2, Hq=2, Hk=2, N=200, budget_tokens=None)
    x = O.SeqInputs.from_workload(w)
    r = O.oracle_decode(x, None, 1.0, 0)
    for (b, hk), res in r.items():
        L = res["len"]
        assert res["sel_tokens"][hk].tolist() == list(range(L))
        qt = torch.from_numpy(x.q[b, hk].astype(np.float32)).view(1, 1, 1, 128)
        kt = torch.from_numpy(x.k[b, hk, :L].astype(np.float32)).view(1, 1, L, 128)
        vt = torch.from_numpy(x.v[b, hk, :L].astype(np.float32)).view(1, 1, L, 128)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).view(128).numpy()
        np.testing.assert_allclose(res["out"][hk], ref, atol=2e-6)


def test_heavy_keys_are_kept():
    w = W.tiny(device="cpu", N=1024, n_heavy=4)
    x = O.SeqInputs.from_workload(w)
    r = O.oracle_decode(x, None, 0.85, 0)[(0, 0)]
    assert set(w.heavy[(0, 0)]) <= set(r["sel_tokens"][0].tolist())
    assert 0 < r["kstar"][0] < 1024


def test_workload_generator_is_seeded():
    a = W.random_small(3, paged=True)
    b = W.random_small(3, paged=True)
    assert torch.equal(a.k, b.k) and torch.equal(a.page_table, b.page_table)
    assert torch.equal(a.seq_lens, b.seq_lens)
