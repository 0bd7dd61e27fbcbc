"""GPU parity of the token-level label-channel base selector (tw_label_cache,
tw_select_tokens, tw_topp_prune_tokens) against the CPU oracle: bit-exact
label cache and candidate token ids, the top-p selection and attention within
the same bars as the page path, at both key-cache widths."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from _parity import check_attention, compare_selection, np16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from adaptive_top_sparse_quest_b200 import _capi, build
    build.build()
    _capi.load()


def _setup(w, r, key_bits=4, seed=7):
    from adaptive_top_sparse_quest_b200 import label_cache, prepare
    kv, keys, meta, q = prepare(w, "cuda", key_bits)
    ch = W.label_channels(w, r=r, seed=seed)
    ch_t = torch.tensor(ch, dtype=torch.int32, device="cuda")
    labels = label_cache(kv, ch_t)
    return kv, keys, q, ch, ch_t, labels


CASES = [
    dict(seed=71, B=2, Hq=2, Hk=2, N=777, paged=False, budget=160, r=16, gm=0),
    dict(seed=72, B=3, Hq=8, Hk=2, N=1000, paged=True, budget=256, r=8, gm=1),
    dict(seed=73, B=2, Hq=8, Hk=2, N=3000, paged=False, budget=2500, r=32, gm=0),
    dict(seed=74, B=2, Hq=8, Hk=1, N=5000, paged=True, budget=700, r=16, gm=1),
    dict(seed=75, B=4, Hq=4, Hk=4, N=333, paged=False, budget=48, r=4, gm=0),
    dict(seed=76, B=1, Hq=4, Hk=2, N=12000, paged=False, budget=9000, r=16, gm=1),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"s{c['seed']}")
@pytest.mark.parametrize("key_bits", [4, 2])
def test_label_path_parity(c, key_bits):
    from adaptive_top_sparse_quest_b200 import select_tokens, sparse_decode, topp_prune_tokens
    w = W.random_small(c["seed"], B=c["B"], Hq=c["Hq"], Hk=c["Hk"], N=c["N"], paged=c["paged"],
                       budget_tokens=c["budget"], group_mode=c["gm"])
    kv, keys, q, ch, ch_t, labels = _setup(w, c["r"], key_bits)
    cand, ncand = select_tokens(q, kv, labels, ch_t, c["budget"])
    idx, count = topp_prune_tokens(q, kv, keys, cand, ncand, w.p, c["gm"])
    out, lse = sparse_decode(q, kv, idx, count, c["gm"])
    torch.cuda.synchronize()
    x = O.SeqInputs.from_workload(w)
    G = w.Hq // w.Hk
    group_sets = c["gm"] == 1 or G == 1
    lab = np16(labels)
    cand_n, ncand_n, idx_n, count_n = np16(cand), np16(ncand), np16(idx), np16(count)
    out_n, lse_n = np16(out), np16(lse)
    cuts = sets = 0
    for b in range(w.B):
        for hk in range(w.Hk):
            res = O.oracle_unit(x, b, hk, c["budget"], w.p, c["gm"], key_bits=key_bits,
                                label_channels=ch)
            L = res["len"]
            k_seq = O.sequence_rows(x.k, x.page_table, b, hk, L)
            assert np.array_equal(O.sequence_rows(lab, x.page_table, b, hk, L).view(np.uint16),
                                  O.label_cache(k_seq, ch[hk]).view(np.uint16)), (b, hk)
            n = int(ncand_n[b, hk])
            assert cand_n[b, hk, :n].tolist() == res["cand_tokens"].tolist(), (b, hk)
            for hq in range(hk * G, (hk + 1) * G):
                s = b * w.Hk + hk if group_sets else b * w.Hq + hq
                toks = idx_n[s, :int(count_n[s])]
                if not group_sets or hq == hk * G:
                    near, cut = compare_selection(toks, res, hq, w.p)
                    cuts += cut
                    sets += 1
                check_attention(out_n[b, hq], float(lse_n[b, hq]), x, b, hq, toks, hk)
    assert cuts <= max(1, sets // 20)


def test_select_tokens_with_many_ties_is_exact():
    """Integer-valued keys on the label channels make most scores tie; the
    token ids must still equal the oracle's (ties to the lower index)."""
    from adaptive_top_sparse_quest_b200 import select_tokens
    w = W.random_small(77, B=2, Hq=4, Hk=2, N=4100, budget_tokens=1000, group_mode=1)
    w.k.copy_(torch.round(w.k.float() * 2).clamp(-3, 3).half())
    kv, keys, q, ch, ch_t, labels = _setup(w, 4)
    cand, ncand = select_tokens(q, kv, labels, ch_t, 1000)
    torch.cuda.synchronize()
    x = O.SeqInputs.from_workload(w)
    for b in range(w.B):
        for hk in range(w.Hk):
            L = int(x.seq_lens[b])
            k_seq = O.sequence_rows(x.k, x.page_table, b, hk, L)
            ref = O.select_tokens(O.label_scores(x.q[b, 2 * hk:2 * hk + 2],
                                                 O.label_cache(k_seq, ch[hk]), ch[hk]), 1000)
            n = int(ncand[b, hk])
            assert np16(cand)[b, hk, :n].tolist() == ref.tolist(), (b, hk)


def test_label_step_matches_single_calls():
    from adaptive_top_sparse_quest_b200 import (LabelDecodeStep, select_tokens, sparse_decode,
                                                topp_prune_tokens)
    w = W.random_small(78, B=2, Hq=8, Hk=2, N=2500, paged=True, budget_tokens=600, group_mode=1)
    kv, keys, q, ch, ch_t, labels = _setup(w, 16)
    step = LabelDecodeStep(kv, keys, labels, ch_t, w.Hq, 600, w.p, 1)
    step(q)
    cand, ncand = select_tokens(q, kv, labels, ch_t, 600)
    idx, count = topp_prune_tokens(q, kv, keys, cand, ncand, w.p, 1)
    out, lse = sparse_decode(q, kv, idx, count, 1)
    torch.cuda.synchronize()
    assert torch.equal(step.count, count) and torch.equal(step.ncand, ncand)
    for s in range(count.shape[0]):
        n = int(count[s])
        assert torch.equal(step.idx[s, :n], idx[s, :n])
    assert torch.equal(step.out, out) and torch.equal(step.lse, lse)
