"""GPU parity of the incremental decode append (tw_append_keys and the step's
append_keys option): after building the int4 cache and page metadata for
shorter lengths and appending tokens one at a time, the cache must equal the
CPU oracle's from-scratch build for the final lengths bit for bit."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from _parity import gpu_meta, gpu_rows, np16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from adaptive_top_sparse_quest_b200 import _capi, build
    build.build()
    _capi.load()


def _start_lengths(final, steps):
    """Start lengths `steps` tokens short of the final ones (at least 0), with
    the boundary cases forced in: a sequence starting empty, one starting on a
    page boundary and one starting mid-page."""
    start = [max(0, int(x) - steps) for x in final]
    if len(start) > 1:
        start[1] = 0
    if len(start) > 2 and final[2] > 32:
        start[2] = 32 - steps % 16 if steps < 32 else 16
    return start


def _check_cache(w, codes, scales, zeros, meta, key_bits=4):
    x = O.SeqInputs.from_workload(w)
    table = x.page_table
    for b in range(w.B):
        L = int(w.seq_lens[b])
        for hk in range(w.Hk):
            ks = O.sequence_rows(x.k, table, b, hk, L)
            rc, rs, rz = O.quantize_keys(ks, key_bits)
            assert np.array_equal(gpu_rows(codes, table, b, hk, L), rc), (b, hk)
            assert np.array_equal(gpu_rows(scales, table, b, hk, L).view(np.uint16),
                                  rs.view(np.uint16)), (b, hk)
            assert np.array_equal(gpu_rows(zeros, table, b, hk, L).view(np.uint16),
                                  rz.view(np.uint16)), (b, hk)
            assert np.array_equal(gpu_meta(meta, table, b, hk, L).view(np.uint16),
                                  O.page_meta(ks, L).view(np.uint16)), (b, hk)


CASES = [
    dict(seed=41, B=4, Hq=4, Hk=2, N=300, paged=False, steps=1, bits=4),
    dict(seed=42, B=4, Hq=8, Hk=2, N=400, paged=True, steps=1, bits=4),
    dict(seed=43, B=3, Hq=4, Hk=4, N=500, paged=False, steps=37, bits=4),
    dict(seed=44, B=5, Hq=8, Hk=1, N=700, paged=True, steps=40, bits=4),
    dict(seed=46, B=4, Hq=4, Hk=2, N=300, paged=False, steps=1, bits=2),
    dict(seed=47, B=5, Hq=8, Hk=1, N=700, paged=True, steps=40, bits=2),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"s{c['seed']}")
def test_append_matches_rebuild(c):
    from adaptive_top_sparse_quest_b200 import append_keys, prepare
    w = W.random_small(c["seed"], B=c["B"], Hq=c["Hq"], Hk=c["Hk"], N=c["N"], paged=c["paged"],
                       budget_tokens=None, min_len=0)
    final = [int(x) for x in w.seq_lens]
    start = _start_lengths(final, c["steps"])
    w0 = dataclasses.replace(w, seq_lens=torch.tensor(start, dtype=torch.int32))
    kv, keys, meta, _ = prepare(w0, "cuda", c["bits"])
    fin = torch.tensor(final, dtype=torch.int32, device="cuda")
    for _ in range(max(f - s for f, s in zip(final, start))):
        torch.minimum(kv.seq_lens + 1, fin, out=kv.seq_lens)
        append_keys(kv, keys, meta)
    torch.cuda.synchronize()
    assert [int(x) for x in kv.seq_lens.cpu()] == final
    _check_cache(w, np16(keys.codes), np16(keys.scales), np16(keys.zeros), np16(meta), c["bits"])


def test_step_with_append_equals_append_then_step():
    from adaptive_top_sparse_quest_b200 import DecodeStep, append_keys, prepare
    w = W.random_small(45, B=3, Hq=8, Hk=2, N=900, paged=True, budget_tokens=256,
                       group_mode=1, min_len=40)
    final = [int(x) for x in w.seq_lens]
    start = [f - 1 for f in final]
    w0 = dataclasses.replace(w, seq_lens=torch.tensor(start, dtype=torch.int32))
    # fused: the step appends the newest token itself
    kv, keys, meta, q = prepare(w0, "cuda")
    kv.seq_lens += 1
    fused = DecodeStep(kv, keys, meta, w.Hq, 256, w.p, 1, append_keys=True)
    fused(q)
    assert fused.kernel_names()[0] == "append_keys"
    # separate: append, then a plain step
    kv2, keys2, meta2, q2 = prepare(w0, "cuda")
    kv2.seq_lens += 1
    append_keys(kv2, keys2, meta2)
    plain = DecodeStep(kv2, keys2, meta2, w.Hq, 256, w.p, 1)
    plain(q2)
    torch.cuda.synchronize()
    for a, b in [(keys.codes, keys2.codes), (keys.scales, keys2.scales),
                 (keys.zeros, keys2.zeros), (meta, meta2), (fused.count, plain.count),
                 (fused.out, plain.out)]:
        assert torch.equal(a, b)
    n = fused.count.cpu()
    for s in range(n.numel()):
        assert torch.equal(fused.idx[s, :n[s]], plain.idx[s, :n[s]])
    _check_cache(w, np16(keys.codes), np16(keys.scales), np16(keys.zeros), np16(meta))
