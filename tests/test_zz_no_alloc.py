"""The allocation-free top-p entry point (tw_topp_prune_noalloc).

Callers such as a runtime that records the decode step into a CUDA graph with
allocation forbidden, or a plugin whose enqueue hook may not allocate, cannot
hand the library a workspace; this entry point keeps its scratch in a fixed
array inside the library.  It must give the same selection as tw_topp_prune
with a caller workspace, on two calls in a row (the shared array keeps the
previous call's contents), and reject shapes whose scratch does not fit.
Collected last on purpose: it runs after every other test, and also alone."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from adaptive_top_sparse_quest_b200 import _capi, build
    build.build()
    return _capi.load()


def _noalloc(lib, q, kv, keys, cand, ncand, p, gm, capacity, U):
    idx = torch.full((U, capacity), -7, dtype=torch.int32, device=q.device)
    count = torch.full((U,), -7, dtype=torch.int32, device=q.device)
    s = kv.struct()
    st = lib.tw_topp_prune_noalloc(q.data_ptr(), q.shape[1], ctypes.byref(s),
                                   keys.codes.data_ptr(), keys.scales.data_ptr(),
                                   keys.zeros.data_ptr(),
                                   None if cand is None else cand.data_ptr(),
                                   0 if cand is None else cand.shape[-1],
                                   None if ncand is None else ncand.data_ptr(), p, gm,
                                   idx.data_ptr(), capacity, count.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    return st, idx, count


@pytest.mark.parametrize("case", [
    dict(seed=31, B=2, Hq=8, Hk=2, N=1500, paged=True, budget=512, p=0.85, gm=1),
    dict(seed=32, B=2, Hq=4, Hk=4, N=3000, paged=False, budget=None, p=0.9, gm=0),
])
def test_noalloc_matches_workspace_call_twice(lib, case):
    from adaptive_top_sparse_quest_b200 import _capi, prepare, select_pages, topp_prune
    w = W.random_small(case["seed"], B=case["B"], Hq=case["Hq"], Hk=case["Hk"], N=case["N"],
                       paged=case["paged"], budget_tokens=case["budget"], p=case["p"],
                       group_mode=case["gm"])
    kv, keys, meta, q = prepare(w, "cuda")
    cand = ncand = None
    if case["budget"]:
        cand, ncand = select_pages(q, kv, meta, case["budget"])
    idx_ref, cnt_ref = topp_prune(q, kv, keys, cand, ncand, case["p"], case["gm"])
    torch.cuda.synchronize()
    U, capacity = idx_ref.shape
    for _ in range(2):
        st, idx, cnt = _noalloc(lib, q, kv, keys, cand, ncand, case["p"], case["gm"], capacity, U)
        assert st == _capi.TW_OK, lib.tw_status_string(st)
        torch.cuda.synchronize()
        c_ref = cnt_ref.cpu().numpy()
        assert np.array_equal(cnt.cpu().numpy(), c_ref)
        a, r = idx.cpu().numpy(), idx_ref.cpu().numpy()
        for u in range(U):
            assert np.array_equal(a[u, :c_ref[u]], r[u, :c_ref[u]])


def test_noalloc_rejects_oversized_scratch(lib):
    from adaptive_top_sparse_quest_b200 import _capi
    # B * Hk * capacity * G * 4 bytes of logits alone exceed the 8 MiB array
    s = _capi.TwKv()
    s.k = s.v = 1 << 20
    s.batch, s.num_kv_heads, s.max_seq_len = 8, 8, 65536
    s.page_size, s.head_dim = 16, 128
    p = 1 << 20
    st = lib.tw_topp_prune_noalloc(p, 8, ctypes.byref(s), p, p, p, None, 0, None, 0.9, 1, p,
                                   65536, p, None)
    assert st == _capi.TW_ERR_CAPACITY


def _scratch_need(B, Hk, G, capacity):
    """Bytes of the array a call needs: a 256-byte status word, then the logits
    of the selection sets, B * Hk * G * lcap floats with lcap = capacity rounded
    up to a multiple of 64, the region rounded up to 256 bytes."""
    lcap = (capacity + 63) // 64 * 64
    return 256 + (B * Hk * G * lcap * 4 + 255) // 256 * 256


def test_noalloc_limit_just_above_is_rejected_on_the_host(lib):
    from adaptive_top_sparse_quest_b200 import _capi
    cap = 2097089   # lcap 2097152: 256 + 8 MiB, one region step over the array
    assert _scratch_need(1, 1, 1, cap) > 8 << 20
    s = _capi.TwKv()
    s.k = s.v = 1 << 20
    s.batch, s.num_kv_heads, s.max_seq_len = 1, 1, 4096
    s.page_size, s.head_dim = 16, 128
    p = 1 << 20
    st = lib.tw_topp_prune_noalloc(p, 1, ctypes.byref(s), p, p, p, None, 0, None, 0.9, 0, p,
                                   cap, p, None)
    assert st == _capi.TW_ERR_CAPACITY


def test_noalloc_limit_just_below_runs_and_matches(lib):
    """capacity 2097088 needs exactly the 8 MiB of the array and must run."""
    from adaptive_top_sparse_quest_b200 import _capi, prepare, topp_prune
    cap = 2097088
    assert _scratch_need(1, 1, 1, cap) == 8 << 20
    w = W.random_small(33, B=1, Hq=1, Hk=1, N=4096, budget_tokens=None, p=0.9, group_mode=0)
    kv, keys, meta, q = prepare(w, "cuda")
    idx_ref, cnt_ref = topp_prune(q, kv, keys, None, None, 0.9, 0, capacity=cap)
    for _ in range(2):
        st, idx, cnt = _noalloc(lib, q, kv, keys, None, None, 0.9, 0, cap, 1)
        assert st == _capi.TW_OK, lib.tw_status_string(st)
        torch.cuda.synchronize()
        n = int(cnt_ref[0])
        assert int(cnt[0]) == n
        assert torch.equal(idx[0, :n], idx_ref[0, :n])
