"""GPU check of tw_decode_step_host: the step with its query read from and its
output written to pinned host memory (copy kernels in the step's launch
chain) gives the same bits as the device-buffer step, step after step, and
rejects pageable host memory before launching anything."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from adaptive_top_sparse_quest_b200 import _capi, build
    build.build()
    _capi.load()


@pytest.mark.parametrize("paged,budget,gm", [(False, 512, 0), (True, 256, 1), (True, None, 1)])
def test_host_staged_step_matches_device_step(paged, budget, gm):
    from adaptive_top_sparse_quest_b200 import DecodeStep, prepare
    w = W.random_small(51, B=3, Hq=8, Hk=2, N=2000, paged=paged, budget_tokens=budget,
                       group_mode=gm)
    kv, keys, meta, q = prepare(w, "cuda")
    dev = DecodeStep(kv, keys, meta, w.Hq, budget, w.p, gm)
    host = DecodeStep(kv, keys, meta, w.Hq, budget, w.p, gm)
    rng = torch.Generator().manual_seed(5)
    out_host = torch.empty(tuple(q.shape), dtype=torch.float16).pin_memory()
    for i in range(4):   # a different query each step through the same buffers
        qi = (q.float().cpu() + 0.1 * i * torch.randn(q.shape, generator=rng)).half()
        q_host = qi.pin_memory()
        host.run_host(q_host, out_host)
        dev(qi.cuda())
        torch.cuda.synchronize()
        assert torch.equal(out_host, dev.out.cpu()), i
        assert torch.equal(host.lse, dev.lse) and torch.equal(host.count, dev.count), i
        assert torch.equal(host._q_stage.cpu(), qi), i


def test_host_staged_step_rejects_pageable_memory():
    from adaptive_top_sparse_quest_b200 import DecodeStep, _capi, prepare
    w = W.random_small(52, B=2, Hq=4, Hk=2, N=600, budget_tokens=128, group_mode=1)
    kv, keys, meta, q = prepare(w, "cuda")
    step = DecodeStep(kv, keys, meta, w.Hq, 128, w.p, 1)
    step(q)
    torch.cuda.synchronize()
    before = step.out.clone()
    s = step._struct(q)
    lib = _capi.load()
    pageable_q = np.zeros(q.numel() + 64, np.uint16)
    pageable_o = np.zeros(q.numel() + 64, np.uint16)
    qa = pageable_q.ctypes.data + (-pageable_q.ctypes.data) % 16
    oa = pageable_o.ctypes.data + (-pageable_o.ctypes.data) % 16
    pinned = torch.empty(tuple(q.shape), dtype=torch.float16).pin_memory()
    st = torch.cuda.current_stream().cuda_stream
    assert lib.tw_decode_step_host(ctypes.byref(s), qa, oa, st) == _capi.TW_ERR_INVALID_ARG
    assert lib.tw_decode_step_host(ctypes.byref(s), pinned.data_ptr(), oa, st) == \
        _capi.TW_ERR_INVALID_ARG
    assert lib.tw_decode_step_host(ctypes.byref(s), pinned.data_ptr() + 2, pinned.data_ptr(),
                                   st) == _capi.TW_ERR_INVALID_ARG     # misaligned
    assert lib.tw_decode_step_host(ctypes.byref(s), None, pinned.data_ptr(), st) == \
        _capi.TW_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.equal(step.out, before)   # nothing ran
    step(q)                                # and the stream is still usable
    torch.cuda.synchronize()
    assert torch.equal(step.out, before)
