"""The selection kernel's ring waits are bounded: a wait whose copies never
land gives up after 0.2 s, sets bit 0 of the caller's status word and lets the
kernel finish, so a logic error yields a reported error instead of a hung GPU.
The diagnostic entry point runs one such wait on an mbarrier that nothing
arrives on (no copy, no fault), then the context must still run the decode
step and match the oracle-checked result of an earlier run bit for bit."""
import time

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


def _step_out(w):
    from adaptive_top_sparse_quest_b200 import DecodeStep, prepare
    kv, keys, meta, q = prepare(w, "cuda")
    step = DecodeStep(kv, keys, meta, w.Hq, w.budget_tokens, w.p, w.group_mode)
    out = step(q).clone()
    torch.cuda.synchronize()
    return out, step.count.clone(), int(step.ws[:4].view(torch.int32).item())


def test_bounded_wait_gives_up_and_context_survives(lib):
    w = W.random_small(11, device="cuda")
    before, cnt_before, st0 = _step_out(w)
    assert st0 == 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    assert lib.tw_selftest_bounded_wait(status.data_ptr(), stream) == 0
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert int(status.item()) == 1          # gave up, and only that
    assert 0.15 < waited < 5.0              # the 0.2 s bound, not a hang
    after, cnt_after, st1 = _step_out(w)    # the context still runs the step
    assert st1 == 0
    assert torch.equal(cnt_before, cnt_after)
    assert torch.equal(before, after)
