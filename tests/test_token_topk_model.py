"""A CPU model of the token top-k kernel's arithmetic (label-channel selector):
the 12 + 10 + 10-bit digit passes with each thread owning a contiguous run of
bins from the top, the scan that finds the crossing thread and digit, and the
in-order compaction (4 tokens per thread, 2048 per round) with its output
position g + min(e, need).  Checked against the oracle's token selection on
ragged sizes, heavy ties and -0 / +0.  It pins the kernel's design; the GPU
parity tests check the kernel itself."""
import numpy as np
import pytest

import oracle as O

def fkey(f):
    """Float -> uint32 key ordered like the value, -0 folded onto +0."""
    f = np.asarray(f, np.float32) + np.float32(0.0)
    u = f.view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)

def model_select(scores, budget, THREADS=512, PER=4):
    n = len(scores); K = min(budget, n)
    out = np.full(max(K, 1), -1, np.int64)
    if K <= 0: return out[:0]
    if K == n: return np.arange(n)
    keys = fkey(scores)
    prefix = 0; pmask = 0; need = K
    for sh, w in ((20, 12), (10, 10), (0, 10)):
        nb = 1 << w; dmask = nb - 1
        hist = np.zeros(nb, np.int64)
        m = (keys & pmask) == prefix
        np.add.at(hist, ((keys[m] >> sh) & dmask).astype(np.int64), 1)
        per = nb // THREADS
        mine = np.array([sum(hist[nb - tid * per - k] for k in range(1, per + 1)) for tid in range(THREADS)])
        above = np.concatenate([[0], np.cumsum(mine)[:-1]])
        hits = [tid for tid in range(THREADS) if above[tid] < need <= above[tid] + mine[tid]]
        assert len(hits) == 1, hits
        tid = hits[0]; acc = above[tid]; top = nb - tid * per
        for k in range(1, per + 1):
            c = hist[top - k]
            if acc + c >= need:
                D = top - k; sel_above = acc; break
            acc += c
        prefix |= D << sh; pmask |= dmask << sh; need -= sel_above
    T = prefix
    run_gt = run_eq = 0
    for base in range(0, n, THREADS * PER):
        fl = []
        for tid in range(THREADS):
            t0 = base + tid * PER
            gt = [(t0 + k < n) and keys[t0 + k] > T for k in range(PER)]
            eq = [(t0 + k < n) and keys[t0 + k] == T for k in range(PER)]
            fl.append((t0, gt, eq))
        cg = np.array([sum(f[1]) for f in fl]); ce = np.array([sum(f[2]) for f in fl])
        exg = np.concatenate([[0], np.cumsum(cg)[:-1]]); exe = np.concatenate([[0], np.cumsum(ce)[:-1]])
        for tid, (t0, gt, eq) in enumerate(fl):
            g = run_gt + exg[tid]; e = run_eq + exe[tid]
            for k in range(PER):
                if gt[k]:
                    pos = g + min(e, need); assert pos < K; out[pos] = t0 + k; g += 1
                elif eq[k]:
                    if e < need:
                        pos = g + e; assert pos < K; out[pos] = t0 + k
                    e += 1
        run_gt += cg.sum(); run_eq += ce.sum()
    assert (out >= 0).all()
    return out


@pytest.mark.parametrize("n", [1, 2, 5, 100, 2047, 2048, 2049, 5000, 9000])
@pytest.mark.parametrize("kind", ["rand", "ties", "neg", "zero"])
def test_model_matches_oracle_selection(n, kind):
    rng = np.random.default_rng(n)
    if kind == "rand":
        s = rng.standard_normal(n).astype(np.float32)
    elif kind == "ties":
        s = rng.integers(-3, 4, n).astype(np.float32)
    elif kind == "neg":
        s = -np.abs(rng.standard_normal(n)).astype(np.float32)
        s[::7] = -0.0
    else:
        s = np.zeros(n, np.float32)
        s[::3] = -0.0
    for budget in sorted({1, 2, n // 3 + 1, n - 1, n, n + 5}):
        if budget >= 1:
            assert np.array_equal(model_select(s, budget), O.select_tokens(s, budget)), budget
