"""CPU model of the GPU's top-p threshold search (host logic, no GPU).

The kernel finds theta on the fp32 bit pattern of the weights with exact
integer masses (each weight truncated to a multiple of 2^-40): a first 12-bit
digit, then either two more digits (9 + 9 bits) or, when the first digit's
bin holds at most 1024 weights over the cluster, the same two digits run on a
gathered list of that bin's weights alone (no cluster reduction); a list of at
most 128 is sorted by one warp instead and cut where the running mass reaches
the target.  Both must give the same theta and tie count as a brute-force sort of
the integer masses; the kept set is every weight above theta plus the r_need
lowest-position weights equal to it."""
import math

import numpy as np
import pytest

SCALE = float(2 ** 40)
EPS = 1e-12
BIN_LIST = 1024


def masses(w32):
    return np.floor(w32.astype(np.float64) * SCALE).astype(np.uint64)


def target(total, p):
    t = math.ceil((p - EPS) * float(total))
    return min(int(total), max(1, t))


def digit_search(keys, F, T, first_only=False):
    """The digit steps: returns (prefix, pmask, A) after 1 or 3 digits."""
    prefix, pmask, A = 0, 0, 0
    steps = [(18, 0xFFF), (9, 0x1FF), (0, 0x1FF)]
    for k, (shift, dm) in enumerate(steps):
        inr = (keys & pmask) == prefix
        dg = (keys >> shift) & dm
        hist = np.zeros(dm + 1, np.uint64)
        np.add.at(hist, dg[inr], F[inr])
        suffix = np.cumsum(hist[::-1])[::-1]          # mass of digits >= d
        above = np.concatenate([suffix[1:], [0]]).astype(np.uint64)
        d = int(np.nonzero((A + suffix >= T) & (A + above < T))[0][0])
        A += int(above[d])
        prefix |= d << shift
        pmask |= dm << shift
        if first_only:
            break
    return prefix, pmask, A


def small_bin(keys, F, T, prefix, pmask, A):
    """The GPU's resolution of a small first-digit bin: digits 2 and 3 over the
    bin's weights gathered into one list (their order in the list is
    arbitrary: the CTAs' lists are concatenated)."""
    idx = np.nonzero((keys & pmask) == prefix)[0]
    if len(idx) == 0 or len(idx) > BIN_LIST:
        return None
    if len(idx) <= 128:
        # one warp sorts the list descending and cuts where the running mass
        # reaches the target; the list's mass above theta joins A
        order = sorted((int(keys[i]) for i in idx), reverse=True)
        cum = A
        for k in order:
            f = int(masses(np.array([k], np.uint32).view(np.float32))[0])
            cum += f
            if cum >= T and cum - f < T:
                theta = k
                break
        A += sum(int(F[i]) for i in idx if int(keys[i]) > theta)
        Ft = max(1, int(masses(np.array([theta], np.uint32).view(np.float32))[0]))
        return theta, (T - A + Ft - 1) // Ft
    perm = np.random.default_rng(len(idx)).permutation(len(idx))
    lk, lF = keys[idx][perm], F[idx][perm]
    for shift, dm in ((9, 0x1FF), (0, 0x1FF)):
        sel = (lk & pmask) == prefix
        hist = np.zeros(dm + 1, dtype=object)
        for k, f in zip(lk[sel], lF[sel]):
            hist[(int(k) >> shift) & dm] += int(f)
        suffix = np.cumsum(hist[::-1])[::-1]
        above = np.concatenate([suffix[1:], [0]])
        d = int(np.nonzero((A + suffix >= T) & (A + above < T))[0][0])
        A += int(above[d])
        prefix |= d << shift
        pmask |= dm << shift
    Ft = max(1, int(masses(np.array([prefix], np.uint32).view(np.float32))[0]))
    return prefix, (T - A + Ft - 1) // Ft


def brute(keys, F, T):
    order = sorted(range(len(keys)), key=lambda i: (-int(keys[i]), i))
    cum = 0
    for j, i in enumerate(order):
        cum += int(F[i])
        if cum >= T:
            theta = int(keys[i])
            ties = sum(1 for i2 in order[:j + 1] if keys[i2] == theta)
            return theta, ties, sorted(order[:j + 1])
    raise AssertionError("no cut")


def kept(keys, theta, r_need):
    out, eq = [], 0
    for i, k in enumerate(keys):
        if k > theta:
            out.append(i)
        elif k == theta and eq < r_need:
            out.append(i)
            eq += 1
    return out


CASES = [("gauss", 4096, 0.85), ("gauss", 700, 0.5), ("spiky", 2048, 0.9),
         ("ties", 1000, 0.85), ("few_levels", 3000, 0.7), ("uniform", 999, 0.9)]


@pytest.mark.parametrize("kind,n,p", CASES)
def test_search_paths_agree_with_brute_force(kind, n, p):
    rng = np.random.default_rng(hash(kind) % 1000 + n)
    for trial in range(6):
        if kind == "gauss":
            l = rng.standard_normal(n) * (1.0 + trial)
        elif kind == "spiky":
            l = rng.standard_normal(n)
            l[rng.integers(0, n, 5)] += 8.0
        elif kind == "ties":
            l = np.round(rng.standard_normal(n) * 2) / 2   # many exactly equal logits
        elif kind == "few_levels":
            l = rng.integers(0, 4, n).astype(np.float64)
        else:
            l = np.zeros(n)
        w = np.exp(l - l.max())
        w32 = (w / w.sum()).astype(np.float32)
        keys = w32.view(np.uint32).astype(np.int64)
        F = masses(w32)
        T = target(int(F.sum()), p)
        theta_b, ties_b, sel_b = brute(keys, F, T)
        # three digits
        prefix, _, A = digit_search(keys, F, T)
        Ft = max(1, int(masses(np.array([prefix], np.uint32).view(np.float32))[0]))
        r_need = (T - A + Ft - 1) // Ft
        assert (prefix, r_need) == (theta_b, ties_b)
        assert kept(keys, prefix, r_need) == sel_b
        # first digit, then the small bin when it applies
        prefix1, pmask1, A1 = digit_search(keys, F, T, first_only=True)
        res = small_bin(keys, F, T, prefix1, pmask1, A1)
        if res is not None:
            assert res == (theta_b, ties_b)
            assert kept(keys, *res) == sel_b


def test_small_bin_path_is_taken_on_spread_weights():
    rng = np.random.default_rng(3)
    l = rng.standard_normal(8192) * 1.7
    w = np.exp(l - l.max())
    w32 = (w / w.sum()).astype(np.float32)
    keys = w32.view(np.uint32).astype(np.int64)
    F = masses(w32)
    T = target(int(F.sum()), 0.85)
    prefix1, pmask1, A1 = digit_search(keys, F, T, first_only=True)
    assert small_bin(keys, F, T, prefix1, pmask1, A1) is not None


def test_small_bin_path_is_taken_on_unit_variance_logits():
    """8192 candidates with logits of unit spread (the Llama-shaped workloads)
    put about 70 weights in the threshold's first-digit bin: more than a warp,
    within the 256 the CTA-wide resolution takes."""
    rng = np.random.default_rng(5)
    taken = 0
    for trial in range(8):
        l = rng.standard_normal(8192)
        w = np.exp(l - l.max())
        w32 = (w / w.sum()).astype(np.float32)
        keys = w32.view(np.uint32).astype(np.int64)
        F = masses(w32)
        T = target(int(F.sum()), 0.85)
        prefix1, pmask1, A1 = digit_search(keys, F, T, first_only=True)
        in_bin = int(((keys & pmask1) == prefix1).sum())
        res = small_bin(keys, F, T, prefix1, pmask1, A1)
        if res is not None:
            taken += 1
            theta_b, ties_b, sel_b = brute(keys, F, T)
            assert res == (theta_b, ties_b)
        assert in_bin > 32
    assert taken == 8
