"""CPU model of the GPU's top-p threshold search (host logic, no GPU).

The kernel finds theta on the fp32 bit pattern of the weights with exact
integer masses (each weight truncated to a multiple of 2^-40): a first 12-bit
digit, then either two more digits (9 + 9 bits) or, when the first digit's
bin holds at most 32 weights, a direct resolution of that bin (sort by weight
descending and position ascending, cut where the running mass reaches the
target).  Both must give the same theta and tie count as a brute-force sort of
the integer masses; the kept set is every weight above theta plus the r_need
lowest-position weights equal to it."""
import math

import numpy as np
import pytest

SCALE = float(2 ** 40)
EPS = 1e-12
BIN_LIST = 32


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
    idx = np.nonzero((keys & pmask) == prefix)[0]
    if len(idx) > BIN_LIST:
        return None
    order = sorted(idx, key=lambda i: (-int(keys[i]), i))
    cum = A
    for j, i in enumerate(order):
        cum += int(F[i])
        if cum >= T and cum - int(F[i]) < T:
            ties = sum(1 for i2 in order[:j + 1] if keys[i2] == keys[i])
            return int(keys[i]), ties
    raise AssertionError("no cut")


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
