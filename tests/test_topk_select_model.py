"""CPU model of the GPU's page top-K_p radix select (host logic, no GPU).

Every CTA of a unit's cluster holds all P page-score keys (order-preserving
u32 images of the fp32 scores) and selects the K largest, ties to the lower
page: digits of 10 bits taken below the common bit prefix of the smallest and
largest key, each round histogramming the keys that match the prefix so far
and finding the digit d where the count from the top first reaches the
number still needed; when the keys of that digit are exactly the ones still
needed, the search ends and all of them are kept.  The kept set is every key
above the final prefix plus the `need` lowest-index keys equal to it (or
every key at or above it after the early exit).  It must equal a brute-force
sort by (key descending, index ascending)."""
import numpy as np
import pytest

BITS = 10


def radix_select(keys, K):
    keys = [int(k) for k in keys]
    kmin, kmax = min(keys), max(keys)
    nb = (kmin ^ kmax).bit_length()
    pmask = 0 if nb >= 32 else (~((1 << nb) - 1)) & 0xFFFFFFFF
    prefix = kmin & pmask
    need = K
    whole = False
    while nb > 0:
        width = min(BITS, nb)
        shift = nb - width
        dm = (1 << width) - 1
        nb = shift
        hist = [0] * (1 << width)
        for k in keys:
            if (k & pmask) == prefix:
                hist[(k >> shift) & dm] += 1
        above = 0
        for d in range(len(hist) - 1, -1, -1):
            here = above + hist[d]
            if here >= need > above:
                break
            above = here
        need -= above
        prefix |= d << shift
        pmask |= dm << shift
        if hist[d] == need:   # the digit's keys are exactly the ones still needed
            whole = True
            break
    if whole:   # every key at or above the prefix (its bits below the digit are zero)
        return sorted(i for i, k in enumerate(keys) if k >= prefix)
    sel = [i for i, k in enumerate(keys) if k > prefix]
    eq = [i for i, k in enumerate(keys) if k == prefix]
    return sorted(sel + eq[:need])


def brute(keys, K):
    order = sorted(range(len(keys)), key=lambda i: (-int(keys[i]), i))
    return sorted(order[:K])


@pytest.mark.parametrize("kind", ["normal", "ties", "few", "prefix", "equal"])
@pytest.mark.parametrize("P,K", [(1, 1), (7, 3), (64, 64), (512, 128), (2048, 512), (3000, 1)])
def test_radix_select_matches_brute_force(kind, P, K):
    rng = np.random.default_rng(P * 31 + K)
    f = rng.standard_normal(P).astype(np.float32)
    if kind == "ties":
        f = np.round(f * 4) / 4
    elif kind == "few":
        f = rng.integers(0, 3, P).astype(np.float32)
    elif kind == "prefix":
        f = (1000.0 + rng.integers(0, 50, P)).astype(np.float32)   # long common bit prefix
    elif kind == "equal":
        f = np.full(P, 2.5, np.float32)
    bits = f.view(np.uint32).astype(np.int64)
    keys = np.where(bits >> 31, (~bits) & 0xFFFFFFFF, bits | 0x80000000)   # order-preserving image
    K = min(K, P)
    assert radix_select(keys, K) == brute(keys, K)
