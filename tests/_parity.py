"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, and compare with the stated
tolerances."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O

# Selected-set tolerance: a token may differ only if its oracle weight is within
# THETA_REL of the oracle threshold, or it is the single token at the cut when
# the oracle's cumulative mass there is within CUT_ABS of p.
THETA_REL = 1e-6
CUT_ABS = 1e-5
# attention output tolerance (max abs error against the oracle's fp64 result)
OUT_ABS = 2e-3
LSE_ABS = 1e-4


def np16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def gpu_rows(arr: np.ndarray, page_table, b, h, L):
    return O.sequence_rows(arr, page_table, b, h, L)


def gpu_meta(meta: np.ndarray, page_table, b, h, L):
    P = (L + 15) // 16
    if page_table is None:
        return meta[b, h, :P]
    return np.stack([meta[page_table[b, pg], h] for pg in range(P)]) if P else meta[0, h, :0]


def compare_selection(gpu_tokens, res: dict, head: int, p: float):
    """Compare a GPU selection (token ids) with the oracle's for one set.

    Returns (n_near_theta, n_cut); raises AssertionError on any other mismatch."""
    g = np.asarray(gpu_tokens, np.int64)
    assert np.all(np.diff(g) > 0), "GPU indices must be strictly ascending"
    toks = res["cand_tokens"]
    o = res["sel_tokens"][head]
    w = res["weights"][head]
    theta = res["theta"][head]
    pos_of = {int(t): i for i, t in enumerate(toks)}
    assert all(int(t) in pos_of for t in g), "GPU selected a non-candidate token"
    diff = set(g.tolist()) ^ set(o.tolist())
    near = {t for t in diff if abs(w[pos_of[t]] - theta) <= THETA_REL * theta}
    rest = diff - near
    n_cut = 0
    if rest:
        order = res["sorted_order"][head]
        cs = res["cumsum"][head]
        k = res["kstar"][head]
        assert len(rest) == 1, f"{len(rest)} tokens differ beyond tolerance (k*={k})"
        t = next(iter(rest))
        i = pos_of[t]
        dropped_cut = t in set(o.tolist()) and i == order[k - 1] and k >= 2 and \
            abs(cs[k - 2] - p) <= CUT_ABS
        added_next = t not in set(o.tolist()) and k < len(order) and i == order[k] and \
            abs(cs[k - 1] - p) <= CUT_ABS
        assert dropped_cut or added_next, \
            f"token {t} (w={w[i]:.3e}, theta={theta:.3e}) differs beyond tolerance"
        n_cut = 1
    return len(near), n_cut


def check_attention(out_gpu: np.ndarray, lse_gpu, x: O.SeqInputs, b: int, hq: int,
                    tokens, hk: int):
    L = int(x.seq_lens[b])
    k_seq = O.sequence_rows(x.k, x.page_table, b, hk, L)
    v_seq = O.sequence_rows(x.v, x.page_table, b, hk, L)
    t = np.asarray(tokens, np.int64)
    ref, lse = O.sparse_attention(x.q[b, hq], k_seq[t], v_seq[t])
    err = np.abs(out_gpu.astype(np.float64) - ref).max()
    assert err <= OUT_ABS, f"attention max abs error {err:.3e}"
    if lse_gpu is not None:
        if math.isinf(lse):
            assert math.isinf(lse_gpu) and lse_gpu < 0
        else:
            assert abs(lse_gpu - lse) <= LSE_ABS * max(1.0, abs(lse)), (lse_gpu, lse)
    return err
