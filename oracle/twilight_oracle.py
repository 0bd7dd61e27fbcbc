"""Plain, slow CPU oracle of Twilight's decode-time hierarchical top-p path.

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference arm may import this module.  It shares no code,
tables or helpers with the CUDA library and never imports it.

Source: "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning"
(Lin, Tang, Yang, Wang, Tang, Tian, Stoica, Han, Gao; arXiv 2502.02770).
The pages that describe it fix the following, and each function below cites
which part it follows:
  * select-then-prune: a base sparse-attention algorithm pre-selects tokens,
    then top-p (nucleus) thresholding runs over the attention weights of those
    candidates, so the budget adapts per head / per query
    (atlas.scime.ai summary, "Approach"; abstract);
  * the weights are estimated from a 4-bit quantised key cache, and the
    threshold is found by binary-search top-p kernels ("Approach"); 4-bit is
    preferred to 2-bit for stable cumulative weights (table of measured
    effects, quantisation ablation row);
  * under GQA the dynamic budget is group-wise, not head-wise ("Limitations");
  * Quest is a base selector whose top-k works on a per-page max-pooled
    layout ("Surprising findings"), hence page-level pre-selection;
  * the INT4 key cache costs about 1/8 of the KV cache ("Limitations");
  * p is about 0.85 (table of measured effects, top-p ablation row).

Readings taken where the pages are silent (all also listed in the design
notes of this repository):
  R1 quantisation: per token, per group of 32 channels, asymmetric with a
     float zero point equal to the group minimum and an fp16 scale
     (max - min) / 15; codes 0..15 packed two per byte, even channel in the
     low nibble; all arithmetic in IEEE fp32 round-to-nearest in the order
     written below; scale == 0 gives code 0.
  R2 min / max of fp16 values use the IEEE totalOrder (-0 < +0), so the
     stored bit pattern is unique.
  R3 Quest page bound: score = sum_j max(q_j * min_j, q_j * max_j) (Quest's
     published criterion; the pages give no formula), no 1/sqrt(d) (it does
     not change the ranking), no forced pages.  Under GQA the KV head's score
     is the sum of its query heads' scores.  Summed in fp32 in one fixed
     order (below) so that the page ranking is a deterministic integer result.
  R4 keep K_p = min(floor(budget / 16), pages) pages with the largest score,
     ties to the lower page index, returned in ascending page order.
  R5 weights are the softmax over the candidate set only; under GQA in group
     mode a token's weight is the mean over the group's heads of the
     per-head normalised weights.
  R6 top-p: sort descending (ties to ascending token index), keep the
     shortest prefix whose cumulative weight is >= p - MASS_EPS; p >= 1 keeps
     all.  MASS_EPS = 1e-12 makes ties that are exact in real arithmetic (for
     instance n uniform weights with p * n an integer) resolve the way exact
     arithmetic does instead of by the last bit of a rounded sum.
  R7 sparse attention over the selected fp16 K/V rows, softmax scale
     1/sqrt(128); out = 0 and lse = -inf for an empty selection.
  R8 the 2-bit key cache of the quantisation ablation (4-bit preferred to
     2-bit for stable cumulative weights, table of measured effects) is R1
     with 3 in place of 15: scale = fp16_rn((max - min) / 3), codes 0..3,
     four per byte, channel 4i + j in bits 2j, 2j + 1 of byte i.
  R9 the Double-Sparsity-style base selector (DS is named as a base selector
     Twilight builds on: "Builds on", "Key results"; the pages give no
     mechanism) is read as DS's published idea, synthetic: per KV head a set
     of r "label" channels (given as input; real DS finds them by offline
     calibration on trained weights), a label cache holding those channels of
     every key, a token-level score
         s_h[t] = sum_j q_h[c_j] * k_t[c_j]   (fp32, products exact, summed
                  j = 0 .. r-1 left to right; group heads added in order)
     and the min(budget, len) tokens with the largest score (ties to the lower
     token index) as the candidate set, ascending.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

HEAD_DIM = 128
PAGE = 16
GROUP = 32
NGROUPS = HEAD_DIM // GROUP
MASS_EPS = 1e-12

__all__ = [
    "HEAD_DIM", "PAGE", "GROUP", "MASS_EPS", "fp16_min", "fp16_max", "quantize_keys", "unpack_codes",
    "dequantize_keys", "page_meta", "quest_page_scores", "select_pages", "candidate_tokens",
    "estimate_logits", "softmax_weights", "group_weights", "topp_select", "sparse_attention",
    "SeqInputs", "sequence_rows", "oracle_unit", "oracle_decode", "int4_cache_bytes_per_token",
    "key_cache_bytes_per_token", "kv_cache_bytes_per_token", "KEY_BITS", "retained_mass",
    "label_cache", "label_scores", "select_tokens",
]

KEY_BITS = (4, 2)   # key-cache widths: 4-bit (R1) and the ablation's 2-bit (R8)


# ----------------------------------------------------------------------------- R2
def _fp16_order_key(x: np.ndarray) -> np.ndarray:
    """Integer key that orders fp16 values by IEEE totalOrder (-0 sorts below +0)."""
    bits = np.ascontiguousarray(x, dtype=np.float16).view(np.uint16).astype(np.int32)
    neg = (bits & 0x8000) != 0
    return np.where(neg, -(bits & 0x7FFF) - 1, bits)


def fp16_min(x: np.ndarray, axis: int) -> np.ndarray:
    """Exact fp16 minimum along `axis` under totalOrder (reading R2)."""
    key = _fp16_order_key(x)
    i = np.expand_dims(np.argmin(key, axis=axis), axis)
    return np.take_along_axis(np.asarray(x, np.float16), i, axis=axis).squeeze(axis)


def fp16_max(x: np.ndarray, axis: int) -> np.ndarray:
    """Exact fp16 maximum along `axis` under totalOrder (reading R2)."""
    key = _fp16_order_key(x)
    i = np.expand_dims(np.argmax(key, axis=axis), axis)
    return np.take_along_axis(np.asarray(x, np.float16), i, axis=axis).squeeze(axis)


# ----------------------------------------------------------------------------- R1, R8
def _levels(bits: int) -> int:
    if bits not in KEY_BITS:
        raise ValueError(f"key cache width must be one of {KEY_BITS}, got {bits}")
    return (1 << bits) - 1


def quantize_keys(k: np.ndarray, bits: int = 4):
    """Per-token asymmetric key quantisation, group 32 (reading R1; R8 for 2 bits).

    The 4-bit key cache used to estimate attention weights: atlas.scime.ai
    summary, "Approach"; the 2-bit width is the one its quantisation ablation
    row compares against (table of measured effects).

    k: fp16 [..., 128].  Returns codes uint8 [..., 128 * bits / 8], scales fp16
    [..., 4] and zeros fp16 [..., 4].  With n = 2^bits - 1 (15 or 3), per group
    of 32 channels, in IEEE fp32 round-to-nearest:
        mn, mx = exact fp16 min / max of the group
        scale  = fp16_rn( (f32(mx) - f32(mn)) / n )
        code   = clamp( rint_even( (f32(x) - f32(mn)) / f32(scale) ), 0, n )
                 (0 when scale == 0)
        zero   = mn
    Packing: 8 / bits codes per byte, channel (8 / bits) * i + j in bits
    bits * j .. bits * j + bits - 1 of byte i (4-bit: even channel in the low
    nibble).
    """
    n = _levels(bits)
    k = np.asarray(k, dtype=np.float16)
    lead = k.shape[:-1]
    x = k.reshape(lead + (NGROUPS, GROUP))
    mn = fp16_min(x, axis=-1)                                    # [..., 4] fp16
    mx = fp16_max(x, axis=-1)
    d = mx.astype(np.float32) - mn.astype(np.float32)            # fp32 RN
    scale = (d / np.float32(n)).astype(np.float16)               # fp32 RN, then fp16 RN
    num = x.astype(np.float32) - mn.astype(np.float32)[..., None]
    sc = scale.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = num / sc                                         # fp32 RN
    code = np.where(sc == 0, np.float32(0), np.clip(np.rint(ratio), 0, n)).astype(np.uint8)
    code = code.reshape(lead + (HEAD_DIM,))
    per = 8 // bits
    packed = np.zeros(lead + (HEAD_DIM // per,), dtype=np.uint8)
    for j in range(per):
        packed |= (code[..., j::per] << (bits * j)).astype(np.uint8)
    return packed, scale, mn.copy()


def unpack_codes(codes: np.ndarray, bits: int = 4) -> np.ndarray:
    """uint8 [..., 128 * bits / 8] -> int codes [..., 128] (the packing of quantize_keys)."""
    n = _levels(bits)
    per = 8 // bits
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape[:-1] + (HEAD_DIM,), dtype=np.int64)
    for j in range(per):
        out[..., j::per] = (codes >> (bits * j)) & n
    return out


def dequantize_keys(codes, scales, zeros, bits: int = 4) -> np.ndarray:
    """k_hat = zero_g + scale_g * code, in fp64 from the stored fp16 scale and zero."""
    c = unpack_codes(codes, bits).astype(np.float64)
    lead = c.shape[:-1]
    c = c.reshape(lead + (NGROUPS, GROUP))
    s = np.asarray(scales, np.float16).astype(np.float64)[..., None]
    z = np.asarray(zeros, np.float16).astype(np.float64)[..., None]
    return (z + s * c).reshape(lead + (HEAD_DIM,))


def key_cache_bytes_per_token(bits: int = 4, with_scale_zero: bool = True) -> int:
    """Bytes of the quantised key cache per token per KV head: 128 * bits / 8 B
    of codes, plus an fp16 scale and an fp16 zero for each of the 4 groups."""
    _levels(bits)
    return HEAD_DIM * bits // 8 + (2 * 2 * NGROUPS if with_scale_zero else 0)


def int4_cache_bytes_per_token(with_scale_zero: bool = True) -> int:
    """Bytes of the 4-bit key cache per token per KV head: 64 B of codes, plus an
    fp16 scale and an fp16 zero for each of the 4 groups."""
    return key_cache_bytes_per_token(4, with_scale_zero)


def kv_cache_bytes_per_token() -> int:
    """fp16 K and V bytes per token per KV head."""
    return 2 * 2 * HEAD_DIM


# ----------------------------------------------------------------------------- meta
def page_meta(k_seq: np.ndarray, length: int) -> np.ndarray:
    """Quest page metadata: per page of 16 tokens, the channel-wise exact fp16 min
    and max of the keys over the page's valid tokens (a partial last page uses
    only tokens < length).  Returns [P][2][128] fp16, row 0 = min, row 1 = max.

    Quest's page-level pre-selection is the base selector the pages build on
    (atlas.scime.ai summary, "Surprising findings": per-page max pooling).
    """
    P = (length + PAGE - 1) // PAGE
    out = np.empty((P, 2, HEAD_DIM), dtype=np.float16)
    for pg in range(P):
        rows = np.asarray(k_seq[pg * PAGE:min(length, (pg + 1) * PAGE)], np.float16)
        out[pg, 0] = fp16_min(rows, axis=0)
        out[pg, 1] = fp16_max(rows, axis=0)
    return out


# ----------------------------------------------------------------------------- R3
def quest_page_scores(q_group: np.ndarray, meta: np.ndarray) -> np.ndarray:
    """Quest upper bound of q.k over each page (reading R3), fp32.

    q_group: fp16 [G][128] (the query heads that share this KV head; G = 1 for
    MHA).  meta: fp16 [P][2][128].  For each head,
        t_j = max(q_j * min_j, q_j * max_j)            (exact in fp32)
    is summed in this fixed fp32 order: channels are split into 16 chunks of 8
    consecutive channels, each chunk summed left to right, then the 16 chunk
    sums c_0..c_15 are combined as a_i = c_i + c_{i+8} (i < 8),
    b_i = a_i + a_{i+4} (i < 4), d_i = b_i + b_{i+2} (i < 2), score = d_0 + d_1.
    Heads of a group are added in head order: ((s_0 + s_1) + s_2) + s_3.
    """
    q = np.asarray(q_group, np.float16).astype(np.float32)
    mn = np.asarray(meta[:, 0, :], np.float16).astype(np.float32)
    mx = np.asarray(meta[:, 1, :], np.float16).astype(np.float32)
    P = meta.shape[0]
    total = None
    for g in range(q.shape[0]):
        t = np.maximum(q[g] * mn, q[g] * mx)                     # [P][128] fp32, exact
        ch = t.reshape(P, 16, 8)
        c = ch[:, :, 0].copy()
        for j in range(1, 8):
            c = c + ch[:, :, j]
        a = c[:, :8] + c[:, 8:]
        b = a[:, :4] + a[:, 4:]
        d = b[:, :2] + b[:, 2:]
        s = d[:, 0] + d[:, 1]
        total = s if total is None else total + s
    if total is None:
        total = np.zeros(P, np.float32)
    return total.astype(np.float32)


def select_pages(scores: np.ndarray, budget_tokens: int) -> np.ndarray:
    """Top-K_p pages by score, K_p = min(floor(budget/16), P); ties to the lower
    page index; returned ascending (reading R4)."""
    P = len(scores)
    kp = min(budget_tokens // PAGE, P)
    order = np.lexsort((np.arange(P), -np.asarray(scores, np.float64)))
    return np.sort(order[:kp]).astype(np.int64)


# ----------------------------------------------------------------------------- R9
def label_cache(k_seq: np.ndarray, channels) -> np.ndarray:
    """The label cache of a token-level base selector (reading R9): the fp16
    values of the given channels of every key, [T][r], exact copies."""
    ch = np.asarray(channels, np.int64)
    return np.asarray(k_seq, np.float16)[:, ch].copy()


def label_scores(q_group: np.ndarray, labels: np.ndarray, channels) -> np.ndarray:
    """Token scores from the label channels (reading R9), fp32.  For each query
    head h of the group, s_h[t] = sum over j = 0 .. r-1, left to right, of
    q_h[c_j] * label[t][j] (each product exact in fp32, each add rounded);
    heads are added in order: ((s_0 + s_1) + s_2) + ...  Returns [T]."""
    q = np.asarray(q_group, np.float16).astype(np.float32)[:, np.asarray(channels, np.int64)]
    lab = np.asarray(labels, np.float16).astype(np.float32)
    total = None
    for h in range(q.shape[0]):
        s = np.zeros(lab.shape[0], np.float32)
        for j in range(lab.shape[1]):
            s = s + q[h, j] * lab[:, j]
        total = s if total is None else total + s
    if total is None:
        total = np.zeros(lab.shape[0], np.float32)
    return total.astype(np.float32)


def select_tokens(scores: np.ndarray, budget_tokens: int) -> np.ndarray:
    """Token-level top-k (reading R9): the min(budget, T) tokens with the
    largest score, ties to the lower token index, returned ascending."""
    T = len(scores)
    k = min(int(budget_tokens), T)
    order = np.lexsort((np.arange(T), -np.asarray(scores, np.float64)))
    return np.sort(order[:k]).astype(np.int64)


def candidate_tokens(pages: Optional[np.ndarray], length: int) -> np.ndarray:
    """Token indices (ascending) of the candidate pages, valid tokens only; None
    means every token of the sequence is a candidate (base = full attention)."""
    if pages is None:
        return np.arange(length, dtype=np.int64)
    toks = [np.arange(pg * PAGE, min(length, (pg + 1) * PAGE)) for pg in pages]
    if not toks:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate(toks).astype(np.int64)


# ----------------------------------------------------------------------------- R5, R6
def estimate_logits(q_group: np.ndarray, codes, scales, zeros, bits: int = 4) -> np.ndarray:
    """Estimated attention logits from the quantised key cache, fp64:
        l[i, h] = (q_h . k_hat_i) / sqrt(128),  k_hat = zero + scale * code.
    (atlas.scime.ai summary, "Approach": weights estimated from INT4 keys;
    `bits` = 2 for the ablation's 2-bit cache.)  Returns [C][G]."""
    khat = dequantize_keys(codes, scales, zeros, bits)           # [C][128] fp64
    q = np.asarray(q_group, np.float16).astype(np.float64)       # [G][128]
    return (khat @ q.T) / math.sqrt(HEAD_DIM)


def softmax_weights(logits: np.ndarray) -> np.ndarray:
    """Normalised attention weights over the candidate set, fp64 (reading R5)."""
    l = np.asarray(logits, np.float64)
    if l.size == 0:
        return l.copy()
    e = np.exp(l - l.max())
    return e / e.sum()


def group_weights(logits: np.ndarray) -> np.ndarray:
    """Group-wise weights under GQA: the mean over the group's heads of each
    head's normalised weights (atlas.scime.ai summary, "Limitations": budgets
    become group-wise under GQA; reading R5).  logits: [C][G]."""
    l = np.asarray(logits, np.float64)
    return np.mean(np.stack([softmax_weights(l[:, h]) for h in range(l.shape[1])], 1), axis=1)


def topp_select(w: np.ndarray, p: float):
    """Top-p (nucleus) selection over candidate weights (reading R6).

    Sort descending with ties to the ascending candidate position, keep the
    shortest prefix with cumulative weight >= p - MASS_EPS (fp64 cumulative
    sum).  Without
    ties this is {i : w_i >= theta} for the largest theta whose retained mass is
    >= p.  p >= 1 keeps every candidate.

    Returns (selected positions ascending, theta, k_star, sorted order, cumsum).
    """
    w = np.asarray(w, np.float64)
    n = len(w)
    order = np.lexsort((np.arange(n), -w))
    cs = np.cumsum(w[order])
    if n == 0:
        return np.zeros(0, np.int64), 0.0, 0, order, cs
    if p >= 1.0:
        k = n
    else:
        k = int(np.searchsorted(cs, p - MASS_EPS, side="left")) + 1
        k = min(k, n)
    sel = np.sort(order[:k]).astype(np.int64)
    theta = float(w[order[k - 1]])
    return sel, theta, k, order, cs


# ----------------------------------------------------------------------------- R7
def sparse_attention(q: np.ndarray, k_rows: np.ndarray, v_rows: np.ndarray):
    """Exact softmax attention of one query over the given fp16 K/V rows, fp64:
    s_i = q.k_i / sqrt(128), out = sum softmax(s)_i v_i, lse = log sum exp s."""
    k_rows = np.asarray(k_rows, np.float16).astype(np.float64)
    v_rows = np.asarray(v_rows, np.float16).astype(np.float64)
    if k_rows.shape[0] == 0:
        return np.zeros(HEAD_DIM, np.float64), -math.inf
    qf = np.asarray(q, np.float16).astype(np.float64)
    s = (k_rows @ qf) / math.sqrt(HEAD_DIM)
    m = s.max()
    e = np.exp(s - m)
    L = e.sum()
    return (e @ v_rows) / L, float(m + math.log(L))


def retained_mass(q: np.ndarray, k_rows: np.ndarray, selected: np.ndarray) -> float:
    """Exact attention mass that a selection keeps: the sum over the selected
    rows of the fp64 softmax of q . k / sqrt(128) over all the given rows (the
    candidate set).  The cumulative attention weight whose stability the
    quantisation ablation measures (atlas.scime.ai summary, table of measured
    effects).  An empty candidate set keeps mass 0."""
    k_rows = np.asarray(k_rows, np.float16).astype(np.float64)
    if k_rows.shape[0] == 0:
        return 0.0
    s = (k_rows @ np.asarray(q, np.float16).astype(np.float64)) / math.sqrt(HEAD_DIM)
    e = np.exp(s - s.max())
    return float(e[np.asarray(selected, np.int64)].sum() / e.sum())


# ----------------------------------------------------------------------------- layout
class SeqInputs:
    """numpy views of one decode-layer input, in either layout.

    contiguous: k, v [B][Hk][N][128];  paged: k, v [pages][Hk][16][128] with
    page_table [B][max_pages]."""

    def __init__(self, q, k, v, seq_lens, page_table=None, Hk=None):
        self.q = np.asarray(q, np.float16)
        self.k = np.asarray(k, np.float16)
        self.v = np.asarray(v, np.float16)
        self.seq_lens = np.asarray(seq_lens, np.int64)
        self.page_table = None if page_table is None else np.asarray(page_table, np.int64)
        self.B, self.Hq = self.q.shape[0], self.q.shape[1]
        self.Hk = self.k.shape[1]

    @classmethod
    def from_workload(cls, w):
        t = lambda x: None if x is None else x.detach().cpu().numpy()
        return cls(t(w.q), t(w.k), t(w.v), t(w.seq_lens), t(w.page_table))


def sequence_rows(arr: np.ndarray, page_table, b: int, h: int, length: int) -> np.ndarray:
    """The first `length` rows [length][...] of sequence b, KV head h."""
    if page_table is None:
        return arr[b, h, :length]
    P = (length + PAGE - 1) // PAGE
    pages = [arr[page_table[b, pg], h] for pg in range(P)]
    if not pages:
        return arr[0, h, :0]
    return np.concatenate(pages, 0)[:length]


def oracle_unit(x: SeqInputs, b: int, hk: int, budget_tokens: Optional[int], p: float,
                group_mode: int, sel_override: Optional[dict] = None,
                key_bits: int = 4, label_channels=None) -> dict:
    """Every result of the decode path for one (sequence, KV head).

    Returns a dict with the quantised key cache (`key_bits` wide), page meta,
    page scores, candidate pages and tokens, fp64 logits, per-set weights /
    selections / thresholds, and the attention output of each query head of the
    group.  `sel_override` maps a query head to the selected token list to
    attend over (used to check the attention stage on another implementation's
    selection).  With `label_channels` ([Hk][r]) and a budget, the base
    selector is the token-level label-channel one (R9) instead of Quest's
    pages: "pages" is then None and "label_scores" holds the token scores."""
    L = int(x.seq_lens[b])
    G = x.Hq // x.Hk
    heads = list(range(hk * G, (hk + 1) * G))
    k_seq = sequence_rows(x.k, x.page_table, b, hk, L)
    v_seq = sequence_rows(x.v, x.page_table, b, hk, L)
    codes, scales, zeros = quantize_keys(k_seq, key_bits)
    meta = page_meta(k_seq, L)
    qg = x.q[b, heads]
    res = {"len": L, "codes": codes, "scales": scales, "zeros": zeros, "meta": meta}
    if budget_tokens is None:
        pages, scores = None, None
        toks = candidate_tokens(None, L)
    elif label_channels is not None:
        ch = np.asarray(label_channels, np.int64)[hk]
        pages, scores = None, None
        res["label_scores"] = label_scores(qg, label_cache(k_seq, ch), ch)
        toks = select_tokens(res["label_scores"], budget_tokens)
    else:
        scores = quest_page_scores(qg, meta)
        pages = select_pages(scores, budget_tokens)
        toks = candidate_tokens(pages, L)
    res.update(scores=scores, pages=pages, cand_tokens=toks)
    logits = estimate_logits(qg, codes[toks], scales[toks], zeros[toks], key_bits)   # [C][G]
    res["logits"] = logits
    sets = {}
    if group_mode and G > 1:
        w = group_weights(logits)
        sel, theta, k, order, cs = topp_select(w, p)
        for h in heads:
            sets[h] = (w, sel, theta, k, order, cs)
    else:
        for gi, h in enumerate(heads):
            w = softmax_weights(logits[:, gi])
            sets[h] = topp_select(w, p)
            sets[h] = (w,) + sets[h]
    res["weights"] = {h: s[0] for h, s in sets.items()}
    res["sel_pos"] = {h: s[1] for h, s in sets.items()}
    res["sel_tokens"] = {h: toks[s[1]] for h, s in sets.items()}
    res["theta"] = {h: s[2] for h, s in sets.items()}
    res["kstar"] = {h: s[3] for h, s in sets.items()}
    res["sorted_order"] = {h: s[4] for h, s in sets.items()}
    res["cumsum"] = {h: s[5] for h, s in sets.items()}
    outs, lses = {}, {}
    for h in heads:
        t = res["sel_tokens"][h] if sel_override is None else np.asarray(sel_override[h], np.int64)
        outs[h], lses[h] = sparse_attention(x.q[b, h], k_seq[t], v_seq[t])
    res["out"], res["lse"] = outs, lses
    return res


def oracle_decode(x: SeqInputs, budget_tokens: Optional[int], p: float, group_mode: int,
                  units=None, key_bits: int = 4) -> dict:
    """oracle_unit over the given (b, hk) units (default: all)."""
    if units is None:
        units = [(b, h) for b in range(x.B) for h in range(x.Hk)]
    return {u: oracle_unit(x, u[0], u[1], budget_tokens, p, group_mode, key_bits=key_bits)
            for u in units}
