"""Seeded synthetic inputs for the Twilight decode path.

This module only draws random tensors and lays them out; it holds none of the
method's arithmetic (no quantisation, scoring, softmax or selection).  Both the
CPU oracle side (tests, the timed CPU baseline) and the CUDA side (tests,
bench, smoke) take their inputs from here, so the two implementations see the
same bytes.

Workloads follow the synthetic shapes used to stand in for the LongBench /
RULER / PG-19 runs of "Twilight: Adaptive Attention Sparsity with Hierarchical
Top-p Pruning" (atlas.scime.ai summary, "Experimental setup"): the layer shapes
of Llama-2-7B (MHA, 32 heads) and Llama-3.1-8B (GQA, 32 query / 8 KV heads),
head_dim 128, fp16 K/V drawn from N(0, 1), with planted heavy keys so that the
attention distribution is skewed the way long-context attention is.

Layouts (all fp16, head_dim = 128, page = 16 tokens):
  contiguous: K, V [B][Hk][N][128]
  paged:      K, V pool [num_pages][Hk][16][128]; page_table [B][max_pages]
              int32 maps (sequence, logical page) -> pool page.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

HEAD_DIM = 128
PAGE = 16


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hk: int
    N: int                      # max tokens per sequence (allocation)
    q: torch.Tensor             # [B][Hq][128] fp16
    k: torch.Tensor             # contiguous [B][Hk][N][128] or pool [P][Hk][16][128]
    v: torch.Tensor
    seq_lens: torch.Tensor      # [B] int32
    page_table: Optional[torch.Tensor] = None   # [B][max_pages] int32 (paged only)
    budget_tokens: Optional[int] = None         # None: candidates = every token
    p: float = 0.85
    group_mode: int = 0         # 1: one top-p set per KV group
    heavy: Optional[dict] = None  # {(b, hk): [token positions]} planted heavy keys

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    @property
    def max_pages(self) -> int:
        return (self.N + PAGE - 1) // PAGE

    def to(self, device) -> "Workload":
        w = dataclasses.replace(self)
        for f in ("q", "k", "v", "seq_lens", "page_table"):
            t = getattr(self, f)
            if t is not None:
                setattr(w, f, t.to(device))
        return w


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn_half(shape, g, device, chunk_elems: int = 1 << 28) -> torch.Tensor:
    """N(0,1) drawn in fp32 and rounded to fp16, in chunks to bound the fp32 peak."""
    out = torch.empty(shape, dtype=torch.float16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=g, device=device, dtype=torch.float32).half()
    return out


def _distinct_positions(n_pick: int, length: int, g, device) -> list:
    perm = torch.randperm(length, generator=g, device=device)[:n_pick]
    return sorted(int(x) for x in perm.cpu())


def _outlier_channels(t: torch.Tensor, channels, factor: float) -> None:
    """Scale the given head_dim channels of every row by `factor` (in place)."""
    for c in channels:
        t[..., c] = (t[..., c].float() * factor).half()


def tiny(seed: int = 1235, device="cpu", N: int = 4096, n_heavy: int = 8,
         p: float = 0.85) -> Workload:
    """Single head, context N, candidates = all tokens, `n_heavy` keys set to 4*q/|q|."""
    g = _gen(seed, device)
    q = _randn_half((1, 1, HEAD_DIM), g, device)
    k = _randn_half((1, 1, N, HEAD_DIM), g, device)
    v = _randn_half((1, 1, N, HEAD_DIM), g, device)
    qf = q[0, 0].float()
    heavy_vec = (4.0 * qf / qf.norm()).half()
    pos = _distinct_positions(n_heavy, N, g, device)
    for t in pos:
        k[0, 0, t] = heavy_vec
    lens = torch.full((1,), N, dtype=torch.int32, device=device)
    return Workload("tiny_1h_4k", 1, 1, 1, N, q, k, v, lens, None, None, p, 0,
                    {(0, 0): pos})


def llama2_mha(seed: int = 1236, device="cpu", N: int = 32768, H: int = 32,
               budget_tokens: int = 8192, p: float = 0.85) -> Workload:
    """Llama-2-7B decode layer: 32 heads MHA, context N, 4 outlier channels x8 in K and V."""
    g = _gen(seed, device)
    q = _randn_half((1, H, HEAD_DIM), g, device)
    k = _randn_half((1, H, N, HEAD_DIM), g, device)
    v = _randn_half((1, H, N, HEAD_DIM), g, device)
    ch = sorted(int(c) for c in torch.randperm(HEAD_DIM, generator=g, device=device)[:4].cpu())
    _outlier_channels(k, ch, 8.0)
    _outlier_channels(v, ch, 8.0)
    lens = torch.full((1,), N, dtype=torch.int32, device=device)
    return Workload(f"llama2_7b_mha_b1_h{H}_n{N}", 1, H, H, N, q, k, v, lens, None,
                    budget_tokens, p, 0, {"outlier_channels": ch})


HEAVY_PER_KV_HEAD = (0, 1, 2, 4, 8, 16, 32, 64)


def llama3_gqa(seed: int = 1237, device="cpu", N: int = 131072, Hq: int = 32, Hk: int = 8,
               budget_tokens: int = 8192, p: float = 0.85, group_mode: int = 1) -> Workload:
    """Llama-3.1-8B GQA layer: 32 query / 8 KV heads; KV head j gets
    HEAVY_PER_KV_HEAD[j % 8] keys set to 8*qbar/|qbar| (qbar = the group's mean query)."""
    g = _gen(seed, device)
    G = Hq // Hk
    q = _randn_half((1, Hq, HEAD_DIM), g, device)
    k = _randn_half((1, Hk, N, HEAD_DIM), g, device)
    v = _randn_half((1, Hk, N, HEAD_DIM), g, device)
    heavy = {}
    for j in range(Hk):
        n_h = HEAVY_PER_KV_HEAD[j % len(HEAVY_PER_KV_HEAD)]
        qbar = q[0, j * G:(j + 1) * G].float().mean(0)
        vec = (8.0 * qbar / qbar.norm()).half()
        pos = _distinct_positions(n_h, N, g, device) if n_h else []
        for t in pos:
            k[0, j, t] = vec
        heavy[(0, j)] = pos
    lens = torch.full((1,), N, dtype=torch.int32, device=device)
    return Workload(f"llama3_8b_gqa_b1_hq{Hq}_hk{Hk}_n{N}", 1, Hq, Hk, N, q, k, v, lens, None,
                    budget_tokens, p, group_mode, heavy)


def batched_paged(seed: int = 1238, device="cpu", B: int = 16, H: int = 32,
                  len_lo: int = 8192, len_hi: int = 32768, budget_tokens: int = 4096,
                  p: float = 0.9, Hk: Optional[int] = None) -> Workload:
    """B sequences with lengths ~ U[len_lo, len_hi], KV in 16-token pages placed by a
    seeded permutation in one pool; page_table entries past a sequence's end are 0."""
    g = _gen(seed, device)
    Hk = H if Hk is None else Hk
    lens = torch.randint(len_lo, len_hi + 1, (B,), generator=g, device=device, dtype=torch.int64)
    lens_l = [int(x) for x in lens.cpu()]
    pages = [(L + PAGE - 1) // PAGE for L in lens_l]
    max_pages = max(pages)
    total = sum(pages)
    perm = torch.randperm(total, generator=g, device=device).to(torch.int32)
    table = torch.zeros((B, max_pages), dtype=torch.int32, device=device)
    off = 0
    for b in range(B):
        table[b, :pages[b]] = perm[off:off + pages[b]]
        off += pages[b]
    q = _randn_half((B, H, HEAD_DIM), g, device)
    k = _randn_half((total, Hk, PAGE, HEAD_DIM), g, device)
    v = _randn_half((total, Hk, PAGE, HEAD_DIM), g, device)
    return Workload(f"paged_b{B}_h{H}_len{len_lo}-{len_hi}", B, H, Hk, max_pages * PAGE, q, k, v,
                    lens.to(torch.int32), table, budget_tokens, p, 0, None)


SWEEP_TAU = (0.25, 0.5, 1.0, 2.0)
SWEEP_P = (0.7, 0.85, 0.95, 0.99)


def concentration_sweep(seed: int = 1239, device="cpu", B: int = 4, Hk: int = 8, G: int = 4,
                        N: int = 65536) -> Workload:
    """Base = full attention (all tokens are candidates), GQA with group-wise top-p.
    Per (b, kv head), 2**u heavy keys (u ~ U{0..8}) set to 8*qbar/|qbar|.  The
    temperature tau and p of a sweep point are applied with `sweep_point`."""
    g = _gen(seed, device)
    Hq = Hk * G
    q = _randn_half((B, Hq, HEAD_DIM), g, device)
    k = _randn_half((B, Hk, N, HEAD_DIM), g, device)
    v = _randn_half((B, Hk, N, HEAD_DIM), g, device)
    heavy = {}
    us = torch.randint(0, 9, (B, Hk), generator=g, device=device).cpu()
    for b in range(B):
        for j in range(Hk):
            n_h = 2 ** int(us[b, j])
            qbar = q[b, j * G:(j + 1) * G].float().mean(0)
            vec = (8.0 * qbar / qbar.norm()).half()
            pos = _distinct_positions(n_h, N, g, device)
            for t in pos:
                k[b, j, t] = vec
            heavy[(b, j)] = pos
    lens = torch.full((B,), N, dtype=torch.int32, device=device)
    return Workload(f"sweep_b{B}_hk{Hk}_g{G}_n{N}", B, Hq, Hk, N, q, k, v, lens, None, None,
                    0.85, 1, heavy)


def sweep_point(w: Workload, tau: float, p: float) -> Workload:
    """The sweep's query temperature: q scaled by 1/tau (rounded to fp16), and its p."""
    out = dataclasses.replace(w)
    out.q = (w.q.float() / tau).half()
    out.p = p
    out.name = f"{w.name}_tau{tau}_p{p}"
    return out


def random_small(seed: int, device="cpu", B: int = 2, Hq: int = 4, Hk: int = 2, N: int = 777,
                 paged: bool = False, ragged: bool = True, budget_tokens: Optional[int] = 160,
                 p: float = 0.85, group_mode: int = 0, n_heavy: int = 3,
                 min_len: int = 1) -> Workload:
    """Small seeded case with ragged lengths (not multiples of 16 or 32) for parity tests."""
    g = _gen(seed, device)
    if ragged:
        lens = torch.randint(min_len, N + 1, (B,), generator=g, device=device, dtype=torch.int64)
        lens[0] = N
    else:
        lens = torch.full((B,), N, dtype=torch.int64, device=device)
    lens_l = [int(x) for x in lens.cpu()]
    q = _randn_half((B, Hq, HEAD_DIM), g, device)
    G = Hq // Hk
    if paged:
        pages = [(L + PAGE - 1) // PAGE for L in lens_l]
        max_pages = (N + PAGE - 1) // PAGE
        total = sum(pages)
        perm = torch.randperm(max(total, 1), generator=g, device=device).to(torch.int32)
        table = torch.zeros((B, max_pages), dtype=torch.int32, device=device)
        off = 0
        for b in range(B):
            table[b, :pages[b]] = perm[off:off + pages[b]]
            off += pages[b]
        k = _randn_half((max(total, 1), Hk, PAGE, HEAD_DIM), g, device)
        v = _randn_half((max(total, 1), Hk, PAGE, HEAD_DIM), g, device)
        Nalloc = max_pages * PAGE
    else:
        table = None
        k = _randn_half((B, Hk, N, HEAD_DIM), g, device)
        v = _randn_half((B, Hk, N, HEAD_DIM), g, device)
        Nalloc = N
    heavy = {}
    for b in range(B):
        for j in range(Hk):
            L = lens_l[b]
            nh = min(n_heavy, L)
            pos = _distinct_positions(nh, L, g, device) if nh > 0 else []
            qbar = q[b, j * G:(j + 1) * G].float().mean(0)
            vec = (4.0 * qbar / qbar.norm()).half()
            for t in pos:
                if paged:
                    k[table[b, t // PAGE], j, t % PAGE] = vec
                else:
                    k[b, j, t] = vec
            heavy[(b, j)] = pos
    w = Workload(f"small_s{seed}", B, Hq, Hk, Nalloc, q, k, v, lens.to(torch.int32), table,
                 budget_tokens, p, group_mode, heavy)
    return w


def label_channels(w: Workload, r: int = 16, seed: int = 7) -> list:
    """Label channels [Hk][r] for a token-level base selector: a seeded stand-in
    for offline calibration on trained weights.  The workload's planted outlier
    channels (if any) come first, then distinct seeded random channels."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    planted = []
    if isinstance(w.heavy, dict):
        planted = [int(c) for c in w.heavy.get("outlier_channels", [])][:r]
    out = []
    for _ in range(w.Hk):
        rest = [int(c) for c in torch.randperm(HEAD_DIM, generator=g) if int(c) not in planted]
        out.append(planted + rest[:r - len(planted)])
    return out


CONFIGS = {
    "tiny": tiny,
    "llama2_mha": llama2_mha,
    "llama3_gqa": llama3_gqa,
    "batched_paged": batched_paged,
    "sweep": concentration_sweep,
}
