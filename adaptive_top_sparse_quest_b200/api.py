"""PyTorch-facing binding of the Twilight sm_100a library.

Every function here only checks tensor dtypes / shapes, allocates outputs with
PyTorch (device memory and streams are the only things PyTorch provides) and
calls the C ABI on the current CUDA stream.  All computation happens in the
CUDA kernels of libtwilight.so.

Method: "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning"
(arXiv 2502.02770): Quest page pre-selection, top-p pruning of the candidates'
attention weights estimated from a 4-bit key cache (or the 2-bit cache of its
quantisation ablation, KVCache.key_bits = 2), exact sparse attention over the
survivors.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import torch

from . import _capi
from ._capi import TwKv, TwStep, check

HEAD_DIM = 128
PAGE = 16


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _need(t: torch.Tensor, dtype, name: str):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


KEY_BITS = (4, 2)


@dataclasses.dataclass
class KVCache:
    """fp16 K/V in the contiguous [B][Hk][N][128] layout, or a paged pool
    [pages][Hk][16][128] with page_table [B][max_pages].  key_bits is the width
    of the quantised key cache that goes with it (4, or 2)."""
    k: torch.Tensor
    v: Optional[torch.Tensor]
    seq_lens: torch.Tensor
    page_table: Optional[torch.Tensor] = None
    key_bits: int = 4

    def __post_init__(self):
        _need(self.k, torch.float16, "k")
        if self.v is not None:
            _need(self.v, torch.float16, "v")
            if self.v.shape != self.k.shape:
                raise ValueError("k and v must have the same shape")
        _need(self.seq_lens, torch.int32, "seq_lens")
        if self.k.shape[-1] != HEAD_DIM:
            raise ValueError("head_dim must be 128")
        if self.page_table is not None:
            _need(self.page_table, torch.int32, "page_table")
            if self.k.dim() != 4 or self.k.shape[2] != PAGE:
                raise ValueError("paged k must be [pages][Hk][16][128]")
        elif self.k.dim() != 4:
            raise ValueError("contiguous k must be [B][Hk][N][128]")
        if self.key_bits not in KEY_BITS:
            raise ValueError(f"key_bits must be one of {KEY_BITS}")

    @property
    def code_bytes(self) -> int:
        """Bytes of codes per token row: 128 * key_bits / 8."""
        return HEAD_DIM * self.key_bits // 8

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    @property
    def B(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def Hk(self) -> int:
        return int(self.k.shape[1])

    @property
    def N(self) -> int:
        return int(self.page_table.shape[1]) * PAGE if self.paged else int(self.k.shape[2])

    @property
    def max_pages(self) -> int:
        return (self.N + PAGE - 1) // PAGE

    def struct(self) -> TwKv:
        s = TwKv()
        s.k = _ptr(self.k)
        s.v = _ptr(self.v)
        s.batch = self.B
        s.num_kv_heads = self.Hk
        s.max_seq_len = self.N
        s.seq_lens = _ptr(self.seq_lens)
        s.page_table = _ptr(self.page_table)
        s.max_pages_per_seq = int(self.page_table.shape[1]) if self.paged else 0
        s.num_pool_pages = int(self.k.shape[0]) if self.paged else 0
        s.page_size = PAGE
        s.head_dim = HEAD_DIM
        s.key_bits = self.key_bits
        return s

    def row_shape(self, last: int):
        """Shape of a per-token companion array (codes, scales, zeros)."""
        if self.paged:
            return (self.k.shape[0], self.Hk, PAGE, last)
        return (self.B, self.Hk, self.N, last)

    def meta_shape(self):
        if self.paged:
            return (self.k.shape[0], self.Hk, 2, HEAD_DIM)
        return (self.B, self.Hk, self.max_pages, 2, HEAD_DIM)

    @classmethod
    def from_workload(cls, w, key_bits: int = 4) -> "KVCache":
        return cls(w.k, w.v, w.seq_lens, w.page_table, key_bits)


@dataclasses.dataclass
class Int4Keys:
    """The quantised key cache (4-bit, or 2-bit when its KVCache says so)."""
    codes: torch.Tensor    # uint8  [..][128 * key_bits / 8]
    scales: torch.Tensor   # fp16   [..][4]
    zeros: torch.Tensor    # fp16   [..][4]


def _check_keys(kv: KVCache, keys: Int4Keys) -> None:
    if tuple(keys.codes.shape) != kv.row_shape(kv.code_bytes):
        raise ValueError(f"codes must be {kv.row_shape(kv.code_bytes)} for "
                         f"{kv.key_bits}-bit keys, got {tuple(keys.codes.shape)}")


def quantize_keys(kv: KVCache, out: Optional[Int4Keys] = None, stream=None) -> Int4Keys:
    """Per-token asymmetric key cache (group 32, kv.key_bits wide): tw_quantize_keys."""
    lib = _capi.load()
    if out is None:
        dev = kv.k.device
        out = Int4Keys(torch.zeros(kv.row_shape(kv.code_bytes), dtype=torch.uint8, device=dev),
                       torch.zeros(kv.row_shape(4), dtype=torch.float16, device=dev),
                       torch.zeros(kv.row_shape(4), dtype=torch.float16, device=dev))
    _check_keys(kv, out)
    s = kv.struct()
    check(lib.tw_quantize_keys(ctypes.byref(s), _ptr(out.codes), _ptr(out.scales),
                               _ptr(out.zeros), _stream(stream)), "tw_quantize_keys")
    return out


def page_meta(kv: KVCache, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Quest per-page channel-wise key min / max: tw_page_meta."""
    lib = _capi.load()
    if out is None:
        out = torch.zeros(kv.meta_shape(), dtype=torch.float16, device=kv.k.device)
    s = kv.struct()
    check(lib.tw_page_meta(ctypes.byref(s), _ptr(out), _stream(stream)), "tw_page_meta")
    return out


def append_keys(kv: KVCache, keys: Int4Keys, meta: Optional[torch.Tensor] = None,
                stream=None) -> None:
    """tw_append_keys: quantise the newest token (position seq_lens[b] - 1) of
    every sequence into `keys` and fold it into `meta` (if given).  The caller
    writes that token's K / V rows and raises seq_lens first."""
    lib = _capi.load()
    _check_keys(kv, keys)
    s = kv.struct()
    check(lib.tw_append_keys(ctypes.byref(s), _ptr(keys.codes), _ptr(keys.scales),
                             _ptr(keys.zeros), _ptr(meta), _stream(stream)), "tw_append_keys")


def workspace_bytes(B: int, Hq: int, Hk: int, N: int, capacity: int) -> int:
    lib = _capi.load()
    n = ctypes.c_size_t(0)
    check(lib.tw_workspace_size(B, Hq, Hk, N, capacity, ctypes.byref(n)), "tw_workspace_size")
    return int(n.value)


def new_workspace(B, Hq, Hk, N, capacity, device) -> torch.Tensor:
    """A workspace with its device status word (the first 4 bytes) zeroed."""
    ws = torch.empty(max(workspace_bytes(B, Hq, Hk, N, capacity), 256), dtype=torch.uint8,
                     device=device)
    ws[:256].zero_()
    return ws


def device_status(ws: torch.Tensor) -> int:
    """The workspace's device status word (synchronises): 0, or bit 0 set when a
    bounded wait of the selection kernel gave up (that call's outputs are
    invalid; the C API calls it TW_ERR_TIMEOUT)."""
    return int(ws[:4].view(torch.int32).item())


def budget_pages(budget_tokens: Optional[int], kv: KVCache) -> int:
    return min(budget_tokens // PAGE, kv.max_pages)


def select_pages(q: torch.Tensor, kv: KVCache, meta: torch.Tensor, budget_tokens: int,
                 ws: Optional[torch.Tensor] = None, stream=None):
    """Quest top-K_p pages per (b, KV head): tw_select_pages -> (cand_pages, ncand)."""
    lib = _capi.load()
    _need(q, torch.float16, "q")
    Hq = int(q.shape[1])
    stride = max(1, budget_pages(budget_tokens, kv))
    cand = torch.zeros((kv.B, kv.Hk, stride), dtype=torch.int32, device=q.device)
    ncand = torch.zeros((kv.B, kv.Hk), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = new_workspace(kv.B, Hq, kv.Hk, kv.N, 1, q.device)
    s = kv.struct()
    check(lib.tw_select_pages(_ptr(q), Hq, ctypes.byref(s), _ptr(meta), int(budget_tokens),
                              _ptr(cand), stride, _ptr(ncand), _ptr(ws), ws.numel(),
                              _stream(stream)), "tw_select_pages")
    return cand, ncand


def num_sets(kv: KVCache, Hq: int, group_mode: int) -> int:
    return kv.B * kv.Hk if (group_mode or Hq == kv.Hk) else kv.B * Hq


def topp_prune(q: torch.Tensor, kv: KVCache, keys: Int4Keys, cand: Optional[torch.Tensor],
               ncand: Optional[torch.Tensor], p: float, group_mode: int = 0,
               capacity: Optional[int] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Twilight top-p pruning of the candidates: tw_topp_prune -> (idx, count)."""
    lib = _capi.load()
    _need(q, torch.float16, "q")
    _check_keys(kv, keys)
    Hq = int(q.shape[1])
    stride = int(cand.shape[-1]) if cand is not None else 0
    if capacity is None:
        capacity = min(stride, kv.max_pages) * PAGE if cand is not None else kv.N
        capacity = max(capacity, 1)
    U = num_sets(kv, Hq, group_mode)
    idx = torch.zeros((U, capacity), dtype=torch.int32, device=q.device)
    count = torch.zeros((U,), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = new_workspace(kv.B, Hq, kv.Hk, kv.N, capacity, q.device)
    s = kv.struct()
    check(lib.tw_topp_prune(_ptr(q), Hq, ctypes.byref(s), _ptr(keys.codes), _ptr(keys.scales),
                            _ptr(keys.zeros), _ptr(cand), stride, _ptr(ncand), float(p),
                            int(group_mode), _ptr(idx), capacity, _ptr(count), _ptr(ws),
                            ws.numel(), _stream(stream)), "tw_topp_prune")
    return idx, count


def sparse_decode(q: torch.Tensor, kv: KVCache, idx: torch.Tensor, count: torch.Tensor,
                  group_mode: int = 0, ws: Optional[torch.Tensor] = None, with_lse: bool = True,
                  stream=None):
    """Exact attention over the selected tokens: tw_sparse_decode -> (out, lse)."""
    lib = _capi.load()
    _need(q, torch.float16, "q")
    _need(idx, torch.int32, "idx")
    Hq = int(q.shape[1])
    capacity = int(idx.shape[-1])
    out = torch.empty((kv.B, Hq, HEAD_DIM), dtype=torch.float16, device=q.device)
    lse = torch.empty((kv.B, Hq), dtype=torch.float32, device=q.device) if with_lse else None
    if ws is None:
        ws = new_workspace(kv.B, Hq, kv.Hk, kv.N, capacity, q.device)
    s = kv.struct()
    check(lib.tw_sparse_decode(_ptr(q), Hq, ctypes.byref(s), _ptr(idx), capacity, _ptr(count),
                               int(group_mode), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                               _stream(stream)), "tw_sparse_decode")
    return out, lse


class DecodeStep:
    """Pre-allocated buffers for repeated tw_decode_step calls on one shape.

    budget_tokens None (or <= 0) means base = full attention (every token is a
    candidate); otherwise Quest keeps budget_tokens // 16 pages first.
    append_keys: each call first folds the newest token of every sequence into
    the int4 cache and the page metadata (tw_append_keys inside the step)."""

    def __init__(self, kv: KVCache, keys: Int4Keys, meta: Optional[torch.Tensor], Hq: int,
                 budget_tokens: Optional[int], p: float, group_mode: int = 0,
                 with_lse: bool = True, append_keys: bool = False):
        _check_keys(kv, keys)
        self.kv, self.keys, self.meta = kv, keys, meta
        self.append = bool(append_keys)
        self.Hq = Hq
        self.budget = int(budget_tokens) if budget_tokens and budget_tokens > 0 else 0
        self.p = float(p)
        self.group_mode = int(group_mode)
        dev = kv.k.device
        if self.budget:
            self.cand_stride = max(1, budget_pages(self.budget, kv))
            self.capacity = self.cand_stride * PAGE
        else:
            self.cand_stride = 1
            self.capacity = max(kv.N, 1)
        self.cand = torch.zeros((kv.B, kv.Hk, self.cand_stride), dtype=torch.int32, device=dev)
        self.ncand = torch.zeros((kv.B, kv.Hk), dtype=torch.int32, device=dev)
        U = num_sets(kv, Hq, group_mode)
        self.idx = torch.zeros((U, self.capacity), dtype=torch.int32, device=dev)
        self.count = torch.zeros((U,), dtype=torch.int32, device=dev)
        self.out = torch.zeros((kv.B, Hq, HEAD_DIM), dtype=torch.float16, device=dev)
        self.lse = torch.zeros((kv.B, Hq), dtype=torch.float32, device=dev) if with_lse else None
        self.ws = new_workspace(kv.B, Hq, kv.Hk, kv.N, self.capacity, dev)
        self._q = None
        self._s = None
        self._q_stage = None   # device staging of the query for run_host

    def _struct(self, q: torch.Tensor) -> TwStep:
        if self._s is not None and self._q is q:
            return self._s
        _need(q, torch.float16, "q")
        if tuple(q.shape) != (self.kv.B, self.Hq, HEAD_DIM):
            raise ValueError(f"q must be [{self.kv.B}][{self.Hq}][128]")
        s = TwStep()
        s.q = _ptr(q)
        s.num_q_heads = self.Hq
        s.kv = self.kv.struct()
        s.codes, s.scales, s.zeros = (_ptr(self.keys.codes), _ptr(self.keys.scales),
                                      _ptr(self.keys.zeros))
        s.meta = _ptr(self.meta)
        s.budget_tokens = self.budget
        s.p = self.p
        s.group_mode = self.group_mode
        s.cand_pages, s.cand_stride, s.ncand = _ptr(self.cand), self.cand_stride, _ptr(self.ncand)
        s.idx, s.capacity, s.count = _ptr(self.idx), self.capacity, _ptr(self.count)
        s.out, s.lse = _ptr(self.out), _ptr(self.lse)
        s.ws, s.ws_bytes = _ptr(self.ws), self.ws.numel()
        s.append_keys = 1 if self.append else 0
        self._q, self._s = q, s
        return s

    def __call__(self, q: torch.Tensor, stream=None) -> torch.Tensor:
        lib = _capi.load()
        s = self._struct(q)
        check(lib.tw_decode_step(ctypes.byref(s), _stream(stream)), "tw_decode_step")
        return self.out

    def run_host(self, q_host: torch.Tensor, out_host: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        """One step with the query taken from, and the output returned to,
        pinned host memory (tw_decode_step_host): the copies run as kernels of
        the step's launch chain.  q_host / out_host: pinned CPU fp16
        [B][Hq][128].  The step's device q / out buffers serve as staging.
        Synchronise the stream before reading out_host."""
        lib = _capi.load()
        shape = (self.kv.B, self.Hq, HEAD_DIM)
        if out_host is None:
            out_host = torch.empty(shape, dtype=torch.float16).pin_memory()
        for t, name in ((q_host, "q_host"), (out_host, "out_host")):
            if t.dtype != torch.float16 or t.is_cuda or not t.is_pinned() or \
                    not t.is_contiguous() or tuple(t.shape) != shape:
                raise ValueError(f"{name} must be a contiguous pinned CPU fp16 tensor {shape}")
        if self._q_stage is None:
            self._q_stage = torch.empty(shape, dtype=torch.float16, device=self.kv.k.device)
        s = self._struct(self._q_stage)
        check(lib.tw_decode_step_host(ctypes.byref(s), q_host.data_ptr(), out_host.data_ptr(),
                                      _stream(stream)), "tw_decode_step_host")
        return out_host

    def kernel_names(self):
        lib = _capi.load()
        s = self._struct(self._q) if self._q is not None else None
        if s is None:
            raise RuntimeError("call the step once before asking for kernel names")
        n = lib.tw_decode_step_num_kernels(ctypes.byref(s))
        return [lib.tw_decode_step_kernel_name(ctypes.byref(s), i).decode() for i in range(n)]

    def profiled(self, q: torch.Tensor, events, stream=None) -> None:
        """Run one step recording events[0] before and events[i+1] after kernel i."""
        lib = _capi.load()
        s = self._struct(q)
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        check(lib.tw_decode_step_profiled(ctypes.byref(s), arr, len(events), _stream(stream)),
              "tw_decode_step_profiled")


def prepare(w, device=None, key_bits: int = 4):
    """Move a workload to the GPU and build its quantised key cache (key_bits
    wide) and page metadata with the library.  Returns (kv, keys, meta, q)."""
    if device is not None:
        w = w.to(device)
    kv = KVCache.from_workload(w, key_bits)
    keys = quantize_keys(kv)
    meta = page_meta(kv)
    return kv, keys, meta, w.q


# ----------------------------------------------------------------------------- label selector
def label_cache(kv: KVCache, channels: torch.Tensor, out: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """Label cache of the token-level label-channel selector (tw_label_cache):
    the fp16 values of channels[h] (int32 CUDA [Hk][r]) of every key row."""
    lib = _capi.load()
    _need(channels, torch.int32, "channels")
    r = int(channels.shape[-1])
    if tuple(channels.shape) != (kv.Hk, r):
        raise ValueError(f"channels must be [{kv.Hk}][r]")
    if out is None:
        out = torch.zeros(kv.row_shape(r), dtype=torch.float16, device=kv.k.device)
    s = kv.struct()
    check(lib.tw_label_cache(ctypes.byref(s), _ptr(channels), r, _ptr(out), _stream(stream)),
          "tw_label_cache")
    return out


def _check_labels(kv: KVCache, labels: torch.Tensor, channels: torch.Tensor) -> int:
    """Label cache and channels of a KV cache: fp16 rows of r values, int32
    [Hk][r] channels.  Returns r."""
    _need(labels, torch.float16, "labels")
    _need(channels, torch.int32, "channels")
    r = int(channels.shape[-1]) if channels.dim() == 2 else -1
    if tuple(channels.shape) != (kv.Hk, r) or not 1 <= r <= 32:
        raise ValueError(f"channels must be int32 [{kv.Hk}][r] with 1 <= r <= 32")
    if tuple(labels.shape) != kv.row_shape(r):
        raise ValueError(f"labels must be {kv.row_shape(r)}, got {tuple(labels.shape)}")
    return r


def _check_cand_tokens(kv: KVCache, cand: torch.Tensor, ncand: torch.Tensor) -> int:
    """Token candidates [B][Hk][stride] and their counts [B][Hk] (int32).
    Returns stride."""
    _need(cand, torch.int32, "cand")
    _need(ncand, torch.int32, "ncand")
    stride = int(cand.shape[-1]) if cand.dim() == 3 else -1
    if tuple(cand.shape) != (kv.B, kv.Hk, stride) or stride < 1:
        raise ValueError(f"cand must be int32 [{kv.B}][{kv.Hk}][stride]")
    if tuple(ncand.shape) != (kv.B, kv.Hk):
        raise ValueError(f"ncand must be int32 [{kv.B}][{kv.Hk}]")
    return stride


def token_workspace_bytes(B, Hq, Hk, N, cand_stride, capacity, key_bits=4) -> int:
    lib = _capi.load()
    n = ctypes.c_size_t(0)
    check(lib.tw_token_workspace_size(B, Hq, Hk, N, cand_stride, capacity, key_bits,
                                      ctypes.byref(n)), "tw_token_workspace_size")
    return int(n.value)


def _token_ws(kv, Hq, stride, capacity, device):
    n = max(token_workspace_bytes(kv.B, Hq, kv.Hk, kv.N, stride, capacity, kv.key_bits), 256)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()   # the device status word
    return ws


def select_tokens(q: torch.Tensor, kv: KVCache, labels: torch.Tensor, channels: torch.Tensor,
                  budget_tokens: int, ws: Optional[torch.Tensor] = None, stream=None):
    """Token-level label-channel pre-selection (tw_select_tokens) ->
    (cand_tokens [B][Hk][stride], ncand [B][Hk]), stride = min(budget, N)."""
    lib = _capi.load()
    _need(q, torch.float16, "q")
    Hq = int(q.shape[1])
    r = _check_labels(kv, labels, channels)
    stride = max(1, min(int(budget_tokens), kv.N))
    cand = torch.zeros((kv.B, kv.Hk, stride), dtype=torch.int32, device=q.device)
    ncand = torch.zeros((kv.B, kv.Hk), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = _token_ws(kv, Hq, stride, stride, q.device)
    s = kv.struct()
    check(lib.tw_select_tokens(_ptr(q), Hq, ctypes.byref(s), _ptr(labels), _ptr(channels), r,
                               int(budget_tokens), _ptr(cand), stride, _ptr(ncand), _ptr(ws),
                               ws.numel(), _stream(stream)), "tw_select_tokens")
    return cand, ncand


def topp_prune_tokens(q: torch.Tensor, kv: KVCache, keys: Int4Keys, cand: torch.Tensor,
                      ncand: torch.Tensor, p: float, group_mode: int = 0,
                      capacity: Optional[int] = None, ws: Optional[torch.Tensor] = None,
                      stream=None):
    """Twilight top-p over token candidates (tw_topp_prune_tokens) -> (idx, count)."""
    lib = _capi.load()
    _need(q, torch.float16, "q")
    _check_keys(kv, keys)
    Hq = int(q.shape[1])
    stride = _check_cand_tokens(kv, cand, ncand)
    capacity = stride if capacity is None else int(capacity)
    U = num_sets(kv, Hq, group_mode)
    idx = torch.zeros((U, capacity), dtype=torch.int32, device=q.device)
    count = torch.zeros((U,), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = _token_ws(kv, Hq, stride, capacity, q.device)
    s = kv.struct()
    check(lib.tw_topp_prune_tokens(_ptr(q), Hq, ctypes.byref(s), _ptr(keys.codes),
                                   _ptr(keys.scales), _ptr(keys.zeros), _ptr(cand), stride,
                                   _ptr(ncand), float(p), int(group_mode), _ptr(idx), capacity,
                                   _ptr(count), _ptr(ws), ws.numel(), _stream(stream)),
          "tw_topp_prune_tokens")
    return idx, count


class LabelDecodeStep:
    """A decode step with the token-level label-channel base selector:
    tw_select_tokens -> tw_topp_prune_tokens -> tw_sparse_decode on one
    stream with pre-allocated buffers (no host synchronisation)."""

    NAMES = ("select_tokens", "topp_prune_tokens", "sparse_decode")
    LAUNCHES = 2 + 4 + 2   # kernels of the three calls

    def __init__(self, kv: KVCache, keys: Int4Keys, labels: torch.Tensor, channels: torch.Tensor,
                 Hq: int, budget_tokens: int, p: float, group_mode: int = 0,
                 with_lse: bool = True):
        _check_keys(kv, keys)
        _check_labels(kv, labels, channels)
        self.kv, self.keys, self.labels, self.channels = kv, keys, labels, channels
        self.Hq, self.budget, self.p, self.group_mode = Hq, int(budget_tokens), float(p), \
            int(group_mode)
        dev = kv.k.device
        self.stride = max(1, min(self.budget, kv.N))
        self.capacity = self.stride
        self.cand = torch.zeros((kv.B, kv.Hk, self.stride), dtype=torch.int32, device=dev)
        self.ncand = torch.zeros((kv.B, kv.Hk), dtype=torch.int32, device=dev)
        U = num_sets(kv, Hq, group_mode)
        self.idx = torch.zeros((U, self.capacity), dtype=torch.int32, device=dev)
        self.count = torch.zeros((U,), dtype=torch.int32, device=dev)
        self.out = torch.zeros((kv.B, Hq, HEAD_DIM), dtype=torch.float16, device=dev)
        self.lse = torch.zeros((kv.B, Hq), dtype=torch.float32, device=dev) if with_lse else None
        n = max(token_workspace_bytes(kv.B, Hq, kv.Hk, kv.N, self.stride, self.capacity,
                                      kv.key_bits),
                workspace_bytes(kv.B, Hq, kv.Hk, kv.N, self.capacity), 256)
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)
        self.ws[:256].zero_()   # the device status word
        self._kvs = kv.struct()
        self._q_stage = None

    def _calls(self, q: torch.Tensor, stream):
        lib = _capi.load()
        st = _stream(stream)
        kvs, ws, nws = ctypes.byref(self._kvs), _ptr(self.ws), self.ws.numel()
        r = int(self.channels.shape[-1])
        yield lambda: check(lib.tw_select_tokens(
            _ptr(q), self.Hq, kvs, _ptr(self.labels), _ptr(self.channels), r, self.budget,
            _ptr(self.cand), self.stride, _ptr(self.ncand), ws, nws, st), "tw_select_tokens")
        yield lambda: check(lib.tw_topp_prune_tokens(
            _ptr(q), self.Hq, kvs, _ptr(self.keys.codes), _ptr(self.keys.scales),
            _ptr(self.keys.zeros), _ptr(self.cand), self.stride, _ptr(self.ncand), self.p,
            self.group_mode, _ptr(self.idx), self.capacity, _ptr(self.count), ws, nws, st),
            "tw_topp_prune_tokens")
        yield lambda: check(lib.tw_sparse_decode(
            _ptr(q), self.Hq, kvs, _ptr(self.idx), self.capacity, _ptr(self.count),
            self.group_mode, _ptr(self.out), _ptr(self.lse), ws, nws, st), "tw_sparse_decode")

    def __call__(self, q: torch.Tensor, stream=None) -> torch.Tensor:
        _need(q, torch.float16, "q")
        for call in self._calls(q, stream):
            call()
        return self.out

    def kernel_names(self):
        return list(self.NAMES)

    def profiled(self, q: torch.Tensor, events, stream=None) -> None:
        """One step with events[0] before and events[i + 1] after call i."""
        s = torch.cuda.current_stream() if stream is None else stream
        events[0].record(s)
        for i, call in enumerate(self._calls(q, stream)):
            call()
            events[i + 1].record(s)

    def run_host(self, q_host: torch.Tensor, out_host: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        """One step from and to pinned host memory (copy-engine transfers)."""
        if out_host is None:
            out_host = torch.empty(tuple(self.out.shape), dtype=torch.float16).pin_memory()
        if self._q_stage is None:
            self._q_stage = torch.empty(tuple(self.out.shape), dtype=torch.float16,
                                        device=self.kv.k.device)
        self._q_stage.copy_(q_host, non_blocking=True)
        self(self._q_stage, stream)
        out_host.copy_(self.out, non_blocking=True)
        return out_host
