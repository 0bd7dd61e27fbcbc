#!/usr/bin/env python
"""Benchmark of one Twilight decode step per layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
                    [--key-bits 4|2]

A step is one pass of the whole hot path over one decode layer: Quest page
scores + top-K_p pages -> int4 weight estimate + top-p threshold + index
compaction -> split-K sparse attention + log-sum-exp merge (the KV cache, its
4-bit key companion and the page metadata are built beforehand, as at
prefill).  The default workload is the Llama-2-7B-shaped MHA layer: batch 1, 32
heads, context 32768, Quest budget 8192 tokens, p = 0.85.  --key-bits 2 runs
the same step on the 2-bit key cache of the paper's quantisation ablation.

The timed region replays the step over R independent copies of the cache in
rotation, so the bytes touched between two visits of a copy exceed the 126 MB
L2.  Times are CUDA events on the launching stream, max over ranks.  With N > 1
(torchrun) each rank runs an independent replica on its own GPU: the path has
no exchange step, so there is no collective on the data path.

--impl reference times the CPU oracle on the host cores on a bounded sample of
the same workload and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "µs per decode step (top-p prune + sparse attn) per layer; achieved HBM GB/s"
UNIT = "us/step"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "ncu_traffic.json")
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="batched_paged",
                    choices=["llama2_mha", "llama3_gqa", "batched_paged", "sweep", "tiny"])
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other workloads' step times in the JSON line")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--copies", type=int, default=0,
                    help="rotating cache copies (0: enough to exceed L2 several times)")
    ap.add_argument("--key-bits", type=int, default=4, choices=[4, 2],
                    help="width of the quantised key cache used for the weight estimate")
    ap.add_argument("--selector", default="quest", choices=["quest", "label"],
                    help="base selector: Quest pages, or token-level label channels "
                         "(synthetic Double Sparsity, 16 channels per KV head)")
    ap.add_argument("--batch", type=int, default=0,
                    help="batched_paged only: this many sequences instead of 16 (a smaller "
                         "case of the same workload, for profiler captures that must stay "
                         "small on the device)")
    return ap.parse_args()


def make_workload(name, device, batch=0):
    import workloads as W
    if batch > 0:
        if name != "batched_paged":
            raise SystemExit("--batch applies to batched_paged only")
        return W.batched_paged(device=device, B=batch)
    return W.CONFIGS[name](device=device)


def workload_config(w, key_bits=4, selector="quest"):
    c = {"workload": w.name, "batch": w.B, "q_heads": w.Hq, "kv_heads": w.Hk,
         "context": w.N, "paged": w.paged, "budget_tokens": w.budget_tokens, "p": w.p,
         "group_mode": w.group_mode, "head_dim": 128, "page_size": 16, "key_bits": key_bits,
         "key_group": 32, "selector": selector}
    if selector == "label":
        c["label_channels"] = LABEL_R
    return c


def l2_policy(copies, copy_bytes):
    return (f"inputs larger than L2: {copies} rotating cache copies, "
            f"{copy_bytes / 1e9:.2f} GB each")


# Device sources of the kernels the traffic record measures (and the headers
# they include): the record is used only while these bytes are unchanged.
TRAFFIC_SOURCES = ("cache_build.cu", "decode.cu", "host_io.cu", "resolve.cu", "select_prune.cu",
                   "tw_bulk.cuh", "tw_common.cuh", "tw_kernels.h")


def _code_only(text: str) -> str:
    """C++ source without comments or blank lines: what a comment edit leaves alone."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def src_hash():
    """Hash of the measured kernels' device sources (code only), so that an ncu
    capture stays attached to the code it was taken on."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "adaptive_top_sparse_quest_b200", "csrc")
    for f in TRAFFIC_SOURCES:
        h.update(f.encode())
        h.update(_code_only(open(os.path.join(d, f)).read()).encode())
    return h.hexdigest()[:16]


def reduce_max(x: float, world: int, device) -> float:
    """Max of a per-rank time over all ranks (the job's time is its slowest rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_step(max_elapsed_ms: float, steps: int, world: int) -> float:
    """Replicas: every rank runs `steps` independent decode steps, so the job
    completes steps * world steps in the slowest rank's time."""
    return max_elapsed_ms * 1e3 / (steps * world)


def hbm_peak():
    try:
        pk = json.load(open(PEAKS_PATH))
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while load runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if not (t0 <= ts <= t1):
                continue
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle
def _oracle_unit_inputs(x, w_cpu, b, hk, key_bits, label_channels):
    """One (sequence, KV head) unit's cache companions, built as at prefill
    (outside every timed region)."""
    import oracle as O
    G = x.Hq // x.Hk
    L = int(x.seq_lens[b])
    k_seq = O.sequence_rows(x.k, x.page_table, b, hk, L)
    v_seq = O.sequence_rows(x.v, x.page_table, b, hk, L)
    codes, scales, zeros = O.quantize_keys(k_seq, key_bits)
    meta = O.page_meta(k_seq, L) if w_cpu.budget_tokens else None
    labels = O.label_cache(k_seq, label_channels[hk]) if label_channels is not None else None
    return dict(L=L, k=k_seq, v=v_seq, codes=codes, scales=scales, zeros=zeros, meta=meta,
                labels=labels, qg=x.q[b, hk * G:(hk + 1) * G], hk=hk)


def _oracle_unit_step(u, w_cpu, G, key_bits, label_channels):
    """The oracle's decode step of one unit: base selector, quantised-key
    estimate, top-p, sparse attention."""
    import oracle as O
    qg = u["qg"]
    if u["labels"] is not None:
        toks = O.select_tokens(O.label_scores(qg, u["labels"], label_channels[u["hk"]]),
                               w_cpu.budget_tokens)
    else:
        pages = None
        if w_cpu.budget_tokens:
            pages = O.select_pages(O.quest_page_scores(qg, u["meta"]), w_cpu.budget_tokens)
        toks = O.candidate_tokens(pages, u["L"])
    lg = O.estimate_logits(qg, u["codes"][toks], u["scales"][toks], u["zeros"][toks], key_bits)
    if w_cpu.group_mode and G > 1:
        sel = O.topp_select(O.group_weights(lg), w_cpu.p)[0]
        sels = [sel] * G
    else:
        sels = [O.topp_select(O.softmax_weights(lg[:, g]), w_cpu.p)[0] for g in range(G)]
    for g in range(G):
        t = toks[sels[g]]
        O.sparse_attention(qg[g], u["k"][t], u["v"][t])


def _single_thread_blas():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except Exception:
        return None


def cpu_step_sample(w_cpu, seconds: float, max_units=None, key_bits=4, label_channels=None):
    """Time the oracle's decode step (page scores, top-K_p, quantised-key
    estimate, top-p, sparse attention) on (b, kv head) units of the workload
    until `seconds` of CPU work, single-threaded; the key cache and page
    metadata are built first, untimed, as at prefill.  Returns (us per full
    step, units timed, total units, threads).  With label_channels the base
    selector is the token-level label-channel one instead of Quest's pages."""
    limiter = _single_thread_blas()
    import numpy as np

    import oracle as O
    x = O.SeqInputs.from_workload(w_cpu)
    G = x.Hq // x.Hk
    units = [(b, h) for b in range(x.B) for h in range(x.Hk)]
    order = np.random.default_rng(0).permutation(len(units))
    spent, n = 0.0, 0
    for ui in order:
        if max_units is not None and n >= max_units:
            break
        b, hk = units[ui]
        u = _oracle_unit_inputs(x, w_cpu, b, hk, key_bits, label_channels)
        t0 = time.perf_counter()
        _oracle_unit_step(u, w_cpu, G, key_bits, label_channels)
        spent += time.perf_counter() - t0
        n += 1
        if spent >= seconds:
            break
    if limiter is not None and hasattr(limiter, "unregister"):
        limiter.unregister()
    return spent / n * len(units) * 1e6, n, len(units), 1


def cpu_step_all_cores(w_cpu, per_unit_us: float, seconds: float, key_bits=4,
                       label_channels=None):
    """The same oracle step on all host cores: a thread pool with one worker
    per core runs whole units concurrently (numpy releases the interpreter
    lock in its array work; each worker's BLAS is single-threaded).  About
    `seconds` of wall time from the single-thread per-unit cost; the inputs of
    the sampled units are built first, untimed.  Returns (us per full step,
    units timed, total units, threads)."""
    import concurrent.futures as cf

    import numpy as np

    import oracle as O
    limiter = _single_thread_blas()
    threads = os.cpu_count() or 1
    x = O.SeqInputs.from_workload(w_cpu)
    G = x.Hq // x.Hk
    units = [(b, h) for b in range(x.B) for h in range(x.Hk)]
    want = int(seconds * 1e6 / max(per_unit_us, 1.0) * threads)
    n = max(threads, min(want, 4 * threads, len(units)))
    n = min(n, len(units))
    order = np.random.default_rng(1).permutation(len(units))[:n]
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        prepared = list(ex.map(lambda i: _oracle_unit_inputs(x, w_cpu, *units[i], key_bits,
                                                             label_channels), order))
        t0 = time.perf_counter()
        list(ex.map(lambda u: _oracle_unit_step(u, w_cpu, G, key_bits, label_channels),
                    prepared))
        wall = time.perf_counter() - t0
    if limiter is not None and hasattr(limiter, "unregister"):
        limiter.unregister()
    return wall / n * len(units) * 1e6, n, len(units), threads


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    # the same seeded workload as the GPU arm: generated where that arm generates
    # it (the device generator draws other numbers than the host one), then
    # brought to the host for the oracle
    gen = "cuda" if torch.cuda.is_available() else "cpu"
    w = make_workload(args.config, gen, args.batch)
    if gen != "cpu":
        w = w.to("cpu")
        torch.cuda.empty_cache()
    chans = None
    if args.selector == "label":
        import workloads as W
        chans = W.label_channels(w, r=LABEL_R)
    per = []
    for i in range(args.warmup + args.steps):
        us, n, tot, cores = cpu_step_sample(w, 0.0, max_units=1, key_bits=args.key_bits,
                                            label_channels=chans)
        if i >= args.warmup:
            per.append(us)
    value = statistics.mean(per)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": value / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, key_bits=args.key_bits, selector=args.selector),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"each step: 1 random (sequence, KV head) unit of {tot}, "
                                   "scaled by the unit count"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
LABEL_R = 16


def label_algorithmic_bytes(w, step, key_bits=4):
    """Bytes the label-selector step must move (per call): the label cache
    (2 B per label channel per token per KV head) and the scores written and
    read back (4 + 4 B); the candidates' quantised keys read, copied and read
    again by the estimate (3 x (128 * key_bits / 8 + 16) B); the selected
    tokens' fp16 K+V rows (512 B per token per set)."""
    import torch
    toks = int(w.seq_lens.to(torch.int64).sum()) * w.Hk
    cand_tokens = int(step.ncand.to(torch.int64).sum())
    kept = step.count.to(torch.int64).cpu()
    return {"select_tokens": toks * (2 * LABEL_R + 8),
            "topp_prune_tokens": cand_tokens * 3 * (128 * key_bits // 8 + 16),
            "sparse_decode": int(kept.sum()) * 512}, cand_tokens, kept


def algorithmic_bytes(w, step, key_bits=4):
    """Bytes the step must move (per kernel): the selection kernel reads the
    page metadata (512 B per page per KV head) and the quantised candidate keys
    (128 * key_bits / 8 B of codes + 16 B of scales and zeros per candidate
    token per KV head: 80 B at 4 bits, 48 B at 2 bits); the attention kernel
    reads the fp16 K+V rows of the selected tokens (512 B per token per set)."""
    import torch
    lens = w.seq_lens.to(torch.int64).cpu()
    pages = (lens + 15) // 16
    meta_b = int(pages.sum()) * w.Hk * 512 if w.budget_tokens else 0
    if w.budget_tokens:
        nc = step.ncand.to(torch.int64).cpu()          # [B][Hk] pages
        cand_tokens = 0
        for b in range(w.B):
            for h in range(w.Hk):
                # every candidate page is full except possibly the sequence's last page
                n = int(nc[b, h]) * 16
                last = int(lens[b]) - (int(pages[b]) - 1) * 16
                sel = step.cand[b, h, :int(nc[b, h])].cpu()
                if int(pages[b]) - 1 in sel.tolist():
                    n -= 16 - last
                cand_tokens += n
    else:
        cand_tokens = int(lens.sum()) * w.Hk
    int4_b = cand_tokens * (128 * key_bits // 8 + 16)
    kept = step.count.to(torch.int64).cpu()
    kv_b = int(kept.sum()) * 512
    first = "select_prune" if w.budget_tokens else "prune"
    return {first: meta_b + int4_b, "sparse_decode": kv_b}, cand_tokens, kept


PER_CONFIGS = ("llama2_mha", "llama3_gqa", "sweep")
NOMINAL_HBM_GBS = 8000.0


def time_workload(w, dev, key_bits, steps, warmup):
    """Device time of the decode step on another workload (the same rotating
    cache copies and CUDA-event timing as the headline), with its algorithmic
    bytes and roofline fractions."""
    import torch

    from adaptive_top_sparse_quest_b200 import DecodeStep, KVCache, page_meta, quantize_keys
    kv0 = KVCache.from_workload(w, key_bits)
    keys0 = quantize_keys(kv0)
    meta0 = page_meta(kv0)
    torch.cuda.synchronize()
    copy_bytes = sum(t.numel() * t.element_size() for t in
                     (w.k, w.v, keys0.codes, keys0.scales, keys0.zeros, meta0))
    R = 1
    while R * min(copy_bytes, 4 * 114e6) < 4 * L2_BYTES and R < 16:
        R += 1
    R = max(R, 4)
    steps_l = []
    for r in range(R):
        if r == 0:
            kv, keys, meta = kv0, keys0, meta0
        else:
            kv = KVCache(w.k.clone(), w.v.clone(), w.seq_lens.clone(),
                         None if w.page_table is None else w.page_table.clone(), key_bits)
            keys = type(keys0)(keys0.codes.clone(), keys0.scales.clone(), keys0.zeros.clone())
            meta = meta0.clone()
        steps_l.append(DecodeStep(kv, keys, meta, w.Hq, w.budget_tokens, w.p, w.group_mode))
    q = w.q.contiguous()
    for i in range(max(3, warmup)):
        steps_l[i % R](q)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st = torch.cuda.current_stream()
    e0.record(st)
    for i in range(steps):
        steps_l[i % R](q)
    e1.record(st)
    e1.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / steps
    kb, cand_tokens, kept = algorithmic_bytes(w, steps_l[0], key_bits)
    total = sum(kb.values())
    peak, peak_kind = hbm_peak()
    gbs = total / (us * 1e-6) / 1e9
    out = {"workload": w.name, "us_per_step": us, "bytes_per_step": total, "hbm_gbs": gbs,
           "frac_of_measured": gbs / peak, "frac_of_nominal_8000": gbs / NOMINAL_HBM_GBS,
           "peak_kind": peak_kind, "kept_tokens_mean": float(kept.double().mean()),
           "candidates_per_set": cand_tokens / max(1, w.B * w.Hk), "steps": steps,
           "l2": l2_policy(R, copy_bytes)}
    del steps_l, kv0, keys0, meta0
    torch.cuda.empty_cache()
    return out


def per_config_times(headline, dev, key_bits, steps, warmup):
    """The other single-GPU workloads' step times (the sweep at tau = 1, p = 0.85)."""
    import workloads as W
    res = {}
    for name in PER_CONFIGS:
        if name == headline:
            continue
        if name == "sweep":
            w = W.sweep_point(W.concentration_sweep(device=dev), 1.0, 0.85)
        else:
            w = W.CONFIGS[name](device=dev)
        res[name] = time_workload(w, dev, key_bits, steps, warmup)
        del w
    return res


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    from adaptive_top_sparse_quest_b200 import (DecodeStep, KVCache, LabelDecodeStep, _capi,
                                                append_keys, label_cache, page_meta,
                                                quantize_keys)
    from adaptive_top_sparse_quest_b200 import build as _b
    _b.build()
    _capi.load()

    w = make_workload(args.config, dev, args.batch)
    kv0 = KVCache.from_workload(w, args.key_bits)
    keys0 = quantize_keys(kv0)
    meta0 = page_meta(kv0)
    torch.cuda.synchronize()
    copy_bytes = sum(t.numel() * t.element_size() for t in
                     (w.k, w.v, keys0.codes, keys0.scales, keys0.zeros, meta0))
    touched_est = 114e6
    R = 1
    while R * min(copy_bytes, 4 * touched_est) < 4 * L2_BYTES and R < 16:
        R += 1
    R = max(R, 4)
    if args.copies > 0:
        R = args.copies

    # cache-build kernels timed once (GB/s over K read + int4/meta written)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    quantize_keys(kv0, keys0)
    ev[1].record()
    page_meta(kv0, meta0)
    ev[2].record()
    torch.cuda.synchronize()
    build_ms = (ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]))
    # incremental append of each sequence's newest token (idempotent at fixed
    # lengths, so it can be repeated): mean of 20 calls after 3 warm-up calls
    for _ in range(3):
        append_keys(kv0, keys0, meta0)
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record()
    for _ in range(20):
        append_keys(kv0, keys0, meta0)
    eb.record()
    torch.cuda.synchronize()
    append_us = ea.elapsed_time(eb) * 1e3 / 20

    label = args.selector == "label"
    if label and not w.budget_tokens:
        raise SystemExit("--selector label needs a workload with a token budget")
    if label:
        import workloads as W
        channels = torch.tensor(W.label_channels(w, r=LABEL_R), dtype=torch.int32, device=dev)

    def make_step(kv, keys, meta, p):
        if label:
            return LabelDecodeStep(kv, keys, label_cache(kv, channels), channels, w.Hq,
                                   w.budget_tokens, p, w.group_mode)
        return DecodeStep(kv, keys, meta, w.Hq, w.budget_tokens, p, w.group_mode)

    steps = []
    for r in range(R):
        if r == 0:
            kv, keys, meta = kv0, keys0, meta0
        else:
            kv = KVCache(w.k.clone(), w.v.clone(), w.seq_lens.clone(),
                         None if w.page_table is None else w.page_table.clone(), args.key_bits)
            keys = type(keys0)(keys0.codes.clone(), keys0.scales.clone(), keys0.zeros.clone())
            meta = meta0.clone()
        steps.append(make_step(kv, keys, meta, w.p))
    q = w.q.contiguous()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    for i in range(args.warmup):
        steps[i % R](q)
    barrier()
    t_start = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        steps[i % R](q)
    e1.record(stream)
    e1.synchronize()
    barrier()
    t_end = time.time()
    elapsed_ms = e0.elapsed_time(e1)
    # keep the GPU under the same load long enough for nvidia-smi to sample clocks
    t_load_end = t_end
    if sampler and t_end - t_start < 0.6:
        n_extra = 0
        while time.time() - t_end < 0.6:
            for _ in range(200):
                steps[n_extra % R](q)
                n_extra += 1
            torch.cuda.synchronize()
        t_load_end = time.time()
    elapsed_ms = reduce_max(elapsed_ms, world, dev)
    us_per_step = elapsed_ms * 1e3 / args.steps
    value = whole_job_us_per_step(elapsed_ms, args.steps, world)

    # per-kernel durations: the same step with an event after each kernel
    names = steps[0].kernel_names()
    nk = len(names)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(4)]
    for es in evs:
        for e in es:
            e.record(stream)
    torch.cuda.synchronize()
    per = [[] for _ in range(nk)]
    nprof = max(8, min(args.steps, 400))
    for i in range(nprof):
        es = evs[i % 4]
        steps[i % R].profiled(q, es)
        if i % 4 == 3 or i == nprof - 1:
            torch.cuda.synchronize()
            for j in range(i - (i % 4), i + 1):
                ej = evs[j % 4]
                for k in range(nk):
                    per[k].append(ej[k].elapsed_time(ej[k + 1]) * 1e3)
    kernel_us = {names[k]: statistics.mean(per[k]) for k in range(nk)}

    # end to end through the public API with host buffers: every step takes q
    # from pinned host memory and returns the attention output to pinned host
    # memory (DecodeStep.run_host: the two copies are kernels of the step's
    # launch chain)
    q_host = q.cpu().pin_memory()
    out_host = torch.empty(steps[0].out.shape, dtype=steps[0].out.dtype).pin_memory()
    for i in range(max(3, args.warmup)):
        steps[i % R].run_host(q_host, out_host)
    barrier()
    e0.record(stream)
    for i in range(args.steps):
        steps[i % R].run_host(q_host, out_host)
    e1.record(stream)
    e1.synchronize()
    barrier()
    e2e_us = whole_job_us_per_step(reduce_max(e0.elapsed_time(e1), world, dev), args.steps, world)

    if sampler:
        sampler.stop()
    # exact attention mass each query head's selection keeps, through the
    # library alone: exp(lse over the selection - lse over every candidate),
    # the second lse from the same step run with p = 1 (outside the timed region)
    steps[0](q)
    lse_p = steps[0].lse.double().clone()
    full = make_step(steps[0].kv, steps[0].keys, getattr(steps[0], "meta", None), 1.0)
    full(q)
    torch.cuda.synchronize()
    retained = torch.exp(lse_p - full.lse.double()).flatten().cpu()
    del full
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    if label:
        kb, cand_tokens, kept = label_algorithmic_bytes(w, steps[0], args.key_bits)
    else:
        kb, cand_tokens, kept = algorithmic_bytes(w, steps[0], args.key_bits)
    toks_total = int(w.seq_lens.to(torch.int64).sum()) * w.Hk
    pages_total = int(((w.seq_lens.to(torch.int64) + 15) // 16).sum()) * w.Hk
    total_b = sum(kb.values())
    peak, peak_kind = hbm_peak()
    dom = max(kb, key=lambda k: kernel_us.get(k, 0.0) if kb[k] > 0 else -1)
    dom_us = kernel_us[dom]
    achieved = kb[dom] / (dom_us * 1e-6) / 1e9
    traffic = None
    try:   # ncu DRAM bytes per launch, valid only for the sources they were taken on
        tr = json.load(open(TRAFFIC_PATH))
        sect = "kernels" if args.key_bits == 4 else f"kernels_key_bits_{args.key_bits}"
        if label:
            sect = "kernels_label_selector"
        if tr.get("src_hash") == src_hash() and tr.get("workload") == w.name:
            traffic = tr.get(sect, {}).get(dom, {}).get("dram_bytes_per_launch")
    except Exception:
        pass
    clocks = sampler.summary(t_start - 0.05, t_load_end + 0.05) if sampler else None

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        w_cpu = w.to("cpu")
        cpu_us, n_units, tot_units, cores = cpu_step_sample(
            w_cpu, args.cpu_seconds, key_bits=args.key_bits,
            label_channels=W.label_channels(w, r=LABEL_R) if label else None)
        per_unit = cpu_us / tot_units
        all_us, n_all, _, threads = cpu_step_all_cores(
            w_cpu, per_unit, args.cpu_seconds, key_bits=args.key_bits,
            label_channels=W.label_channels(w, r=LABEL_R) if label else None)
        cpu = {"value": cpu_us, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n_units} of {tot_units} (sequence, KV head) units of the same "
                         f"workload, single-threaded numpy, scaled to the full step",
               "all_cores": {"value": all_us, "unit": UNIT, "cores": threads,
                             "nproc": os.cpu_count(),
                             "sample": f"{n_all} of {tot_units} units run concurrently by "
                                       f"{threads} worker threads, wall time scaled to the "
                                       f"full step"}}

    sets = kept.numel()
    cands_per_set = cand_tokens / max(1, w.B * w.Hk)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": value / 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, args.key_bits, args.selector),
        "l2": l2_policy(R, copy_bytes),
        "hbm_gbs": total_b / (us_per_step * 1e-6) / 1e9,
        "hbm_frac_of_measured": total_b / (us_per_step * 1e-6) / 1e9 / peak,
        "bytes_per_step": total_b,
        "kv_tokens_scanned_per_s": cand_tokens / (us_per_step * 1e-6),
        "kept_tokens": {"mean": float(kept.double().mean()), "min": int(kept.min()),
                        "max": int(kept.max()), "sets": sets,
                        "candidates_per_set": cands_per_set},
        "pruned_frac": 1.0 - float(kept.double().mean()) / max(1.0, cands_per_set),
        "retained_mass": {"p": w.p, "mean": float(retained.mean()),
                          "std": float(retained.std()) if retained.numel() > 1 else 0.0,
                          "min": float(retained.min()), "max": float(retained.max()),
                          "heads": retained.numel()},
        "step_us": us_per_step,
        "kernel_us_serialised": kernel_us,
        "kernel_us_note": "each kernel bracketed by events with no overlap between kernels "
                          "(programmatic dependent launch off); step_us is the overlapped step",
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "algorithmic_bytes": kb[dom]},
        "cache_build": {
            "quantize_keys_gbs": toks_total * (256 + 80) / (build_ms[0] * 1e-3) / 1e9,
            "page_meta_gbs": (toks_total * 256 + pages_total * 512) / (build_ms[1] * 1e-3) / 1e9,
            "append_keys_us": append_us},
        "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": q.numel() * q.element_size(),
                "d2h_bytes_per_step": steps[0].out.numel() * steps[0].out.element_size()},
        "gpu_launches": args.steps * (LabelDecodeStep.LAUNCHES if label else nk),
        "e2e_gpu_launches": args.steps * ((LabelDecodeStep.LAUNCHES if label else nk) + 2),
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if world == 1 and not args.no_per_config and args.selector == "quest":
        del steps
        torch.cuda.empty_cache()
        line["per_config"] = per_config_times(args.config, dev, args.key_bits,
                                              max(20, min(args.steps, 200)), args.warmup)
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
