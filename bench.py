#!/usr/bin/env python
"""Benchmark of the QUOKA prefill-chunk step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path -- (a) mean query and SQ, (b) top-NQ
queries, (c) normalise + group mean, (d) cosine score + max, (e) top-BSA keys,
(f) gather of the selected rows, (g) sparse GQA attention -- over one chunk
of synthetic input resident in HBM. The default workload is the Qwen3-4B-shaped layer at
T = 32768 prior keys (b=1, nq=32, nkv=8, d=128, BCP=512, NQ=32, BSA=4096).

Timing: W warm-up steps, then exactly K timed steps bracketed by a barrier and
a device synchronisation; before every timed step the L2 is flushed by writing
a 256 MiB buffer (outside the timed events); each step is timed with CUDA
events on the launching stream, placed only at the step's two ends; the step
is quoka_prefill_chunk (the whole path in one C-ABI call, its kernels
overlapping at their edges through programmatic dependent launch, as they
do for a user); under torchrun the maximum over ranks is reported. A second
pass of K steps runs the same kernels through the three part calls
(quoka_select | quoka_gather_kv | quoka_sparse_gqa_attn_gathered) with an
event at every boundary, for the breakdown (ms_select, ms_gather,
ms_attention) and the rooflines. For a single-chunk workload, `decode`
reports a decode step (BCP = 1, NQ = 1) on the same cache: the whole step
through quoka_prefill_chunk (which takes the short-chunk attention) and, on
its selection, that attention alone against the prefill attention kernels.
Rank 0 prints one JSON line.

--impl reference times the CPU oracle (numpy float64) on the host cores
instead, on a bounded per-step sample of the same workload (one KV head's
group per step, 1/nkv of the work), and reports the same metric.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "prefill chunk-tokens/sec at T=32K (keys-scored/sec, % HBM and tensor-pipe peak alongside)"
UNIT = "chunk-tokens/s"
FLUSH_BYTES = 256 << 20
def kernels_per_chunk(T, bsa_eff):
    """Our kernel launches in one chunk's step: query select, group mean,
    scoring (T > 0), top-k and gather (BSA_eff > 0), attention."""
    return 2 + (1 if T > 0 else 0) + (2 if bsa_eff > 0 else 0) + 1


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _profiled_traffic(profile_name: str, *source_rel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's
    sources (hashed in the given order) still match the value recorded with
    the counters (else None: the counters describe an older kernel)."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", profile_name)
    srcs = [os.path.join(ROOT, r) for r in source_rel]
    if not (os.path.exists(prof) and all(os.path.exists(x) for x in srcs)):
        return None
    want, traffic = None, None
    with open(prof) as f:
        for line in f:
            line = line.strip()
            if line.startswith("traffic_bytes_per_launch:"):
                traffic = int(line.split(":")[1])
            elif line.startswith("source_sha256_16:"):
                want = line.split(":")[1].strip()
    m = hashlib.sha256()
    for x in srcs:
        with open(x, "rb") as f:
            m.update(f.read())
    have = m.hexdigest()[:16]
    return traffic if (want is not None and have == want) else None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"quoka_clocks_{os.getpid()}_{gpu_index}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- workload

def max_over_ranks(values, world: int, device="cpu"):
    """Per-rank timings -> their maximum over the ranks of the default
    process group, on every rank (the values themselves at world 1)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_throughput(world: int, units_per_rank: float, ms_step: float) -> float:
    """Whole-job units per second: every rank processes units_per_rank per
    step (weak scaling, replicas), the step taking ms_step (the slowest
    rank's time)."""
    return world * units_per_rank / (ms_step / 1e3)


def make_inputs(name: str, rank: int):
    from sparse_kv_selection_quoka_b200 import inputs
    w = inputs._lookup(name)
    if name.startswith("sweep"):
        return w, inputs.make_sweep(seed=w.seed + 7919 * rank)
    x = inputs.make_chunk(w.b, w.nq, w.nkv, w.d, w.T, w.BCP, w.NQ, w.BSA, dtype=w.dtype,
                          structure=w.structure, seed=w.seed + 7919 * rank)
    return w, x


def attn_flops(b, nq, d, BCP, bsa_eff):
    return 4.0 * d * b * nq * (BCP * bsa_eff + BCP * (BCP + 1) / 2.0)


def select_bytes(b, nq, nkv, d, T, BCP, bsa_eff, es):
    return b * nkv * T * d * es + b * nq * BCP * d * es + b * nkv * bsa_eff * 4


def gather_bytes(b, nkv, d, bsa_eff, es):
    """Step (f): the selected K and V rows read once and written once, and
    the index list read."""
    return b * nkv * bsa_eff * (4 * d * es + 4)


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import sparse_kv_selection_quoka_b200 as q
    from sparse_kv_selection_quoka_b200 import inputs

    q.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w, x = make_inputs(args.workload, rank)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    es = 2 if w.dtype == "bf16" else 4
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(tdt).to(dev)

    sweep = w.name.startswith("sweep")
    if sweep:
        Qs, Ks, Vs = (to_dev(a) for a in (x.Qs, x.Ks, x.Vs))
        L = x.BCP
        chunks = []
        for c in range(x.n_chunks):
            T = c * L
            bsa = x.budget(T)
            views = (Qs[:, :, T:T + L], Ks[:, :, :T], Vs[:, :, :T], Ks[:, :, T:T + L], Vs[:, :, T:T + L])
            ws = q.workspace_for(views[0], views[1], x.NQ, bsa)
            O = torch.empty((w.b, w.nq, L, w.d), dtype=tdt, device=dev)
            kv_idx = torch.empty((w.b, w.nkv, min(bsa, T)), dtype=torch.int32, device=dev)
            kv_count = torch.empty((w.b, w.nkv), dtype=torch.int32, device=dev)
            sel_kv = tuple(torch.empty((w.b, w.nkv, min(bsa, T), w.d), dtype=tdt, device=dev) for _ in range(2))
            chunks.append((views, bsa, ws, O, kv_idx, kv_count, T, sel_kv))
    else:
        Q, K, V, Kc, Vc = (to_dev(a) for a in (x.Q, x.K, x.V, x.Kc, x.Vc))
        bsa_eff = min(w.BSA, w.T)
        ws = q.workspace_for(Q, K, w.NQ, w.BSA)
        O = torch.empty((w.b, w.nq, w.BCP, w.d), dtype=tdt, device=dev)
        kv_idx = torch.empty((w.b, w.nkv, bsa_eff), dtype=torch.int32, device=dev)
        kv_count = torch.empty((w.b, w.nkv), dtype=torch.int32, device=dev)
        sel_kv = tuple(torch.empty((w.b, w.nkv, bsa_eff, w.d), dtype=tdt, device=dev) for _ in range(2))
        chunks = [((Q, K, V, Kc, Vc), w.BSA, ws, O, kv_idx, kv_count, w.T, sel_kv)]

    def one_chunk(ch, evs=None):
        """Steps (a)-(e) | (f) | (g) through the public calls; with `evs`
        (three events) each boundary is recorded, so every part is timed on
        its own: quoka_sparse_gqa_attn with a full workspace runs exactly
        the gather and attention kernels below."""
        (Qv, Kv, Vv, Kcv, Vcv), bsa, wsb, Ob, idx, cnt, _, (Ks, Vs) = ch
        q.quoka_select(Qv, Kv, w.NQ, bsa, kv_idx=idx, kv_count=cnt, ws=wsb, stream=stream)
        if evs is not None:
            evs[0].record(stream)
        q.quoka_gather_kv(Kv, Vv, idx, cnt, Ksel=Ks, Vsel=Vs, ws=wsb, stream=stream)
        if evs is not None:
            evs[1].record(stream)
        q.quoka_sparse_gqa_attn_gathered(Qv, Ks, Vs, cnt, Kcv, Vcv, O=Ob, ws=wsb, stream=stream)

    def whole_chunk(ch):
        """Steps (a)-(g) as one call, quoka_prefill_chunk: the same kernels as
        one_chunk, chained on the stream with no event in between."""
        (Qv, Kv, Vv, Kcv, Vcv), bsa, wsb, Ob, idx, _, _, _ = ch
        q.quoka_prefill_chunk(Qv, Kv, Vv, Kcv, Vcv, w.NQ, bsa, O=Ob, kv_idx=idx,
                              ws=wsb, stream=stream)

    for _ in range(args.warmup):
        for ch in chunks:
            one_chunk(ch)
            whole_chunk(ch)
    torch.cuda.synchronize()
    status = q.quoka_get_device_status(chunks[-1][2])
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    # a short untimed burst so the sampler sees the GPU under load
    for _ in range(max(3, args.warmup)):
        for ch in chunks:
            one_chunk(ch)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    n_ev = len(chunks)
    # The step: quoka_prefill_chunk per chunk with events only at the step's
    # two ends, so the kernels overlap at their edges as they do for a user
    # (programmatic dependent launch within the call).
    t_step = 0.0
    per_chunk = [0.0] * n_ev
    step_evs = []
    for _ in range(args.steps):
        flush.fill_(1)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        for ch in chunks:
            whole_chunk(ch)
        e[1].record(stream)
        step_evs.append(e)
    torch.cuda.synchronize()
    for e in step_evs:
        t_step += e[0].elapsed_time(e[1])
    # The parts, timed in a second pass with an event at every boundary
    # (which serialises the parts): select (a)-(e), gather (f), attention (g).
    if world > 1:
        torch.distributed.barrier()
    t_sel, t_gather, t_attn = 0.0, 0.0, 0.0
    evs = []
    for _ in range(args.steps):
        flush.fill_(1)
        step_evs = []
        for ch in chunks:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            e[0].record(stream)
            one_chunk(ch, evs=e[1:4])
            e[4].record(stream)
            step_evs.append(e)
        evs.append(step_evs)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    for step_evs in evs:
        for c, e in enumerate(step_evs):
            a, g, bms = e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[4])
            t_sel += a
            t_gather += g
            t_attn += bms
            per_chunk[c] += a + g + bms
    clocks = sampler.stop()

    K_ = args.steps
    ms_step, ms_sel, ms_gather, ms_attn = max_over_ranks(
        [t_step / K_, t_sel / K_, t_gather / K_, t_attn / K_], world, dev)

    tokens_per_step = w.b * (w.T if sweep else w.BCP)
    if sweep:
        tokens_per_step = w.b * x.n_chunks * x.BCP
    value = job_throughput(world, tokens_per_step, ms_step)

    hbm, tf_burst, tf_sus, peak_src = _peaks()
    if sweep:
        flops = sum(attn_flops(w.b, w.nq, w.d, x.BCP, min(ch[1], ch[6])) for ch in chunks)
        sbytes = sum(select_bytes(w.b, w.nq, w.nkv, w.d, ch[6], x.BCP, min(ch[1], ch[6]), es) for ch in chunks)
        gbytes = sum(gather_bytes(w.b, w.nkv, w.d, min(ch[1], ch[6]), es) for ch in chunks)
        keys = sum(w.b * w.nkv * ch[6] for ch in chunks)
    else:
        flops = attn_flops(w.b, w.nq, w.d, w.BCP, min(w.BSA, w.T))
        sbytes = select_bytes(w.b, w.nq, w.nkv, w.d, w.T, w.BCP, min(w.BSA, w.T), es)
        gbytes = gather_bytes(w.b, w.nkv, w.d, min(w.BSA, w.T), es)
        keys = w.b * w.nkv * w.T
    attn_tflops = flops / (ms_attn / 1e3) / 1e12
    sel_gbs = sbytes / (ms_sel / 1e3) / 1e9
    out = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": K_,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded; shapes and value structure of the workload, see DESIGN.md)",
        "config": {"workload": w.name, "b": w.b, "nq": w.nq, "nkv": w.nkv, "d": w.d,
                   "T": w.T, "BCP": w.BCP, "NQ": w.NQ, "BSA": w.BSA, "parallelism": f"replicas{world}",
                   "l2": "flushed before every timed step (256 MiB write, untimed)"},
        "keys_scored_per_s": world * keys / (ms_sel / 1e3),
        "keys_scored_per_s_query_heads": world * keys * (w.nq // w.nkv) / (ms_sel / 1e3),
        "ms_select": ms_sel,
        "ms_gather": ms_gather,
        "ms_attention": ms_attn,
        "roofline": {"kernel": "sparse GQA attention (tcgen05)" if w.dtype == "bf16" else "sparse GQA attention (fp32 CUDA cores)",
                     "bound": "tensor", "achieved": attn_tflops, "peak": tf_burst,
                     "unit": "TFLOP/s", "frac": attn_tflops / tf_burst,
                     "traffic": (_profiled_traffic("attn_tma_qwen3-4b_T32k.md",
                                                   "sparse_kv_selection_quoka_b200/csrc/attn_tma.cu",
                                                   "sparse_kv_selection_quoka_b200/csrc/attn_common.cuh")
                                 if w.name == "qwen3-4b_T32k" and w.dtype == "bf16" else None),
                     "peak_kind": f"bf16 dense, burst, {peak_src}",
                     "algorithmic_flops_per_launch": flops / max(1, len(chunks))},
        "roofline_select": {"steps": "(a)-(e)", "bound": "hbm", "achieved": sel_gbs, "peak": hbm,
                            "unit": "GB/s", "frac": sel_gbs / hbm, "frac_of_8TBs": sel_gbs / 8000.0,
                            "algorithmic_bytes_per_step": sbytes},
        "roofline_gather": {"steps": "(f)", "bound": "hbm", "achieved": gbytes / (ms_gather / 1e3) / 1e9,
                            "peak": hbm, "unit": "GB/s", "frac": gbytes / (ms_gather / 1e3) / 1e9 / hbm,
                            "algorithmic_bytes_per_step": gbytes},
        "clocks": clocks,
        "gpu_launches": sum(kernels_per_chunk(ch[6], min(ch[1], ch[6])) for ch in chunks) * K_,
    }
    if sweep:
        out["per_chunk_ms"] = [p / K_ for p in per_chunk]
    else:
        out["decode"] = measure_decode(q, w, dev, stream, flush, Q, K, V, Kc, Vc, min(K_, 50))
    if not args.no_e2e:
        out["e2e"] = run_e2e(args, w, x, chunks, q, dev, stream, tokens_per_step, world, sweep)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, x, sweep)
    return out


def measure_decode(q, w, dev, stream, flush, Q, K, V, Kc, Vc, steps):
    """A decode step on the workload's cache: BCP = 1 (the chunk's first
    token), NQ = 1, the same T and BSA, through quoka_prefill_chunk (which
    takes the short-chunk attention), L2 flushed before every timed call;
    then, on that step's selection, the short-chunk attention alone
    (quoka_decode_attn) and the prefill attention kernels on the same
    selection (quoka_sparse_gqa_attn: gather, then 128-row tiles)."""
    Q1, Kc1, Vc1 = (a[:, :, :1].contiguous() for a in (Q, Kc, Vc))
    bsa_eff = min(w.BSA, w.T)
    ws = q.workspace_for(Q1, K, 1, w.BSA)
    O1 = torch.empty_like(Q1)
    idx = torch.empty((w.b, w.nkv, bsa_eff), dtype=torch.int32, device=dev)
    cnt = torch.full((w.b, w.nkv), bsa_eff, dtype=torch.int32, device=dev)
    wsa = torch.empty(max(256, q.quoka_attn_workspace_size(w.b, w.nkv, w.d, bsa_eff, Q1.dtype)),
                      dtype=torch.uint8, device=dev)
    wsd = torch.empty(q.quoka_decode_workspace_size(w.b, w.nq, w.nkv, w.d, 1, bsa_eff, Q1.dtype),
                      dtype=torch.uint8, device=dev)
    calls = {
        "ms_step": lambda: q.quoka_prefill_chunk(Q1, K, V, Kc1, Vc1, 1, w.BSA, O=O1, kv_idx=idx, ws=ws,
                                                 stream=stream),
        "ms_attention": lambda: q.quoka_decode_attn(Q1, K, V, idx, cnt, Kc1, Vc1, O=O1, ws=wsd, stream=stream),
        "ms_attention_prefill_kernels": lambda: q.quoka_sparse_gqa_attn(Q1, K, V, idx, cnt, Kc1, Vc1, O=O1,
                                                                        ws=wsa, stream=stream),
    }
    out = {"BCP": 1, "NQ": 1, "steps": steps}
    for name, f in calls.items():
        for _ in range(3):
            f()
        evs = []
        for _ in range(steps):
            flush.fill_(1)
            # a short device-side wait after the flush: these calls take less
            # GPU time than their host-side argument marshalling, and the
            # wait lets the host enqueue the whole call before the timed
            # region starts, so the events see the device's time only
            torch.cuda._sleep(200000)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            e[0].record(stream)
            f()
            e[1].record(stream)
            evs.append(e)
        torch.cuda.synchronize()
        out[name] = sum(a.elapsed_time(b) for a, b in evs) / steps
    for wsx in (ws, wsd):
        if q.quoka_get_device_status(wsx) != 0:
            raise RuntimeError("device status after the decode measurement")
    es = 2 if Q1.dtype == torch.bfloat16 else 4
    nbytes = (2 * w.b * w.nkv * bsa_eff * w.d + 2 * w.b * w.nq * w.d + 2 * w.b * w.nkv * w.d) * es
    gbs = nbytes / (out["ms_attention"] / 1e3) / 1e9
    hbm = _peaks()[0]
    out["attention_bytes"] = nbytes
    out["attention_gbs"] = gbs
    out["attention_frac_hbm"] = gbs / hbm
    return out


def run_e2e(args, w, x, chunks, q, dev, stream, tokens_per_step, world, sweep):
    """The same metric through the public whole-step call with host buffers:
    every step copies that step's inputs from pinned host memory to the
    device, runs quoka_prefill_chunk, and copies the output back."""
    tdt = chunks[0][3].dtype
    hosts, devs, outs = [], [], []
    h2d = d2h = 0
    if sweep:
        # the whole sequence's inputs are uploaded once per step
        host = [torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(tdt).pin_memory()
                for a in (x.Qs, x.Ks, x.Vs)]
        dbuf = [torch.empty_like(h, device=dev) for h in host]
        h2d = sum(h.numel() * h.element_size() for h in host)
    else:
        host = [torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(tdt).pin_memory()
                for a in (x.Q, x.K, x.V, x.Kc, x.Vc)]
        dbuf = [torch.empty_like(h, device=dev) for h in host]
        h2d = sum(h.numel() * h.element_size() for h in host)
    O_host = [torch.empty(ch[3].shape, dtype=tdt).pin_memory() for ch in chunks]
    d2h = sum(o.numel() * o.element_size() for o in O_host)

    def step():
        for h, d_ in zip(host, dbuf):
            d_.copy_(h, non_blocking=True)
        if sweep:
            Qs, Ks, Vs = dbuf
            for c, ch in enumerate(chunks):
                T = ch[6]
                L = x.BCP
                q.quoka_prefill_chunk(Qs[:, :, T:T + L], Ks[:, :, :T], Vs[:, :, :T], Ks[:, :, T:T + L],
                                      Vs[:, :, T:T + L], w.NQ, ch[1], O=ch[3], ws=ch[2], stream=stream)
                O_host[c].copy_(ch[3], non_blocking=True)
        else:
            Q, K, V, Kc, Vc = dbuf
            ch = chunks[0]
            q.quoka_prefill_chunk(Q, K, V, Kc, Vc, w.NQ, w.BSA, O=ch[3], ws=ch[2], stream=stream)
            O_host[0].copy_(ch[3], non_blocking=True)

    for _ in range(max(1, args.warmup // 2)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(1, min(args.steps, 50))
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = max_over_ranks([e0.elapsed_time(e1) / n], world, dev)[0]
    return {"value": job_throughput(world, tokens_per_step, ms), "unit": UNIT, "ms_per_step": ms,
            "steps": n, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "call": "quoka_prefill_chunk (C ABI) with pinned-host inputs copied in and O copied out every step"}


# ---------------------------------------------------------------- CPU oracle

def _blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"), default=1)
    except Exception:
        return os.cpu_count() or 1


def _oracle_head_step(x, j):
    """Steps (a)-(g) of the oracle for KV head j and its G query heads only
    (1/nkv of the workload; heads are independent through every step)."""
    from oracle import quoka_oracle as orc
    G = x.Q.shape[1] // x.K.shape[1]
    Qj = x.Q[:, j * G:(j + 1) * G]
    sl = slice(j, j + 1)
    return orc.prefill_chunk(Qj, x.K[:, sl], x.V[:, sl], x.Kc[:, sl], x.Vc[:, sl], x.NQ, x.BSA)


def cpu_baseline(w, x, sweep, budget_s=12.0):
    """The oracle as it stands on the host cores, on a bounded sample of the
    workload: whole KV-head groups (1/nkv of a step each) until ~budget_s."""
    if sweep:
        x = x.chunk(x.n_chunks // 2)
    t0 = time.perf_counter()
    n = 0
    while True:
        _oracle_head_step(x, n % w.nkv)
        n += 1
        if time.perf_counter() - t0 >= budget_s or n >= 4 * w.nkv:
            break
    dt = time.perf_counter() - t0
    tokens = x.Q.shape[0] * x.Q.shape[2] * n / w.nkv
    return {"value": tokens / dt, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{n} KV-head groups ({n}/{w.nkv} of a step) of workload {w.name}"
                      + (" (chunk 32 of the sweep)" if sweep else "") + f", {dt:.1f} s",
            "host_cpu_count": os.cpu_count()}


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: each step is one KV-head group of
    the workload (1/nkv of the work), on the host cores."""
    if rank != 0:
        return None
    from sparse_kv_selection_quoka_b200 import inputs
    w, x = make_inputs(args.workload, 0)
    if w.name.startswith("sweep"):
        x = x.chunk(x.n_chunks // 2)
    for s in range(args.warmup):
        _oracle_head_step(x, s % w.nkv)
    t0 = time.perf_counter()
    for s in range(args.steps):
        _oracle_head_step(x, s % w.nkv)
    dt = time.perf_counter() - t0
    ms_sample = dt / args.steps * 1e3
    ms_step = ms_sample * w.nkv
    tokens = x.Q.shape[0] * x.Q.shape[2]
    value = tokens / (ms_step / 1e3)
    cores = _blas_threads()
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": w.name, "b": w.b, "nq": w.nq, "nkv": w.nkv, "d": w.d, "T": w.T,
                       "BCP": w.BCP, "NQ": w.NQ, "BSA": w.BSA, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"one KV-head group (1/{w.nkv} of the step) per timed step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="qwen3-4b_T32k")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out))
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(out))
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
