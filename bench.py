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
With the default workload, `per_workload` repeats the measurement (without
the e2e, decode and oracle legs) on the Llama-shaped layer at T = 8192, the
chunked-prefill sweep (b = 8, 64 chunks of 256, with its per-chunk time
curve) and the 128K-key layer. Rank 0 prints one JSON line.

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
# device-side wait (clock cycles, ~100 µs) enqueued after each flush, outside
# the timed events: the host's argument marshalling for a call can take
# longer than the call's device time, and the wait lets the host enqueue the
# whole timed region before the device reaches it
HOST_LEAD_CYCLES = 200000
DEFAULT_WORKLOAD = "qwen3-4b_T32k"
# measured beside the default workload in every default run
OTHER_WORKLOADS = ("llama3.2-3b_T8k", "sweep_b8_S16k", "long_T128k_G8")


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

def kernels_per_chunk(w, T, bsa_eff):
    """Our kernel launches in one quoka_prefill_chunk call on a bf16, d = 128
    workload: query select + group mean (one fused kernel for BCP <= 512,
    NQ <= 32, G <= 8 or for one query, else two), the scoring (T > 0), the
    top-k and the gather (BSA_eff > 0), and the attention (a short chunk's
    takes two; so do split key ranges, with their merge)."""
    G = w.nq // w.nkv
    fused = w.dtype == "bf16" and w.d == 128 and ((w.BCP <= 512 and w.NQ <= 32 and G <= 8)
                                                   or (w.BCP == 1 and G <= 32))
    short = G * w.BCP <= 64
    n = (1 if fused else 2) + (1 if T > 0 else 0)
    if bsa_eff > 0:
        n += 1 if short else 2
        # the merge of the attention's split key ranges (few query tiles)
        tiles = w.b * w.nq * ((w.BCP + 127) // 128)
        if not short and w.dtype == "bf16" and w.d == 128 and 2 * tiles <= 148:
            if min(4, 148 // tiles, ((bsa_eff + 127) // 128 + 1) // 2) >= 2:
                n += 1
    return n + (2 if short else 1)


class WorkloadRun:
    """Device buffers of one workload on this rank: a list of chunks (one,
    or the sweep's 64), each with its strided input views, its workspace and
    its outputs, all resident in HBM before any timing."""

    def __init__(self, q, name, rank, dev):
        self.w, self.x = make_inputs(name, rank)
        w, x = self.w, self.x
        self.sweep = w.name.startswith("sweep")
        self.tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.es = 2 if w.dtype == "bf16" else 4
        tdt = self.tdt

        def to_dev(a):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(tdt).to(dev)

        self.chunks = []
        if self.sweep:
            self.Qs, self.Ks, self.Vs = (to_dev(a) for a in (x.Qs, x.Ks, x.Vs))
            L = x.BCP
            for c in range(x.n_chunks):
                T = c * L
                views = (self.Qs[:, :, T:T + L], self.Ks[:, :, :T], self.Vs[:, :, :T],
                         self.Ks[:, :, T:T + L], self.Vs[:, :, T:T + L])
                self.chunks.append(self._chunk(q, views, x.budget(T), T, L, dev))
            self.BCP = L
        else:
            self.dev_inputs = [to_dev(a) for a in (x.Q, x.K, x.V, x.Kc, x.Vc)]
            self.chunks.append(self._chunk(q, tuple(self.dev_inputs), w.BSA, w.T, w.BCP, dev))
            self.BCP = w.BCP

    def _chunk(self, q, views, bsa, T, L, dev):
        w = self.w
        be = min(bsa, T)
        return {
            "views": views, "bsa": bsa, "T": T, "bsa_eff": be,
            "ws": q.workspace_for(views[0], views[1], w.NQ, bsa),
            "O": torch.empty((w.b, w.nq, L, w.d), dtype=self.tdt, device=dev),
            "kv_idx": torch.empty((w.b, w.nkv, be), dtype=torch.int32, device=dev),
            "kv_count": torch.empty((w.b, w.nkv), dtype=torch.int32, device=dev),
            "sel": tuple(torch.empty((w.b, w.nkv, be, w.d), dtype=self.tdt, device=dev) for _ in range(2)),
        }

    # the work of one step, in both forms
    def whole(self, q, ch, stream):
        """Steps (a)-(g) as one call, quoka_prefill_chunk."""
        Qv, Kv, Vv, Kcv, Vcv = ch["views"]
        q.quoka_prefill_chunk(Qv, Kv, Vv, Kcv, Vcv, self.w.NQ, ch["bsa"], O=ch["O"], kv_idx=ch["kv_idx"],
                              ws=ch["ws"], stream=stream)

    def parts(self, q, ch, stream, evs=None):
        """Steps (a)-(e) | (f) | (g) through the three part calls; with `evs`
        (two events) each boundary is recorded, so every part is timed on
        its own."""
        Qv, Kv, Vv, Kcv, Vcv = ch["views"]
        Ks, Vs = ch["sel"]
        q.quoka_select(Qv, Kv, self.w.NQ, ch["bsa"], kv_idx=ch["kv_idx"], kv_count=ch["kv_count"], ws=ch["ws"],
                       stream=stream)
        if evs is not None:
            evs[0].record(stream)
        q.quoka_gather_kv(Kv, Vv, ch["kv_idx"], ch["kv_count"], Ksel=Ks, Vsel=Vs, ws=ch["ws"], stream=stream)
        if evs is not None:
            evs[1].record(stream)
        q.quoka_sparse_gqa_attn_gathered(Qv, Ks, Vs, ch["kv_count"], Kcv, Vcv, O=ch["O"], ws=ch["ws"],
                                         stream=stream)

    # algorithmic work of one step
    def flops(self):
        w = self.w
        return sum(attn_flops(w.b, w.nq, w.d, self.BCP, ch["bsa_eff"]) for ch in self.chunks)

    def select_bytes(self):
        w = self.w
        return sum(select_bytes(w.b, w.nq, w.nkv, w.d, ch["T"], self.BCP, ch["bsa_eff"], self.es)
                   for ch in self.chunks)

    def gather_bytes(self):
        w = self.w
        return sum(gather_bytes(w.b, w.nkv, w.d, ch["bsa_eff"], self.es) for ch in self.chunks)

    def keys(self):
        return sum(self.w.b * self.w.nkv * ch["T"] for ch in self.chunks)

    def tokens(self):
        return self.w.b * self.BCP * len(self.chunks)

    def launches(self):
        return sum(kernels_per_chunk(self.w, ch["T"], ch["bsa_eff"]) for ch in self.chunks)

    def status_ok(self, q):
        return all(q.quoka_get_device_status(ch["ws"]) == 0 for ch in self.chunks)


def time_run(q, run, steps, warmup, flush, stream, world, dev, sampler=None):
    """W warm-up steps, then K timed steps of quoka_prefill_chunk (events at
    the step's two ends only, L2 flushed before each step, outside the
    events), then K steps of the part calls with an event at every
    boundary. Timings are maxima over the ranks."""
    for _ in range(warmup):
        for ch in run.chunks:
            run.parts(q, ch, stream)
            run.whole(q, ch, stream)
    torch.cuda.synchronize()
    if not run.status_ok(q):
        raise RuntimeError(f"device status after the warm-up of {run.w.name}")
    if sampler is not None:
        sampler.start()
        time.sleep(0.3)
        # a short untimed burst so the sampler sees the GPU under load
        for _ in range(max(3, warmup)):
            for ch in run.chunks:
                run.whole(q, ch, stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    step_evs = []
    for _ in range(steps):
        flush.fill_(1)
        # a device-side wait after the flush (outside the events) keeps the
        # host's enqueueing ahead of the device, so that no host-side gap
        # falls inside a timed region
        torch.cuda._sleep(HOST_LEAD_CYCLES * len(run.chunks))
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        for ch in run.chunks:
            run.whole(q, ch, stream)
        e[1].record(stream)
        step_evs.append(e)
    torch.cuda.synchronize()
    t_step = sum(a.elapsed_time(b) for a, b in step_evs)
    if world > 1:
        torch.distributed.barrier()
    n = len(run.chunks)
    per_chunk = [0.0] * n
    t_sel = t_gather = t_attn = 0.0
    evs = []
    for _ in range(steps):
        flush.fill_(1)
        one = []
        for ch in run.chunks:
            torch.cuda._sleep(HOST_LEAD_CYCLES)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            e[0].record(stream)
            run.parts(q, ch, stream, evs=e[1:3])
            e[3].record(stream)
            one.append(e)
        evs.append(one)
    torch.cuda.synchronize()
    for one in evs:
        for c, e in enumerate(one):
            a, g, at = e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])
            t_sel += a
            t_gather += g
            t_attn += at
            per_chunk[c] += a + g + at
    clocks = sampler.stop() if sampler is not None else None
    if world > 1:
        torch.distributed.barrier()
    if not run.status_ok(q):
        raise RuntimeError(f"device status after timing {run.w.name}")
    vals = max_over_ranks([t_step / steps, t_sel / steps, t_gather / steps, t_attn / steps]
                          + [p / steps for p in per_chunk], world, dev)
    return {"ms_step": vals[0], "ms_select": vals[1], "ms_gather": vals[2], "ms_attention": vals[3],
            "per_chunk_ms": vals[4:], "clocks": clocks}


def rooflines(run, t, world):
    """Throughput and roofline figures of a timed run (see time_run)."""
    hbm, tf_burst, _, peak_src = _peaks()
    w = run.w
    flops, sbytes, gbytes = run.flops(), run.select_bytes(), run.gather_bytes()
    attn_tflops = flops / (t["ms_attention"] / 1e3) / 1e12
    sel_gbs = sbytes / (t["ms_select"] / 1e3) / 1e9
    g_gbs = gbytes / (t["ms_gather"] / 1e3) / 1e9
    return {
        "value": job_throughput(world, run.tokens(), t["ms_step"]),
        "keys_scored_per_s": world * run.keys() / (t["ms_select"] / 1e3),
        "keys_scored_per_s_query_heads": world * run.keys() * (w.nq // w.nkv) / (t["ms_select"] / 1e3),
        "roofline": {"kernel": ("sparse GQA attention (tcgen05)" if w.dtype == "bf16"
                                else "sparse GQA attention (fp32 CUDA cores)"),
                     "bound": "tensor", "achieved": attn_tflops, "peak": tf_burst, "unit": "TFLOP/s",
                     "frac": attn_tflops / tf_burst, "traffic": None,
                     "peak_kind": f"bf16 dense, burst, {peak_src}",
                     "algorithmic_flops_per_launch": flops / max(1, len(run.chunks))},
        "roofline_select": {"steps": "(a)-(e)", "bound": "hbm", "achieved": sel_gbs, "peak": hbm, "unit": "GB/s",
                            "frac": sel_gbs / hbm, "frac_of_8TBs": sel_gbs / 8000.0,
                            "algorithmic_bytes_per_step": sbytes},
        "roofline_gather": {"steps": "(f)", "bound": "hbm", "achieved": g_gbs, "peak": hbm, "unit": "GB/s",
                            "frac": g_gbs / hbm, "algorithmic_bytes_per_step": gbytes},
    }


def run_ours(args, rank, world, local_rank):
    import sparse_kv_selection_quoka_b200 as q

    q.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    run = WorkloadRun(q, args.workload, rank, dev)
    w = run.w
    sampler = ClockSampler(local_rank)
    t = time_run(q, run, args.steps, args.warmup, flush, stream, world, dev, sampler=sampler)
    rf = rooflines(run, t, world)
    K_ = args.steps
    out = {
        "metric": METRIC,
        "value": rf["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": K_,
        "warmup": args.warmup,
        "ms_per_step": t["ms_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded; the workload's shapes and planted value structure)",
        "config": {"workload": w.name, "b": w.b, "nq": w.nq, "nkv": w.nkv, "d": w.d,
                   "T": w.T, "BCP": w.BCP, "NQ": w.NQ, "BSA": w.BSA, "parallelism": f"replicas{world}",
                   "l2": "flushed before every timed step (256 MiB write, untimed)"},
        "keys_scored_per_s": rf["keys_scored_per_s"],
        "keys_scored_per_s_query_heads": rf["keys_scored_per_s_query_heads"],
        "ms_select": t["ms_select"],
        "ms_gather": t["ms_gather"],
        "ms_attention": t["ms_attention"],
        "roofline": rf["roofline"],
        "roofline_select": rf["roofline_select"],
        "roofline_gather": rf["roofline_gather"],
        "clocks": t["clocks"],
        "gpu_launches": run.launches() * K_,
    }
    if w.name == "qwen3-4b_T32k" and w.dtype == "bf16":
        out["roofline"]["traffic_from_committed_profile"] = _profiled_traffic(
            "attn_tma_qwen3-4b_T32k.md", "sparse_kv_selection_quoka_b200/csrc/attn_tma.cu",
            "sparse_kv_selection_quoka_b200/csrc/attn_common.cuh")
    if run.sweep:
        out["per_chunk_ms"] = t["per_chunk_ms"]
    else:
        Q, K, V, Kc, Vc = run.dev_inputs
        out["decode"] = measure_decode(q, w, dev, stream, flush, Q, K, V, Kc, Vc, min(K_, 50))
    if not args.no_e2e:
        out["e2e"] = run_e2e(args, run, q, dev, stream, world)
    if not args.no_other_workloads and args.workload == DEFAULT_WORKLOAD:
        out["per_workload"] = other_workloads(q, args, rank, world, dev, stream, flush, exclude=w.name)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(run.w, run.x, run.sweep)
    return out


def other_workloads(q, args, rank, world, dev, stream, flush, exclude):
    """The same measurement (no e2e, decode or oracle legs) on the other
    bf16 workloads: the Llama-shaped layer, the chunked-prefill sweep (with
    its per-chunk time curve) and the 128K-key layer."""
    out = {}
    for name in OTHER_WORKLOADS:
        if name == exclude:
            continue
        run = WorkloadRun(q, name, rank, dev)
        steps = max(3, min(args.steps, 50 if not run.sweep else 10))
        t = time_run(q, run, steps, 3, flush, stream, world, dev)
        rf = rooflines(run, t, world)
        w = run.w
        entry = {"config": {"b": w.b, "nq": w.nq, "nkv": w.nkv, "d": w.d, "T": w.T, "BCP": w.BCP, "NQ": w.NQ,
                            "BSA": w.BSA if not run.sweep else "25% of T (min 256)"},
                 "steps": steps, "ms_per_step": t["ms_step"], "value": rf["value"], "unit": UNIT,
                 "keys_scored_per_s": rf["keys_scored_per_s"], "ms_select": t["ms_select"],
                 "ms_gather": t["ms_gather"], "ms_attention": t["ms_attention"], "roofline": rf["roofline"],
                 "roofline_select": rf["roofline_select"], "roofline_gather": rf["roofline_gather"],
                 "gpu_launches": run.launches() * steps}
        if run.sweep:
            entry["per_chunk_ms"] = t["per_chunk_ms"]
        out[name] = entry
        del run
        torch.cuda.empty_cache()
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
            torch.cuda._sleep(HOST_LEAD_CYCLES)
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


def run_e2e(args, run, q, dev, stream, world):
    """The same metric through the public whole-step call with host buffers:
    every step copies that step's inputs from pinned host memory to the
    device, runs quoka_prefill_chunk, and copies the output back."""
    x, w, tdt = run.x, run.w, run.tdt
    arrays = (x.Qs, x.Ks, x.Vs) if run.sweep else (x.Q, x.K, x.V, x.Kc, x.Vc)
    host = [torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(tdt).pin_memory() for a in arrays]
    dbuf = [torch.empty_like(h, device=dev) for h in host]
    h2d = sum(h.numel() * h.element_size() for h in host)
    O_host = [torch.empty(ch["O"].shape, dtype=tdt).pin_memory() for ch in run.chunks]
    d2h = sum(o.numel() * o.element_size() for o in O_host)

    def step():
        for h, d_ in zip(host, dbuf):
            d_.copy_(h, non_blocking=True)
        if run.sweep:
            Qs, Ks, Vs = dbuf
            L = run.BCP
            for c, ch in enumerate(run.chunks):
                T = ch["T"]
                q.quoka_prefill_chunk(Qs[:, :, T:T + L], Ks[:, :, :T], Vs[:, :, :T], Ks[:, :, T:T + L],
                                      Vs[:, :, T:T + L], w.NQ, ch["bsa"], O=ch["O"], ws=ch["ws"], stream=stream)
                O_host[c].copy_(ch["O"], non_blocking=True)
        else:
            Q, K, V, Kc, Vc = dbuf
            ch = run.chunks[0]
            q.quoka_prefill_chunk(Q, K, V, Kc, Vc, w.NQ, w.BSA, O=ch["O"], ws=ch["ws"], stream=stream)
            O_host[0].copy_(ch["O"], non_blocking=True)

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
    # what bounds it: the host-to-device copy of the inputs, alone
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(n):
        for h, d_ in zip(host, dbuf):
            d_.copy_(h, non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    ms_h2d = max_over_ranks([e2.elapsed_time(e3) / n], world, dev)[0]
    return {"value": job_throughput(world, run.tokens(), ms), "unit": UNIT, "ms_per_step": ms,
            "steps": n, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "h2d_gbs_in_step": h2d / (ms / 1e3) / 1e9,
            "ms_h2d_copies_alone": ms_h2d, "h2d_gbs_alone": h2d / (ms_h2d / 1e3) / 1e9,
            "call": "quoka_prefill_chunk (C ABI) with pinned-host inputs copied in and O copied out every step; "
                    "the input copy bounds it"}


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


def _time_oracle_groups(x, nkv, budget_s, max_groups):
    """Times whole KV-head groups of the oracle until budget_s or
    max_groups; returns (groups, seconds)."""
    t0 = time.perf_counter()
    n = 0
    while True:
        _oracle_head_step(x, n % nkv)
        n += 1
        if time.perf_counter() - t0 >= budget_s or n >= max_groups:
            break
    return n, time.perf_counter() - t0


def cpu_baseline(w, x, sweep, budget_s=10.0):
    """The oracle as it stands on the host cores, on a bounded sample of the
    workload: whole KV-head groups (1/nkv of a step each), timed with the
    BLAS pool at its default size (all cores) and again with one thread."""
    if sweep:
        x = x.chunk(x.n_chunks // 2)
    tokens_per_group = x.Q.shape[0] * x.Q.shape[2] / w.nkv
    n, dt = _time_oracle_groups(x, w.nkv, budget_s, 2 * w.nkv)
    out = {"value": tokens_per_group * n / dt, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
           "sample": f"{n} KV-head groups (each 1/{w.nkv} of a step) of workload {w.name}"
                     + (" (chunk 32 of the sweep)" if sweep else "") + f", {dt:.1f} s",
           "host_cpu_count": os.cpu_count()}
    try:
        import threadpoolctl
        with threadpoolctl.threadpool_limits(1):
            n1, dt1 = _time_oracle_groups(x, w.nkv, budget_s, w.nkv)
        out["one_thread"] = {"value": tokens_per_group * n1 / dt1, "unit": UNIT, "cores": 1,
                             "sample": f"{n1} KV-head groups, {dt1:.1f} s"}
    except ImportError:
        out["one_thread"] = None
    return out


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm. Its step is a bounded sample of
    the workload: one KV-head group (the G query heads of one KV head over
    the whole chunk, 1/nkv of the work, heads being independent through
    every step). ms_per_step is the measured time of that sample, and the
    metric counts the chunk tokens it stands for (BCP * b / nkv)."""
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
    ms_step = dt / args.steps * 1e3
    tokens = x.Q.shape[0] * x.Q.shape[2] / w.nkv
    value = tokens / (ms_step / 1e3)
    cores = _blas_threads()
    sample = f"one KV-head group per step (1/{w.nkv} of a step of {w.name}: {tokens:g} chunk-tokens' worth)"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": w.name, "b": w.b, "nq": w.nq, "nkv": w.nkv, "d": w.d, "T": w.T,
                       "BCP": w.BCP, "NQ": w.NQ, "BSA": w.BSA, "parallelism": "host cores",
                       "sample": sample, "sampled_fraction_of_step": 1.0 / w.nkv},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the per_workload block (the other bf16 workloads)")
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
