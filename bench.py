"""Benchmark of the HySparse MQA forward path on B200.

One step = one pass of the whole forward path over one batch of synthetic
input: hs_block_score -> hs_select_topk -> hs_sparse_mqa_fwd, plus
hs_swa_mqa_fwd over the same q, k, v.  Default workload: one document of
4096 tokens, 64 query heads over one KV head, Dk 576 (512 latent + 64 RoPE),
Dv 512, bf16, block 64, top-16, window 512.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  Timing: W untimed warm-up steps; then K
steps, each bracketed by CUDA events on the launching stream with an L2
flush (a 512 MiB write) between steps outside the events; barrier +
synchronize around the timed loop; max over ranks.  Under torchrun every
rank runs its own replica of the workload (weak scaling, no data-path
collective: documents are independent).

``--impl reference`` times the float64 CPU oracle (the only reference this
path has) on a bounded sample of query rows of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_mqa_b200 import hs, synth, workloads  # noqa: E402

METRIC = "HySparse fwd tokens/s at 64 heads, Dk576/Dv512; % of bf16 tensor peak"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=workloads.MAIN.name)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the (separately timed) backward of the two attention steps")
    ap.add_argument("--no-full-layer", action="store_true",
                    help="skip the (separately timed) full layer's fused forward")
    ap.add_argument("--no-swa-layer", action="store_true",
                    help="skip the (separately timed) combined SWA layer")
    ap.add_argument("--cpu-rows", type=int, default=4096,
                    help="query rows of the oracle sample (cpu_baseline / reference arm); "
                         "4096 covers the main workload whole")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-setting timings of the packed, long-context and "
                         "sweep workloads")
    return ap.parse_args()


def ncu_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu record, or
    None when the kernel source changed since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        rec = json.load(open(p))[kernel]
        src = open(os.path.join(ROOT, rec["source"]), "rb").read()
    except (OSError, KeyError, ValueError):
        return None
    if hashlib.sha256(src).hexdigest() != rec["sha256"]:
        return None
    return rec["bytes"]


NOMINAL_BF16_TFLOPS = 2250.0   # dense bf16, per GPU (context only)
# a step at least this long keeps the GPU under sustained load (the clocks
# settle under the power cap): its tensor kernels are measured against the
# sustained bf16 peak, shorter steps against the burst peak
LONG_STEP_MS = 20.0
NOMINAL_HBM_GBS = 8000.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------------------
# algorithmic work (valid (query, key) pairs only)
# ---------------------------------------------------------------------------

def causal_pairs(docs):
    return sum(n * (n + 1) // 2 for n in docs)


def window_pairs(docs, W):
    tot = 0
    for n in docs:
        m = min(n, W)
        tot += m * (m + 1) // 2 + (n - m) * W
    return tot


def select_bytes(docs, B, topk):
    """Algorithmic bytes of step 2: each query t reads its candidates'
    scores, blocks 0 .. bq(t) of its row (4 bytes each), and writes topk
    ids (4 bytes each)."""
    tot = 0
    for n in docs:
        full, rem = divmod(n, B)  # blocks with all B queries, then a partial one
        tot += B * full * (full + 1) // 2 + rem * (full + 1)
    return 4.0 * tot + 4.0 * sum(docs) * topk


def sparse_pairs(idx, cu, B):
    """sum_t |S_t| from the selected blocks (keys of each block up to t)."""
    idx = idx.cpu().numpy().astype(np.int64)
    tot = 0
    for d in range(len(cu) - 1):
        bos, eos = cu[d], cu[d + 1]
        if eos <= bos:
            continue
        t = np.arange(bos, eos)[:, None]
        b = idx[bos:eos]
        lo = bos + b * B
        cnt = np.minimum(lo + B, t + 1) - lo
        tot += int(np.where(b >= 0, np.clip(cnt, 0, B), 0).sum())
    return tot


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons during the timed region.  NVML is
    read from a background thread every 2 ms (a timed region of a few tens
    of milliseconds still gets samples); without NVML, nvidia-smi -lms runs
    as a child process.  start() returns once the first sample is in, so the
    timed region that follows is covered from its first step."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.nvml = None
        self.lines = []
        self.sm = []
        self.reasons = set()
        self.smax = None
        self.source = None
        self._stop = threading.Event()

    def _start_nvml(self):
        import pynvml
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(self.dev)
        bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
        h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}

        def poll():
            while not self._stop.is_set():
                self.sm.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                for nm, b in bits.items():
                    if r & b:
                        self.reasons.add(nm)
                time.sleep(0.002)

        self.nvml = pynvml
        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        self.source = "nvml"

    def _start_smi(self):
        self.proc = subprocess.Popen(
            ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
             "--format=csv,noheader,nounits", "-lms", "20"],
            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        self.source = "nvidia-smi"

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            if self._stop.is_set():
                break
            self.sm.append(sm)
            self.smax = smax
            for nm, val in zip(self.NAMES, parts[5:9]):
                if val.lower().startswith("active"):
                    self.reasons.add(nm)

    def start(self):
        try:
            self._start_nvml()
        except Exception:
            try:
                self._start_smi()
            except (OSError, FileNotFoundError):
                self.proc = None
                return
        t0 = time.time()
        while not self.sm and time.time() - t0 < 5.0:
            time.sleep(0.001)
        self.sm.clear()  # keep only samples taken from here on
        self.reasons.clear()

    def stop(self):
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock source unavailable"]}
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.thread.join(timeout=5)
        sm = list(self.sm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax,
                "reasons": sorted(self.reasons), "samples": len(sm), "source": self.source}


# ---------------------------------------------------------------------------
# the oracle on a bounded sample (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(wl, rows_n, seed=0):
    """Inputs and a row sample for the oracle (host tensors, same recipe)."""
    import oracle.hysparse as O  # test infrastructure: the CPU baseline only
    inp = synth.make_inputs(wl.total_tokens, wl.num_heads, wl.dk, wl.dv, dtype=wl.dtype,
                            seed=seed, device="cpu", doc_lengths=wl.docs())
    f = lambda t: t.double().numpy()
    host = (f(inp.q), f(inp.k), f(inp.v), f(inp.sink), inp.cu_seqlens.tolist())
    per_doc = max(2, rows_n // len(wl.docs()))
    rows = synth.sample_rows(inp.cu_seqlens, per_doc, seed)
    return O, host, rows


def oracle_step(O, host, rows, wl):
    q, k, v, s, cu = host
    bs = O.block_score(q, k, cu, wl.block_size, rows=rows)
    idx = O.select_topk(bs["block_score"], cu, wl.block_size, wl.topk, rows=rows,
                        total_tokens=wl.total_tokens)
    O.sparse_mqa_fwd(q, k, v, idx, cu, wl.block_size, sink=s, rows=rows)
    O.swa_mqa_fwd(q, k, v, cu, wl.window, sink=s, rows=rows)


def cpu_cores():
    try:
        aff = len(os.sched_getaffinity(0))
    except AttributeError:
        aff = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        blas = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        blas = aff
    return min(aff, blas), aff, blas


def run_cpu_baseline(wl, rows_n, steps=1):
    O, host, rows = oracle_sample(wl, rows_n)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle_step(O, host, rows, wl)
    dt = time.perf_counter() - t0
    used, aff, blas = cpu_cores()
    what = ("all %d query rows of %s (the whole workload)" % (len(rows), wl.name)
            if len(rows) == wl.total_tokens else "%d query rows of %s" % (len(rows), wl.name))
    return {"value": len(rows) * steps / dt, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": "%s, all four steps, float64 NumPy, %d step(s), %.1f s; "
                      "os.cpu_count() %d, affinity %d cores, BLAS threads %d" % (
                          what, steps, dt, os.cpu_count() or 0, aff, blas)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas; control plane only)
# ---------------------------------------------------------------------------

def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a host scalar over all ranks (the device-timed region of the
    slowest rank defines the job's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens(tokens_per_rank, world):
    """Whole-job units: every rank processes its own replica of the workload
    (independent documents, no data-path collective)."""
    return tokens_per_rank * world


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

class Step:
    """Preallocated buffers and the four C-ABI calls of one forward step."""

    def __init__(self, inp, wl):
        self.inp, self.wl = inp, wl
        T, H = inp.total_tokens, wl.num_heads
        nb = hs.nbmax(inp.max_seqlen, wl.block_size)
        dev = inp.q.device
        f32 = torch.float32
        self.lse1 = torch.empty((T, H), device=dev, dtype=f32)
        self.bs = torch.empty((T, nb), device=dev, dtype=f32)
        self.idx = torch.empty((T, wl.topk), device=dev, dtype=torch.int32)
        self.out = torch.empty((T, H, wl.dv), device=dev, dtype=inp.q.dtype)
        self.lse = torch.empty((T, H), device=dev, dtype=f32)
        self.wout = torch.empty_like(self.out)
        self.wlse = torch.empty_like(self.lse)
        need = hs.workspace_size(hs.HS_OP_BLOCK_SCORE, T, len(wl.docs()), inp.max_seqlen, H,
                                 wl.dk, wl.dv, inp.q.dtype, wl.block_size)
        self.ws = torch.empty(max(need, 1), device=dev, dtype=torch.uint8)

    def score(self):
        i, w = self.inp, self.wl
        hs.hs_block_score(i.q, i.k, i.cu_seqlens, i.max_seqlen, w.block_size, out_lse=self.lse1,
                          out_block_score=self.bs, workspace=self.ws)

    def select(self):
        i, w = self.inp, self.wl
        hs.hs_select_topk(self.bs, i.cu_seqlens, i.max_seqlen, w.block_size, w.topk,
                          out_idx=self.idx)

    def sparse(self):
        i, w = self.inp, self.wl
        hs.hs_sparse_mqa_fwd(i.q, i.k, i.v, self.idx, i.cu_seqlens, i.max_seqlen, w.block_size,
                             i.sink, out=self.out, lse=self.lse)

    def swa(self):
        i, w = self.inp, self.wl
        hs.hs_swa_mqa_fwd(i.q, i.k, i.v, i.cu_seqlens, i.max_seqlen, w.window, i.sink,
                          out=self.wout, lse=self.wlse)

    PHASES = ("score", "select", "sparse", "swa")

    def run(self, events=None):
        for n, ph in enumerate(self.PHASES):
            if events is not None:
                events[n].record()
            getattr(self, ph)()
        if events is not None:
            events[len(self.PHASES)].record()


def run_ours(args, wl, world, rank):
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = synth.make_inputs(wl.total_tokens, wl.num_heads, wl.dk, wl.dv, dtype=wl.dtype, seed=rank,
                            device=dev, doc_lengths=wl.docs())
    step = Step(inp, wl)
    flush = torch.empty(512 * 1024 * 1024, device=dev, dtype=torch.uint8)
    for _ in range(max(3, args.warmup)):
        step.run()
    torch.cuda.synchronize()
    hs.poll_status(dev)
    cu = inp.cu_seqlens.cpu().tolist()

    nph = len(Step.PHASES)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(args.steps)]
    clocks = ClockSampler(dev.index) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    for s in range(args.steps):
        flush.fill_(s & 0xff)  # evict L2 between steps (outside the events)
        gpu_busy()
        step.run(evs[s])
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    hs.poll_status(dev)

    per_phase = [[evs[s][p].elapsed_time(evs[s][p + 1]) for s in range(args.steps)]
                 for p in range(nph)]
    step_ms = [sum(per_phase[p][s] for p in range(nph)) for s in range(args.steps)]
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    tokens = job_tokens(wl.total_tokens, world)
    value = tokens / (ms_per_step / 1e3)

    pk = peaks()
    H = wl.num_heads
    flops = {
        "score": 2.0 * H * wl.dk * causal_pairs(wl.docs()),
        "sparse": 2.0 * H * (wl.dk + wl.dv) * sparse_pairs(step.idx, cu, wl.block_size),
        "swa": 2.0 * H * (wl.dk + wl.dv) * window_pairs(wl.docs(), wl.window),
    }
    nb = hs.nbmax(inp.max_seqlen, wl.block_size)
    sel_bytes = select_bytes(wl.docs(), wl.block_size, wl.topk)
    avg = {ph: statistics.mean(per_phase[p]) for p, ph in enumerate(Step.PHASES)}
    sustained = sum(avg.values()) >= LONG_STEP_MS and pk.get("bf16_tflops_sustained")
    tpk = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    kernels = {}
    for ph in ("score", "sparse", "swa"):
        tf = flops[ph] / (avg[ph] / 1e3) / 1e12
        kernels[ph] = {"ms": avg[ph], "tflops": tf, "frac_of_bf16_peak": tf / tpk,
                       "frac_of_nominal_bf16": tf / NOMINAL_BF16_TFLOPS,
                       "algorithmic_flops": flops[ph],
                       "path": "tcgen05" if hs.path(
                           {"score": 0, "sparse": 2, "swa": 3}[ph], wl.dtype, H, wl.dk, wl.dv,
                           wl.block_size) == hs.HS_PATH_TCGEN05 else "simt"}
    sel_gbs = sel_bytes / (avg["select"] / 1e3) / 1e9
    # gather traffic of the sparse step: every valid (query, key) pair moves one
    # K row and one V row from L2 to an SM (the unique KV is only T rows)
    kernels["sparse"]["gather_bytes_l2_to_sm"] = 2.0 * (wl.dk + wl.dv) * flops["sparse"] / (
        2.0 * H * (wl.dk + wl.dv))
    kernels["sparse"]["unique_kv_bytes"] = 2.0 * (wl.dk + wl.dv) * wl.total_tokens
    kernels["select"] = {"ms": avg["select"], "gbs": sel_gbs, "frac_of_hbm": sel_gbs / pk["hbm_gbs"],
                         "frac_of_nominal_hbm": sel_gbs / NOMINAL_HBM_GBS,
                         "algorithmic_bytes": sel_bytes, "path": "simt"}
    dom = max(("score", "sparse", "swa"), key=lambda ph: avg[ph])
    roof = {"bound": "tensor", "achieved": kernels[dom]["tflops"], "peak": tpk,
            "unit": "TFLOP/s", "frac": kernels[dom]["tflops"] / tpk,
            "traffic": ncu_traffic(dom) if wl.name == workloads.MAIN.name else None,
            "kernel": dom,
            "peak_source": "%s bf16 %s (MEASURED_PEAKS.json)" % (
                pk["source"], "sustained: step >= %g ms" % LONG_STEP_MS if sustained else "burst")}
    contraction_tflops = (flops["score"] + flops["sparse"] + flops["swa"]) / (
        (avg["score"] + avg["sparse"] + avg["swa"]) / 1e3) / 1e12

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(inp, wl, step, max(3, min(args.steps, 10)), world)
    bwd = None
    if not args.no_backward:
        bwd = run_backward(inp, wl, step, cu, pk)
    full = None
    if not args.no_full_layer:
        full = run_full_layer(inp, wl, pk, flush, avg["score"])
    layer = None
    if not args.no_swa_layer:
        layer = run_swa_layer(inp, wl, step, pk, flush, flops["sparse"] + flops["swa"],
                              avg["sparse"] + avg["swa"])
    other = None
    if not args.no_workloads and world == 1 and wl.name == workloads.MAIN.name:
        torch.cuda.empty_cache()
        other = run_workloads(pk, flush)

    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded N(0,1) q/k/v/sink, torch generator on device)",
        "config": {"workload": wl.name, "tokens_per_gpu": wl.total_tokens, "num_heads": H,
                   "dk": wl.dk, "dv": wl.dv, "block_size": wl.block_size, "topk": wl.topk,
                   "window": wl.window, "docs": len(wl.docs()), "parallelism": "replicas x%d" % world,
                   "l2": "flushed between steps (512 MiB write outside the timed events)",
                   "step": "block_score + select_topk + sparse_mqa + swa_mqa"},
        "roofline": roof,
        "kernels": kernels,
        "score_select_sparse_tokens_per_s": tokens / ((avg["score"] + avg["select"] + avg["sparse"]) / 1e3),
        "contraction_tflops": contraction_tflops,
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
        "e2e": e2e,
        "backward": bwd,
        "full_layer": full,
        "swa_layer": layer,
        "workloads": other,
    }
    return res


def gpu_busy():
    """Keeps the GPU busy (~0.1 ms spin, outside the timed events) while the
    host enqueues the next timed calls, so that their events measure device
    time only, not the host's launch overhead."""
    torch.cuda._sleep(200000)


def _timed(fn, flush, reps, warm=2):
    """CUDA-event milliseconds of fn() per call (mean of reps), L2 flushed
    before each call outside the events, after warm untimed calls."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for r in range(reps):
        flush.fill_(r & 0xff)
        gpu_busy()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.mean(ts)


def run_workloads(pk, flush, reps=3):
    """Per-setting numbers of the other workloads: the packed 16384-token
    one, the 65536-token long context, the 4 x 32768 sparsity sweep (top-k 8,
    16, 32, 64; block scoring depends on no top-k, so it is timed once for
    the four) and the sweep's separate SWA-only layer (Dk 192 / Dv 128,
    windows 256, 1024, 4096).  Each kernel: CUDA-event time per call (mean of
    `reps`, L2 flushed before each, two untimed calls first), its
    algorithmic work and the fraction of the bf16 peak; a step of 20 ms or
    more is measured against the sustained peak, shorter ones against the
    burst peak.  SM clocks are sampled during each workload's timed calls."""
    dev = torch.device("cuda", torch.cuda.current_device())
    res = {}

    def frac_of(ms_total):
        sus = ms_total >= LONG_STEP_MS and pk.get("bf16_tflops_sustained")
        return (pk["bf16_tflops_sustained"] if sus else pk["bf16_tflops"]), \
            ("sustained" if sus else "burst")

    def kern(ms, fl, peak):
        tf = fl / (ms / 1e3) / 1e12
        return {"ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / peak, "algorithmic_flops": fl}

    def one(wl, topks, with_swa=True, swa_only=False):
        inp = synth.make_inputs(wl.total_tokens, wl.num_heads, wl.dk, wl.dv, dtype=wl.dtype,
                                seed=0, device=dev, doc_lengths=wl.docs())
        cu = inp.cu_seqlens.cpu().tolist()
        H, T = wl.num_heads, wl.total_tokens
        clocks = ClockSampler(dev.index)
        clocks.start()
        out = {}
        if swa_only:
            o = torch.empty((T, H, wl.dv), device=dev, dtype=wl.dtype)
            l = torch.empty((T, H), device=dev, dtype=torch.float32)
            ms = _timed(lambda: hs.hs_swa_mqa_fwd(inp.q, inp.k, inp.v, inp.cu_seqlens,
                                                  inp.max_seqlen, wl.window, inp.sink, out=o,
                                                  lse=l), flush, reps)
            peak, kind = frac_of(ms)
            out = {"swa": kern(ms, 2.0 * H * (wl.dk + wl.dv) * window_pairs(wl.docs(), wl.window),
                               peak),
                   "tokens_per_s": T / (ms / 1e3), "peak": kind}
        else:
            step = Step(inp, wl)
            ms_score = _timed(step.score, flush, reps)
            per_k = {}
            for k in topks:
                w2 = workloads.Workload(wl.name, T, H, wl.dk, wl.dv, wl.dtype, wl.block_size, k,
                                        wl.window, wl.doc_lengths)
                st = Step(inp, w2)
                st.bs, st.ws, st.lse1 = step.bs, step.ws, step.lse1
                ms_sel = _timed(st.select, flush, reps)
                ms_sp = _timed(st.sparse, flush, reps)
                ms_tot = ms_score + ms_sel + ms_sp
                peak, kind = frac_of(ms_tot)
                pairs = sparse_pairs(st.idx, cu, wl.block_size)
                sel_bytes = select_bytes(wl.docs(), wl.block_size, k)
                per_k[k] = {
                    "score": kern(ms_score, 2.0 * H * wl.dk * causal_pairs(wl.docs()), peak),
                    "select": {"ms": ms_sel, "gbs": sel_bytes / (ms_sel / 1e3) / 1e9,
                               "frac_of_hbm": sel_bytes / (ms_sel / 1e3) / 1e9 / pk["hbm_gbs"],
                               "algorithmic_bytes": sel_bytes},
                    "sparse": kern(ms_sp, 2.0 * H * (wl.dk + wl.dv) * pairs, peak),
                    "score_select_sparse_tokens_per_s": T / (ms_tot / 1e3), "peak": kind}
                del st
            if with_swa:
                ms_swa = _timed(step.swa, flush, reps)
                k0 = topks[0]
                peak = pk["bf16_tflops_sustained"] if per_k[k0]["peak"] == "sustained" \
                    else pk["bf16_tflops"]
                per_k[k0]["swa"] = kern(ms_swa, 2.0 * H * (wl.dk + wl.dv) *
                                        window_pairs(wl.docs(), wl.window), peak)
                tot = ms_score + per_k[k0]["select"]["ms"] + per_k[k0]["sparse"]["ms"] + ms_swa
                per_k[k0]["step_tokens_per_s"] = T / (tot / 1e3)
            out = per_k[topks[0]] if len(topks) == 1 else {"topk_%d" % k: v for k, v in per_k.items()}
            del step
        out["clocks"] = clocks.stop()
        out["config"] = {"tokens": T, "docs": len(wl.docs()), "num_heads": H, "dk": wl.dk,
                         "dv": wl.dv, "block_size": wl.block_size, "window": wl.window}
        del inp
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        return out

    t0 = time.perf_counter()
    res[workloads.PACKED.name] = one(workloads.PACKED, [workloads.PACKED.topk])
    res[workloads.LONG.name] = one(workloads.LONG, [workloads.LONG.topk])
    sw = workloads.sweep(16)
    res["sweep_4x32768_H64_dk576_dv512_bf16_B64"] = one(sw, [8, 16, 32, 64], with_swa=False)
    for w in (256, 1024, 4096):
        wl = workloads.sweep_swa(w)
        res[wl.name] = one(wl, [], swa_only=True)
    hs.poll_status(dev)
    res["wall_s"] = time.perf_counter() - t0
    return res


def run_swa_layer(inp, wl, step, pk, flush, flops, separate_ms, reps=3):
    """The combined SWA layer (window branch + sparse branch, gated sum), not
    part of the headline step: the step's q, k, v serve as both the layer's
    own and the shared KV and the step's block lists as the full layer's;
    per-(token, head) gates are uniform random.  CUDA-event time per call
    with L2 flushed before each; algorithmic work = the two branches'."""
    T, H = wl.total_tokens, wl.num_heads
    dev = inp.q.device
    g = torch.Generator(device=dev)
    g.manual_seed(321)
    gw = torch.rand((T, H), generator=g, device=dev)
    gs = torch.rand((T, H), generator=g, device=dev)
    out = torch.empty((T, H, wl.dv), device=dev, dtype=inp.q.dtype)
    lw = torch.empty((T, H), device=dev, dtype=torch.float32)
    ls = torch.empty_like(lw)

    def fn():
        hs.hs_swa_layer_fwd(inp.q, inp.k, inp.v, inp.k, inp.v, step.idx, inp.cu_seqlens,
                            inp.max_seqlen, wl.window, wl.block_size, inp.sink, inp.sink, gw, gs,
                            out=out, lse_swa=lw, lse_sparse=ls)

    fn()
    torch.cuda.synchronize()
    ts = []
    for r in range(reps):
        flush.fill_(r & 0xff)
        gpu_busy()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    hs.poll_status(dev)
    ms = statistics.mean(ts)
    tf = flops / (ms / 1e3) / 1e12
    return {"ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / pk["bf16_tflops"],
            "algorithmic_flops": flops, "calls_timed": reps,
            "separate_sparse_plus_swa_ms": separate_ms, "tokens_per_s": T / (ms / 1e3),
            "path": "tcgen05" if hs.path(hs.HS_OP_SWA_LAYER, wl.dtype, H, wl.dk, wl.dv,
                                         wl.block_size) == hs.HS_PATH_TCGEN05 else "simt",
            "launches_per_call": 2}


def run_full_layer(inp, wl, pk, flush, score_ms, reps=3):
    """The full layer's forward with step 1 fused in (not part of the
    headline step, which uses step 1 alone): CUDA-event time per call with L2
    flushed before each, one untimed call first.  Algorithmic work per causal
    (query, key) pair and head: 2 Dk (scores) + 2 Dv (PV) flops."""
    T, H = wl.total_tokens, wl.num_heads
    dev = inp.q.device
    nb = hs.nbmax(inp.max_seqlen, wl.block_size)
    out = torch.empty((T, H, wl.dv), device=dev, dtype=inp.q.dtype)
    lse = torch.empty((T, H), device=dev, dtype=torch.float32)
    bs = torch.empty((T, nb), device=dev, dtype=torch.float32)
    ws = torch.empty(max(1, hs.workspace_size(hs.HS_OP_BLOCK_SCORE_ATTN, T, len(wl.docs()),
                                              inp.max_seqlen, H, wl.dk, wl.dv, wl.dtype,
                                              wl.block_size)), device=dev, dtype=torch.uint8)

    def fn():
        hs.hs_block_score_attn_fwd(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen,
                                   wl.block_size, out=out, lse=lse, out_block_score=bs,
                                   workspace=ws)

    fn()
    torch.cuda.synchronize()
    ts = []
    for r in range(reps):
        flush.fill_(r & 0xff)
        gpu_busy()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    hs.poll_status(dev)
    ms = statistics.mean(ts)
    fl = 2.0 * H * (wl.dk + wl.dv) * causal_pairs(wl.docs())
    tf = fl / (ms / 1e3) / 1e12
    return {"ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / pk["bf16_tflops"],
            "frac_of_nominal_bf16": tf / NOMINAL_BF16_TFLOPS, "algorithmic_flops": fl,
            "calls_timed": reps, "block_score_step_ms": score_ms,
            "tokens_per_s": T / (ms / 1e3),
            "path": "tcgen05" if hs.path(hs.HS_OP_BLOCK_SCORE_ATTN, wl.dtype, H, wl.dk, wl.dv,
                                         wl.block_size) == hs.HS_PATH_TCGEN05 else "simt",
            "outputs": "out, lse, block_score (dense causal attention + step 1, no sink)"}


def run_backward(inp, wl, step, cu, pk, reps=2):
    """Backward of the two attention steps on the same inputs (not part of the
    headline step): CUDA-event time per call, one untimed call first.
    Algorithmic work per valid (query, key) pair and head: recomputed scores
    (2 Dk), dp (2 Dv), dq (2 Dk), dk (2 Dk), dv (2 Dv) flops."""
    T, H = wl.total_tokens, wl.num_heads
    g = torch.Generator(device=inp.q.device)
    g.manual_seed(123)
    dout = torch.randn((T, H, wl.dv), generator=g, device=inp.q.device).to(wl.dtype)
    ws = torch.empty(hs.workspace_size(hs.HS_OP_SPARSE_MQA_BWD, T, len(wl.docs()), inp.max_seqlen,
                                       H, wl.dk, wl.dv, wl.dtype, wl.block_size),
                     device=inp.q.device, dtype=torch.uint8)
    calls = {
        "sparse": lambda: hs.hs_sparse_mqa_bwd(inp.q, inp.k, inp.v, step.idx, inp.cu_seqlens,
                                               inp.max_seqlen, wl.block_size, step.out, step.lse,
                                               dout, inp.sink, workspace=ws),
        "swa": lambda: hs.hs_swa_mqa_bwd(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.max_seqlen,
                                         wl.window, step.wout, step.wlse, dout, inp.sink,
                                         workspace=ws),
    }
    pairs = {"sparse": sparse_pairs(step.idx, cu, wl.block_size),
             "swa": window_pairs(wl.docs(), wl.window)}
    res = {}
    for name, fn in calls.items():
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            gpu_busy()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ms = statistics.mean(ts)
        fl = 2.0 * H * (3 * wl.dk + 2 * wl.dv) * pairs[name]
        tf = fl / (ms / 1e3) / 1e12
        res[name] = {"ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / pk["bf16_tflops"],
                     "algorithmic_flops": fl, "calls_timed": reps,
                     "path": {hs.HS_PATH_MMA: "tcgen05",
                              hs.HS_PATH_SIMT: "simt"}.get(
                         hs.path(hs.HS_OP_SPARSE_MQA_BWD if name == "sparse" else hs.HS_OP_SWA_MQA_BWD,
                                 wl.dtype, H, wl.dk, wl.dv, wl.block_size), "other")}
    hs.poll_status(inp.q.device)
    return res


def run_e2e(inp, wl, step, steps, world):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory, runs the four calls and copies its
    outputs back, all inside the timed region.  Consecutive steps overlap as
    in a serving loop: two device buffer sets, and the input copies, the
    kernels and the output copies on three streams ordered by events (step
    s + 1's inputs and step s - 1's outputs cross PCIe while step s runs)."""
    import dataclasses
    dev = inp.q.device
    hq = inp.q.cpu().pin_memory()
    hk = inp.k.cpu().pin_memory()
    hv = inp.v.cpu().pin_memory()
    hsink = inp.sink.cpu().pin_memory()
    hcu = inp.cu_seqlens.cpu().pin_memory()
    inp2 = dataclasses.replace(inp, q=torch.empty_like(inp.q), k=torch.empty_like(inp.k),
                               v=torch.empty_like(inp.v), sink=torch.empty_like(inp.sink),
                               cu_seqlens=torch.empty_like(inp.cu_seqlens))
    sets = [(inp, step), (inp2, Step(inp2, wl))]
    outs = [[st.out, st.lse, st.wout, st.wlse, st.idx] for _, st in sets]
    houts = [[torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in oo] for oo in outs]
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hsink, hcu))
    d2h = sum(t.numel() * t.element_size() for t in houts[0])
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def issue(n):
        k = n % 2
        ip, st = sets[k]
        with torch.cuda.stream(s_in):
            if n >= 2:
                s_in.wait_event(ev_run[k])  # step n - 2 has read this set's inputs
            ip.q.copy_(hq, non_blocking=True)
            ip.k.copy_(hk, non_blocking=True)
            ip.v.copy_(hv, non_blocking=True)
            ip.sink.copy_(hsink, non_blocking=True)
            ip.cu_seqlens.copy_(hcu, non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[k])
            if n >= 2:
                s_run.wait_event(ev_out[k])  # step n - 2's outputs have left this set
            st.run()
            ev_run[k].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[k])
            for o, h in zip(outs[k], houts[k]):
                h.copy_(o, non_blocking=True)
            ev_out[k].record(s_out)

    for n in range(2):
        issue(n)
    torch.cuda.synchronize()
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(dev)
    a.record(cur)
    for st_ in (s_in, s_run, s_out):
        st_.wait_event(a)
    for n in range(steps):
        issue(n + 2)
    for k in range(2):
        cur.wait_event(ev_out[k])
    b.record(cur)
    torch.cuda.synchronize()
    hs.poll_status(dev)
    ms = max_over_ranks(a.elapsed_time(b), world) / steps
    return {"value": wl.total_tokens * world / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": ms,
            "overlap": "steps pipelined: H2D, kernels and D2H on three streams, two buffer sets"}


# ---------------------------------------------------------------------------
# reference arm: the oracle on host cores
# ---------------------------------------------------------------------------

def run_reference(args, wl):
    O, host, rows = oracle_sample(wl, args.cpu_rows)
    for _ in range(max(0, min(args.warmup, 1))):
        oracle_step(O, host, rows[:2], wl)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(O, host, rows, wl)
    dt = time.perf_counter() - t0
    value = len(rows) * args.steps / dt
    used, aff, blas = cpu_cores()
    cb = {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
          "sample": "%d query rows of %s per step (all four steps, float64 NumPy); affinity %d "
                    "cores, BLAS threads %d" % (len(rows), wl.name, aff, blas)}
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1), CPU generator)",
            "config": {"workload": wl.name, "sample_rows_per_step": int(len(rows))},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    wl = workloads.ALL[args.workload]
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        if args.steps > 3:  # keep the CPU arm within minutes: fewer rows per step
            args.cpu_rows = max(8, args.cpu_rows * 3 // args.steps)
        print(json.dumps(run_reference(args, wl)), flush=True)
        return 0
    world, rank, local = dist_init(args)
    res = run_ours(args, wl, world, rank)
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            res["cpu_baseline"] = run_cpu_baseline(wl, args.cpu_rows)
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
