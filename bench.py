"""Benchmark of the paged multi-adapter LoRA delta on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the page-in call for
the batch's adapter set (LRU touch; no copies when all are resident), then the
segment build, the grouped paged shrink and the grouped expand over all
projections of one layer (decode batches of up to 1024 tokens: all three in one
persistent kernel).  Default workload: the LLaMA-7B decode layer
(7 projections, 256 tokens, 1000 resident rank-16 adapters, Zipf 1.0, fp16).

Timing: CUDA events on the compute stream right around the library's kernels
(per kernel: events the library records between them, slora_set_phase_events;
per step: events around the call).  L2 is flushed (a 256 MiB write) and y reset
before every step, outside the timed events, and a spin kernel then holds the
GPU for about 100 us, so that the host has enqueued the whole step before the
start event is reached: the timed region holds the step's device work back to
back, without the host's enqueue latency (Python marshalling and the library's
planning), as when a serving loop runs ahead of the GPU.  N > 1 (torchrun): every rank
runs an independent replica (no collective on the data path); the step time
is the max over ranks (NCCL all-reduce of the timings only).

The reference arm (--impl reference) is the fp64 CPU oracle, timed on the
host cores over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "LoRA-delta tokens/s at LLaMA-7B shapes, 1 B200; % of HBM/tensor roofline"
UNIT = "tokens/s"
FALLBACK_HBM = 6650.0
FALLBACK_BF16 = 1590.0


FALLBACK_BF16_SUSTAINED = 1400.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM, FALLBACK_BF16, "fallback"


def bf16_sustained():
    """The bf16 peak for a kernel timed inside a long step (the power-capped
    loop figure), else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m.get("bf16_tflops_sustained", m["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_BF16_SUSTAINED, "fallback"


# ---------------------------------------------------------------------------
# DRAM traffic per launch from a committed ncu capture (profiles/traffic.json),
# valid only while the kernel's source file is the one that was captured
# GPU cycles of the spin kernel ahead of each timed step (about 100 us at the
# B200's 1.965 GHz): longer than the host takes to enqueue one step.
HOLD_CYCLES = 200_000

KERNEL_SOURCE = {"stream": "stream.cu", "fused": "fused.cu", "token": "token.cu", "shrink": "bgmv.cu",
                 "expand": "bgmv.cu", "segments": "bgmv.cu", "sgmv_shrink": "sgmv.cu", "sgmv_expand": "sgmv.cu",
                 "linear": "linear.cu"}


def source_sha(name: str) -> str:
    import hashlib
    path = os.path.join(ROOT, "gather_lora_paged_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def ncu_traffic(workload: str, kernel: str):
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            e = json.load(f)[workload][kernel]
        if e["source_sha256"] != source_sha(KERNEL_SOURCE[kernel]):
            return None  # the kernel changed since the counters were taken
        return int(e["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------
# data-parallel replicas: rank k runs workload `config` with its own batch
# (seeded by k), no collective on the data path; timings are reduced by max.
def replica_workload(config: int, rank: int) -> W.Workload:
    return W.config(config, replica=rank)


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The job's time for a per-rank device time: the max over all ranks."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_step: int, steps: int, t_ms: float) -> float:
    """Whole-job tokens/s: every rank processed `steps` batches of
    `tokens_per_step` tokens in (at most) t_ms."""
    return world * tokens_per_step * steps / (t_ms / 1e3)


# ---------------------------------------------------------------------------
# algorithmic bytes / flops (each touched adapter and each distinct input read
# once, y read and written once)
def algorithmic(w: W.Workload, tokens=None, wbytes=2):
    """wbytes: bytes per adapter weight (2: 16-bit pages, 1: e4m3 codes; the
    per-row scales add r floats per tensor, counted too)."""
    idx = w.idx if tokens is None else w.idx[tokens]
    T = idx.size
    esz = 2
    touched = np.unique(idx[idx >= 0])
    r_sum = int(w.ranks[touched].sum())
    din = sum(p.d_in for p in w.projs)
    dout = sum(p.d_out for p in w.projs)
    xin = sum(w.x_dim(n) for n in w.x_names)
    n_t = len(w.projs)
    A_bytes = r_sum * din * wbytes + (4 * r_sum * n_t if wbytes == 1 else 0)
    B_bytes = r_sum * dout * wbytes + (4 * r_sum * n_t if wbytes == 1 else 0)
    x_bytes = T * xin * esz
    y_bytes = 2 * T * dout * esz
    r_tok = w.ranks[idx[idx >= 0]].astype(np.int64)
    flops = int(2 * r_tok.sum() * (din + dout))
    return dict(shrink_bytes=A_bytes + x_bytes, expand_bytes=B_bytes + y_bytes,
                total_bytes=A_bytes + B_bytes + x_bytes + y_bytes, flops=flops,
                touched=int(touched.size))


# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every 2 ms through
    NVML while the timed passes run (read-only queries)."""

    PERIOD = 0.002
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.h = None
        self.stop_ev = threading.Event()

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            pr = torch.cuda.get_device_properties(self.index)
            bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def start(self):
        try:
            import pynvml
            self.nv = pynvml
            self.h = self._handle()
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.h = None

    def _reasons(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(f(self.h))

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append((float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)),
                                     self._reasons()))
            except Exception:
                pass
            self.stop_ev.wait(self.PERIOD)

    def stop(self):
        if self.h is None:
            return None
        self.stop_ev.set()
        self.t.join(timeout=5)
        if not self.samples:
            return None
        reasons = sorted({n for _, m in self.samples for bit, n in self.REASONS.items() if m & bit})
        return {"sm_mhz": float(np.median([c for c, _ in self.samples])), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "source": "nvml, every 2 ms across the per-kernel, timed and warm-L2 passes"}


# ---------------------------------------------------------------------------
class DecodeRun:
    """Decode step: page-in call for the batch's adapter set (LRU touch), then
    the delta over all projections: one persistent kernel for batches of up to
    1024 tokens, else (or with split=True) segment build, grouped shrink and
    grouped expand."""
    FUSED_MAX_T = 1024

    def __init__(self, w, path="auto", weights="16", pool="all"):
        import torch

        import gather_lora_paged_b200 as G
        import harness as H
        self.G, self.H, self.w = G, H, w
        self.wbytes = 1 if weights == "e4m3" else 2
        dp = {"auto": G.SLORA_DECODE_AUTO, "split": G.SLORA_DECODE_SPLIT, "fused": G.SLORA_DECODE_FUSED,
              "stream": G.SLORA_DECODE_STREAM}[path]
        wf = G.SLORA_WEIGHTS_E4M3 if weights == "e4m3" else G.SLORA_WEIGHTS_16
        kw = {}
        if pool == "touched":  # only the batch's adapters: the same kernel work in a smaller pool
            t = sorted(set(w.touched().tolist()))
            d = G.make_desc(w.dtype, [p.d_in for p in w.projs], [p.d_out for p in w.projs], w.n_adapters,
                            int(w.ranks.max()), 1, w.page_elems, 0, weight_format=wf)
            kw = {"resident": t, "n_pages": int(sum(G.slora_pages_for_rank(d, int(w.ranks[a])) for a in t))}
        self.pb = H.PoolBuild(w, decode_path=dp, weight_format=wf, **kw)
        kind = G.slora_decode_kind(self.pb.h, w.T)
        self.phases = {G.SLORA_KIND_TOKEN: ("token",), G.SLORA_KIND_STREAM: ("stream",),
                       G.SLORA_KIND_FUSED: ("fused",)}.get(kind, ("segments", "shrink", "expand"))
        self.ncu_names = self.phases
        self.ten = H.Tensors(w)
        self.d_idx = torch.from_numpy(w.idx).cuda()
        self.touched = w.touched().tolist()

    def set_events(self, evs):
        self.G.slora_set_phase_events(self.pb.h, evs)

    def step(self, stream, outer=None, ten=None, ins=None):
        """One step on `stream`; `ten` / `ins` select another set of device
        buffers (x, y and the batch description) than the default one."""
        G = self.G
        ten = ten or self.ten
        d_idx = ins[0] if ins else self.d_idx
        G.slora_adapter_page_in(self.pb.h, self.touched, stream)
        if outer:
            outer[0].record(stream)
        G.slora_lora_delta(self.pb.h, *ten.args(), d_idx, self.w.T, stream)
        if outer:
            outer[1].record(stream)

    def inputs(self):  # device tensors refreshed from the host in the e2e run
        return [self.d_idx]


class PrefillRun(DecodeRun):
    """Prefill step: page-in call, request -> segment merge on the device, and
    the tensor-core SGMV (plan, shrink, expand) over all projections."""
    def __init__(self, w):
        import torch
        super().__init__(w)
        self.phases = ("plan", "shrink", "expand")
        self.ncu_names = ("plan", "sgmv_shrink", "sgmv_expand")
        n = w.req_adapter.size
        self.n = n
        self.d_rs = torch.from_numpy(w.req_start).cuda()
        self.d_ra = torch.from_numpy(w.req_adapter).cuda()
        self.ss = torch.zeros(n + 1, dtype=torch.int32, device="cuda")
        self.sa = torch.zeros(n, dtype=torch.int32, device="cuda")
        self.S = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(self, stream, outer=None, ten=None, ins=None):
        G = self.G
        ten = ten or self.ten
        d_rs, d_ra = ins if ins else (self.d_rs, self.d_ra)
        G.slora_adapter_page_in(self.pb.h, self.touched, stream)
        if outer:
            outer[0].record(stream)
        G.slora_build_sgmv_segments(self.pb.h, d_rs, d_ra, self.n, self.ss, self.sa, self.S, stream)
        G.slora_sgmv(self.pb.h, *ten.args(), self.ss, self.sa, self.n, self.w.T, stream)
        if outer:
            outer[1].record(stream)

    def inputs(self):
        return [self.d_rs, self.d_ra]


def run_ours(args, rank, world):
    import torch

    import harness as H

    dev = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(dev)
    w = replica_workload(args.config, rank)
    if args.config == 4:
        return run_mixed(args, rank, world, w)
    if args.linear:
        return run_linear(args, rank, world, w)
    R = PrefillRun(w) if args.config == 3 else DecodeRun(w, path=args.path, weights=args.weights, pool=args.pool)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for e in ev + outer:  # torch creates the CUDA event on first record
        e.record()
    torch.cuda.synchronize()
    alg = algorithmic(w, wbytes=getattr(R, "wbytes", 2))

    def prep():
        R.ten.reset()
        flush.zero_()
        torch.cuda._sleep(HOLD_CYCLES)

    for _ in range(args.warmup):
        prep()
        R.step(stream)
    torch.cuda.synchronize()
    st, code, info = R.G.slora_check_device(R.pb.h)
    assert st == 0, (code, info)

    # pass 1: per-kernel device times (library events between its kernels)
    nk = len(R.phases)
    pev = ev[:2] if nk == 1 else ev
    clocks = ClockSampler(dev)
    clocks.start()
    R.set_events(pev)
    kt = [0.0] * nk
    for _ in range(args.steps):
        prep()
        R.step(stream)
        pev[-1].synchronize()
        for i in range(nk):
            kt[i] += pev[i].elapsed_time(pev[i + 1])
    R.set_events([])
    # pass 2 (the timed region): whole steps, kernels back to back; the L2
    # flush ahead of each step keeps the GPU busy while the host enqueues it
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_step = 0.0
    per_step = []
    for _ in range(args.steps):
        prep()
        R.step(stream, outer)
        outer[1].synchronize()
        per_step.append(outer[0].elapsed_time(outer[1]))
        t_step += per_step[-1]
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t_step = max_over_ranks(t_step, world, "cuda")
    K = args.steps
    ms = t_step / K
    value = job_throughput(world, w.T, K, t_step)
    ms_median = max_over_ranks(float(np.median(per_step)), world, "cuda")

    # warm L2: the same steps without the flush (y still reset before each)
    Kw = min(K, 500)
    t_warm = 0.0
    for _ in range(Kw):
        R.ten.reset()
        torch.cuda._sleep(HOLD_CYCLES)
        R.step(stream, outer)
        outer[1].synchronize()
        t_warm += outer[0].elapsed_time(outer[1])
    clk = clocks.stop()
    t_warm = max_over_ranks(t_warm, world, "cuda")
    warm = {"value": job_throughput(world, w.T, Kw, t_warm), "ms_per_step": t_warm / Kw, "steps": Kw,
            "l2": "not flushed between steps"}

    # end to end through the C ABI with host buffers (pinned): every step copies
    # its x, y and batch description in from pinned host memory and its y back
    # out, all inside the timed region.  Consecutive steps are pipelined as a
    # serving loop runs them: two sets of device buffers, the host->device copies
    # of step i + 1 on one stream while step i computes on another and its
    # device->host copy runs on a third (PCIe is full duplex).
    hx = {n: H.pinned(w.x(n)) for n in w.x_names}
    hy = [H.pinned(w.y_in(p)) for p in range(len(w.projs))]
    hout = [[torch.empty_like(t).pin_memory() for t in hy] for _ in range(2)]
    hins = [t.cpu().pin_memory() for t in R.inputs()]
    sets = [(R.ten, R.inputs()), (H.Tensors(w), [t.clone() for t in R.inputs()])]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_in + ev_comp + ev_out:
        e.record()
    torch.cuda.synchronize()

    def e2e_step(i):
        b = i & 1
        ten, ins = sets[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_out[b])  # the copy-out of step i - 2 read this y
            for n in w.x_names:
                ten.x[n].view(torch.int16).copy_(hx[n], non_blocking=True)
            for p in range(len(w.projs)):
                ten.y[p].view(torch.int16).copy_(hy[p], non_blocking=True)
            for d, h in zip(ins, hins):
                d.copy_(h, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        R.step(stream, ten=ten, ins=ins)
        ev_comp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            for p in range(len(w.projs)):
                hout[b][p].copy_(ten.y[p].view(torch.int16), non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    n_e2e = max(10, min(K, 200))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record(s_in)
    for i in range(n_e2e):
        e2e_step(i)
    s_out.wait_event(ev_out[(n_e2e - 1) & 1])
    e1.record(s_out)
    e1.synchronize()
    tot = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
    h2d = sum(t.numel() * 2 for t in hx.values()) + sum(t.numel() * 2 for t in hy) + \
        sum(t.numel() * t.element_size() for t in hins)
    d2h = sum(t.numel() * 2 for t in hout[0])
    e2e = {"value": job_throughput(world, w.T, n_e2e, tot), "unit": UNIT,
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "ms_per_step": tot / n_e2e,
           "pipelining": "two device buffer sets; copy-in, compute and copy-out streams"}

    hbm, tc, src = peaks()
    kt = [t / K for t in kt]
    names = R.phases
    if nk == 1:  # one kernel runs the whole step
        i_dom, dom_bytes = 0, alg["total_bytes"]
    else:
        i_dom = 1 if kt[1] >= kt[2] else 2
        dom_bytes = alg["shrink_bytes"] if i_dom == 1 else alg["expand_bytes"]
    achieved = dom_bytes / (kt[i_dom] / 1e3) / 1e9
    step_gbs = alg["total_bytes"] / (ms / 1e3) / 1e9
    tflops = alg["flops"] / (ms / 1e3) / 1e12
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_median": ms_median,
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": W.DTYPE_NAME[w.dtype],
        "data": "synthetic (seeded N(0,1) activations, N(0,1/sqrt(d_in)) A, N(0,1/sqrt(r)) B; "
                "Zipf or uniform adapter ids)",
        "config": {"workload": w.name + ("_e4m3pages" if getattr(R, "wbytes", 2) == 1 else ""),
                   "tokens_per_step": w.T, "projections": len(w.projs),
                   "adapters": w.n_adapters, "touched_adapters": alg["touched"],
                   "adapter_weights": "e4m3 codes + fp32 row scales" if getattr(R, "wbytes", 2) == 1
                   else W.DTYPE_NAME[w.dtype],
                   "accumulate": "f32", "l2": "flushed before every step (256 MiB write)",
                   "host_enqueue": "not timed: a ~100 us spin kernel precedes each step's start event",
                   "pool": "the batch's adapters only" if getattr(args, "pool", "all") == "touched"
                   else "every adapter of the workload",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": names[i_dom], "achieved": achieved, "peak": hbm,
                     "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": ncu_traffic(w.name, R.ncu_names[i_dom]),
                     "peak_source": src, "alg_bytes_per_launch": dom_bytes},
        "step_roofline": {"achieved": step_gbs, "peak": hbm, "unit": "GB/s",
                          "frac": step_gbs / hbm, "alg_bytes_per_step": alg["total_bytes"],
                          "flops_per_step": alg["flops"],
                          "tensor_tflops": tflops, "tensor_frac_of_bf16_peak": tflops / tc,
                          "kernel_ms": dict(zip(names, kt))},
        "e2e": e2e,
        "warm_l2": warm,
        "gpu_launches": (4 if args.config == 3 else len(R.phases)) * K,
        "clocks": clk,
    }
    R.pb.close()
    return out


# ---------------------------------------------------------------------------
def run_linear(args, rank, world, w):
    """The prefill linear layer with its delta in one tensor-core kernel
    (slora_sgmv_linear): y = x . W0 + delta for the 7 projections of the
    layer, with random-init base weights.  Timed with L2 flushed before each
    step, and once more with every segment's adapter set to -1 (the base
    GEMM alone, same kernel) to give the delta's overhead."""
    import torch

    import gather_lora_paged_b200 as G
    import harness as H
    dev = int(os.environ.get("LOCAL_RANK", 0))
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    w0s = [H.to_device(w.w0(p), w.dtype) for p in range(len(w.projs))]
    rs, ra = w.req_start, w.req_adapter
    ss, sa = [0], []
    for q in range(ra.size):  # merged segments covering [0, T)
        if sa and sa[-1] == ra[q]:
            ss[-1] = int(rs[q + 1])
        else:
            sa.append(int(ra[q]))
            ss.append(int(rs[q + 1]))
    d_ss = torch.tensor(ss, dtype=torch.int32, device="cuda")
    d_sa = torch.tensor(sa, dtype=torch.int32, device="cuda")
    d_none = torch.full_like(d_sa, -1)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    projs, xs, ldx, ys, ldy = ten.args()
    ldw = [t.stride(0) for t in w0s]

    def step(ads):
        G.slora_sgmv_linear(pb.h, projs, xs, ldx, w0s, ldw, ys, ldy, d_ss, ads, len(sa), w.T, stream)

    for _ in range(args.warmup):
        flush.zero_()
        step(d_sa)
    torch.cuda.synchronize()
    st, code, info = G.slora_check_device(pb.h)
    assert st == 0, (code, info)
    clocks = ClockSampler(dev)
    clocks.start()
    res = {}
    for name, ads in (("lora", d_sa), ("base", d_none)):
        if world > 1:
            torch.distributed.barrier()
        t = 0.0
        for _ in range(args.steps):
            flush.zero_()
            e0.record(stream)
            step(ads)
            e1.record(stream)
            e1.synchronize()
            t += e0.elapsed_time(e1)
        res[name] = max_over_ranks(t, world, "cuda") / args.steps
    clk = clocks.stop()
    K = args.steps
    ms = res["lora"]
    din = [p.d_in for p in w.projs]
    dout = [p.d_out for p in w.projs]
    base_flops = 2 * w.T * sum(a * b for a, b in zip(din, dout))
    alg = algorithmic(w)
    flops = base_flops + alg["flops"]
    tflops = flops / (ms / 1e3) / 1e12
    peak, src = bf16_sustained()
    out = {
        "metric": METRIC, "value": job_throughput(world, w.T, K, ms * K), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": W.DTYPE_NAME[w.dtype],
        "data": "synthetic (seeded N(0,1) activations; N(0,1/sqrt(d_in)) base weights and A; "
                "N(0,1/sqrt(r)) B)",
        "config": {"workload": w.name + "_linear_layer", "tokens_per_step": w.T, "projections": len(w.projs),
                   "segments": len(sa), "accumulate": "f32", "l2": "flushed before every step (256 MiB write)",
                   "what": "y = x.W0 + (alpha/r)(x.A).B in one tcgen05 kernel per layer (base GEMM fused "
                           "with the delta)", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "kernel": "linear", "achieved": tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": tflops / peak, "traffic": ncu_traffic(w.name, "linear"),
                     "peak_source": src, "flops_per_step": flops},
        "lora_overhead": {"base_only_ms": res["base"], "with_delta_ms": ms,
                          "overhead_frac": ms / res["base"] - 1.0},
        "gpu_launches": 2 * K,
        "clocks": clk,
    }
    pb.close()
    return out


# ---------------------------------------------------------------------------
def pcie_h2d_peak(nbytes=1 << 30, reps=5):
    """Measured pinned host -> device copy bandwidth (GB/s), one large copy."""
    import torch
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best = 0.0
    for _ in range(reps):
        e0.record()
        d.copy_(h, non_blocking=True)
        e1.record()
        e1.synchronize()
        best = max(best, nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9)
    del h, d
    return best


def run_mixed(args, rank, world, w):
    """The mixed step (decode batch + prefill requests, 30% of the adapters
    cold): page-in of the cold adapters from pinned host memory on a side
    stream, then the BGMV and SGMV compute.  Each timed step is preceded,
    untimed, by the restore of the pool (cold set evicted, fillers back) and
    an L2 flush."""
    import torch

    import harness as H
    mode = {"kernel": H.G.SLORA_PAGEIN_KERNEL, "memcpy": H.G.SLORA_PAGEIN_MEMCPY}[args.pagein]
    M = H.MixedStep(w, pagein_mode=mode)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    K = min(args.steps, 20)
    Wm = max(3, min(args.warmup, 5))
    for _ in range(Wm):
        M.ten.reset()
        M.step(stream)
        M.restore(stream)
    st, code, info = H.G.slora_check_device(M.h)
    assert st == 0, (code, info)
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", 0)))
    clocks.start()
    t_step = t_page = t_comp = 0.0
    paged = 0
    for _ in range(K):
        M.ten.reset()
        flush.zero_()
        s0 = H.G.slora_pool_stats(M.h)
        M.step(stream, ev[0], ev[1], ev[2])
        ev[2].synchronize()
        paged += H.G.slora_pool_stats(M.h)["bytes_paged_in"] - s0["bytes_paged_in"]
        t_step += ev[0].elapsed_time(ev[2])
        t_page += ev[0].elapsed_time(ev[1])
        t_comp += ev[1].elapsed_time(ev[2])
        M.restore(stream)
    clk = clocks.stop()
    paged_steps = paged / K
    t_step = max_over_ranks(t_step, world, "cuda")
    ms, ms_page, ms_comp = t_step / K, t_page / K, t_comp / K
    value = job_throughput(world, w.T, K, t_step)

    # e2e: the same step with x, y and the batch description copied from
    # pinned host memory and y copied back, all inside the timed region
    hx = {n: H.pinned(w.x(n)) for n in w.x_names}
    hy = [H.pinned(w.y_in(p)) for p in range(len(w.projs))]
    hout = [torch.empty_like(t).pin_memory() for t in hy]
    dins = [M.d_idx, M.d_rs, M.d_ra]
    hins = [t.cpu().pin_memory() for t in dins]
    xs = {n: M.ten.x[n].view(torch.int16) for n in w.x_names}
    ys = [t.view(torch.int16) for t in M.ten.y]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, min(K, 10))
    tot = 0.0
    for _ in range(n_e2e):
        e0.record(stream)
        for n in w.x_names:
            xs[n].copy_(hx[n], non_blocking=True)
        for p in range(len(w.projs)):
            ys[p].copy_(hy[p], non_blocking=True)
        for d, h in zip(dins, hins):
            d.copy_(h, non_blocking=True)
        M.step(stream)
        for p in range(len(w.projs)):
            hout[p].copy_(ys[p], non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
        M.restore(stream)
    tot = max_over_ranks(tot, world, "cuda")
    h2d = sum(t.numel() * 2 for t in hx.values()) + sum(t.numel() * 2 for t in hy) + \
        sum(t.numel() * t.element_size() for t in hins)
    d2h = sum(t.numel() * 2 for t in hout)

    pre = prefetch_leg(M, w, stream)

    peak_pcie = pcie_h2d_peak()
    hbm, tc, src = peaks()
    alg = algorithmic(w)
    comp_gbs = alg["total_bytes"] / (ms_comp / 1e3) / 1e9
    page_gbs = paged_steps / (ms_page / 1e3) / 1e9
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": W.DTYPE_NAME[w.dtype],
        "data": "synthetic (seeded N(0,1) activations, N(0,1/sqrt(d_in)) A, N(0,1/sqrt(r)) B; "
                "Zipf adapter ids)",
        "config": {"workload": w.name, "tokens_per_step": w.T, "decode_tokens": w.n_decode,
                   "prefill_requests": M.n_req, "projections": len(w.projs),
                   "adapters": w.n_adapters, "touched_adapters": int(M.U.size),
                   "cold_adapters": int(M.cold.size), "pool_pages": M.n_pages,
                   "pagein_mode": args.pagein, "accumulate": "f32",
                   "l2": "flushed before every step (256 MiB write)",
                   "parallelism": f"replicas x{world}"},
        "pagein": {"ms": ms_page, "bytes_per_step": int(paged_steps),
                   "expected_bytes": M.cold_bytes(), "achieved_gbs": page_gbs,
                   "pcie_h2d_peak_gbs": peak_pcie, "frac": page_gbs / peak_pcie,
                   "peak_source": "pinned 1 GiB cudaMemcpyAsync, measured in this run"},
        "roofline": {"bound": "hbm", "kernel": "compute (BGMV decode + SGMV prefill)",
                     "achieved": comp_gbs, "peak": hbm, "unit": "GB/s", "frac": comp_gbs / hbm,
                     "traffic": None, "peak_source": src,
                     "alg_bytes_per_launch": alg["total_bytes"], "compute_ms": ms_comp},
        "e2e": {"value": job_throughput(world, w.T, n_e2e, tot), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": tot / n_e2e},
        # page-in gather, the decode delta (one or three kernels), request
        # merge, SGMV plan, shrink, expand
        "gpu_launches": (5 + H.G.slora_decode_kernels(M.h, w.n_decode)) * K,
        "clocks": clk,
        "prefetch": pre,
    }
    M.close()
    return out


def prefetch_leg(M, w, stream):
    """Two device-timed measurements of adapter prefetch, after the timed
    steps (pool restored: cold adapters out, fillers in).
    rare_adapter: one cold adapter of the largest rank paged in alone on the
    side stream (its copy time: what a request for a rare adapter waits).
    prefetched_step: the step with its cold adapters prefetched beforehand
    (while a step that names only the warm set is current, so the fillers are
    older and may be evicted); its page-in then finds every adapter resident."""
    import torch

    import harness as H
    G = H.G
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for e in (e0, e1):
        e.record()  # torch creates the CUDA event on its first record
    torch.cuda.synchronize()
    a = int(M.cold[np.argmax(w.ranks[M.cold])])
    e0.record(M.side)
    G.slora_adapter_page_in(M.h, [a], M.side, e1)
    e1.synchronize()
    rare_ms = e0.elapsed_time(e1)
    rare_bytes = int(w.ranks[a]) * sum(p.d_in + p.d_out for p in w.projs) * 2
    G.slora_adapter_evict(M.h, a, stream)
    back = [f for f in M.fillers if not G.slora_adapter_is_resident(M.h, f)]
    G.slora_adapter_page_in(M.h, list(M.warm) + back, M.side)     # the "current" step
    M.side.synchronize()
    n = G.slora_adapter_prefetch(M.h, M.cold.tolist(), 1 << 40, M.side)
    M.side.synchronize()
    s0 = G.slora_pool_stats(M.h)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    M.ten.reset()
    M.step(stream, ev[0], ev[1], ev[2])
    ev[2].synchronize()
    s1 = G.slora_pool_stats(M.h)
    out = {"rare_adapter": {"id": a, "rank": int(w.ranks[a]), "bytes": rare_bytes, "ms": rare_ms,
                            "gbs": rare_bytes / (rare_ms / 1e3) / 1e9},
           "prefetched_adapters": n, "cold_adapters": int(M.cold.size),
           "prefetched_step": {"ms": ev[0].elapsed_time(ev[2]), "pagein_ms": ev[0].elapsed_time(ev[1]),
                               "hits": s1["hits"] - s0["hits"],
                               "copied_bytes": s1["bytes_paged_in"] - s0["bytes_paged_in"]}}
    M.restore(stream)
    return out


# ---------------------------------------------------------------------------
def oracle_step(w: W.Workload, tokens, threads):
    import harness as H
    import oracle
    for p in range(len(w.projs)):
        x, idx, y, A_t, B = H.oracle_inputs(w, p, tokens)
        oracle.lora_delta(w.dtype, x, idx, y, w.ranks, np.full(w.n_adapters, w.alpha), A_t, B,
                          n_threads=threads)


def cpu_baseline(w: W.Workload, budget_s=10.0):
    """The oracle, as it stands, on the host cores over a bounded sample of the
    workload: whole steps when one fits the budget, else seeded uniform token
    subsets (all projections of each sampled token) for about the budget."""
    threads = os.cpu_count() or 1
    w.prefetch_adapters(w.touched().tolist())
    rng = np.random.default_rng(0)
    # cost of one token, from a small subset after a warm-up call (neither counted)
    oracle_step(w, np.arange(min(w.T, 2)), threads)
    probe = np.sort(rng.choice(w.T, size=min(w.T, 2 * threads), replace=False))
    t0 = time.perf_counter()
    oracle_step(w, probe, threads)
    per_tok = (time.perf_counter() - t0) / probe.size
    if per_tok * w.T <= budget_s:
        t0 = time.perf_counter()
        oracle_step(w, None, threads)
        n_steps = 1
        while time.perf_counter() - t0 < budget_s and n_steps < 50:
            oracle_step(w, None, threads)
            n_steps += 1
        dt = time.perf_counter() - t0
        n_tok = n_steps * w.T
        sample = (f"{n_steps} whole step(s) of {w.name} ({w.T} tokens x {len(w.projs)} "
                  f"projections each), fp64 loops, {threads} threads")
    else:
        chunk = min(w.T, 4 * threads)
        t0 = time.perf_counter()
        n_tok = 0
        while n_tok == 0 or time.perf_counter() - t0 < budget_s:
            oracle_step(w, np.sort(rng.choice(w.T, size=chunk, replace=False)), threads)
            n_tok += chunk
        dt = time.perf_counter() - t0
        sample = (f"{n_tok} tokens of {w.name} drawn uniformly in subsets of {chunk} (all "
                  f"{len(w.projs)} projections of each; a whole step of {w.T} tokens would "
                  f"take about {per_tok * w.T:.0f} s), fp64 loops, {threads} threads")
    # the same loops on one host thread, over a token subset sized to ~3 s
    t1 = time.perf_counter()
    n1 = 0
    while time.perf_counter() - t1 < 3.0 and n1 < w.T:
        tok = np.sort(rng.choice(w.T, size=min(8, w.T), replace=False))
        oracle_step(w, tok, 1)
        n1 += tok.size
    d1 = time.perf_counter() - t1
    return {"value": n_tok / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": sample, "seconds": dt,
            "single_thread": {"value": n1 / d1, "unit": UNIT, "cores": 1,
                              "sample": f"{n1} tokens of the same workload (all {len(w.projs)} "
                                        f"projections), fp64 loops, 1 thread", "seconds": d1}}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = W.config(args.config)
    for _ in range(args.warmup):
        pass
    cb = cpu_baseline(w, budget_s=max(5.0, min(60.0, 2.0 * args.steps)))
    return {"metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * w.T / cb["value"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "tokens_per_step": w.T},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", default="auto", choices=["auto", "split", "fused", "stream"],
                    help="decode kernels: the library's choice, the three-kernel path (segment "
                         "build, shrink, expand) or the one persistent kernel")
    ap.add_argument("--linear", action="store_true",
                    help="--config 3: the whole linear layer (base GEMM + delta) in one kernel")
    ap.add_argument("--pool", default="all", choices=["all", "touched"],
                    help="decode: a pool of every adapter of the workload, or of the batch's adapters only "
                         "(the same kernel work; smaller device footprint for profiler captures)")
    ap.add_argument("--weights", default="16", choices=["16", "e4m3"],
                    help="decode: adapter pages in the pool's 16-bit dtype or as e4m3 codes")
    ap.add_argument("--pagein", default="kernel", choices=["kernel", "memcpy"],
                    help="page-in mode of the mixed workload (--config 4)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out))
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    out = run_ours(args, rank, world)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(W.config(args.config))
        print(json.dumps(out))
    if world > 1:
        import torch
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
