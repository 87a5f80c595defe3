"""Builds library pools and device tensors for the synthetic workloads.

Shared by the GPU tests and bench.py.  Plumbing only: it allocates memory,
registers adapters and pages them in through the library's C ABI (via the
Python binding); it computes nothing of the method itself.
"""
from __future__ import annotations

import numpy as np

import gather_lora_paged_b200 as G
import workloads as W


def torch_dtype(dtype):
    import torch
    return torch.float16 if dtype == W.F16 else torch.bfloat16


def to_device(bits: np.ndarray, dtype, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch_dtype(dtype))


def from_device(t) -> np.ndarray:
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def pinned(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).pin_memory()


class PoolBuild:
    """A pool holding a workload's adapters.

    resident: adapter ids paged in at build time (default: all).
    n_pages: pool size (default: exactly the pages of all adapters)."""

    def __init__(self, w: W.Workload, resident=None, n_pages=None, max_tokens=None,
                 pagein_mode=G.SLORA_PAGEIN_KERNEL, threads=8, chunk=256):
        import torch
        self.w = w
        d_in = [p.d_in for p in w.projs]
        d_out = [p.d_out for p in w.projs]
        max_rank = int(w.ranks.max())
        desc = G.make_desc(w.dtype, d_in, d_out, w.n_adapters, max_rank, 1, w.page_elems, 0)
        self.need = np.array([G.slora_pages_for_rank(desc, int(r)) for r in w.ranks], np.int64)
        if n_pages is None:
            n_pages = int(self.need.sum())
        self.pool = G.Pool(w.dtype, d_in, d_out, w.n_adapters, max_rank,
                           max_tokens or max(w.T, 1), w.page_elems, n_pages, pagein_mode)
        if w.shuffle_pages:
            G.slora_pool_set_page_order(self.pool.h, W.page_order(n_pages, w.seed))
        # host weights: own data for touched adapters, one pinned filler per rank
        touched = set(w.touched().tolist()) | set(int(a) for a in w.extra_touched)
        w.prefetch_adapters(sorted(touched), threads)
        self.host = {}
        fill = {}
        for a in range(w.n_adapters):
            r = int(w.ranks[a])
            if a in touched:
                A_t, B = w.adapter(a)
                self.host[a] = ([pinned(x) for x in A_t], [pinned(x) for x in B])
            else:
                if r not in fill:
                    A_t, B = w.adapter(a)
                    fill[r] = ([pinned(x) for x in A_t], [pinned(x) for x in B])
                self.host[a] = fill[r]
            hA, hB = self.host[a]
            G.slora_adapter_register(self.pool.h, a, r, w.alpha, hA, hB)
        ids = list(range(w.n_adapters)) if resident is None else [int(a) for a in resident]
        side = torch.cuda.Stream()
        for i in range(0, len(ids), chunk):
            G.slora_adapter_page_in(self.pool.h, ids[i:i + chunk], side)
        side.synchronize()

    @property
    def h(self):
        return self.pool.h

    def close(self):
        self.pool.close()


class Tensors:
    """Device x (one per distinct input) and y (one per projection) of a workload."""

    def __init__(self, w: W.Workload, device="cuda"):
        self.w = w
        self.x = {n: to_device(w.x(n), w.dtype, device) for n in w.x_names}
        self.y0 = [to_device(w.y_in(p), w.dtype, device) for p in range(len(w.projs))]
        self.y = [t.clone() for t in self.y0]

    def reset(self):
        for a, b in zip(self.y, self.y0):
            a.copy_(b)

    def args(self, projs=None):
        projs = list(range(len(self.w.projs))) if projs is None else projs
        xs = [self.x[self.w.projs[p].x_name] for p in projs]
        ys = [self.y[p] for p in projs]
        return (projs, xs, [x.stride(0) for x in xs], ys, [y.stride(0) for y in ys])


def oracle_inputs(w: W.Workload, p: int, tokens=None):
    """(x bits, idx, y_in bits, A_t list, B list) of projection p for the oracle,
    restricted to `tokens` (row indices) when given."""
    proj = w.projs[p]
    x = w.x(proj.x_name)
    y = w.y_in(p)
    idx = w.idx
    if tokens is not None:
        x, y, idx = x[tokens], y[tokens], idx[tokens]
    used = set(np.unique(idx[idx >= 0]).tolist())
    A_t = [None] * w.n_adapters
    B = [None] * w.n_adapters
    for a in used:
        At_all, B_all = w.adapter(a)
        A_t[a], B[a] = At_all[p], B_all[p]
    return x, idx, y, A_t, B


def tolerance_check(got_bits: np.ndarray, ref: np.ndarray, dtype):
    """The acceptance bound: |gpu - oracle| <= 1e-2 * max|oracle| + 1e-3,
    elementwise over one projection's output.  Returns (ok, max_err, bound)."""
    got = decode(got_bits, dtype)
    err = np.abs(got - ref)
    bound = 1e-2 * float(np.abs(ref).max(initial=0.0)) + 1e-3
    return bool(np.all(err <= bound)), float(err.max(initial=0.0)), bound


def decode(bits: np.ndarray, dtype) -> np.ndarray:
    bits = np.asarray(bits, np.uint16)
    if dtype == W.F16:
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class MixedStep:
    """The mixed serving step: a decode batch (one adapter per token) and
    prefill requests (one adapter per request) in one batch, with a share of
    the step's adapters cold (in pinned host memory only).

    Pool: sized 1.25x the pages of the step's adapter set; filled at build
    time with the warm adapters plus untouched "filler" adapters until no
    filler fits, so the cold adapters can only come in by LRU eviction.

    step(): page-in of the whole adapter set on a side stream (the cold ones
    are copied, evicting fillers), the compute stream waits on its done event,
    then the fused BGMV delta over the decode tokens and the SGMV over the
    prefill requests.  restore(): evicts the cold set again and pages the
    evicted fillers back (outside any timed region), so that every step pays
    the same page-in."""

    def __init__(self, w: W.Workload, pagein_mode=G.SLORA_PAGEIN_KERNEL, headroom=1.25):
        import torch
        self.w = w
        d_in = [p.d_in for p in w.projs]
        d_out = [p.d_out for p in w.projs]
        desc = G.make_desc(w.dtype, d_in, d_out, w.n_adapters, int(w.ranks.max()), 1, w.page_elems, 0)
        need = np.array([G.slora_pages_for_rank(desc, int(r)) for r in w.ranks], np.int64)
        self.U = w.touched()
        self.warm, self.cold = W.cold_split(w)
        n_pages = int(np.ceil(headroom * need[self.U].sum()))
        used = int(need[self.warm].sum())
        touched = set(self.U.tolist())
        fillers = []
        for a in range(w.n_adapters):
            if a not in touched and need[a] > 0 and used + need[a] <= n_pages:
                fillers.append(a)
                used += int(need[a])
        self.fillers = fillers
        self.n_pages = n_pages
        self.need = need
        self.pb = PoolBuild(w, resident=list(self.warm) + fillers, n_pages=n_pages,
                            pagein_mode=pagein_mode)
        self.ten = Tensors(w)
        nd = w.n_decode
        self.d_idx = torch.from_numpy(w.idx[:nd].copy()).cuda()
        self.n_req = int(w.req_adapter.size)
        self.d_rs = torch.from_numpy(w.req_start).cuda()
        self.d_ra = torch.from_numpy(w.req_adapter).cuda()
        self.ss = torch.zeros(self.n_req + 1, dtype=torch.int32, device="cuda")
        self.sa = torch.zeros(self.n_req, dtype=torch.int32, device="cuda")
        self.S = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.side = torch.cuda.Stream()
        self.ids = self.U.tolist()
        self.ev_start = torch.cuda.Event()
        self.ev_paged = torch.cuda.Event()
        for e in (self.ev_start, self.ev_paged):
            e.record()  # torch creates the CUDA event on first record
        torch.cuda.synchronize()

    @property
    def h(self):
        return self.pb.h

    def cold_bytes(self) -> int:
        """Weight bytes of the cold adapters (what one step copies)."""
        w = self.w
        per_rank = sum(p.d_in + p.d_out for p in w.projs) * 2
        return int(sum(int(w.ranks[a]) * per_rank for a in self.cold))

    def step(self, stream, start=None, paged=None, end=None):
        """start/end: events recorded on `stream` around the step; paged: the
        page-in's done event (created by the caller, timing enabled)."""
        w = self.w
        start = start or self.ev_start
        paged = paged or self.ev_paged
        if not paged.cuda_event:
            paged.record(self.side)
        start.record(stream)
        self.side.wait_event(start)
        G.slora_adapter_page_in(self.h, self.ids, self.side, paged)
        stream.wait_event(paged)
        if w.n_decode:
            G.slora_lora_delta(self.h, *self.ten.args(), self.d_idx, w.n_decode, stream)
        if self.n_req:
            G.slora_build_sgmv_segments(self.h, self.d_rs, self.d_ra, self.n_req, self.ss, self.sa,
                                        self.S, stream)
            G.slora_sgmv(self.h, *self.ten.args(), self.ss, self.sa, self.n_req, w.T, stream)
        if end is not None:
            end.record(stream)

    def restore(self, stream):
        for a in self.cold.tolist():
            G.slora_adapter_evict(self.h, int(a), stream)
        back = [f for f in self.fillers if not G.slora_adapter_is_resident(self.h, f)]
        if back:
            G.slora_adapter_page_in(self.h, back, self.side)
        self.side.synchronize()
        stream.synchronize()

    def close(self):
        self.pb.close()
