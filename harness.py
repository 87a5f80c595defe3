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


def pinned_bytes(codes: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).pin_memory()


class PoolBuild:
    """A pool holding a workload's adapters.

    resident: adapter ids paged in at build time (default: all).
    n_pages: pool size (default: exactly the pages of all adapters)."""

    def __init__(self, w: W.Workload, resident=None, n_pages=None, max_tokens=None,
                 pagein_mode=G.SLORA_PAGEIN_KERNEL, threads=8, chunk=256,
                 decode_path=G.SLORA_DECODE_AUTO, weight_format=G.SLORA_WEIGHTS_16):
        import torch
        self.w = w
        self.q8 = weight_format == G.SLORA_WEIGHTS_E4M3
        d_in = [p.d_in for p in w.projs]
        d_out = [p.d_out for p in w.projs]
        max_rank = int(w.ranks.max())
        desc = G.make_desc(w.dtype, d_in, d_out, w.n_adapters, max_rank, 1, w.page_elems, 0,
                           weight_format=weight_format)
        self.need = np.array([G.slora_pages_for_rank(desc, int(r)) for r in w.ranks], np.int64)
        if n_pages is None:
            n_pages = int(self.need.sum())
        self.pool = G.Pool(w.dtype, d_in, d_out, w.n_adapters, max_rank,
                           max_tokens or max(w.T, 1), w.page_elems, n_pages, pagein_mode,
                           decode_path=decode_path, weight_format=weight_format)
        if w.shuffle_pages:
            G.slora_pool_set_page_order(self.pool.h, W.page_order(n_pages, w.seed))
        # host weights: own data for touched adapters, one pinned filler per rank
        touched = set(w.touched().tolist()) | set(int(a) for a in w.extra_touched)
        w.prefetch_adapters(sorted(touched), threads)
        self.host = {}
        fill = {}
        self.q8w = {}  # e4m3 pools: adapter -> (codes A_t, scales A_t, codes B, scales B) per projection
        store, qstore = {}, {}
        for a in range(w.n_adapters):
            r = int(w.ranks[a])
            key = a if a in touched else ("fill", r)
            if key not in store:
                A_t, B = w.adapter(a)
                if self.q8:
                    qa = [G.slora_quantize_e4m3_rows(w.dtype, x) for x in A_t]
                    qb = [G.slora_quantize_e4m3_rows(w.dtype, x) for x in B]
                    qstore[key] = ([c for c, _ in qa], [s for _, s in qa], [c for c, _ in qb],
                                   [s for _, s in qb])
                    store[key] = ([pinned_bytes(c) for c, _ in qa], [pinned_bytes(c) for c, _ in qb])
                else:
                    store[key] = ([pinned(x) for x in A_t], [pinned(x) for x in B])
            self.host[a] = store[key]
            hA, hB = store[key]
            if self.q8:
                self.q8w[a] = qstore[key]
                cA, sA, cB, sB = self.q8w[a]
                G.slora_adapter_register_e4m3(self.pool.h, a, r, w.alpha, hA, sA, hB, sB)
            else:
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


def oracle_inputs_q8(pb: PoolBuild, p: int, tokens=None):
    """(x bits, idx, y_in bits, codes A_t, scales A_t, codes B, scales B) of
    projection p for the 8-bit oracle, with the codes and scales the pool
    holds; restricted to `tokens` when given."""
    w = pb.w
    x, idx, y, _, _ = oracle_inputs(w, p, tokens)
    n = w.n_adapters
    qa, sa, qb, sb = [None] * n, [None] * n, [None] * n, [None] * n
    for a in set(np.unique(idx[idx >= 0]).tolist()):
        cA, sA, cB, sB = pb.q8w[a]
        qa[a], sa[a], qb[a], sb[a] = cA[p], sA[p], cB[p], sB[p]
    return x, idx, y, qa, sa, qb, sb


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


def tile_tokens(req_start, req_adapter, tile=128, per_tile=1, seed=0, offset=0):
    """Token indices that touch every tile the prefill path computes: for each
    request and for each merged segment (neighbouring requests on one adapter),
    its first and last token and `per_tile` random tokens of every `tile`-token
    tile counted from its start; plus one random token of every `tile`-token
    window of the whole range.  `offset` is added to every index."""
    rng = np.random.default_rng(seed)
    rs = np.asarray(req_start, np.int64)
    ra = np.asarray(req_adapter)
    spans = [(int(rs[q]), int(rs[q + 1])) for q in range(ra.size) if rs[q + 1] > rs[q]]
    q = 0
    while q < ra.size:  # merged segments
        e = q
        while e + 1 < ra.size and ra[e + 1] == ra[q]:
            e += 1
        if rs[e + 1] > rs[q]:
            spans.append((int(rs[q]), int(rs[e + 1])))
        q = e + 1
    lo, hi = int(rs[0]), int(rs[-1])
    spans += [(b, min(b + tile, hi)) for b in range(lo, hi, tile)]
    out = set()
    for b, e in spans:
        out.update((b, e - 1))
        for t0 in range(b, e, tile):
            t1 = min(t0 + tile, e)
            out.update(int(v) for v in rng.integers(t0, t1, size=per_tile))
    return np.array(sorted(out), np.int64) + offset


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
