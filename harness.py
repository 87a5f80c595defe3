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
