"""Prefetch on the GPU, at LLaMA-7B decode shapes (1000 rank-16 adapters).

The batch's adapters are split into two halves served by two consecutive
steps.  While the first step computes, the second step's adapters are
prefetched on a side stream into a pool so tight that older, untouched
adapters must be evicted for them; the second step's page_in then finds them
resident (hits, no copies) and its compute must see their bytes.  Every token
gets its delta exactly once, checked against the fp64 oracle, and the
prefetched pages hold the registered host bytes bit for bit.
"""
import numpy as np
import pytest

import gather_lora_paged_b200 as G
import harness as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def test_prefetched_adapters_serve_the_next_step():
    import torch
    w = W.config(1)
    ids = w.touched()
    A_set, B_set = ids[::2], ids[1::2]
    touched = set(ids.tolist())
    fill = [a for a in range(w.n_adapters) if a not in touched][:len(B_set)]
    d_in = [p.d_in for p in w.projs]
    d_out = [p.d_out for p in w.projs]
    desc = G.make_desc(w.dtype, d_in, d_out, w.n_adapters, int(w.ranks.max()), 1, w.page_elems, 0)
    per = G.slora_pages_for_rank(desc, 16)
    pb = H.PoolBuild(w, resident=fill, n_pages=per * (len(A_set) + len(B_set)))
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    ten = H.Tensors(w)
    in_A = np.isin(w.idx, A_set)
    idx_A = torch.from_numpy(np.where(in_A, w.idx, -1).astype(np.int32)).cuda()
    idx_B = torch.from_numpy(np.where(~in_A, w.idx, -1).astype(np.int32)).cuda()

    ev_a, ev_b = torch.cuda.Event(), torch.cuda.Event()
    for e in (ev_a, ev_b):
        e.record()  # torch creates the CUDA event on its first record
    G.slora_adapter_page_in(pb.h, A_set.tolist(), side, ev_a)   # fits in the free pages
    stream.wait_event(ev_a)
    G.slora_lora_delta(pb.h, *ten.args(), idx_A, w.T, stream)
    # the next step's adapters come in while this one computes
    s0 = G.slora_pool_stats(pb.h)
    assert G.slora_adapter_prefetch(pb.h, B_set.tolist(), 1 << 40, side) == len(B_set)
    s1 = G.slora_pool_stats(pb.h)
    assert s1["prefetched"] - s0["prefetched"] == len(B_set)
    assert all(G.slora_adapter_is_resident(pb.h, int(a)) for a in A_set)   # the step's set stays
    assert not any(G.slora_adapter_is_resident(pb.h, a) for a in fill)      # older ones made room
    G.slora_adapter_page_in(pb.h, B_set.tolist(), side, ev_b)
    s2 = G.slora_pool_stats(pb.h)
    assert s2["page_ins"] == s1["page_ins"] and s2["hits"] - s1["hits"] == len(B_set)
    stream.wait_event(ev_b)
    G.slora_lora_delta(pb.h, *ten.args(), idx_B, w.T, stream)
    torch.cuda.synchronize()
    st, code, info = G.slora_check_device(pb.h)
    assert st == 0, (code, info)

    tokens = np.arange(w.T)
    for p in range(len(w.projs)):
        x, idx, y, A_t, B = H.oracle_inputs(w, p, tokens)
        ref = oracle.lora_delta(w.dtype, x, idx, y, w.ranks, np.full(w.n_adapters, w.alpha), A_t, B,
                                n_threads=16)
        ok, err, bound = H.tolerance_check(H.from_device(ten.y[p]), ref, w.dtype)
        assert ok, (w.projs[p].name, err, bound)
    for a in B_set[:6].tolist():
        A_t, B = w.adapter(a)
        for p in (0, 4, 6):
            gA = np.zeros_like(A_t[p])
            gB = np.zeros_like(B[p])
            G.slora_debug_gather(pb.h, a, p, gA, gB)
            assert np.array_equal(gA, A_t[p]) and np.array_equal(gB, B[p]), (a, p)
    pb.close()
