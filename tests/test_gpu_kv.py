"""KV-cache blocks and adapters in one pool on the GPU (LLaMA-7B decode shapes).

KV blocks take pages by evicting adapters older than the current step; the
caller writes them while a step computes; the next step's page-in evicts
adapters but never KV pages.  Checked: the KV bytes survive bit for bit, every
token's delta matches the fp64 oracle, adapters paged into pages that KV blocks
returned hold their host bytes bit for bit.
"""
import numpy as np
import pytest

import gather_lora_paged_b200 as G
import harness as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def _gather_ok(pb, w, a, projs=(0, 4, 6)):
    hA, hB = pb.host[a]
    for p in projs:
        gA = np.zeros(hA[p].shape, np.uint16)
        gB = np.zeros(hB[p].shape, np.uint16)
        G.slora_debug_gather(pb.h, a, p, gA, gB)
        if not (np.array_equal(gA, hA[p].numpy().view(np.uint16)) and
                np.array_equal(gB, hB[p].numpy().view(np.uint16))):
            return False
    return True


def test_kv_blocks_share_the_pool_with_adapters():
    import torch
    w = W.config(1)
    U = w.touched()
    A_set, B_set = U[:60], U[60:]
    touched = set(U.tolist())
    F = [a for a in range(w.n_adapters) if a not in touched][:40]
    d_in = [p.d_in for p in w.projs]
    d_out = [p.d_out for p in w.projs]
    desc = G.make_desc(w.dtype, d_in, d_out, w.n_adapters, int(w.ranks.max()), 1, w.page_elems, 0)
    per = G.slora_pages_for_rank(desc, 16)
    n_kv = per * 30
    pb = H.PoolBuild(w, resident=F, n_pages=per * (len(A_set) + len(F)) + per * 10)
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    ten = H.Tensors(w)
    in_A = np.isin(w.idx, A_set)
    idx_A = torch.from_numpy(np.where(in_A, w.idx, -1).astype(np.int32)).cuda()
    idx_B = torch.from_numpy(np.where(~in_A, w.idx, -1).astype(np.int32)).cuda()
    ev = [torch.cuda.Event() for _ in range(3)]
    for e in ev:
        e.record()  # torch creates the CUDA event on its first record

    G.slora_adapter_page_in(pb.h, A_set.tolist(), side, ev[0])
    stream.wait_event(ev[0])
    G.slora_lora_delta(pb.h, *ten.args(), idx_A, w.T, stream)
    # KV blocks: 10 adapters' worth of free pages plus 20 fillers evicted
    kv = G.slora_kv_alloc(pb.h, n_kv, stream, ev[1])
    assert len(set(kv)) == n_kv and G.slora_pool_stats(pb.h)["kv_pages"] == n_kv
    assert sum(G.slora_adapter_is_resident(pb.h, a) for a in F) == 20
    assert all(G.slora_adapter_is_resident(pb.h, int(a)) for a in A_set)
    P = w.page_elems
    flat = pb.pool.pages.view(torch.int16)
    pos = (torch.tensor(kv, dtype=torch.int64, device="cuda")[:, None] * P +
           torch.arange(P, device="cuda")[None, :]).reshape(-1)
    pattern = (torch.arange(pos.numel(), device="cuda") * 7919 % 65521 - 32760).to(torch.int16)
    stream.wait_event(ev[1])
    flat[pos] = pattern
    # the next step: its page-in evicts the other fillers and part of A, never KV pages
    G.slora_adapter_page_in(pb.h, B_set.tolist(), side, ev[2])
    stream.wait_event(ev[2])
    G.slora_lora_delta(pb.h, *ten.args(), idx_B, w.T, stream)
    torch.cuda.synchronize()
    st, code, info = G.slora_check_device(pb.h)
    assert st == 0, (code, info)
    assert torch.equal(flat[pos], pattern)
    assert not any(G.slora_adapter_is_resident(pb.h, a) for a in F)
    for p in range(len(w.projs)):
        x, idx, y, A_t, B = H.oracle_inputs(w, p, np.arange(w.T))
        ref = oracle.lora_delta(w.dtype, x, idx, y, w.ranks, np.full(w.n_adapters, w.alpha), A_t, B,
                                n_threads=16)
        ok, err, bound = H.tolerance_check(H.from_device(ten.y[p]), ref, w.dtype)
        assert ok, (w.projs[p].name, err, bound)
    assert all(_gather_ok(pb, w, int(a)) for a in B_set[:5])
    # KV blocks return their pages; fillers come back into them
    chk = flat[pos].to(torch.int32).sum()     # a last read of the KV pages on `stream`
    G.slora_kv_free(pb.h, kv, stream)
    back = F[:25]
    G.slora_adapter_page_in(pb.h, back, side, ev[0])
    stream.wait_event(ev[0])
    torch.cuda.synchronize()
    assert int(chk) == int(pattern.to(torch.int32).sum())
    assert G.slora_pool_stats(pb.h)["kv_pages"] == 0
    assert all(_gather_ok(pb, w, a) for a in back)
    assert G.slora_check_device(pb.h)[0] == 0
    pb.close()
