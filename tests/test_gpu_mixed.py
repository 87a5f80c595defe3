"""The mixed serving step at LLaMA-70B shapes: 1024 decode tokens (BGMV) and
8 prefill requests of 512 tokens (SGMV) in one batch, 2000 registered
adapters of ranks 8..128, 30% of the step's adapters cold.

The cold adapters come in from pinned host memory on a side stream and take
their pages from untouched adapters by LRU eviction; the step's output is
checked against the fp64 oracle on every decode token and on tokens covering
every 128-token tile of the prefill requests, the cold
adapters' pages against their host bytes (bit-exact), and a second step,
after the pool has been put back, must give bit-identical output.
"""
import numpy as np
import pytest

import gather_lora_paged_b200 as G
import harness as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def _sample(w, seed=11):
    """Every decode token (the decode batch is one kernel's whole work), and on
    the prefill side every 128-token tile of every request (two random tokens
    per tile plus each request's first and last token)."""
    dec = np.arange(w.n_decode)
    pre = H.tile_tokens(w.req_start - w.n_decode, w.req_adapter, per_tile=2, seed=seed,
                        offset=w.n_decode)
    return np.unique(np.concatenate([dec, pre]))


@pytest.mark.parametrize("mode", [G.SLORA_PAGEIN_KERNEL, G.SLORA_PAGEIN_MEMCPY])
def test_mixed_step_with_cold_adapters(mode):
    import torch
    w = W.config(4)
    M = H.MixedStep(w, pagein_mode=mode)
    stream = torch.cuda.current_stream()
    s0 = G.slora_pool_stats(M.h)
    assert all(not G.slora_adapter_is_resident(M.h, int(a)) for a in M.cold)
    M.step(stream)
    torch.cuda.synchronize()
    st, code, info = G.slora_check_device(M.h)
    assert st == 0, (code, info)
    s1 = G.slora_pool_stats(M.h)
    assert s1["page_ins"] - s0["page_ins"] == M.cold.size
    assert s1["bytes_paged_in"] - s0["bytes_paged_in"] == M.cold_bytes()
    assert s1["evictions"] > s0["evictions"]          # the cold set had to evict fillers
    assert all(G.slora_adapter_is_resident(M.h, int(a)) for a in M.U)

    # cold adapters' pages hold exactly the registered host bytes
    for a in M.cold[:6].tolist():
        A_t, B = w.adapter(a)
        for p in (0, 4, 6):
            gA = np.zeros_like(A_t[p])
            gB = np.zeros_like(B[p])
            G.slora_debug_gather(M.h, a, p, gA, gB)
            assert np.array_equal(gA, A_t[p]) and np.array_equal(gB, B[p]), (a, p)

    tokens = _sample(w)
    first = [H.from_device(t) for t in M.ten.y]
    for p in range(len(w.projs)):
        x, idx, y, A_t, B = H.oracle_inputs(w, p, tokens)
        ref = oracle.lora_delta(w.dtype, x, idx, y, w.ranks, np.full(w.n_adapters, w.alpha), A_t, B,
                                n_threads=16)
        ok, err, bound = H.tolerance_check(first[p][tokens], ref, w.dtype)
        assert ok, (w.projs[p].name, err, bound)

    # put the pool back (cold evicted, fillers in) and run the step again
    M.restore(stream)
    assert all(not G.slora_adapter_is_resident(M.h, int(a)) for a in M.cold)
    M.ten.reset()
    M.step(stream)
    torch.cuda.synchronize()
    assert G.slora_check_device(M.h)[0] == 0
    for p in range(len(w.projs)):
        assert np.array_equal(first[p], H.from_device(M.ten.y[p])), w.projs[p].name
    M.close()
