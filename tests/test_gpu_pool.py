"""GPU: the page-table gather and the segment builds are bit-exact.

* every page-table gather of a paged-in adapter returns the registered host
  bytes exactly (shuffled pool, mixed ranks, tensors spanning pages, pages
  reused after LRU eviction, both page-in modes);
* the device segment build equals the oracle's stable counting sort bit for
  bit; the request merge equals the oracle's merge;
* bad adapter ids are recorded in the device error word, never trapped.
"""
import numpy as np
import pytest

import gather_lora_paged_b200 as G
import harness as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def _custom(dtype, projs, ranks, idx, page_elems, shuffle, seed):
    return W.Workload(99, "custom", dtype, projs, len(idx), np.asarray(idx, np.int32),
                      np.asarray(ranks, np.int32), page_elems, shuffle, seed,
                      n_decode=len(idx))


def _gather_all(pb, ids):
    w = pb.w
    for a in ids:
        r = int(w.ranks[a])
        if r == 0:
            continue
        A_t, B = w.adapter(a)
        for p, pr in enumerate(w.projs):
            ga = np.empty((r, pr.d_in), np.uint16)
            gb = np.empty((r, pr.d_out), np.uint16)
            G.slora_debug_gather(pb.h, a, p, ga, gb)
            assert np.array_equal(ga, A_t[p]), (a, p, "A")
            assert np.array_equal(gb, B[p]), (a, p, "B")


@pytest.mark.parametrize("mode", [G.SLORA_PAGEIN_KERNEL, G.SLORA_PAGEIN_MEMCPY])
def test_gather_bit_exact_shuffled_mixed_ranks(mode):
    projs = [W.Proj("a", 1024, 2048, "x"), W.Proj("b", 2048, 1024, "x2"),
             W.Proj("c", 1088, 192, "x3")]
    ranks = [0, 8, 16, 24, 40, 64, 8, 16]
    w = _custom(W.BF16, projs, ranks, list(range(8)), 512, True, 7)
    pb = H.PoolBuild(w, pagein_mode=mode)
    _gather_all(pb, range(8))
    s = pb.pool.stats()
    assert s["free_pages"] == 0 and s["resident"] == 8
    pb.close()


def test_gather_after_lru_reuse():
    import torch
    projs = [W.Proj("a", 1024, 1024, "x")]
    ranks = [16] * 6
    w = _custom(W.F16, projs, ranks, list(range(6)), 1024, True, 3)
    # pool fits 3 adapters of rank 16 (32 pages each)
    pb = H.PoolBuild(w, resident=[0, 1, 2], n_pages=96)
    side = torch.cuda.Stream()
    G.slora_adapter_page_in(pb.h, [3, 4], side)      # evicts 0 and 1
    side.synchronize()
    assert [G.slora_adapter_is_resident(pb.h, a) for a in range(6)] == \
        [False, False, True, True, True, False]
    _gather_all(pb, [2, 3, 4])
    G.slora_adapter_page_in(pb.h, [0], side)          # evicts 2 (oldest unpinned)
    side.synchronize()
    _gather_all(pb, [0, 3, 4])
    pb.close()


@pytest.mark.parametrize("T", [0, 1, 7, 300, 1024, 5000])
def test_segments_bit_exact(T):
    import torch
    rng = np.random.default_rng(T)
    n_ad = 50
    projs = [W.Proj("a", 64, 64, "x")]
    ranks = rng.choice([0, 8], n_ad)
    w = _custom(W.F16, projs, ranks, np.zeros(max(T, 1), np.int32), 512, False, 1)
    pb = H.PoolBuild(w, max_tokens=max(T, 1))
    idx = rng.integers(-1, n_ad, T).astype(np.int32)
    hot = rng.random(T) < 0.5          # skew: half the tokens on three adapters
    idx[hot] = rng.integers(0, 3, int(hot.sum()))
    d_idx = torch.from_numpy(idx).cuda() if T else torch.zeros(1, dtype=torch.int32, device="cuda")
    perm = torch.full((max(T, 1),), -7, dtype=torch.int32, device="cuda")
    ss = torch.full((max(T, 1) + 1,), -7, dtype=torch.int32, device="cuda")
    sa = torch.full((max(T, 1),), -7, dtype=torch.int32, device="cuda")
    S = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.slora_build_segments(pb.h, d_idx, T, perm, ss, sa, S)
    torch.cuda.synchronize()
    ref_perm, ref_ss, ref_sa = oracle.segments(idx, n_ad)
    n = int(S.item())
    assert n == len(ref_sa)
    assert np.array_equal(perm.cpu().numpy()[:ref_ss[-1]], ref_perm)
    assert np.array_equal(ss.cpu().numpy()[:n + 1], ref_ss)
    assert np.array_equal(sa.cpu().numpy()[:n], ref_sa)
    assert G.slora_check_device(pb.h)[0] == 0
    pb.close()


def test_segments_flag_bad_ids_and_non_resident():
    import torch
    projs = [W.Proj("a", 64, 64, "x")]
    w = _custom(W.F16, projs, [8, 8, 8], [0], 512, False, 1)
    pb = H.PoolBuild(w, resident=[0, 1], max_tokens=16)
    for bad, code in (([0, 1, 5, 1], 1), ([0, 2, 1], 2)):
        idx = np.array(bad, np.int32)
        d_idx = torch.from_numpy(idx).cuda()
        perm = torch.zeros(16, dtype=torch.int32, device="cuda")
        ss = torch.zeros(17, dtype=torch.int32, device="cuda")
        sa = torch.zeros(16, dtype=torch.int32, device="cuda")
        S = torch.zeros(1, dtype=torch.int32, device="cuda")
        G.slora_build_segments(pb.h, d_idx, len(bad), perm, ss, sa, S)
        st, c, info = G.slora_check_device(pb.h)
        assert st == 6 and c == code and bad[info] in (5, 2)
        ok = np.array([a if a in (0, 1) else -1 for a in bad], np.int32)
        ref_perm, ref_ss, ref_sa = oracle.segments(ok, 3)
        assert np.array_equal(perm.cpu().numpy()[:ref_ss[-1]], ref_perm)
        assert G.slora_check_device(pb.h)[0] == 0      # cleared
    pb.close()


@pytest.mark.parametrize("seed", range(3))
def test_merge_requests_bit_exact(seed):
    import torch
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 3000))
    lens = rng.integers(0, 5, n)
    lens[rng.random(n) < 0.1] = 0
    req_start = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    req_ad = rng.integers(-1, 4, n).astype(np.int32)
    ref_ss, ref_sa = oracle.merge_requests(req_start, req_ad)
    projs = [W.Proj("a", 64, 64, "x")]
    w = _custom(W.F16, projs, [8], [0], 512, False, 1)
    pb = H.PoolBuild(w, max_tokens=4)
    ss = torch.full((n + 1,), -7, dtype=torch.int32, device="cuda")
    sa = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    S = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.slora_build_sgmv_segments(pb.h, torch.from_numpy(req_start).cuda(),
                                torch.from_numpy(req_ad).cuda(), n, ss, sa, S)
    torch.cuda.synchronize()
    m = int(S.item())
    assert m == len(ref_sa)
    assert np.array_equal(ss.cpu().numpy()[:m + 1], ref_ss)
    assert np.array_equal(sa.cpu().numpy()[:m], ref_sa)
    # the tail is padded with empty segments (start = end = T, no adapter)
    assert np.all(ss.cpu().numpy()[m:] == req_start[-1])
    assert np.all(sa.cpu().numpy()[m:] == -1)
    pb.close()
