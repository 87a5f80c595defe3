"""GPU parity of the tensor-core SGMV prefill path with the fp64 oracle.

Segments are contiguous token ranges with one adapter each; the oracle sees
the same thing as a per-token adapter index.  Bound per projection output, as
for the decode path: |gpu - oracle| <= 1e-2 * max|oracle| + 1e-3, plus the
tighter arithmetic bound on the small cases (the rank-r intermediate enters
the tensor cores as two 16-bit halves, so it keeps ~2x16 bits).
"""
import numpy as np
import pytest

import gather_lora_paged_b200 as G
import harness as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def _tight_ok(got_bits, ref, dtype):
    got = H.decode(got_bits, dtype)
    rel = 2.0 ** -8 if dtype == W.F16 else 2.0 ** -7
    bound = rel * np.abs(ref) + 2.0 ** -12 * np.abs(ref).max(initial=0.0) + 1e-6
    return bool(np.all(np.abs(got - ref) <= bound))


def _segment_workload(dtype, projs, ranks, seg_lens, seg_ads, page_elems=1024, seed=13):
    idx = np.concatenate([np.full(n, a, np.int32) for n, a in zip(seg_lens, seg_ads)] +
                         [np.zeros(0, np.int32)])
    req_start = np.concatenate([[0], np.cumsum(seg_lens)]).astype(np.int32)
    return W.Workload(95, "sgmv", dtype, projs, int(idx.size), idx, np.asarray(ranks, np.int32),
                      page_elems, True, seed, req_start=req_start,
                      req_adapter=np.asarray(seg_ads, np.int32), n_decode=0)


def _run_sgmv(pb, ten, w, seg_start, seg_ad):
    import torch
    ss = torch.from_numpy(np.asarray(seg_start, np.int32)).cuda()
    sa = torch.from_numpy(np.asarray(seg_ad, np.int32)).cuda()
    G.slora_sgmv(pb.h, *ten.args(), ss, sa, len(seg_ad), w.T)
    torch.cuda.synchronize()
    st, code, info = G.slora_check_device(pb.h)
    assert st == 0, (code, info)


def _check(w, ten, tokens=None, tight=True, threads=16):
    for p in range(len(w.projs)):
        x, idx, y, A_t, B = H.oracle_inputs(w, p, tokens)
        ref = oracle.lora_delta(w.dtype, x, idx, y, w.ranks, np.full(w.n_adapters, w.alpha), A_t, B,
                                n_threads=threads)
        got = H.from_device(ten.y[p])
        if tokens is not None:
            got = got[tokens]
        ok, err, bound = H.tolerance_check(got, ref, w.dtype)
        assert ok, (w.projs[p].name, err, bound)
        if tight:
            assert _tight_ok(got, ref, w.dtype), w.projs[p].name


@pytest.mark.parametrize("dtype", [W.BF16, W.F16])
def test_sgmv_ragged_segments(dtype):
    """Tiles with 1, 127, 128, 129, 300 tokens, an empty segment, a segment
    without adapter, ranks 8..128 (not all multiples of 16), projections that
    share x (one group) and one that does not; d_out not a multiple of 256."""
    projs = [W.Proj("q", 512, 320, "a"), W.Proj("k", 512, 192, "a"), W.Proj("o", 384, 1088, "b")]
    ranks = [8, 16, 24, 64, 128, 0, 40]
    seg_lens = [1, 127, 128, 129, 300, 0, 5, 64, 33]
    seg_ads = [0, 1, 2, 3, 4, 1, -1, 6, 5]
    w = _segment_workload(dtype, projs, ranks, seg_lens, seg_ads, page_elems=512)
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    _run_sgmv(pb, ten, w, w.req_start, w.req_adapter)
    _check(w, ten)
    # deterministic
    first = [H.from_device(t) for t in ten.y]
    ten.reset()
    _run_sgmv(pb, ten, w, w.req_start, w.req_adapter)
    assert all(np.array_equal(a, H.from_device(b)) for a, b in zip(first, ten.y))
    pb.close()


def test_sgmv_merged_requests_match_unmerged():
    """Neighbouring requests on one adapter, merged by the device request
    merge, give the same result as the unmerged request list."""
    import torch
    projs = [W.Proj("q", 256, 256, "a")]
    seg_lens = [100, 60, 200, 7, 7]
    seg_ads = [1, 1, 0, 0, 1]
    w = _segment_workload(W.BF16, projs, [16, 32], seg_lens, seg_ads)
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    _run_sgmv(pb, ten, w, w.req_start, w.req_adapter)
    unmerged = H.from_device(ten.y[0])
    ten.reset()
    n = len(seg_ads)
    ss = torch.zeros(n + 1, dtype=torch.int32, device="cuda")
    sa = torch.zeros(n, dtype=torch.int32, device="cuda")
    S = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.slora_build_sgmv_segments(pb.h, torch.from_numpy(w.req_start).cuda(),
                                torch.from_numpy(w.req_adapter).cuda(), n, ss, sa, S)
    torch.cuda.synchronize()
    m = int(S.item())
    assert m == 3
    G.slora_sgmv(pb.h, *ten.args(), ss, sa, m, w.T)
    torch.cuda.synchronize()
    assert np.array_equal(H.from_device(ten.y[0]), unmerged)
    _check(w, ten)
    pb.close()


def test_sgmv_bad_segment_is_skipped():
    import torch
    projs = [W.Proj("q", 256, 256, "a")]
    w = _segment_workload(W.BF16, projs, [16, 16], [10, 10], [0, 1])
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    ss = torch.tensor([0, 10, 25], dtype=torch.int32, device="cuda")   # second runs past T = 20
    sa = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    G.slora_sgmv(pb.h, *ten.args(), ss, sa, 2, w.T)
    st, code, info = G.slora_check_device(pb.h)
    assert st == 6 and code == 6 and info == 1
    got = H.from_device(ten.y[0])
    assert np.array_equal(got[10:], w.y_in(0)[10:])
    pb.close()


def test_sgmv_prefill_config_every_tile():
    """The LLaMA-7B prefill workload (32 requests of 64..1024 tokens, 64
    adapters of rank 16/32/64, bf16) in the launch configuration bench.py
    times; every projection against the oracle on tokens that touch every
    128-token tile of every request and merged segment (two random tokens per
    tile, plus each one's first and last token) and every 128-token window."""
    w = W.config(3)
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    _run_sgmv(pb, ten, w, w.req_start, w.req_adapter)
    tokens = H.tile_tokens(w.req_start, w.req_adapter, per_tile=2, seed=7)
    assert tokens.size > 300
    _check(w, ten, tokens=tokens, tight=True, threads=32)
    pb.close()
