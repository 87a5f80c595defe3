"""GPU parity of the whole prefill linear layer with its LoRA delta in one
tensor-core kernel, y = x . W0 + (alpha/r) (x . A) . B per segment, against
the fp64 oracle (oracle_linear + the delta oracle).

Bound per projection output, as for the other paths:
|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3, plus the tighter arithmetic
bound (fp32 accumulation in tensor memory, one rounding of y; t enters the
tensor cores as two 16-bit halves).
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


def _seg_workload(dtype, projs, ranks, seg_lens, seg_ads, page_elems=1024, seed=19):
    idx = np.concatenate([np.full(n, a, np.int32) for n, a in zip(seg_lens, seg_ads)] +
                         [np.zeros(0, np.int32)])
    req_start = np.concatenate([[0], np.cumsum(seg_lens)]).astype(np.int32)
    return W.Workload(93, "linear", dtype, projs, int(idx.size), idx, np.asarray(ranks, np.int32),
                      page_elems, True, seed, req_start=req_start,
                      req_adapter=np.asarray(seg_ads, np.int32), n_decode=0)


def _run(pb, w, ten, w0s, seg_start=None, seg_ad=None):
    import torch
    ss = torch.from_numpy(np.asarray(w.req_start if seg_start is None else seg_start, np.int32)).cuda()
    sa = torch.from_numpy(np.asarray(w.req_adapter if seg_ad is None else seg_ad, np.int32)).cuda()
    projs, xs, ldx, ys, ldy = ten.args()
    G.slora_sgmv_linear(pb.h, projs, xs, ldx, w0s, [t.stride(0) for t in w0s], ys, ldy, ss, sa,
                        int(sa.numel()), w.T)
    torch.cuda.synchronize()
    st, code, info = G.slora_check_device(pb.h)
    assert st == 0, (code, info)


def _check(w, ten, tokens=None, tight=True, threads=16):
    for p in range(len(w.projs)):
        x, idx, _, A_t, B = H.oracle_inputs(w, p, tokens)
        ref = oracle.linear_lora(w.dtype, x, w.w0(p), idx, w.ranks, np.full(w.n_adapters, w.alpha), A_t, B,
                                 n_threads=threads)
        got = H.from_device(ten.y[p])
        if tokens is not None:
            got = got[tokens]
        ok, err, bound = H.tolerance_check(got, ref, w.dtype)
        assert ok, (w.projs[p].name, err, bound)
        if tight:
            assert _tight_ok(got, ref, w.dtype), w.projs[p].name


@pytest.mark.parametrize("dtype", [W.BF16, W.F16])
def test_linear_ragged_segments(dtype):
    """Tiles of 1, 127, 128, 129, 300 tokens, an empty segment, segments
    without adapter and with a rank-0 adapter, ranks 8..64 (not all multiples
    of 16), projections sharing x and one that does not, d_out not a multiple
    of 128; every output element against the oracle."""
    projs = [W.Proj("q", 512, 320, "a"), W.Proj("k", 512, 192, "a"), W.Proj("o", 384, 1088, "b")]
    ranks = [8, 16, 24, 64, 40, 0]
    seg_lens = [1, 127, 128, 129, 300, 0, 5, 64, 33]
    seg_ads = [0, 1, 2, 3, 4, 1, -1, 5, 4]
    w = _seg_workload(dtype, projs, ranks, seg_lens, seg_ads, page_elems=512)
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    w0s = [H.to_device(w.w0(p), dtype) for p in range(len(projs))]
    _run(pb, w, ten, w0s)
    _check(w, ten)
    first = [H.from_device(t) for t in ten.y]
    ten.reset()
    _run(pb, w, ten, w0s)                     # deterministic
    assert all(np.array_equal(a, H.from_device(b)) for a, b in zip(first, ten.y))
    pb.close()


def test_linear_without_adapters_is_the_base_gemm():
    """Every segment without adapter: y = x . W0, against the oracle and
    against torch's fp64 matmul on the CPU."""
    import torch
    projs = [W.Proj("q", 1024, 640, "a")]
    w = _seg_workload(W.BF16, projs, [16], [200, 57], [-1, -1])
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    w0s = [H.to_device(w.w0(0), W.BF16)]
    _run(pb, w, ten, w0s)
    _check(w, ten)
    X = torch.from_numpy(H.decode(w.x("a"), W.BF16))
    ref = (X @ torch.from_numpy(H.decode(w.w0(0), W.BF16)).T).numpy()
    assert H.tolerance_check(H.from_device(ten.y[0]), ref, W.BF16)[0]
    pb.close()


def test_linear_bad_segments_are_reported():
    import torch
    projs = [W.Proj("q", 256, 256, "a")]
    w = _seg_workload(W.BF16, projs, [16, 16], [10, 10], [0, 1])
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    w0s = [H.to_device(w.w0(0), W.BF16)]
    ss = torch.tensor([0, 10, 25], dtype=torch.int32, device="cuda")   # runs past T = 20
    sa = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    projs_, xs, ldx, ys, ldy = ten.args()
    G.slora_sgmv_linear(pb.h, projs_, xs, ldx, w0s, [256], ys, ldy, ss, sa, 2, w.T)
    st, code, info = G.slora_check_device(pb.h)
    assert st == 6 and code == 6 and info == 1
    pb.close()


def test_linear_prefill_config_every_tile():
    """The LLaMA-7B prefill workload (32 requests of 64..1024 tokens, 64
    adapters of rank 16/32/64, bf16, 7 projections with random-init base
    weights) against the oracle on a random token of every 128-token tile of
    every merged segment (the kernel's tiles) and both ends of each."""
    w = W.config(3)
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    w0s = [H.to_device(w.w0(p), w.dtype) for p in range(len(w.projs))]
    # merged segments (neighbouring requests on one adapter), covering [0, T)
    rs, ra = w.req_start, w.req_adapter
    ss, sa = [0], []
    for q in range(ra.size):
        if sa and sa[-1] == ra[q]:
            ss[-1] = int(rs[q + 1])
        else:
            sa.append(int(ra[q]))
            ss.append(int(rs[q + 1]))
    _run(pb, w, ten, w0s, ss, sa)
    rng = np.random.default_rng(5)
    tokens = set()
    for b, e in zip(ss[:-1], ss[1:]):          # the kernel's tiles: 128 tokens from each segment start
        tokens.update((b, e - 1))
        tokens.update(int(rng.integers(t0, min(t0 + 128, e))) for t0 in range(b, e, 128))
    tokens = np.array(sorted(tokens))
    _check(w, ten, tokens=tokens, tight=True, threads=32)
    pb.close()
