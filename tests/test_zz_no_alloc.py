"""GPU: slora_lora_delta_noalloc, the decode delta whose scratch lives in the
library's fixed device array (for callers that cannot allocate device memory
where they run the delta, such as a plug-in whose host framework owns every
device allocation), checked on two calls in a row against the fp64 oracle
(the acceptance bound and the tighter arithmetic bound) and against
slora_lora_delta on the same inputs (bit for bit); a call whose scratch need
exceeds the array is refused.  Every decode path (the streaming-task kernel, the
persistent kernel, three kernels) runs through it.

Kept in its own file, named to be collected last, so that a run stopping at the
first failure has already run every other test.  It builds its own pools, so
it passes alone in a fresh process as well as after the other tests.
"""
import numpy as np
import pytest

import gather_lora_paged_b200 as G
import harness as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def _ragged_workload():
    rng = np.random.default_rng(41)
    projs = [W.Proj("q", 1088, 2112, "a"), W.Proj("k", 1088, 192, "a"),
             W.Proj("o", 2112, 1088, "b")]
    ranks = [0, 8, 16, 24, 64, 3]
    counts = [2, 1, 20, 3, 5, 6]
    idx = np.concatenate([np.full(c, a) for a, c in enumerate(counts)] + [np.full(3, -1)])
    idx = idx[rng.permutation(idx.size)].astype(np.int32)
    return W.Workload(97, "noalloc", W.BF16, projs, idx.size, idx, np.asarray(ranks, np.int32),
                      512, True, 11, n_decode=idx.size)


def _tight_ok(got_bits, ref, dtype):
    got = H.decode(got_bits, dtype)
    rel = 2.0 ** -8 if dtype == W.F16 else 2.0 ** -7
    bound = rel * np.abs(ref) + 2.0 ** -12 * np.abs(ref).max(initial=0.0) + 1e-6
    return bool(np.all(np.abs(got - ref) <= bound))


@pytest.mark.parametrize("path", [G.SLORA_DECODE_STREAM, G.SLORA_DECODE_FUSED, G.SLORA_DECODE_SPLIT],
                         ids=["stream", "fused", "split"])
@pytest.mark.parametrize("make", [lambda: W.config(0), _ragged_workload], ids=["tiny", "ragged"])
def test_noalloc_matches_oracle_twice(make, path):
    import torch
    w = make()
    pb = H.PoolBuild(w, decode_path=path)
    idx = torch.from_numpy(w.idx).cuda()
    refs = []
    for p in range(len(w.projs)):
        x, idx_np, y, A_t, B = H.oracle_inputs(w, p)
        refs.append(oracle.lora_delta(w.dtype, x, idx_np, y, w.ranks, np.full(w.n_adapters, w.alpha),
                                      A_t, B))
    base = H.Tensors(w)
    G.slora_lora_delta(pb.h, *base.args(), idx, w.T)
    torch.cuda.synchronize()
    assert G.slora_check_device(pb.h)[0] == 0
    expect = [H.from_device(t) for t in base.y]
    ten = H.Tensors(w)
    for call in range(2):              # two calls in a row share the static scratch
        ten.reset()
        G.slora_lora_delta_noalloc(pb.h, *ten.args(), idx, w.T)
        torch.cuda.synchronize()
        assert G.slora_check_device(pb.h)[0] == 0
        for p in range(len(w.projs)):
            got = H.from_device(ten.y[p])
            ok, err, bound = H.tolerance_check(got, refs[p], w.dtype)
            assert ok, (call, w.projs[p].name, err, bound)
            assert _tight_ok(got, refs[p], w.dtype), (call, w.projs[p].name)
            # the same kernels on the same inputs: the same bits as slora_lora_delta
            assert np.array_equal(got, expect[p]), (call, w.projs[p].name)
    pb.close()


def test_noalloc_sizes_scratch_by_the_projections_named():
    """The scratch a call needs grows with the projections it names, not with
    every projection of the pool: one projection of a LLaMA-70B rank-128 pool
    at 2000 tokens fits the array, all seven do not."""
    import torch
    T = 2000
    projs = W.llama_layer(8192, 28672, 1024)
    d_in = [p.d_in for p in projs]
    d_out = [p.d_out for p in projs]
    pool = G.Pool(W.BF16, d_in, d_out, 1, 128, T, 8192, 1)
    idx = torch.full((T,), -1, dtype=torch.int32, device="cuda")   # no adapter: y unchanged
    xs = {n: torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
          for n, d in (("attn", 8192), ("o", 8192), ("mlp", 8192), ("down", 28672))}
    ys = [torch.ones((T, p.d_out), dtype=torch.bfloat16, device="cuda") for p in projs]
    G.slora_lora_delta_noalloc(pool.h, [0], [xs["attn"]], [8192], [ys[0]], [ys[0].stride(0)], idx, T)
    torch.cuda.synchronize()
    assert bool((ys[0] == 1).all())
    xa = [xs[p.x_name] for p in projs]
    with pytest.raises(G.SloraError) as e:
        G.slora_lora_delta_noalloc(pool.h, list(range(7)), xa, [x.stride(0) for x in xa], ys,
                                   [y.stride(0) for y in ys], idx, T)
    assert e.value.status == 1 and "scratch" in e.value.message
    pool.close()


def test_noalloc_rejects_oversized_call():
    import torch
    # the down projection of a 7B layer at rank 128: the fp32 partials of
    # 4096 tokens need far more than the fixed array holds
    T = 4096
    projs = W.llama_layer(4096, 11008)
    d_in = [p.d_in for p in projs]
    d_out = [p.d_out for p in projs]
    pool = G.Pool(W.F16, d_in, d_out, 1, 128, T, 8192, 1)
    y = torch.zeros((T, 4096), dtype=torch.float16, device="cuda")
    x = torch.zeros((T, 11008), dtype=torch.float16, device="cuda")
    idx = torch.zeros(T, dtype=torch.int32, device="cuda")
    with pytest.raises(G.SloraError) as e:
        G.slora_lora_delta_noalloc(pool.h, [6], [x], [11008], [y], [4096], idx, T)
    assert e.value.status == 1 and "scratch" in e.value.message
    assert G.slora_noalloc_scratch_bytes() == 8 << 20
    pool.close()
