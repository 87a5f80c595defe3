"""GPU: slora_lora_delta_noalloc, the decode delta whose scratch lives in the
library's fixed device array (for callers that cannot allocate device memory
where they run it, e.g. while a stream is being captured into a CUDA graph),
gives the same result as slora_lora_delta on the same inputs, on two calls in
a row, and refuses a call whose scratch need exceeds the array.

Kept in its own file, named to be collected last, so that a run stopping at the
first failure has already run every other test.  It builds its own pools, so
it passes alone in a fresh process as well as after the other tests.
"""
import numpy as np
import pytest

import gather_lora_paged_b200 as G
import harness as H
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


@pytest.mark.parametrize("make", [lambda: W.config(0), _ragged_workload], ids=["tiny", "ragged"])
def test_noalloc_matches_lora_delta_twice(make):
    import torch
    w = make()
    pb = H.PoolBuild(w)
    idx = torch.from_numpy(w.idx).cuda()
    ref = H.Tensors(w)
    G.slora_lora_delta(pb.h, *ref.args(), idx, w.T)
    torch.cuda.synchronize()
    expect = [H.from_device(t) for t in ref.y]
    ten = H.Tensors(w)
    for call in range(2):              # two calls in a row share the static scratch
        ten.reset()
        G.slora_lora_delta_noalloc(pb.h, *ten.args(), idx, w.T)
        torch.cuda.synchronize()
        assert G.slora_check_device(pb.h)[0] == 0
        for p in range(len(w.projs)):
            got = H.from_device(ten.y[p])
            ok, err, bound = H.tolerance_check(got, H.decode(expect[p], w.dtype), w.dtype)
            assert ok, (call, w.projs[p].name, err, bound)
    pb.close()


def test_noalloc_rejects_oversized_call():
    import torch
    # 7B decode layer at rank 128: the fp32 partials of 2048 tokens need far
    # more than the fixed array holds
    T = 2048
    projs = W.llama_layer(4096, 11008)
    idx = np.zeros(T, np.int32)
    w = W.Workload(96, "big", W.F16, projs, T, idx, np.array([128], np.int32), 8192, False, 3,
                   n_decode=T)
    d_in = [p.d_in for p in projs]
    d_out = [p.d_out for p in projs]
    pool = G.Pool(w.dtype, d_in, d_out, 1, 128, T, 8192, 1)
    y = torch.zeros((T, 4096), dtype=torch.float16, device="cuda")
    x = torch.zeros((T, 4096), dtype=torch.float16, device="cuda")
    with pytest.raises(G.SloraError) as e:
        G.slora_lora_delta_noalloc(pool.h, [0], [x], [4096], [y], [4096],
                                   torch.from_numpy(idx).cuda(), T)
    assert e.value.status == 1 and "scratch" in e.value.message
    assert G.slora_noalloc_scratch_bytes() == 8 << 20
    pool.close()
