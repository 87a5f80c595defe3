"""GPU parity of the decode delta with 8-bit adapter pages (e4m3 codes, one
fp32 scale per rank row) against the fp64 8-bit oracle (oracle_lora_delta_q8)
on the same codes and scales.

The codes come from the library's host row quantiser, which the CPU tests pin
bit for bit to the oracle's brute-force quantiser.  Bound per projection output,
as for 16-bit pages: |gpu - oracle| <= 1e-2 * max|oracle| + 1e-3, plus the
tighter arithmetic bound (fp32 accumulation, one rounding of y): the weights
are exact in the kernel (every e4m3 value is an fp16 value) and the scales are
applied in fp32.
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


def _run_and_check(w, tokens=None, tight=True, threads=16, path=G.SLORA_DECODE_AUTO):
    import torch
    pb = H.PoolBuild(w, weight_format=G.SLORA_WEIGHTS_E4M3, decode_path=path)
    ten = H.Tensors(w)
    idx = torch.from_numpy(w.idx).cuda()
    G.slora_lora_delta(pb.h, *ten.args(), idx, w.T)
    torch.cuda.synchronize()
    st, code, info = G.slora_check_device(pb.h)
    assert st == 0, (code, info)
    for p in range(len(w.projs)):
        x, idx_np, y, qa, sa, qb, sb = H.oracle_inputs_q8(pb, p, tokens)
        ref = oracle.lora_delta_q8(w.dtype, x, idx_np, y, w.ranks, np.full(w.n_adapters, w.alpha),
                                   qa, sa, qb, sb, n_threads=threads)
        got = H.from_device(ten.y[p])
        if tokens is not None:
            got = got[tokens]
        ok, err, bound = H.tolerance_check(got, ref, w.dtype)
        assert ok, (w.projs[p].name, err, bound)
        if tight:
            assert _tight_ok(got, ref, w.dtype), w.projs[p].name
    return pb, ten


def _ragged(dtype):
    rng = np.random.default_rng(57)
    projs = [W.Proj("q", 1088, 2112, "a"), W.Proj("k", 1088, 192, "a"),
             W.Proj("o", 2112, 1088, "b"), W.Proj("d", 3136, 1024, "c")]
    ranks = [0, 8, 16, 24, 40, 64, 3, 13, 128]
    counts = [2, 1, 30, 3, 5, 2, 9, 1, 6]
    idx = np.concatenate([np.full(c, a) for a, c in enumerate(counts)] + [np.full(4, -1)])
    idx = idx[rng.permutation(idx.size)].astype(np.int32)
    return W.Workload(94, "q8", dtype, projs, idx.size, idx, np.asarray(ranks, np.int32), 512, True, 9,
                      n_decode=idx.size)


def test_q8_tiny():
    pb, _ = _run_and_check(W.config(0))
    pb.close()


@pytest.mark.parametrize("path", [G.SLORA_DECODE_STREAM, G.SLORA_DECODE_FUSED], ids=["stream", "fused"])
@pytest.mark.parametrize("dtype", [W.F16, W.BF16])
def test_q8_ragged(dtype, path):
    """Ranks not multiples of 8, rank 0, tokens without adapter, rows that
    straddle 512-element pages (1024 codes), shared x across projections, on
    both one-kernel paths; the pages hold exactly the registered codes."""
    w = _ragged(dtype)
    pb, ten = _run_and_check(w, path=path)
    for a in (2, 5, 8):
        cA, _, cB, _ = pb.q8w[a]
        for p in range(len(w.projs)):
            gA = np.zeros(cA[p].shape, np.uint8)
            gB = np.zeros(cB[p].shape, np.uint8)
            G.slora_debug_gather(pb.h, a, p, gA, gB)
            assert np.array_equal(gA, cA[p]) and np.array_equal(gB, cB[p]), (a, p)
    pb.close()


@pytest.mark.parametrize("cfg", [1, 2])
def test_q8_full_size_configs(cfg):
    """The LLaMA-7B (fp16) and LLaMA-13B (bf16, shuffled pool, ranks 8..64)
    decode layers with 8-bit pages, every output element against the oracle;
    the pool takes about half the pages of the 16-bit one."""
    w = W.config(cfg)
    pb, _ = _run_and_check(w, tight=False)
    d16 = G.make_desc(w.dtype, [p.d_in for p in w.projs], [p.d_out for p in w.projs], w.n_adapters,
                      int(w.ranks.max()), 1, w.page_elems, 0)
    d8 = G.make_desc(w.dtype, [p.d_in for p in w.projs], [p.d_out for p in w.projs], w.n_adapters,
                     int(w.ranks.max()), 1, w.page_elems, 0, weight_format=G.SLORA_WEIGHTS_E4M3)
    r = int(w.ranks.max())
    assert G.slora_pages_for_rank(d8, r) <= (G.slora_pages_for_rank(d16, r) + 14) // 2 + 14
    pb.close()


def test_q8_pool_refuses_other_paths():
    import torch
    w = W.config(0)
    pb = H.PoolBuild(w, weight_format=G.SLORA_WEIGHTS_E4M3)
    ten = H.Tensors(w)
    idx = torch.from_numpy(w.idx).cuda()
    t = torch.zeros((w.T, 16), dtype=torch.float32, device="cuda")
    x = ten.x["x"]
    with pytest.raises(G.SloraError) as e:
        G.slora_bgmv_shrink(pb.h, 0, x, x.stride(0), idx, w.T, t, 16)
    assert e.value.status == 9
    A_t, B = w.adapter(0)
    with pytest.raises(G.SloraError) as e:
        G.slora_adapter_register(pb.h, 0, 8, 16.0, [H.pinned(A_t[0])], [H.pinned(B[0])])
    assert e.value.status == 1
    pb.close()
