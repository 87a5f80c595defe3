"""GPU parity of the decode path (segment build + paged shrink + expand) with
the fp64 oracle, on the same seeded inputs.  Every decode path is checked: the
one kernel of streaming tasks (SLORA_DECODE_STREAM, the default for 17..1024
tokens), the persistent bulk-copy kernel (SLORA_DECODE_FUSED) and the
three-kernel path (SLORA_DECODE_SPLIT, every batch above 1024 tokens); the
last two must agree bit for bit (same fp32 partials, same summation order),
and every path must give the same bits on a repeated call.

Acceptance bound, per projection output y_out:
    |gpu - oracle| <= 1e-2 * max|oracle| + 1e-3   (elementwise)
A second, tighter bound derived from the arithmetic is also checked on the
small cases: the kernel accumulates in fp32 and rounds y once, so the error is
half an output ulp plus fp32 accumulation noise, well under
2^-8 |oracle| + 2^-12 max|oracle| (fp16) or 2^-7 |oracle| + 2^-12 max|oracle|
(bf16).  A dropped term or a wrong index fails it by orders of magnitude.
"""
import numpy as np
import pytest

import gather_lora_paged_b200 as G
import harness as H
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def _custom(dtype, projs, ranks, idx, page_elems=1024, shuffle=True, seed=5):
    return W.Workload(98, "custom", dtype, projs, len(idx), np.asarray(idx, np.int32),
                      np.asarray(ranks, np.int32), page_elems, shuffle, seed,
                      n_decode=len(idx))


def _tight_ok(got_bits, ref, dtype):
    got = H.decode(got_bits, dtype)
    rel = 2.0 ** -8 if dtype == W.F16 else 2.0 ** -7
    bound = rel * np.abs(ref) + 2.0 ** -12 * np.abs(ref).max(initial=0.0) + 1e-6
    return bool(np.all(np.abs(got - ref) <= bound))


def _check_all(w, ten, tokens=None, tight=False, threads=8):
    for p in range(len(w.projs)):
        x, idx, y, A_t, B = H.oracle_inputs(w, p, tokens)
        ref = oracle.lora_delta(w.dtype, x, idx, y, w.ranks, np.full(w.n_adapters, w.alpha),
                                A_t, B, n_threads=threads)
        got = H.from_device(ten.y[p])
        if tokens is not None:
            got = got[tokens]
        ok, err, bound = H.tolerance_check(got, ref, w.dtype)
        assert ok, (w.projs[p].name, err, bound)
        if tight:
            assert _tight_ok(got, ref, w.dtype), w.projs[p].name


def _run_delta(pb, ten, w):
    import torch
    idx = torch.from_numpy(w.idx).cuda()
    G.slora_lora_delta(pb.h, *ten.args(), idx, w.T)
    torch.cuda.synchronize()
    st, code, info = G.slora_check_device(pb.h)
    assert st == 0, (code, info)


def test_tiny_config():
    w = W.config(0)
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    _run_delta(pb, ten, w)
    _check_all(w, ten, tight=True)
    pb.close()


PATHS = [G.SLORA_DECODE_FUSED, G.SLORA_DECODE_SPLIT]
ALL_PATHS = [G.SLORA_DECODE_STREAM, G.SLORA_DECODE_FUSED, G.SLORA_DECODE_SPLIT]
ALL_IDS = ["stream", "fused", "split"]


@pytest.mark.parametrize("path", ALL_PATHS, ids=ALL_IDS)
@pytest.mark.parametrize("dtype", [W.F16, W.BF16])
def test_ragged_mixed(dtype, path):
    """Ragged everything: d_in not a multiple of the 1024-element chunk nor of
    256, ranks not multiples of 8, rank 0, tokens without adapter, segments of
    1, 2, 3, 4, 5..40 tokens (all token classes), shared x across projections."""
    rng = np.random.default_rng(17)
    projs = [W.Proj("q", 1088, 2112, "a"), W.Proj("k", 1088, 192, "a"),
             W.Proj("o", 2112, 1088, "b"), W.Proj("d", 3136, 1024, "c")]
    ranks = [0, 8, 16, 24, 40, 64, 3, 13, 8, 16, 32, 128]
    counts = [2, 1, 40, 3, 5, 2, 9, 1, 4, 0, 7, 6]
    idx = np.concatenate([np.full(c, a) for a, c in enumerate(counts)] + [np.full(5, -1)])
    idx = idx[rng.permutation(idx.size)].astype(np.int32)
    w = _custom(dtype, projs, ranks, idx, page_elems=512)
    pb = H.PoolBuild(w, decode_path=path)
    ten = H.Tensors(w)
    _run_delta(pb, ten, w)
    _check_all(w, ten, tight=True)
    # deterministic: a second run from the same y_in is bit-identical
    first = [H.from_device(t) for t in ten.y]
    ten.reset()
    _run_delta(pb, ten, w)
    assert all(np.array_equal(a, H.from_device(b)) for a, b in zip(first, ten.y))
    pb.close()


def test_unfused_shrink_expand():
    import torch
    rng = np.random.default_rng(3)
    projs = [W.Proj("q", 2048, 1024, "a")]
    ranks = [8, 16, 64, 0]
    idx = rng.integers(-1, 4, 45).astype(np.int32)
    w = _custom(W.BF16, projs, ranks, idx)
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    d_idx = torch.from_numpy(idx).cuda()
    ldt = 64
    t = torch.full((w.T, ldt), float("nan"), dtype=torch.float32, device="cuda")
    x = ten.x["a"]
    G.slora_bgmv_shrink(pb.h, 0, x, x.stride(0), d_idx, w.T, t, ldt)
    torch.cuda.synchronize()
    # t against fp64 x . A (through the oracle with B = I and alpha = r)
    X = H.decode(w.x("a"), w.dtype)
    tt = t.cpu().numpy().astype(np.float64)
    for i, a in enumerate(idx):
        r = ranks[a] if a >= 0 else 0
        if r:
            ref = X[i] @ H.decode(w.adapter(a)[0][0], w.dtype).T
            assert np.allclose(tt[i, :r], ref, rtol=1e-5, atol=1e-5 * np.abs(ref).max())
        assert np.all(tt[i, r:] == 0)
    G.slora_bgmv_expand(pb.h, 0, t, ldt, d_idx, w.T, ten.y[0], ten.y[0].stride(0))
    torch.cuda.synchronize()
    _check_all(w, ten, tight=True)
    pb.close()


@pytest.mark.parametrize("T", [1, 5, 16])
def test_small_batch_token_path(T):
    """Batches of up to 16 tokens run as one CTA per token on 16-bit pools
    (the default path): ranks up to 128, rank 0, tokens without adapter and
    tokens sharing one, projections sharing x, rows across 512-element pages;
    every element against the oracle at the tight bound."""
    import torch
    rng = np.random.default_rng(300 + T)
    projs = [W.Proj("q", 1088, 2112, "a"), W.Proj("k", 1088, 192, "a"), W.Proj("d", 3136, 1024, "c")]
    ranks = [8, 128, 0, 24, 3]
    idx = rng.integers(-1, len(ranks), T).astype(np.int32)
    if T > 2:
        idx[1] = idx[0] = 1                      # two tokens on the rank-128 adapter
    w = _custom(W.BF16, projs, ranks, idx, page_elems=512)
    pb = H.PoolBuild(w)
    assert G.slora_decode_kernels(pb.h, T) == 1
    ten = H.Tensors(w)
    _run_delta(pb, ten, w)
    _check_all(w, ten, tight=True)
    pb.close()


@pytest.mark.parametrize("path", [G.SLORA_DECODE_AUTO] + ALL_PATHS, ids=["auto"] + ALL_IDS)
@pytest.mark.parametrize("T", [4, 40])
def test_degenerate_batches(T, path):
    import torch
    projs = [W.Proj("q", 1024, 1024, "a")]
    idx = np.resize(np.array([-1, -1, 1, -1], np.int32), T)
    w = _custom(W.F16, projs, [16, 0], idx)
    pb = H.PoolBuild(w, decode_path=path)
    ten = H.Tensors(w)
    for _ in range(2):               # no adapter / rank 0 only: y unchanged
        _run_delta(pb, ten, w)
        assert np.array_equal(H.from_device(ten.y[0]), w.y_in(0))
    idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.slora_lora_delta(pb.h, *ten.args(), idx, 0)     # T = 0 is a no-op
    torch.cuda.synchronize()
    assert np.array_equal(H.from_device(ten.y[0]), w.y_in(0))
    pb.close()


def test_single_shared_adapter_is_a_gemm():
    """One adapter for every token: y + s (X A) B, checked against the oracle
    and, independently, against torch fp64 matmuls on the CPU."""
    projs = [W.Proj("q", 2048, 3072, "a")]
    w = _custom(W.BF16, projs, [32], np.zeros(70, np.int32))
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    _run_delta(pb, ten, w)
    _check_all(w, ten, tight=True)
    X = H.decode(w.x("a"), w.dtype)
    A_t, B = w.adapter(0)
    ref = H.decode(w.y_in(0), w.dtype) + (16.0 / 32) * (X @ H.decode(A_t[0], w.dtype).T) @ \
        H.decode(B[0], w.dtype)
    ok, err, bound = H.tolerance_check(H.from_device(ten.y[0]), ref, w.dtype)
    assert ok, (err, bound)
    pb.close()


@pytest.mark.parametrize("T", [4, 24])
def test_bad_token_is_skipped_and_reported(T):
    import torch
    projs = [W.Proj("q", 1024, 1024, "a")]
    idx = np.resize(np.array([0, 1, 1, 0], np.int32), T)
    idx[2] = 7                                        # the one bad id
    w = _custom(W.F16, projs, [16, 8], np.where(idx == 7, 1, idx).astype(np.int32))
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    G.slora_lora_delta(pb.h, *ten.args(), torch.from_numpy(idx).cuda(), T)
    st, code, info = G.slora_check_device(pb.h)
    assert st == 6 and code == 1 and info == 2
    got = H.from_device(ten.y[0])
    assert np.array_equal(got[2], w.y_in(0)[2])       # bad token untouched
    ok_idx = np.where(idx == 7, -1, idx).astype(np.int32)
    x, _, y, A_t, B = H.oracle_inputs(w, 0)
    ref = oracle.lora_delta(w.dtype, x, ok_idx, y, w.ranks, [16.0, 16.0], A_t, B)
    assert H.tolerance_check(got, ref, w.dtype)[0]
    pb.close()


@pytest.mark.parametrize("cfg", [1, 2])
def test_full_size_configs_stream(cfg):
    """The LLaMA-7B and LLaMA-13B decode layers on the streaming-stage kernel
    (the default for the 256-token layer), every output element against the
    oracle, and a repeated call bit-identical."""
    w = W.config(cfg)
    pb = H.PoolBuild(w, decode_path=G.SLORA_DECODE_STREAM)
    assert G.slora_decode_kernels(pb.h, w.T) == 1
    ten = H.Tensors(w)
    _run_delta(pb, ten, w)
    _check_all(w, ten, threads=16)
    first = [H.from_device(t) for t in ten.y]
    ten.reset()
    _run_delta(pb, ten, w)
    assert all(np.array_equal(a, H.from_device(b)) for a, b in zip(first, ten.y))
    pb.close()


@pytest.mark.parametrize("path", [G.SLORA_DECODE_STREAM, G.SLORA_DECODE_FUSED], ids=["stream", "fused"])
@pytest.mark.parametrize("cfg", [1, 2])
def test_one_kernel_many_calls_bit_identical(cfg, path):
    """Forty calls of a one-kernel decode path on one pool, L2 flushed before
    each, give the same bits every time.  The schedule (which CTA takes which
    chunk of tasks, when a stage's copy lands) differs from call to call while
    the arithmetic order does not, so a difference can only come from a race:
    an expand task reading t partials before they are visible, or a bulk copy
    overwriting a stage slot before every read of it has taken its value."""
    import hashlib
    import torch
    w = W.config(cfg)
    pb = H.PoolBuild(w, decode_path=path)
    ten = H.Tensors(w)
    idx = torch.from_numpy(w.idx).cuda()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    digests = []
    for _ in range(40):
        ten.reset()
        flush.zero_()
        G.slora_lora_delta(pb.h, *ten.args(), idx, w.T)
        torch.cuda.synchronize()
        assert G.slora_check_device(pb.h)[0] == 0
        h = hashlib.sha1()
        for t in ten.y:
            h.update(H.from_device(t).tobytes())
        digests.append(h.hexdigest())
    assert len(set(digests)) == 1, [i for i, d in enumerate(digests) if d != digests[0]]
    pb.close()


@pytest.mark.parametrize("cfg", [1, 2])
def test_full_size_configs(cfg):
    """LLaMA-7B (fp16, 1000 adapters r=16, Zipf 1.0, T=256) and LLaMA-13B (bf16,
    2000 adapters r in {8..64}, Zipf 1.2, shuffled pool, T=512) decode layers,
    on the one-kernel path, every output element compared; then the
    three-kernel path on the same pool layout must give the same bits."""
    w = W.config(cfg)
    pb = H.PoolBuild(w, decode_path=G.SLORA_DECODE_FUSED)
    ten = H.Tensors(w)
    _run_delta(pb, ten, w)
    _check_all(w, ten, threads=16)
    fused = [H.from_device(t) for t in ten.y]
    pb.close()
    pb = H.PoolBuild(w, decode_path=G.SLORA_DECODE_SPLIT)
    ten.reset()
    _run_delta(pb, ten, w)
    for p in range(len(w.projs)):
        assert np.array_equal(fused[p], H.from_device(ten.y[p])), w.projs[p].name
    pb.close()


@pytest.mark.parametrize("T", [1, 2, 33, 1024])
def test_fused_matches_split_bitwise(T):
    """Token counts at the edges of the one-kernel path (1 token, 2, a ragged
    33, the 1024-token limit) with Zipf-skewed ids over mixed ranks: the fused
    kernel and the three-kernel path give identical bits, and both match the
    oracle on sampled tokens."""
    rng = np.random.default_rng(100 + T)
    projs = [W.Proj("q", 2048, 2048, "a"), W.Proj("v", 2048, 512, "a"), W.Proj("d", 5504, 2048, "c")]
    n_ad = 64
    ranks = rng.choice(np.array([8, 16, 32, 64, 128, 24], np.int32), n_ad)
    idx = W.zipf_ids(rng, n_ad, 1.1, T)
    if T > 2:
        idx[rng.random(T) < 0.1] = -1
    w = _custom(W.BF16, projs, ranks, idx, page_elems=8192, shuffle=True, seed=31)
    outs = []
    for path in PATHS:
        pb = H.PoolBuild(w, decode_path=path)
        ten = H.Tensors(w)
        _run_delta(pb, ten, w)
        outs.append([H.from_device(t) for t in ten.y])
        pb.close()
    for p in range(len(projs)):
        assert np.array_equal(outs[0][p], outs[1][p]), projs[p].name
    tokens = np.arange(T) if T <= 64 else np.sort(rng.choice(T, 96, replace=False))
    _check_all(w, ten, tokens=tokens, tight=True, threads=16)


@pytest.mark.parametrize("T", [17, 33, 700, 1024])
def test_stream_edges(T):
    """The streaming-task kernel at the edges of its range (17 tokens, a ragged
    33, 700, the 1024-token limit) with Zipf-skewed ids over mixed ranks up to
    128, one hot adapter holding more than one shrink token tile, and rows
    across 8192-element pages: sampled tokens against the oracle at the tight
    bound, and a repeated call bit-identical."""
    rng = np.random.default_rng(500 + T)
    projs = [W.Proj("q", 2048, 2048, "a"), W.Proj("v", 2048, 512, "a"), W.Proj("d", 5504, 2048, "c")]
    n_ad = 64
    ranks = rng.choice(np.array([8, 16, 32, 64, 128, 24, 5], np.int32), n_ad)
    idx = W.zipf_ids(rng, n_ad, 1.1, T)
    idx[: T // 3] = 7                            # a hot adapter: tokens spread over the batch
    idx = idx[rng.permutation(T)]
    if T > 2:
        idx[rng.random(T) < 0.1] = -1
    w = _custom(W.BF16, projs, ranks, idx, page_elems=8192, shuffle=True, seed=37)
    pb = H.PoolBuild(w, decode_path=G.SLORA_DECODE_STREAM)
    ten = H.Tensors(w)
    _run_delta(pb, ten, w)
    first = [H.from_device(t) for t in ten.y]
    tokens = np.arange(T) if T <= 64 else np.sort(rng.choice(T, 96, replace=False))
    _check_all(w, ten, tokens=tokens, tight=True, threads=16)
    ten.reset()
    _run_delta(pb, ten, w)
    assert all(np.array_equal(a, H.from_device(b)) for a, b in zip(first, ten.y))
    pb.close()


def test_many_single_stage_tasks_repeatable():
    """Thousands of rank-8 segments: every shrink and expand task is one stage,
    so the producers run many tasks ahead of the consumers and reuse the x / y
    staging buffers at their fastest rate.  Sampled tokens against the oracle,
    and three repeated calls bit-identical."""
    import torch
    rng = np.random.default_rng(21)
    projs = [W.Proj("a", 1024, 2048, "x"), W.Proj("b", 1024, 1024, "x"), W.Proj("c", 2048, 1024, "z")]
    n_ad, T = 1500, 4096
    idx = W.zipf_ids(rng, n_ad, 0.6, T)
    idx[rng.random(T) < 0.05] = -1
    w = _custom(W.BF16, projs, np.full(n_ad, 8), idx, page_elems=1024, shuffle=True, seed=23)
    pb = H.PoolBuild(w)
    ten = H.Tensors(w)
    d_idx = torch.from_numpy(w.idx).cuda()
    outs = []
    for _ in range(3):
        ten.reset()
        G.slora_lora_delta(pb.h, *ten.args(), d_idx, w.T)
        torch.cuda.synchronize()
        assert G.slora_check_device(pb.h)[0] == 0
        outs.append([H.from_device(t) for t in ten.y])
    for rep in outs[1:]:
        assert all(np.array_equal(a, b) for a, b in zip(outs[0], rep))
    tokens = np.sort(rng.choice(T, size=256, replace=False))
    _check_all(w, ten, tokens=tokens)
    pb.close()
