"""The seeded input recipe (workloads.py) against its own description: the
16-bit rounding, the finite Zipf law of adapter ids, the layer shapes of the
configs, and reproducible, distinct replica batches.  CPU only."""
import numpy as np
import pytest

import workloads as W


def test_bf16_and_f16_rounding_match_reference_conversions():
    import torch
    rng = np.random.default_rng(0)
    v = rng.standard_normal(50000).astype(np.float32) * rng.choice([1e-4, 1, 300], 50000).astype(np.float32)
    # exact ties between two bf16 neighbours (lower 16 bits 0x8000)
    ties = (rng.integers(0, 2 ** 31, 2000, dtype=np.uint32) & np.uint32(0x7FFF0000)) | np.uint32(0x8000)
    v = np.concatenate([v, ties.view(np.float32)])
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(W.to_bits(W.BF16, v), ref)
    assert np.array_equal(W.to_bits(W.F16, v[np.abs(v) < 6e4]),
                          v[np.abs(v) < 6e4].astype(np.float16).view(np.uint16))


def test_zipf_ids_follow_the_finite_zipf_law():
    n_ids, s, n = 40, 1.0, 200000
    ids = W.zipf_ids(np.random.default_rng(1), n_ids, s, n)
    assert ids.min() >= 0 and ids.max() < n_ids
    p = (np.arange(1, n_ids + 1) ** -s)
    p /= p.sum()
    obs = np.bincount(ids, minlength=n_ids)
    chi2 = float(((obs - n * p) ** 2 / (n * p)).sum())
    assert chi2 < 80.0          # 39 degrees of freedom: a right sampler exceeds 80 w.p. 1.2e-4


@pytest.mark.parametrize("cfg,H,M,KV", [(1, 4096, 11008, 4096), (2, 5120, 13824, 5120),
                                        (4, 8192, 28672, 1024)])
def test_layer_shapes(cfg, H, M, KV):
    w = W.config(cfg)
    shapes = {p.name: (p.d_in, p.d_out) for p in w.projs}
    assert shapes == {"q": (H, H), "k": (H, KV), "v": (H, KV), "o": (H, H), "gate": (H, M),
                      "up": (H, M), "down": (M, H)}
    assert len(w.x_names) == 4          # attn input shared by q, k, v; gate and up share theirs


def test_config_batches():
    w1 = W.config(1)
    assert (w1.T, w1.n_adapters, set(w1.ranks.tolist()), w1.dtype) == (256, 1000, {16}, W.F16)
    w3 = W.config(3)
    lens = np.diff(w3.req_start)
    assert w3.T == 18768 and lens.size == 32 and lens.min() >= 64 and lens.max() <= 1024
    assert set(w3.ranks.tolist()) <= {16, 32, 64}
    w4 = W.config(4)
    warm, cold = W.cold_split(w4)
    assert w4.n_decode == 1024 and w4.T == 1024 + 8 * 512
    assert cold.size == round(0.3 * w4.touched().size) and not set(cold) & set(warm)


def test_replicas_are_reproducible_and_distinct():
    a, b, c = W.config(1, replica=1), W.config(1, replica=1), W.config(1, replica=2)
    assert np.array_equal(a.idx, b.idx) and not np.array_equal(a.idx, c.idx)
    assert np.array_equal(a.x("attn"), b.x("attn"))
