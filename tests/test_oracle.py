"""Pins for the fp64 CPU oracle, against things other than itself.

Each check is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong scale) fails at least one:
  * a hand-derived worked example (tests/golden/tiny_delta.json);
  * the exact fp16/bf16 decoders against numpy's own conversions;
  * brute force with the dense update W_delta = A.B (numpy fp64) on tiny,
    deliberately non-square shapes;
  * closed forms: rank 0 / zero A / zero B / adapter -1 leave y unchanged,
    one shared adapter equals one ordinary GEMM, rank 1 is an outer product,
    A = I gives y + s.x.B;
  * invariants: token permutation, linearity in the scale, additivity over a
    split of the tokens, thread count.
"""
import json
import os

import numpy as np
import pytest

import oracle
from workloads import BF16, F16, to_bits
import workloads as W


def _bits(dtype, a):
    return to_bits(dtype, np.asarray(a, np.float32))


def _dec(dtype, bits):
    bits = np.asarray(bits, np.uint16)
    if dtype == F16:
        return bits.view(np.float16).astype(np.float64)
    with np.errstate(invalid="ignore"):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rand_case(rng, dtype, T, d_in, d_out, ranks, p_none=0.2):
    n_ad = len(ranks)
    x = _bits(dtype, rng.standard_normal((T, d_in)))
    y = _bits(dtype, rng.standard_normal((T, d_out)))
    idx = rng.integers(0, n_ad, T).astype(np.int32)
    idx[rng.random(T) < p_none] = -1
    A_t = [_bits(dtype, rng.standard_normal((r, d_in)) / np.sqrt(d_in)) for r in ranks]
    B = [_bits(dtype, rng.standard_normal((r, d_out)) / np.sqrt(max(r, 1))) for r in ranks]
    return x, y, idx, A_t, B


def _dense_ref(dtype, x, y, idx, ranks, alphas, A_t, B):
    """numpy fp64: y + s_a * x @ (A @ B), with A = A_t.T built explicitly."""
    X = _dec(dtype, x)
    Y = _dec(dtype, y).copy()
    for i, a in enumerate(idx):
        if a < 0 or ranks[a] == 0:
            continue
        A = _dec(dtype, A_t[a]).T          # d_in x r
        Bm = _dec(dtype, B[a])             # r x d_out
        W = A @ Bm                         # dense d_in x d_out update
        Y[i] += (alphas[a] / ranks[a]) * (X[i] @ W)
    return Y


# --------------------------------------------------------------------------
def test_decoders_match_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    for dtype in (F16, BF16):
        ref = _dec(dtype, bits)
        got = oracle.decode16(bits, dtype)
        fin = np.isfinite(ref)
        assert np.array_equal(got[fin], ref[fin])
        assert np.array_equal(np.isnan(got), np.isnan(ref))
        assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_golden_tiny_delta(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "tiny_delta.json")))
    dt = F16
    ranks = np.array(g["ranks"], np.int32)
    A_t = [_bits(dt, np.array(a, np.float32).reshape(r, 3)) for a, r in zip(g["A_t"], ranks)]
    B = [_bits(dt, np.array(b, np.float32).reshape(r, 2)) for b, r in zip(g["B"], ranks)]
    y = oracle.lora_delta(dt, _bits(dt, g["x"]), g["idx"], _bits(dt, g["y_in"]), ranks,
                          np.full(3, g["alpha"]), A_t, B)
    assert np.array_equal(y, np.array(g["y_out"], np.float64))


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_bruteforce_dense_update(dtype, seed):
    rng = np.random.default_rng(seed)
    ranks = [3, 8, 1, 5]
    T, d_in, d_out = 13, 24, 40           # non-square on purpose
    x, y, idx, A_t, B = _rand_case(rng, dtype, T, d_in, d_out, ranks)
    alphas = np.array([16.0, 16.0, 2.0, 16.0])
    got = oracle.lora_delta(dtype, x, idx, y, ranks, alphas, A_t, B)
    ref = _dense_ref(dtype, x, y, idx, ranks, alphas, A_t, B)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_identity_cases():
    rng = np.random.default_rng(7)
    dt = F16
    T, d_in, d_out = 9, 16, 24
    x, y, idx, A_t, B = _rand_case(rng, dt, T, d_in, d_out, [4, 4, 0, 4], p_none=0.3)
    A_t[1] = np.zeros_like(A_t[1])       # zero A
    B[3] = np.zeros_like(B[3])           # zero B
    got = oracle.lora_delta(dt, x, idx, y, [4, 4, 0, 4], np.full(4, 16.0), A_t, B)
    Y = _dec(dt, y)
    for i, a in enumerate(idx):
        if a in (-1, 1, 2, 3):           # none, zero A, rank 0, zero B
            assert np.array_equal(got[i], Y[i])
    assert not np.array_equal(got[idx == 0], Y[idx == 0]) or not np.any(idx == 0)


@pytest.mark.parametrize("dtype", [F16, BF16])
def test_shared_adapter_is_one_gemm(dtype):
    rng = np.random.default_rng(11)
    T, d_in, d_out, r = 17, 32, 48, 8
    x, y, _, A_t, B = _rand_case(rng, dtype, T, d_in, d_out, [r])
    idx = np.zeros(T, np.int32)
    got = oracle.lora_delta(dtype, x, idx, y, [r], [16.0], A_t, B)
    X, Y = _dec(dtype, x), _dec(dtype, y)
    ref = Y + (16.0 / r) * np.matmul(np.matmul(X, _dec(dtype, A_t[0]).T), _dec(dtype, B[0]))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_rank_one_is_outer_product():
    rng = np.random.default_rng(5)
    dt = BF16
    T, d_in, d_out = 6, 20, 12
    x, y, _, A_t, B = _rand_case(rng, dt, T, d_in, d_out, [1])
    idx = np.zeros(T, np.int32)
    got = oracle.lora_delta(dt, x, idx, y, [1], [16.0], A_t, B)
    X, Y = _dec(dt, x), _dec(dt, y)
    a, b = _dec(dt, A_t[0])[0], _dec(dt, B[0])[0]
    ref = Y + 16.0 * np.outer(X @ a, b)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_identity_A_gives_x_B():
    rng = np.random.default_rng(6)
    dt = F16
    T, r, d_out = 5, 8, 16
    x, y, _, _, B = _rand_case(rng, dt, T, r, d_out, [r])
    A_t = [_bits(dt, np.eye(r))]
    got = oracle.lora_delta(dt, x, np.zeros(T, np.int32), y, [r], [16.0], A_t, B)
    ref = _dec(dt, y) + (16.0 / r) * (_dec(dt, x) @ _dec(dt, B[0]))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_invariants_permutation_scale_split_threads():
    rng = np.random.default_rng(21)
    dt = BF16
    ranks = [8, 16, 4]
    T, d_in, d_out = 31, 40, 24
    x, y, idx, A_t, B = _rand_case(rng, dt, T, d_in, d_out, ranks)
    al = np.array([16.0, 16.0, 16.0])
    base = oracle.lora_delta(dt, x, idx, y, ranks, al, A_t, B)
    # token permutation
    perm = rng.permutation(T)
    got = oracle.lora_delta(dt, x[perm], idx[perm], y[perm], ranks, al, A_t, B)
    assert np.array_equal(got, base[perm])
    # linear in the scale (x2 is exact in binary)
    Y = _dec(dt, y)
    got2 = oracle.lora_delta(dt, x, idx, y, ranks, 2 * al, A_t, B)
    assert np.array_equal(got2 - Y, 2 * (base - Y))
    # additivity over a split of the tokens by adapter
    parts = np.zeros_like(base)
    for a in [-1, 0, 1, 2]:
        m = idx == a
        if m.any():
            parts[m] = oracle.lora_delta(dt, x[m], idx[m], y[m], ranks, al, A_t, B)
    assert np.array_equal(parts, base)
    # thread count does not change the result
    assert np.array_equal(oracle.lora_delta(dt, x, idx, y, ranks, al, A_t, B, n_threads=4), base)


def test_rejects_bad_index():
    rng = np.random.default_rng(1)
    x, y, idx, A_t, B = _rand_case(rng, F16, 4, 8, 8, [2])
    with pytest.raises(ValueError):
        oracle.lora_delta(F16, x, np.array([0, 1, 0, 0]), y, [2], [16.0], A_t, B)


# --------------------------------------------------------------------------
def test_segments_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "segments.json")))
    d = g["decode"]
    perm, ss, sa = oracle.segments(d["idx"], d["max_adapters"])
    assert perm.tolist() == d["perm"]
    assert ss.tolist() == d["seg_start"]
    assert sa.tolist() == d["seg_adapter"]
    p = g["prefill"]
    ss, sa = oracle.merge_requests(p["req_start"], p["req_adapter"])
    assert ss.tolist() == p["seg_start"] and sa.tolist() == p["seg_adapter"]


@pytest.mark.parametrize("seed", range(5))
def test_segments_bruteforce(seed):
    rng = np.random.default_rng(seed)
    T, n_ad = int(rng.integers(0, 300)), int(rng.integers(1, 50))
    idx = rng.integers(-1, n_ad, T).astype(np.int32)
    perm, ss, sa = oracle.segments(idx, n_ad)
    # brute force: python sort by (adapter, position) over the valid tokens
    ref = sorted([i for i in range(T) if idx[i] >= 0], key=lambda i: (idx[i], i))
    assert perm.tolist() == ref
    assert ss[0] == 0 and ss[-1] == len(ref)
    for s in range(len(sa)):
        toks = perm[ss[s]:ss[s + 1]]
        assert toks.size > 0 and np.all(idx[toks] == sa[s])
    assert np.all(np.diff(sa) > 0)
    assert set(sa.tolist()) == set(idx[idx >= 0].tolist())


def test_pages_needed_closed_form():
    # 7B layer, rank 16, 16 KB pages of fp16 (8192 elements):
    # 4096-wide tensors take 16*4096/8192 = 8 pages, 11008-wide ones ceil(22.5..) = 22
    d_in = [4096] * 6 + [11008]
    d_out = [4096] * 4 + [11008] * 2 + [4096]
    assert oracle.pages_needed(16, d_in, d_out, 8192) == 4 * 16 + 2 * (8 + 22) + (22 + 8)
    # one row per page (1024-element rows, 1024-element pages): 2*r pages per projection
    assert oracle.pages_needed(8, [1024], [1024], 1024) == 16
    assert oracle.pages_needed(0, [1024], [1024], 1024) == 0
    # a 1024-wide output of rank 8 fits one 8192-element page
    assert oracle.pages_needed(8, [8192], [1024], 8192) == 8 + 1


def test_lru_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "lru_trace.json")))
    status, res, ev = oracle.lru_run(g["need"], g["capacity"], g["calls"])
    assert status.tolist() == g["status"]
    for c in range(len(g["calls"])):
        assert np.flatnonzero(res[c]).tolist() == g["resident"][c]
    assert ev == g["evicted"]


@pytest.mark.parametrize("seed", range(4))
def test_lru_invariants(seed):
    rng = np.random.default_rng(seed)
    n_ad = 30
    need = rng.integers(1, 6, n_ad)
    cap = 40
    calls = [rng.choice(n_ad, size=int(rng.integers(1, 8)), replace=True).tolist()
             for _ in range(60)]
    status, res, ev = oracle.lru_run(need, cap, calls)
    last = {}
    prev = np.zeros(n_ad, bool)
    for c, ids in enumerate(calls):
        if status[c] == 0:
            assert res[c][ids].all()
            assert not set(ev[c]) & set(ids)
            assert need[res[c]].sum() <= cap
            # each victim was at least as old as every unpinned survivor
            for v in ev[c]:
                for a in np.flatnonzero(res[c] & prev):
                    if a not in ids:
                        assert (last.get(v, -1), v) <= (last.get(a, -1), a)
            for a in ids:
                last[a] = c
        else:
            assert status[c] == 2 and ev[c] == []
            assert np.array_equal(res[c], prev)
        prev = res[c]


# A prefetch trace worked by hand from the rules (pages: a0..a2 need 4, a3
# needs 2, a4 needs 0; capacity 10; E = page-in calls so far):
#  1 page_in [0]          E=1  {0}
#  2 page_in [1]          E=2  {0,1}            free 2
#  3 prefetch [2,3] b=100 room = 2 + 4 (a0, age 1 < 2) = 6: a2 (4) and a3 (2)
#                         fit; a0 evicted           {1,2,3}
#  4 prefetch [4,0] b=3   room = 0 (all ages are 2): a4 (0 pages) fits, a0
#                         does not                  {1,2,3,4}
#  5 page_in [2,0]   E=3  a0 needs 4, free 0: oldest unpinned of age 2 is a1
#                         (lowest id)               {0,2,3,4}
#  6 prefetch [1] b=4     room = 2 (a3) + 0 (a4) < 4: skipped
#  7 page_in []      E=4
#  8 prefetch [1] b=10    room = 10; evicts a3, a4 (age 2, ids 3, 4), then a0
#                         (age 3, before a2 by id)  {1,2}
PREFETCH_TRACE = dict(
    need=[4, 4, 4, 2, 0], capacity=10,
    calls=[("page_in", [0], 0), ("page_in", [1], 0), ("prefetch", [2, 3], 100),
           ("prefetch", [4, 0], 3), ("page_in", [2, 0], 0), ("prefetch", [1], 4),
           ("page_in", [], 0), ("prefetch", [1], 10)],
    resident=[[0], [0, 1], [1, 2, 3], [1, 2, 3, 4], [0, 2, 3, 4], [0, 2, 3, 4], [0, 2, 3, 4],
              [1, 2]])


def test_prefetch_rules_hand_trace():
    t = PREFETCH_TRACE
    status, res = oracle.lru_prefetch_run(t["need"], t["capacity"], t["calls"])
    assert status.tolist() == [0] * len(t["calls"])
    assert [np.flatnonzero(r).tolist() for r in res] == t["resident"]


def test_prefetch_without_prefetch_calls_is_lru():
    rng = np.random.default_rng(3)
    need = rng.integers(0, 6, 25)
    calls = [rng.choice(25, size=int(rng.integers(1, 6))).tolist() for _ in range(50)]
    s1, r1, _ = oracle.lru_run(need, 30, calls)
    s2, r2 = oracle.lru_prefetch_run(need, 30, [("page_in", c, 0) for c in calls])
    assert np.array_equal(s1, s2) and np.array_equal(r1, r2)


# KV blocks sharing the pool, worked by hand (a0, a1 need 4 pages, a2 needs 2;
# capacity 10):
#  1 page_in [0]   E=1  {0}              used 4
#  2 kv_alloc 4         free 6 -> kv 4   {0}
#  3 page_in [1]   E=2  free 2 < 4: a0 (oldest) evicted   {1}
#  4 kv_alloc 4         free 2; a1 has age 2 = E, not evictable: OOM
#  5 page_in [2]   E=3  free 2 fits a2   {1,2}
#  6 kv_alloc 4         free 0; a1 (age 2 < 3) evicted -> kv 8   {2}
#  7 kv_free 6          kv 2
#  8 page_in [0,1] E=4  free 6 < 8: a2 evicted   {0,1}
KV_TRACE = dict(
    need=[4, 4, 2], capacity=10,
    calls=[("page_in", [0], 0), ("kv_alloc", [], 4), ("page_in", [1], 0), ("kv_alloc", [], 4),
           ("page_in", [2], 0), ("kv_alloc", [], 4), ("kv_free", [], 6), ("page_in", [0, 1], 0)],
    status=[0, 0, 0, 2, 0, 0, 0, 0],
    resident=[[0], [0], [1], [1], [1, 2], [2], [2], [0, 1]])


# Explicit eviction, worked by hand from the rules (a0..a2 need 4 pages, a3
# needs 2; capacity 10; E = page-in calls so far):
#  1 page_in [0]      E=1  {0}        used 4   age a0=1
#  2 page_in [1]      E=2  {0,1}      used 8   a1=2
#  3 evict [2]        a2 is not resident: NOT_RESIDENT (3), nothing changes
#  4 evict [0]        {1}, used 4; E stays 2, no age moves
#  5 prefetch [2,3,0] b=100
#                     room = free 6 + adapters older than E (none: a1's age is
#                     E) = 6: a2 (4) and a3 (2) fit, a0 does not   {1,2,3}
#                     (had the evict bumped E, a1 would count as older and a0
#                     would fit; had it kept a0's pages, only a3 would fit)
#  6 evict [3]        {1,2}, used 8 (between a prefetch and a page-in)
#  7 page_in [0] E=3  needs 4, free 2 (a3's pages): oldest unpinned of age 2
#                     are a1 and a2, lower id first: a1 evicted   {0,2}  a0=3
#  8 page_in [3] E=4  a3 fits the 2 free pages   {0,2,3}  a3=4
#  9 evict [3]        {0,2}; ages stay a0=3, a2=2
# 10 page_in [1] E=5  needs 4, free 2: a2 (age 2) goes before a0 (age 3)
#                     {0,1}  (had the evict refreshed the residents' ages,
#                     a0 and a2 would tie and a0 would go)
# 11 evict [7]        id out of range: ARG (1), nothing changes
EVICT_TRACE = dict(
    need=[4, 4, 4, 2], capacity=10,
    calls=[("page_in", [0], 0), ("page_in", [1], 0), ("evict", [2], 0), ("evict", [0], 0),
           ("prefetch", [2, 3, 0], 100), ("evict", [3], 0), ("page_in", [0], 0),
           ("page_in", [3], 0), ("evict", [3], 0), ("page_in", [1], 0), ("evict", [7], 0)],
    status=[0, 0, 3, 0, 0, 0, 0, 0, 0, 0, 1],
    resident=[[0], [0, 1], [0, 1], [1], [1, 2, 3], [1, 2], [0, 2], [0, 2, 3], [0, 2], [0, 1],
              [0, 1]])


def test_evict_hand_trace():
    t = EVICT_TRACE
    status, res = oracle.lru_prefetch_run(t["need"], t["capacity"], t["calls"])
    assert status.tolist() == t["status"]
    assert [np.flatnonzero(r).tolist() for r in res] == t["resident"]


def test_kv_blocks_hand_trace():
    t = KV_TRACE
    status, res = oracle.lru_prefetch_run(t["need"], t["capacity"], t["calls"])
    assert status.tolist() == t["status"]
    assert [np.flatnonzero(r).tolist() for r in res] == t["resident"]


# ---------------------------------------------------------------------------
# 8-bit adapter weights (e4m3 codes with one fp32 scale per rank row)

def test_e4m3_decoder_matches_torch_for_all_codes():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert got[0x7e] == 448.0 and got[0x01] == 2.0 ** -9 and np.isnan(got[0x7f])


def test_e4m3_quantizer_round_trip_ties_and_torch():
    import torch
    finite = np.array([c for c in range(256) if c not in (0x7f, 0xff)], np.uint8)
    vals = oracle.decode_e4m3(finite)
    assert np.array_equal(oracle.quantize_e4m3(vals, 1.0), finite)      # exact values map back
    # midpoints of neighbouring positive codes go to the even code
    pos = np.arange(0, 0x7e, dtype=np.uint8)
    lo, hi = oracle.decode_e4m3(pos), oracle.decode_e4m3(pos + 1)
    mids = oracle.quantize_e4m3((lo + hi) / 2, 1.0)
    assert np.array_equal(mids, np.where(pos % 2 == 0, pos, pos + 1).astype(np.uint8))
    # random fp32 inputs: torch's float -> e4m3 conversion rounds to nearest even too
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(20000) * rng.choice([1e-3, 0.1, 1, 30, 200], 20000)).astype(np.float32)
    v = np.clip(v, -448, 448)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.quantize_e4m3(v.astype(np.float64), 1.0), ref)
    assert oracle.quantize_e4m3([1e6, -1e6], 1.0).tolist() == [0x7e, 0xfe]   # saturates
    assert oracle.quantize_e4m3([3.0, -2.0], 0.0).tolist() == [0, 0]


def test_e4m3_row_quantisation_error_bound():
    rng = np.random.default_rng(1)
    rows = rng.standard_normal((16, 300)) * rng.uniform(1e-3, 10, (16, 1))
    rows[3] = 0.0
    codes, scales = oracle.quantize_rows_e4m3(rows)
    deq = oracle.decode_e4m3(codes) * scales[:, None].astype(np.float64)
    s = scales[:, None].astype(np.float64)
    # half an ulp: 2^-4 of the magnitude for normals, 2^-10 of the scale below them
    bound = np.maximum(np.abs(rows) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(deq - rows) <= bound)
    assert np.all(deq[3] == 0) and scales[3] == 0
    assert np.all(np.abs(oracle.decode_e4m3(codes)).max(axis=1)[scales > 0] <= 448)


def _q8_case(seed, T=9, d_in=96, d_out=80, ranks=(4, 8, 0)):
    rng = np.random.default_rng(seed)
    x = to_bits(F16, rng.standard_normal((T, d_in)).astype(np.float32))
    y = to_bits(F16, rng.standard_normal((T, d_out)).astype(np.float32))
    idx = rng.integers(-1, len(ranks), T).astype(np.int32)
    finite = np.array([c for c in range(256) if c not in (0x7f, 0xff)], np.uint8)
    qA = [rng.choice(finite, (r, d_in)) for r in ranks]
    qB = [rng.choice(finite, (r, d_out)) for r in ranks]
    return x, y, idx, np.array(ranks, np.int32), qA, qB


def test_q8_delta_with_unit_scales_is_the_16bit_delta():
    """e4m3 values are exact in fp16: with scales 1 the 8-bit delta must equal
    the 16-bit oracle on the decoded weights, bit for bit."""
    x, y, idx, ranks, qA, qB = _q8_case(2)
    ones = [np.ones(r, np.float32) for r in ranks]
    got = oracle.lora_delta_q8(F16, x, idx, y, ranks, np.full(3, 16.0), qA, ones, qB, ones)
    to16 = lambda q: oracle.decode_e4m3(q).astype(np.float16).view(np.uint16)
    ref = oracle.lora_delta(F16, x, idx, y, ranks, np.full(3, 16.0), [to16(q) for q in qA],
                            [to16(q) for q in qB])
    assert np.array_equal(got, ref)


def test_q8_delta_scales_enter_per_row():
    x, y, idx, ranks, qA, qB = _q8_case(3)
    ones = [np.ones(r, np.float32) for r in ranks]
    base = oracle.lora_delta_q8(F16, x, idx, y, ranks, np.full(3, 16.0), qA, ones, qB, ones)
    # powers of two cancel exactly: (2 sA) with (sB / 2)
    two = [np.full(r, 2.0, np.float32) for r in ranks]
    half = [np.full(r, 0.5, np.float32) for r in ranks]
    assert np.array_equal(base, oracle.lora_delta_q8(F16, x, idx, y, ranks, np.full(3, 16.0),
                                                     qA, two, qB, half))
    # zeroing one row's scale removes exactly that rank row's contribution
    sA = [np.ones(r, np.float32) for r in ranks]
    sA[1][5] = 0.0
    qA2 = [q.copy() for q in qA]
    qA2[1][5] = 0
    a = oracle.lora_delta_q8(F16, x, idx, y, ranks, np.full(3, 16.0), qA, sA, qB, ones)
    b = oracle.lora_delta_q8(F16, x, idx, y, ranks, np.full(3, 16.0), qA2, ones, qB, ones)
    assert np.array_equal(a, b)


# ---------------------------------------------------------------------------
# The base linear map and the whole layer Y = X.W0 + (alpha/r).((X.A).B)

def test_linear_lora_hand_example():
    """Worked by hand: x = [[1, 2, 3], [0.5, -1, 2]], W0 (2 x 3, a linear
    layer's weight) = [[1, 0, -1], [2, 1, 0.5]] gives X.W0 = [[-2, 5.5],
    [-1.5, 1]]; token 0 uses a rank-1 adapter with alpha 2 (scale 2),
    A_t = [[1, 1, 0]] (t = 3) and B = [[0.5, -1]] (delta [3, -6]); token 1 has
    no adapter.  Y = [[1, -0.5], [-1.5, 1]]."""
    f = lambda a: W.to_bits(W.F16, np.asarray(a, np.float32))
    x = f([[1, 2, 3], [0.5, -1, 2]])
    w0 = f([[1, 0, -1], [2, 1, 0.5]])
    y = oracle.linear_lora(W.F16, x, w0, np.array([0, -1]), [1], [2.0], [f([[1, 1, 0]])], [f([[0.5, -1]])])
    assert np.array_equal(y, [[1.0, -0.5], [-1.5, 1.0]])
    assert np.array_equal(oracle.linear(W.F16, x, w0), [[-2.0, 5.5], [-1.5, 1.0]])


def _layer_inputs(seed, dtype=W.BF16, T=9, d_in=96, d_out=80):
    rng = np.random.default_rng(seed)
    x = W.to_bits(dtype, rng.standard_normal((T, d_in)).astype(np.float32))
    w0 = W.to_bits(dtype, (rng.standard_normal((d_out, d_in)) / np.sqrt(d_in)).astype(np.float32))
    ranks = [4, 8]
    A_t = [W.to_bits(dtype, rng.standard_normal((r, d_in)).astype(np.float32)) for r in ranks]
    B = [W.to_bits(dtype, rng.standard_normal((r, d_out)).astype(np.float32)) for r in ranks]
    idx = rng.integers(-1, 2, T).astype(np.int32)
    return x, w0, idx, ranks, A_t, B


def test_linear_lora_with_zero_base_is_the_delta():
    x, w0, idx, ranks, A_t, B = _layer_inputs(1)
    zero_w = np.zeros_like(w0)
    y = oracle.linear_lora(W.BF16, x, zero_w, idx, ranks, [16.0, 16.0], A_t, B)
    ref = oracle.lora_delta(W.BF16, x, idx, np.zeros((x.shape[0], w0.shape[0]), np.uint16), ranks,
                            [16.0, 16.0], A_t, B)
    assert np.array_equal(y, ref)          # 0 + delta: bit for bit


def test_linear_lora_without_adapters_is_a_matmul():
    x, w0, idx, ranks, A_t, B = _layer_inputs(2)
    X = H_decode(x, W.BF16)
    Wm = H_decode(w0, W.BF16)
    ref = X @ Wm.T                          # numpy's fp64 matmul (another summation order)
    for ids in (np.full(x.shape[0], -1, np.int32), idx):
        zA = [np.zeros_like(a) for a in A_t] if ids is idx else A_t
        y = oracle.linear_lora(W.BF16, x, w0, ids, ranks, [16.0, 16.0], zA, B)
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_linear_is_linear_in_the_weight():
    x, w0, _, _, _, _ = _layer_inputs(3, dtype=W.F16)
    rng = np.random.default_rng(4)
    # two weights whose sum is exact in fp16 (small integers)
    w1 = W.to_bits(W.F16, rng.integers(-4, 5, w0.shape).astype(np.float32))
    w2 = W.to_bits(W.F16, rng.integers(-4, 5, w0.shape).astype(np.float32))
    ws = W.to_bits(W.F16, (H_decode(w1, W.F16) + H_decode(w2, W.F16)).astype(np.float32))
    a, b, c = (oracle.linear(W.F16, x, w) for w in (w1, w2, ws))
    assert np.allclose(a + b, c, rtol=1e-13, atol=1e-13 * np.abs(c).max())


def H_decode(bits, dtype):
    bits = np.asarray(bits, np.uint16)
    if dtype == W.F16:
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
