"""The C-ABI library loads and exports every entry point include/slora.h
declares; sizing and host-side pool logic (LRU, page accounting, OOM, fault
injection, batch checks) run without a GPU on a host_only pool and agree with
the oracle's LRU rules."""
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
import gather_lora_paged_b200 as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "slora.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(slora_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = G.lib()
    names = _declared()
    assert len(names) >= 20
    out = subprocess.run(["nm", "-D", "--defined-only", G.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(slora_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(L, n)


def test_desc_layout_matches_header():
    # int32 x 22, then int64 page_elems at byte 88 (see slora_pool_desc)
    assert G.PoolDesc.page_elems.offset == 88
    assert G.PoolDesc.dev_pool.offset == 104
    assert G.PoolDesc.host_only.offset == 136
    assert __import__("ctypes").sizeof(G.PoolDesc) == 168


LAYER7B = ([4096] * 6 + [11008], [4096] * 4 + [11008] * 2 + [4096])


def test_sizing_matches_oracle_page_count():
    d = G.make_desc(G.SLORA_F16, *LAYER7B, 1000, 64, 256, 8192, 10)
    for r in (0, 8, 16, 24, 64):
        assert G.slora_pages_for_rank(d, r) == oracle.pages_needed(r, *LAYER7B, 8192)
    assert G.slora_tables_bytes(d) > 0 and G.slora_scratch_bytes(d) > 0
    # e4m3 weights: a page of page_elems 16-bit units holds 2 * page_elems codes
    d8 = G.make_desc(G.SLORA_F16, *LAYER7B, 1000, 64, 256, 8192, 10, weight_format=G.SLORA_WEIGHTS_E4M3)
    for r in (0, 3, 8, 16, 24, 64):
        assert G.slora_pages_for_rank(d8, r) == oracle.pages_needed(r, *LAYER7B, 2 * 8192)
    # the tables grow by the row-scale table of every adapter
    assert G.slora_tables_bytes(d8) >= G.slora_tables_bytes(d) + 4 * 1000 * 7 * 2 * 64


def test_e4m3_pool_registration_and_lru():
    """A host-only e4m3 pool: registration needs codes and scales (and the
    16-bit call is refused), pages are counted at two codes per unit, LRU as
    for 16-bit pools."""
    pool = G.Pool(G.SLORA_F16, [1024, 2048], [2048, 1024], 8, 32, 64, 1024, 192, host_only=True,
                  weight_format=G.SLORA_WEIGHTS_E4M3)
    codes = np.zeros(16, np.uint8)
    sc = np.ones(32, np.float32)
    with pytest.raises(G.SloraError) as e:
        G.slora_adapter_register(pool.h, 0, 8, 16.0, [codes, codes], [codes, codes])
    assert e.value.status == 1
    with pytest.raises(G.SloraError) as e:   # a negative scale
        G.slora_adapter_register_e4m3(pool.h, 0, 8, 16.0, [codes, codes], [-sc, sc], [codes, codes],
                                      [sc, sc])
    assert e.value.status == 1
    for a in range(4):
        G.slora_adapter_register_e4m3(pool.h, a, 32, 16.0, [codes, codes], [sc, sc], [codes, codes],
                                      [sc, sc])
    need = pool.pages_for_rank(32)
    assert need == 2 * (32 * 1024 // 2048 + 32 * 2048 // 2048)      # 96: half of the 16-bit count
    pool.page_in([0, 1])
    pool.page_in([2])                  # 192 pages hold two adapters: the oldest (0) goes
    assert [G.slora_adapter_is_resident(pool.h, a) for a in range(4)] == [0, 1, 1, 0]


def _host_pool(n_pages=100, max_adapters=40, max_rank=32, page=1024):
    return G.Pool(G.SLORA_F16, [1024, 2048], [2048, 1024], max_adapters, max_rank, 64, page,
                  n_pages, host_only=True)


def _register_all(pool, ranks):
    dummy = np.zeros(16, np.uint16)
    for a, r in enumerate(ranks):
        pool.register(a, int(r), 16.0, [dummy, dummy], [dummy, dummy])


@pytest.mark.parametrize("seed", range(4))
def test_lru_matches_oracle(seed):
    rng = np.random.default_rng(seed)
    n_ad = 40
    ranks = rng.choice([0, 8, 16, 32], n_ad)
    pool = _host_pool()
    _register_all(pool, ranks)
    need = [pool.pages_for_rank(int(r)) for r in ranks]
    calls = [rng.choice(n_ad, size=int(rng.integers(1, 7))).tolist() for _ in range(80)]
    calls.insert(10, [n_ad + 3])  # invalid id
    status, resident, evicted = oracle.lru_run(need, 100, calls)
    for c, ids in enumerate(calls):
        st = 0
        try:
            pool.page_in(ids)
        except G.SloraError as e:
            st = e.status
        assert st == status[c], (c, ids, st, status[c])
        got = [G.slora_adapter_is_resident(pool.h, a) for a in range(n_ad)]
        assert got == resident[c].tolist(), c
    s = pool.stats()
    assert s["free_pages"] == 100 - sum(need[a] for a in range(n_ad) if resident[-1][a])
    assert s["evictions"] == sum(len(e) for e in evicted)


def test_lru_golden_trace_through_the_library(golden_dir):
    import json
    g = json.load(open(os.path.join(golden_dir, "lru_trace.json")))
    # pages: d_in 1024, d_out 1024, page 1024 -> 2*rank pages per adapter
    ranks = [n // 2 for n in g["need"]]
    pool = G.Pool(G.SLORA_F16, [1024], [1024], len(ranks), 8, 16, 1024, g["capacity"],
                  host_only=True)
    _register_all(pool, ranks)
    assert [pool.pages_for_rank(r) for r in ranks] == g["need"]
    for c, ids in enumerate(g["calls"]):
        st = 0
        try:
            pool.page_in(ids)
        except G.SloraError as e:
            st = e.status
        assert st == g["status"][c]
        res = [a for a in range(len(ranks)) if G.slora_adapter_is_resident(pool.h, a)]
        assert res == g["resident"][c]


def test_oom_and_injection_leave_pool_unchanged():
    pool = _host_pool(n_pages=30)
    _register_all(pool, [16] * 10)   # 16*(1024+2048)*2/1024 = 96 pages each > 30
    with pytest.raises(G.SloraError) as e:
        pool.page_in([0])
    assert e.value.status == 2
    pool2 = _host_pool()
    _register_all(pool2, [8] * 10)   # 48 pages each
    pool2.page_in([0])
    before = pool2.stats()
    G.slora_inject_fault(pool2.h, 0)
    with pytest.raises(G.SloraError) as e:
        pool2.page_in([1])
    assert e.value.status == 8
    assert pool2.stats() == before
    pool2.page_in([1])  # disarmed after firing
    assert G.slora_adapter_is_resident(pool2.h, 1)


def test_unregistered_and_batch_checks():
    pool = _host_pool()
    _register_all(pool, [8, 8, 8])
    with pytest.raises(G.SloraError) as e:
        pool.page_in([5])
    assert e.value.status == 7
    pool.page_in([0, 1])
    G.slora_check_batch(pool.h, [0, 1, -1, 0])
    with pytest.raises(G.SloraError) as e:
        G.slora_check_batch(pool.h, [2])
    assert e.value.status == 3
    with pytest.raises(G.SloraError) as e:
        G.slora_check_batch(pool.h, [0, 99])
    assert e.value.status == 1
    pool.page_in([1])                   # 0 stays resident but is no longer in the step's set
    with pytest.raises(G.SloraError):
        G.slora_check_batch(pool.h, [0])
    G.slora_adapter_evict(pool.h, 1)
    assert not G.slora_adapter_is_resident(pool.h, 1)


def test_page_order_validation():
    pool = _host_pool(n_pages=10)
    with pytest.raises(G.SloraError):
        G.slora_pool_set_page_order(pool.h, [0, 1, 2])
    with pytest.raises(G.SloraError):
        G.slora_pool_set_page_order(pool.h, [0] * 10)
    G.slora_pool_set_page_order(pool.h, list(range(9, -1, -1)))


def test_host_only_pool_refuses_compute():
    pool = _host_pool()
    with pytest.raises(G.SloraError) as e:
        G.slora_lora_delta(pool.h, [0], [0], [1024], [0], [2048], 0, 0)
    assert e.value.status == 9


def test_bad_desc_rejected():
    d = G.make_desc(G.SLORA_F16, [100], [128], 4, 16, 8, 1024, 4, host_only=True)
    with pytest.raises(G.SloraError):
        G.slora_pool_create(d)   # 100 is not a multiple of 64
    d = G.make_desc(G.SLORA_F16, [128], [128], 4, 16, 8, 1000, 4, host_only=True)
    with pytest.raises(G.SloraError):
        G.slora_pool_create(d)   # page size not a power of two


def test_event_without_cuda_handle_is_refused():
    """A torch event that was never recorded has no CUDA handle (0); passing
    it as NULL would drop the page-in completion signal, so the binding
    refuses it."""
    class Unrecorded:
        cuda_event = 0
    with pytest.raises(ValueError):
        G._event(Unrecorded())
    assert G._event(None) is None and G._event(1234) == 1234


@pytest.mark.parametrize("seed", range(4))
def test_prefetch_matches_oracle(seed):
    """page_in and prefetch calls interleaved: the library's residency after
    every call agrees with the oracle's restatement of the rules."""
    rng = np.random.default_rng(100 + seed)
    n_ad = 40
    ranks = rng.choice([0, 8, 16, 32], n_ad)
    pool = _host_pool()
    _register_all(pool, ranks)
    need = [pool.pages_for_rank(int(r)) for r in ranks]
    calls = []
    for _ in range(150):
        ids = rng.choice(n_ad, size=int(rng.integers(1, 7))).tolist()
        if rng.random() < 0.4:
            calls.append(("prefetch", ids, int(rng.integers(0, 160))))
        else:
            calls.append(("page_in", ids, 0))
    calls.insert(7, ("prefetch", [n_ad + 1], 50))     # invalid id
    status, resident = oracle.lru_prefetch_run(need, 100, calls)
    n_pre = 0
    for c, (kind, ids, budget) in enumerate(calls):
        st = 0
        try:
            if kind == "page_in":
                pool.page_in(ids)
            else:
                n_pre += G.slora_adapter_prefetch(pool.h, ids, budget)
        except G.SloraError as e:
            st = e.status
        assert st == status[c], (c, kind, ids, st, status[c])
        got = [G.slora_adapter_is_resident(pool.h, a) for a in range(n_ad)]
        assert got == resident[c].tolist(), (c, kind, ids, budget)
    assert pool.stats()["prefetched"] == n_pre > 0


def test_prefetch_keeps_the_step_set_and_needs_a_page_in():
    pool = _host_pool(n_pages=150)              # rank 8: 48 pages each -> 3 fit
    _register_all(pool, [8] * 6)
    pool.page_in([0])
    pool.page_in([1, 2])                         # the step's set; 0 is older
    assert G.slora_adapter_prefetch(pool.h, [3, 4], 1000) == 1   # room for one: evicts 0
    res = [G.slora_adapter_is_resident(pool.h, a) for a in range(6)]
    assert res == [False, True, True, True, False, False]
    G.slora_check_batch(pool.h, [1, 2, -1])      # the step's set is unchanged
    with pytest.raises(G.SloraError) as e:
        G.slora_check_batch(pool.h, [3])         # prefetched, not yet named
    assert e.value.status == 3
    # nothing older than the step is left: a second prefetch cannot evict
    assert G.slora_adapter_prefetch(pool.h, [4, 5], 1000) == 0
    before = pool.stats()
    pool.page_in([3, 1])                         # finds 3 resident: two hits, no copy
    after = pool.stats()
    assert after["hits"] - before["hits"] == 2 and after["page_ins"] == before["page_ins"]
    G.slora_check_batch(pool.h, [3, 1])
    assert after["bytes_prefetched"] == 2 * 8 * (1024 + 2048 + 2048 + 1024)
    # a budget smaller than one adapter skips it; rank 0 needs no pages
    with pytest.raises(G.SloraError) as e:
        G.slora_adapter_prefetch(pool.h, [4], -1)
    assert e.value.status == 1
    assert G.slora_adapter_prefetch(pool.h, [4], 47) == 0


def _decayed_scores(trace, n_ad, half_life):
    """Popularity by its definition: over an adapter's last 32 namings by a
    page-in call, the sum of 2^(-age / half_life), age in page-in calls."""
    E = len(trace)
    scores = {}
    for a in range(n_ad):
        epochs = [e + 1 for e, ids in enumerate(trace) if a in ids][-32:]
        if epochs:
            scores[a] = sum(2.0 ** (-(E - e) / half_life) for e in epochs)
    return scores


@pytest.mark.parametrize("half_life", [1.0, 4.0, 50.0])
def test_prefetch_candidates_rank_by_decayed_popularity(half_life):
    rng = np.random.default_rng(7)
    n_ad = 12
    pool = _host_pool(n_pages=100)              # two rank-8 adapters fit
    _register_all(pool, [8] * n_ad)
    # skewed traffic: adapter 0 named in most calls (more than 32 times)
    trace = []
    for _ in range(60):
        ids = sorted({int(i) for i in (rng.zipf(1.6, 2) - 1) % n_ad})
        pool.page_in(ids)
        trace.append(set(ids))
    sc = _decayed_scores(trace, n_ad, half_life)
    want = [a for a in sc if not G.slora_adapter_is_resident(pool.h, a)]
    got = G.slora_prefetch_candidates(pool.h, half_life, n_ad)
    assert sorted(got) == sorted(want)
    for u, v in zip(got, got[1:]):               # most popular first, ties by id
        assert sc[u] > sc[v] * (1 + 1e-12) or (abs(sc[u] - sc[v]) <= 1e-12 * sc[u] and u < v)
    assert G.slora_prefetch_candidates(pool.h, half_life, 2) == got[:2]
    with pytest.raises(G.SloraError):
        G.slora_prefetch_candidates(pool.h, 0.0, 4)


def test_prefetch_hand_trace_through_the_library():
    from test_oracle import PREFETCH_TRACE as t
    ranks = [n // 2 for n in t["need"]]          # d_in = d_out = page = 1024: 2 r pages
    pool = G.Pool(G.SLORA_F16, [1024], [1024], len(ranks), 8, 16, 1024, t["capacity"],
                  host_only=True)
    _register_all(pool, ranks)
    for c, (kind, ids, budget) in enumerate(t["calls"]):
        if kind == "page_in":
            pool.page_in(ids)
        else:
            G.slora_adapter_prefetch(pool.h, ids, budget)
        assert [a for a in range(len(ranks)) if G.slora_adapter_is_resident(pool.h, a)] == \
            t["resident"][c], c


def test_kv_hand_trace_through_the_library():
    from test_oracle import KV_TRACE as t
    ranks = [n // 2 for n in t["need"]]
    pool = G.Pool(G.SLORA_F16, [1024], [1024], len(ranks), 8, 16, 1024, t["capacity"],
                  host_only=True)
    _register_all(pool, ranks)
    held = []
    for c, (kind, ids, n) in enumerate(t["calls"]):
        st = 0
        try:
            if kind == "page_in":
                pool.page_in(ids)
            elif kind == "kv_alloc":
                held += G.slora_kv_alloc(pool.h, n)
            else:
                G.slora_kv_free(pool.h, held[:n])
                held = held[n:]
        except G.SloraError as e:
            st = e.status
        assert st == t["status"][c], c
        assert [a for a in range(len(ranks)) if G.slora_adapter_is_resident(pool.h, a)] == \
            t["resident"][c], c
    assert pool.stats()["kv_pages"] == len(held) == 2


def test_evict_hand_trace_through_the_library():
    from test_oracle import EVICT_TRACE as t
    ranks = [n // 2 for n in t["need"]]          # d_in = d_out = page = 1024: 2 r pages
    pool = G.Pool(G.SLORA_F16, [1024], [1024], len(ranks), 8, 16, 1024, t["capacity"],
                  host_only=True)
    _register_all(pool, ranks)
    for c, (kind, ids, budget) in enumerate(t["calls"]):
        st = 0
        try:
            if kind == "page_in":
                pool.page_in(ids)
            elif kind == "prefetch":
                G.slora_adapter_prefetch(pool.h, ids, budget)
            else:
                G.slora_adapter_evict(pool.h, ids[0])
        except G.SloraError as e:
            st = e.status
        assert st == t["status"][c], c
        assert [a for a in range(len(ranks)) if G.slora_adapter_is_resident(pool.h, a)] == \
            t["resident"][c], c


@pytest.mark.parametrize("seed", range(4))
def test_kv_blocks_and_prefetch_match_oracle(seed):
    rng = np.random.default_rng(200 + seed)
    n_ad = 30
    ranks = rng.choice([0, 8, 16], n_ad)
    pool = _host_pool(n_pages=160)
    _register_all(pool, ranks)
    need = [pool.pages_for_rank(int(r)) for r in ranks]
    held, calls, got_status, got_res = [], [], [], []
    for _ in range(160):
        u = rng.random()
        if u < 0.45:
            call = ("page_in", rng.choice(n_ad, size=int(rng.integers(1, 5))).tolist(), 0)
        elif u < 0.6:
            call = ("prefetch", rng.choice(n_ad, size=int(rng.integers(1, 5))).tolist(),
                    int(rng.integers(0, 120)))
        elif u < 0.75:
            call = ("kv_alloc", [], int(rng.integers(0, 60)))
        elif u < 0.9:
            call = ("kv_free", [], int(rng.integers(0, len(held) + 1)))
        else:
            call = ("evict", [int(rng.integers(0, n_ad))], 0)
        kind, ids, n = call
        st = 0
        try:
            if kind == "page_in":
                pool.page_in(ids)
            elif kind == "prefetch":
                G.slora_adapter_prefetch(pool.h, ids, n)
            elif kind == "kv_alloc":
                held += G.slora_kv_alloc(pool.h, n)
            elif kind == "evict":
                G.slora_adapter_evict(pool.h, ids[0])
            else:
                pick = set(rng.choice(len(held), size=n, replace=False).tolist())
                G.slora_kv_free(pool.h, [held[i] for i in sorted(pick)])
                held = [h for i, h in enumerate(held) if i not in pick]
        except G.SloraError as e:
            st = e.status
        calls.append(call)
        got_status.append(st)
        got_res.append([G.slora_adapter_is_resident(pool.h, a) for a in range(n_ad)])
        assert len(set(held)) == len(held)
        s = pool.stats()
        assert s["kv_pages"] == len(held)
        assert s["free_pages"] + len(held) + sum(need[a] for a in range(n_ad) if got_res[-1][a]) == 160
    status, res = oracle.lru_prefetch_run(need, 160, calls)
    assert got_status == status.tolist()
    assert got_res == res.tolist()
    assert 2 in got_status                       # the trace reached an OOM


def test_kv_free_checks_ids_and_pages_are_never_evicted():
    pool = _host_pool(n_pages=100)
    _register_all(pool, [8, 8])                  # 48 pages each
    kv = G.slora_kv_alloc(pool.h, 40)
    assert len(set(kv)) == 40 and pool.stats()["kv_pages"] == 40
    with pytest.raises(G.SloraError) as e:       # 96 pages needed, only 60 are not KV
        pool.page_in([0, 1])
    assert e.value.status == 2
    pool.page_in([0])
    for bad in ([kv[0], kv[0]], [kv[0], 10 ** 6], [i for i in range(100) if i not in kv][:1]):
        with pytest.raises(G.SloraError) as e:
            G.slora_kv_free(pool.h, bad)
        assert e.value.status == 1
    assert pool.stats()["kv_pages"] == 40        # nothing changed
    with pytest.raises(G.SloraError):
        G.slora_pool_set_page_order(pool.h, list(range(100)))
    G.slora_kv_free(pool.h, kv[:36])
    pool.page_in([0, 1])                         # 12 free + 36 returned = 48
    assert G.slora_adapter_is_resident(pool.h, 0) and G.slora_adapter_is_resident(pool.h, 1)
    assert pool.stats()["free_pages"] == 0


@pytest.mark.parametrize("dtype", [G.SLORA_F16, G.SLORA_BF16])
def test_e4m3_row_quantiser_matches_oracle(dtype):
    """The library's host quantiser (frexp / rint) against the oracle's
    (nearest code by trying every code), codes and scales bit for bit."""
    rng = np.random.default_rng(dtype)
    rows = rng.standard_normal((40, 257)) * rng.choice([1e-6, 1e-3, 1.0, 50.0, 3e3], (40, 1))
    rows = np.clip(rows, -6e4, 6e4)         # finite in fp16
    rows[5] = 0.0
    rows[6, :] = 0.0
    rows[6, 3] = -0.0
    rows[7, 10] = 1e-7                       # lone tiny value: subnormal codes
    bits = __import__("workloads").to_bits(dtype, rows.astype(np.float32))
    codes, scales = G.slora_quantize_e4m3_rows(dtype, bits)
    vals = oracle.decode16(bits, dtype)
    ref_codes, ref_scales = oracle.quantize_rows_e4m3(vals)
    assert np.array_equal(scales.view(np.uint32), ref_scales.view(np.uint32))
    assert np.array_equal(codes, ref_codes)
    assert scales[5] == 0 and not codes[5].any()
    nan = bits.copy()
    nan[2, 2] = 0x7E00 if dtype == G.SLORA_F16 else 0x7FC0
    with pytest.raises(G.SloraError) as e:
        G.slora_quantize_e4m3_rows(dtype, nan)
    assert e.value.status == 1


def test_pool_convenience_methods():
    pool = _host_pool(n_pages=100)
    _register_all(pool, [8, 8, 8])
    pool.page_in([0])
    assert pool.prefetch([1, 2], 1000) == 1            # 52 free pages: one rank-8 adapter
    kv = pool.kv_alloc(4)
    assert pool.stats()["kv_pages"] == 4
    pool.kv_free(kv)
    pool.page_in([0])
    assert pool.prefetch_candidates(2.0, 5) == []      # only adapter 0 was ever named, and it is resident


@pytest.mark.parametrize("fmt", [G.SLORA_WEIGHTS_16, G.SLORA_WEIGHTS_E4M3], ids=["16bit", "e4m3"])
def test_decode_path_policy(fmt):
    """Kernels a decode call launches, per path and token count (host logic):
    AUTO runs up to 16 tokens of a 16-bit pool as one CTA per token, 17..1024
    on the streaming-stage kernel and more on the three-kernel path; an e4m3
    pool takes the streaming kernel up to 1024 tokens; the one-kernel paths
    hand calls above 1024 tokens to the three-kernel path."""
    want = {
        G.SLORA_DECODE_AUTO: {1: 1, 16: 1, 17: 1, 512: 1, 513: 1, 1024: 1, 1025: 3},
        G.SLORA_DECODE_SPLIT: {1: 3, 256: 3, 1025: 3},
        G.SLORA_DECODE_FUSED: {1: 1, 1024: 1, 1025: 3},
        G.SLORA_DECODE_STREAM: {1: 1, 1024: 1, 1025: 3},
    }
    for path, cases in want.items():
        pool = G.Pool(G.SLORA_F16, [1024], [1024], 4, 16, 2048, 1024, 64, host_only=True,
                      decode_path=path, weight_format=fmt)
        for T, k in cases.items():
            assert G.slora_decode_kernels(pool.h, T) == k, (path, T)
            kind = G.slora_decode_kind(pool.h, T)
            assert (kind == G.SLORA_KIND_SPLIT) == (k == 3), (path, T, kind)
            if path == G.SLORA_DECODE_STREAM and T <= 1024:
                assert kind == G.SLORA_KIND_STREAM
            if path == G.SLORA_DECODE_FUSED and T <= 1024:
                assert kind == G.SLORA_KIND_FUSED
            if path == G.SLORA_DECODE_AUTO and T <= 16 and fmt == G.SLORA_WEIGHTS_16:
                assert kind == G.SLORA_KIND_TOKEN
            if path == G.SLORA_DECODE_AUTO and (T > 16 or fmt != G.SLORA_WEIGHTS_16) and T <= 1024:
                assert kind == G.SLORA_KIND_STREAM
        assert G.slora_decode_kernels(pool.h, 0) == 0
        assert G.slora_decode_kind(pool.h, 0) == G.SLORA_KIND_NONE
        pool.close()
