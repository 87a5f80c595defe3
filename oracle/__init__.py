"""Python face of the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE: only tests/, the package smoke entry and bench.py's CPU
baseline leg import this module.  It shares no code with the CUDA path; inputs
are numpy arrays of raw 16-bit patterns (np.uint16) plus int32 index arrays.
Every function cites, in oracle.c, the passage of the pages it follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

F16, BF16 = 0, 1


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_long
        L.oracle_decode16.argtypes = [i32, P, i64, P]
        L.oracle_lora_delta.argtypes = [i32, i32, i32, i32, P, i64, P, P, i64, i32, P, P, P, P,
                                        P, i32]
        L.oracle_segments.argtypes = [P, i32, i32, P, P, P, P]
        L.oracle_merge_requests.argtypes = [P, P, i32, P, P, P]
        L.oracle_pages_needed.argtypes = [i32, i32, P, P, i64]
        L.oracle_pages_needed.restype = i64
        L.oracle_lru_run.argtypes = [i32, P, i64, i32, P, P, P, P, P, P]
        L.oracle_lru_prefetch_run.argtypes = [i32, P, i64, i32, P, P, P, P, P, P]
        L.oracle_decode_e4m3.argtypes = [P, i64, P]
        L.oracle_quantize_e4m3.argtypes = [P, i64, ctypes.c_double, P]
        L.oracle_linear.argtypes = [i32, i32, i32, i32, P, i64, P, i64, P, i32]
        L.oracle_lora_delta_q8.argtypes = [i32, i32, i32, i32, P, i64, P, P, i64, i32, P, P, P, P,
                                           P, P, P, i32]
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def decode16(bits, dtype):
    bits = _c(bits, np.uint16)
    out = np.empty(bits.shape, np.float64)
    rc = lib().oracle_decode16(dtype, _p(bits), bits.size, _p(out))
    assert rc == 0
    return out


def lora_delta(dtype, x, idx, y_in, ranks, alphas, A_t, B, n_threads=1):
    """fp64 y_out = y_in + (alpha_a / r_a) * (x_i . A_a) . B_a per token.

    x: (T, d_in) uint16 bits; idx: (T,) int; y_in: (T, d_out) bits or None;
    ranks: (n_adapters,) int; alphas: (n_adapters,) float; A_t[a]: (r_a, d_in)
    bits (A transposed, rank-major); B[a]: (r_a, d_out) bits.  A_t[a]/B[a] may
    be None for adapters no token uses.
    """
    x = _c(x, np.uint16)
    T, d_in = x.shape
    idx = _c(idx, np.int32)
    n_ad = len(ranks)
    d_out = None
    for b in B:
        if b is not None and b.size:
            d_out = b.shape[1]
            break
    if y_in is not None:
        y_in = _c(y_in, np.uint16)
        d_out = y_in.shape[1]
    assert d_out is not None, "d_out unknown: pass y_in or one non-empty B"
    ranks = _c(ranks, np.int32)
    alphas = _c(alphas, np.float64)
    keep = []
    pa = (ctypes.c_void_p * max(n_ad, 1))()
    pb = (ctypes.c_void_p * max(n_ad, 1))()
    for a in range(n_ad):
        if A_t[a] is not None and ranks[a] > 0:
            at = _c(A_t[a], np.uint16)
            bb = _c(B[a], np.uint16)
            assert at.shape == (ranks[a], d_in) and bb.shape == (ranks[a], d_out)
            keep += [at, bb]
            pa[a] = at.ctypes.data
            pb[a] = bb.ctypes.data
    y_out = np.empty((T, d_out), np.float64)
    rc = lib().oracle_lora_delta(dtype, T, d_in, d_out, _p(x), d_in, _p(idx),
                                 _p(y_in) if y_in is not None else None, d_out, n_ad,
                                 _p(ranks), _p(alphas), ctypes.cast(pa, ctypes.c_void_p),
                                 ctypes.cast(pb, ctypes.c_void_p), _p(y_out), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_lora_delta: invalid argument")
    return y_out


def decode_e4m3(codes):
    """e4m3 codes (uint8) -> exact fp64 values (NaN for 0x7f / 0xff)."""
    codes = _c(codes, np.uint8)
    out = np.empty(codes.shape, np.float64)
    lib().oracle_decode_e4m3(_p(codes), codes.size, _p(out))
    return out


def quantize_e4m3(values, scale):
    """Nearest e4m3 codes of values / scale (ties: even fraction; saturating
    at +-448); all zero codes when scale == 0."""
    v = _c(values, np.float64)
    out = np.empty(v.shape, np.uint8)
    if lib().oracle_quantize_e4m3(_p(v), v.size, float(scale), _p(out)) != 0:
        raise ValueError("oracle_quantize_e4m3: invalid argument")
    return out


def quantize_rows_e4m3(values):
    """Per-row quantisation of a (rows, n) fp64 array: scale = max|row| / 448
    stored as fp32, codes = nearest e4m3 of row / scale.  Returns (codes,
    scales)."""
    values = np.asarray(values, np.float64)
    scales = (np.abs(values).max(axis=1, initial=0.0) / 448.0).astype(np.float32)
    codes = np.stack([quantize_e4m3(row, float(s)) for row, s in zip(values, scales)]) \
        if values.shape[0] else np.zeros(values.shape, np.uint8)
    return codes, scales


def linear(dtype, x, w0, n_threads=1):
    """fp64 y = x . W0 for x (T, d_in) bits and w0 (d_out, d_in) bits (the
    layout of a linear layer's weight)."""
    x = _c(x, np.uint16)
    w0 = _c(w0, np.uint16)
    T, d_in = x.shape
    d_out = w0.shape[0]
    assert w0.shape[1] == d_in
    y = np.empty((T, d_out), np.float64)
    if lib().oracle_linear(dtype, T, d_in, d_out, _p(x), d_in, _p(w0), d_in, _p(y), int(n_threads)) != 0:
        raise ValueError("oracle_linear: invalid argument")
    return y


def linear_lora(dtype, x, w0, idx, ranks, alphas, A_t, B, n_threads=1):
    """fp64 Y = X.W0 + (alpha_a / r_a) (x_i . A_a) . B_a per token: the base
    linear map plus the delta (the delta starts from zero)."""
    x = _c(x, np.uint16)
    zero = np.zeros((x.shape[0], np.asarray(w0).shape[0]), np.uint16)
    return linear(dtype, x, w0, n_threads) + lora_delta(dtype, x, idx, zero, ranks, alphas, A_t, B,
                                                         n_threads)


def lora_delta_q8(dtype, x, idx, y_in, ranks, alphas, qA_t, sA, qB, sB, n_threads=1):
    """As lora_delta, with adapter a's weights as e4m3 codes qA_t[a] (r_a,
    d_in), qB[a] (r_a, d_out) and fp32 row scales sA[a], sB[a] (r_a,)."""
    x = _c(x, np.uint16)
    T, d_in = x.shape
    idx = _c(idx, np.int32)
    n_ad = len(ranks)
    y_in = _c(y_in, np.uint16)
    d_out = y_in.shape[1]
    ranks = _c(ranks, np.int32)
    alphas = _c(alphas, np.float64)
    keep = []
    ptr = [(ctypes.c_void_p * max(n_ad, 1))() for _ in range(4)]
    for a in range(n_ad):
        if qA_t[a] is not None and ranks[a] > 0:
            arrs = [_c(qA_t[a], np.uint8), _c(sA[a], np.float32), _c(qB[a], np.uint8),
                    _c(sB[a], np.float32)]
            assert arrs[0].shape == (ranks[a], d_in) and arrs[2].shape == (ranks[a], d_out)
            assert arrs[1].shape == arrs[3].shape == (ranks[a],)
            keep += arrs
            for q in range(4):
                ptr[q][a] = arrs[q].ctypes.data
    y_out = np.empty((T, d_out), np.float64)
    rc = lib().oracle_lora_delta_q8(dtype, T, d_in, d_out, _p(x), d_in, _p(idx), _p(y_in), d_out,
                                    n_ad, _p(ranks), _p(alphas),
                                    *[ctypes.cast(q, ctypes.c_void_p) for q in ptr], _p(y_out),
                                    int(n_threads))
    if rc != 0:
        raise ValueError("oracle_lora_delta_q8: invalid argument")
    return y_out


def segments(idx, max_adapters):
    """Stable counting sort by adapter: (perm, seg_start, seg_adapter)."""
    idx = _c(idx, np.int32)
    T = idx.size
    perm = np.full(T, -1, np.int32)
    ss = np.zeros(T + 1, np.int32)
    sa = np.zeros(max(T, 1), np.int32)
    S = np.zeros(1, np.int32)
    rc = lib().oracle_segments(_p(idx), T, max_adapters, _p(perm), _p(ss), _p(sa), _p(S))
    if rc != 0:
        raise ValueError("oracle_segments: invalid argument")
    S = int(S[0])
    return perm[: ss[S]].copy(), ss[: S + 1].copy(), sa[:S].copy()


def merge_requests(req_start, req_adapter):
    req_start = _c(req_start, np.int32)
    req_adapter = _c(req_adapter, np.int32)
    n = req_adapter.size
    ss = np.zeros(n + 1, np.int32)
    sa = np.zeros(max(n, 1), np.int32)
    S = np.zeros(1, np.int32)
    rc = lib().oracle_merge_requests(_p(req_start), _p(req_adapter), n, _p(ss), _p(sa), _p(S))
    if rc != 0:
        raise ValueError("oracle_merge_requests: invalid argument")
    S = int(S[0])
    return ss[: S + 1].copy(), sa[:S].copy()


def pages_needed(rank, d_in, d_out, page_elems):
    d_in = _c(d_in, np.int32)
    d_out = _c(d_out, np.int32)
    return int(lib().oracle_pages_needed(int(rank), d_in.size, _p(d_in), _p(d_out),
                                         int(page_elems)))


def lru_run(need, capacity, calls):
    """Run the LRU rules over `calls` (a list of id lists).

    Returns (status[c], resident[c, a] bool, evicted ids per call)."""
    need = _c(need, np.int64)
    n_ad = need.size
    off = np.zeros(len(calls) + 1, np.int32)
    for c, ids in enumerate(calls):
        off[c + 1] = off[c] + len(ids)
    ids = _c(np.concatenate([np.asarray(c, np.int32) for c in calls]) if calls else
             np.zeros(0, np.int32), np.int32)
    status = np.zeros(len(calls), np.int32)
    resident = np.zeros((len(calls), n_ad), np.uint8)
    evicted = np.zeros(max(n_ad * len(calls), 1), np.int32)
    eoff = np.zeros(len(calls) + 1, np.int32)
    lib().oracle_lru_run(n_ad, _p(need), int(capacity), len(calls), _p(off), _p(ids),
                         _p(status), _p(resident), _p(evicted), _p(eoff))
    ev = [evicted[eoff[c]:eoff[c + 1]].tolist() for c in range(len(calls))]
    return status, resident.astype(bool), ev


def lru_prefetch_run(need, capacity, calls):
    """Run the LRU rules with prefetch and KV-block calls over `calls`, a
    list of (kind, ids, n): kind "page_in", "prefetch" (n = page budget),
    "kv_alloc" or "kv_free" (n pages; ids unused), "evict" (ids = [one id]).

    Returns (status[c], resident[c, a] bool)."""
    need = _c(need, np.int64)
    n_ad = need.size
    kinds = {"page_in": 0, "prefetch": 1, "kv_alloc": 2, "kv_free": 3, "evict": 4}
    kind = _c([kinds[k] for k, _, _ in calls], np.int32)
    budget = _c([int(b) for _, _, b in calls], np.int64)
    off = np.zeros(len(calls) + 1, np.int32)
    for c, (_, ids, _) in enumerate(calls):
        off[c + 1] = off[c] + len(ids)
    ids = _c(np.concatenate([np.asarray(i, np.int32) for _, i, _ in calls]) if calls else
             np.zeros(0, np.int32), np.int32)
    status = np.zeros(len(calls), np.int32)
    resident = np.zeros((len(calls), n_ad), np.uint8)
    lib().oracle_lru_prefetch_run(n_ad, _p(need), int(capacity), len(calls), _p(kind), _p(budget),
                                  _p(off), _p(ids), _p(status), _p(resident))
    return status, resident.astype(bool)


def n_threads_default():
    return os.cpu_count() or 1
