"""Python binding of the sm_100a paged multi-adapter LoRA delta library.

Every `slora_*` function here has the name, arguments and meaning of the C
entry point of the same name in include/slora.h; the binding only marshals
arguments (tensors -> device pointers, streams -> handles) and turns a failing
status into SloraError.  All arithmetic runs in the library's CUDA kernels.
PyTorch is used for device memory, pinned host memory and streams only.

`Pool` is a convenience owner of the caller-side buffers a pool needs (page
storage, tables, scratch) plus the pinned host copies of registered weights.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int32, c_int64, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libslora.so")

SLORA_F16, SLORA_BF16 = 0, 1
SLORA_PAGEIN_KERNEL, SLORA_PAGEIN_MEMCPY = 0, 1
SLORA_DECODE_AUTO, SLORA_DECODE_SPLIT, SLORA_DECODE_FUSED, SLORA_DECODE_STREAM = 0, 1, 2, 3
SLORA_KIND_NONE, SLORA_KIND_TOKEN, SLORA_KIND_STREAM, SLORA_KIND_FUSED, SLORA_KIND_SPLIT = 0, 1, 2, 3, 4
SLORA_WEIGHTS_16, SLORA_WEIGHTS_E4M3 = 0, 1
MAX_PROJ = 8

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "OOM", 3: "NOT_RESIDENT", 4: "CUDA", 5: "TIMEOUT",
          6: "DEVICE_CHECK", 7: "NOT_REGISTERED", 8: "INJECTED", 9: "UNSUPPORTED"}


class SloraError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status
        self.message = message


class PoolDesc(ctypes.Structure):
    _fields_ = [("dtype", c_int32), ("n_proj", c_int32), ("d_in", c_int32 * MAX_PROJ),
                ("d_out", c_int32 * MAX_PROJ), ("max_adapters", c_int32), ("max_rank", c_int32),
                ("max_tokens", c_int32), ("pagein_mode", c_int32), ("page_elems", c_int64),
                ("n_pages", c_int64), ("dev_pool", c_void_p), ("dev_tables", c_void_p),
                ("dev_scratch", c_void_p), ("scratch_bytes", c_size_t), ("host_only", c_int32),
                ("decode_path", c_int32), ("weight_format", c_int32), ("reserved", c_int32 * 5)]


class PoolStats(ctypes.Structure):
    _fields_ = [(n, c_int64) for n in ("page_ins", "hits", "evictions", "bytes_paged_in",
                                       "free_pages", "resident", "copy_calls", "epoch",
                                       "prefetched", "bytes_prefetched", "kv_pages")]


_lib = None


def lib():
    """Load libslora.so; fails loudly when the CUDA library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with gather_lora_paged_b200/build.py")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64 = c_void_p, c_int32, c_int64
    sig = {
        "slora_tables_bytes": ([POINTER(PoolDesc)], c_size_t),
        "slora_scratch_bytes": ([POINTER(PoolDesc)], c_size_t),
        "slora_pages_for_rank": ([POINTER(PoolDesc), I32], I64),
        "slora_pool_create": ([POINTER(PoolDesc), POINTER(c_void_p)], I32),
        "slora_pool_destroy": ([P], I32),
        "slora_last_error": ([P], ctypes.c_char_p),
        "slora_pool_set_page_order": ([P, P, I64], I32),
        "slora_adapter_register": ([P, I32, I32, c_float, P, P], I32),
        "slora_adapter_register_e4m3": ([P, I32, I32, c_float, P, P, P, P], I32),
        "slora_adapter_page_in": ([P, P, I32, P, P], I32),
        "slora_adapter_prefetch": ([P, P, I32, I64, P, P, POINTER(c_int32)], I32),
        "slora_prefetch_candidates": ([P, ctypes.c_double, I32, P, POINTER(c_int32)], I32),
        "slora_quantize_e4m3_rows": ([I32, P, I64, I64, P, P], I32),
        "slora_kv_alloc": ([P, I64, P, P, P], I32),
        "slora_kv_free": ([P, P, I64, P], I32),
        "slora_adapter_evict": ([P, I32, P], I32),
        "slora_adapter_is_resident": ([P, I32, POINTER(c_int32)], I32),
        "slora_check_batch": ([P, P, I32], I32),
        "slora_build_segments": ([P, P, I32, P, P, P, P, P], I32),
        "slora_build_sgmv_segments": ([P, P, P, I32, P, P, P, P], I32),
        "slora_bgmv_shrink": ([P, I32, P, I64, P, I32, P, I64, P], I32),
        "slora_bgmv_expand": ([P, I32, P, I64, P, I32, P, I64, P], I32),
        "slora_lora_delta": ([P, I32, P, P, P, P, P, P, I32, P], I32),
        "slora_sgmv": ([P, I32, P, P, P, P, P, P, P, I32, I32, P], I32),
        "slora_sgmv_linear": ([P, I32, P, P, P, P, P, P, P, P, P, I32, I32, P], I32),
        "slora_debug_gather": ([P, I32, I32, P, P], I32),
        "slora_check_device": ([P, P, POINTER(c_int32), POINTER(c_int32)], I32),
        "slora_pool_stats": ([P, POINTER(PoolStats)], I32),
        "slora_inject_fault": ([P, I32], I32),
        "slora_set_phase_events": ([P, P, I32], I32),
        "slora_lora_delta_noalloc": ([P, I32, P, P, P, P, P, P, I32, P], I32),
        "slora_noalloc_scratch_bytes": ([], c_size_t),
        "slora_decode_kernels": ([P, I32], I32),
        "slora_decode_kind": ([P, I32], I32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


# ---------------------------------------------------------------------------
# marshalling helpers
def _ptr(t) -> int | None:
    """Device/host pointer of a tensor, an int, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    return t.ctypes.data  # numpy array (host memory)


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _event(e) -> int | None:
    if e is None:
        return None
    if isinstance(e, int):
        return e
    h = e.cuda_event
    if not h:
        # torch creates the CUDA event on its first record(); passing NULL
        # would silently drop the completion signal
        raise ValueError("event has no CUDA handle yet: record it once before passing it")
    return h


def _arr(ctype, vals):
    a = (ctype * max(len(vals), 1))()
    for i, v in enumerate(vals):
        a[i] = v if v is not None else 0
    return a


def _check(pool, status: int):
    if status != 0:
        msg = lib().slora_last_error(pool).decode() if pool else ""
        raise SloraError(status, msg)


# ---------------------------------------------------------------------------
# the C ABI, one function each
def slora_tables_bytes(desc: PoolDesc) -> int:
    return lib().slora_tables_bytes(ctypes.byref(desc))


def slora_scratch_bytes(desc: PoolDesc) -> int:
    return lib().slora_scratch_bytes(ctypes.byref(desc))


def slora_pages_for_rank(desc: PoolDesc, rank: int) -> int:
    return lib().slora_pages_for_rank(ctypes.byref(desc), rank)


def slora_pool_create(desc: PoolDesc) -> int:
    h = c_void_p()
    st = lib().slora_pool_create(ctypes.byref(desc), ctypes.byref(h))
    if st != 0:
        raise SloraError(st, "slora_pool_create (set SLORA_LOG=1 for the reason)")
    return h.value


def slora_pool_destroy(pool: int) -> None:
    _check(None, lib().slora_pool_destroy(pool))


def slora_last_error(pool: int) -> str:
    return lib().slora_last_error(pool).decode()


def slora_pool_set_page_order(pool: int, order) -> None:
    import numpy as np
    o = np.ascontiguousarray(order, np.int32)
    _check(pool, lib().slora_pool_set_page_order(pool, o.ctypes.data, o.size))


def slora_adapter_register(pool: int, id: int, rank: int, alpha: float, host_A_t, host_B) -> None:
    pa = _arr(c_void_p, [_ptr(t) for t in host_A_t])
    pb = _arr(c_void_p, [_ptr(t) for t in host_B])
    _check(pool, lib().slora_adapter_register(pool, id, rank, alpha, ctypes.cast(pa, c_void_p),
                                              ctypes.cast(pb, c_void_p)))


def slora_adapter_register_e4m3(pool: int, id: int, rank: int, alpha: float, codes_A_t, scales_A_t,
                                codes_B, scales_B) -> None:
    """codes_*: pinned host tensors (uint8); scales_*: host float32 arrays (one per rank row)."""
    ca = _arr(c_void_p, [_ptr(t) for t in codes_A_t])
    sa = _arr(c_void_p, [_ptr(t) for t in scales_A_t])
    cb = _arr(c_void_p, [_ptr(t) for t in codes_B])
    sb = _arr(c_void_p, [_ptr(t) for t in scales_B])
    _check(pool, lib().slora_adapter_register_e4m3(pool, id, rank, alpha, ctypes.cast(ca, c_void_p),
                                                   ctypes.cast(sa, c_void_p), ctypes.cast(cb, c_void_p),
                                                   ctypes.cast(sb, c_void_p)))


def slora_adapter_page_in(pool: int, ids, side_stream=None, done_event=None) -> None:
    a = _arr(c_int32, [int(i) for i in ids])
    _check(pool, lib().slora_adapter_page_in(pool, ctypes.cast(a, c_void_p), len(ids),
                                             _stream(side_stream), _event(done_event)))


def slora_adapter_prefetch(pool: int, ids, max_pages: int, side_stream=None, done_event=None) -> int:
    """Returns the number of adapters whose copies were enqueued."""
    a = _arr(c_int32, [int(i) for i in ids])
    n_done = c_int32(0)
    _check(pool, lib().slora_adapter_prefetch(pool, ctypes.cast(a, c_void_p), len(ids), int(max_pages),
                                              _stream(side_stream), _event(done_event),
                                              ctypes.byref(n_done)))
    return n_done.value


def slora_prefetch_candidates(pool: int, half_life: float, max_n: int) -> list:
    out = (c_int32 * max(int(max_n), 1))()
    n = c_int32(0)
    _check(pool, lib().slora_prefetch_candidates(pool, float(half_life), int(max_n),
                                                 ctypes.cast(out, c_void_p), ctypes.byref(n)))
    return [int(out[i]) for i in range(n.value)]


def slora_quantize_e4m3_rows(dtype: int, bits):
    """(rows, n) 16-bit host values -> (codes uint8 (rows, n), scales float32 (rows,))."""
    import numpy as np
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    rows, n = bits.shape
    codes = np.empty((rows, n), np.uint8)
    scales = np.empty(max(rows, 1), np.float32)
    _check(None, lib().slora_quantize_e4m3_rows(dtype, bits.ctypes.data, rows, n, codes.ctypes.data,
                                                scales.ctypes.data))
    return codes, scales[:rows]


def slora_kv_alloc(pool: int, n: int, stream=None, done_event=None) -> list:
    """Returns the page ids taken for KV blocks."""
    out = (c_int32 * max(int(n), 1))()
    _check(pool, lib().slora_kv_alloc(pool, int(n), ctypes.cast(out, c_void_p), _stream(stream),
                                      _event(done_event)))
    return [int(out[i]) for i in range(int(n))]


def slora_kv_free(pool: int, ids, stream=None) -> None:
    a = _arr(c_int32, [int(i) for i in ids])
    _check(pool, lib().slora_kv_free(pool, ctypes.cast(a, c_void_p), len(ids), _stream(stream)))


def slora_adapter_evict(pool: int, id: int, stream=None) -> None:
    _check(pool, lib().slora_adapter_evict(pool, id, _stream(stream)))


def slora_adapter_is_resident(pool: int, id: int) -> bool:
    out = c_int32()
    _check(pool, lib().slora_adapter_is_resident(pool, id, ctypes.byref(out)))
    return bool(out.value)


def slora_check_batch(pool: int, idx_host) -> None:
    import numpy as np
    a = np.ascontiguousarray(idx_host, np.int32)
    _check(pool, lib().slora_check_batch(pool, a.ctypes.data, a.size))


def slora_build_segments(pool: int, idx, T: int, perm, seg_start, seg_adapter, S_out,
                         stream=None) -> None:
    _check(pool, lib().slora_build_segments(pool, _ptr(idx), T, _ptr(perm), _ptr(seg_start),
                                            _ptr(seg_adapter), _ptr(S_out), _stream(stream)))


def slora_build_sgmv_segments(pool: int, req_start, req_adapter, n: int, seg_start, seg_adapter,
                              S_out, stream=None) -> None:
    _check(pool, lib().slora_build_sgmv_segments(pool, _ptr(req_start), _ptr(req_adapter), n,
                                                 _ptr(seg_start), _ptr(seg_adapter), _ptr(S_out),
                                                 _stream(stream)))


def slora_bgmv_shrink(pool: int, proj: int, x, ldx: int, idx, T: int, t, ldt: int,
                      stream=None) -> None:
    _check(pool, lib().slora_bgmv_shrink(pool, proj, _ptr(x), ldx, _ptr(idx), T, _ptr(t), ldt,
                                         _stream(stream)))


def slora_bgmv_expand(pool: int, proj: int, t, ldt: int, idx, T: int, y, ldy: int,
                      stream=None) -> None:
    _check(pool, lib().slora_bgmv_expand(pool, proj, _ptr(t), ldt, _ptr(idx), T, _ptr(y), ldy,
                                         _stream(stream)))


def _slot_arrays(projs, x, ldx, y, ldy):
    n = len(projs)
    return (n, _arr(c_int32, projs), _arr(c_void_p, [_ptr(v) for v in x]), _arr(c_int64, ldx),
            _arr(c_void_p, [_ptr(v) for v in y]), _arr(c_int64, ldy))


def slora_lora_delta(pool: int, projs, x, ldx, y, ldy, idx, T: int, stream=None) -> None:
    n, pp, px, plx, py, ply = _slot_arrays(projs, x, ldx, y, ldy)
    c = lambda a: ctypes.cast(a, c_void_p)  # noqa: E731
    _check(pool, lib().slora_lora_delta(pool, n, c(pp), c(px), c(plx), c(py), c(ply), _ptr(idx),
                                        T, _stream(stream)))


def slora_lora_delta_noalloc(pool: int, projs, x, ldx, y, ldy, idx, T: int, stream=None) -> None:
    """slora_lora_delta with the library's fixed scratch array (no caller scratch)."""
    n, pp, px, plx, py, ply = _slot_arrays(projs, x, ldx, y, ldy)
    c = lambda a: ctypes.cast(a, c_void_p)  # noqa: E731
    _check(pool, lib().slora_lora_delta_noalloc(pool, n, c(pp), c(px), c(plx), c(py), c(ply),
                                                _ptr(idx), T, _stream(stream)))


def slora_noalloc_scratch_bytes() -> int:
    return lib().slora_noalloc_scratch_bytes()


def slora_sgmv(pool: int, projs, x, ldx, y, ldy, seg_start, seg_adapter, S: int, T: int,
               stream=None) -> None:
    n, pp, px, plx, py, ply = _slot_arrays(projs, x, ldx, y, ldy)
    c = lambda a: ctypes.cast(a, c_void_p)  # noqa: E731
    _check(pool, lib().slora_sgmv(pool, n, c(pp), c(px), c(plx), c(py), c(ply), _ptr(seg_start),
                                  _ptr(seg_adapter), S, T, _stream(stream)))


def slora_sgmv_linear(pool: int, projs, x, ldx, w0, ldw, y, ldy, seg_start, seg_adapter, S: int, T: int,
                      stream=None) -> None:
    """y = x . W0 + delta per projection (w0[k]: d_out x d_in device tensors)."""
    n, pp, px, plx, py, ply = _slot_arrays(projs, x, ldx, y, ldy)
    pw = _arr(c_void_p, [_ptr(t) for t in w0])
    plw = _arr(c_int64, [int(v) for v in ldw])
    c = lambda a: ctypes.cast(a, c_void_p)  # noqa: E731
    _check(pool, lib().slora_sgmv_linear(pool, n, c(pp), c(px), c(plx), c(pw), c(plw), c(py), c(ply),
                                         _ptr(seg_start), _ptr(seg_adapter), S, T, _stream(stream)))


def slora_debug_gather(pool: int, id: int, proj: int, host_A_t, host_B) -> None:
    _check(pool, lib().slora_debug_gather(pool, id, proj, _ptr(host_A_t), _ptr(host_B)))


def slora_check_device(pool: int, stream=None):
    code, info = c_int32(), c_int32()
    st = lib().slora_check_device(pool, _stream(stream), ctypes.byref(code), ctypes.byref(info))
    if st not in (0, 6):
        _check(pool, st)
    return st, code.value, info.value


def slora_pool_stats(pool: int) -> dict:
    s = PoolStats()
    _check(pool, lib().slora_pool_stats(pool, ctypes.byref(s)))
    return {f: getattr(s, f) for f, _ in PoolStats._fields_}


def slora_decode_kernels(pool: int, T: int) -> int:
    """Kernels slora_lora_delta launches for T tokens on this pool (1 or 3)."""
    return int(lib().slora_decode_kernels(pool, int(T)))


def slora_decode_kind(pool: int, T: int) -> int:
    """SLORA_KIND_* of the kernels a decode call of T tokens takes."""
    return int(lib().slora_decode_kind(pool, int(T)))


def slora_set_phase_events(pool: int, events) -> None:
    a = _arr(c_void_p, [_event(e) for e in events])
    _check(pool, lib().slora_set_phase_events(pool, ctypes.cast(a, c_void_p), len(events)))


def slora_inject_fault(pool: int, after: int) -> None:
    _check(pool, lib().slora_inject_fault(pool, after))


# ---------------------------------------------------------------------------
def make_desc(dtype, d_in, d_out, max_adapters, max_rank, max_tokens, page_elems, n_pages,
              pagein_mode=SLORA_PAGEIN_KERNEL, host_only=False,
              decode_path=SLORA_DECODE_AUTO, weight_format=SLORA_WEIGHTS_16) -> PoolDesc:
    d = PoolDesc()
    d.dtype = dtype
    d.n_proj = len(d_in)
    for i, (a, b) in enumerate(zip(d_in, d_out)):
        d.d_in[i] = a
        d.d_out[i] = b
    d.max_adapters = max_adapters
    d.max_rank = max_rank
    d.max_tokens = max_tokens
    d.pagein_mode = pagein_mode
    d.page_elems = page_elems
    d.n_pages = n_pages
    d.host_only = 1 if host_only else 0
    d.decode_path = decode_path
    d.weight_format = weight_format
    return d


class Pool:
    """Owns the caller-side buffers of one pool (device pages, tables, scratch
    as torch tensors) and the pinned host copies of registered adapters."""

    def __init__(self, dtype, d_in, d_out, max_adapters, max_rank, max_tokens, page_elems,
                 n_pages, pagein_mode=SLORA_PAGEIN_KERNEL, host_only=False, device="cuda",
                 decode_path=SLORA_DECODE_AUTO, weight_format=SLORA_WEIGHTS_16):
        self.desc = make_desc(dtype, d_in, d_out, max_adapters, max_rank, max_tokens, page_elems,
                              n_pages, pagein_mode, host_only, decode_path, weight_format)
        self.host_only = host_only
        self.keep = {}
        if not host_only:
            import torch
            tdt = torch.float16 if dtype == SLORA_F16 else torch.bfloat16
            self.pages = torch.empty(max(n_pages * page_elems, 8), dtype=tdt, device=device)
            self.tables = torch.empty(slora_tables_bytes(self.desc), dtype=torch.uint8,
                                      device=device)
            sb = slora_scratch_bytes(self.desc)
            self.scratch = torch.empty(sb, dtype=torch.uint8, device=device)
            self.desc.dev_pool = self.pages.data_ptr()
            self.desc.dev_tables = self.tables.data_ptr()
            self.desc.dev_scratch = self.scratch.data_ptr()
            self.desc.scratch_bytes = sb
        self.h = slora_pool_create(self.desc)

    def close(self):
        if self.h:
            slora_pool_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def pages_for_rank(self, r):
        return slora_pages_for_rank(self.desc, r)

    def register(self, id, rank, alpha, A_t, B, pinned=None):
        """A_t[p], B[p]: host tensors (pinned torch tensors) or numpy uint16
        arrays, which are copied into pinned memory owned by this object."""
        if not self.host_only and pinned is None:
            import numpy as np
            import torch

            def pin(a):
                if isinstance(a, np.ndarray):
                    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()
                return a
            A_t = [pin(a) for a in A_t]
            B = [pin(b) for b in B]
        self.keep[id] = (A_t, B)
        slora_adapter_register(self.h, id, rank, alpha, A_t, B)

    def page_in(self, ids, side_stream=None, done_event=None):
        slora_adapter_page_in(self.h, list(ids), side_stream, done_event)

    def prefetch(self, ids, max_pages, side_stream=None, done_event=None) -> int:
        return slora_adapter_prefetch(self.h, list(ids), max_pages, side_stream, done_event)

    def prefetch_candidates(self, half_life, max_n) -> list:
        return slora_prefetch_candidates(self.h, half_life, max_n)

    def kv_alloc(self, n, stream=None, done_event=None) -> list:
        return slora_kv_alloc(self.h, n, stream, done_event)

    def kv_free(self, ids, stream=None) -> None:
        slora_kv_free(self.h, list(ids), stream)

    def stats(self):
        return slora_pool_stats(self.h)
