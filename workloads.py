"""Seeded synthetic inputs for the paged multi-adapter LoRA delta.

This module only draws random numbers and arranges them; it holds none of the
method's arithmetic.  Both the tests (for the CUDA path and the oracle) and
bench.py use it, so that the two sides see identical inputs.

Value recipe (the pages publish no datasets for this op; these stand in for
the serving traces the pages evaluate on):
  * x ~ N(0, 1), y_in ~ N(0, 1) (y_in stands for the base output X.W0);
  * A ~ N(0, std = 1/sqrt(d_in)), B ~ N(0, std = 1/sqrt(r)), alpha = 16;
  * the base weight of a projection (for the whole linear layer) W0 ~
    N(0, std = 1/sqrt(d_in)), stored as d_out rows of d_in;
  * values are drawn in fp32 and rounded to nearest-even into fp16 or bf16;
  * adapter per token: uniform (the tiny case) or a finite Zipf law
    P(id = j) ~ (j + 1)^(-s) over j in [0, N), drawn by inverse CDF.
Every stream has its own counter-style seed [base_seed, tag, ...] so that one
adapter's weights can be drawn without drawing the others'.

Adapters that no token of the workload touches ("fillers") share one set of
host weights per rank; they still get pages of their own in the pool.  Their
values never reach an output.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

F16, BF16 = 0, 1
DTYPE_NAME = {F16: "f16", BF16: "bf16"}
ALPHA = 16.0

# stream tags
_T_IDX, _T_RANK, _T_X, _T_Y, _T_AD, _T_FILL, _T_REQ, _T_COLD, _T_W0 = range(9)


def _rng(*key):
    return np.random.Generator(np.random.PCG64([int(k) for k in key]))


def to_bits(dtype: int, a: np.ndarray) -> np.ndarray:
    """fp32 values -> fp16/bf16 bit patterns (round to nearest even)."""
    a = np.ascontiguousarray(a, np.float32)
    if dtype == F16:
        return a.astype(np.float16).view(np.uint16)
    u = a.view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >>
            np.uint32(16)).astype(np.uint16)


def normal_bits(rng, shape, std, dtype):
    v = rng.standard_normal(int(np.prod(shape)), dtype=np.float32)
    if std != 1.0:
        v *= np.float32(std)
    return to_bits(dtype, v).reshape(shape)


def zipf_ids(rng, n_ids: int, s: float, size: int) -> np.ndarray:
    w = (np.arange(1, n_ids + 1, dtype=np.float64)) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(size)
    return np.minimum(np.searchsorted(cdf, u, side="right"), n_ids - 1).astype(np.int32)


@dataclasses.dataclass
class Proj:
    name: str
    d_in: int
    d_out: int
    x_name: str  # projections sharing x_name read the same input rows


def llama_layer(H: int, M: int, KV: int | None = None) -> list[Proj]:
    KV = H if KV is None else KV
    return [Proj("q", H, H, "attn"), Proj("k", H, KV, "attn"), Proj("v", H, KV, "attn"),
            Proj("o", H, H, "o"), Proj("gate", H, M, "mlp"), Proj("up", H, M, "mlp"),
            Proj("down", M, H, "down")]


@dataclasses.dataclass
class Workload:
    cfg: int
    name: str
    dtype: int
    projs: list
    T: int
    idx: np.ndarray            # (T,) int32 adapter per token, -1 = none
    ranks: np.ndarray          # (n_adapters,) int32
    page_elems: int
    shuffle_pages: bool
    seed: int
    # prefill requests (SGMV): token range [req_start[q], req_start[q+1]) uses req_adapter[q]
    req_start: np.ndarray | None = None
    req_adapter: np.ndarray | None = None
    n_decode: int = 0          # tokens [0, n_decode) are decode tokens (per-token idx)
    cold_frac: float = 0.0
    alpha: float = ALPHA
    _cache: dict = dataclasses.field(default_factory=dict, repr=False)

    @property
    def n_adapters(self) -> int:
        return int(self.ranks.size)

    @property
    def x_names(self) -> list[str]:
        out = []
        for p in self.projs:
            if p.x_name not in out:
                out.append(p.x_name)
        return out

    def x_dim(self, x_name: str) -> int:
        return next(p.d_in for p in self.projs if p.x_name == x_name)

    def touched(self) -> np.ndarray:
        ids = self.idx[self.idx >= 0]
        return np.unique(ids).astype(np.int32)

    def x(self, x_name: str) -> np.ndarray:
        key = ("x", x_name)
        if key not in self._cache:
            k = self.x_names.index(x_name)
            self._cache[key] = normal_bits(_rng(self.seed, _T_X, k), (self.T, self.x_dim(x_name)),
                                           1.0, self.dtype)
        return self._cache[key]

    def y_in(self, p: int) -> np.ndarray:
        key = ("y", p)
        if key not in self._cache:
            self._cache[key] = normal_bits(_rng(self.seed, _T_Y, p),
                                           (self.T, self.projs[p].d_out), 1.0, self.dtype)
        return self._cache[key]

    def w0(self, p: int) -> np.ndarray:
        """The base weight of projection p as a linear layer stores it: d_out
        rows of d_in, N(0, std = 1/sqrt(d_in)) (random-init stand-in for the
        model's weight)."""
        key = ("w0", p)
        if key not in self._cache:
            pr = self.projs[p]
            self._cache[key] = normal_bits(_rng(self.seed, _T_W0, p), (pr.d_out, pr.d_in),
                                           1.0 / np.sqrt(pr.d_in), self.dtype)
        return self._cache[key]

    def _draw_adapter(self, key_rng, r):
        A_t, B = [], []
        for p in self.projs:
            A_t.append(normal_bits(key_rng, (r, p.d_in), 1.0 / np.sqrt(p.d_in), self.dtype))
            B.append(normal_bits(key_rng, (r, p.d_out), 1.0 / np.sqrt(max(r, 1)), self.dtype))
        return A_t, B

    def adapter(self, a: int, filler_ok: bool = True):
        """(A_t[p] (r x d_in), B[p] (r x d_out)) bit arrays of adapter a.

        Adapters in `touched_set` get weights of their own; the others share a
        per-rank filler when filler_ok."""
        r = int(self.ranks[a])
        own = (not filler_ok) or a in self._touched_set()
        key = ("ad", a) if own else ("fill", r)
        if key not in self._cache:
            rng = _rng(self.seed, _T_AD, a) if own else _rng(self.seed, _T_FILL, r)
            self._cache[key] = self._draw_adapter(rng, r)
        return self._cache[key]

    def prefetch_adapters(self, ids, threads: int = 8):
        ids = [int(a) for a in ids]
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(self.adapter, ids))

    def _touched_set(self):
        if "touched" not in self._cache:
            self._cache["touched"] = set(self.touched().tolist()) | set(self.extra_touched)
        return self._cache["touched"]

    extra_touched: tuple = ()

    def drop(self, prefix):
        for k in [k for k in self._cache if isinstance(k, tuple) and k[0] == prefix]:
            del self._cache[k]


# ----------------------------------------------------------------------------
# The five workloads.  Seeds are 1000 + config index.

def _cfg0(T=8, seed=1000):
    idx = _rng(seed, _T_IDX).integers(0, 4, size=T).astype(np.int32)
    return Workload(0, "tiny_decode_1proj_d1024_T8_fp16", F16, [Proj("p", 1024, 1024, "x")], T,
                    idx, np.array([8, 8, 16, 16], np.int32), 1024, False, seed, n_decode=T)


def _cfg1(T=256, n_adapters=1000, seed=1001):
    idx = zipf_ids(_rng(seed, _T_IDX), n_adapters, 1.0, T)
    return Workload(1, "llama7b_decode_layer_T256_1000ad_r16_fp16", F16, llama_layer(4096, 11008),
                    T, idx, np.full(n_adapters, 16, np.int32), 8192, False, seed, n_decode=T)


def _cfg2(T=512, n_adapters=2000, seed=1002):
    idx = zipf_ids(_rng(seed, _T_IDX), n_adapters, 1.2, T)
    ranks = _rng(seed, _T_RANK).choice(np.array([8, 16, 32, 64], np.int32), n_adapters)
    return Workload(2, "llama13b_decode_layer_T512_2000ad_r8-64_bf16_shuffled", BF16,
                    llama_layer(5120, 13824), T, idx, ranks.astype(np.int32), 8192, True, seed,
                    n_decode=T)


def _cfg3(n_req=32, n_adapters=64, lo=64, hi=1024, seed=1003):
    rng = _rng(seed, _T_REQ)
    lens = rng.integers(lo, hi + 1, size=n_req)
    req_ad = rng.integers(0, n_adapters, size=n_req).astype(np.int32)
    req_start = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(req_start[-1])
    idx = np.repeat(req_ad, lens).astype(np.int32)
    ranks = _rng(seed, _T_RANK).choice(np.array([16, 32, 64], np.int32), n_adapters)
    return Workload(3, "llama7b_sgmv_prefill_32req_64-1024tok_64ad_r16-64_bf16", BF16,
                    llama_layer(4096, 11008), T, idx, ranks.astype(np.int32), 8192, False, seed,
                    req_start=req_start, req_adapter=req_ad, n_decode=0)


def _cfg4(n_dec=1024, n_req=8, req_len=512, n_adapters=2000, seed=1004):
    rng = _rng(seed, _T_IDX)
    dec = zipf_ids(rng, n_adapters, 1.0, n_dec)
    req_ad = zipf_ids(rng, n_adapters, 1.0, n_req)
    idx = np.concatenate([dec, np.repeat(req_ad, req_len)]).astype(np.int32)
    req_start = (n_dec + np.arange(n_req + 1) * req_len).astype(np.int32)
    ranks = _rng(seed, _T_RANK).choice(np.array([8, 16, 32, 64, 128], np.int32), n_adapters)
    return Workload(4, "llama70b_mixed_1024dec_8x512prefill_2000ad_r8-128_bf16_30pct_cold", BF16,
                    llama_layer(8192, 28672, 1024), n_dec + n_req * req_len, idx,
                    ranks.astype(np.int32), 8192, True, seed, req_start=req_start,
                    req_adapter=req_ad.astype(np.int32), n_decode=n_dec, cold_frac=0.3)


BUILDERS = {0: _cfg0, 1: _cfg1, 2: _cfg2, 3: _cfg3, 4: _cfg4}


def config(i: int, replica: int = 0, **kw) -> Workload:
    """Workload i.  Replica k > 0 (one per data-parallel rank) draws its own
    batch, activations and weights from seed 1000 + i + 10000 k."""
    if replica:
        kw["seed"] = 1000 + i + 10000 * int(replica)
    return BUILDERS[i](**kw)


def cold_split(w: Workload):
    """Seeded split of the touched adapters into (warm, cold) for the mixed
    workload: cold_frac of them start outside the pool."""
    t = w.touched()
    rng = _rng(w.seed, _T_COLD)
    perm = rng.permutation(t.size)
    n_cold = int(round(w.cold_frac * t.size))
    cold = np.sort(t[perm[:n_cold]])
    warm = np.sort(t[perm[n_cold:]])
    return warm.astype(np.int32), cold.astype(np.int32)


def page_order(n_pages: int, seed: int) -> np.ndarray:
    """A seeded permutation of page ids (the 'shuffled pool')."""
    return _rng(seed, 99).permutation(n_pages).astype(np.int32)
