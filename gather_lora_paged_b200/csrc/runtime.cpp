// runtime.cpp -- host side of the C ABI in include/slora.h: the paged adapter
// pool (free pages, per-adapter page lists, LRU residency), page-in planning
// and submission, argument validation and kernel launches.
//
// Sources for the behaviour (see include/slora.h for the full citations):
//   "Paper explainer: S-LoRA", section "Unified Paging": adapters live in host
//   RAM, are paged into VRAM on demand and evicted least-recently-used first.
//   "Multi-LoRA serving: S-LoRA, Punica, SGMV, vLLM", section on the unified
//   paged pool: fixed-size non-contiguous pages, asynchronous PCIe page-in on
//   dedicated streams overlapped with compute.
#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <set>
#include <string>
#include <thread>
#include <unordered_set>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "slora_internal.h"

using namespace slora;

namespace slora {
cudaError_t launch_sgmv(const BgmvParams& p, int dtype, const int32_t* seg_start,
                        const int32_t* seg_adapter, int S, int T, int sm_count, cudaStream_t s,
                        void* scratch, int max_tokens, int64_t n_pages, cudaEvent_t const* ev, int n_ev);
size_t sgmv_scratch_bytes(const slora_pool_desc& d);
cudaError_t launch_linear(const BgmvParams& bp, int dtype, const void* const* w0, const int64_t* ldw,
                          const int32_t* seg_start, const int32_t* seg_adapter, int S, int T, int sm_count,
                          cudaStream_t st, void* scratch, int max_tokens, int64_t n_pages);
}  // namespace slora

namespace {

constexpr int kStagingSlots = 4;
constexpr double kWaitSeconds = 30.0;

int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Size of a rank x dim weight tensor in the pool's 16-bit units: one element
// each, or (e4m3 weights) two codes each.
int64_t tensor_units(const slora_pool_desc& d, int64_t rank, int64_t dim) {
  return d.weight_format == SLORA_WEIGHTS_E4M3 ? rank * dim / 2 : rank * dim;
}
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// An NVTX range around each C-ABI call that enqueues work or changes the pool,
// so that profilers show the library's calls on the timeline (no cost when no
// tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kUseHistory = 32;  // page_in namings kept per adapter for the prefetch policy

struct Adapter {
  bool registered = false;
  bool resident = false;
  int rank = 0;
  float alpha = 0.f;
  const void* host_A[kMaxSlots] = {};
  const void* host_B[kMaxSlots] = {};
  const void* map_A[kMaxSlots] = {};  // device-usable addresses of the pinned copies
  const void* map_B[kMaxSlots] = {};
  int64_t last_use = -1;       // LRU age: epoch of the last page_in naming it, or of its prefetch
  int64_t named = -1;          // epoch of the last page_in naming it (compute may use it iff == epoch)
  int64_t uses[kUseHistory];   // epochs of its most recent page_in namings (a ring)
  int n_uses = 0;              // namings recorded so far
  std::vector<int32_t> pages;  // tensor order (p, A), (p, B)
  std::vector<float> qs;       // e4m3 weights: row scales [projection][A_t, B][rank]
};

struct FreePage {
  int32_t id;
  int64_t free_epoch;  // compute epoch that last may have read it (-1: none)
  int rel = -1;        // release event of the KV-block owner that freed it (-1: none)
};

constexpr int kRelRing = 64;  // events marking the last use of freed KV blocks

struct Staging {
  void* host = nullptr;
  size_t cap = 0;
  cudaEvent_t done = nullptr;
  bool pending = false;
};

// Table layout inside dev_tables.
struct TableLayout {
  size_t off_rank, off_scale, off_err, off_list, off_qscale, off_desc, desc_cap, total;
};

// Row scales of e4m3 weights, per adapter: [projection][A_t, B][max_rank] floats.
size_t qscale_floats(const slora_pool_desc& d) {
  return d.weight_format == SLORA_WEIGHTS_E4M3 ? (size_t)d.n_proj * 2 * (size_t)d.max_rank : 0;
}

// Scratch layout inside dev_scratch.
struct ScratchLayout {
  size_t off_ready, off_meta, off_perm, off_seg_start, off_seg_adapter, off_seg_rank, off_shrink_pre,
      off_expand_pre, off_tpart, off_sgmv, total;
  int64_t tpart_floats, rk8;
  int MS;
};

int64_t list_stride_of(const slora_pool_desc& d, int* listA, int* listB) {
  int64_t off = 0;
  for (int p = 0; p < d.n_proj; ++p) {
    listA[p] = (int)off;
    off += cdiv64(tensor_units(d, d.max_rank, d.d_in[p]), d.page_elems);
    listB[p] = (int)off;
    off += cdiv64(tensor_units(d, d.max_rank, d.d_out[p]), d.page_elems);
  }
  for (int p = d.n_proj; p < kMaxSlots; ++p) listA[p] = listB[p] = 0;
  return off > 0 ? off : 1;
}

TableLayout table_layout(const slora_pool_desc& d) {
  int la[kMaxSlots], lb[kMaxSlots];
  const int64_t stride = list_stride_of(d, la, lb);
  TableLayout L;
  size_t o = 0;
  L.off_rank = o;
  o = align_up(o + 4 * (size_t)d.max_adapters, 256);
  L.off_scale = o;
  o = align_up(o + 4 * (size_t)d.max_adapters, 256);
  L.off_err = o;
  o = align_up(o + 16, 256);
  L.off_list = o;
  o = align_up(o + 4 * (size_t)d.max_adapters * stride, 256);
  L.off_qscale = o;
  o = align_up(o + 4 * (size_t)d.max_adapters * qscale_floats(d), 256);
  L.off_desc = o;
  L.desc_cap = align_up(sizeof(PageInHeader) + 4 * (size_t)d.max_adapters +
                            (sizeof(PageInNew) + 4 * (size_t)stride + 4 * qscale_floats(d) + 32) *
                                (size_t)d.max_adapters,
                        256);
  o += L.desc_cap;
  L.total = o;
  return L;
}

ScratchLayout scratch_layout(const slora_pool_desc& d) {
  ScratchLayout L;
  const int64_t T = d.max_tokens;
  L.MS = (int)std::min<int64_t>(T, d.max_adapters);
  if (L.MS < 1) L.MS = 1;
  int64_t sum_ns = 0;
  for (int p = 0; p < d.n_proj; ++p) sum_ns += cdiv64(d.d_in[p], kPartK);
  L.rk8 = std::max<int64_t>(8, (d.max_rank + 7) / 8 * 8);
  L.tpart_floats = sum_ns * T * L.rk8;
  size_t o = 0;
  L.off_ready = o;  // first in every layout: zero between calls (see kFReadyCap)
  o = align_up(o + kFReadyBytes, 256);
  L.off_meta = o;
  o = align_up(o + 4 * kMetaCount, 256);
  L.off_perm = o;
  o = align_up(o + 4 * (size_t)T, 256);
  L.off_seg_start = o;
  o = align_up(o + 4 * (size_t)(L.MS + 1), 256);
  L.off_seg_adapter = o;
  o = align_up(o + 4 * (size_t)L.MS, 256);
  L.off_seg_rank = o;
  o = align_up(o + 4 * (size_t)L.MS, 256);
  L.off_shrink_pre = o;
  o = align_up(o + 4 * (size_t)(L.MS + 1), 256);
  L.off_expand_pre = o;
  o = align_up(o + 4 * (size_t)(L.MS + 1), 256);
  L.off_tpart = o;
  o = align_up(o + 4 * (size_t)L.tpart_floats, 256);
  L.off_sgmv = o;
  o = align_up(o + sgmv_scratch_bytes(d), 256);
  L.total = o;
  return L;
}

const char* status_name(slora_status_t s) {
  switch (s) {
    case SLORA_OK: return "ok";
    case SLORA_ERR_INVALID_ARG: return "invalid argument";
    case SLORA_ERR_OOM: return "out of pages";
    case SLORA_ERR_NOT_RESIDENT: return "adapter not resident";
    case SLORA_ERR_CUDA: return "CUDA error";
    case SLORA_ERR_TIMEOUT: return "timeout";
    case SLORA_ERR_DEVICE_CHECK: return "device check";
    case SLORA_ERR_NOT_REGISTERED: return "adapter not registered";
    case SLORA_ERR_INJECTED: return "injected failure";
    case SLORA_ERR_UNSUPPORTED: return "unsupported";
  }
  return "?";
}

}  // namespace

struct slora_pool {
  slora_pool_desc d;
  int listA[kMaxSlots], listB[kMaxSlots];
  int64_t list_stride = 0;
  TableLayout tl;
  ScratchLayout sl;
  std::vector<Adapter> ad;
  std::deque<FreePage> free_pages;
  std::set<std::pair<int64_t, int>> lru;  // (last_use, id) of resident adapters
  int64_t epoch = 0;
  cudaEvent_t ev[kEventRing] = {};
  int64_t ev_epoch[kEventRing];
  Staging stg[kStagingSlots];
  int next_stg = 0;
  cudaEvent_t pagein_done = nullptr;
  bool pagein_pending = false;
  std::vector<uint8_t> kv_page;       // 1: the page is held as a KV block
  int64_t kv_held = 0;
  cudaEvent_t rel_ev[kRelRing] = {};
  int64_t n_rel = 0;                  // release events recorded so far
  PoolDev pd{};
  int sm_count = 148;
  int grid_shrink = 0, grid_expand = 0, grid_stream = 0;
  int inject_after = -1;
  cudaEvent_t phase_ev[8] = {};
  int n_phase = 0;
  slora_pool_stats_t st{};
  std::string err;

  slora_status_t fail(slora_status_t s, const std::string& m) {
    err = std::string(status_name(s)) + ": " + m;
    if (getenv("SLORA_LOG")) fprintf(stderr, "slora: %s\n", err.c_str());
    return s;
  }
  slora_status_t cuda_fail(cudaError_t e, const char* where) {
    err = std::string("CUDA error in ") + where + ": " + cudaGetErrorString(e);
    if (getenv("SLORA_LOG")) fprintf(stderr, "slora: %s\n", err.c_str());
    cudaGetLastError();  // a non-sticky error must not resurface at the next launch check
    return SLORA_ERR_CUDA;
  }
  int64_t pages_for(int rank) const {
    int64_t n = 0;
    for (int p = 0; p < d.n_proj; ++p)
      n += cdiv64(tensor_units(d, rank, d.d_in[p]), d.page_elems) +
           cdiv64(tensor_units(d, rank, d.d_out[p]), d.page_elems);
    return n;
  }
  bool e4m3() const { return d.weight_format == SLORA_WEIGHTS_E4M3; }
  char* tables() const { return static_cast<char*>(d.dev_tables); }
  char* scratch() const { return static_cast<char*>(d.dev_scratch); }
};

#define CUDA_TRY(pool, call)                                  \
  do {                                                        \
    cudaError_t e_ = (call);                                  \
    if (e_ != cudaSuccess) return (pool)->cuda_fail(e_, #call); \
  } while (0)

// ---------------------------------------------------------------------------
// helpers
namespace {

slora_status_t validate_desc(const slora_pool_desc* d, std::string* why) {
  auto bad = [&](const char* m) {
    *why = m;
    return SLORA_ERR_INVALID_ARG;
  };
  if (!d) return bad("desc is NULL");
  if (d->dtype != SLORA_F16 && d->dtype != SLORA_BF16) return bad("dtype must be F16 or BF16");
  if (d->n_proj < 1 || d->n_proj > SLORA_MAX_PROJ) return bad("n_proj out of range");
  for (int p = 0; p < d->n_proj; ++p)
    if (d->d_in[p] <= 0 || d->d_out[p] <= 0 || d->d_in[p] % 64 || d->d_out[p] % 64 ||
        d->d_in[p] > 32768)
      return bad("d_in/d_out must be positive multiples of 64, d_in <= 32768");
  if (d->max_adapters < 1 || d->max_adapters > 16384) return bad("max_adapters out of [1, 16384]");
  if (d->max_rank < 0 || d->max_rank > 128) return bad("max_rank out of [0, 128]");
  if (d->max_tokens < 1 || d->max_tokens > (1 << 20)) return bad("max_tokens out of [1, 2^20]");
  if (d->page_elems < 512 || (d->page_elems & (d->page_elems - 1))) return bad("page_elems must be a power of two >= 512");
  if (d->n_pages < 0 || d->n_pages > (int64_t)INT32_MAX) return bad("n_pages out of range");
  if (d->pagein_mode != SLORA_PAGEIN_KERNEL && d->pagein_mode != SLORA_PAGEIN_MEMCPY)
    return bad("pagein_mode");
  if (d->decode_path < SLORA_DECODE_AUTO || d->decode_path > SLORA_DECODE_STREAM) return bad("decode_path");
  if (d->weight_format != SLORA_WEIGHTS_16 && d->weight_format != SLORA_WEIGHTS_E4M3) return bad("weight_format");
  if (!d->host_only) {
    if (!d->dev_pool && d->n_pages > 0) return bad("dev_pool is NULL");
    if (!d->dev_tables || !d->dev_scratch) return bad("dev_tables/dev_scratch is NULL");
    if ((uintptr_t)d->dev_pool % 16 || (uintptr_t)d->dev_tables % 256 || (uintptr_t)d->dev_scratch % 256)
      return bad("misaligned device buffer (pool 16 B, tables and scratch 256 B)");
    if (d->scratch_bytes < scratch_layout(*d).total) return bad("scratch_bytes below slora_scratch_bytes()");
  }
  return SLORA_OK;
}

// Device-side wait (no host block) for the compute of `epoch` to finish.
cudaError_t wait_epoch(slora_pool* P, cudaStream_t s, int64_t epoch) {
  if (epoch < 0) return cudaSuccess;
  const int slot = (int)(epoch % kEventRing);
  if (P->ev_epoch[slot] >= epoch) return cudaStreamWaitEvent(s, P->ev[slot], 0);
  return cudaSuccess;
}

// Timing hook: with 2 events only the call's start and end are recorded (the
// kernels stay back to back); with >= 4 also the boundaries between kernels.
void phase(slora_pool* P, int k, int last, cudaStream_t s) {
  if (P->n_phase == 2) {
    if (k == 0) cudaEventRecord(P->phase_ev[0], s);
    else if (k == last) cudaEventRecord(P->phase_ev[1], s);
  } else if (P->n_phase >= 4 && k < P->n_phase) {
    cudaEventRecord(P->phase_ev[k], s);
  }
}

cudaError_t record_epoch(slora_pool* P, cudaStream_t s) {
  const int slot = (int)(P->epoch % kEventRing);
  const cudaError_t e = cudaEventRecord(P->ev[slot], s);
  if (e == cudaSuccess) P->ev_epoch[slot] = P->epoch;
  return e;
}

// Bounded host wait on an event.
slora_status_t wait_event_bounded(slora_pool* P, cudaEvent_t e) {
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    cudaError_t q = cudaEventQuery(e);
    if (q == cudaSuccess) return SLORA_OK;
    if (q != cudaErrorNotReady) return P->cuda_fail(q, "cudaEventQuery");
    if (std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count() > kWaitSeconds)
      return P->fail(SLORA_ERR_TIMEOUT, "page-in staging slot did not drain");
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

void fill_pool_dev(slora_pool* P) {
  P->pd.pool = static_cast<uint16_t*>(P->d.dev_pool);
  int sh = 0;
  while ((1ll << sh) < P->d.page_elems) ++sh;
  P->pd.page_shift = sh;
  P->pd.max_adapters = P->d.max_adapters;
  P->pd.max_rank = P->d.max_rank;
  P->pd.list_stride = P->list_stride;
  P->pd.rank = reinterpret_cast<int32_t*>(P->tables() + P->tl.off_rank);
  P->pd.scale = reinterpret_cast<float*>(P->tables() + P->tl.off_scale);
  P->pd.page_list = reinterpret_cast<int32_t*>(P->tables() + P->tl.off_list);
  P->pd.err = reinterpret_cast<int32_t*>(P->tables() + P->tl.off_err);
  P->pd.qscale = P->e4m3() ? reinterpret_cast<float*>(P->tables() + P->tl.off_qscale) : nullptr;
  P->pd.wfmt = P->d.weight_format;
  P->pd.n_proj = P->d.n_proj;
}

ScratchDev scratch_at(char* b, const ScratchLayout& L) {
  ScratchDev s{};
  s.meta = reinterpret_cast<int32_t*>(b + L.off_meta);
  s.perm = reinterpret_cast<int32_t*>(b + L.off_perm);
  s.seg_start = reinterpret_cast<int32_t*>(b + L.off_seg_start);
  s.seg_adapter = reinterpret_cast<int32_t*>(b + L.off_seg_adapter);
  s.seg_rank = reinterpret_cast<int32_t*>(b + L.off_seg_rank);
  s.ready = reinterpret_cast<int32_t*>(b + L.off_ready);
  s.shrink_prefix = reinterpret_cast<int32_t*>(b + L.off_shrink_pre);
  s.expand_prefix = reinterpret_cast<int32_t*>(b + L.off_expand_pre);
  s.MS = L.MS;
  return s;
}

ScratchDev scratch_dev(slora_pool* P) { return scratch_at(P->scratch(), P->sl); }

// Points each slot's t at its share of the fp32 partials region (position-
// ordered rows of rk8 * nsplit floats for T tokens).  False when they do not fit.
bool assign_partials(BgmvParams& bp, float* base, int64_t cap_floats, int64_t T, int64_t rk8) {
  int64_t off = 0;
  for (int k = 0; k < bp.n_slots; ++k) {
    SlotDev& S = bp.slot[k];
    S.t = base + off;
    S.t_rs = rk8 * S.nsplit;
    S.t_ns = S.nsplit;
    S.t_by_token = 0;
    S.tout = nullptr;
    S.ldt_out = 0;
    off += (int64_t)S.nsplit * T * rk8;
  }
  return off <= cap_floats;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// Builds the slot / group blocks of a compute call.  x may be NULL per slot
// when do_shrink == 0.
slora_status_t plan_slots(slora_pool* P, BgmvParams& bp, int n, const int32_t* projs,
                          const void* const* x, const int64_t* ldx, void* const* y,
                          const int64_t* ldy, int T, bool need_x, bool need_y) {
  if (n < 1 || n > kMaxSlots) return P->fail(SLORA_ERR_INVALID_ARG, "n out of [1, 8]");
  if (!projs) return P->fail(SLORA_ERR_INVALID_ARG, "projs is NULL");
  bp.n_slots = n;
  bp.n_groups = 0;
  for (int k = 0; k < n; ++k) {
    const int p = projs[k];
    if (p < 0 || p >= P->d.n_proj) return P->fail(SLORA_ERR_INVALID_ARG, "projection id out of range");
    SlotDev& S = bp.slot[k];
    S = SlotDev{};
    S.d_in = P->d.d_in[p];
    S.d_out = P->d.d_out[p];
    S.listA = P->listA[p];
    S.listB = P->listB[p];
    S.proj = p;
    S.nsplit = (int)cdiv64(S.d_in, kPartK);
    if (need_x) {
      if (!x || !ldx || !x[k]) return P->fail(SLORA_ERR_INVALID_ARG, "x is NULL");
      if (ldx[k] < S.d_in || ldx[k] % 8 || !aligned16(x[k]))
        return P->fail(SLORA_ERR_INVALID_ARG, "x must be 16-byte aligned with ldx >= d_in, ldx % 8 == 0");
      S.x = static_cast<const uint16_t*>(x[k]);
      S.ldx = ldx[k];
    }
    if (need_y) {
      if (!y || !ldy || !y[k]) return P->fail(SLORA_ERR_INVALID_ARG, "y is NULL");
      if (ldy[k] < S.d_out || ldy[k] % 8 || !aligned16(y[k]))
        return P->fail(SLORA_ERR_INVALID_ARG, "y must be 16-byte aligned with ldy >= d_out, ldy % 8 == 0");
      S.y = static_cast<uint16_t*>(y[k]);
      S.ldy = ldy[k];
    }
    // x-sharing groups
    int g = -1;
    if (need_x)
      for (int q = 0; q < bp.n_groups; ++q)
        if (bp.group[q].x == S.x && bp.group[q].ldx == S.ldx && bp.group[q].d_in == S.d_in) g = q;
    if (g < 0) {
      g = bp.n_groups++;
      bp.group[g] = GroupDev{};
      bp.group[g].x = S.x;
      bp.group[g].ldx = S.ldx;
      bp.group[g].d_in = S.d_in;
    }
    S.group = g;
    S.gpos = bp.group[g].n;
    bp.group[g].slot[bp.group[g].n++] = k;
  }
  if (!assign_partials(bp, reinterpret_cast<float*>(P->scratch() + P->sl.off_tpart), P->sl.tpart_floats,
                       P->d.max_tokens, P->sl.rk8))
    return P->fail(SLORA_ERR_INVALID_ARG, "too many projections in one call for the scratch size");
  if (T < 0 || T > P->d.max_tokens) return P->fail(SLORA_ERR_INVALID_ARG, "T out of [0, max_tokens]");
  return SLORA_OK;
}

void base_params(slora_pool* P, BgmvParams& bp) {
  bp = BgmvParams{};
  bp.pool = P->pd;
  bp.sc = scratch_dev(P);
  bp.max_tokens = P->d.max_tokens;
}

slora_status_t need_device(slora_pool* P) {
  if (P->d.host_only) return P->fail(SLORA_ERR_UNSUPPORTED, "pool was created host_only");
  return SLORA_OK;
}

// Whether a decode call of T tokens runs as one CTA per token (AUTO, 16-bit
// weights, at most kTokenMaxT tokens: a latency-bound batch).
bool token_path(const slora_pool* P, int T) {
  return P->d.decode_path == SLORA_DECODE_AUTO && P->d.weight_format == SLORA_WEIGHTS_16 && T <= kTokenMaxT;
}

// Whether a decode call of T tokens runs as the one persistent kernel.
bool fused_path(const slora_pool* P, int T) {
  return T <= kFMaxT && P->d.decode_path == SLORA_DECODE_FUSED;
}

// Whether a decode call of T tokens runs as the one kernel of streaming stages.
// AUTO takes it for 17..kFMaxT tokens (16-bit) and for every call of an e4m3
// pool up to kFMaxT: on B200 it is the faster of the measured kernels at 256,
// 512 and 1024 tokens (LLaMA-7B, -13B and -70B layers); larger 16-bit calls
// take the three-kernel path, which has no token limit.
bool stream_path(const slora_pool* P, int T) {
  if (T > kFMaxT) return false;
  if (P->d.decode_path == SLORA_DECODE_STREAM) return true;
  return P->d.decode_path == SLORA_DECODE_AUTO && !token_path(P, T);
}

// The decode delta's kernels for a planned call (both phases): the one
// persistent kernel or the three-kernel path (fused_path); timing events
// (slora_set_phase_events) bracket each kernel when `timed`.
slora_status_t enqueue_delta(slora_pool* P, BgmvParams& bp, const int32_t* idx, int T, cudaStream_t st,
                             bool timed) {
  bp.do_shrink = 1;
  bp.do_expand = 1;
  if (P->e4m3() && !fused_path(P, T) && !stream_path(P, T))
    return P->fail(SLORA_ERR_UNSUPPORTED, "e4m3 weights: decode calls of up to 1024 tokens on a one-kernel path");
  if (token_path(P, T)) {
    if (timed) phase(P, 0, 1, st);
    CUDA_TRY(P, launch_token(bp, P->d.dtype, idx, T, st));
    if (timed) phase(P, 1, 1, st);
    return SLORA_OK;
  }
  if (stream_path(P, T)) {
    if (timed) phase(P, 0, 1, st);
    CUDA_TRY(P, launch_stream(bp, P->d.dtype, idx, T, P->grid_stream, st));
    if (timed) phase(P, 1, 1, st);
    return SLORA_OK;
  }
  if (fused_path(P, T)) {
    const int grid = std::max(1, std::min(P->sm_count, fused_grid_bound(bp, T)));
    if (timed) phase(P, 0, 1, st);
    CUDA_TRY(P, launch_fused(bp, P->d.dtype, idx, T, grid, st));
    if (timed) phase(P, 1, 1, st);
    return SLORA_OK;
  }
  if (timed) phase(P, 0, 3, st);
  CUDA_TRY(P, launch_segments(bp, idx, T, st));
  if (timed) phase(P, 1, 3, st);
  CUDA_TRY(P, launch_shrink(bp, P->d.dtype, P->grid_shrink, st));
  if (timed) phase(P, 2, 3, st);
  CUDA_TRY(P, launch_expand(bp, P->d.dtype, P->grid_expand, st));
  if (timed) phase(P, 3, 3, st);
  return SLORA_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// The fused decode delta on a caller-chosen scratch region instead of the
// pool's dev_scratch; used by the no-allocation entry point (noalloc.cu).
// Kernels, launch order and arithmetic are those of slora_lora_delta; only the
// scratch addresses differ, laid out for this call's T tokens.
namespace slora {
slora_status_t lora_delta_on_scratch(slora_pool* P, int32_t n, const int32_t* projs,
                                     const void* const* x, const int64_t* ldx, void* const* y,
                                     const int64_t* ldy, const int32_t* idx, int32_t T,
                                     cudaStream_t st, void* scratch, size_t scratch_cap) {
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  if (T > 0 && !idx) return P->fail(SLORA_ERR_INVALID_ARG, "idx is NULL");
  BgmvParams bp;
  base_params(P, bp);
  s = plan_slots(P, bp, n, projs, x, ldx, y, ldy, T, true, true);
  if (s) return s;
  if (T == 0) return SLORA_OK;
  slora_pool_desc dd = P->d;
  dd.max_tokens = T;
  const ScratchLayout L = scratch_layout(dd);
  // the decode part of the layout: tables, then the fp32 partials of the
  // projections this call names (not of every projection of the pool)
  int64_t part_floats = 0;
  for (int k = 0; k < bp.n_slots; ++k) part_floats += (int64_t)bp.slot[k].nsplit * T * L.rk8;
  const size_t need = L.off_tpart + 4 * (size_t)part_floats;
  if (need > scratch_cap)
    return P->fail(SLORA_ERR_INVALID_ARG,
                   "this call needs " + std::to_string(need) + " bytes of scratch; the static "
                   "no-allocation scratch holds " + std::to_string(scratch_cap) +
                   " (fewer tokens, projections or a smaller max_rank fit)");
  char* b = static_cast<char*>(scratch);
  bp.max_tokens = T;
  bp.sc = scratch_at(b, L);
  if (!assign_partials(bp, reinterpret_cast<float*>(b + L.off_tpart), part_floats, T, L.rk8))
    return P->fail(SLORA_ERR_INVALID_ARG, "too many projections in one call");
  s = enqueue_delta(P, bp, idx, T, st, false);
  if (s) return s;
  CUDA_TRY(P, record_epoch(P, st));
  return SLORA_OK;
}
}  // namespace slora

// ---------------------------------------------------------------------------
// C ABI
extern "C" {

size_t slora_tables_bytes(const slora_pool_desc* d) {
  std::string why;
  if (!d || d->max_adapters < 1 || d->n_proj < 1 || d->n_proj > SLORA_MAX_PROJ || d->page_elems < 1) return 0;
  return table_layout(*d).total;
}

size_t slora_scratch_bytes(const slora_pool_desc* d) {
  if (!d || d->max_tokens < 1 || d->n_proj < 1 || d->n_proj > SLORA_MAX_PROJ) return 0;
  return scratch_layout(*d).total;
}

int64_t slora_pages_for_rank(const slora_pool_desc* d, int32_t rank) {
  if (!d || rank < 0 || d->page_elems < 1) return -1;
  int64_t n = 0;
  for (int p = 0; p < d->n_proj && p < SLORA_MAX_PROJ; ++p)
    n += cdiv64(tensor_units(*d, rank, d->d_in[p]), d->page_elems) +
         cdiv64(tensor_units(*d, rank, d->d_out[p]), d->page_elems);
  return n;
}

slora_status_t slora_pool_create(const slora_pool_desc* desc, slora_pool** out) {
  NvtxRange nvtx_("slora_pool_create");
  if (!out) return SLORA_ERR_INVALID_ARG;
  *out = nullptr;
  std::string why;
  slora_status_t s = validate_desc(desc, &why);
  if (s != SLORA_OK) {
    if (getenv("SLORA_LOG")) fprintf(stderr, "slora_pool_create: %s\n", why.c_str());
    return s;
  }
  slora_pool* P = new slora_pool();
  P->d = *desc;
  P->list_stride = list_stride_of(P->d, P->listA, P->listB);
  P->tl = table_layout(P->d);
  P->sl = scratch_layout(P->d);
  P->ad.resize(P->d.max_adapters);
  for (int64_t pg = 0; pg < P->d.n_pages; ++pg) P->free_pages.push_back({(int32_t)pg, -1, -1});
  P->kv_page.assign((size_t)P->d.n_pages, 0);
  for (int i = 0; i < kEventRing; ++i) P->ev_epoch[i] = -1;
  P->st.free_pages = P->d.n_pages;
  if (!P->d.host_only) {
    fill_pool_dev(P);
    cudaError_t e = cudaSuccess;
    int dev = 0;
    if (e == cudaSuccess) e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&P->sm_count, cudaDevAttrMultiProcessorCount, dev);
    for (int i = 0; i < kEventRing && e == cudaSuccess; ++i)
      e = cudaEventCreateWithFlags(&P->ev[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&P->pagein_done, cudaEventDisableTiming);
    for (int i = 0; i < kRelRing && e == cudaSuccess; ++i)
      e = cudaEventCreateWithFlags(&P->rel_ev[i], cudaEventDisableTiming);
    for (int i = 0; i < kStagingSlots && e == cudaSuccess; ++i)
      e = cudaEventCreateWithFlags(&P->stg[i].done, cudaEventDisableTiming);
    // tables: rank = -1 (0xff bytes), scale = 0, err = 0, page lists = -1
    if (e == cudaSuccess) e = cudaMemset(P->tables(), 0, P->tl.off_list);
    if (e == cudaSuccess) e = cudaMemset(P->tables() + P->tl.off_rank, 0xff, 4 * (size_t)P->d.max_adapters);
    if (e == cudaSuccess)
      e = cudaMemset(P->tables() + P->tl.off_list, 0xff, 4 * (size_t)P->d.max_adapters * P->list_stride);
    if (e == cudaSuccess) e = cudaMemset(P->scratch(), 0, P->sl.off_perm);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
      if (getenv("SLORA_LOG")) fprintf(stderr, "slora_pool_create: %s\n", cudaGetErrorString(e));
      slora_pool_destroy(P);
      return SLORA_ERR_CUDA;
    }
    P->grid_shrink = P->sm_count * occupancy_blocks(0);
    P->grid_expand = P->sm_count * occupancy_blocks(1);
    P->grid_stream = P->sm_count * stream_blocks_per_sm(P->d.max_adapters);
  }
  *out = P;
  return SLORA_OK;
}

slora_status_t slora_pool_destroy(slora_pool* P) {
  NvtxRange nvtx_("slora_pool_destroy");
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (!P->d.host_only) {
    if (P->pagein_done) {
      if (P->pagein_pending) wait_event_bounded(P, P->pagein_done);
      cudaEventDestroy(P->pagein_done);
    }
    for (int i = 0; i < kStagingSlots; ++i) {
      if (P->stg[i].done) {
        if (P->stg[i].pending) wait_event_bounded(P, P->stg[i].done);
        cudaEventDestroy(P->stg[i].done);
      }
      if (P->stg[i].host) cudaFreeHost(P->stg[i].host);
    }
    for (int i = 0; i < kEventRing; ++i)
      if (P->ev[i]) cudaEventDestroy(P->ev[i]);
    for (int i = 0; i < kRelRing; ++i)
      if (P->rel_ev[i]) cudaEventDestroy(P->rel_ev[i]);
  }
  delete P;
  return SLORA_OK;
}

const char* slora_last_error(const slora_pool* P) { return P ? P->err.c_str() : "pool is NULL"; }

slora_status_t slora_pool_set_page_order(slora_pool* P, const int32_t* order, int64_t n) {
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (!order || n != P->d.n_pages) return P->fail(SLORA_ERR_INVALID_ARG, "order must list n_pages ids");
  if (!P->lru.empty() || P->kv_held) return P->fail(SLORA_ERR_INVALID_ARG, "only allowed while no page is held");
  std::vector<char> seen(n, 0);
  for (int64_t i = 0; i < n; ++i) {
    if (order[i] < 0 || order[i] >= n || seen[order[i]]) return P->fail(SLORA_ERR_INVALID_ARG, "order is not a permutation");
    seen[order[i]] = 1;
  }
  std::deque<FreePage> fp;
  for (int64_t i = 0; i < n; ++i) fp.push_back({order[i], -1, -1});
  P->free_pages.swap(fp);
  return SLORA_OK;
}

static slora_status_t register_impl(slora_pool* P, int32_t id, int32_t rank, float alpha,
                                    const void* const* host_A_t, const void* const* host_B,
                                    const float* const* scales_A_t, const float* const* scales_B) {
  if (id < 0 || id >= P->d.max_adapters) return P->fail(SLORA_ERR_INVALID_ARG, "adapter id out of range");
  if (rank < 0 || rank > P->d.max_rank) return P->fail(SLORA_ERR_INVALID_ARG, "rank out of [0, max_rank]");
  Adapter& A = P->ad[id];
  if (A.resident) return P->fail(SLORA_ERR_INVALID_ARG, "adapter is resident; evict it first");
  if (rank > 0 && (!host_A_t || !host_B)) return P->fail(SLORA_ERR_INVALID_ARG, "weight pointers are NULL");
  const bool q8 = P->e4m3();
  if (q8 && rank > 0 && (!scales_A_t || !scales_B)) return P->fail(SLORA_ERR_INVALID_ARG, "scale pointers are NULL");
  Adapter N;
  N.registered = true;
  N.rank = rank;
  N.alpha = alpha;
  N.last_use = A.last_use;
  if (q8) N.qs.assign((size_t)P->d.n_proj * 2 * rank, 0.f);
  for (int p = 0; p < P->d.n_proj && rank > 0; ++p) {
    if (!host_A_t[p] || !host_B[p]) return P->fail(SLORA_ERR_INVALID_ARG, "weight pointer is NULL");
    if (!aligned16(host_A_t[p]) || !aligned16(host_B[p]))
      return P->fail(SLORA_ERR_INVALID_ARG, "weights must be 16-byte aligned");
    if (q8) {
      if (!scales_A_t[p] || !scales_B[p]) return P->fail(SLORA_ERR_INVALID_ARG, "scale pointer is NULL");
      for (int k = 0; k < rank; ++k) {
        const float a = scales_A_t[p][k], b = scales_B[p][k];
        if (!(a >= 0.f) || !(b >= 0.f) || !std::isfinite(a) || !std::isfinite(b))
          return P->fail(SLORA_ERR_INVALID_ARG, "scales must be finite and non-negative");
        N.qs[((size_t)p * 2 + 0) * rank + k] = a;
        N.qs[((size_t)p * 2 + 1) * rank + k] = b;
      }
    }
    N.host_A[p] = host_A_t[p];
    N.host_B[p] = host_B[p];
    N.map_A[p] = host_A_t[p];
    N.map_B[p] = host_B[p];
    if (!P->d.host_only) {
      for (int m = 0; m < 2; ++m) {
        const void* h = m ? host_B[p] : host_A_t[p];
        cudaPointerAttributes at;
        cudaError_t e = cudaPointerGetAttributes(&at, h);
        if (e != cudaSuccess || at.type != cudaMemoryTypeHost) {
          cudaGetLastError();
          return P->fail(SLORA_ERR_INVALID_ARG, "weights must be in pinned host memory");
        }
        void* dp = nullptr;
        e = cudaHostGetDevicePointer(&dp, const_cast<void*>(h), 0);
        if (e != cudaSuccess) {
          cudaGetLastError();
          return P->fail(SLORA_ERR_INVALID_ARG, "pinned weights are not mapped for the device");
        }
        (m ? N.map_B[p] : N.map_A[p]) = dp;
      }
    }
  }
  A = N;
  return SLORA_OK;
}

slora_status_t slora_adapter_register(slora_pool* P, int32_t id, int32_t rank, float alpha,
                                      const void* const* host_A_t, const void* const* host_B) {
  NvtxRange nvtx_("slora_adapter_register");
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (P->e4m3()) return P->fail(SLORA_ERR_INVALID_ARG, "the pool holds e4m3 weights: use slora_adapter_register_e4m3");
  return register_impl(P, id, rank, alpha, host_A_t, host_B, nullptr, nullptr);
}

slora_status_t slora_adapter_register_e4m3(slora_pool* P, int32_t id, int32_t rank, float alpha,
                                           const void* const* codes_A_t, const float* const* scales_A_t,
                                           const void* const* codes_B, const float* const* scales_B) {
  NvtxRange nvtx_("slora_adapter_register_e4m3");
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (!P->e4m3()) return P->fail(SLORA_ERR_INVALID_ARG, "the pool holds 16-bit weights: use slora_adapter_register");
  return register_impl(P, id, rank, alpha, codes_A_t, codes_B, scales_A_t, scales_B);
}

static void evict_one(slora_pool* P, int id) {
  Adapter& A = P->ad[id];
  P->lru.erase({A.last_use, id});
  for (int32_t pg : A.pages) P->free_pages.push_back({pg, A.last_use, -1});
  A.pages.clear();
  A.resident = false;
  P->st.evictions++;
}

// Shared by page_in and prefetch.  page_in (prefetch = false): every id
// becomes resident, evicting LRU adapters not named; the named set becomes
// the step's set.  prefetch: the non-resident ids, in order, that fit in
// max_pages (and in the free pages plus the pages of adapters older than the
// current step) become resident; nothing the current step or an earlier
// prefetch of this step holds is evicted, and the step's set is unchanged.
static slora_status_t page_in_impl(slora_pool* P, const int32_t* ids, int32_t n, void* side_stream,
                                   void* done_event, bool prefetch, int64_t max_pages, int32_t* n_done) {
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (n < 0 || (n > 0 && !ids)) return P->fail(SLORA_ERR_INVALID_ARG, "ids");
  if (prefetch && max_pages < 0) return P->fail(SLORA_ERR_INVALID_ARG, "max_pages < 0");
  cudaStream_t side = static_cast<cudaStream_t>(side_stream);
  std::vector<int> uniq;
  std::unordered_set<int> pinned;
  for (int i = 0; i < n; ++i) {
    const int a = ids[i];
    if (a < 0 || a >= P->d.max_adapters) return P->fail(SLORA_ERR_INVALID_ARG, "adapter id out of range");
    if (!P->ad[a].registered) return P->fail(SLORA_ERR_NOT_REGISTERED, "adapter " + std::to_string(a));
    if (pinned.insert(a).second) uniq.push_back(a);
  }
  std::vector<int> missing;
  int64_t need = 0;
  std::vector<int> victims;
  if (!prefetch) {
    for (int a : uniq)
      if (!P->ad[a].resident) {
        missing.push_back(a);
        need += P->pages_for(P->ad[a].rank);
      }
    // LRU victims: oldest first, equal ages lower id first (std::set order)
    int64_t avail = (int64_t)P->free_pages.size();
    for (auto it = P->lru.begin(); avail < need && it != P->lru.end(); ++it) {
      if (pinned.count(it->second)) continue;
      victims.push_back(it->second);
      avail += (int64_t)P->ad[it->second].pages.size();
    }
    if (avail < need)
      return P->fail(SLORA_ERR_OOM, "cannot fit " + std::to_string(need) + " pages with all unpinned adapters evicted");
  } else {
    // evictable: resident adapters older than the current step (the step's
    // set and this step's prefetches have last_use == epoch)
    int64_t cap = (int64_t)P->free_pages.size();
    for (const auto& e : P->lru)
      if (e.first < P->epoch) cap += (int64_t)P->ad[e.second].pages.size();
    const int64_t limit = std::min(cap, max_pages);
    for (int a : uniq) {
      if (P->ad[a].resident) continue;
      const int64_t np = P->pages_for(P->ad[a].rank);
      if (need + np > limit) continue;  // does not fit: try the next one
      missing.push_back(a);
      need += np;
    }
    int64_t avail = (int64_t)P->free_pages.size();
    for (auto it = P->lru.begin(); avail < need && it != P->lru.end(); ++it) {
      if (it->first >= P->epoch) break;  // std::set order: the rest are as new
      victims.push_back(it->second);
      avail += (int64_t)P->ad[it->second].pages.size();
    }
  }
  if (n_done) *n_done = 0;
  if (P->inject_after >= 0 && !missing.empty()) {
    if (P->inject_after == 0) {
      P->inject_after = -1;
      return P->fail(SLORA_ERR_INJECTED, "planted page-in copy failure");
    }
    P->inject_after--;
  }
  // staging slot (device mode)
  Staging* stg = nullptr;
  if (!P->d.host_only && !missing.empty()) {
    stg = &P->stg[P->next_stg];
    if (stg->pending) {
      slora_status_t ws = wait_event_bounded(P, stg->done);
      if (ws != SLORA_OK) return ws;
      stg->pending = false;
    }
  }
  // ---- commit host state
  std::set<int> rel_wait;  // release events of freed KV blocks among the pages taken
  for (int v : victims) evict_one(P, v);
  int64_t wait_ep = -1;
  for (int v : victims) wait_ep = std::max(wait_ep, P->ad[v].last_use);
  for (int a : missing) {
    Adapter& A = P->ad[a];
    const int64_t np = P->pages_for(A.rank);
    A.pages.resize(np);
    for (int64_t i = 0; i < np; ++i) {
      FreePage f = P->free_pages.front();
      P->free_pages.pop_front();
      A.pages[i] = f.id;
      wait_ep = std::max(wait_ep, f.free_epoch);
      if (f.rel >= 0) rel_wait.insert(f.rel);
    }
    A.resident = true;
    if (!prefetch) P->st.page_ins++;
    (prefetch ? P->st.bytes_prefetched : P->st.bytes_paged_in) +=
        [&] { int64_t s = 0; for (int p = 0; p < P->d.n_proj; ++p)
                s += 2 * (tensor_units(P->d, A.rank, P->d.d_in[p]) + tensor_units(P->d, A.rank, P->d.d_out[p]));
              return s; }();
  }
  if (!prefetch) {
    P->st.hits += (int64_t)(uniq.size() - missing.size());
    P->epoch++;
    for (int a : uniq) {
      Adapter& A = P->ad[a];
      if (A.resident && A.last_use >= 0) P->lru.erase({A.last_use, a});
      A.last_use = P->epoch;
      A.named = P->epoch;
      A.uses[A.n_uses % kUseHistory] = P->epoch;
      A.n_uses++;
      P->lru.insert({A.last_use, a});
    }
  } else {
    // as recent as the current step's set in the LRU order; usable by a
    // compute call only once a later page_in names it
    for (int a : missing) {
      Adapter& A = P->ad[a];
      A.last_use = P->epoch;
      P->lru.insert({A.last_use, a});
    }
    P->st.prefetched += (int64_t)missing.size();
  }
  P->st.epoch = P->epoch;
  P->st.free_pages = (int64_t)P->free_pages.size();
  P->st.resident = (int64_t)P->lru.size();
  if (n_done) *n_done = (int32_t)missing.size();
  if (P->d.host_only) return SLORA_OK;

  // ---- device work on the side stream
  if (!missing.empty() || !victims.empty()) {
    // descriptor
    const int64_t stride = P->list_stride;
    size_t off_evict = align_up(sizeof(PageInHeader), 16);
    size_t off_new = align_up(off_evict + 4 * victims.size(), 16);
    size_t off_lists = align_up(off_new + sizeof(PageInNew) * missing.size(), 16);
    size_t off_qs = align_up(off_lists + 4 * (size_t)stride * missing.size(), 16);
    size_t bytes = off_qs;
    for (int a : missing) bytes += 4 * P->ad[a].qs.size();
    if (!stg) {
      stg = &P->stg[P->next_stg];
      if (stg->pending) {
        slora_status_t ws = wait_event_bounded(P, stg->done);
        if (ws != SLORA_OK) return ws;
        stg->pending = false;
      }
    }
    if (bytes > P->tl.desc_cap) return P->fail(SLORA_ERR_INVALID_ARG, "page-in descriptor exceeds its area");
    if (stg->cap < bytes) {
      if (stg->host) cudaFreeHost(stg->host);
      stg->host = nullptr;
      stg->cap = 0;
      size_t cap = std::max<size_t>(bytes, 1 << 20);
      CUDA_TRY(P, cudaHostAlloc(&stg->host, cap, cudaHostAllocDefault));
      stg->cap = cap;
    }
    char* h = static_cast<char*>(stg->host);
    PageInHeader* H = reinterpret_cast<PageInHeader*>(h);
    H->n_new = (int32_t)missing.size();
    H->n_evict = (int32_t)victims.size();
    H->n_proj = P->d.n_proj;
    H->copy_data = P->d.pagein_mode == SLORA_PAGEIN_KERNEL;
    H->list_stride = stride;
    H->off_evict = (int64_t)off_evict;
    H->off_new = (int64_t)off_new;
    int32_t* ev = reinterpret_cast<int32_t*>(h + off_evict);
    for (size_t i = 0; i < victims.size(); ++i) ev[i] = victims[i];
    PageInNew* nw = reinterpret_cast<PageInNew*>(h + off_new);
    int64_t units = 0;
    size_t qs_at = off_qs;
    for (size_t i = 0; i < missing.size(); ++i) {
      const Adapter& A = P->ad[missing[i]];
      PageInNew& w = nw[i];
      memset(&w, 0, sizeof(w));
      w.id = missing[i];
      w.rank = A.rank;
      w.scale = A.rank > 0 ? A.alpha / (float)A.rank : 0.f;
      w.n_units = (int32_t)A.pages.size();
      w.unit_base = units;
      units += (int64_t)A.pages.size();
      w.list_off = (int64_t)(off_lists + 4 * (size_t)stride * i);
      w.qs_off = A.qs.empty() ? -1 : (int64_t)qs_at;
      if (!A.qs.empty()) {
        memcpy(h + qs_at, A.qs.data(), 4 * A.qs.size());
        qs_at += 4 * A.qs.size();
      }
      for (int p = 0; p < P->d.n_proj; ++p) {
        w.host[p][0] = static_cast<const uint16_t*>(A.map_A[p]);
        w.host[p][1] = static_cast<const uint16_t*>(A.map_B[p]);
      }
      int32_t* row = reinterpret_cast<int32_t*>(h + w.list_off);
      for (int64_t e = 0; e < stride; ++e) row[e] = -1;
      int64_t c = 0;
      for (int p = 0; p < P->d.n_proj; ++p) {
        const int64_t na = cdiv64(tensor_units(P->d, A.rank, P->d.d_in[p]), P->d.page_elems);
        for (int64_t j = 0; j < na; ++j) row[P->listA[p] + j] = A.pages[c++];
        const int64_t nb = cdiv64(tensor_units(P->d, A.rank, P->d.d_out[p]), P->d.page_elems);
        for (int64_t j = 0; j < nb; ++j) row[P->listB[p] + j] = A.pages[c++];
      }
    }
    H->total_units = units;
    // device-side ordering: previous page-in done (descriptor area), and the
    // compute that last read the pages being reused
    if (P->pagein_pending) CUDA_TRY(P, cudaStreamWaitEvent(side, P->pagein_done, 0));
    CUDA_TRY(P, wait_epoch(P, side, wait_ep));
    for (int r : rel_wait) CUDA_TRY(P, cudaStreamWaitEvent(side, P->rel_ev[r], 0));
    char* desc_dev = P->tables() + P->tl.off_desc;
    CUDA_TRY(P, cudaMemcpyAsync(desc_dev, h, bytes, cudaMemcpyHostToDevice, side));
    CUDA_TRY(P, cudaEventRecord(stg->done, side));
    stg->pending = true;
    P->next_stg = (P->next_stg + 1) % kStagingSlots;
    int grid = (int)std::min<int64_t>(std::max<int64_t>(units, 1), 2 * (int64_t)P->sm_count);
    if (missing.size() > (size_t)grid) grid = (int)std::min<size_t>(missing.size(), 4096);
    int u_in[kMaxSlots], u_out[kMaxSlots];  // tensor widths in 16-bit units
    for (int q = 0; q < kMaxSlots; ++q) {
      u_in[q] = P->e4m3() ? P->d.d_in[q] / 2 : P->d.d_in[q];
      u_out[q] = P->e4m3() ? P->d.d_out[q] / 2 : P->d.d_out[q];
    }
    CUDA_TRY(P, launch_page_in(P->pd, u_in, u_out, P->listA, P->listB, desc_dev, units, grid, side));
    P->st.copy_calls++;
    if (P->d.pagein_mode == SLORA_PAGEIN_MEMCPY) {
      const int64_t Pb = P->d.page_elems * 2;
      for (int a : missing) {
        const Adapter& A = P->ad[a];
        int64_t c = 0;
        for (int t = 0; t < 2 * P->d.n_proj; ++t) {
          const int p = t >> 1;
          const int64_t nel = tensor_units(P->d, A.rank, (t & 1) ? P->d.d_out[p] : P->d.d_in[p]);
          const int64_t np = cdiv64(nel, P->d.page_elems);
          const char* src = static_cast<const char*>((t & 1) ? A.host_B[p] : A.host_A[p]);
          int64_t j = 0;
          while (j < np) {
            int64_t run = 1;
            while (j + run < np && A.pages[c + j + run] == A.pages[c + j] + run) ++run;
            const int64_t bytes_run = std::min(run * P->d.page_elems, nel - j * P->d.page_elems) * 2;
            char* dst = static_cast<char*>(P->d.dev_pool) + (int64_t)A.pages[c + j] * Pb;
            CUDA_TRY(P, cudaMemcpyAsync(dst, src + j * Pb, bytes_run, cudaMemcpyHostToDevice, side));
            P->st.copy_calls++;
            j += run;
          }
          c += np;
        }
      }
    }
    CUDA_TRY(P, cudaEventRecord(P->pagein_done, side));
    P->pagein_pending = true;
  }
  // compute that waits on done_event must also see the copies of an earlier
  // prefetch (or page-in) of the adapters named here, made on any stream
  if (missing.empty() && victims.empty() && P->pagein_pending)
    CUDA_TRY(P, cudaStreamWaitEvent(side, P->pagein_done, 0));
  if (done_event) CUDA_TRY(P, cudaEventRecord(static_cast<cudaEvent_t>(done_event), side));
  return SLORA_OK;
}

slora_status_t slora_adapter_page_in(slora_pool* P, const int32_t* ids, int32_t n, void* side_stream,
                                     void* done_event) {
  NvtxRange nvtx_("slora_adapter_page_in");
  return page_in_impl(P, ids, n, side_stream, done_event, false, 0, nullptr);
}

slora_status_t slora_adapter_prefetch(slora_pool* P, const int32_t* ids, int32_t n, int64_t max_pages,
                                      void* side_stream, void* done_event, int32_t* n_done) {
  NvtxRange nvtx_("slora_adapter_prefetch");
  return page_in_impl(P, ids, n, side_stream, done_event, true, max_pages, n_done);
}

slora_status_t slora_prefetch_candidates(const slora_pool* Pc, double half_life, int32_t max_n, int32_t* out,
                                         int32_t* n_out) {
  slora_pool* P = const_cast<slora_pool*>(Pc);
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (!(half_life > 0) || max_n < 0 || (max_n > 0 && !out) || !n_out)
    return P->fail(SLORA_ERR_INVALID_ARG, "prefetch_candidates arguments");
  std::vector<std::pair<double, int>> cand;  // (-score, id)
  for (int a = 0; a < P->d.max_adapters; ++a) {
    const Adapter& A = P->ad[a];
    if (!A.registered || A.resident || A.n_uses == 0) continue;
    double score = 0.0;
    const int k = std::min(A.n_uses, kUseHistory);
    for (int j = 0; j < k; ++j) score += std::exp2(-(double)(P->epoch - A.uses[j]) / half_life);
    cand.push_back({-score, a});
  }
  std::sort(cand.begin(), cand.end());
  const int m = std::min<int64_t>(max_n, (int64_t)cand.size());
  for (int i = 0; i < m; ++i) out[i] = cand[i].second;
  *n_out = m;
  return SLORA_OK;
}

slora_status_t slora_kv_alloc(slora_pool* P, int64_t n, int32_t* ids_out, void* stream, void* done_event) {
  NvtxRange nvtx_("slora_kv_alloc");
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (n < 0 || (n > 0 && !ids_out)) return P->fail(SLORA_ERR_INVALID_ARG, "kv_alloc arguments");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // room: free pages, then adapters older than the current step, LRU first
  std::vector<int> victims;
  int64_t avail = (int64_t)P->free_pages.size();
  for (auto it = P->lru.begin(); avail < n && it != P->lru.end(); ++it) {
    if (it->first >= P->epoch) break;  // std::set order: the rest are as new
    victims.push_back(it->second);
    avail += (int64_t)P->ad[it->second].pages.size();
  }
  if (avail < n)
    return P->fail(SLORA_ERR_OOM, "cannot take " + std::to_string(n) + " pages for KV blocks");
  int64_t wait_ep = -1;
  for (int v : victims) {
    wait_ep = std::max(wait_ep, P->ad[v].last_use);
    evict_one(P, v);
  }
  std::set<int> rel_wait;
  for (int64_t i = 0; i < n; ++i) {
    FreePage f = P->free_pages.front();
    P->free_pages.pop_front();
    ids_out[i] = f.id;
    P->kv_page[f.id] = 1;
    wait_ep = std::max(wait_ep, f.free_epoch);
    if (f.rel >= 0) rel_wait.insert(f.rel);
  }
  P->kv_held += n;
  P->st.free_pages = (int64_t)P->free_pages.size();
  P->st.resident = (int64_t)P->lru.size();
  if (P->d.host_only) return SLORA_OK;
  // the evicted adapters leave the device table; the pages are the caller's
  // once the compute, page-in copies and KV owners that last touched them are done
  // (table writes join the page-in chain, so a later page-in of the same
  // adapter on another stream lands after them)
  if (P->pagein_pending) CUDA_TRY(P, cudaStreamWaitEvent(st, P->pagein_done, 0));
  for (int v : victims) CUDA_TRY(P, cudaMemsetAsync(P->pd.rank + v, 0xff, 4, st));
  if (!victims.empty()) {
    CUDA_TRY(P, cudaEventRecord(P->pagein_done, st));
    P->pagein_pending = true;
  }
  CUDA_TRY(P, wait_epoch(P, st, wait_ep));
  for (int r : rel_wait) CUDA_TRY(P, cudaStreamWaitEvent(st, P->rel_ev[r], 0));
  if (done_event) CUDA_TRY(P, cudaEventRecord(static_cast<cudaEvent_t>(done_event), st));
  return SLORA_OK;
}

slora_status_t slora_kv_free(slora_pool* P, const int32_t* ids, int64_t n, void* stream) {
  NvtxRange nvtx_("slora_kv_free");
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (n < 0 || (n > 0 && !ids)) return P->fail(SLORA_ERR_INVALID_ARG, "kv_free arguments");
  std::unordered_set<int32_t> seen;
  for (int64_t i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= P->d.n_pages || !P->kv_page[ids[i]] || !seen.insert(ids[i]).second)
      return P->fail(SLORA_ERR_INVALID_ARG, "page " + std::to_string(ids[i]) + " is not a held KV page");
  int rel = -1;
  if (!P->d.host_only && stream && n > 0) {
    // reusing a slot: the work it marked is long done (64 releases ago); make sure
    rel = (int)(P->n_rel % kRelRing);
    if (P->n_rel >= kRelRing) {
      slora_status_t ws = wait_event_bounded(P, P->rel_ev[rel]);
      if (ws != SLORA_OK) return ws;
    }
    CUDA_TRY(P, cudaEventRecord(P->rel_ev[rel], static_cast<cudaStream_t>(stream)));
    P->n_rel++;
  }
  for (int64_t i = 0; i < n; ++i) {
    P->kv_page[ids[i]] = 0;
    P->free_pages.push_back({ids[i], -1, rel});
  }
  P->kv_held -= n;
  P->st.free_pages = (int64_t)P->free_pages.size();
  return SLORA_OK;
}

slora_status_t slora_adapter_evict(slora_pool* P, int32_t id, void* stream) {
  NvtxRange nvtx_("slora_adapter_evict");
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (id < 0 || id >= P->d.max_adapters) return P->fail(SLORA_ERR_INVALID_ARG, "adapter id out of range");
  if (!P->ad[id].resident) return P->fail(SLORA_ERR_NOT_RESIDENT, "adapter " + std::to_string(id));
  if (!P->d.host_only) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (P->pagein_pending) CUDA_TRY(P, cudaStreamWaitEvent(st, P->pagein_done, 0));
    CUDA_TRY(P, cudaMemsetAsync(P->pd.rank + id, 0xff, 4, st));
    CUDA_TRY(P, cudaEventRecord(P->pagein_done, st));  // a later page-in lands after it
    P->pagein_pending = true;
  }
  evict_one(P, id);
  P->st.free_pages = (int64_t)P->free_pages.size();
  P->st.resident = (int64_t)P->lru.size();
  return SLORA_OK;
}

slora_status_t slora_adapter_is_resident(const slora_pool* P, int32_t id, int32_t* out) {
  if (!P || !out || id < 0 || id >= P->d.max_adapters) return SLORA_ERR_INVALID_ARG;
  *out = P->ad[id].resident ? 1 : 0;
  return SLORA_OK;
}

int32_t slora_decode_kernels(const slora_pool* P, int32_t T) {
  if (!P || T <= 0) return 0;
  return token_path(P, T) || fused_path(P, T) || stream_path(P, T) ? 1 : 3;
}

int32_t slora_decode_kind(const slora_pool* P, int32_t T) {
  if (!P || T <= 0) return SLORA_KIND_NONE;
  if (token_path(P, T)) return SLORA_KIND_TOKEN;
  if (stream_path(P, T)) return SLORA_KIND_STREAM;
  if (fused_path(P, T)) return SLORA_KIND_FUSED;
  return SLORA_KIND_SPLIT;
}

slora_status_t slora_check_batch(const slora_pool* Pc, const int32_t* idx_host, int32_t T) {
  slora_pool* P = const_cast<slora_pool*>(Pc);
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (T < 0 || (T > 0 && !idx_host)) return P->fail(SLORA_ERR_INVALID_ARG, "idx");
  for (int i = 0; i < T; ++i) {
    const int a = idx_host[i];
    if (a == -1) continue;
    if (a < -1 || a >= P->d.max_adapters) return P->fail(SLORA_ERR_INVALID_ARG, "token " + std::to_string(i) + ": adapter id out of range");
    if (!P->ad[a].resident || P->ad[a].named != P->epoch)
      return P->fail(SLORA_ERR_NOT_RESIDENT, "token " + std::to_string(i) + ": adapter " + std::to_string(a) +
                                                 " is not in the latest page-in set");
  }
  return SLORA_OK;
}

slora_status_t slora_build_segments(slora_pool* P, const int32_t* idx, int32_t T, int32_t* perm,
                                    int32_t* seg_start, int32_t* seg_adapter, int32_t* S_out, void* stream) {
  NvtxRange nvtx_("slora_build_segments");
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  if (T < 0 || T > P->d.max_tokens || (T > 0 && !idx) || !perm || !seg_start || !seg_adapter || !S_out)
    return P->fail(SLORA_ERR_INVALID_ARG, "build_segments arguments");
  BgmvParams bp;
  base_params(P, bp);
  bp.n_slots = 0;
  bp.n_groups = 0;
  bp.sc.perm = perm;
  bp.sc.seg_start = seg_start;
  bp.sc.seg_adapter = seg_adapter;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUDA_TRY(P, launch_segments(bp, idx, T, st));
  CUDA_TRY(P, cudaMemcpyAsync(S_out, bp.sc.meta + kMetaS, 4, cudaMemcpyDeviceToDevice, st));
  return SLORA_OK;
}

slora_status_t slora_build_sgmv_segments(slora_pool* P, const int32_t* req_start, const int32_t* req_adapter,
                                         int32_t n, int32_t* seg_start, int32_t* seg_adapter, int32_t* S_out,
                                         void* stream) {
  NvtxRange nvtx_("slora_build_sgmv_segments");
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  if (n < 0 || !req_start || (n > 0 && !req_adapter) || !seg_start || !seg_adapter || !S_out)
    return P->fail(SLORA_ERR_INVALID_ARG, "build_sgmv_segments arguments");
  CUDA_TRY(P, launch_merge_requests(req_start, req_adapter, n, seg_start, seg_adapter, S_out,
                                    static_cast<cudaStream_t>(stream)));
  return SLORA_OK;
}

slora_status_t slora_lora_delta(slora_pool* P, int32_t n, const int32_t* projs, const void* const* x,
                                const int64_t* ldx, void* const* y, const int64_t* ldy, const int32_t* idx,
                                int32_t T, void* stream) {
  NvtxRange nvtx_("slora_lora_delta");
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  if (T > 0 && !idx) return P->fail(SLORA_ERR_INVALID_ARG, "idx is NULL");
  BgmvParams bp;
  base_params(P, bp);
  s = plan_slots(P, bp, n, projs, x, ldx, y, ldy, T, true, true);
  if (s) return s;
  if (T == 0) return SLORA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = enqueue_delta(P, bp, idx, T, st, true);
  if (s) return s;
  CUDA_TRY(P, record_epoch(P, st));
  return SLORA_OK;
}

slora_status_t slora_bgmv_shrink(slora_pool* P, int32_t proj, const void* x, int64_t ldx, const int32_t* idx,
                                 int32_t T, float* t, int64_t ldt, void* stream) {
  NvtxRange nvtx_("slora_bgmv_shrink");
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  if (P->e4m3()) return P->fail(SLORA_ERR_UNSUPPORTED, "slora_bgmv_shrink takes 16-bit weights only");
  if (T > 0 && (!idx || !t)) return P->fail(SLORA_ERR_INVALID_ARG, "idx / t is NULL");
  if (ldt < P->d.max_rank || ((uintptr_t)t & 15) || ldt % 8)
    return P->fail(SLORA_ERR_INVALID_ARG, "t: ldt >= max_rank, ldt % 8 == 0, 16-byte aligned");
  BgmvParams bp;
  base_params(P, bp);
  const void* xs[1] = {x};
  const int64_t lx[1] = {ldx};
  s = plan_slots(P, bp, 1, &proj, xs, lx, nullptr, nullptr, T, true, false);
  if (s) return s;
  if (T == 0) return SLORA_OK;
  bp.slot[0].tout = t;
  bp.slot[0].ldt_out = ldt;
  bp.do_shrink = 1;
  bp.do_expand = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUDA_TRY(P, cudaMemsetAsync(t, 0, sizeof(float) * (size_t)T * ldt, st));
  phase(P, 0, 3, st);
  CUDA_TRY(P, launch_segments(bp, idx, T, st));
  phase(P, 1, 3, st);
  CUDA_TRY(P, launch_shrink(bp, P->d.dtype, P->grid_shrink, st));
  phase(P, 2, 3, st);
  CUDA_TRY(P, launch_reduce_t(bp, T, st));
  phase(P, 3, 3, st);
  CUDA_TRY(P, record_epoch(P, st));
  return SLORA_OK;
}

slora_status_t slora_bgmv_expand(slora_pool* P, int32_t proj, const float* t, int64_t ldt, const int32_t* idx,
                                 int32_t T, void* y, int64_t ldy, void* stream) {
  NvtxRange nvtx_("slora_bgmv_expand");
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  if (P->e4m3()) return P->fail(SLORA_ERR_UNSUPPORTED, "slora_bgmv_expand takes 16-bit weights only");
  if (T > 0 && (!idx || !t)) return P->fail(SLORA_ERR_INVALID_ARG, "idx / t is NULL");
  if (ldt < P->d.max_rank || ((uintptr_t)t & 15) || ldt % 8)
    return P->fail(SLORA_ERR_INVALID_ARG, "t: ldt >= max_rank, ldt % 8 == 0, 16-byte aligned");
  BgmvParams bp;
  base_params(P, bp);
  void* ys[1] = {y};
  const int64_t ly[1] = {ldy};
  s = plan_slots(P, bp, 1, &proj, nullptr, nullptr, ys, ly, T, false, true);
  if (s) return s;
  if (T == 0) return SLORA_OK;
  bp.slot[0].t = const_cast<float*>(t);
  bp.slot[0].t_rs = ldt;
  bp.slot[0].t_ns = 1;
  bp.slot[0].t_by_token = 1;
  bp.do_shrink = 0;
  bp.do_expand = 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  phase(P, 0, 2, st);
  CUDA_TRY(P, launch_segments(bp, idx, T, st));
  phase(P, 1, 2, st);
  CUDA_TRY(P, launch_expand(bp, P->d.dtype, P->grid_expand, st));
  phase(P, 2, 2, st);
  CUDA_TRY(P, record_epoch(P, st));
  return SLORA_OK;
}

slora_status_t slora_sgmv(slora_pool* P, int32_t n, const int32_t* projs, const void* const* x,
                          const int64_t* ldx, void* const* y, const int64_t* ldy, const int32_t* seg_start,
                          const int32_t* seg_adapter, int32_t S, int32_t T, void* stream) {
  NvtxRange nvtx_("slora_sgmv");
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  if (P->e4m3()) return P->fail(SLORA_ERR_UNSUPPORTED, "slora_sgmv takes 16-bit weights only");
  if (S < 0 || (S > 0 && (!seg_start || !seg_adapter))) return P->fail(SLORA_ERR_INVALID_ARG, "segments");
  BgmvParams bp;
  base_params(P, bp);
  s = plan_slots(P, bp, n, projs, x, ldx, y, ldy, T, true, true);
  if (s) return s;
  if (S == 0 || T == 0) return SLORA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (S > P->d.max_tokens) return P->fail(SLORA_ERR_INVALID_ARG, "more segments than max_tokens");
  cudaError_t e = launch_sgmv(bp, P->d.dtype, seg_start, seg_adapter, S, T, P->sm_count, st,
                              P->scratch() + P->sl.off_sgmv, P->d.max_tokens, P->d.n_pages, P->phase_ev,
                              P->n_phase);
  if (e == cudaErrorNotSupported) return P->fail(SLORA_ERR_UNSUPPORTED, "SGMV shape not supported");
  if (e != cudaSuccess) return P->cuda_fail(e, "SGMV launch");
  CUDA_TRY(P, record_epoch(P, st));
  return SLORA_OK;
}

slora_status_t slora_sgmv_linear(slora_pool* P, int32_t n, const int32_t* projs, const void* const* x,
                                 const int64_t* ldx, const void* const* w0, const int64_t* ldw, void* const* y,
                                 const int64_t* ldy, const int32_t* seg_start, const int32_t* seg_adapter,
                                 int32_t S, int32_t T, void* stream) {
  NvtxRange nvtx_("slora_sgmv_linear");
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  if (P->e4m3()) return P->fail(SLORA_ERR_UNSUPPORTED, "slora_sgmv_linear takes 16-bit weights only");
  if (P->d.max_rank > 64) return P->fail(SLORA_ERR_UNSUPPORTED, "slora_sgmv_linear: max_rank above 64");
  if (S < 1 || !seg_start || !seg_adapter) return P->fail(SLORA_ERR_INVALID_ARG, "segments");
  if (T < 1) return P->fail(SLORA_ERR_INVALID_ARG, "T must be positive");
  BgmvParams bp;
  base_params(P, bp);
  s = plan_slots(P, bp, n, projs, x, ldx, y, ldy, T, true, true);
  if (s) return s;
  if (!w0 || !ldw) return P->fail(SLORA_ERR_INVALID_ARG, "w0 is NULL");
  for (int k = 0; k < n; ++k)
    if (!w0[k] || !aligned16(w0[k]) || ldw[k] < bp.slot[k].d_in || ldw[k] % 8)
      return P->fail(SLORA_ERR_INVALID_ARG, "w0 must be 16-byte aligned with ldw >= d_in, ldw % 8 == 0");
  if (S > P->d.max_tokens) return P->fail(SLORA_ERR_INVALID_ARG, "more segments than max_tokens");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  phase(P, 0, 1, st);
  cudaError_t e = launch_linear(bp, P->d.dtype, w0, ldw, seg_start, seg_adapter, S, T, P->sm_count, st,
                                P->scratch() + P->sl.off_sgmv, P->d.max_tokens, P->d.n_pages);
  if (e == cudaErrorNotSupported) return P->fail(SLORA_ERR_UNSUPPORTED, "linear layer shape not supported");
  if (e != cudaSuccess) return P->cuda_fail(e, "linear layer launch");
  phase(P, 1, 1, st);
  CUDA_TRY(P, record_epoch(P, st));
  return SLORA_OK;
}

slora_status_t slora_debug_gather(slora_pool* P, int32_t id, int32_t proj, void* host_A_t, void* host_B) {
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  if (id < 0 || id >= P->d.max_adapters || proj < 0 || proj >= P->d.n_proj)
    return P->fail(SLORA_ERR_INVALID_ARG, "id / proj out of range");
  if (!P->ad[id].resident) return P->fail(SLORA_ERR_NOT_RESIDENT, "adapter " + std::to_string(id));
  const int r = P->ad[id].rank;
  if (r == 0) return SLORA_OK;
  // Debug path: uses its own temporary device buffer.  Widths in 16-bit units.
  const int w_in = P->e4m3() ? P->d.d_in[proj] / 2 : P->d.d_in[proj];
  const int w_out = P->e4m3() ? P->d.d_out[proj] / 2 : P->d.d_out[proj];
  const size_t na = (size_t)r * w_in * 2, nb = (size_t)r * w_out * 2;
  void* buf = nullptr;
  CUDA_TRY(P, cudaMalloc(&buf, na + nb));
  cudaError_t e = launch_gather_debug(P->pd, id, w_in, P->listA[proj], r, static_cast<uint16_t*>(buf), 0);
  if (e == cudaSuccess)
    e = launch_gather_debug(P->pd, id, w_out, P->listB[proj], r,
                            reinterpret_cast<uint16_t*>(static_cast<char*>(buf) + na), 0);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess && host_A_t) e = cudaMemcpy(host_A_t, buf, na, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && host_B) e = cudaMemcpy(host_B, static_cast<char*>(buf) + na, nb, cudaMemcpyDeviceToHost);
  cudaFree(buf);
  if (e != cudaSuccess) return P->cuda_fail(e, "debug_gather");
  return SLORA_OK;
}

slora_status_t slora_check_device(slora_pool* P, void* stream, int32_t* code, int32_t* info) {
  NvtxRange nvtx_("slora_check_device");
  if (!P) return SLORA_ERR_INVALID_ARG;
  slora_status_t s = need_device(P);
  if (s) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUDA_TRY(P, cudaStreamSynchronize(st));
  int32_t w[2] = {0, 0};
  CUDA_TRY(P, cudaMemcpy(w, P->pd.err, 8, cudaMemcpyDeviceToHost));
  if (code) *code = w[0];
  if (info) *info = w[1];
  if (w[0] == 0) return SLORA_OK;
  CUDA_TRY(P, cudaMemset(P->pd.err, 0, 8));
  return P->fail(SLORA_ERR_DEVICE_CHECK, "kernel recorded code " + std::to_string(w[0]) + " at " + std::to_string(w[1]));
}

// ---------------------------------------------------------------------------
// Host-side quantisation of adapter rows to e4m3 (the registration step of
// 8-bit adapter pages).

// Exact value of a 16-bit element: fp16 (1/5/10) or bf16 (1/8/7).
static double value16(int dtype, uint16_t h) {
  if (dtype == SLORA_BF16) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
  }
  const int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v = e == 0 ? std::ldexp((double)m, -24)
                    : e == 31 ? (m ? NAN : INFINITY) : std::ldexp((double)(m | 1024), e - 25);
  return s ? -v : v;
}

// e4m3 code of a finite q, rounded to nearest with ties to an even fraction,
// saturating at +-448: the exponent from frexp, the 3 fraction bits by one
// rint (the current rounding mode, nearest-even) of the exactly scaled value.
static uint8_t e4m3_of(double q) {
  const uint8_t sign = std::signbit(q) ? 0x80 : 0x00;
  const double a = std::fabs(q);
  if (a >= 448.0) return sign | 0x7e;
  int e;
  std::frexp(a, &e);  // a = m * 2^e, m in [0.5, 1)
  int code;
  if (a < 0.015625) {  // below 2^-6: subnormal steps of 2^-9
    code = (int)std::rint(std::ldexp(a, 9));  // 8 carries into the first normal code
  } else {
    const int E = e - 1;                                     // a in [2^E, 2^(E+1))
    const int f = (int)std::rint(std::ldexp(a, 3 - E)) - 8;  // 0..8
    code = ((E + 7) << 3) + f;                               // f = 8 carries into the exponent
  }
  return sign | (uint8_t)std::min(code, 0x7e);
}

slora_status_t slora_quantize_e4m3_rows(int32_t dtype, const uint16_t* in, int64_t rows, int64_t n,
                                        uint8_t* codes, float* scales) {
  if ((dtype != SLORA_F16 && dtype != SLORA_BF16) || rows < 0 || n < 0 ||
      (rows > 0 && n > 0 && (!in || !codes)) || (rows > 0 && !scales))
    return SLORA_ERR_INVALID_ARG;
  for (int64_t r = 0; r < rows; ++r) {
    const uint16_t* row = in + r * n;
    double amax = 0.0;
    for (int64_t j = 0; j < n; ++j) {
      const double v = value16(dtype, row[j]);
      if (!std::isfinite(v)) return SLORA_ERR_INVALID_ARG;
      amax = std::max(amax, std::fabs(v));
    }
    const float sc = (float)(amax / 448.0);
    scales[r] = sc;
    for (int64_t j = 0; j < n; ++j)
      codes[r * n + j] = sc == 0.0f ? 0 : e4m3_of(value16(dtype, row[j]) / (double)sc);
  }
  return SLORA_OK;
}

slora_status_t slora_pool_stats(const slora_pool* P, slora_pool_stats_t* out) {
  if (!P || !out) return SLORA_ERR_INVALID_ARG;
  *out = P->st;
  out->free_pages = (int64_t)P->free_pages.size();
  out->resident = (int64_t)P->lru.size();
  out->epoch = P->epoch;
  out->kv_pages = P->kv_held;
  return SLORA_OK;
}

slora_status_t slora_set_phase_events(slora_pool* P, void* const* events, int32_t n) {
  if (!P) return SLORA_ERR_INVALID_ARG;
  if (n < 0 || n > 8 || n == 1 || n == 3 || (n > 0 && !events))
    return P->fail(SLORA_ERR_INVALID_ARG, "events: n must be 0, 2 or 4..8");
  for (int i = 0; i < n; ++i) {
    if (!events[i]) return P->fail(SLORA_ERR_INVALID_ARG, "event is NULL");
    P->phase_ev[i] = static_cast<cudaEvent_t>(events[i]);
  }
  P->n_phase = n;
  return SLORA_OK;
}

slora_status_t slora_inject_fault(slora_pool* P, int32_t after) {
  if (!P) return SLORA_ERR_INVALID_ARG;
  P->inject_after = after < 0 ? -1 : after;
  return SLORA_OK;
}

}  // extern "C"
