// bgmv.cu -- decode-path kernels of the paged multi-adapter LoRA delta (sm_100a).
//
//   k_segments   one CTA: validates the token -> adapter index vector, builds
//                the per-adapter segments with a stable counting sort, and
//                plans the shrink / expand work lists (segment grouping as in
//                "Multi-LoRA serving: S-LoRA, Punica, SGMV, vLLM", SGMV section:
//                an index vector maps each token to its adapter).
//   k_shrink     t[i, k] = sum_j x[i, j] * A_a[j, k]  (first SGMV phase, d -> r),
//                A_a gathered from the paged pool through the page table
//                ("Paper explainer: S-LoRA", BGMV kernel section: weights fetched
//                from paged memory by adapter id).  fp32 accumulation; d_in is
//                split in fixed chunks whose fp32 partials are summed, in chunk
//                order, by the last task to finish (deterministic).
//   k_expand     y[i, l] <- round(y[i, l] + (alpha/r) * sum_k t[i, k] * B_a[k, l])
//                (second phase, r -> d_out, with the residual add fused into the
//                output store: "Multi-LoRA serving", metrics section).
//   k_page_in    copies newly resident adapters from pinned host memory into
//                their scattered pages and updates the page table.
//
// Shrink and expand are persistent (one CTA of 8 warps per SM).  Every warp
// runs its own two-slot pipeline: while it computes on one shared-memory slot,
// the bulk-copy engine fills the other with the next task's page-gathered rows
// (cp.async.bulk, completion counted on an mbarrier).  A task reads one adapter
// tile once and applies it to every token of its segment that the task covers,
// so each touched adapter is streamed from HBM about once per step.  The three
// kernels are chained with programmatic dependent launch.
#include <algorithm>

#include "dev_common.cuh"

namespace slora {

// Task shapes.  A shrink task covers NT tokens x kRB rank rows x kShrinkKT of
// d_in; an expand task NTE tokens x kELC outputs (all rank rows).
constexpr int kCW = 8;                        // consumer warps per CTA
constexpr int kProd = 4;                      // producer warps (interleaved ring stages)
constexpr int kPipeThreads = (kCW + kProd) * 32;
constexpr int kDescInts = 32;                 // per-stage descriptor (task fields)
constexpr int kRB = 16;                       // shrink task: rank rows (2 per consumer warp)
constexpr int kELC = kCW * 256;               // expand task: outputs (256 per consumer warp)

// ---------------------------------------------------------------------------
// Task schedule of the persistent CTAs.  The first rounds are static: CTA b
// takes tasks b, b + G, b + 2G, ... (G = gridDim.x) for m_static tasks; the
// rest, the last fifth of the rounds but at least two, are claimed from a
// global counter, so that CTAs that drew cheaper tasks take more of them and
// all finish close together.  The kProd producer warps each walk the CTA's
// whole (task, stage) sequence: the first warp to reach a dynamic CTA-local
// ordinal n claims its task with one atomicAdd and publishes the index in
// slot n % kTix, the others read it there.  The walking cursors stay within
// 3 kProd stage positions of one another (a producer cannot issue a stage
// before the ring slot it reuses has been consumed), so a slot is never
// reused before every warp has read it.
constexpr int kTix = 32;
static_assert(3 * kProd < kTix, "claim slots");
struct TaskClaims {
  int next;       // next dynamic ordinal to claim
  int m_static;   // static ordinals per CTA
  int ord[kTix];  // ordinal published in each slot
  int id[kTix];   // its task index
};
__device__ __forceinline__ int static_rounds(int total) {
  const int rounds = total / (int)gridDim.x;
  return max(0, rounds - max(2, rounds / 5));
}
// One thread, before the CTA barrier.
__device__ __forceinline__ void claims_init(TaskClaims& C, int total) {
  C.m_static = static_rounds(total);
  C.next = C.m_static;
  for (int i = 0; i < kTix; ++i) C.ord[i] = -1;
}
// Task index of CTA-local ordinal n, for every lane of the calling warp (n
// warp-uniform); -1 if the wait for its publication gave up (error recorded).
__device__ __forceinline__ int task_of(TaskClaims& C, int n, int* counter, int32_t* err) {
  if (n < C.m_static) return (int)blockIdx.x + n * (int)gridDim.x;
  int id = -1;
  if ((threadIdx.x & 31) == 0) {
    const int slot = n % kTix;
    if (atomicCAS(&C.next, n, n + 1) == n) {
      id = C.m_static * (int)gridDim.x + atomicAdd(counter, 1);
      st_volatile_s32(&C.id[slot], id);
      __threadfence_block();
      st_volatile_s32(&C.ord[slot], n);
    } else {
      long long t0 = -1;
      for (uint32_t it = 0;; ++it) {
        if (ld_volatile_s32(&C.ord[slot]) == n) {
          __threadfence_block();
          id = ld_volatile_s32(&C.id[slot]);
          break;
        }
        if ((it & 63) == 0) {
          const long long now = clock64();
          if (t0 < 0) t0 = now;
          else if (now - t0 > kWaitLimit) {
            record_error(err, 4, (int)blockIdx.x);
            break;
          }
        }
        __nanosleep(32);
      }
    }
  }
  return __shfl_sync(FULL_MASK, id, 0);
}

// Touch every 64-byte line of a kernel's parameter block once, so that the
// first lookups that index its group and slot tables with runtime values do
// not each wait on a constant-cache miss.  Runs before the grid dependency
// resolves (or, in k_segments, beside the histogram reset).
template <class Params>
__device__ __forceinline__ void warm_params(const Params& p, int* sink) {
  constexpr int kLines = (int)((sizeof(Params) + 63) / 64);
  if ((int)threadIdx.x < kLines) {
    const int v = reinterpret_cast<const int*>(&p)[threadIdx.x * 16];
    if (v == 0x5a5a5a5a) *sink = v;  // keeps the load; the value is never used
  }
}

// k_segments: one CTA of 1024 threads.  Dynamic smem: max_adapters ints.
// Output: perm, segments (start, adapter, rank) and, per segment, the number
// of shrink and expand tasks before it (prefix sums in segment-major order).
__device__ __forceinline__ void seg_task_counts(const BgmvParams& p, int n, int r, int& shr, int& exp) {
  shr = exp = 0;
  if (n == 0 || r <= 0) return;
  const int nt = nt_class(n), ntg = cdiv_i(n, nt), nte = cdiv_i(n, nte_class(n));
  if (p.do_shrink)
    for (int g = 0; g < p.n_groups; ++g)
      shr += cdiv_i(p.group[g].n * r, kRB) * ntg * cdiv_i(p.group[g].d_in, kShrinkKT);
  if (p.do_expand)
    for (int k = 0; k < p.n_slots; ++k) exp += nte * cdiv_i(p.slot[k].d_out, kELC);
}

// L2 hint for the page lists (A_t and B of every projection of the call) of
// the adapters of tokens blockIdx.x and blockIdx.x + gridDim.x: warp w < 2
// takes one token, lane 2k + h the list of projection k, half h.  Runs in a
// persistent kernel's prologue, while k_segments builds the segment table;
// idx and the pool tables are final by then (k_segments, which this kernel
// follows, started only after all earlier work of the stream).
__device__ __forceinline__ void prefetch_token_page_lists(const BgmvParams& p) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int i = (int)blockIdx.x + w * (int)gridDim.x;
  if (w >= 2 || p.idx == nullptr || i >= p.T || lane >= 2 * p.n_slots) return;
  const int a = p.idx[i];
  if (a < 0 || a >= p.pool.max_adapters) return;
  const int r = p.pool.rank[a];
  if (r <= 0) return;
  const SlotDev& L = p.slot[lane >> 1];
  const int h = lane & 1;
  const int64_t np = ((int64_t)r * (h ? L.d_out : L.d_in) + (1ll << p.pool.page_shift) - 1) >> p.pool.page_shift;
  const int32_t* row = p.pool.page_list + (int64_t)a * p.pool.list_stride + (h ? L.listB : L.listA);
  const uintptr_t e = reinterpret_cast<uintptr_t>(row + np);
  for (uintptr_t l = reinterpret_cast<uintptr_t>(row) & ~(uintptr_t)127; l < e; l += 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(l));
}

// Histogram entries pack the adapter's token count (< 2^21) with its rank + 1
// (bits 21 and up), so that the segment pass needs no second rank lookup.
constexpr int kHistRankShift = 21;

__global__ void __launch_bounds__(1024, 1) k_segments(const __grid_constant__ BgmvParams p,
                                                   const int32_t* __restrict__ idx, int T) {
  extern __shared__ int hist[];
  __shared__ int4 sh[32];
  __shared__ __align__(16) int ck[1024];  // keys of one scatter chunk
  __shared__ int sink;
  const int tid = threadIdx.x, nth = blockDim.x;
  const int MA = p.pool.max_adapters;
  const ScratchDev& sc = p.sc;
  griddep_launch();  // the next kernel may start its prologue; it waits for this grid
  warm_params(p, &sink);

  for (int a = tid; a < MA; a += nth) hist[a] = 0;
  __syncthreads();
  int key0 = -1;  // adapter of token tid when it is valid (the first scatter chunk)
  for (int i = tid; i < T; i += nth) {
    const int a = idx[i];
    if (a == -1) continue;
    if (a < -1 || a >= MA) {
      record_error(p.pool.err, 1, i);
      continue;
    }
    const int r = p.pool.rank[a];
    if (r < 0) {
      record_error(p.pool.err, 2, i);
      continue;
    }
    atomicOr(&hist[a], (r + 1) << kHistRankShift);
    atomicAdd(&hist[a], 1);
    if (i == tid) key0 = a;
  }
  __syncthreads();

  // Each thread owns a contiguous adapter range; the segments it creates form
  // a contiguous range of segment indices.
  const int E = (MA + nth - 1) / nth;
  const int a0 = min(tid * E, MA), a1 = min(a0 + E, MA);
  int4 c = make_int4(0, 0, 0, 0);  // tokens, segments, shrink tasks, expand tasks
  for (int a = a0; a < a1; ++a) {
    const int h = hist[a];
    if (h == 0) continue;
    const int n = h & ((1 << kHistRankShift) - 1), r = (h >> kHistRankShift) - 1;
    int x, z;
    seg_task_counts(p, n, r, x, z);
    c.x += n;
    c.y += 1;
    c.z += x;
    c.w += z;
  }
  int4 tot;
  const int4 base = block_exscan4(c, &tot, sh);
  const int n_valid = tot.x, S = tot.y, t_shr = tot.z, t_exp = tot.w;
  int cbase = base.x, sb = base.y, b_shr = base.z, b_exp = base.w;
  for (int a = a0; a < a1; ++a) {
    const int h = hist[a];
    hist[a] = cbase;  // becomes the scatter cursor
    if (h == 0) continue;
    const int n = h & ((1 << kHistRankShift) - 1), r = (h >> kHistRankShift) - 1;
    int x, z;
    seg_task_counts(p, n, r, x, z);
    sc.seg_start[sb] = cbase;
    sc.seg_adapter[sb] = a;
    sc.seg_rank[sb] = r;
    sc.shrink_prefix[sb] = b_shr;
    sc.expand_prefix[sb] = b_exp;
    ++sb;
    cbase += n;
    b_shr += x;
    b_exp += z;
  }
  if (tid == 0) {
    sc.seg_start[S] = n_valid;
    sc.shrink_prefix[S] = t_shr;
    sc.expand_prefix[S] = t_exp;
    sc.meta[kMetaS] = S;
    sc.meta[kMetaValid] = n_valid;
    sc.meta[kMetaShrinkTotal] = t_shr;
    sc.meta[kMetaExpandTotal] = t_exp;
    sc.meta[kMetaShrinkClaim] = 0;
    sc.meta[kMetaExpandClaim] = 0;
  }
  __syncthreads();

  // Stable scatter, one chunk of blockDim.x tokens at a time: a token's place
  // among its adapter's tokens of the chunk is the number of equal keys in
  // earlier warps (counted from the chunk's keys in shared memory) plus the
  // number in earlier lanes of its own warp.
  const int lane = tid & 31, warp = tid >> 5;
  for (int c0 = 0; c0 < T; c0 += nth) {
    const int i = c0 + tid;
    int a = key0;
    if (c0 > 0) {
      a = i < T ? idx[i] : -1;
      if (!(a >= 0 && a < MA && p.pool.rank[a] >= 0)) a = -1;
    }
    ck[tid] = a;
    __syncthreads();
    const unsigned m = __match_any_sync(FULL_MASK, a);
    if (a >= 0) {
      int before = __popc(m & ((1u << lane) - 1));
      const int4* k4 = reinterpret_cast<const int4*>(ck);
      for (int j = 0; j < warp * 8; ++j) {  // the 32 * warp keys of earlier warps
        const int4 v = k4[j];
        before += (v.x == a) + (v.y == a) + (v.z == a) + (v.w == a);
      }
      sc.perm[hist[a] + before] = i;
    }
    __syncthreads();  // every cursor read before the chunk's counts are added
    if (a >= 0 && lane == __ffs(m) - 1) atomicAdd(&hist[a], __popc(m));
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Segment table as seen by the persistent kernels: staged in shared memory
// when it fits (one round trip per CTA), else read from global memory.
constexpr int kSegCap = 1024;
constexpr int kSegSmemInts = 4 * kSegCap + 2;
struct SegView {
  const int32_t* start;   // [S + 1]
  const int32_t* adapter; // [S]
  const int32_t* rank;    // [S]
  const int32_t* prefix;  // [S + 1] tasks before each segment
  int S;
};

__device__ SegView stage_segments(const ScratchDev& sc, int S, bool shrink, int32_t* sm) {
  SegView v;
  v.S = S;
  const int32_t* pre = shrink ? sc.shrink_prefix : sc.expand_prefix;
  if (S > kSegCap) {
    v.start = sc.seg_start;
    v.adapter = sc.seg_adapter;
    v.rank = sc.seg_rank;
    v.prefix = pre;
    return v;
  }
  int32_t* st = sm;
  int32_t* ad = sm + (kSegCap + 1);
  int32_t* rk = ad + kSegCap;
  int32_t* pf = rk + kSegCap;
  for (int i = threadIdx.x; i <= S; i += blockDim.x) {
    st[i] = sc.seg_start[i];
    pf[i] = pre[i];
    if (i < S) {
      ad[i] = sc.seg_adapter[i];
      rk[i] = sc.seg_rank[i];
    }
  }
  __syncthreads();
  v.start = st;
  v.adapter = ad;
  v.rank = rk;
  v.prefix = pf;
  return v;
}

// ---------------------------------------------------------------------------
// Shrink and expand run as warp-specialised persistent CTAs: kProd producer
// warps take turns along the CTA's (task, stage) sequence and fill a ring of
// shared-memory stages with page-gathered bulk copies (cp.async.bulk,
// completion counted on the stage's `full` mbarrier); kCW consumer warps each
// compute a fixed slice of every stage and release it on the stage's `empty`
// mbarrier.  Page ids and token ids are looked up two of a producer's stages
// before the stage is issued.  Stages hold whole 4 KiB row slices: the copy
// engine's cost per request makes 1 KiB copies top out near 60% of HBM
// bandwidth, and a consumer warp needs a full row slice per stage to keep its
// fixed per-stage cost small.
// ---------------------------------------------------------------------------
// Shrink task = (group g, segment, kRB rank rows, NT tokens, kShrinkKT slice
// of d_in).  The task's x rows (NT x up to kShrinkKT elements) are copied
// once, with its first stage, into one of two x buffers (alternating with the
// CTA's task count); its A rows stream through a kSNS-stage ring kSRows at a
// time, each stage holding kSRows row slices of up to kShrinkKT elements
// (4 KiB copies, cut only at page boundaries).  Consumer warp w owns stage row
// w and writes one fp32 partial per (row, token) of the slice; the expand sums
// the partials of a row in index order.
constexpr int kSRows = 8;                        // A rows per shrink stage (one per consumer warp)
constexpr int kSNS = 4;                          // shrink ring stages
constexpr int kSStageBytes = kSRows * 2 * kShrinkKT;
constexpr int kSRingBytes = kSNS * kSStageBytes;
constexpr int kXBufBytes = 4 * 2 * kShrinkKT;    // up to 4 tokens x kShrinkKT elements
static_assert(kPartK == kShrinkKT && kCW == kSRows, "shrink stage mapping");
static_assert(kSRows * kMaxPieces <= 64, "two lookups per lane");
static_assert(kSNS % kProd == 0 || kProd % kSNS == 0, "ring slots per producer");

struct STask {
  int g, a, r, seg0, n, nt, rg, tg, split, nst, nrows, ntok, xb;
};
static_assert(sizeof(STask) / 4 + 2 <= kDescInts, "descriptor too small");

__device__ __forceinline__ void decode_shrink(const BgmvParams& p, const SegView& V, int task, int ord, STask& t) {
  const int s = find_seg(V.prefix, V.S, task);
  int q = task - V.prefix[s];
  t.a = V.adapter[s];
  t.seg0 = V.start[s];
  t.n = V.start[s + 1] - t.seg0;
  t.r = V.rank[s];
  t.nt = nt_class(t.n);
  const int n_tg = cdiv_i(t.n, t.nt);
  int g = 0;
  for (; g < p.n_groups - 1; ++g) {  // the group owning local task q
    const int cnt = cdiv_i(p.group[g].n * t.r, kRB) * n_tg * cdiv_i(p.group[g].d_in, kShrinkKT);
    if (q < cnt) break;
    q -= cnt;
  }
  t.g = g;
  const int d_in = p.group[g].d_in;
  const int n_split = cdiv_i(d_in, kShrinkKT);
  t.tg = q % n_tg;
  q /= n_tg;
  t.split = q % n_split;
  t.rg = q / n_split;
  t.nrows = min(kRB, p.group[g].n * t.r - t.rg * kRB);
  t.nst = cdiv_i(t.nrows, kSRows);
  t.ntok = min(t.nt, t.n - t.tg * t.nt);
  t.xb = ord & 1;  // CTA-local task ordinal parity
}

struct SCursor {  // a point of the producer's (task, stage) sequence
  STask t;
  int task, ord, st;  // task index, CTA-local task ordinal, stage
  bool valid;
};

__device__ __forceinline__ void scursor_next(const BgmvParams& p, const SegView& V, int total, TaskClaims& cl,
                                             SCursor& c) {
  if (!c.valid) return;
  if (++c.st < c.t.nst) return;
  c.st = 0;
  ++c.ord;
  c.task = task_of(cl, c.ord, p.sc.meta + kMetaShrinkClaim, p.pool.err);
  c.valid = c.task >= 0 && c.task < total;
  if (c.valid) decode_shrink(p, V, c.task, c.ord, c.t);
}

// Per-lane lookups of a shrink stage: entry e = lane + 32 u (u = 0, 1),
// e < kSRows * kMaxPieces, copies piece e % kMaxPieces of stage row
// e / kMaxPieces (aux0[u] = its page id); on a task's first stage lane
// l < ntok also copies token row l (aux1 = token).
__device__ __forceinline__ void shrink_lookup(const BgmvParams& p, const SCursor& c, int32_t (&aux0)[2],
                                              int32_t& aux1) {
  const int lane = threadIdx.x & 31;
  aux0[0] = aux0[1] = -1;
  aux1 = -1;
  if (!c.valid) return;
  const STask& t = c.t;
  const GroupDev& G = p.group[t.g];
  const int k0 = t.split * kShrinkKT;
  const int L = min(kShrinkKT, G.d_in - k0);
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int e = lane + 32 * u;
    const int i = e / kMaxPieces, q = e % kMaxPieces;
    if (i < kSRows && c.st * kSRows + i < t.nrows) {
      const int rho = t.rg * kRB + c.st * kSRows + i;
      const int j = rho / t.r, k = rho % t.r;
      const int64_t f0 = (int64_t)k * G.d_in + k0;
      int64_t b, en;
      if (piece_range(p.pool, f0, f0 + L, q, b, en)) aux0[u] = page_id(p.pool, t.a, p.slot[G.slot[j]].listA, b);
    }
  }
  if (c.st == 0 && lane < t.ntok) aux1 = __ldg(p.sc.perm + t.seg0 + t.tg * t.nt + lane);
}

__device__ __forceinline__ void shrink_issue(const BgmvParams& p, const SCursor& c, const int32_t (&aux0)[2],
                                             int32_t aux1, unsigned char* buf, unsigned char* xbuf, int32_t* desc,
                                             uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const STask& t = c.t;
  const GroupDev& G = p.group[t.g];
  const int k0 = t.split * kShrinkKT;
  const int L = min(kShrinkKT, G.d_in - k0);
  const int rows = min(kSRows, t.nrows - c.st * kSRows);
  if (lane == 0) {
    const int32_t* src = reinterpret_cast<const int32_t*>(&t);
    for (int q = 0; q < (int)(sizeof(STask) / 4); ++q) desc[q] = src[q];
    desc[kDescInts - 2] = c.st;
    desc[kDescInts - 1] = 1;
    mbar_expect_tx(bar, 2u * L * (rows + (c.st == 0 ? t.ntok : 0)));
  }
  __syncwarp();
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    if (aux0[u] >= 0) {
      const int e = lane + 32 * u;
      const int i = e / kMaxPieces, q = e % kMaxPieces;
      const int rho = t.rg * kRB + c.st * kSRows + i;
      const int64_t f0 = (int64_t)(rho % t.r) * G.d_in + k0;
      int64_t b, en;
      piece_range(p.pool, f0, f0 + L, q, b, en);
      bulk_g2s(buf + i * 2 * kShrinkKT + 2 * (b - f0), page_ptr(p.pool, aux0[u], b), (uint32_t)(2 * (en - b)), bar);
    }
  }
  if (aux1 >= 0) bulk_g2s(xbuf + lane * 2 * kShrinkKT, G.x + (int64_t)aux1 * G.ldx + k0, 2u * L, bar);
}

template <int DT, int NT>
__device__ __forceinline__ void shrink_consume(const BgmvParams& p, const STask& t, int st,
                                               const unsigned char* buf, const unsigned char* xb) {
  const int lane = threadIdx.x & 31, cw = (threadIdx.x >> 5) - kProd;
  if (st * kSRows + cw >= t.nrows) return;  // warp-uniform
  const GroupDev& G = p.group[t.g];
  const int L = min(kShrinkKT, G.d_in - t.split * kShrinkKT);
  // four accumulator chains per token (256-element chunk c feeds chain c % 4),
  // summed in chain order
  constexpr int kC = kShrinkKT / 256;
  float acc[4][NT];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) acc[c][tt] = 0.f;
  const unsigned char* arow = buf + cw * 2 * kShrinkKT;
#pragma unroll
  for (int c0 = 0; c0 < kC; c0 += 4) {
    const int e0 = c0 * 256 + lane * 8;
    if (e0 >= L) break;
    uint4 av[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) av[c] = e0 + c * 256 < L ? lds128(arow + 2 * (e0 + c * 256)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) {
      if (tt >= t.ntok) break;
      uint4 xv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        xv[c] = e0 + c * 256 < L ? lds128(xb + tt * 2 * kShrinkKT + 2 * (e0 + c * 256)) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float s0 = acc[c][tt];
        s0 = fma2_16<DT>(av[c].x, xv[c].x, s0);
        s0 = fma2_16<DT>(av[c].y, xv[c].y, s0);
        s0 = fma2_16<DT>(av[c].z, xv[c].z, s0);
        s0 = fma2_16<DT>(av[c].w, xv[c].w, s0);
        acc[c][tt] = s0;
      }
    }
  }
  float v[NT];
#pragma unroll
  for (int tt = 0; tt < NT; ++tt) v[tt] = (acc[0][tt] + acc[1][tt]) + (acc[2][tt] + acc[3][tt]);
  // sum over lanes; lane tt < ntok stores the partial of (row, token tt)
  const float val = lane_transpose_reduce<NT>(v);
  const int rho = t.rg * kRB + st * kSRows + cw;
  const int j = rho / t.r, k = rho % t.r;
  const SlotDev& S = p.slot[G.slot[j]];
  if (lane < NT && lane < t.ntok) {
    const int pos = t.seg0 + t.tg * t.nt + lane;
    S.t[(int64_t)pos * S.t_rs + (int64_t)k * S.t_ns + t.split] = val;
  }
}

template <int DT>
__global__ void __launch_bounds__(kPipeThreads, 1) k_shrink(const __grid_constant__ BgmvParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[kSNS], empty[kSNS];
  __shared__ int xdone[2];  // consumer warps done with each x buffer (kCW per task)
  __shared__ TaskClaims claims;
  __shared__ int warm_sink;
  __shared__ int32_t desc[kSNS][kDescInts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* xbufs = smem + kSRingBytes;
  int32_t* segsm = reinterpret_cast<int32_t*>(xbufs + 2 * kXBufBytes);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    xdone[0] = xdone[1] = 0;
    fence_mbar_init();
  }
  warm_params(p, &warm_sink);
  prefetch_token_page_lists(p);
  griddep_wait();
  const int S = p.sc.meta[kMetaS];
  const int total = p.sc.meta[kMetaShrinkTotal];
  const SegView V = stage_segments(p.sc, S, true, segsm);
  if (threadIdx.x == 0) claims_init(claims, total);
  __syncthreads();
  if (warp < kProd) {
    // producer `warp` issues the stages at positions warp, warp + kProd, ...
    // of the CTA's (task, stage) sequence, into ring slots of the same parity
    SCursor A, B;
    A.task = task_of(claims, 0, p.sc.meta + kMetaShrinkClaim, p.pool.err);
    A.ord = 0;
    A.st = 0;
    A.valid = A.task >= 0 && A.task < total;
    if (A.valid) decode_shrink(p, V, A.task, 0, A.t);
    for (int q = 0; q < warp; ++q) scursor_next(p, V, total, claims, A);
    // page ids of a position are looked up two of this warp's issues ahead;
    // A's lookups are in flight while B is walked
    int32_t a0[2], a1, b0[2], b1;
    shrink_lookup(p, A, a0, a1);
    B = A;
    for (int q = 0; q < kProd; ++q) scursor_next(p, V, total, claims, B);
    shrink_lookup(p, B, b0, b1);
    uint32_t eparity = 0;
    int ring = warp % kSNS, uses = 0;
    bool ok = true;
    while (A.valid) {
      if (uses >= kSNS / kProd) {
        if (!mbar_wait(&empty[ring], (eparity >> ring) & 1, p.pool.err)) break;
        eparity ^= 1u << ring;
      }
      if (A.st == 0) {  // the x buffer of CTA task n is free once tasks n - 2, n - 4, ... are consumed
        const int n = A.ord;
        if (n >= 2) ok = counter_wait(&xdone[n & 1], kCW * (n >> 1), p.pool.err);
        if (!ok) break;
      }
      shrink_issue(p, A, a0, a1, smem + ring * kSStageBytes, xbufs + A.t.xb * kXBufBytes, desc[ring], &full[ring]);
      a0[0] = b0[0];
      a0[1] = b0[1];
      a1 = b1;
      A = B;
      for (int q = 0; q < kProd; ++q) scursor_next(p, V, total, claims, B);
      shrink_lookup(p, B, b0, b1);
      ring = (ring + kProd) % kSNS;
      ++uses;
    }
    // end marker at this producer's next position (the consumers stop at the
    // first one in sequence order)
    if (uses >= kSNS / kProd) mbar_wait(&empty[ring], (eparity >> ring) & 1, p.pool.err);
    if (lane == 0) {
      desc[ring][kDescInts - 1] = 0;
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&full[ring])) : "memory");
    }
  } else {
    // consumers
    uint32_t fparity = 0;
    int ring = 0;
    for (;;) {
      if (!mbar_wait(&full[ring], (fparity >> ring) & 1, p.pool.err)) break;
      fparity ^= 1u << ring;
      if (desc[ring][kDescInts - 1] == 0) break;
      STask t;
      int32_t* dst = reinterpret_cast<int32_t*>(&t);
#pragma unroll
      for (int q = 0; q < (int)(sizeof(STask) / 4); ++q) dst[q] = desc[ring][q];
      const int st = desc[ring][kDescInts - 2];
      const unsigned char* buf = smem + ring * kSStageBytes;
      const unsigned char* xb = xbufs + t.xb * kXBufBytes;
      if (DT == SLORA_BF16) {
        switch (t.nt) {
          case 1: shrink_consume<SLORA_BF16, 1>(p, t, st, buf, xb); break;
          case 2: shrink_consume<SLORA_BF16, 2>(p, t, st, buf, xb); break;
          default: shrink_consume<SLORA_BF16, 4>(p, t, st, buf, xb); break;
        }
      } else {
        switch (t.nt) {
          case 1: shrink_consume<SLORA_F16, 1>(p, t, st, buf, xb); break;
          case 2: shrink_consume<SLORA_F16, 2>(p, t, st, buf, xb); break;
          default: shrink_consume<SLORA_F16, 4>(p, t, st, buf, xb); break;
        }
      }
      // the slot's generic-proxy reads before the next bulk copy into it
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&empty[ring])) : "memory");
        if (st == t.nst - 1) atomicAdd(&xdone[t.xb], 1);
      }
      ring = (ring + 1) % kSNS;
    }
  }
  griddep_launch();
}

// ---------------------------------------------------------------------------
// Expand task = (projection slot k, segment, NTE tokens, kELC outputs); stages
// of kER rank rows.  Stage layout: B row i at i * 4 KiB, then the t partials
// of token t at kEXT + t * kER * t_ns * 4 B.  The task's y rows (NTE x kELC
// outputs) are copied with its first stage into one of two y buffers
// (alternating with the CTA's task count) and read back at its last stage.
// Consumer warp w owns outputs [256 w, 256 w + 256) of the task.
constexpr int kER = 8;                           // expand stage: rank rows
constexpr int kEXT = kER * 2 * kELC;             // B rows of a stage
constexpr int kETMax = 4 * kER * 32 * 4;         // t partials: 4 tokens x kER rows x <= 32 partials
constexpr int kEStageBytes = kEXT + kETMax;
constexpr int kENS = 4;                          // expand ring stages
constexpr int kERingBytes = kENS * kEStageBytes;
constexpr int kYBufBytes = 4 * 2 * kELC;         // up to 4 tokens x kELC outputs
static_assert(kER * 4 == 32, "one lane per (token, row) for four tokens");
static_assert(kER * kMaxPieces <= 64, "two lookups per lane");

struct ETask {
  int k, a, r, seg0, n, nt, tg, lc, nst, ntok, yb, tok0, tok1, tok2, tok3;
};
static_assert(sizeof(ETask) / 4 + 2 <= kDescInts, "descriptor too small");

__device__ __forceinline__ void decode_expand(const BgmvParams& p, const SegView& V, int task, int ord, ETask& t) {
  const int s = find_seg(V.prefix, V.S, task);
  int q = task - V.prefix[s];
  t.a = V.adapter[s];
  t.seg0 = V.start[s];
  t.n = V.start[s + 1] - t.seg0;
  t.r = V.rank[s];
  t.nt = nte_class(t.n);
  const int n_tg = cdiv_i(t.n, t.nt);
  int k = 0;
  for (; k < p.n_slots - 1; ++k) {  // the projection owning local task q
    const int cnt = n_tg * cdiv_i(p.slot[k].d_out, kELC);
    if (q < cnt) break;
    q -= cnt;
  }
  t.k = k;
  t.tg = q % n_tg;
  t.lc = q / n_tg;
  t.nst = cdiv_i(t.r, kER);
  t.ntok = min(t.nt, t.n - t.tg * t.nt);
  t.yb = ord & 1;  // CTA-local task ordinal parity
  t.tok0 = t.tok1 = t.tok2 = t.tok3 = 0;
}

struct ECursor {
  ETask t;
  int task, ord, st;
  bool valid;
};

__device__ __forceinline__ void ecursor_next(const BgmvParams& p, const SegView& V, int total, TaskClaims& cl,
                                             ECursor& c) {
  if (!c.valid) return;
  if (++c.st < c.t.nst) return;
  c.st = 0;
  ++c.ord;
  c.task = task_of(cl, c.ord, p.sc.meta + kMetaExpandClaim, p.pool.err);
  c.valid = c.task >= 0 && c.task < total;
  if (c.valid) decode_expand(p, V, c.task, c.ord, c.t);
}

// Per-lane lookups of an expand stage: entry e = lane + 32 u (u = 0, 1),
// e < kER * kMaxPieces, copies piece e % kMaxPieces of stage row
// e / kMaxPieces (aux0[u] = page id); lane l < ntok holds token l (aux1).
__device__ __forceinline__ void expand_lookup(const BgmvParams& p, const ECursor& c, int32_t (&aux0)[2],
                                              int32_t& aux1) {
  const int lane = threadIdx.x & 31;
  aux0[0] = aux0[1] = -1;
  aux1 = -1;
  if (!c.valid) return;
  const ETask& t = c.t;
  const SlotDev& L = p.slot[t.k];
  const int l0 = t.lc * kELC;
  const int Lo = min(kELC, L.d_out - l0);
  const int r0 = c.st * kER;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int e = lane + 32 * u;
    const int i = e / kMaxPieces, q = e % kMaxPieces;
    if (i < kER && r0 + i < t.r) {
      const int64_t f0 = (int64_t)(r0 + i) * L.d_out + l0;
      int64_t b, en;
      if (piece_range(p.pool, f0, f0 + Lo, q, b, en)) aux0[u] = page_id(p.pool, t.a, L.listB, b);
    }
  }
  if (lane < t.ntok) aux1 = __ldg(p.sc.perm + t.seg0 + t.tg * t.nt + lane);
}

__device__ __forceinline__ void expand_issue(const BgmvParams& p, const ECursor& c, const int32_t (&aux0)[2],
                                             int32_t aux1, unsigned char* buf, unsigned char* ybuf, int32_t* desc,
                                             uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const ETask& t = c.t;
  const SlotDev& L = p.slot[t.k];
  const int l0 = t.lc * kELC;
  const int Lo = min(kELC, L.d_out - l0);
  const int r0 = c.st * kER;
  const int nrows = min(kER, t.r - r0);
  const uint32_t tbytes = 4u * kER * L.t_ns;
  const int tk0 = __shfl_sync(FULL_MASK, aux1, 0), tk1 = __shfl_sync(FULL_MASK, aux1, 1);
  const int tk2 = __shfl_sync(FULL_MASK, aux1, 2), tk3 = __shfl_sync(FULL_MASK, aux1, 3);
  if (lane == 0) {
    ETask u = t;
    u.tok0 = tk0;
    u.tok1 = tk1;
    u.tok2 = tk2;
    u.tok3 = tk3;
    const int32_t* src = reinterpret_cast<const int32_t*>(&u);
    for (int q = 0; q < (int)(sizeof(ETask) / 4); ++q) desc[q] = src[q];
    desc[kDescInts - 2] = c.st;
    desc[kDescInts - 1] = 1;
    mbar_expect_tx(bar, 2u * Lo * nrows + tbytes * t.ntok + (c.st == 0 ? 2u * Lo * t.ntok : 0u));
  }
  __syncwarp();
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    if (aux0[u] >= 0) {
      const int e = lane + 32 * u;
      const int i = e / kMaxPieces, q = e % kMaxPieces;
      const int64_t f0 = (int64_t)(r0 + i) * L.d_out + l0;
      int64_t b, en;
      piece_range(p.pool, f0, f0 + Lo, q, b, en);
      bulk_g2s(buf + i * 2 * kELC + 2 * (b - f0), page_ptr(p.pool, aux0[u], b), (uint32_t)(2 * (en - b)), bar);
    }
  }
  if (lane < t.ntok) {
    const int64_t row = L.t_by_token ? (int64_t)aux1 : (int64_t)(t.seg0 + t.tg * t.nt + lane);
    bulk_g2s(buf + kEXT + lane * tbytes, L.t + row * L.t_rs + (int64_t)r0 * L.t_ns, tbytes, bar);
    if (c.st == 0) bulk_g2s(ybuf + lane * 2 * kELC, L.y + (int64_t)aux1 * L.ldy + l0, 2u * Lo, bar);
  }
}

template <int DT, int NT>
__device__ __forceinline__ void expand_consume(const BgmvParams& p, const ETask& t, int st,
                                               const unsigned char* buf, const unsigned char* yb,
                                               float (&acc)[4][8]) {
  const int lane = threadIdx.x & 31, cw = (threadIdx.x >> 5) - kProd;
  const SlotDev& L = p.slot[t.k];
  const int l0 = t.lc * kELC;
  const int Lo = min(kELC, L.d_out - l0);
  const int l = cw * 256 + lane * 8;
  const bool act = l < Lo;
  const int r0 = st * kER;
  const int nrows = min(kER, t.r - r0);
  // t of (token tt, row kk) summed over the t_ns partials by lane kER tt + kk
  float tsum = 0.f;
  {
    const int tt = lane / kER, kk = lane % kER;
    if (tt < t.ntok && kk < nrows) {
      const float* src = reinterpret_cast<const float*>(buf + kEXT + tt * 4 * kER * L.t_ns) + kk * L.t_ns;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;  // four chains; fixed association
      int c = 0;
      for (; c + 4 <= L.t_ns; c += 4) {
        s0 += src[c];
        s1 += src[c + 1];
        s2 += src[c + 2];
        s3 += src[c + 3];
      }
      for (; c < L.t_ns; ++c) s0 += src[c];
      tsum = (s0 + s1) + (s2 + s3);
    }
  }
  float tv[NT][kER];  // broadcast by every lane, before the lane-dependent part
#pragma unroll
  for (int tt = 0; tt < NT; ++tt)
#pragma unroll
    for (int kk = 0; kk < kER; ++kk) tv[tt][kk] = __shfl_sync(FULL_MASK, tsum, kER * tt + kk);
  if (act) {
#pragma unroll
    for (int kk = 0; kk < kER; ++kk) {
      if (kk >= nrows) break;
      float bf[8];
      unpack8<DT>(lds128(buf + kk * 2 * kELC + 2 * l), bf);
#pragma unroll
      for (int tt = 0; tt < NT; ++tt)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[tt][e] = fmaf(tv[tt][kk], bf[e], acc[tt][e]);
    }
  }
  if (st != t.nst - 1) return;
  const float s_a = __ldg(p.pool.scale + t.a);
  const int tokv[4] = {t.tok0, t.tok1, t.tok2, t.tok3};
#pragma unroll
  for (int tt = 0; tt < NT; ++tt) {
    if (act && tt < t.ntok) {
      float yf[8];
      unpack8<DT>(lds128(yb + tt * 2 * kELC + 2 * l), yf);
      uint4 o;
      o.x = pack2<DT>(fmaf(s_a, acc[tt][0], yf[0]), fmaf(s_a, acc[tt][1], yf[1]));
      o.y = pack2<DT>(fmaf(s_a, acc[tt][2], yf[2]), fmaf(s_a, acc[tt][3], yf[3]));
      o.z = pack2<DT>(fmaf(s_a, acc[tt][4], yf[4]), fmaf(s_a, acc[tt][5], yf[5]));
      o.w = pack2<DT>(fmaf(s_a, acc[tt][6], yf[6]), fmaf(s_a, acc[tt][7], yf[7]));
      *reinterpret_cast<uint4*>(L.y + (int64_t)tokv[tt] * L.ldy + l0 + l) = o;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[tt][e] = 0.f;
  }
}

template <int DT>
__global__ void __launch_bounds__(kPipeThreads, 1) k_expand(const __grid_constant__ BgmvParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[kENS], empty[kENS];
  __shared__ int ydone[2];  // consumer warps done with each y buffer (kCW per task)
  __shared__ TaskClaims claims;
  __shared__ int warm_sink;
  __shared__ int32_t desc[kENS][kDescInts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* ybufs = smem + kERingBytes;
  int32_t* segsm = reinterpret_cast<int32_t*>(ybufs + 2 * kYBufBytes);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kENS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    ydone[0] = ydone[1] = 0;
    fence_mbar_init();
  }
  warm_params(p, &warm_sink);
  griddep_wait();
  const int S = p.sc.meta[kMetaS];
  const int total = p.sc.meta[kMetaExpandTotal];
  const SegView V = stage_segments(p.sc, S, false, segsm);
  if (threadIdx.x == 0) claims_init(claims, total);
  __syncthreads();
  if (warp < kProd) {
    // producer `warp` issues the stages at positions warp, warp + kProd, ...
    // of the CTA's (task, stage) sequence, into ring slots of the same parity
    ECursor A, B;
    A.task = task_of(claims, 0, p.sc.meta + kMetaExpandClaim, p.pool.err);
    A.ord = 0;
    A.st = 0;
    A.valid = A.task >= 0 && A.task < total;
    if (A.valid) decode_expand(p, V, A.task, 0, A.t);
    for (int q = 0; q < warp; ++q) ecursor_next(p, V, total, claims, A);
    // page ids of a position are looked up two of this warp's issues ahead;
    // A's lookups are in flight while B is walked
    int32_t a0[2], a1, b0[2], b1;
    expand_lookup(p, A, a0, a1);
    B = A;
    for (int q = 0; q < kProd; ++q) ecursor_next(p, V, total, claims, B);
    expand_lookup(p, B, b0, b1);
    uint32_t eparity = 0;
    int ring = warp % kENS, uses = 0;
    while (A.valid) {
      if (uses >= kENS / kProd) {
        if (!mbar_wait(&empty[ring], (eparity >> ring) & 1, p.pool.err)) break;
        eparity ^= 1u << ring;
      }
      if (A.st == 0) {  // the y buffer of CTA task n is free once tasks n - 2, n - 4, ... are consumed
        const int n = A.ord;
        if (n >= 2 && !counter_wait(&ydone[n & 1], kCW * (n >> 1), p.pool.err)) break;
      }
      expand_issue(p, A, a0, a1, smem + ring * kEStageBytes, ybufs + A.t.yb * kYBufBytes, desc[ring],
                   &full[ring]);
      a0[0] = b0[0];
      a0[1] = b0[1];
      a1 = b1;
      A = B;
      for (int q = 0; q < kProd; ++q) ecursor_next(p, V, total, claims, B);
      expand_lookup(p, B, b0, b1);
      ring = (ring + kProd) % kENS;
      ++uses;
    }
    // end marker at this producer's next position (the consumers stop at the
    // first one in sequence order)
    if (uses >= kENS / kProd) mbar_wait(&empty[ring], (eparity >> ring) & 1, p.pool.err);
    if (lane == 0) {
      desc[ring][kDescInts - 1] = 0;
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&full[ring])) : "memory");
    }
  } else {
    float acc[4][8];
#pragma unroll
    for (int tt = 0; tt < 4; ++tt)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[tt][e] = 0.f;
    uint32_t fparity = 0;
    int ring = 0;
    for (;;) {
      if (!mbar_wait(&full[ring], (fparity >> ring) & 1, p.pool.err)) break;
      fparity ^= 1u << ring;
      if (desc[ring][kDescInts - 1] == 0) break;
      ETask t;
      int32_t* dst = reinterpret_cast<int32_t*>(&t);
#pragma unroll
      for (int q = 0; q < (int)(sizeof(ETask) / 4); ++q) dst[q] = desc[ring][q];
      const int st = desc[ring][kDescInts - 2];
      const unsigned char* buf = smem + ring * kEStageBytes;
      const unsigned char* yb = ybufs + t.yb * kYBufBytes;
      switch (t.nt) {
        case 1: expand_consume<DT, 1>(p, t, st, buf, yb, acc); break;
        case 2: expand_consume<DT, 2>(p, t, st, buf, yb, acc); break;
        default: expand_consume<DT, 4>(p, t, st, buf, yb, acc); break;
      }
      // the slot's generic-proxy reads before the next bulk copy into it
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&empty[ring])) : "memory");
        if (st == t.nst - 1) atomicAdd(&ydone[t.yb], 1);
      }
      ring = (ring + 1) % kENS;
    }
  }
  griddep_launch();
}

// ---------------------------------------------------------------------------
// slora_bgmv_shrink's output: t_out[token][k] = sum over the d_in slices.
__global__ void __launch_bounds__(256) k_reduce_t(const __grid_constant__ BgmvParams p) {
  griddep_wait();
  const SlotDev& L = p.slot[0];
  const int S = p.sc.meta[kMetaS];
  const int n_valid = p.sc.meta[kMetaValid];
  const int RK = (int)(L.t_rs / L.t_ns);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < (int64_t)n_valid * RK;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int pos = (int)(e / RK), k = (int)(e % RK);
    const int s = S > 0 ? find_seg(p.sc.seg_start, S, pos) : 0;
    if (k >= p.sc.seg_rank[s]) continue;
    float acc = 0.f;
    for (int c = 0; c < L.t_ns; ++c) acc += L.t[(int64_t)pos * L.t_rs + (int64_t)k * L.t_ns + c];
    L.tout[(int64_t)p.sc.perm[pos] * L.ldt_out + k] = acc;
  }
}

// ---------------------------------------------------------------------------
// Prefill segments from requests (one CTA of 1024 threads).
__global__ void __launch_bounds__(1024) k_merge_requests(const int32_t* __restrict__ req_start,
                                                         const int32_t* __restrict__ req_adapter,
                                                         int n, int32_t* seg_start,
                                                         int32_t* seg_adapter, int32_t* S_out) {
  __shared__ int sh[32];
  const int tid = threadIdx.x, nth = blockDim.x;
  const int E = (n + nth - 1) / nth;
  const int q0 = min(tid * E, n), q1 = min(q0 + E, n);
  // last non-empty request before each position (max-scan of indices)
  int last = -1;
  for (int q = q0; q < q1; ++q)
    if (req_start[q + 1] > req_start[q]) last = q;
  int total;
  int prev = block_exscan<true>(last, &total, sh);  // last non-empty strictly before q0
  int cnt = 0;
  {
    int pv = prev;
    for (int q = q0; q < q1; ++q) {
      if (req_start[q + 1] <= req_start[q]) continue;
      if (pv < 0 || req_adapter[pv] != req_adapter[q]) ++cnt;
      pv = q;
    }
  }
  int S;
  int base = block_exscan<false>(cnt, &S, sh);
  for (int q = q0; q < q1; ++q) {
    if (req_start[q + 1] <= req_start[q]) continue;
    if (prev < 0 || req_adapter[prev] != req_adapter[q]) {
      seg_start[base] = req_start[q];
      seg_adapter[base] = req_adapter[q];
      ++base;
    }
    prev = q;
  }
  const int end = n > 0 ? req_start[n] : 0;
  if (tid == 0) {
    seg_start[S] = end;
    *S_out = S;
  }
  // pad to n segments with empty ones, so the arrays can go to slora_sgmv with S = n
  for (int q = S + tid; q < n; q += nth) {
    seg_start[q + 1] = end;
    seg_adapter[q] = -1;
  }
}

// ---------------------------------------------------------------------------
// Page-in: each CTA copies whole pages; the descriptor lives in pinned host
// memory (read through its device-mapped address).
struct PageInConst {
  int d_in[kMaxSlots], d_out[kMaxSlots], listA[kMaxSlots], listB[kMaxSlots];
};

__global__ void __launch_bounds__(256) k_page_in(PoolDev P, PageInConst C, const char* desc,
                                                 int64_t total_units) {
  const PageInHeader* H = reinterpret_cast<const PageInHeader*>(desc);
  const int n_new = H->n_new, n_proj = H->n_proj;
  const PageInNew* NW = reinterpret_cast<const PageInNew*>(desc + H->off_new);
  const int32_t* EV = reinterpret_cast<const int32_t*>(desc + H->off_evict);
  const int64_t P_el = 1ll << P.page_shift;
  // table updates: evictions, then new entries
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e < H->n_evict; e += blockDim.x) P.rank[EV[e]] = -1;
  for (int u = blockIdx.x; u < n_new; u += gridDim.x) {
    const PageInNew& w = NW[u];
    const int32_t* row = reinterpret_cast<const int32_t*>(desc + w.list_off);
    for (int64_t e = threadIdx.x; e < H->list_stride; e += blockDim.x)
      P.page_list[(int64_t)w.id * H->list_stride + e] = row[e];
    if (threadIdx.x == 0) {
      P.rank[w.id] = w.rank;
      P.scale[w.id] = w.scale;
    }
    if (w.qs_off >= 0) {  // e4m3 row scales into the adapter's table row
      const float* qs = reinterpret_cast<const float*>(desc + w.qs_off);
      for (int e = threadIdx.x; e < n_proj * 2 * w.rank; e += blockDim.x) {
        const int t = e / w.rank, k = e % w.rank;
        P.qscale[((int64_t)w.id * n_proj * 2 + t) * P.max_rank + k] = qs[e];
      }
    }
  }
  if (!H->copy_data) return;
  for (int64_t u = blockIdx.x; u < total_units; u += gridDim.x) {
    // adapter owning unit u
    int lo = 0, hi = n_new - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (NW[mid].unit_base <= u) lo = mid;
      else hi = mid - 1;
    }
    const PageInNew& w = NW[lo];
    const int32_t* row = reinterpret_cast<const int32_t*>(desc + w.list_off);
    int64_t c = u - w.unit_base;
    // tensor owning page c: order (p, A), (p, B) over p
    int tensor = 0;
    int64_t nel = 0;
    int lofs = 0;
    for (tensor = 0; tensor < 2 * n_proj; ++tensor) {
      const int pj = tensor >> 1;
      nel = (int64_t)w.rank * ((tensor & 1) ? C.d_out[pj] : C.d_in[pj]);
      const int64_t np = (nel + P_el - 1) / P_el;
      if (c < np) {
        lofs = (tensor & 1) ? C.listB[pj] : C.listA[pj];
        break;
      }
      c -= np;
    }
    const uint16_t* src = w.host[tensor >> 1][tensor & 1] + c * P_el;
    uint16_t* dst = P.pool + ((int64_t)row[lofs + c] << P.page_shift);
    const int64_t n_el = min(P_el, nel - c * P_el);
    const int nv = (int)(P_el / 8), nv_src = (int)(n_el / 8);
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    for (int v = threadIdx.x; v < nv; v += 4 * blockDim.x) {
      uint4 t[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int vv = v + j * blockDim.x;
        t[j] = vv < nv_src ? s4[vv] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int vv = v + j * blockDim.x;
        if (vv < nv) d4[vv] = t[j];
      }
    }
  }
}

// Debug read-back of one tensor into a dense device buffer.
__global__ void k_gather_debug(PoolDev P, int id, int d, int list_off, int rank, uint16_t* out) {
  const int64_t nv = (int64_t)rank * d / 8;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nv;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t f = v * 8;
    reinterpret_cast<uint4*>(out)[v] = *reinterpret_cast<const uint4*>(page_addr(P, id, list_off, f));
  }
}

// ---------------------------------------------------------------------------
// Launchers.
constexpr int kDynSmem = kERingBytes + 2 * kYBufBytes + 4 * kSegSmemInts;  // expand: ring, y, segments
constexpr int kSDynSmem = kSRingBytes + 2 * kXBufBytes + 4 * kSegSmemInts;  // shrink: ring, x, segments
static_assert(kSDynSmem <= 227 * 1024 - 2048 && kDynSmem <= 227 * 1024 - 2048, "shared memory");
template <typename Kern>
static cudaError_t launch_dependent(Kern kernel, int grid, int block, size_t smem, cudaStream_t s,
                                    const BgmvParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

static bool g_attrs_done = false;
static cudaError_t set_attrs() {
  if (g_attrs_done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k_segments, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_shrink<SLORA_F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSDynSmem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_shrink<SLORA_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSDynSmem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_expand<SLORA_F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_expand<SLORA_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem);
  if (e == cudaSuccess) g_attrs_done = true;
  return e;
}

cudaError_t launch_segments(BgmvParams& p, const int32_t* idx, int T, cudaStream_t s) {
  p.idx = idx;
  p.T = T;
  cudaError_t ea = set_attrs();
  if (ea != cudaSuccess) return ea;
  const size_t smem = sizeof(int) * (size_t)p.pool.max_adapters;
  k_segments<<<1, 1024, smem, s>>>(p, idx, T);
  return cudaGetLastError();
}

cudaError_t launch_shrink(const BgmvParams& p, int dtype, int grid, cudaStream_t s) {
  cudaError_t ea = set_attrs();
  if (ea != cudaSuccess) return ea;
  if (dtype == SLORA_BF16) return launch_dependent(k_shrink<SLORA_BF16>, grid, kPipeThreads, kSDynSmem, s, p);
  return launch_dependent(k_shrink<SLORA_F16>, grid, kPipeThreads, kSDynSmem, s, p);
}

cudaError_t launch_expand(const BgmvParams& p, int dtype, int grid, cudaStream_t s) {
  cudaError_t ea = set_attrs();
  if (ea != cudaSuccess) return ea;
  if (dtype == SLORA_BF16) return launch_dependent(k_expand<SLORA_BF16>, grid, kPipeThreads, kDynSmem, s, p);
  return launch_dependent(k_expand<SLORA_F16>, grid, kPipeThreads, kDynSmem, s, p);
}

cudaError_t launch_reduce_t(const BgmvParams& p, int T, cudaStream_t s) {
  const int64_t n = (int64_t)T * (p.slot[0].t_rs / p.slot[0].t_ns);
  const int grid = (int)std::min<int64_t>(std::max<int64_t>((n + 255) / 256, 1), 1184);
  return launch_dependent(k_reduce_t, grid, 256, 0, s, p);
}

cudaError_t launch_merge_requests(const int32_t* req_start, const int32_t* req_adapter, int n,
                                  int32_t* seg_start, int32_t* seg_adapter, int32_t* S_out,
                                  cudaStream_t s) {
  k_merge_requests<<<1, 1024, 0, s>>>(req_start, req_adapter, n, seg_start, seg_adapter, S_out);
  return cudaGetLastError();
}

cudaError_t launch_page_in(const PoolDev& pool, const int* d_in, const int* d_out,
                           const int* listA, const int* listB, const void* desc_dev,
                           int64_t total_units, int grid, cudaStream_t s) {
  PageInConst C;
  for (int i = 0; i < kMaxSlots; ++i) {
    C.d_in[i] = d_in[i];
    C.d_out[i] = d_out[i];
    C.listA[i] = listA[i];
    C.listB[i] = listB[i];
  }
  k_page_in<<<grid, 256, 0, s>>>(pool, C, reinterpret_cast<const char*>(desc_dev), total_units);
  return cudaGetLastError();
}

cudaError_t launch_gather_debug(const PoolDev& pool, int id, int d, int list_off, int rank,
                                uint16_t* out_dev, cudaStream_t s) {
  const int64_t nv = (int64_t)rank * d / 8;
  int grid = (int)((nv + 255) / 256);
  if (grid < 1) grid = 1;
  if (grid > 4096) grid = 4096;
  k_gather_debug<<<grid, 256, 0, s>>>(pool, id, d, list_off, rank, out_dev);
  return cudaGetLastError();
}

// Resident CTAs per SM of the persistent decode kernels (shared memory bound).
int occupancy_blocks(int which) {
  set_attrs();
  int n = 0;
  if (which == 0) cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_shrink<SLORA_F16>, kPipeThreads, kSDynSmem);
  else cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_expand<SLORA_F16>, kPipeThreads, kDynSmem);
  return n > 0 ? n : 1;
}

}  // namespace slora
