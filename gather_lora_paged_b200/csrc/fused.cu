// fused.cu -- the decode delta as one persistent kernel (sm_100a).
//
// One launch computes, for a decode batch in which every token names its own
// adapter (-1: none),
//     y_i <- y_i + (alpha_a / r_a) * ((x_i . A_a) . B_a)
// over up to eight projections of one layer: the two phases of the SGMV
// formulation ("Multi-LoRA serving: S-LoRA, Punica, SGMV, vLLM", SGMV section:
// shrink d -> r, then expand r -> d_out), the whole heterogeneous batch in one
// launch with the weights fetched from paged memory by adapter id ("Paper
// explainer: S-LoRA", BGMV kernel section), several LoRA linear maps in one
// kernel ("Multi-LoRA inference optimisation", the remark on merging them).
//
// Structure (one CTA per SM, all CTAs resident: cooperative launch):
//  1. Every CTA builds the batch's segment table in shared memory -- a stable
//     counting sort of the tokens by adapter id, then per segment the number
//     and byte cost of its shrink and expand tasks.  All CTAs compute the same
//     table, so no separate kernel and no grid barrier is needed.
//  2. Shrink tasks (segment, x group, 16 rank rows, 2048-wide slice of d_in, up
//     to 8 tokens) leave one fp32 partial per (token, rank row, slice) in
//     scratch; expand tasks (segment, projection, 2048 outputs, up to 4 tokens)
//     sum their rank rows' partials in slice order and update y in place,
//     rounding once.  Each CTA takes a contiguous, byte-balanced range of the
//     shrink tasks, then one of the expand tasks.  The expand ranges are
//     offset by half a range, so the shrink tasks an expand task needs ran
//     about half a phase earlier; it still waits (bounded) on a counter per
//     (segment, x group) that shrink consumers bump once their partials are
//     visible.
//  3. Inside a CTA a resolver warp walks the CTA's stage sequence ahead of the
//     copies and fetches the page ids of every stage's row slices straight into
//     shared memory with asynchronous 4-byte copies (cp.async: several stages'
//     lookups in flight, so page-table misses in L2 do not stall it); an issuer
//     warp turns resolved stages into bulk copies (cp.async.bulk, completion
//     counted on the stage's mbarrier) into a ring of shared-memory stages;
//     eight consumer warps compute on each stage; a signaller warp publishes
//     each finished shrink task to the other CTAs (a gpu-scope fence, then the
//     ready counter), so no compute warp ever waits on global visibility.
// Arithmetic is that of the three-kernel path in bgmv.cu: fp32 accumulation,
// partials summed in slice order, one rounding of y.
#include "dev_common.cuh"

namespace slora {

namespace {

constexpr int kFCW = 8;                        // consumer warps
constexpr int kFW0 = 3;                        // first consumer warp (after resolver, issuer, signaller)
constexpr int kFThreads = (kFW0 + kFCW) * 32;
constexpr int kFNS = 4;                        // ring stages
constexpr int kFLook = 12;                     // resolved stages held ahead of the issuer
constexpr int kFLookAhead = 4;                 // stages of page-id copies in flight in the resolver
constexpr int kFXYBufs = 4;                    // x / y buffers: a task's buffer is free once
                                               // the task kFXYBufs earlier is consumed
constexpr int kFSigQ = 32;                     // shrink tasks queued for the signaller
constexpr int kFRows = 8;                      // row slices per stage (one per consumer warp)
constexpr int kFKT = 2048;                     // slice length (elements)
constexpr int kFRB = 16;                       // shrink task: rank rows
constexpr int kFELC = kFCW * 256;              // expand task: outputs (256 per consumer warp)
constexpr int kFRowBytes = 2 * kFKT;
constexpr int kFTBytes = 4 * kFRows * 16 * 4;  // t partials of a stage: 4 tokens x 8 rows x <= 16 slices
constexpr int kFEXT = kFRows * kFRowBytes;     // offset of the t partials in a stage
constexpr int kFStageBytes = kFEXT + kFTBytes;
constexpr int kFXYBytes = 4 * kFRowBytes;      // x or y rows of <= 4 tokens
constexpr int kFRankShift = 21;                // histogram entry: count | (rank + 1) << 21
constexpr int kFTabBytes = ((2 * kFMaxT + 8 * kFSegCap + 8 * (kFSegCap + 1)) + 15) / 16 * 16;
constexpr int kFDynSmem = kFNS * kFStageBytes + kFXYBufs * kFXYBytes + kFTabBytes;
static_assert(kFLookAhead < kFLook, "lookahead within the resolved-stage ring");
static_assert(kFKT == kPartK && kFKT == kShrinkKT, "partials are per 2048-element slice");
static_assert(kFRows * kMaxPieces <= 64, "two lookups per lane");
static_assert(kFThreads % 4 == 0 && kFMaxT % 4 == 0, "int4 alignment of the prologue arrays");

// One stage of the CTA's sequence, as the resolver decodes it and the issuer
// hands it to the consumers.
struct FDesc {
  int kind;      // 0: end of the sequence, 1: shrink, 2: expand
  int gk;        // x group (shrink) or projection slot (expand)
  int a, r;      // adapter, rank
  int seg;       // segment index
  int pos0;      // position (token order of the segment table) of the task's first token
  int ntok, nt;  // tokens of the task, token class (template NT)
  int st, nst;   // stage of the task, stages of the task
  int ch;        // d_in slice (shrink) or 2048-output chunk (expand)
  int rb;        // shrink: block of 16 rank rows of the group
  int nrows;     // shrink: rank rows of the task
  int buf;       // x / y buffer of the task
  int need;      // expand: value of the ready counter once its partials are in
  int m;         // task ordinal within the CTA (issuer)
  float s_a;     // expand: alpha / r of the adapter (fetched by the resolver)
  int tok[8];    // token ids at positions pos0 .. pos0 + ntok (resolver)
};
constexpr int kFDescInts = (int)(sizeof(FDesc) / 4);
constexpr int kFDescHead = kFDescInts - 9;  // fields before s_a and tok

struct FLook {
  FDesc d;
  int32_t pg[64];  // page id of each (row slice, piece) entry, -1 when unused
  float qs[8];     // e4m3 weights: the scales of the stage's row slices
};

struct FRanges {
  int S;             // segments
  int n_s, n_e;      // shrink / expand tasks
  int s0, s1;        // this CTA's shrink tasks
  int e0, e1;        // this CTA's expand tasks (virtual: index mod n_e)
  int last;          // this CTA finished last (clears the ready counters)
};

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* c) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
  return v;
}

// Bounded wait (one thread) until the global counter *c reaches target.
__device__ bool ready_wait(const int32_t* c, int target, int32_t* err) {
  long long t0 = -1;
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire_gpu(c) >= target) return true;
    if ((it & 15) == 0) {
      const long long now = clock64();
      if (t0 < 0) t0 = now;
      else if (now - t0 > kWaitLimit) {
        record_error(err, 4, (int)blockIdx.x);
        return false;
      }
    }
    __nanosleep(64);
  }
}

// Task counts and byte cost (256-byte units) of one segment of n tokens on a
// rank-r adapter.  Cost: the bytes each task streams through the copy ring
// (a token group after the first re-reads the rows, from L2 mostly, but its
// stages take the ring just the same), activations, and 2 KB per stage.
__device__ void seg_costs(const BgmvParams& p, int n, int r, int& n_s, int& n_e, int& c_s, int& c_e) {
  n_s = n_e = c_s = c_e = 0;
  if (n <= 0 || r <= 0) return;
  const int ntg = cdiv_i(n, nt_class(n)), nte = cdiv_i(n, nte_class(n));
  int64_t bs = 0, be = 0;
  for (int g = 0; g < p.n_groups; ++g) {
    const GroupDev& G = p.group[g];
    const int rows = G.n * r, ns = cdiv_i(G.d_in, kFKT);
    const int tasks = cdiv_i(rows, kFRB) * ntg * ns;
    n_s += tasks;
    bs += 2ll * G.d_in * ((int64_t)rows * ntg + n) + 2048ll * 2 * tasks;
  }
  for (int k = 0; k < p.n_slots; ++k) {
    const SlotDev& L = p.slot[k];
    const int tasks = nte * cdiv_i(L.d_out, kFELC);
    n_e += tasks;
    be += 2ll * L.d_out * ((int64_t)r * nte + 2 * n) + 2048ll * cdiv_i(r, kFRows) * tasks;
  }
  c_s = (int)(bs >> 8);
  c_e = (int)(be >> 8);
}

// Task index at cost position pos: the segment holding pos, then a share of
// its tasks proportional to the position inside it.
__device__ int task_at(const int* pre, const int* cpre, int S, int64_t pos) {
  int lo = 0, hi = S;
  while (lo < hi) {  // largest s with cpre[s] <= pos
    const int mid = (lo + hi + 1) >> 1;
    if (cpre[mid] <= pos) lo = mid;
    else hi = mid - 1;
  }
  if (lo >= S) return pre[S];
  const int64_t c = cpre[lo + 1] - cpre[lo];
  const int nt = pre[lo + 1] - pre[lo];
  const int q = c > 0 ? (int)(((pos - cpre[lo]) * nt) / c) : 0;
  return pre[lo] + min(q, nt);
}

__device__ __forceinline__ void seg_unpack(const int* sega, const int* segb, int s, int& start, int& n, int& a,
                                           int& r) {
  const int u = sega[s], v = segb[s];
  start = u & 0xffff;
  n = u >> 16;
  a = v & 0xffff;
  r = v >> 16;
}

// Shrink task: within a segment, groups in order; within a group, tasks run
// over (rank-row block, d_in slice, token group) with the token group fastest,
// so consecutive tasks stream the same row slices (the repeats hit L2).
__device__ void decode_s(const BgmvParams& p, const int* spre, const int* sega, const int* segb, int S, int task,
                         FDesc& d) {
  const int s = find_seg(spre, S, task);
  int q = task - spre[s];
  int start, n;
  seg_unpack(sega, segb, s, start, n, d.a, d.r);
  d.kind = 1;
  d.seg = s;
  d.nt = nt_class(n);
  const int ntg = cdiv_i(n, d.nt);
  int g = 0;
  for (; g < p.n_groups - 1; ++g) {
    const int cnt = cdiv_i(p.group[g].n * d.r, kFRB) * ntg * cdiv_i(p.group[g].d_in, kFKT);
    if (q < cnt) break;
    q -= cnt;
  }
  d.gk = g;
  const int ns = cdiv_i(p.group[g].d_in, kFKT);
  const int tg = q % ntg;
  q /= ntg;
  d.ch = q % ns;
  d.rb = q / ns;
  d.nrows = min(kFRB, p.group[g].n * d.r - d.rb * kFRB);
  d.nst = cdiv_i(d.nrows, kFRows);
  d.pos0 = start + tg * d.nt;
  d.ntok = min(d.nt, n - tg * d.nt);
  d.st = 0;
  d.need = 0;
}

// Expand task: within a segment, slots in order; within a slot, (output chunk,
// token group) with the token group fastest.
__device__ void decode_e(const BgmvParams& p, const int* epre, const int* sega, const int* segb, int S, int task,
                         FDesc& d) {
  const int s = find_seg(epre, S, task);
  int q = task - epre[s];
  int start, n;
  seg_unpack(sega, segb, s, start, n, d.a, d.r);
  d.kind = 2;
  d.seg = s;
  d.nt = nte_class(n);
  const int ntg = cdiv_i(n, d.nt);
  int k = 0;
  for (; k < p.n_slots - 1; ++k) {
    const int cnt = ntg * cdiv_i(p.slot[k].d_out, kFELC);
    if (q < cnt) break;
    q -= cnt;
  }
  d.gk = k;
  const int tg = q % ntg;
  d.ch = q / ntg;
  d.nst = cdiv_i(d.r, kFRows);
  d.pos0 = start + tg * d.nt;
  d.ntok = min(d.nt, n - tg * d.nt);
  d.st = 0;
  d.rb = 0;
  d.nrows = d.r;
  // the shrink tasks of (segment, the slot's x group): one ready count each
  const GroupDev& G = p.group[p.slot[k].group];
  d.need = cdiv_i(G.n * d.r, kFRB) * cdiv_i(n, nt_class(n)) * cdiv_i(G.d_in, kFKT);
}

__device__ __forceinline__ void cp_async4(int32_t* dst, const int32_t* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Weight elements of a tensor are 16-bit elements (WF = 0) or e4m3 codes (WF =
// 1, two to a 16-bit unit); a page holds page_elems units.  Piece q of the
// weight range [f0, f1) cut at page boundaries, and the address of element f.
template <int WF>
__device__ __forceinline__ bool wpiece(const PoolDev& P, int64_t f0, int64_t f1, int q, int64_t& b, int64_t& e) {
  const int sh = P.page_shift + WF;
  const int64_t pb0 = ((f0 >> sh) + 1) << sh;
  b = q == 0 ? f0 : pb0 + (int64_t)(q - 1) * (1ll << sh);
  e = pb0 + (int64_t)q * (1ll << sh);
  if (e > f1) e = f1;
  return b < f1;
}
template <int WF>
__device__ __forceinline__ const unsigned char* wptr(const PoolDev& P, int32_t pg, int64_t f) {
  return reinterpret_cast<const unsigned char*>(P.pool) + ((int64_t)pg << (P.page_shift + 1)) +
         ((f & ((1ll << (P.page_shift + WF)) - 1)) << (1 - WF));
}

// Page ids of a stage's row slices, fetched into pg[] with asynchronous copies
// (the caller commits them as one group): entry e = lane + 32 u is piece e % 5
// of row slice e / 5 (-1 where there is none).  e4m3 weights: lane i < 8 also
// fetches the scale of row slice i into qs[i].
template <int WF>
__device__ __forceinline__ void stage_lookups(const BgmvParams& p, const FDesc& d, int32_t* pg, float* qs) {
  const int lane = threadIdx.x & 31;
  const int64_t row0 = (int64_t)d.a * p.pool.list_stride;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int e = lane + 32 * u;
    const int i = e / kMaxPieces, q = e % kMaxPieces;
    const int32_t* src = nullptr;
    if (d.kind == 1) {
      const GroupDev& G = p.group[d.gk];
      const int k0 = d.ch * kFKT;
      const int L = min(kFKT, G.d_in - k0);
      if (i < kFRows && d.st * kFRows + i < d.nrows) {
        const int rho = d.rb * kFRB + d.st * kFRows + i;
        const int j = rho / d.r, k = rho % d.r;
        const int64_t f0 = (int64_t)k * G.d_in + k0;
        int64_t b, en;
        if (wpiece<WF>(p.pool, f0, f0 + L, q, b, en))
          src = p.pool.page_list + row0 + p.slot[G.slot[j]].listA + (b >> (p.pool.page_shift + WF));
      }
    } else if (d.kind == 2) {
      const SlotDev& L = p.slot[d.gk];
      const int l0 = d.ch * kFELC;
      const int Lo = min(kFELC, L.d_out - l0);
      const int r0 = d.st * kFRows;
      if (i < kFRows && r0 + i < d.r) {
        const int64_t f0 = (int64_t)(r0 + i) * L.d_out + l0;
        int64_t b, en;
        if (wpiece<WF>(p.pool, f0, f0 + Lo, q, b, en))
          src = p.pool.page_list + row0 + L.listB + (b >> (p.pool.page_shift + WF));
      }
    }
    if (src) cp_async4(pg + e, src);
    else pg[e] = -1;
  }
  if (WF == 1 && lane < kFRows) {
    const float* qsrc = nullptr;
    if (d.kind == 1 && d.st * kFRows + lane < d.nrows) {
      const int rho = d.rb * kFRB + d.st * kFRows + lane;
      const int proj = p.slot[p.group[d.gk].slot[rho / d.r]].proj;
      qsrc = p.pool.qscale + ((int64_t)(d.a * p.pool.n_proj + proj) * 2 + 0) * p.pool.max_rank + rho % d.r;
    } else if (d.kind == 2 && d.st * kFRows + lane < d.r) {
      const int proj = p.slot[d.gk].proj;
      qsrc = p.pool.qscale + ((int64_t)(d.a * p.pool.n_proj + proj) * 2 + 1) * p.pool.max_rank + d.st * kFRows + lane;
    }
    if (qsrc) cp_async4(reinterpret_cast<int32_t*>(qs + lane), reinterpret_cast<const int32_t*>(qsrc));
    else qs[lane] = 0.f;
  }
}

// e4m3 pair -> f16 pair (exact: every e4m3 value is an fp16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((unsigned short)two));
  return r;
}
// Eight e4m3 codes -> fp32, exactly.
__device__ __forceinline__ void unpack8_e4m3(const uint2& v, float* f) {
  const uint32_t w[2] = {v.x, v.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    h2x2f(e4m3x2_to_f16x2(w[i] & 0xffffu), f[4 * i], f[4 * i + 1]);
    h2x2f(e4m3x2_to_f16x2(w[i] >> 16), f[4 * i + 2], f[4 * i + 3]);
  }
}
// acc + a.lo * x.lo + a.hi * x.hi for an e4m3 code pair a and a 16-bit pair x.
template <int DT>
__device__ __forceinline__ float fma2_e4m3(uint32_t a2, uint32_t x2, float acc) {
  const uint32_t h = e4m3x2_to_f16x2(a2);
  if (DT == SLORA_F16) return fma2_16<SLORA_F16>(h, x2, acc);
  float a0, a1;
  h2x2f(h, a0, a1);
  acc = fmaf(a0, __uint_as_float(x2 << 16), acc);
  return fmaf(a1, __uint_as_float(x2 & 0xffff0000u), acc);
}
__device__ __forceinline__ uint2 lds64(const unsigned char* p) { return *reinterpret_cast<const uint2*>(p); }

// ---------------------------------------------------------------------------
// Consumers.  Shrink: warp w owns row slice w of the stage and writes one fp32
// partial per (row, token) of the slice; four accumulator chains per token
// (256-element chunk c feeds chain c % 4), summed in chain order.
template <int DT, int NT, int WF>
__device__ __forceinline__ void f_shrink(const BgmvParams& p, const FDesc& t, int cw, const unsigned char* buf,
                                         const unsigned char* xb, const float* qs) {
  const int lane = threadIdx.x & 31;
  if (t.st * kFRows + cw >= t.nrows) return;  // warp-uniform
  const GroupDev& G = p.group[t.gk];
  const int L = min(kFKT, G.d_in - t.ch * kFKT);
  constexpr int kC = kFKT / 256;
  float acc[4][NT];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) acc[c][tt] = 0.f;
  const unsigned char* arow = buf + cw * kFRowBytes;
#pragma unroll
  for (int c0 = 0; c0 < kC; c0 += 4) {
    const int e0 = c0 * 256 + lane * 8;
    if (e0 >= L) break;
    uint4 av[4];  // 16-bit weights: 8 elements; e4m3: 8 codes in .x, .y
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (WF == 1) {
        const uint2 v = e0 + c * 256 < L ? lds64(arow + (e0 + c * 256)) : make_uint2(0, 0);
        av[c] = make_uint4(v.x, v.y, 0, 0);
      } else {
        av[c] = e0 + c * 256 < L ? lds128(arow + 2 * (e0 + c * 256)) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) {
      if (tt >= t.ntok) break;
      uint4 xv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        xv[c] = e0 + c * 256 < L ? lds128(xb + tt * kFRowBytes + 2 * (e0 + c * 256)) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float s0 = acc[c][tt];
        if (WF == 1) {
          s0 = fma2_e4m3<DT>(av[c].x & 0xffffu, xv[c].x, s0);
          s0 = fma2_e4m3<DT>(av[c].x >> 16, xv[c].y, s0);
          s0 = fma2_e4m3<DT>(av[c].y & 0xffffu, xv[c].z, s0);
          s0 = fma2_e4m3<DT>(av[c].y >> 16, xv[c].w, s0);
        } else {
          s0 = fma2_16<DT>(av[c].x, xv[c].x, s0);
          s0 = fma2_16<DT>(av[c].y, xv[c].y, s0);
          s0 = fma2_16<DT>(av[c].z, xv[c].z, s0);
          s0 = fma2_16<DT>(av[c].w, xv[c].w, s0);
        }
        acc[c][tt] = s0;
      }
    }
  }
  float v[NT];
#pragma unroll
  for (int tt = 0; tt < NT; ++tt) v[tt] = (acc[0][tt] + acc[1][tt]) + (acc[2][tt] + acc[3][tt]);
  float val = lane_transpose_reduce<NT>(v);  // lane tt < NT holds token tt's sum
  if (WF == 1) val *= qs[cw];               // the row's scale
  const int rho = t.rb * kFRB + t.st * kFRows + cw;
  const int j = rho / t.r, k = rho % t.r;
  const SlotDev& S = p.slot[G.slot[j]];
  if (lane < NT && lane < t.ntok)
    S.t[(int64_t)(t.pos0 + lane) * S.t_rs + (int64_t)k * S.t_ns + t.ch] = val;
}

// Expand: warp w owns outputs [256 w, 256 w + 256) of the task's chunk, lane l
// eight consecutive ones; acc (token x output) runs over the task's stages.
template <int DT, int NT, int WF>
__device__ __forceinline__ void f_expand(const BgmvParams& p, const FDesc& t, int cw, const unsigned char* buf,
                                         const unsigned char* yb, const float* qs, float (&acc)[4][8]) {
  const int lane = threadIdx.x & 31;
  const SlotDev& L = p.slot[t.gk];
  const int l0 = t.ch * kFELC;
  const int Lo = min(kFELC, L.d_out - l0);
  const int l = cw * 256 + lane * 8;
  const bool act = l < Lo;
  const int r0 = t.st * kFRows;
  const int nrows = min(kFRows, t.r - r0);
  // t of (token tt, row kk): lane kFRows tt + kk sums the t_ns slice partials
  float tsum = 0.f;
  {
    const int tt = lane / kFRows, kk = lane % kFRows;
    if (tt < t.ntok && kk < nrows) {
      const float* src = reinterpret_cast<const float*>(buf + kFEXT + tt * 4 * kFRows * L.t_ns) + kk * L.t_ns;
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
      if (WF == 1) tsum *= qs[kk];  // B's row scale folded into t
    }
  }
  float tv[NT][kFRows];
#pragma unroll
  for (int tt = 0; tt < NT; ++tt)
#pragma unroll
    for (int kk = 0; kk < kFRows; ++kk) tv[tt][kk] = __shfl_sync(FULL_MASK, tsum, kFRows * tt + kk);
  if (act) {
#pragma unroll
    for (int kk = 0; kk < kFRows; ++kk) {
      if (kk >= nrows) break;
      float bf[8];
      if (WF == 1) unpack8_e4m3(lds64(buf + kk * kFRowBytes + l), bf);
      else unpack8<DT>(lds128(buf + kk * kFRowBytes + 2 * l), bf);
#pragma unroll
      for (int tt = 0; tt < NT; ++tt)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[tt][e] = fmaf(tv[tt][kk], bf[e], acc[tt][e]);
    }
  }
  if (t.st != t.nst - 1) return;
  const float s_a = t.s_a;
#pragma unroll
  for (int tt = 0; tt < NT; ++tt) {
    if (act && tt < t.ntok) {
      float yf[8];
      unpack8<DT>(lds128(yb + tt * kFRowBytes + 2 * l), yf);
      uint4 o;
      o.x = pack2<DT>(fmaf(s_a, acc[tt][0], yf[0]), fmaf(s_a, acc[tt][1], yf[1]));
      o.y = pack2<DT>(fmaf(s_a, acc[tt][2], yf[2]), fmaf(s_a, acc[tt][3], yf[3]));
      o.z = pack2<DT>(fmaf(s_a, acc[tt][4], yf[4]), fmaf(s_a, acc[tt][5], yf[5]));
      o.w = pack2<DT>(fmaf(s_a, acc[tt][6], yf[6]), fmaf(s_a, acc[tt][7], yf[7]));
      *reinterpret_cast<uint4*>(L.y + (int64_t)t.tok[tt] * L.ldy + l0 + l) = o;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[tt][e] = 0.f;
  }
}

// The resolver's position in the CTA's stage sequence.
struct FCursor {
  FDesc d;
  int ph;     // 0: shrink range, 1: expand range, 2: past the end
  int v;      // task (virtual index in the expand range)
};

__device__ __forceinline__ void cursor_task(const BgmvParams& p, const FRanges& R, const int* spre, const int* epre,
                                            const int* sega, const int* segb, FCursor& c) {
  // move to the first phase with a task left at or after c.v, decode it
  for (;;) {
    if (c.ph == 0) {
      if (c.v < R.s1) {
        decode_s(p, spre, sega, segb, R.S, c.v, c.d);
        return;
      }
      c.ph = 1;
      c.v = R.e0;
    }
    if (c.ph == 1) {
      if (c.v < R.e1) {
        decode_e(p, epre, sega, segb, R.S, c.v % R.n_e, c.d);
        return;
      }
      c.ph = 2;
    }
    c.d.kind = 0;
    c.d.st = 0;
    c.d.nst = 1;
    return;
  }
}

__device__ __forceinline__ void cursor_next(const BgmvParams& p, const FRanges& R, const int* spre, const int* epre,
                                            const int* sega, const int* segb, FCursor& c) {
  if (c.ph == 2) return;
  if (++c.d.st < c.d.nst) return;
  ++c.v;
  cursor_task(p, R, spre, epre, sega, segb, c);
}

template <int DT, int WF>
__global__ void __launch_bounds__(kFThreads, 1) k_delta(const __grid_constant__ BgmvParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[kFNS], empty[kFNS];
  __shared__ FLook look[kFLook];
  __shared__ FDesc desc[kFNS];
  __shared__ float dqs[kFNS][8];  // e4m3: row scales of each ring stage
  __shared__ int resolved, issued, xydone[kFXYBufs], warm_sink;
  __shared__ int sigq[kFSigQ], sig_n, sig_done;
  __shared__ FRanges R;
  unsigned char* ring = smem;
  unsigned char* xy = smem + kFNS * kFStageBytes;
  unsigned char* tab = xy + kFXYBufs * kFXYBytes;
  uint16_t* perm = reinterpret_cast<uint16_t*>(tab);
  int* sega = reinterpret_cast<int*>(tab + 2 * kFMaxT);  // start | n << 16
  int* segb = sega + kFSegCap;                           // adapter | rank << 16
  int* spre = segb + kFSegCap;                           // shrink tasks before each segment
  int* epre = spre + kFSegCap + 1;                       // expand tasks before each segment
  const int tid = threadIdx.x, nth = blockDim.x, warp = tid >> 5, lane = tid & 31;
  const int T = p.T, MA = p.pool.max_adapters;
  int32_t* err = p.pool.err;

  {  // touch every 64-byte line of the parameter block once, so that later
     // lookups with runtime indices (groups, slots) hit the constant cache
    constexpr int kLines = (int)((sizeof(BgmvParams) + 63) / 64);
    if (tid < kLines) {
      const int v = reinterpret_cast<const int*>(&p)[tid * 16];
      if (v == 0x5a5a5a5a) warm_sink = v;  // keeps the load; the value is never used
    }
  }
  if (tid == 0) {
    for (int s = 0; s < kFNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFCW);
    }
    resolved = issued = sig_n = sig_done = 0;
    for (int b = 0; b < kFXYBufs; ++b) xydone[b] = 0;
    fence_mbar_init();
  }

  // ---- 1. the segment table (prologue scratch lives in the ring area) -----
  int* hist = reinterpret_cast<int*>(ring);
  int* keys = hist + ((MA + 3) & ~3);
  int* ck = keys + kFMaxT;
  int4* sh4 = reinterpret_cast<int4*>(ck + kFThreads);
  int* cpre_s = reinterpret_cast<int*>(sh4 + 32);
  int* cpre_e = cpre_s + kFSegCap + 1;
  for (int a = tid; a < MA; a += nth) hist[a] = 0;
  __syncthreads();
  for (int i = tid; i < T; i += nth) {
    const int a = p.idx[i];
    int key = -1;
    if (a != -1) {
      if (a < -1 || a >= MA) {
        if (blockIdx.x == 0) record_error(err, 1, i);
      } else {
        const int r = p.pool.rank[a];
        if (r < 0) {
          if (blockIdx.x == 0) record_error(err, 2, i);
        } else {
          atomicOr(&hist[a], (r + 1) << kFRankShift);
          atomicAdd(&hist[a], 1);
          key = a;
        }
      }
    }
    keys[i] = key;
  }
  __syncthreads();
  // segments: each thread owns a contiguous adapter range
  {
    const int E = (MA + nth - 1) / nth;
    const int a0 = min(tid * E, MA), a1 = min(a0 + E, MA);
    int4 c = make_int4(0, 0, 0, 0);
    for (int a = a0; a < a1; ++a) {
      const int h = hist[a];
      if (h == 0) continue;
      c.x += h & ((1 << kFRankShift) - 1);
      c.y += 1;
    }
    int4 tot;
    const int4 base = block_exscan4(c, &tot, sh4);
    int cb = base.x, sb = base.y;
    for (int a = a0; a < a1; ++a) {
      const int h = hist[a];
      hist[a] = cb;  // becomes the scatter cursor
      if (h == 0) continue;
      const int n = h & ((1 << kFRankShift) - 1), r = (h >> kFRankShift) - 1;
      sega[sb] = cb | (n << 16);
      segb[sb] = a | (r << 16);
      ++sb;
      cb += n;
    }
    if (tid == 0) R.S = tot.y;
  }
  __syncthreads();
  const int S = R.S;
  // L2 hint for the page lists of segments b, b + G, ... (every CTA a share)
  for (int s = (int)blockIdx.x; s < S; s += (int)gridDim.x) {
    const int v = segb[s], a = v & 0xffff, r = v >> 16;
    if (r <= 0) continue;
    const int32_t* row = p.pool.page_list + (int64_t)a * p.pool.list_stride;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(row) & ~(uintptr_t)127;
    const uintptr_t e = reinterpret_cast<uintptr_t>(row + p.pool.list_stride);
    for (uintptr_t l = b0 + 128 * (uintptr_t)tid; l < e; l += 128 * (uintptr_t)nth)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(l));
  }
  // stable scatter, one chunk of nth tokens at a time: a token's place among
  // its adapter's tokens of the chunk = equal keys in earlier warps (counted
  // from the chunk's keys) + equal keys in earlier lanes of its own warp
  for (int c0 = 0; c0 < T; c0 += nth) {
    const int i = c0 + tid;
    const int a = i < T ? keys[i] : -1;
    ck[tid] = a;
    __syncthreads();
    const unsigned m = __match_any_sync(FULL_MASK, a);
    if (a >= 0) {
      int before = __popc(m & ((1u << lane) - 1));
      const int4* k4 = reinterpret_cast<const int4*>(ck);
      for (int j = 0; j < warp * 8; ++j) {
        const int4 v = k4[j];
        before += (v.x == a) + (v.y == a) + (v.z == a) + (v.w == a);
      }
      perm[hist[a] + before] = (uint16_t)i;
    }
    __syncthreads();
    if (a >= 0 && lane == __ffs(m) - 1) atomicAdd(&hist[a], __popc(m));
    __syncthreads();
  }
  // task counts and costs per segment, prefix sums
  {
    const int E = (S + nth - 1) / nth;
    const int s0 = min(tid * E, S), s1 = min(s0 + E, S);
    int4 c = make_int4(0, 0, 0, 0);
    for (int s = s0; s < s1; ++s) {
      int ns, ne, cs, ce;
      seg_costs(p, sega[s] >> 16, segb[s] >> 16, ns, ne, cs, ce);
      c.x += ns;
      c.y += ne;
      c.z += cs;
      c.w += ce;
    }
    int4 tot;
    const int4 base = block_exscan4(c, &tot, sh4);
    int4 run = base;
    for (int s = s0; s < s1; ++s) {
      spre[s] = run.x;
      epre[s] = run.y;
      cpre_s[s] = run.z;
      cpre_e[s] = run.w;
      int ns, ne, cs, ce;
      seg_costs(p, sega[s] >> 16, segb[s] >> 16, ns, ne, cs, ce);
      run.x += ns;
      run.y += ne;
      run.z += cs;
      run.w += ce;
    }
    if (tid == 0) {
      spre[S] = tot.x;
      epre[S] = tot.y;
      cpre_s[S] = tot.z;
      cpre_e[S] = tot.w;
    }
  }
  __syncthreads();
  // this CTA's ranges: shrink [b, b + 1) / G of the cost, expand offset by half
  if (tid == 0) {
    const int64_t G = gridDim.x, b = blockIdx.x;
    const int64_t CS = cpre_s[S], CE = cpre_e[S];
    R.n_s = spre[S];
    R.n_e = epre[S];
    R.s0 = task_at(spre, cpre_s, S, b * CS / G);
    R.s1 = task_at(spre, cpre_s, S, (b + 1) * CS / G);
    auto vtask = [&](int64_t pos) {
      return pos < CE ? task_at(epre, cpre_e, S, pos) : R.n_e + task_at(epre, cpre_e, S, pos - CE);
    };
    R.e0 = CE > 0 ? vtask((2 * b + 1) * CE / (2 * G)) : 0;
    R.e1 = CE > 0 ? vtask((2 * b + 3) * CE / (2 * G)) : 0;
    R.last = 0;
  }
  __syncthreads();

  // ---- 2. the pipeline ----------------------------------------------------
  if (warp == 0) {
    // resolver: decode the sequence into the lookahead slots; page ids (and the
    // expand scale) arrive by cp.async, kFLookAhead stages of them in flight
    FCursor cur;
    cur.ph = 0;
    cur.v = R.s0;
    cursor_task(p, R, spre, epre, sega, segb, cur);
    int n = 0;
    bool ended = false;
    for (;; ++n) {
      if (n >= kFLook && !counter_wait(&issued, n - kFLook + 1, err)) break;
      FLook& L = look[n % kFLook];
      if (lane == 0) {
        const int32_t* src = reinterpret_cast<const int32_t*>(&cur.d);
        int32_t* dst = reinterpret_cast<int32_t*>(&L.d);
        for (int q = 0; q < kFDescHead; ++q) dst[q] = src[q];
        if (cur.d.kind == 2) cp_async4(reinterpret_cast<int32_t*>(&L.d.s_a),
                                       reinterpret_cast<const int32_t*>(p.pool.scale + cur.d.a));
        else L.d.s_a = 0.f;
      }
      if (lane < 8) L.d.tok[lane] = (cur.d.kind != 0 && lane < cur.d.ntok) ? (int)perm[cur.d.pos0 + lane] : 0;
      if (cur.d.kind != 0) stage_lookups<WF>(p, cur.d, L.pg, L.qs);
      asm volatile("cp.async.commit_group;" ::: "memory");
      if (n >= kFLookAhead) {  // stages up to n - kFLookAhead are complete
        asm volatile("cp.async.wait_group %0;" ::"n"(kFLookAhead) : "memory");
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          st_volatile_s32(&resolved, n - kFLookAhead + 1);
        }
      }
      if (cur.d.kind == 0) {
        ended = true;
        break;
      }
      cursor_next(p, R, spre, epre, sega, segb, cur);
    }
    // the last stages (through the end marker); after a failed wait only the
    // stages written so far
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      st_volatile_s32(&resolved, ended ? n + 1 : n);
    }
  } else if (warp == 1) {
    // issuer: resolved stages -> bulk copies into the ring
    uint32_t eparity = 0;
    int m = -1;          // task ordinal
    bool sig_end = false;
    for (int n = 0;; ++n) {
      if (!counter_wait(&resolved, n + 1, err)) break;
      const FLook& L = look[n % kFLook];
      FDesc d;
      {
        const int32_t* src = reinterpret_cast<const int32_t*>(&L.d);
        int32_t* dst = reinterpret_cast<int32_t*>(&d);
#pragma unroll
        for (int q = 0; q < kFDescInts; ++q) dst[q] = src[q];
      }
      const int32_t pg0 = L.pg[lane], pg1 = L.pg[lane + 32];
      const float qsl = WF == 1 ? L.qs[lane & 7] : 0.f;
      const int tokl = L.d.tok[lane & 7];  // token of position pos0 + lane (lane < ntok)
      if (!sig_end && d.kind != 1) {  // no shrink task follows: tell the signaller
        if (lane == 0) {
          if (m + 1 >= kFSigQ) counter_wait(&sig_done, m + 2 - kFSigQ, err);
          sigq[(m + 1) % kFSigQ] = -1;
          __threadfence_block();
          st_volatile_s32(&sig_n, m + 2);
        }
        sig_end = true;
      }
      const int ring_i = n % kFNS;
      if (n >= kFNS) {
        if (!mbar_wait(&empty[ring_i], (eparity >> ring_i) & 1, err)) break;
        eparity ^= 1u << ring_i;
      }
      if (d.kind == 0) {
        if (lane == 0) {
          desc[ring_i].kind = 0;
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&full[ring_i])) : "memory");
        }
        break;
      }
      if (d.st == 0) {
        ++m;
        const int b = m % kFXYBufs;  // free once the task kFXYBufs earlier is consumed
        if (m >= kFXYBufs && !counter_wait(&xydone[b], kFCW * (m / kFXYBufs), err)) break;
        if (d.kind == 1) {  // queue the shrink task for the signaller
          int ok = 1;
          if (lane == 0) {
            if (m >= kFSigQ) ok = counter_wait(&sig_done, m + 1 - kFSigQ, err) ? 1 : 0;
            sigq[m % kFSigQ] = d.seg * p.n_groups + d.gk;
            __threadfence_block();
            st_volatile_s32(&sig_n, m + 1);
          }
          if (!__shfl_sync(FULL_MASK, ok, 0)) break;
        } else {  // expand: the partials of its (segment, x group) must be in
          int ok = 1;
          if (lane == 0)
            ok = ready_wait(p.sc.ready + d.seg * p.n_groups + p.slot[d.gk].group, d.need, err) ? 1 : 0;
          ok = __shfl_sync(FULL_MASK, ok, 0);
          __syncwarp();
          if (!ok) break;
          asm volatile("fence.proxy.async.global;" ::: "memory");  // partials written by other SMs' stores
        }
      }
      d.m = m;
      d.buf = m % kFXYBufs;
      unsigned char* stage = ring + ring_i * kFStageBytes;
      unsigned char* xyb = xy + d.buf * kFXYBytes;
      const int32_t pgs[2] = {pg0, pg1};
      if (d.kind == 1) {
        const GroupDev& G = p.group[d.gk];
        const int k0 = d.ch * kFKT;
        const int Lk = min(kFKT, G.d_in - k0);
        const int rows = min(kFRows, d.nrows - d.st * kFRows);
        if (WF == 1 && lane < 8) dqs[ring_i][lane] = qsl;
        if (lane == 0) {
          int32_t* dd = reinterpret_cast<int32_t*>(&desc[ring_i]);
          const int32_t* ss = reinterpret_cast<const int32_t*>(&d);
          for (int q = 0; q < kFDescInts; ++q) dd[q] = ss[q];
          mbar_expect_tx(&full[ring_i], (2u - WF) * Lk * rows + (d.st == 0 ? 2u * Lk * d.ntok : 0u));
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (pgs[u] >= 0) {
            const int e = lane + 32 * u;
            const int i = e / kMaxPieces, q = e % kMaxPieces;
            const int rho = d.rb * kFRB + d.st * kFRows + i;
            const int64_t f0 = (int64_t)(rho % d.r) * G.d_in + k0;
            int64_t b, en;
            wpiece<WF>(p.pool, f0, f0 + Lk, q, b, en);
            bulk_g2s(stage + i * kFRowBytes + (2 - WF) * (b - f0), wptr<WF>(p.pool, pgs[u], b),
                     (uint32_t)((2 - WF) * (en - b)), &full[ring_i]);
          }
        }
        if (d.st == 0 && lane < d.ntok)
          bulk_g2s(xyb + lane * kFRowBytes, G.x + (int64_t)tokl * G.ldx + k0, 2u * Lk, &full[ring_i]);
      } else {
        const SlotDev& L2 = p.slot[d.gk];
        const int l0 = d.ch * kFELC;
        const int Lo = min(kFELC, L2.d_out - l0);
        const int r0 = d.st * kFRows;
        const int nrows = min(kFRows, d.r - r0);
        const uint32_t tbytes = 4u * kFRows * L2.t_ns;
        if (WF == 1 && lane < 8) dqs[ring_i][lane] = qsl;
        if (lane == 0) {
          int32_t* dd = reinterpret_cast<int32_t*>(&desc[ring_i]);
          const int32_t* ss = reinterpret_cast<const int32_t*>(&d);
          for (int q = 0; q < kFDescInts; ++q) dd[q] = ss[q];
          mbar_expect_tx(&full[ring_i],
                         (2u - WF) * Lo * nrows + tbytes * d.ntok + (d.st == 0 ? 2u * Lo * d.ntok : 0u));
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (pgs[u] >= 0) {
            const int e = lane + 32 * u;
            const int i = e / kMaxPieces, q = e % kMaxPieces;
            const int64_t f0 = (int64_t)(r0 + i) * L2.d_out + l0;
            int64_t b, en;
            wpiece<WF>(p.pool, f0, f0 + Lo, q, b, en);
            bulk_g2s(stage + i * kFRowBytes + (2 - WF) * (b - f0), wptr<WF>(p.pool, pgs[u], b),
                     (uint32_t)((2 - WF) * (en - b)), &full[ring_i]);
          }
        }
        if (lane < d.ntok) {
          bulk_g2s(stage + kFEXT + lane * tbytes, L2.t + (int64_t)(d.pos0 + lane) * L2.t_rs + (int64_t)r0 * L2.t_ns,
                   tbytes, &full[ring_i]);
          if (d.st == 0)
            bulk_g2s(xyb + lane * kFRowBytes, L2.y + (int64_t)tokl * L2.ldy + l0, 2u * Lo, &full[ring_i]);
        }
      }
      __syncwarp();
      if (lane == 0) st_volatile_s32(&issued, n + 1);
    }
    if (!sig_end && lane == 0) {  // an early exit: release the signaller
      sigq[(m + 1) % kFSigQ] = -1;
      __threadfence_block();
      st_volatile_s32(&sig_n, m + 2);
    }
  } else if (warp == 2) {
    // signaller: shrink task m's partials are in once all consumer warps have
    // finished it; publish them to the other CTAs in task order
    for (int m = 0;; ++m) {
      if (!counter_wait(&sig_n, m + 1, err)) break;
      const int v = ld_volatile_s32(&sigq[m % kFSigQ]);
      if (v < 0) break;
      if (!counter_wait(&xydone[m % kFXYBufs], kFCW * (m / kFXYBufs + 1), err)) break;
      if (lane == 0) {
        __threadfence();  // the consumers' partials (ordered before their xydone arrivals)
        atomicAdd(p.sc.ready + v, 1);
        st_volatile_s32(&sig_done, m + 1);
      }
      __syncwarp();
    }
  } else {
    // consumers
    const int cw = warp - kFW0;
    float acc[4][8];
#pragma unroll
    for (int tt = 0; tt < 4; ++tt)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[tt][e] = 0.f;
    uint32_t fparity = 0;
    for (int n = 0;; ++n) {
      const int ring_i = n % kFNS;
      if (!mbar_wait(&full[ring_i], (fparity >> ring_i) & 1, err)) break;
      fparity ^= 1u << ring_i;
      FDesc t;
      {
        const int32_t* src = reinterpret_cast<const int32_t*>(&desc[ring_i]);
        int32_t* dst = reinterpret_cast<int32_t*>(&t);
#pragma unroll
        for (int q = 0; q < kFDescInts; ++q) dst[q] = src[q];
      }
      if (t.kind == 0) break;
      const unsigned char* buf = ring + ring_i * kFStageBytes;
      const unsigned char* xyb = xy + t.buf * kFXYBytes;
      const bool last = t.st == t.nst - 1;
      if (t.kind == 1) {
        const float* qs = dqs[ring_i];
        switch (t.nt) {
          case 1: f_shrink<DT, 1, WF>(p, t, cw, buf, xyb, qs); break;
          case 2: f_shrink<DT, 2, WF>(p, t, cw, buf, xyb, qs); break;
          default: f_shrink<DT, 4, WF>(p, t, cw, buf, xyb, qs); break;
        }
      } else {
        const float* qs = dqs[ring_i];
        switch (t.nt) {
          case 1: f_expand<DT, 1, WF>(p, t, cw, buf, xyb, qs, acc); break;
          case 2: f_expand<DT, 2, WF>(p, t, cw, buf, xyb, qs, acc); break;
          default: f_expand<DT, 4, WF>(p, t, cw, buf, xyb, qs, acc); break;
        }
      }
      // the slot's generic-proxy reads before the next bulk copy into it
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      // a shrink task's t partials, stored by every lane, visible to the whole
      // GPU before the signaller counts the task (another warp's fence alone
      // does not order this warp's stores)
      if (last && t.kind == 1) __threadfence();
      __syncwarp();
      if (lane == 0) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&empty[ring_i])) : "memory");
        if (last) {
          __threadfence_block();  // this warp's partial stores before its arrival
          atomicAdd(&xydone[t.buf], 1);
        }
      }
    }
  }

  // ---- 3. the last CTA to finish clears the ready counters ----------------
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    R.last = atomicAdd(p.sc.ready + kFReadyCap, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (R.last) {
    __threadfence();
    for (int i = tid; i < S * p.n_groups; i += nth) p.sc.ready[i] = 0;
    if (tid == 0) p.sc.ready[kFReadyCap] = 0;
  }
}

bool g_fused_attrs = false;

}  // namespace

int fused_grid_bound(const BgmvParams& p, int T) {
  // tasks per phase are at most T x (tasks of one token's segment): each
  // segment has ceil(n / class) <= n token groups
  int64_t ns = 0, ne = 0;
  const int r = std::max(1, p.pool.max_rank);
  for (int g = 0; g < p.n_groups; ++g)
    ns += (int64_t)cdiv_i(p.group[g].n * r, kFRB) * cdiv_i(p.group[g].d_in, kFKT);
  for (int k = 0; k < p.n_slots; ++k) ne += cdiv_i(p.slot[k].d_out, kFELC);
  const int64_t b = (int64_t)T * std::max(ns, ne);
  return (int)std::min<int64_t>(std::max<int64_t>(b, 1), 1 << 20);
}

cudaError_t launch_fused(BgmvParams& p, int dtype, const int32_t* idx, int T, int grid, cudaStream_t s) {
  p.idx = idx;
  p.T = T;
  if (T > kFMaxT || p.sc.ready == nullptr) return cudaErrorInvalidValue;
  if (!g_fused_attrs) {
    cudaError_t e = cudaSuccess;
    const void* ks[4] = {(const void*)k_delta<SLORA_F16, 0>, (const void*)k_delta<SLORA_BF16, 0>,
                         (const void*)k_delta<SLORA_F16, 1>, (const void*)k_delta<SLORA_BF16, 1>};
    for (int i = 0; i < 4 && e == cudaSuccess; ++i)
      e = cudaFuncSetAttribute(ks[i], cudaFuncAttributeMaxDynamicSharedMemorySize, kFDynSmem);
    if (e != cudaSuccess) return e;
    g_fused_attrs = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = kFDynSmem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: expand tasks wait on other CTAs
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const bool q8 = p.pool.wfmt == SLORA_WEIGHTS_E4M3;
  if (dtype == SLORA_BF16)
    return q8 ? cudaLaunchKernelEx(&cfg, k_delta<SLORA_BF16, 1>, p) : cudaLaunchKernelEx(&cfg, k_delta<SLORA_BF16, 0>, p);
  return q8 ? cudaLaunchKernelEx(&cfg, k_delta<SLORA_F16, 1>, p) : cudaLaunchKernelEx(&cfg, k_delta<SLORA_F16, 0>, p);
}

}  // namespace slora
