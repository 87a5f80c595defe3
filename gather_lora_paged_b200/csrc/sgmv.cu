// sgmv.cu -- SGMV prefill path on the 5th-generation tensor cores (sm_100a).
//
// Prefill segments are contiguous token ranges that share one adapter
// ("Multi-LoRA serving: S-LoRA, Punica, SGMV, vLLM", SGMV section: segments of
// tokens per adapter, dispatched to the Tensor Cores; FAQ: ranks padded into
// uniform bands to keep tensor-core alignment).  Per segment the delta is two
// small GEMMs:
//   shrink  t[128 x R] = X[128 x d_in] . A_t^T      (R = projections x rank)
//   expand  y[128 x 128] += s * t[128 x r] . B[r x 128]
// with fp32 accumulators in tensor memory (TMEM).
//
// Operands in shared memory use the 128-byte-swizzled canonical layouts:
//   * X tiles and y tiles come from ordinary tiled TMA loads (64 x 128 boxes);
//   * adapter rows live in scattered pages.  Shrink: the A rows of a stage are
//     copied with per-thread 16-byte cp.async straight into the swizzled
//     K-major layout (by the warps that later run the epilogue).  Expand: the
//     pool is viewed as a 2-D tensor of 64-element rows and TMA tile::gather4
//     fetches four such rows (any four pool rows) per instruction into
//     MN-major atoms of 8 ranks x 64 outputs;
//   * t enters the expand as two 16-bit halves, t = hi + lo with hi = RN(t),
//     lo = RN(t - hi); both products with B are exact in fp32, so the
//     intermediate keeps about twice the 16-bit precision.
// All mbarrier waits are bounded and record an error instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "tc_common.cuh"

namespace slora {

namespace {

using namespace tc;
constexpr int kBK = 64;              // K per stage (one 128-byte swizzle atom)
constexpr int kXTileBytes = kBM * kBK * 2;
constexpr int kShrinkThreads = 192;  // X producer, MMA, 4 A-loader / epilogue warps
constexpr int kALoaders = 128;       // shrink threads copying A rows (warps 2..5)
constexpr int kALag = 2;             // A copy groups in flight per loader thread (1 or 2)
constexpr int kEpiWarps = 8;         // expand epilogue warps (two per TMEM lane quarter)
constexpr int kExpandThreads = 64 + 32 * kEpiWarps;  // producer, MMA, epilogue warps
constexpr int kEN = 128;             // expand outputs per item (MMA N)
constexpr int kAcc = 4;              // expand TMEM accumulators (kAcc x kEN columns)
constexpr int kYTileBytes = kBM * kEN * 2;

struct SgmvPlan {      // scratch arrays of one call
  int32_t* seg_start;  // [S] first token of each segment (0 when skipped)
  int32_t* seg_end;    // [S] one past its last token (0 when skipped)
  int32_t* seg_adapter;
  int32_t* seg_rank;   // 0 when the segment is skipped
  int32_t* shrink_prefix;  // [S + 1]
  int32_t* expand_prefix;  // [S + 1]
  int32_t* meta;           // [0] shrink items, [1] expand items
};

struct SgmvParams {
  CUtensorMap xmap[kMaxSlots];  // per group: X as (d_in, T) with 64 x 128 boxes
  CUtensorMap poolmap;          // the pool as (64, rows) with 64 x 1 boxes (gather4)
  PoolDev pool;
  int n_groups;
  GroupDev group[kMaxSlots];
  int n_slots;
  SlotDev slot[kMaxSlots];
  SgmvPlan plan;
  const int32_t* user_seg_start;
  const int32_t* user_seg_adapter;
  int S, T;
  float* t;             // t of slot k: t + k * t_slot_stride, rows of t_ld floats
  int64_t t_slot_stride;
  int t_ld;
  int64_t pool_rows;    // rows of 64 elements in the pool (out-of-range coordinate)
  int ntot_max;         // max over groups of round_up(n * max_rank, 16)
  int stages;           // shrink pipeline depth
  int s_mq;             // shrink: 128-token tiles per item (share each A stage)
  int s_gorder[kMaxSlots];  // shrink: group indices, most expensive first
  int dtype;
  CUtensorMap ymap[kMaxSlots];  // per slot: y as (d_out, T) with 64 x 128 boxes
  int e_nb, e_ny;       // expand ring depths (B chunks, y tiles)
  int e_pair;           // expand: 128-token tiles per group (1, 2 or 4; one B gather serves them)
  int e_t_half;         // expand: bytes of one t half in shared memory
  int e_b_stage;        // expand: bytes of one B ring stage
};

// ---------------------------------------------------------------------------
// Plan: validate segments, per-segment tile counts, prefix sums (one CTA).
__global__ void __launch_bounds__(1024) k_sgmv_plan(const __grid_constant__ SgmvParams p) {
  __shared__ int sh[32];
  gd_launch();
  const int S = p.S, tid = threadIdx.x, nth = blockDim.x;
  const int E = (S + nth - 1) / nth;
  const int s0 = min(tid * E, S), s1 = min(s0 + E, S);
  int csh = 0, cex = 0;
  for (int s = s0; s < s1; ++s) {
    const int a = p.user_seg_adapter[s];
    const int b0 = p.user_seg_start[s], b1 = p.user_seg_start[s + 1];
    const int n = b1 - b0;
    int r = 0;
    if (b0 < 0 || b1 > p.T || n < 0) rec_err(p.pool.err, 6, s);  // segment outside [0, T)
    else if (a >= 0) {
      if (a >= p.pool.max_adapters) rec_err(p.pool.err, 1, s);
      else if (p.pool.rank[a] < 0) rec_err(p.pool.err, 2, s);
      else r = p.pool.rank[a];
    }
    const int mt = (r > 0 && n > 0) ? cdiv_d(n, kBM) : 0;
    csh += cdiv_d(mt, p.s_mq);
    int ex = 0;
    for (int k = 0; k < p.n_slots; ++k) ex += cdiv_d(p.slot[k].d_out, kEN);
    cex += mt * ex;
  }
  // block exclusive scans (two)
  auto scan = [&](int v, int* total) {
    const int lane = tid & 31, w = tid >> 5, nw = nth >> 5;
    int x = v;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sh[w] = x;
    __syncthreads();
    if (w == 0) {
      int q = lane < nw ? sh[lane] : 0;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, q, o);
        if (lane >= o) q += y;
      }
      sh[lane] = q;
    }
    __syncthreads();
    const int res = (w ? sh[w - 1] : 0) + x - v;
    *total = sh[nw - 1];
    __syncthreads();
    return res;
  };
  int tsh, tex;
  int bsh = scan(csh, &tsh);
  int bex = scan(cex, &tex);
  for (int s = s0; s < s1; ++s) {
    const int a = p.user_seg_adapter[s];
    const int b0 = p.user_seg_start[s], b1 = p.user_seg_start[s + 1];
    const int n = b1 - b0;
    const bool inb = b0 >= 0 && b1 <= p.T && n >= 0;
    const int r = (inb && a >= 0 && a < p.pool.max_adapters && p.pool.rank[a] > 0) ? p.pool.rank[a] : 0;
    const int mt = (r > 0 && n > 0) ? cdiv_d(n, kBM) : 0;
    p.plan.seg_start[s] = mt > 0 ? b0 : 0;
    p.plan.seg_end[s] = mt > 0 ? b1 : 0;
    p.plan.seg_adapter[s] = a;
    p.plan.seg_rank[s] = mt > 0 ? r : 0;
    p.plan.shrink_prefix[s] = bsh;
    p.plan.expand_prefix[s] = bex;
    bsh += cdiv_d(mt, p.s_mq);
    int ex = 0;
    for (int k = 0; k < p.n_slots; ++k) ex += cdiv_d(p.slot[k].d_out, kEN);
    bex += mt * ex;
  }
  if (tid == 0) {
    p.plan.shrink_prefix[S] = tsh;
    p.plan.expand_prefix[S] = tex;
    p.plan.meta[0] = tsh * p.n_groups;  // items: groups (most expensive first) x tile pairs
    p.plan.meta[1] = tex;
  }
}

// ---------------------------------------------------------------------------
// Shrink: one CTA per (segment, group, 128-token tile).
__global__ void __launch_bounds__(kShrinkThreads, 1) k_sgmv_shrink(const __grid_constant__ SgmvParams p) {
  extern __shared__ __align__(1024) unsigned char dsm[];
  __shared__ __align__(8) uint64_t full[8], empty[8], accb;
  __shared__ uint32_t tmem_slot;
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  gd_wait();
  const int total = p.plan.meta[0];
  const int item = blockIdx.x;
  if (item >= total) {
    gd_launch();
    return;
  }
  // items run group-major, the groups in descending cost (so the longest items
  // start first and the last wave is short), then over segments' tile pairs
  const int S = p.S;
  const int per_group = p.plan.shrink_prefix[S];
  const int g = p.s_gorder[item / per_group];
  const int qi = item % per_group;
  const int s = find_ge(p.plan.shrink_prefix, S, qi);
  const int q = qi - p.plan.shrink_prefix[s];
  const int seg0 = p.plan.seg_start[s], seg1 = p.plan.seg_end[s];
  const int mt = cdiv_d(seg1 - seg0, kBM);
  const int MQ = p.s_mq;
  const int mtq = cdiv_d(mt, MQ);
  if (mt <= 0 || q >= mtq || seg0 < 0 || seg1 > p.T) {  // inconsistent plan: record, do nothing
    if (threadIdx.x == 0) rec_err(p.pool.err, 7, item);
    gd_launch();
    return;
  }
  const int m = q * MQ;  // first tile of this item
  const int nq = min(MQ, mt - m);             // tiles of this item (share each A stage)
  const int a = p.plan.seg_adapter[s], r = p.plan.seg_rank[s];
  const GroupDev& G = p.group[g];
  const int R = G.n * r;
  const int NT = (R + 15) & ~15;
  const int row0 = seg0 + m * kBM;
  const int KB = G.d_in / kBK;
  const int ST = p.stages;
  const int stage_bytes = MQ * kXTileBytes + ((p.ntot_max * 128 + 1023) & ~1023);
  uint32_t ncols = 32;
  while ((int)ncols < nq * NT) ncols <<= 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      bar_init(&full[i], 1 + kALoaders);  // X producer (with its bytes) + A loader threads
      bar_init(&empty[i], 1);
    }
    bar_init(&accb, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(&tmem_slot, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // X producer: the stage's token tiles by tiled TMA (streamed once: evict first)
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_first();
      for (int kb = 0; kb < KB && ok; ++kb) {
        const int st = kb % ST;
        if (kb >= ST) ok = bar_wait(&empty[st], ((kb / ST) - 1) & 1, p.pool.err);
        if (!ok) break;
        unsigned char* xs = smem + st * stage_bytes;
        bar_expect(&full[st], nq * kXTileBytes);
        for (int i = 0; i < nq; ++i)
          tma_tile_2d_hint(xs + i * kXTileBytes, &p.xmap[g], kb * kBK, row0 + i * kBM, &full[st], pol_x);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t lbo = 16, sbo = 1024;
      for (int kb = 0; kb < KB && ok; ++kb) {
        const int st = kb % ST;
        ok = bar_wait(&full[st], (kb / ST) & 1, p.pool.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t xs = su32(smem + st * stage_bytes);
        const uint32_t as = xs + MQ * kXTileBytes;
        for (int i = 0; i < nq; ++i)
          for (int c0 = 0; c0 < NT; c0 += 256) {
            const int nc = min(256, NT - c0);
            const uint32_t id = idesc_f16(p.dtype, nc, 0);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t da = sdesc(xs + i * kXTileBytes + kk * 32, lbo, sbo);
              const uint64_t db = sdesc(as + c0 * 128 + kk * 32, lbo, sbo);
              mma_f16(tmem + i * NT + c0, da, db, id, (kb > 0 || kk > 0) ? 1u : 0u);
            }
          }
        mma_commit(&empty[st]);
      }
      mma_commit(&accb);
    }
    __syncwarp();
  } else {
    // warps 2..5 first load A: thread t copies 16-byte chunk t % 8 of rows
    // t / 8 + 16 i of every stage with cp.async into the 128-byte-swizzled
    // K-major layout (rows past R are zero-filled).  Copies are committed one
    // group per stage; a stage is released to the MMA kALag stages later,
    // after its group completed and a proxy fence made it visible to the
    // tensor cores.
    {
      const int et = threadIdx.x - 64, ch = et & 7, r0 = et >> 3;
      const int32_t* plist = p.pool.page_list + (int64_t)a * p.pool.list_stride;
      const int64_t pmask = (1ll << p.pool.page_shift) - 1;
      const uint64_t pol_a = policy_evict_last();  // adapter rows are re-read by every token tile
      const int lag = min(kALag, ST - 1);           // < ST: a stage is released before its slot is reused
      int kb = 0;
      for (; kb < KB && ok; ++kb) {
        const int st = kb % ST;
        if (kb >= ST) ok = bar_wait(&empty[st], ((kb / ST) - 1) & 1, p.pool.err);
        if (!ok) break;
        const uint32_t as = su32(smem + st * stage_bytes + MQ * kXTileBytes);
        for (int rho = r0; rho < NT; rho += 16) {
          const uint32_t dst = as + rho * 128 + ((ch ^ (rho & 7)) << 4);
          if (rho < R) {
            const int sj = rho / r, k = rho - sj * r;
            const int64_t f = (int64_t)k * G.d_in + (int64_t)kb * kBK + ch * 8;
            const int32_t pg = __ldg(plist + p.slot[G.slot[sj]].listA + (f >> p.pool.page_shift));
            const uint16_t* src = p.pool.pool + ((int64_t)pg << p.pool.page_shift) + (f & pmask);
            asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, 16, %2;" ::"r"(dst), "l"(src),
                         "l"(pol_a)
                         : "memory");
          } else {
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, 0;" ::"r"(dst), "l"(p.pool.pool) : "memory");
          }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (kb >= lag) {
          if (lag == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
          else asm volatile("cp.async.wait_group 2;" ::: "memory");
          fence_async_smem();
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&full[(kb - lag) % ST])) : "memory");
        }
      }
      // release the last stages (every group issued completes before exit)
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      fence_async_smem();
      for (int k2 = max(0, kb - lag); k2 < kb; ++k2)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&full[k2 % ST])) : "memory");
    }
    // epilogue warps 2..5: TMEM lanes 32 * (warp % 4)
    ok = bar_wait(&accb, 0, p.pool.err) && ok;
    tc_fence_after();
    const int quarter = warp & 3;
    const int mrow = quarter * 32 + lane;
    for (int ci = 0; ci < nq * NT; ci += 16) {
      const int i = ci / NT, c = ci - i * NT;  // tile, column within it
      const int token = row0 + i * kBM + mrow;
      const bool valid = token < seg1;
      uint32_t v[16];
      tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + ci, v);
      if (!valid || !ok) continue;
      const int sj0 = c / r, k0 = c - sj0 * r;
      if (c + 16 <= R && k0 + 16 <= r && (k0 & 3) == 0) {  // 16 ranks of one slot: vector stores
        float4* tt = reinterpret_cast<float4*>(p.t + (int64_t)G.slot[sj0] * p.t_slot_stride +
                                               (int64_t)token * p.t_ld + k0);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          tt[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                              __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        continue;
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int rho = c + e;
        if (rho < R) {
          const int sj = rho / r, k = rho % r;
          float* tt = p.t + (int64_t)G.slot[sj] * p.t_slot_stride + (int64_t)token * p.t_ld + k;
          *tt = __uint_as_float(v[e]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, ncols);
  gd_launch();
}


// ---------------------------------------------------------------------------
// Expand: persistent CTAs (one per SM) over the item sequence
//   (segment, 128-token tile m, projection slot k, 128-output chunk c)
// in that order; CTA b takes the contiguous item range [b N / G, (b+1) N / G).
// Warp 0 produces: B chunk (r16 ranks x 128 outputs, MN-major atoms, gather4
// from the pages) into an NB-stage ring and the y tile (128 tokens x 128
// outputs, two 64 x 128 TMA boxes) into an NY-stage ring.  Warp 1 issues the
// MMAs into one of kAcc TMEM accumulators of 128 columns.  Warps 2..5 (one
// token row per thread) convert t to hi/lo halves when a new (tile, slot)
// unit starts, and drain each accumulator: y <- RN(y + s * acc) in place in
// shared memory, then 16-byte coalesced stores of the rows inside the segment.

struct ECur {  // a point of the item sequence
  int s, g, k, c, i;  // segment, tile group, slot, chunk, tile within the group
  int mt, nm, nch;    // tiles of segment s, tiles of group g, chunks of slot k
  bool valid;
};

__device__ __forceinline__ int seg_tiles(const SgmvParams& p, int s) {
  return p.plan.seg_rank[s] > 0 ? cdiv_d(p.plan.seg_end[s] - p.plan.seg_start[s], kBM) : 0;
}

// Within a segment the items run over groups of PS consecutive 128-token tiles
// (the last group may be shorter), then slots, then 128-output chunks, then
// the group's tiles: one B chunk serves the group's tiles, one conversion of
// the group's t rows serves all its slot's chunks.  First item of the range
// starting at `item` (< total):
__device__ __forceinline__ void ecur_init(const SgmvParams& p, int item, ECur& e) {
  const int PS = p.e_pair;
  const int s = find_ge(p.plan.expand_prefix, p.S, item);
  int q = item - p.plan.expand_prefix[s];
  int NC = 0;
  for (int k = 0; k < p.n_slots; ++k) NC += cdiv_d(p.slot[k].d_out, kEN);
  e.s = s;
  e.mt = seg_tiles(p, s);
  const int full = e.mt / PS;  // complete groups
  if (q < full * PS * NC) {
    e.g = q / (PS * NC);
    q -= e.g * PS * NC;
    e.nm = PS;
  } else {
    e.g = full;
    q -= full * PS * NC;
    e.nm = e.mt - full * PS;
  }
  const int nm = max(e.nm, 1);
  int kc = q / nm;
  e.i = q - kc * nm;
  int k = 0;
  for (; k < p.n_slots - 1; ++k) {
    const int n = cdiv_d(p.slot[k].d_out, kEN);
    if (kc < n) break;
    kc -= n;
  }
  e.k = k;
  e.nch = cdiv_d(p.slot[k].d_out, kEN);
  e.c = kc;
  e.valid = e.nm > 0 && e.c < e.nch;
}

// Advances to the next item; returns 0 (same B chunk), 1 (new chunk, same
// t rows) or 2 (new t rows: another slot or tile group).
__device__ __forceinline__ int ecur_next(const SgmvParams& p, ECur& e) {
  if (++e.i < e.nm) return 0;
  e.i = 0;
  if (++e.c < e.nch) return 1;
  e.c = 0;
  if (++e.k < p.n_slots) {
    e.nch = cdiv_d(p.slot[e.k].d_out, kEN);
    return 2;
  }
  e.k = 0;
  e.nch = cdiv_d(p.slot[0].d_out, kEN);
  const int PS = p.e_pair;
  if ((++e.g) * PS < e.mt) {
    e.nm = min(PS, e.mt - e.g * PS);
    return 2;
  }
  e.g = 0;
  do {
    ++e.s;
  } while (e.s < p.S && seg_tiles(p, e.s) == 0);
  e.valid = e.s < p.S;
  if (e.valid) {
    e.mt = seg_tiles(p, e.s);
    e.nm = min(PS, e.mt);
  }
  return 2;
}

template <int DT>
__global__ void __launch_bounds__(kExpandThreads, 1) k_sgmv_expand(const __grid_constant__ SgmvParams p) {
  extern __shared__ __align__(1024) unsigned char dsm[];
  __shared__ __align__(8) uint64_t b_full[4], b_empty[4], y_full[4], y_empty[4], a_full[kAcc], a_empty[kAcc];
  __shared__ __align__(8) uint64_t t_full, fin, e_sync;
  __shared__ uint32_t tmem_slot;
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NB = p.e_nb, NY = p.e_ny, PS = p.e_pair;
  const int t_half = p.e_t_half;   // bytes of one t half (hi or lo)
  const int b_stage = p.e_b_stage;
  unsigned char* tbuf = smem;      // PS tiles of (hi, lo)
  unsigned char* bring = smem + PS * 2 * t_half;
  unsigned char* yring = bring + NB * b_stage;

  if (tid == 0) {
    for (int i = 0; i < NB; ++i) {
      bar_init(&b_full[i], 1);
      bar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < NY; ++i) {
      bar_init(&y_full[i], 1);
      bar_init(&y_empty[i], kEpiWarps);
    }
    for (int i = 0; i < kAcc; ++i) {
      bar_init(&a_full[i], 1);
      bar_init(&a_empty[i], kEpiWarps);
    }
    bar_init(&t_full, kEpiWarps);
    bar_init(&fin, 1);
    bar_init(&e_sync, kEpiWarps);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(&tmem_slot, kAcc * kEN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  gd_wait();
  const int total = p.plan.meta[1];
  const int G = gridDim.x;
  const int i0 = (int)(((int64_t)blockIdx.x * total) / G);
  const int i1 = (int)(((int64_t)(blockIdx.x + 1) * total) / G);
  const int n_items = i1 - i0;
  bool ok = true;

  if (n_items > 0 && warp == 0) {
    // ---------------- producer: a B chunk per run of items (gather4 from the
    // pages, MN-major atoms of 8 ranks x 64 outputs), a y tile per item (two
    // tiled TMA boxes)
    ECur e;
    ecur_init(p, i0, e);
    int issued = 0, runs = 0, code = 2;
    const uint64_t pol_y = policy_evict_first(), pol_b = policy_evict_last();
    for (int j = 0; j < n_items && ok; ++j) {
      if (!e.valid) {
        if (lane == 0) rec_err(p.pool.err, 7, i0 + j);
        ok = false;
        break;
      }
      const SlotDev& L = p.slot[e.k];
      const int n0 = e.c * kEN;
      if (code > 0) {  // a new B chunk
        const int a = p.plan.seg_adapter[e.s], r = p.plan.seg_rank[e.s];
        const int r16 = (r + 15) & ~15;
        int rr[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int g = lane + 32 * i, kq = g >> 1, cn = g & 1;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int kr = 4 * kq + u, col = n0 + cn * 64;
            rr[i][u] = (g < r16 / 2 && kr < r && col < L.d_out)
                           ? pool_row(p.pool, a, L.listB, (int64_t)kr * L.d_out + col)
                           : (int)p.pool_rows;
          }
        }
        const int bs = runs % NB;
        if (runs >= NB) ok = bar_wait(&b_empty[bs], ((runs / NB) - 1) & 1, p.pool.err);
        if (!ok) break;
        unsigned char* bt = bring + bs * b_stage;
        if (lane == 0) bar_expect(&b_full[bs], (uint32_t)r16 * (kEN * 2));
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int g = lane + 32 * i, kq = g >> 1, cn = g & 1;
          if (g < r16 / 2)
            tma_gather4_hint(bt + ((4 * kq) >> 3) * 2048 + cn * 1024 + ((4 * kq) & 7) * 128, &p.poolmap, rr[i][0],
                             rr[i][1], rr[i][2], rr[i][3], &b_full[bs], pol_b);
        }
        ++runs;
      }
      const int ys = j % NY;
      if (j >= NY) ok = bar_wait(&y_empty[ys], ((j / NY) - 1) & 1, p.pool.err);
      if (!ok) break;
      if (lane == 0) {
        unsigned char* yt = yring + ys * kYTileBytes;
        const int row0 = p.plan.seg_start[e.s] + (e.g * PS + e.i) * kBM;
        const bool two = n0 + 64 < L.d_out;  // no box lies wholly past d_out
        bar_expect(&y_full[ys], (uint32_t)(two ? kYTileBytes : kYTileBytes / 2));
        tma_tile_2d_hint(yt, &p.ymap[e.k], n0, row0, &y_full[ys], pol_y);
        if (two) tma_tile_2d_hint(yt + kYTileBytes / 2, &p.ymap[e.k], n0 + 64, row0, &y_full[ys], pol_y);
      }
      __syncwarp();
      ++issued;
      code = ecur_next(p, e);
    }
    // every copy issued must land before the CTA may exit (the last phase of
    // each ring stage is not re-armed, so these waits see their own copies)
    if (lane == 0) {
      for (int j = max(0, runs - NB); j < runs; ++j) bar_wait(&b_full[j % NB], (j / NB) & 1, p.pool.err);
      for (int j = max(0, issued - NY); j < issued; ++j) bar_wait(&y_full[j % NY], (j / NY) & 1, p.pool.err);
    }
  } else if (n_items > 0 && warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      ECur e;
      ecur_init(p, i0, e);
      int unit = 0, runs = 0, bs = 0, code = 2;  // bs: B slot of the current run
      const uint32_t id = idesc_f16(p.dtype, kEN, 1);
      for (int j = 0; j < n_items && ok; ++j) {
        if (!e.valid) break;
        const int r16 = (p.plan.seg_rank[e.s] + 15) & ~15;
        const int as = j % kAcc;
        if (code == 2) {  // new t rows
          ok = bar_wait(&t_full, unit & 1, p.pool.err);
          ++unit;
        }
        if (ok && code > 0) {  // new B chunk
          bs = runs % NB;
          ok = bar_wait(&b_full[bs], (runs / NB) & 1, p.pool.err);
          ++runs;
        }
        if (ok && j >= kAcc) ok = bar_wait(&a_empty[as], ((j / kAcc) - 1) & 1, p.pool.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sb = su32(bring + bs * b_stage);
        const uint32_t sh = su32(tbuf + e.i * 2 * t_half), sl = sh + t_half;
        const uint32_t acc = tmem + as * kEN;
        for (int q = 0; q < r16 / 16; ++q)
          mma_f16(acc, sdesc(sh + (q >> 2) * (kBM * 128) + (q & 3) * 32, 16, 1024), sdesc(sb + q * 4096, 1024, 2048),
                  id, q > 0 ? 1u : 0u);
        for (int q = 0; q < r16 / 16; ++q)
          mma_f16(acc, sdesc(sl + (q >> 2) * (kBM * 128) + (q & 3) * 32, 16, 1024), sdesc(sb + q * 4096, 1024, 2048),
                  id, 1u);
        mma_commit(&a_full[as]);
        code = ecur_next(p, e);
        if (code > 0 || j == n_items - 1) mma_commit(&b_empty[bs]);  // the run's last item
      }
      // all MMAs complete before TMEM is released
      mma_commit(&fin);
      bar_wait(&fin, 0, p.pool.err);
    }
    __syncwarp();
  } else if (n_items > 0) {
    // ---------------- epilogue warps 2..9: TMEM lanes 32 * (warp % 4), output
    // columns [64 half, 64 half + 64) of the item with half = (warp - 2) / 4
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int mrow = quarter * 32 + lane;
    const int etid = tid - 64;  // 0 .. 32 * kEpiWarps - 1
    const uint64_t pol_y = policy_evict_first();
    ECur e;
    ecur_init(p, i0, e);
    int code = 2;
    for (int j = 0; j < n_items && ok; ++j) {
      if (!e.valid) break;
      const SlotDev& L = p.slot[e.k];
      const int s = e.s;
      const int a = p.plan.seg_adapter[s], r = p.plan.seg_rank[s];
      const int r16 = (r + 15) & ~15;
      const int seg1 = p.plan.seg_end[s];
      const int row0 = p.plan.seg_start[s] + (e.g * PS + e.i) * kBM;
      const bool valid = row0 + mrow < seg1;
      const int n0 = e.c * kEN;
      // new unit: the t rows of slot k for each tile of the group, as hi / lo
      // halves, K-major 128-byte swizzle (tile i into t buffer i).  The previous
      // unit's MMAs are complete: this thread waited on the accumulator of its
      // last item, committed after them.
      for (int ti = 0; ti < (code == 2 ? e.nm : 0); ++ti) {
        unsigned char* t_hi = tbuf + ti * 2 * t_half;
        unsigned char* t_lo = t_hi + t_half;
        const int token = p.plan.seg_start[s] + (e.g * PS + ti) * kBM + mrow;
        const bool tvalid = token < seg1;
        const float* trow = p.t + (int64_t)e.k * p.t_slot_stride + (int64_t)token * p.t_ld;
        for (int k0 = half * 8; k0 < r16; k0 += 16) {
          float v[8];
          if (tvalid) {
            const float4 f0 = *reinterpret_cast<const float4*>(trow + k0);
            const float4 f1 = *reinterpret_cast<const float4*>(trow + k0 + 4);
            v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w;
            v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (k0 + q >= r) v[q] = 0.f;
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = 0.f;
          }
          uint4 h, l;
          split2<DT>(v[0], v[1], h.x, l.x);
          split2<DT>(v[2], v[3], h.y, l.y);
          split2<DT>(v[4], v[5], h.z, l.z);
          split2<DT>(v[6], v[7], h.w, l.w);
          const int off = (k0 >> 6) * (kBM * 128) + (mrow >> 3) * 1024 + (mrow & 7) * 128 +
                          ((((k0 & 63) >> 3) ^ (mrow & 7)) << 4);
          *reinterpret_cast<uint4*>(t_hi + off) = h;
          *reinterpret_cast<uint4*>(t_lo + off) = l;
        }
      }
      if (code == 2) {
        fence_async_smem();
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&t_full)) : "memory");
      }
      const int as = j % kAcc, ys = j % NY;
      ok = bar_wait(&a_full[as], (j / kAcc) & 1, p.pool.err);
      if (ok) ok = bar_wait(&y_full[ys], (j / NY) & 1, p.pool.err);
      if (!ok) break;
      tc_fence_after();
      const float s_a = __ldg(p.pool.scale + a);
      unsigned char* yt = yring + ys * kYTileBytes;
#pragma unroll
      for (int c4 = 0; c4 < kEN / 32; ++c4) {
        const int cc = half * (kEN / 32) + c4;  // 16-column group of this warp
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + as * kEN + cc * 16, v);
        if (!valid) continue;
        // 16 outputs = chunks ch, ch + 1 (8 outputs each) of box cc / 4
        unsigned char* rowp = yt + (cc >> 2) * (kYTileBytes / 2) + mrow * 128;
        const int ch = (cc & 3) * 2;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4* pp = reinterpret_cast<uint4*>(rowp + (((ch + h) ^ (mrow & 7)) << 4));
          const uint4 yv = *pp;
          const uint32_t w[4] = {yv.x, yv.y, yv.z, yv.w};
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float y0, y1;
            up2<DT>(w[q], y0, y1);
            o[q] = pk2<DT>(fmaf(s_a, __uint_as_float(v[h * 8 + 2 * q]), y0),
                           fmaf(s_a, __uint_as_float(v[h * 8 + 2 * q + 1]), y1));
          }
          *pp = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      tc_fence_before();
      fence_async_smem();  // the tile's new y values, for a TMA store
      __syncwarp();
      if (lane == 0) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&a_empty[as])) : "memory");
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&e_sync)) : "memory");
      }
      // the tile in shared memory is complete once all four warps arrived
      // (a bounded wait, unlike a named barrier, so a warp that gave up
      // cannot hang the others)
      ok = bar_wait(&e_sync, j & 1, p.pool.err);
      if (!ok) break;
      if (row0 + kBM <= seg1) {
        // the whole tile belongs to the segment: one TMA store per box (clipped
        // at d_out); the slot is released once the copy has read it
        if (etid == 0) {
          tma_store_2d_hint(&p.ymap[e.k], n0, row0, yt, pol_y);
          if (n0 + 64 < L.d_out) tma_store_2d_hint(&p.ymap[e.k], n0 + 64, row0, yt + kYTileBytes / 2, pol_y);
          bulk_commit();
          bulk_wait_read();
        }
      } else {
        // the segment ends inside the tile (its other rows are another
        // segment's): coalesced stores of this segment's rows, thread ->
        // (row it * R + etid / 16, 16-byte chunk etid % 16)
        constexpr int kRowsPerIt = 32 * kEpiWarps / 16;
        const int q16 = etid & 15, cb = q16 >> 3, cj = q16 & 7;
        const int col = n0 + q16 * 8;
#pragma unroll 4
        for (int it = 0; it < kBM / kRowsPerIt; ++it) {
          const int row = it * kRowsPerIt + (etid >> 4);
          const int tok = row0 + row;
          if (tok < seg1 && col < L.d_out) {
            const uint4 v = *reinterpret_cast<const uint4*>(yt + cb * (kYTileBytes / 2) + row * 128 +
                                                            ((cj ^ (row & 7)) << 4));
            st_global_v4_hint(L.y + (int64_t)tok * L.ldy + col, v, pol_y);
          }
        }
      }
      fence_async_smem();  // generic-proxy writes of the slot before the next TMA fill
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&y_empty[ys])) : "memory");
      code = ecur_next(p, e);
    }
  }
  if (tid == 64) bulk_wait_all();  // the epilogue's TMA stores are complete
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kAcc * kEN);
  gd_launch();
}

// ---------------------------------------------------------------------------
// Host side.
int round16(int v) { return (v + 15) & ~15; }

template <typename Kern>
cudaError_t launch_pdl(Kern kernel, int grid, int block, size_t smem, cudaStream_t s, const SgmvParams& p) {
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

}  // namespace

// Scratch of the prefill path inside dev_scratch: segment plan + t for up to
// kMaxSlots projection slots of max_tokens rows x round16(max_rank) floats.
size_t sgmv_scratch_bytes(const slora_pool_desc& d) {
  const size_t T = (size_t)d.max_tokens;
  const size_t plan = 4 * (6 * (T + 2) + 16);
  const size_t t = 4 * (size_t)kMaxSlots * T * (size_t)std::max(16, round16(d.max_rank));
  return ((plan + 255) / 256) * 256 + t + 256;
}

static SgmvParams g_sgmv;  // host staging of the (large) parameter block

cudaError_t launch_sgmv(const BgmvParams& bp, int dtype, const int32_t* seg_start, const int32_t* seg_adapter,
                        int S, int T, int sm_count, cudaStream_t st, void* scratch, int max_tokens,
                        int64_t n_pages, cudaEvent_t const* ev, int n_ev) {
  SgmvParams& p = g_sgmv;
  memset(&p, 0, sizeof(p));
  p.pool = bp.pool;
  p.dtype = dtype;
  p.S = S;
  p.T = T;
  p.user_seg_start = seg_start;
  p.user_seg_adapter = seg_adapter;
  p.n_slots = bp.n_slots;
  for (int k = 0; k < bp.n_slots; ++k) p.slot[k] = bp.slot[k];
  // groups: slots sharing x, at most 512 / round16(max_rank) per group (TMEM columns)
  const int r16max = std::max(16, round16(bp.pool.max_rank));
  const int per_group = std::max(1, 512 / r16max);
  p.n_groups = 0;
  for (int g = 0; g < bp.n_groups; ++g) {
    const GroupDev& G = bp.group[g];
    for (int i = 0; i < G.n; i += per_group) {
      GroupDev& H = p.group[p.n_groups++];
      H = G;
      H.n = std::min(per_group, G.n - i);
      for (int j = 0; j < H.n; ++j) H.slot[j] = G.slot[i + j];
    }
  }
  if (p.n_groups > kMaxSlots) return cudaErrorNotSupported;
  int ntot = 16;
  for (int g = 0; g < p.n_groups; ++g) ntot = std::max(ntot, round16(p.group[g].n * bp.pool.max_rank));
  if (ntot > 512) return cudaErrorNotSupported;
  p.ntot_max = ntot;
  p.s_mq = 2 * ntot <= 512 ? 2 : 1;  // two accumulators of NT columns fit in TMEM
  {  // shrink group order: descending bytes per item (X tiles + A rows over d_in)
    int ord[kMaxSlots];
    for (int g = 0; g < p.n_groups; ++g) ord[g] = g;
    auto cost = [&](int g) {
      return (int64_t)p.group[g].d_in * (p.s_mq * kBM + p.group[g].n * bp.pool.max_rank);
    };
    std::stable_sort(ord, ord + p.n_groups, [&](int x, int y) { return cost(x) > cost(y); });
    for (int g = 0; g < p.n_groups; ++g) p.s_gorder[g] = ord[g];
  }
  const int stage_bytes = p.s_mq * kXTileBytes + ((ntot * 128 + 1023) & ~1023);
  p.stages = std::min(8, (225 * 1024) / stage_bytes);
  if (p.stages < 2) return cudaErrorNotSupported;
  // tensor maps
  const int64_t pool_rows = n_pages * ((int64_t)1 << bp.pool.page_shift) / 64;
  if (pool_rows <= 0 || pool_rows >= INT32_MAX) return cudaErrorNotSupported;
  p.pool_rows = pool_rows;
  if (!encode_2d(&p.poolmap, dtype, bp.pool.pool, 64, (uint64_t)pool_rows, 128, 64, 1)) return cudaErrorNotSupported;
  for (int g = 0; g < p.n_groups; ++g) {
    const GroupDev& G = p.group[g];
    if (!encode_2d(&p.xmap[g], dtype, G.x, (uint64_t)G.d_in, (uint64_t)T, (uint64_t)G.ldx * 2, kBK, kBM))
      return cudaErrorNotSupported;
  }
  // scratch: plan arrays then t
  int32_t* pl = static_cast<int32_t*>(scratch);
  const int Tm = max_tokens;
  p.plan.seg_start = pl;
  p.plan.seg_end = pl + (Tm + 2);
  p.plan.seg_adapter = pl + 2 * (Tm + 2);
  p.plan.seg_rank = pl + 3 * (Tm + 2);
  p.plan.shrink_prefix = pl + 4 * (Tm + 2);
  p.plan.expand_prefix = pl + 5 * (Tm + 2);
  p.plan.meta = pl + 6 * (Tm + 2);
  const size_t plan_bytes = ((4 * (6 * ((size_t)Tm + 2) + 16) + 255) / 256) * 256;
  p.t = reinterpret_cast<float*>(static_cast<char*>(scratch) + plan_bytes);
  p.t_ld = r16max;
  p.t_slot_stride = (int64_t)Tm * r16max;
  if (S > Tm) return cudaErrorNotSupported;

  for (int k = 0; k < p.n_slots; ++k) {
    const SlotDev& L = p.slot[k];
    if (!encode_2d(&p.ymap[k], dtype, L.y, (uint64_t)L.d_out, (uint64_t)T, (uint64_t)L.ldy * 2, 64, kBM))
      return cudaErrorNotSupported;
  }
  // expand shared memory: t hi + lo, NB B stages, NY y tiles (deepest rings that fit)
  p.e_t_half = ((r16max + 63) / 64) * (kBM * 128);
  p.e_b_stage = r16max * (kEN * 2);
  // the largest tile group that fits (one B gather serves the group's tiles;
  // measured: 4 tiles with 2 y stages beat 2 tiles with 4), then the deepest
  // y ring that fits
  const size_t smem_cap = 227 * 1024 - 1024;  // dynamic budget minus static barriers
  auto esmem = [&] {
    return (size_t)p.e_pair * 2 * p.e_t_half + (size_t)p.e_nb * p.e_b_stage + (size_t)p.e_ny * kYTileBytes + 1024;
  };
  bool fits = false;
  for (int pair = 4; pair >= 1 && !fits; pair >>= 1)
    for (int ny = 4; ny >= 2 && !fits; --ny) {
      p.e_pair = pair;
      p.e_nb = 2;
      p.e_ny = ny;
      fits = esmem() <= smem_cap;
    }
  if (esmem() > smem_cap) return cudaErrorNotSupported;
  const size_t shrink_smem = (size_t)p.stages * stage_bytes + 1024;
  const size_t expand_smem = esmem();
  cudaError_t ea = cudaFuncSetAttribute(k_sgmv_shrink, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shrink_smem);
  if (ea == cudaSuccess)
    ea = cudaFuncSetAttribute(dtype == SLORA_BF16 ? k_sgmv_expand<SLORA_BF16> : k_sgmv_expand<SLORA_F16>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)expand_smem);
  if (ea != cudaSuccess) return ea;
  const int tiles = (T + kBM - 1) / kBM + S;  // upper bound on 128-token tiles over all segments
  // timing hook: n_ev == 2 brackets the call, n_ev >= 4 also splits it per kernel
  if (n_ev >= 2) cudaEventRecord(ev[0], st);
  k_sgmv_plan<<<1, 1024, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (n_ev >= 4) cudaEventRecord(ev[1], st);
  const int items_ub = (tiles + p.s_mq - 1) / p.s_mq + S;  // >= sum over segments of ceil(tiles / s_mq)
  e = launch_pdl(k_sgmv_shrink, p.n_groups * items_ub, kShrinkThreads, shrink_smem, st, p);
  if (e != cudaSuccess) return e;
  if (n_ev >= 4) cudaEventRecord(ev[2], st);
  // persistent expand: one CTA per SM, each a contiguous range of items
  if (dtype == SLORA_BF16) e = launch_pdl(k_sgmv_expand<SLORA_BF16>, sm_count, kExpandThreads, expand_smem, st, p);
  else e = launch_pdl(k_sgmv_expand<SLORA_F16>, sm_count, kExpandThreads, expand_smem, st, p);
  if (e != cudaSuccess) return e;
  if (n_ev >= 4) cudaEventRecord(ev[3], st);
  else if (n_ev == 2) cudaEventRecord(ev[1], st);
  return cudaSuccess;
}

}  // namespace slora
