// linear.cu -- the prefill linear layer with its LoRA delta in one tcgen05
// kernel (sm_100a):
//
//     Y[i, :] = X[i, :] . W0 + (alpha_a / r_a) . (X[i, :] . A_a) . B_a
//
// for every token i of a segment (request) whose adapter is a, and
// Y[i, :] = X[i, :] . W0 for a segment without one: the scaled form of
// "Multi-LoRA serving: S-LoRA, Punica, SGMV, vLLM" (SGMV section), with the
// delta fused into the linear layer's own output as its metrics section puts
// it, instead of a second pass over X and Y.
//
// A work unit is (128-token tile of one segment, projection, group of up to 8
// output chunks of 128 columns).  For each chunk the K loop streams 64-wide
// blocks of the X tile and of W0 (tiled TMA, 128-byte swizzle) and accumulates
// X . W0 into one of two 128-column TMEM accumulators.  On a unit's first
// chunk the same X blocks also meet the adapter's A rows (copied from their
// pages by four loader warps with cp.async into the K-major swizzled layout):
// t = X . A accumulates into a third TMEM region in the same K loop, so the
// shrink costs no extra pass over X.  The epilogue warps turn t into two
// 16-bit halves (t = hi + lo, hi = RN(s . t), lo = RN(s . t - hi)) in shared
// memory once per unit; after each chunk's K loop the MMA warp adds
// t_hi . B + t_lo . B (B's 128-column chunk gathered from the pages with TMA
// gather4 into MN-major atoms) to the chunk's accumulator.  The epilogue warps
// then store the accumulator's rows that lie inside the segment.
// Warps: 0 TMA producer, 1 MMA issuer, 2..5 A loaders, 6..9 epilogue.
// Adapter ranks up to 64 (round16(r) <= 64: t fits one 64-wide K atom).
#include <algorithm>
#include <cstring>

#include "tc_common.cuh"

namespace slora {

namespace {

using namespace tc;

constexpr int kLK = 64;                        // K per stage (one 128-byte swizzle atom)
constexpr int kLN = 128;                       // output columns per chunk (MMA N)
constexpr int kLXBytes = kBM * kLK * 2;        // X block
constexpr int kLWBytes = kLN * kLK * 2;        // W0 block
constexpr int kLRmax = 64;                     // largest round16(rank)
constexpr int kLABytes = kLRmax * 128;         // A rows of a stage
constexpr int kLStage = kLXBytes + kLWBytes + kLABytes;
constexpr int kLTHalf = kBM * 128;             // t hi or lo: 128 rows x one K atom
constexpr int kLBBytes = kLRmax * kLN * 2;     // B chunk (<= 64 ranks x 128 columns)
constexpr int kLThreads = 320;
constexpr int kLCG = 8;                        // chunks per unit
constexpr int kLMaxSG = 256;                   // (projection, chunk group) pairs
constexpr int kLMaxStages = 4;
constexpr int kLTmemCols = 512;                // two 128-column accumulators + t
constexpr int kLTCol = 2 * kLN;                // TMEM column of t

struct LinParams {
  CUtensorMap xmap[kMaxSlots];   // per slot: X as (d_in, T), 64 x 128 boxes
  CUtensorMap wmap[kMaxSlots];   // per slot: W0 as (d_in, d_out) (rows = output features), 64 x 128 boxes
  CUtensorMap poolmap;           // the pool as rows of 64 elements (gather4 of B rows)
  PoolDev pool;
  int n_slots;
  SlotDev slot[kMaxSlots];
  const int32_t* seg_start;      // [S + 1], covering [0, T)
  const int32_t* seg_adapter;    // [S]
  int S, T;
  int32_t* tile_prefix;          // [S + 1] scratch: 128-token tiles before each segment
  int32_t* seg_rank;             // [S] scratch: rank applied (0: base only)
  int32_t* meta;                 // [0]: tiles
  int n_sg;
  int16_t sg_slot[kLMaxSG], sg_c0[kLMaxSG], sg_nc[kLMaxSG];
  int stages;
  int dtype;
  int64_t pool_rows;
};

struct LUnit {
  int row0, seg_end, a, r, k, c0, nc;
};

// Units run in groups of kLGroup token tiles x every (projection, chunk group):
// the CTAs of one wave then share a few x tiles and W0 chunk groups, which
// stay in L2 while each unit re-reads its x tile once per chunk.
constexpr int kLGroup = 32;
__device__ __forceinline__ void lunit(const LinParams& p, int n_tiles, int u, LUnit& U) {
  const int g = u / (kLGroup * p.n_sg), base = g * kLGroup;
  const int gm = min(kLGroup, n_tiles - base), i = u - base * p.n_sg;
  const int tile = base + i % gm, sgi = i / gm;
  const int s = find_ge(p.tile_prefix, p.S, tile);
  U.row0 = p.seg_start[s] + (tile - p.tile_prefix[s]) * kBM;
  U.seg_end = p.seg_start[s + 1];
  U.r = p.seg_rank[s];
  U.a = U.r > 0 ? p.seg_adapter[s] : -1;
  U.k = p.sg_slot[sgi];
  U.c0 = p.sg_c0[sgi];
  U.nc = p.sg_nc[sgi];
}

// Plan (one CTA): segments must cover [0, T) in order; their 128-token tiles
// are counted and prefix-summed; an adapter that is out of range or not
// resident is recorded (codes 1, 2; info = segment) and its segment gets the
// base map only; a segment outside [0, T) or out of order (code 6) gets no
// tiles.
__global__ void __launch_bounds__(1024) k_linear_plan(const __grid_constant__ LinParams p) {
  __shared__ int sh[32];
  gd_launch();
  const int S = p.S, tid = threadIdx.x, nth = blockDim.x;
  const int E = (S + nth - 1) / nth;
  const int s0 = min(tid * E, S), s1 = min(s0 + E, S);
  int cnt = 0;
  for (int s = s0; s < s1; ++s) {
    const int b0 = p.seg_start[s], b1 = p.seg_start[s + 1];
    const bool inb = b0 >= 0 && b1 <= p.T && b1 >= b0 && (s > 0 || b0 == 0) && (s < S - 1 || b1 == p.T);
    if (!inb) rec_err(p.pool.err, 6, s);
    else cnt += cdiv_d(b1 - b0, kBM);
  }
  const int lane = tid & 31, w = tid >> 5, nw = nth >> 5;
  int x = cnt;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[w] = x;
  __syncthreads();
  if (w == 0) {
    int v = lane < nw ? sh[lane] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    sh[lane] = v;
  }
  __syncthreads();
  int base = (w ? sh[w - 1] : 0) + x - cnt;
  for (int s = s0; s < s1; ++s) {
    const int b0 = p.seg_start[s], b1 = p.seg_start[s + 1];
    const bool inb = b0 >= 0 && b1 <= p.T && b1 >= b0 && (s > 0 || b0 == 0) && (s < S - 1 || b1 == p.T);
    const int a = p.seg_adapter[s];
    int r = 0;
    if (inb && a >= 0) {
      if (a >= p.pool.max_adapters) rec_err(p.pool.err, 1, s);
      else if (p.pool.rank[a] < 0) rec_err(p.pool.err, 2, s);
      else r = p.pool.rank[a];
    }
    p.tile_prefix[s] = base;
    p.seg_rank[s] = r;
    base += inb ? cdiv_d(b1 - b0, kBM) : 0;
  }
  if (tid == nth - 1) {
    p.tile_prefix[S] = base;
    p.meta[0] = base;
  }
}

template <int DT>
__global__ void __launch_bounds__(kLThreads, 1) k_linear(const __grid_constant__ LinParams p) {
  extern __shared__ __align__(1024) unsigned char dsm[];
  __shared__ __align__(8) uint64_t full[kLMaxStages], empty[kLMaxStages], fullA[kLMaxStages];
  __shared__ __align__(8) uint64_t t_full, t_ready, b_full[2], b_empty[2], acc_full[2], acc_empty[2], fin;
  __shared__ uint32_t tmem_slot;
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ST = p.stages;
  unsigned char* tbuf = smem + ST * kLStage;   // t hi, then t lo
  unsigned char* bbuf = tbuf + 2 * kLTHalf;    // two B chunks
  if (tid == 0) {
    for (int i = 0; i < ST; ++i) {
      bar_init(&full[i], 1);
      bar_init(&empty[i], 1);
      bar_init(&fullA[i], 128);
    }
    bar_init(&t_full, 1);
    bar_init(&t_ready, 128);
    for (int i = 0; i < 2; ++i) {
      bar_init(&b_full[i], 1);
      bar_init(&b_empty[i], 1);
      bar_init(&acc_full[i], 1);
      bar_init(&acc_empty[i], 128);
    }
    bar_init(&fin, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(&tmem_slot, kLTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  gd_wait();
  const int n_tiles = p.meta[0];
  const int n_units = n_tiles * p.n_sg;
  int32_t* err = p.pool.err;
  bool ok = true;

  if (warp == 0) {
    // ---- producer: B chunks (gather4 from the pages), X and W0 blocks (TMA)
    const uint64_t pol_keep = policy_evict_last();
    int gs = 0, nb = 0;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      LUnit U;
      lunit(p, n_tiles, u, U);
      const SlotDev& L = p.slot[U.k];
      const int KB = L.d_in / kLK;
      const int r16 = (U.r + 15) & ~15;
      for (int j = 0; j < U.nc && ok; ++j) {
        const int c = U.c0 + j;
        if (U.r > 0) {  // this chunk's B rows: r16 ranks x 128 columns, MN-major atoms
          const int bb = nb & 1;
          int rr[2][4];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int g = lane + 32 * i, kq = g >> 1, cn = g & 1;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int kr = 4 * kq + v, col = c * kLN + cn * 64;
              rr[i][v] = (g < r16 / 2 && kr < U.r && col < L.d_out)
                             ? pool_row(p.pool, U.a, L.listB, (int64_t)kr * L.d_out + col)
                             : (int)p.pool_rows;
            }
          }
          if (nb >= 2) ok = bar_wait(&b_empty[bb], ((nb >> 1) - 1) & 1, err);
          if (!ok) break;
          unsigned char* bt = bbuf + bb * kLBBytes;
          if (lane == 0) bar_expect(&b_full[bb], (uint32_t)r16 * (kLN * 2));
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int g = lane + 32 * i, kq = g >> 1, cn = g & 1;
            if (g < r16 / 2)
              tma_gather4_hint(bt + ((4 * kq) >> 3) * 2048 + cn * 1024 + ((4 * kq) & 7) * 128, &p.poolmap,
                               rr[i][0], rr[i][1], rr[i][2], rr[i][3], &b_full[bb], pol_keep);
          }
          ++nb;
        }
        for (int kb = 0; kb < KB; ++kb, ++gs) {
          const int st = gs % ST;
          if (gs >= ST) ok = bar_wait(&empty[st], ((gs / ST) - 1) & 1, err);
          if (!ok) break;
          if (lane == 0) {
            unsigned char* sp = smem + st * kLStage;
            bar_expect(&full[st], kLXBytes + kLWBytes);
            tma_tile_2d_hint(sp, &p.xmap[U.k], kb * kLK, U.row0, &full[st], pol_keep);
            tma_tile_2d_hint(sp + kLXBytes, &p.wmap[U.k], kb * kLK, c * kLN, &full[st], pol_keep);
          }
          __syncwarp();
        }
      }
    }
    // every copy issued lands before the CTA may exit
    if (lane == 0) {
      for (int g = max(0, gs - ST); g < gs; ++g) bar_wait(&full[g % ST], (g / ST) & 1, err);
      for (int b = max(0, nb - 2); b < nb; ++b) bar_wait(&b_full[b & 1], (b >> 1) & 1, err);
    }
  } else if (warp == 1) {
    // ---- MMA issuer
    if (lane == 0) {
      int gs = 0, q = 0, nb = 0, nt = 0;
      uint32_t apar = 0;
      const uint32_t id_w = idesc_f16(p.dtype, kLN, 0);
      const uint32_t id_b = idesc_f16(p.dtype, kLN, 1);
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        LUnit U;
        lunit(p, n_tiles, u, U);
        const int KB = p.slot[U.k].d_in / kLK;
        const int r16 = (U.r + 15) & ~15;
        const uint32_t id_t = idesc_f16(p.dtype, r16 > 0 ? r16 : 16, 0);
        for (int j = 0; j < U.nc && ok; ++j, ++q) {
          const int ab = q & 1;
          if (q >= 2) ok = bar_wait(&acc_empty[ab], ((q >> 1) - 1) & 1, err);
          if (!ok) break;
          tc_fence_after();
          const bool withA = j == 0 && U.r > 0;
          for (int kb = 0; kb < KB; ++kb, ++gs) {
            const int st = gs % ST;
            ok = bar_wait(&full[st], (gs / ST) & 1, err);
            if (ok && withA) {
              ok = bar_wait(&fullA[st], (apar >> st) & 1, err);
              apar ^= 1u << st;
            }
            if (!ok) break;
            tc_fence_after();
            const uint32_t xs = su32(smem + st * kLStage);
            const uint32_t ws = xs + kLXBytes, as = ws + kLWBytes;
#pragma unroll
            for (int kk = 0; kk < kLK / 16; ++kk)
              mma_f16(tmem + ab * kLN, sdesc(xs + kk * 32, 16, 1024), sdesc(ws + kk * 32, 16, 1024), id_w,
                      (kb > 0 || kk > 0) ? 1u : 0u);
            if (withA) {
#pragma unroll
              for (int kk = 0; kk < kLK / 16; ++kk)
                mma_f16(tmem + kLTCol, sdesc(xs + kk * 32, 16, 1024), sdesc(as + kk * 32, 16, 1024), id_t,
                        (kb > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&empty[st]);
          }
          if (!ok) break;
          if (U.r > 0) {
            if (j == 0) {  // t complete: the epilogue warps convert it; wait for the halves
              mma_commit(&t_full);
              ok = bar_wait(&t_ready, nt & 1, err);
              ++nt;
            }
            const int bb = nb & 1;
            if (ok) ok = bar_wait(&b_full[bb], (nb >> 1) & 1, err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t th = su32(tbuf), tl = th + kLTHalf, sb = su32(bbuf + bb * kLBBytes);
            for (int qq = 0; qq < r16 / 16; ++qq)
              mma_f16(tmem + ab * kLN, sdesc(th + qq * 32, 16, 1024), sdesc(sb + qq * 4096, 1024, 2048), id_b, 1u);
            for (int qq = 0; qq < r16 / 16; ++qq)
              mma_f16(tmem + ab * kLN, sdesc(tl + qq * 32, 16, 1024), sdesc(sb + qq * 4096, 1024, 2048), id_b, 1u);
            mma_commit(&b_empty[bb]);
            ++nb;
          }
          mma_commit(&acc_full[ab]);
        }
      }
      // all MMAs complete before TMEM is released
      mma_commit(&fin);
      bar_wait(&fin, 0, err);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ---- A loaders: on a unit's first chunk, thread et copies 16-byte chunk
    // et % 8 of rows et / 8 + 16 i of each stage's A block (rows past r zero),
    // into the 128-byte-swizzled K-major layout; a stage's rows are released
    // to the MMA (fullA) two stages later, once their copy group completed.
    // The loaders wait for every stage slot in order (not only the ones they
    // fill): an mbarrier phase parity is unambiguous only while the waiter is
    // at most one phase ahead.
    const int et = tid - 64, ch = et & 7, r0 = et >> 3;
    const uint64_t pol = policy_evict_last();
    const int lag = min(2, ST - 1);
    int gs = 0;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      LUnit U;
      lunit(p, n_tiles, u, U);
      const SlotDev& L = p.slot[U.k];
      const int KB = L.d_in / kLK;
      const int r16 = (U.r + 15) & ~15;
      const int32_t* plist = p.pool.page_list + (int64_t)(U.a >= 0 ? U.a : 0) * p.pool.list_stride + L.listA;
      const int64_t pmask = (1ll << p.pool.page_shift) - 1;
      for (int j = 0; j < U.nc && ok; ++j) {
        const bool withA = j == 0 && U.r > 0;
        int kb = 0;
        for (; kb < KB && ok; ++kb) {
          const int g = gs + kb, st = g % ST;
          if (g >= ST) ok = bar_wait(&empty[st], ((g / ST) - 1) & 1, err);
          if (!ok || !withA) continue;
          const uint32_t as = su32(smem + st * kLStage + kLXBytes + kLWBytes);
          for (int rho = r0; rho < r16; rho += 16) {
            const uint32_t dst = as + rho * 128 + ((ch ^ (rho & 7)) << 4);
            if (rho < U.r) {
              const int64_t f = (int64_t)rho * L.d_in + (int64_t)kb * kLK + ch * 8;
              const int32_t pg = __ldg(plist + (f >> p.pool.page_shift));
              const uint16_t* src = p.pool.pool + ((int64_t)pg << p.pool.page_shift) + (f & pmask);
              asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, 16, %2;" ::"r"(dst), "l"(src),
                           "l"(pol)
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
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&fullA[(gs + kb - lag) % ST])) : "memory");
          }
        }
        if (withA) {
          asm volatile("cp.async.wait_group 0;" ::: "memory");
          fence_async_smem();
          for (int k2 = max(0, kb - lag); k2 < kb; ++k2)
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&fullA[(gs + k2) % ST])) : "memory");
        }
        gs += KB;
      }
    }
  } else {
    // ---- epilogue: thread = TMEM lane = tile row quarter * 32 + lane
    const int quarter = warp & 3;
    const int mrow = quarter * 32 + lane;
    int q = 0, nt = 0;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      LUnit U;
      lunit(p, n_tiles, u, U);
      const SlotDev& L = p.slot[U.k];
      const int row = U.row0 + mrow;
      const bool valid = row < U.seg_end;
      if (U.r > 0) {  // t -> s . t as 16-bit halves, K-major swizzled rows
        ok = bar_wait(&t_full, nt & 1, err);
        ++nt;
        if (!ok) break;
        tc_fence_after();
        const int r16 = (U.r + 15) & ~15;
        const float s_a = __ldg(p.pool.scale + U.a);
        unsigned char* t_hi = tbuf;
        unsigned char* t_lo = tbuf + kLTHalf;
        for (int c0 = 0; c0 < r16; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + kLTCol + c0, v);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = (c0 + 8 * h + e < U.r) ? s_a * __uint_as_float(v[8 * h + e]) : 0.f;
            uint4 hi, lo;
            split2<DT>(f[0], f[1], hi.x, lo.x);
            split2<DT>(f[2], f[3], hi.y, lo.y);
            split2<DT>(f[4], f[5], hi.z, lo.z);
            split2<DT>(f[6], f[7], hi.w, lo.w);
            const int k8 = (c0 >> 3) + h;
            const int off = (mrow >> 3) * 1024 + (mrow & 7) * 128 + ((k8 ^ (mrow & 7)) << 4);
            *reinterpret_cast<uint4*>(t_hi + off) = hi;
            *reinterpret_cast<uint4*>(t_lo + off) = lo;
          }
        }
        fence_async_smem();
        tc_fence_before();
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&t_ready)) : "memory");
      }
      for (int j = 0; j < U.nc && ok; ++j, ++q) {
        const int c = U.c0 + j, ab = q & 1;
        ok = bar_wait(&acc_full[ab], (q >> 1) & 1, err);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 2
        for (int cc = 0; cc < kLN / 16; ++cc) {
          uint32_t v[16];
          tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + ab * kLN + cc * 16, v);
          const int col = c * kLN + cc * 16;
          if (valid && col < L.d_out) {
            uint4 o0, o1;
            o0.x = pk2<DT>(__uint_as_float(v[0]), __uint_as_float(v[1]));
            o0.y = pk2<DT>(__uint_as_float(v[2]), __uint_as_float(v[3]));
            o0.z = pk2<DT>(__uint_as_float(v[4]), __uint_as_float(v[5]));
            o0.w = pk2<DT>(__uint_as_float(v[6]), __uint_as_float(v[7]));
            o1.x = pk2<DT>(__uint_as_float(v[8]), __uint_as_float(v[9]));
            o1.y = pk2<DT>(__uint_as_float(v[10]), __uint_as_float(v[11]));
            o1.z = pk2<DT>(__uint_as_float(v[12]), __uint_as_float(v[13]));
            o1.w = pk2<DT>(__uint_as_float(v[14]), __uint_as_float(v[15]));
            uint4* dst = reinterpret_cast<uint4*>(L.y + (int64_t)row * L.ldy + col);
            dst[0] = o0;
            dst[1] = o1;
          }
        }
        tc_fence_before();
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&acc_empty[ab])) : "memory");
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kLTmemCols);
  gd_launch();
}

template <typename Kern>
cudaError_t launch_pdl_l(Kern kernel, int grid, int block, size_t smem, cudaStream_t s, const LinParams& p) {
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

LinParams g_lin;  // host staging of the (large) parameter block

}  // namespace

// Scratch of the linear path: tile prefix, ranks and counters for S segments
// (S <= max_tokens), inside the SGMV part of the pool's scratch.
cudaError_t launch_linear(const BgmvParams& bp, int dtype, const void* const* w0, const int64_t* ldw,
                          const int32_t* seg_start, const int32_t* seg_adapter, int S, int T, int sm_count,
                          cudaStream_t st, void* scratch, int max_tokens, int64_t n_pages) {
  LinParams& p = g_lin;
  memset(&p, 0, sizeof(p));
  p.pool = bp.pool;
  p.dtype = dtype;
  p.S = S;
  p.T = T;
  p.seg_start = seg_start;
  p.seg_adapter = seg_adapter;
  p.n_slots = bp.n_slots;
  if (bp.pool.max_rank > kLRmax) return cudaErrorNotSupported;
  for (int k = 0; k < bp.n_slots; ++k) {
    p.slot[k] = bp.slot[k];
    const SlotDev& L = bp.slot[k];
    if (!encode_2d(&p.xmap[k], dtype, L.x, (uint64_t)L.d_in, (uint64_t)T, (uint64_t)L.ldx * 2, kLK, kBM))
      return cudaErrorNotSupported;
    if (!encode_2d(&p.wmap[k], dtype, w0[k], (uint64_t)L.d_in, (uint64_t)L.d_out, (uint64_t)ldw[k] * 2, kLK, kLN))
      return cudaErrorNotSupported;
  }
  const int64_t pool_rows = n_pages * ((int64_t)1 << bp.pool.page_shift) / 64;
  if (pool_rows <= 0 || pool_rows >= INT32_MAX) return cudaErrorNotSupported;
  p.pool_rows = pool_rows;
  if (!encode_2d(&p.poolmap, dtype, bp.pool.pool, 64, (uint64_t)pool_rows, 128, 64, 1)) return cudaErrorNotSupported;
  // (projection, chunk group) pairs, the largest d_in first
  int order[kMaxSlots];
  for (int k = 0; k < bp.n_slots; ++k) order[k] = k;
  std::stable_sort(order, order + bp.n_slots, [&](int a, int b) { return bp.slot[a].d_in > bp.slot[b].d_in; });
  p.n_sg = 0;
  for (int oi = 0; oi < bp.n_slots; ++oi) {
    const int k = order[oi];
    const int nch = (bp.slot[k].d_out + kLN - 1) / kLN;
    for (int c0 = 0; c0 < nch; c0 += kLCG) {
      if (p.n_sg >= kLMaxSG) return cudaErrorNotSupported;
      p.sg_slot[p.n_sg] = (int16_t)k;
      p.sg_c0[p.n_sg] = (int16_t)c0;
      p.sg_nc[p.n_sg] = (int16_t)std::min(kLCG, nch - c0);
      ++p.n_sg;
    }
  }
  if (S > max_tokens) return cudaErrorNotSupported;
  int32_t* pl = static_cast<int32_t*>(scratch);
  p.tile_prefix = pl;
  p.seg_rank = pl + (max_tokens + 2);
  p.meta = pl + 2 * (max_tokens + 2);
  const size_t fixed = 2 * (size_t)kLTHalf + 2 * (size_t)kLBBytes + 1024;
  const int stages = (int)std::min<size_t>(kLMaxStages, (227 * 1024 - 1024 - fixed) / kLStage);
  if (stages < 2) return cudaErrorNotSupported;
  p.stages = stages;
  const size_t smem = (size_t)stages * kLStage + fixed;
  cudaError_t e = cudaFuncSetAttribute(dtype == SLORA_BF16 ? k_linear<SLORA_BF16> : k_linear<SLORA_F16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_linear_plan<<<1, 1024, 0, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (dtype == SLORA_BF16) return launch_pdl_l(k_linear<SLORA_BF16>, sm_count, kLThreads, smem, st, p);
  return launch_pdl_l(k_linear<SLORA_F16>, sm_count, kLThreads, smem, st, p);
}

}  // namespace slora
