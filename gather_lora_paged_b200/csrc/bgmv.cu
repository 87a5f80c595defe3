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

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "slora_internal.h"

namespace slora {

#define FULL_MASK 0xffffffffu

constexpr int kWarps = 16;                // warps per CTA of shrink / expand
constexpr int kSlots = 2;                 // pipeline slots per warp
constexpr int kSlotBytes = 6 * 1024 + 128; // bytes per slot
constexpr int kSmemBytes = kWarps * kSlots * kSlotBytes;
constexpr int kExpandRows = 4;            // B rows per expand stage
constexpr int kLC = 256;                  // outputs per expand task (8 per lane)
constexpr long long kWaitLimit = 2000000000ll;  // clock cycles before a wait gives up

__host__ __device__ __forceinline__ int cdiv_i(int a, int b) { return (a + b - 1) / b; }

// Task shapes.  Shrink tasks cover NT tokens x RW rank rows x kShrinkKT of
// d_in; expand tasks NTE tokens x kLC outputs.  Slot use per stage: (RW + NT)
// KiB for shrink; 8 B rows, the t partials and y rows for expand.
__host__ __device__ __forceinline__ int nt_class(int n) { return n <= 1 ? 1 : (n == 2 ? 2 : (n <= 4 ? 4 : 8)); }
__host__ __device__ __forceinline__ int rw_of(int nt) { return nt == 1 ? 8 : 4; }
__host__ __device__ __forceinline__ int nte_class(int n) { return n <= 1 ? 1 : (n == 2 ? 2 : 4); }

__device__ __forceinline__ void record_error(int32_t* err, int code, int info) {
  if (atomicCAS(&err[0], 0, code) == 0) atomicExch(&err[1], info);
}

// ---------------------------------------------------------------------------
// PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// Bounded wait on an mbarrier phase; false (and a recorded error) if it gives up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* err) {
  const uint32_t a = smem_u32(bar);
  const long long t0 = clock64();
  for (;;) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if (clock64() - t0 > kWaitLimit) {
      record_error(err, 4, (int)blockIdx.x);
      return false;
    }
  }
}
// Bulk async copy global -> shared, completion counted on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(const unsigned char* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// 16-bit -> fp32 for 8 packed elements.
template <int DT>
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (DT == SLORA_BF16) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    } else {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      float2 g = __half22float2(h);
      f[2 * i] = g.x;
      f[2 * i + 1] = g.y;
    }
  }
}

template <int DT>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  if (DT == SLORA_BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

// Address of flat element f of tensor (adapter a, page-list offset lo).
__device__ __forceinline__ const uint16_t* page_addr(const PoolDev& P, int a, int lo, int64_t f) {
  const int32_t pg = __ldg(P.page_list + (int64_t)a * P.list_stride + lo + (f >> P.page_shift));
  return P.pool + ((int64_t)pg << P.page_shift) + (f & ((1ll << P.page_shift) - 1));
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scans (blockDim.x threads, a multiple of 32).
template <bool kMax>
__device__ int block_exscan(int v, int* total, int* sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int ident = kMax ? -1 : 0;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(FULL_MASK, x, o);
    if (lane >= o) x = kMax ? max(x, y) : x + y;
  }
  int ex = __shfl_up_sync(FULL_MASK, x, 1);
  if (lane == 0) ex = ident;
  if (lane == 31) sh[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = lane < nw ? sh[lane] : ident;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(FULL_MASK, s, o);
      if (lane >= o) s = kMax ? max(s, y) : s + y;
    }
    sh[lane] = s;
  }
  __syncthreads();
  const int wp = w ? sh[w - 1] : ident;
  const int res = kMax ? max(wp, ex) : wp + ex;
  if (total) *total = sh[nw - 1];
  __syncthreads();
  return res;
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
      shr += cdiv_i(p.group[g].n * r, rw_of(nt)) * ntg * cdiv_i(p.group[g].d_in, kShrinkKT);
  if (p.do_expand)
    for (int k = 0; k < p.n_slots; ++k) exp += nte * cdiv_i(p.slot[k].d_out, kLC);
}

__global__ void __launch_bounds__(1024) k_segments(const __grid_constant__ BgmvParams p,
                                                   const int32_t* __restrict__ idx, int T) {
  extern __shared__ int hist[];
  __shared__ int sh[32];
  const int tid = threadIdx.x, nth = blockDim.x;
  const int MA = p.pool.max_adapters;
  const ScratchDev& sc = p.sc;
  griddep_launch();  // the next kernel may start its prologue; it waits for this grid

  for (int a = tid; a < MA; a += nth) hist[a] = 0;
  __syncthreads();
  for (int i = tid; i < T; i += nth) {
    const int a = idx[i];
    if (a == -1) continue;
    if (a < -1 || a >= MA) {
      record_error(p.pool.err, 1, i);
      continue;
    }
    if (p.pool.rank[a] < 0) {
      record_error(p.pool.err, 2, i);
      continue;
    }
    atomicAdd(&hist[a], 1);
  }
  __syncthreads();

  // Each thread owns a contiguous adapter range; the segments it creates form
  // a contiguous range of segment indices.
  const int E = (MA + nth - 1) / nth;
  const int a0 = min(tid * E, MA), a1 = min(a0 + E, MA);
  int cnt = 0, nseg = 0, c_shr = 0, c_exp = 0;
  for (int a = a0; a < a1; ++a) {
    const int n = hist[a];
    if (n == 0) continue;
    int x, z;
    seg_task_counts(p, n, p.pool.rank[a], x, z);
    cnt += n;
    nseg += 1;
    c_shr += x;
    c_exp += z;
  }
  int n_valid, S, t_shr, t_exp;
  int cbase = block_exscan<false>(cnt, &n_valid, sh);
  int sb = block_exscan<false>(nseg, &S, sh);
  int b_shr = block_exscan<false>(c_shr, &t_shr, sh);
  int b_exp = block_exscan<false>(c_exp, &t_exp, sh);
  for (int a = a0; a < a1; ++a) {
    const int n = hist[a];
    hist[a] = cbase;  // becomes the scatter cursor
    if (n == 0) continue;
    const int r = p.pool.rank[a];
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
  }
  __syncthreads();

  // Stable scatter: chunks of 1024 tokens, warps take turns in order.
  const int lane = tid & 31, warp = tid >> 5;
  for (int c0 = 0; c0 < T; c0 += nth) {
    const int i = c0 + tid;
    const int a = i < T ? idx[i] : -1;
    const bool ok = a >= 0 && a < MA && p.pool.rank[a] >= 0;
    const int key = ok ? a : -1;
    const int nw = min(32, (T - c0 + 31) >> 5);
    for (int w = 0; w < nw; ++w) {
      if (warp == w) {
        const unsigned m = __match_any_sync(FULL_MASK, key);
        const int before = __popc(m & ((1u << lane) - 1));
        int cur = 0;
        if (ok) cur = hist[a];
        __syncwarp();
        if (ok) {
          sc.perm[cur + before] = i;
          if (before == 0) hist[a] = cur + __popc(m);
        }
      }
      __syncthreads();
    }
  }
}

// Largest s with prefix[s] <= q (prefix ascending from 0, S >= 1).
__device__ __forceinline__ int find_seg(const int32_t* prefix, int S, int q) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= q) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Sum over the 32 lanes of each of the N values v[0..N); afterwards lane L
// holds the total of value L % N.  N is a power of two <= 32.
template <int N>
__device__ __forceinline__ float lane_transpose_reduce(float (&v)[N]) {
#pragma unroll
  for (int o = 16; o >= N; o >>= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] += __shfl_xor_sync(FULL_MASK, v[i], o);
  }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = N / 2; o >= 1; o >>= 1) {
    const bool up = lane & o;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? v[i] : v[i + o];
      const float keep = up ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(FULL_MASK, send, o);
    }
  }
  return v[0];
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

// Page id of flat element f of tensor (adapter a, page-list offset lo).
__device__ __forceinline__ int32_t page_id(const PoolDev& P, int a, int lo, int64_t f) {
  return __ldg(P.page_list + (int64_t)a * P.list_stride + lo + (f >> P.page_shift));
}
__device__ __forceinline__ const uint16_t* page_ptr(const PoolDev& P, int32_t pg, int64_t f) {
  return P.pool + ((int64_t)pg << P.page_shift) + (f & ((1ll << P.page_shift) - 1));
}

// A paged range [f0, f0 + n) (n <= page size) is copied as piece 0 (the part
// in f0's page) and piece 1 (the rest, if the range crosses a page boundary).
// aux_page: the page id of the lane's piece, looked up one stage ahead.
__device__ __forceinline__ int32_t piece_page(const PoolDev& P, int a, int lo, int64_t f0, int n, int piece) {
  const int64_t pb = ((f0 >> P.page_shift) + 1) << P.page_shift;
  if (piece == 0) return page_id(P, a, lo, f0);
  return (f0 + n > pb) ? page_id(P, a, lo, pb) : -1;
}
__device__ __forceinline__ void piece_copy(const PoolDev& P, int32_t pg, int64_t f0, int n, int piece,
                                           unsigned char* dst, uint64_t* bar) {
  const int64_t pb = ((f0 >> P.page_shift) + 1) << P.page_shift;
  const int64_t f1 = f0 + n;
  if (piece == 0) {
    const int64_t e = f1 < pb ? f1 : pb;
    bulk_g2s(dst, page_ptr(P, pg, f0), (uint32_t)(2 * (e - f0)), bar);
  } else if (f1 > pb) {
    bulk_g2s(dst + 2 * (pb - f0), page_ptr(P, pg, pb), (uint32_t)(2 * (f1 - pb)), bar);
  }
}

// ---------------------------------------------------------------------------
// Shrink.  Task = (group g, segment, RW rank rows, NT tokens, kShrinkKT slice
// of d_in), streamed in stages of kStageK elements.  Slot layout of a stage:
// rank row i at i * 1 KiB, token row t at (RW + t) * 1 KiB.
struct STask {
  int g, a, r, seg0, n, nt, rw, rg, tg, split, nst, nrows, ntok;
};

__device__ __forceinline__ void decode_shrink(const BgmvParams& p, const SegView& V, int task, STask& t) {
  const int s = find_seg(V.prefix, V.S, task);
  int q = task - V.prefix[s];
  t.a = V.adapter[s];
  t.seg0 = V.start[s];
  t.n = V.start[s + 1] - t.seg0;
  t.r = V.rank[s];
  t.nt = nt_class(t.n);
  t.rw = rw_of(t.nt);
  const int n_tg = cdiv_i(t.n, t.nt);
  int g = 0;
  for (; g < p.n_groups - 1; ++g) {  // the group owning local task q
    const int cnt = cdiv_i(p.group[g].n * t.r, t.rw) * n_tg * cdiv_i(p.group[g].d_in, kShrinkKT);
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
  t.nst = cdiv_i(min(kShrinkKT, d_in - t.split * kShrinkKT), kStageK);
  t.nrows = min(t.rw, p.group[g].n * t.r - t.rg * t.rw);
  t.ntok = min(t.nt, t.n - t.tg * t.nt);
}

// Lane roles in a shrink stage: lane i < 16 copies piece 0 of rank row i
// (i < nrows) or token row i - nrows; lane 16 + i copies piece 1 of row i.
// The per-lane lookup (page id or token id) is done one stage ahead.
__device__ __forceinline__ int32_t shrink_lookup(const BgmvParams& p, const STask& t, int st) {
  const int lane = threadIdx.x & 31, i = lane & 15;
  const GroupDev& G = p.group[t.g];
  const int k0 = t.split * kShrinkKT + st * kStageK;
  const int L = min(kStageK, G.d_in - k0);
  if (i < t.nrows) {
    const int rho = t.rg * t.rw + i;
    const int j = rho / t.r, k = rho % t.r;
    return piece_page(p.pool, t.a, p.slot[G.slot[j]].listA, (int64_t)k * G.d_in + k0, L, lane >> 4);
  }
  if (lane < 16 && i < t.nrows + t.ntok) return __ldg(p.sc.perm + t.seg0 + t.tg * t.nt + (i - t.nrows));
  return -1;
}

__device__ __forceinline__ void issue_shrink(const BgmvParams& p, const STask& t, int st, int32_t aux,
                                             unsigned char* buf, uint64_t* bar) {
  const int lane = threadIdx.x & 31, i = lane & 15;
  const GroupDev& G = p.group[t.g];
  const int k0 = t.split * kShrinkKT + st * kStageK;
  const int L = min(kStageK, G.d_in - k0);
  if (lane == 0) mbar_expect_tx(bar, 2u * L * (t.nrows + t.ntok));
  __syncwarp();
  if (i < t.nrows) {
    const int rho = t.rg * t.rw + i;
    const int k = rho % t.r;
    piece_copy(p.pool, aux, (int64_t)k * G.d_in + k0, L, lane >> 4, buf + i * 2 * kStageK, bar);
  } else if (lane < 16 && i < t.nrows + t.ntok) {
    bulk_g2s(buf + (t.rw + i - t.nrows) * 2 * kStageK, G.x + (int64_t)aux * G.ldx + k0, 2u * L, bar);
  }
}

template <int DT, int NT, int RW>
__device__ __forceinline__ void shrink_stage(const BgmvParams& p, const STask& t, int st,
                                             const unsigned char* buf, float (&acc)[32]) {
  const int lane = threadIdx.x & 31;
  const GroupDev& G = p.group[t.g];
  const int k0 = t.split * kShrinkKT + st * kStageK;
  const int L = min(kStageK, G.d_in - k0);
#pragma unroll
  for (int e = lane * 8; e < kStageK; e += 256) {
    if (e >= L) break;
    uint4 av[RW], xv[NT];
#pragma unroll
    for (int i = 0; i < RW; ++i)
      av[i] = i < t.nrows ? lds128(buf + i * 2 * kStageK + 2 * e) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int tt = 0; tt < NT; ++tt)
      xv[tt] = tt < t.ntok ? lds128(buf + (RW + tt) * 2 * kStageK + 2 * e) : make_uint4(0, 0, 0, 0);
    if (NT <= 2) {
      float xf[NT][8];
#pragma unroll
      for (int tt = 0; tt < NT; ++tt) unpack8<DT>(xv[tt], xf[tt]);
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        float af[8];
        unpack8<DT>(av[i], af);
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) {
          float s = acc[i * NT + tt];
#pragma unroll
          for (int q = 0; q < 8; ++q) s = fmaf(af[q], xf[tt][q], s);
          acc[i * NT + tt] = s;
        }
      }
    } else {
      float af[RW][8];
#pragma unroll
      for (int i = 0; i < RW; ++i) unpack8<DT>(av[i], af[i]);
#pragma unroll
      for (int tt = 0; tt < NT; ++tt) {
        float xf[8];
        unpack8<DT>(xv[tt], xf);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          float s = acc[i * NT + tt];
#pragma unroll
          for (int q = 0; q < 8; ++q) s = fmaf(af[i][q], xf[q], s);
          acc[i * NT + tt] = s;
        }
      }
    }
  }
}

// End of a shrink task: sum over lanes and store the fp32 partial of this
// d_in slice, t[pos][k][split], for RW rows x NT tokens.
template <int NT, int RW>
__device__ __forceinline__ void shrink_finish(const BgmvParams& p, const STask& t, float (&acc)[32]) {
  constexpr int N = RW * NT;
  float v[N];
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = acc[i];
  const float val = lane_transpose_reduce<N>(v);
  const int lane = threadIdx.x & 31;
  const int Lx = lane % N;
  const int i = Lx / NT, tt = Lx % NT;
  if (lane < N && i < t.nrows && tt < t.ntok) {
    const int rho = t.rg * RW + i;
    const int j = rho / t.r, k = rho % t.r;
    const SlotDev& S = p.slot[p.group[t.g].slot[j]];
    const int pos = t.seg0 + t.tg * NT + tt;
    S.t[(int64_t)pos * S.t_rs + (int64_t)k * S.t_ns + t.split] = val;
  }
#pragma unroll
  for (int q = 0; q < 32; ++q) acc[q] = 0.f;
}

template <int DT>
__device__ __forceinline__ void shrink_stage_any(const BgmvParams& p, const STask& t, int st,
                                                 const unsigned char* buf, float (&acc)[32]) {
  const bool last = st == t.nst - 1;
  switch (t.nt) {
    case 1: shrink_stage<DT, 1, 8>(p, t, st, buf, acc); if (last) shrink_finish<1, 8>(p, t, acc); break;
    case 2: shrink_stage<DT, 2, 4>(p, t, st, buf, acc); if (last) shrink_finish<2, 4>(p, t, acc); break;
    case 4: shrink_stage<DT, 4, 4>(p, t, st, buf, acc); if (last) shrink_finish<4, 4>(p, t, acc); break;
    default: shrink_stage<DT, 8, 4>(p, t, st, buf, acc); if (last) shrink_finish<8, 4>(p, t, acc); break;
  }
}

template <int DT>
__global__ void __launch_bounds__(kWarps * 32, 1) k_shrink(const __grid_constant__ BgmvParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t bars[kWarps][kSlots];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wbuf = smem + warp * kSlots * kSlotBytes;
  int32_t* segsm = reinterpret_cast<int32_t*>(smem + kSmemBytes);
  if (lane == 0)
    for (int s = 0; s < kSlots; ++s) mbar_init(&bars[warp][s], 1);
  fence_mbar_init();
  griddep_wait();
  const int S = p.sc.meta[kMetaS];
  const int total = p.sc.meta[kMetaShrinkTotal];
  const SegView V = stage_segments(p.sc, S, true, segsm);
  const int NW = gridDim.x * kWarps;
  const int first = blockIdx.x * kWarps + warp;
  if (first >= total) {
    griddep_launch();
    return;
  }
  // Producer and consumer walk the same (task, stage) sequence; the producer
  // issues one stage ahead and looks up its page / token ids one more ahead.
  int ptask = first, pst = 0, pslot = 0;
  STask pt;
  decode_shrink(p, V, ptask, pt);
  bool pvalid = true;
  int32_t aux = shrink_lookup(p, pt, 0);
  auto produce = [&]() {
    issue_shrink(p, pt, pst, aux, wbuf + pslot * kSlotBytes, &bars[warp][pslot]);
    pslot ^= 1;
    if (++pst == pt.nst) {
      pst = 0;
      ptask += NW;
      pvalid = ptask < total;
      if (pvalid) decode_shrink(p, V, ptask, pt);
    }
    if (pvalid) aux = shrink_lookup(p, pt, pst);
  };
  int ctask = first, cst = 0, slot = 0;
  STask ct = pt;
  uint32_t parity = 0;
  float acc[32];
#pragma unroll
  for (int q = 0; q < 32; ++q) acc[q] = 0.f;
  produce();
  for (;;) {
    if (pvalid) produce();
    if (!mbar_wait(&bars[warp][slot], (parity >> slot) & 1, p.pool.err)) break;
    parity ^= 1u << slot;
    shrink_stage_any<DT>(p, ct, cst, wbuf + slot * kSlotBytes, acc);
    __syncwarp();
    fence_proxy_async();
    slot ^= 1;
    if (++cst == ct.nst) {
      cst = 0;
      ctask += NW;
      if (ctask >= total) break;
      decode_shrink(p, V, ctask, ct);
    }
  }
  griddep_launch();
}

// ---------------------------------------------------------------------------
// Expand.  Task = (projection slot k, segment, NTE tokens, kLC outputs),
// streamed in stages of kExpandRows rank rows.  Slot layout of a stage:
// B row i at i * 512 B; t partials of token t at kExpT + t * 8 * t_ns * 4 B;
// y row t (last stage) at kExpY + t * 512 B; t sums at kExpS.
constexpr int kExpT = kExpandRows * 2 * kLC;
constexpr int kExpY = 4 * 1024;
constexpr int kExpS = kExpY + 4 * 2 * kLC;
static_assert(kExpS + 4 * kExpandRows * 4 <= kSlotBytes, "expand slot overflow");

struct ETask {
  int k, a, r, seg0, n, nt, tg, lc, nst, ntok;
};

__device__ __forceinline__ void decode_expand(const BgmvParams& p, const SegView& V, int task, ETask& t) {
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
    const int cnt = n_tg * cdiv_i(p.slot[k].d_out, kLC);
    if (q < cnt) break;
    q -= cnt;
  }
  t.k = k;
  t.tg = q % n_tg;
  t.lc = q / n_tg;
  t.nst = cdiv_i(t.r, kExpandRows);
  t.ntok = min(t.nt, t.n - t.tg * t.nt);
}

// Lane roles in an expand stage: lanes 0-7 copy piece 0 of B rows 0-7,
// lanes 8-15 piece 1; lanes 16-19 the t partials of tokens 0-3; lanes 20-23
// the y rows (last stage).  The lookup (page id / token id) is done a stage ahead.
__device__ __forceinline__ int32_t expand_lookup(const BgmvParams& p, const ETask& t, int st) {
  const int lane = threadIdx.x & 31;
  const SlotDev& L = p.slot[t.k];
  const int l0 = t.lc * kLC;
  const int Lo = min(kLC, L.d_out - l0);
  const int r0 = st * kExpandRows;
  const int nrows = min(kExpandRows, t.r - r0);
  if (lane < 16) {
    const int i = lane & 7;
    if (i >= nrows) return -1;
    return piece_page(p.pool, t.a, L.listB, (int64_t)(r0 + i) * L.d_out + l0, Lo, lane >> 3);
  }
  const int tt = (lane - 16) & 3;
  if (lane < 24 && tt < t.ntok) return __ldg(p.sc.perm + t.seg0 + t.tg * t.nt + tt);
  return -1;
}

__device__ __forceinline__ void issue_expand(const BgmvParams& p, const ETask& t, int st, int32_t aux,
                                             unsigned char* buf, uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const SlotDev& L = p.slot[t.k];
  const int l0 = t.lc * kLC;
  const int Lo = min(kLC, L.d_out - l0);
  const int r0 = st * kExpandRows;
  const int nrows = min(kExpandRows, t.r - r0);
  const bool last = st == t.nst - 1;
  const uint32_t tbytes = 4u * kExpandRows * L.t_ns;
  if (lane == 0) mbar_expect_tx(bar, 2u * Lo * (nrows + (last ? t.ntok : 0)) + tbytes * t.ntok);
  __syncwarp();
  if (lane < 16) {
    const int i = lane & 7;
    if (i < nrows)
      piece_copy(p.pool, aux, (int64_t)(r0 + i) * L.d_out + l0, Lo, lane >> 3, buf + i * 2 * kLC, bar);
  } else if (lane < 20) {
    const int tt = lane - 16;
    if (tt < t.ntok) {
      const int64_t row = L.t_by_token ? (int64_t)aux : (int64_t)(t.seg0 + t.tg * t.nt + tt);
      bulk_g2s(buf + kExpT + tt * tbytes, L.t + row * L.t_rs + (int64_t)r0 * L.t_ns, tbytes, bar);
    }
  } else if (lane < 24 && last) {
    const int tt = lane - 20;
    if (tt < t.ntok) bulk_g2s(buf + kExpY + tt * 2 * kLC, L.y + (int64_t)aux * L.ldy + l0, 2u * Lo, bar);
  }
}

template <int DT>
__device__ __forceinline__ void expand_stage(const BgmvParams& p, const ETask& t, int st, unsigned char* buf,
                                             float (&acc)[4][8], int32_t ctok) {
  const int lane = threadIdx.x & 31;
  const SlotDev& L = p.slot[t.k];
  const int l0 = t.lc * kLC;
  const int Lo = min(kLC, L.d_out - l0);
  const int r0 = st * kExpandRows;
  const int nrows = min(kExpandRows, t.r - r0);
  // t for this stage: lane (tt, kk) sums the t_ns partials, in order
  float* tsum = reinterpret_cast<float*>(buf + kExpS);
  {
    const int tt = lane >> 3, kk = lane & 7;
    if (tt < t.ntok && kk < nrows) {
      const float* src = reinterpret_cast<const float*>(buf + kExpT + tt * 4 * kExpandRows * L.t_ns) + kk * L.t_ns;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;  // four chains; fixed association
      int c = 0;
      for (; c + 4 <= L.t_ns; c += 4) {
        s0 += src[c];
        s1 += src[c + 1];
        s2 += src[c + 2];
        s3 += src[c + 3];
      }
      for (; c < L.t_ns; ++c) s0 += src[c];
      tsum[tt * kExpandRows + kk] = (s0 + s1) + (s2 + s3);
    }
  }
  __syncwarp();
  const int l = lane * 8;
  const bool act = l < Lo;
  if (act) {
#pragma unroll
    for (int kk = 0; kk < kExpandRows; ++kk) {
      if (kk >= nrows) break;
      float bf[8];
      unpack8<DT>(lds128(buf + kk * 2 * kLC + 2 * l), bf);
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        if (tt >= t.ntok) break;
        const float tv = tsum[tt * kExpandRows + kk];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[tt][e] = fmaf(tv, bf[e], acc[tt][e]);
      }
    }
  }
  if (st != t.nst - 1) return;
  const float s_a = __ldg(p.pool.scale + t.a);
#pragma unroll
  for (int tt = 0; tt < 4; ++tt) {
    const int token = __shfl_sync(FULL_MASK, ctok, tt);
    if (act && tt < t.ntok) {
      float yf[8];
      unpack8<DT>(lds128(buf + kExpY + tt * 2 * kLC + 2 * l), yf);
      uint4 o;
      o.x = pack2<DT>(fmaf(s_a, acc[tt][0], yf[0]), fmaf(s_a, acc[tt][1], yf[1]));
      o.y = pack2<DT>(fmaf(s_a, acc[tt][2], yf[2]), fmaf(s_a, acc[tt][3], yf[3]));
      o.z = pack2<DT>(fmaf(s_a, acc[tt][4], yf[4]), fmaf(s_a, acc[tt][5], yf[5]));
      o.w = pack2<DT>(fmaf(s_a, acc[tt][6], yf[6]), fmaf(s_a, acc[tt][7], yf[7]));
      *reinterpret_cast<uint4*>(L.y + (int64_t)token * L.ldy + l0 + l) = o;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[tt][e] = 0.f;
  }
}

template <int DT>
__global__ void __launch_bounds__(kWarps * 32, 1) k_expand(const __grid_constant__ BgmvParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t bars[kWarps][kSlots];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wbuf = smem + warp * kSlots * kSlotBytes;
  int32_t* segsm = reinterpret_cast<int32_t*>(smem + kSmemBytes);
  if (lane == 0)
    for (int s = 0; s < kSlots; ++s) mbar_init(&bars[warp][s], 1);
  fence_mbar_init();
  griddep_wait();
  const int S = p.sc.meta[kMetaS];
  const int total = p.sc.meta[kMetaExpandTotal];
  const SegView V = stage_segments(p.sc, S, false, segsm);
  const int NW = gridDim.x * kWarps;
  const int first = blockIdx.x * kWarps + warp;
  if (first >= total) {
    griddep_launch();
    return;
  }
  int ptask = first, pst = 0, pslot = 0;
  ETask pt;
  decode_expand(p, V, ptask, pt);
  bool pvalid = true;
  int32_t aux = expand_lookup(p, pt, 0);
  auto produce = [&]() {
    issue_expand(p, pt, pst, aux, wbuf + pslot * kSlotBytes, &bars[warp][pslot]);
    pslot ^= 1;
    if (++pst == pt.nst) {
      pst = 0;
      ptask += NW;
      pvalid = ptask < total;
      if (pvalid) decode_expand(p, V, ptask, pt);
    }
    if (pvalid) aux = expand_lookup(p, pt, pst);
  };
  int ctask = first, cst = 0, slot = 0;
  ETask ct = pt;
  auto ctoken = [&]() {  // token ids of the consumer's task, lane tt holds token tt
    return lane < ct.ntok ? __ldg(p.sc.perm + ct.seg0 + ct.tg * ct.nt + lane) : 0;
  };
  int32_t ctok = ctoken();
  uint32_t parity = 0;
  float acc[4][8];
#pragma unroll
  for (int tt = 0; tt < 4; ++tt)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[tt][e] = 0.f;
  produce();
  for (;;) {
    if (pvalid) produce();
    if (!mbar_wait(&bars[warp][slot], (parity >> slot) & 1, p.pool.err)) break;
    parity ^= 1u << slot;
    expand_stage<DT>(p, ct, cst, wbuf + slot * kSlotBytes, acc, ctok);
    __syncwarp();
    fence_proxy_async();
    slot ^= 1;
    if (++cst == ct.nst) {
      cst = 0;
      ctask += NW;
      if (ctask >= total) break;
      decode_expand(p, V, ctask, ct);
      ctok = ctoken();
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
  if (tid == 0) {
    seg_start[S] = n > 0 ? req_start[n] : 0;
    *S_out = S;
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
constexpr int kDynSmem = kSmemBytes + 4 * kSegSmemInts;  // slots + segment table
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
static void set_attrs() {
  if (g_attrs_done) return;
  cudaFuncSetAttribute(k_segments, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
  cudaFuncSetAttribute(k_shrink<SLORA_F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem);
  cudaFuncSetAttribute(k_shrink<SLORA_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem);
  cudaFuncSetAttribute(k_expand<SLORA_F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem);
  cudaFuncSetAttribute(k_expand<SLORA_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem);
  g_attrs_done = true;
}

cudaError_t launch_segments(const BgmvParams& p, const int32_t* idx, int T, cudaStream_t s) {
  set_attrs();
  const size_t smem = sizeof(int) * (size_t)p.pool.max_adapters;
  k_segments<<<1, 1024, smem, s>>>(p, idx, T);
  return cudaGetLastError();
}

cudaError_t launch_shrink(const BgmvParams& p, int dtype, int grid, cudaStream_t s) {
  set_attrs();
  if (dtype == SLORA_BF16) return launch_dependent(k_shrink<SLORA_BF16>, grid, kWarps * 32, kDynSmem, s, p);
  return launch_dependent(k_shrink<SLORA_F16>, grid, kWarps * 32, kDynSmem, s, p);
}

cudaError_t launch_expand(const BgmvParams& p, int dtype, int grid, cudaStream_t s) {
  set_attrs();
  if (dtype == SLORA_BF16) return launch_dependent(k_expand<SLORA_BF16>, grid, kWarps * 32, kDynSmem, s, p);
  return launch_dependent(k_expand<SLORA_F16>, grid, kWarps * 32, kDynSmem, s, p);
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
  if (which == 0) cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_shrink<SLORA_F16>, kWarps * 32, kDynSmem);
  else cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_expand<SLORA_F16>, kWarps * 32, kDynSmem);
  return n > 0 ? n : 1;
}

}  // namespace slora
