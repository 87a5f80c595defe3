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
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "slora_internal.h"

namespace slora {

#define FULL_MASK 0xffffffffu

constexpr int kWarps = 8;                 // warps per CTA of shrink / expand
constexpr int kSlots = 2;                 // pipeline slots per warp
constexpr int kSlotBytes = 12 * 1024;     // bytes per slot
constexpr int kSmemBytes = kWarps * kSlots * kSlotBytes;
constexpr int kExpandRows = 16;           // B rows per expand stage
constexpr int kLC = 256;                  // outputs per expand task (8 per lane)
constexpr long long kWaitLimit = 2000000000ll;  // clock cycles before a wait gives up

__host__ __device__ __forceinline__ int cdiv_i(int a, int b) { return (a + b - 1) / b; }

// Task shapes.  Shrink tasks cover NT tokens x RW rank rows x kShrinkKC of d_in;
// expand tasks NTE tokens x kLC outputs.  Slot use: (RW + NT) KiB for shrink,
// 16 x 512 B + NTE x 512 B for expand; both fit kSlotBytes.
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

// Copies flat elements [f0, f0 + n) of a paged tensor into dst.  The range
// crosses at most one page boundary (n <= page size); piece 0 is the part in
// the first page, piece 1 the rest.  Returns nothing for an empty piece.
__device__ __forceinline__ void bulk_paged_piece(const PoolDev& P, int a, int lo, int64_t f0, int n,
                                                 int piece, unsigned char* dst, uint64_t* bar) {
  const int64_t pb = ((f0 >> P.page_shift) + 1) << P.page_shift;
  const int64_t f1 = f0 + n;
  if (piece == 0) {
    const int64_t e = f1 < pb ? f1 : pb;
    bulk_g2s(dst, page_addr(P, a, lo, f0), (uint32_t)(2 * (e - f0)), bar);
  } else if (f1 > pb) {
    bulk_g2s(dst + 2 * (pb - f0), page_addr(P, a, lo, pb), (uint32_t)(2 * (f1 - pb)), bar);
  }
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
// of shrink tasks, reduction counters and expand tasks before it (prefix sums
// in segment-major task order).

__device__ __forceinline__ void seg_task_counts(const BgmvParams& p, int n, int r, int& shr, int& ctr,
                                                int& exp) {
  shr = ctr = exp = 0;
  if (n == 0 || r <= 0) return;
  const int nt = nt_class(n), ntg = cdiv_i(n, nt), nte = cdiv_i(n, nte_class(n));
  if (p.do_shrink)
    for (int g = 0; g < p.n_groups; ++g) {
      const int nrg = cdiv_i(p.group[g].n * r, rw_of(nt));
      shr += nrg * ntg * cdiv_i(p.group[g].d_in, kShrinkKC);
      ctr += nrg * ntg;
    }
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
  int cnt = 0, nseg = 0, c_shr = 0, c_ctr = 0, c_exp = 0;
  for (int a = a0; a < a1; ++a) {
    const int n = hist[a];
    if (n == 0) continue;
    int x, y, z;
    seg_task_counts(p, n, p.pool.rank[a], x, y, z);
    cnt += n;
    nseg += 1;
    c_shr += x;
    c_ctr += y;
    c_exp += z;
  }
  int n_valid, S, t_shr, t_ctr, t_exp;
  int cbase = block_exscan<false>(cnt, &n_valid, sh);
  int sb = block_exscan<false>(nseg, &S, sh);
  int b_shr = block_exscan<false>(c_shr, &t_shr, sh);
  int b_ctr = block_exscan<false>(c_ctr, &t_ctr, sh);
  int b_exp = block_exscan<false>(c_exp, &t_exp, sh);
  for (int a = a0; a < a1; ++a) {
    const int n = hist[a];
    hist[a] = cbase;  // becomes the scatter cursor
    if (n == 0) continue;
    const int r = p.pool.rank[a];
    int x, y, z;
    seg_task_counts(p, n, r, x, y, z);
    sc.seg_start[sb] = cbase;
    sc.seg_adapter[sb] = a;
    sc.seg_rank[sb] = r;
    sc.shrink_prefix[sb] = b_shr;
    sc.ctr_prefix[sb] = b_ctr;
    sc.expand_prefix[sb] = b_exp;
    ++sb;
    cbase += n;
    b_shr += x;
    b_ctr += y;
    b_exp += z;
  }
  int ctr_total = t_ctr;
  if (ctr_total > sc.ctr_cap) {  // cannot happen with the sizing in slora_scratch_bytes
    if (tid == 0) record_error(p.pool.err, 3, ctr_total);
    ctr_total = t_shr = t_exp = 0;
  }
  if (tid == 0) {
    sc.seg_start[S] = n_valid;
    sc.shrink_prefix[S] = t_shr;
    sc.ctr_prefix[S] = t_ctr;
    sc.expand_prefix[S] = t_exp;
    sc.meta[kMetaS] = S;
    sc.meta[kMetaValid] = n_valid;
    sc.meta[kMetaShrinkTotal] = t_shr;
    sc.meta[kMetaExpandTotal] = t_exp;
    sc.meta[kMetaCtrTotal] = ctr_total;
  }
  for (int c = tid; c < ctr_total; c += nth) sc.ctr[c] = 0;
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
struct SegView {
  const int32_t* start;   // [S + 1]
  const int32_t* adapter; // [S]
  const int32_t* rank;    // [S]
  const int32_t* prefix;  // [S + 1] tasks before each segment
  const int32_t* ctr;     // [S + 1] counters before each segment (shrink only)
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
    v.ctr = sc.ctr_prefix;
    return v;
  }
  int32_t* st = sm;
  int32_t* ad = sm + (kSegCap + 1);
  int32_t* rk = ad + kSegCap;
  int32_t* pf = rk + kSegCap;
  int32_t* ct = pf + (kSegCap + 1);
  for (int i = threadIdx.x; i <= S; i += blockDim.x) {
    st[i] = sc.seg_start[i];
    pf[i] = pre[i];
    if (shrink) ct[i] = sc.ctr_prefix[i];
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
  v.ctr = ct;
  return v;
}
constexpr int kSegSmemInts = 5 * kSegCap + 3;

// ---------------------------------------------------------------------------
// Shrink.
struct STask {
  int g, a, r, seg0, n, nt, rw, rg, tg, kc, n_kc, ci;
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
  int ci = V.ctr[s];
  int g = 0;
  for (; g < p.n_groups - 1; ++g) {  // the group owning local task q
    const int nrg = cdiv_i(p.group[g].n * t.r, t.rw);
    const int cnt = nrg * n_tg * cdiv_i(p.group[g].d_in, kShrinkKC);
    if (q < cnt) break;
    q -= cnt;
    ci += nrg * n_tg;
  }
  t.g = g;
  t.n_kc = cdiv_i(p.group[g].d_in, kShrinkKC);
  t.tg = q % n_tg;
  q /= n_tg;
  t.kc = q % t.n_kc;
  t.rg = q / t.n_kc;
  t.ci = ci + t.rg * n_tg + t.tg;
}

// Slot layout: rank row i at i * 1 KiB, token row t at (rw + t) * 1 KiB.
__device__ __forceinline__ void issue_shrink(const BgmvParams& p, const STask& t, unsigned char* buf,
                                             uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const GroupDev& G = p.group[t.g];
  const int k0 = t.kc * kShrinkKC;
  const int L = min(kShrinkKC, G.d_in - k0);
  const int R = G.n * t.r;
  const int nrows = min(t.rw, R - t.rg * t.rw);
  const int ntok = min(t.nt, t.n - t.tg * t.nt);
  if (lane == 0) mbar_expect_tx(bar, 2u * L * (nrows + ntok));
  __syncwarp();
  const int i = lane & 15;
  if (i < nrows) {
    const int rho = t.rg * t.rw + i;
    const int j = rho / t.r, k = rho % t.r;
    const int lo = p.slot[G.slot[j]].listA;
    bulk_paged_piece(p.pool, t.a, lo, (int64_t)k * G.d_in + k0, L, lane >> 4, buf + i * 2 * kShrinkKC, bar);
  } else if (lane < 16 && i < nrows + ntok) {
    const int tt = i - nrows;
    const int token = __ldg(p.sc.perm + t.seg0 + t.tg * t.nt + tt);
    bulk_g2s(buf + (t.rw + tt) * 2 * kShrinkKC, G.x + (int64_t)token * G.ldx + k0, 2u * L, bar);
  }
}

template <int DT, int NT, int RW>
__device__ __forceinline__ void compute_shrink(const BgmvParams& p, const STask& t,
                                               const unsigned char* buf) {
  const int lane = threadIdx.x & 31;
  const GroupDev& G = p.group[t.g];
  const PoolDev& P = p.pool;
  const int k0 = t.kc * kShrinkKC;
  const int L = min(kShrinkKC, G.d_in - k0);
  const int R = G.n * t.r;
  const int nrows = min(RW, R - t.rg * RW);
  const int ntok = min(NT, t.n - t.tg * NT);

  float acc[RW * NT];
#pragma unroll
  for (int i = 0; i < RW * NT; ++i) acc[i] = 0.f;
#pragma unroll
  for (int e = lane * 8; e < kShrinkKC; e += 256) {
    if (e >= L) break;
    uint4 av[RW], xv[NT];
#pragma unroll
    for (int i = 0; i < RW; ++i) av[i] = i < nrows ? lds128(buf + i * 2 * kShrinkKC + 2 * e) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int tt = 0; tt < NT; ++tt)
      xv[tt] = tt < ntok ? lds128(buf + (RW + tt) * 2 * kShrinkKC + 2 * e) : make_uint4(0, 0, 0, 0);
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

  const float val = lane_transpose_reduce<RW * NT>(acc);
  const int Lx = lane % (RW * NT);
  const int i = Lx / NT, tt = Lx % NT;
  const int rho = t.rg * RW + i;
  const bool mine = lane < RW * NT && i < nrows && tt < ntok;
  const int j = mine ? rho / t.r : 0, k = mine ? rho % t.r : 0;
  const SlotDev& S = p.slot[G.slot[j]];
  const int pos = t.seg0 + t.tg * NT + tt;
  if (t.n_kc == 1) {
    if (mine) {
      const int64_t row = S.t_by_token ? (int64_t)__ldg(p.sc.perm + pos) : (int64_t)pos;
      S.tfin[row * S.ldt + k] = val;
    }
    return;
  }
  if (mine) S.tpart[((int64_t)t.kc * p.max_tokens + pos) * P.max_rank + k] = val;
  __threadfence();
  __syncwarp();
  int old = 0;
  if (lane == 0) old = atomicAdd(p.sc.ctr + t.ci, 1);
  old = __shfl_sync(FULL_MASK, old, 0);
  if (old != t.n_kc - 1) return;
  __threadfence();
  if (mine) {  // last of the n_kc chunk tasks: sum the partials in chunk order
    float s = 0.f;
    for (int c = 0; c < t.n_kc; ++c)
      s += __ldcg(S.tpart + ((int64_t)c * p.max_tokens + pos) * P.max_rank + k);
    const int64_t row = S.t_by_token ? (int64_t)__ldg(p.sc.perm + pos) : (int64_t)pos;
    S.tfin[row * S.ldt + k] = s;
  }
}

template <int DT>
__device__ __forceinline__ void compute_shrink_any(const BgmvParams& p, const STask& t,
                                                   const unsigned char* buf) {
  switch (t.nt) {
    case 1: compute_shrink<DT, 1, 8>(p, t, buf); break;
    case 2: compute_shrink<DT, 2, 4>(p, t, buf); break;
    case 4: compute_shrink<DT, 4, 4>(p, t, buf); break;
    default: compute_shrink<DT, 8, 4>(p, t, buf); break;
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
  int task = blockIdx.x * kWarps + warp;
  STask cur, nxt;
  bool have = task < total;
  if (have) {
    decode_shrink(p, V, task, cur);
    issue_shrink(p, cur, wbuf, &bars[warp][0]);
  }
  int slot = 0;
  uint32_t parity = 0;
  while (have) {
    const int ntask = task + NW;
    const bool hn = ntask < total;
    if (hn) {
      decode_shrink(p, V, ntask, nxt);
      issue_shrink(p, nxt, wbuf + (slot ^ 1) * kSlotBytes, &bars[warp][slot ^ 1]);
    }
    if (!mbar_wait(&bars[warp][slot], (parity >> slot) & 1, p.pool.err)) break;
    parity ^= 1u << slot;
    compute_shrink_any<DT>(p, cur, wbuf + slot * kSlotBytes);
    __syncwarp();
    fence_proxy_async();
    slot ^= 1;
    task = ntask;
    cur = nxt;
    have = hn;
  }
  griddep_launch();
}

// ---------------------------------------------------------------------------
// Expand.
struct ETask {
  int k, a, r, seg0, n, nt, tg, lc, nks;
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
  t.nks = cdiv_i(t.r, kExpandRows);
}

// Slot layout: B row i of this stage at i * 512 B; t values of token t for
// this stage's rank rows at 8 KiB + t * 64 B; in a task's last stage, y row t
// at 8 KiB + 256 B + t * 512 B.
constexpr int kExpTOff = kExpandRows * 2 * kLC;
constexpr int kExpYOff = kExpTOff + 4 * 64;

__device__ __forceinline__ void issue_expand(const BgmvParams& p, const ETask& t, int ks,
                                             unsigned char* buf, uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const SlotDev& L = p.slot[t.k];
  const int l0 = t.lc * kLC;
  const int Lo = min(kLC, L.d_out - l0);
  const int r0 = ks * kExpandRows;
  const int nrows = min(kExpandRows, t.r - r0);
  const int tcols = (nrows + 3) & ~3;  // t floats copied per token (16-byte multiple)
  const bool last = ks == t.nks - 1;
  const int ntok = min(t.nt, t.n - t.tg * t.nt);
  const int nyt = last ? ntok : 0;
  if (lane == 0) mbar_expect_tx(bar, 2u * Lo * (nrows + nyt) + 4u * tcols * ntok);
  __syncwarp();
  const int i = lane & 15;
  if (i < nrows)
    bulk_paged_piece(p.pool, t.a, L.listB, (int64_t)(r0 + i) * L.d_out + l0, Lo, lane >> 4,
                     buf + i * 2 * kLC, bar);
  if (lane < ntok) {
    const int pos = t.seg0 + t.tg * t.nt + lane;
    const int token = __ldg(p.sc.perm + pos);
    const int64_t row = L.t_by_token ? (int64_t)token : (int64_t)pos;
    bulk_g2s(buf + kExpTOff + lane * 64, L.tfin + row * L.ldt + r0, 4u * tcols, bar);
    if (last) bulk_g2s(buf + kExpYOff + lane * 2 * kLC, L.y + (int64_t)token * L.ldy + l0, 2u * Lo, bar);
  }
}

template <int DT>
__device__ __forceinline__ void compute_expand(const BgmvParams& p, const ETask& t, int ks,
                                               const unsigned char* buf, float (&acc)[4][8]) {
  const int lane = threadIdx.x & 31;
  const SlotDev& L = p.slot[t.k];
  const int l0 = t.lc * kLC;
  const int Lo = min(kLC, L.d_out - l0);
  const int r0 = ks * kExpandRows;
  const int nrows = min(kExpandRows, t.r - r0);
  const int ntok = min(t.nt, t.n - t.tg * t.nt);
  const int l = lane * 8;
  const bool act = l < Lo;
  const float* tv = reinterpret_cast<const float*>(buf + kExpTOff);
  if (act) {
#pragma unroll 4
    for (int kk = 0; kk < nrows; ++kk) {
      float bf[8];
      unpack8<DT>(lds128(buf + kk * 2 * kLC + 2 * l), bf);
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        if (tt >= ntok) break;
        const float tvv = tv[tt * 16 + kk];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[tt][e] = fmaf(tvv, bf[e], acc[tt][e]);
      }
    }
  }
  if (ks != t.nks - 1) return;
  const float s_a = __ldg(p.pool.scale + t.a);
  if (act) {
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
      if (tt >= ntok) break;
      const int token = __ldg(p.sc.perm + t.seg0 + t.tg * t.nt + tt);
      float yf[8];
      unpack8<DT>(lds128(buf + kExpYOff + tt * 2 * kLC + 2 * l), yf);
      uint4 o;
      o.x = pack2<DT>(fmaf(s_a, acc[tt][0], yf[0]), fmaf(s_a, acc[tt][1], yf[1]));
      o.y = pack2<DT>(fmaf(s_a, acc[tt][2], yf[2]), fmaf(s_a, acc[tt][3], yf[3]));
      o.z = pack2<DT>(fmaf(s_a, acc[tt][4], yf[4]), fmaf(s_a, acc[tt][5], yf[5]));
      o.w = pack2<DT>(fmaf(s_a, acc[tt][6], yf[6]), fmaf(s_a, acc[tt][7], yf[7]));
      *reinterpret_cast<uint4*>(L.y + (int64_t)token * L.ldy + l0 + l) = o;
    }
  }
#pragma unroll
  for (int tt = 0; tt < 4; ++tt)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[tt][e] = 0.f;
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
  int task = blockIdx.x * kWarps + warp;
  ETask cur, nxt;
  bool have = task < total;
  int ks = 0;
  if (have) {
    decode_expand(p, V, task, cur);
    issue_expand(p, cur, 0, wbuf, &bars[warp][0]);
  }
  float acc[4][8];
#pragma unroll
  for (int tt = 0; tt < 4; ++tt)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[tt][e] = 0.f;
  int slot = 0;
  uint32_t parity = 0;
  while (have) {
    // next stage: the next rank chunk of this task, or the first of the next task
    int nks = ks + 1, ntask = task;
    bool hn = true;
    if (nks >= cur.nks) {
      nks = 0;
      ntask = task + NW;
      hn = ntask < total;
      if (hn) decode_expand(p, V, ntask, nxt);
    } else {
      nxt = cur;
    }
    if (hn) issue_expand(p, nxt, nks, wbuf + (slot ^ 1) * kSlotBytes, &bars[warp][slot ^ 1]);
    if (!mbar_wait(&bars[warp][slot], (parity >> slot) & 1, p.pool.err)) break;
    parity ^= 1u << slot;
    compute_expand<DT>(p, cur, ks, wbuf + slot * kSlotBytes, acc);
    __syncwarp();
    fence_proxy_async();
    slot ^= 1;
    task = ntask;
    ks = nks;
    cur = nxt;
    have = hn;
  }
  griddep_launch();
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
