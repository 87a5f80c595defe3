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
// All three compute kernels are persistent: a grid of (SMs x resident CTAs)
// whose warps pull tasks from a device counter.  A task reads one adapter tile
// once and applies it to every token of its segment that the task covers, so
// each touched adapter is streamed from HBM about once per step.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "slora_internal.h"

namespace slora {

#define FULL_MASK 0xffffffffu

__device__ __forceinline__ int cdiv_i(int a, int b) { return (a + b - 1) / b; }

// Token classes: tasks cover NT tokens of a segment and RW rank rows.
__device__ __forceinline__ int nt_class(int n) { return n <= 1 ? 1 : (n == 2 ? 2 : (n <= 4 ? 4 : 8)); }
__device__ __forceinline__ int rw_of(int nt) { return nt == 1 ? 8 : 4; }
// Expand tasks cover at most 4 tokens (8 fp32 accumulators per token per lane).
__device__ __forceinline__ int nte_class(int n) { return n <= 1 ? 1 : (n == 2 ? 2 : 4); }
// Outputs per expand task: about 16 KB of B per task.
__device__ __forceinline__ int lc_of(int r) {
  int lc = (8192 / (r > 0 ? r : 1)) & ~255;
  return lc < 256 ? 256 : lc;
}

__device__ __forceinline__ void record_error(int32_t* err, int code, int info) {
  if (atomicCAS(&err[0], 0, code) == 0) atomicExch(&err[1], info);
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

__device__ __forceinline__ uint4 ldg_nc(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Address of flat element f of tensor (adapter a, page-list offset lo).
__device__ __forceinline__ const uint16_t* page_addr(const PoolDev& P, int a, int lo, int64_t f) {
  const int32_t pg = __ldg(P.page_list + (int64_t)a * P.list_stride + lo + (f >> P.page_shift));
  return P.pool + ((int64_t)pg << P.page_shift) + (f & ((1ll << P.page_shift) - 1));
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan (blockDim.x threads, multiple of 32).
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

// ---------------------------------------------------------------------------
// k_segments: one CTA of 1024 threads.  Dynamic smem: max_adapters ints.
__global__ void __launch_bounds__(1024) k_segments(const __grid_constant__ BgmvParams p,
                                                   const int32_t* __restrict__ idx, int T) {
  extern __shared__ int hist[];
  __shared__ int sh[32];
  __shared__ int s_tot[4];
  const int tid = threadIdx.x, nth = blockDim.x;
  const int MA = p.pool.max_adapters;
  const ScratchDev& sc = p.sc;

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

  // Per-thread contiguous adapter range -> counts, segment flags -> scans.
  const int E = (MA + nth - 1) / nth;
  const int a0 = min(tid * E, MA), a1 = min(a0 + E, MA);
  int cnt = 0, nseg = 0;
  for (int a = a0; a < a1; ++a) {
    cnt += hist[a];
    nseg += hist[a] > 0;
  }
  int n_valid, S;
  int cbase = block_exscan<false>(cnt, &n_valid, sh);
  int sbase = block_exscan<false>(nseg, &S, sh);
  for (int a = a0; a < a1; ++a) {
    const int h = hist[a];
    if (h > 0) {
      sc.seg_start[sbase] = cbase;
      sc.seg_adapter[sbase] = a;
      ++sbase;
    }
    hist[a] = cbase;  // becomes the scatter cursor
    cbase += h;
  }
  if (tid == 0) {
    sc.seg_start[S] = n_valid;
    sc.meta[kMetaS] = S;
    sc.meta[kMetaValid] = n_valid;
  }
  __syncthreads();

  // Stable scatter: chunks of 1024 tokens, warps take turns in order.
  const int lane = tid & 31, warp = tid >> 5;
  for (int c0 = 0; c0 < T; c0 += nth) {
    const int i = c0 + tid;
    int a = i < T ? idx[i] : -1;
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

  // Work planning, per group (shrink, counters) and per slot (expand).
  const int ES = (S + nth - 1) / nth;
  const int s0 = min(tid * ES, S), s1 = min(s0 + ES, S);
  int tot_shrink = 0, tot_ctr = 0, tot_expand = 0;
  for (int g = 0; g < p.n_groups; ++g) {
    const GroupDev& G = p.group[g];
    const int n_kc = cdiv_i(G.d_in, kShrinkKC);
    int lt = 0, lc = 0;
    for (int s = s0; s < s1; ++s) {
      const int n = sc.seg_start[s + 1] - sc.seg_start[s];
      const int r = p.pool.rank[sc.seg_adapter[s]];
      const int nt = nt_class(n);
      const int ntg = cdiv_i(n, nt), nrg = cdiv_i(G.n * r, rw_of(nt));
      lt += p.do_shrink ? nrg * ntg * n_kc : 0;
      lc += p.do_shrink ? nrg * ntg : 0;
    }
    int tt, tc;
    int bt = block_exscan<false>(lt, &tt, sh);
    int bc = block_exscan<false>(lc, &tc, sh);
    int32_t* pt = sc.shrink_prefix + g * (sc.MS + 1);
    int32_t* pc = sc.ctr_prefix + g * (sc.MS + 1);
    for (int s = s0; s < s1; ++s) {
      const int n = sc.seg_start[s + 1] - sc.seg_start[s];
      const int r = p.pool.rank[sc.seg_adapter[s]];
      const int nt = nt_class(n);
      const int ntg = cdiv_i(n, nt), nrg = cdiv_i(G.n * r, rw_of(nt));
      pt[s] = bt;  // group-local prefix
      pc[s] = tot_ctr + bc;
      bt += p.do_shrink ? nrg * ntg * n_kc : 0;
      bc += p.do_shrink ? nrg * ntg : 0;
    }
    if (tid == 0) pt[S] = tt, pc[S] = tot_ctr + tc;
    tot_shrink += tt;
    tot_ctr += tc;
  }
  for (int k = 0; k < p.n_slots; ++k) {
    const SlotDev& L = p.slot[k];
    int le = 0;
    for (int s = s0; s < s1; ++s) {
      const int n = sc.seg_start[s + 1] - sc.seg_start[s];
      const int r = p.pool.rank[sc.seg_adapter[s]];
      le += (p.do_expand && r > 0) ? cdiv_i(n, nte_class(n)) * cdiv_i(L.d_out, lc_of(r)) : 0;
    }
    int te;
    int be = block_exscan<false>(le, &te, sh);
    int32_t* pe = sc.expand_prefix + k * (sc.MS + 1);
    for (int s = s0; s < s1; ++s) {
      const int n = sc.seg_start[s + 1] - sc.seg_start[s];
      const int r = p.pool.rank[sc.seg_adapter[s]];
      pe[s] = be;
      be += (p.do_expand && r > 0) ? cdiv_i(n, nte_class(n)) * cdiv_i(L.d_out, lc_of(r)) : 0;
    }
    if (tid == 0) pe[S] = te;
    tot_expand += te;
  }
  if (tid == 0) {
    s_tot[0] = tot_shrink;
    s_tot[1] = tot_ctr;
  }
  __syncthreads();
  int ctr_total = s_tot[1];
  if (ctr_total > sc.ctr_cap) {  // cannot happen with the sizing in slora_scratch_bytes
    if (tid == 0) record_error(p.pool.err, 3, ctr_total);
    ctr_total = 0;
    tot_shrink = 0;
    tot_expand = 0;
  }
  for (int c = tid; c < ctr_total; c += nth) sc.ctr[c] = 0;
  if (tid == 0) {
    sc.meta[kMetaShrinkTotal] = tot_shrink;
    sc.meta[kMetaExpandTotal] = tot_expand;
    sc.meta[kMetaCtrTotal] = ctr_total;
    sc.meta[kMetaShrinkWork] = 0;
    sc.meta[kMetaExpandWork] = 0;
  }
}

// Largest s with prefix[s] <= q (prefix ascending, prefix[0] = 0).
__device__ __forceinline__ int find_seg(const int32_t* prefix, int S, int q) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(prefix + mid) <= q) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Sum over the 32 lanes of each of the N values v[0..N); afterwards lane L
// holds the total of value L % N.  N is a power of two <= 32.
template <int N>
__device__ __forceinline__ float lane_transpose_reduce(float (&v)[N]) {
  // fold lanes that share an output first
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
// Shrink task: RW rank rows x NT tokens x one d_in chunk.
template <int DT, int NT, int RW>
__device__ __noinline__ void shrink_task(const BgmvParams& p, const GroupDev& G, int a, int r,
                                            int seg0, int n, int rg, int tg, int kc, int n_kc,
                                            int ci) {
  const int lane = threadIdx.x & 31;
  const PoolDev& P = p.pool;
  const int R = G.n * r;
  const int k0 = kc * kShrinkKC, k1 = min(G.d_in, k0 + kShrinkKC);

  // rows
  int row_lo[RW];
  int64_t row_f[RW];
  bool row_ok[RW];
#pragma unroll
  for (int i = 0; i < RW; ++i) {
    const int rho = rg * RW + i;
    row_ok[i] = rho < R;
    const int j = row_ok[i] ? rho / r : 0, k = row_ok[i] ? rho % r : 0;
    row_lo[i] = p.slot[G.slot[j]].listA;
    row_f[i] = (int64_t)k * G.d_in;
  }
  // tokens
  const uint16_t* xrow[NT];
  bool tok_ok[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int q = tg * NT + t;
    tok_ok[t] = q < n;
    const int token = tok_ok[t] ? __ldg(p.sc.perm + seg0 + q) : 0;
    xrow[t] = G.x + (int64_t)token * G.ldx;
  }

  float acc[RW * NT];
#pragma unroll
  for (int i = 0; i < RW * NT; ++i) acc[i] = 0.f;

#pragma unroll 1
  for (int e0 = k0 + lane * 8; e0 < k1; e0 += 256) {
    uint4 av[RW], xv[NT];
#pragma unroll
    for (int i = 0; i < RW; ++i)
      av[i] = row_ok[i] ? ldg_nc(page_addr(P, a, row_lo[i], row_f[i] + e0)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int t = 0; t < NT; ++t)
      xv[t] = tok_ok[t] ? __ldg(reinterpret_cast<const uint4*>(xrow[t] + e0)) : make_uint4(0, 0, 0, 0);
    if (NT <= 2) {  // few tokens: unpack x once, stream the rows
      float xf[NT][8];
#pragma unroll
      for (int t = 0; t < NT; ++t) unpack8<DT>(xv[t], xf[t]);
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        float af[8];
        unpack8<DT>(av[i], af);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          float s = acc[i * NT + t];
#pragma unroll
          for (int e = 0; e < 8; ++e) s = fmaf(af[e], xf[t][e], s);
          acc[i * NT + t] = s;
        }
      }
    } else {        // many tokens: unpack the rows once, stream the tokens
      float af[RW][8];
#pragma unroll
      for (int i = 0; i < RW; ++i) unpack8<DT>(av[i], af[i]);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float xf[8];
        unpack8<DT>(xv[t], xf);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          float s = acc[i * NT + t];
#pragma unroll
          for (int e = 0; e < 8; ++e) s = fmaf(af[i][e], xf[e], s);
          acc[i * NT + t] = s;
        }
      }
    }
  }

  const float v = lane_transpose_reduce<RW * NT>(acc);
  const int L = lane % (RW * NT);
  const int i = L / NT, t = L % NT;
  const int rho = rg * RW + i;
  const int q = tg * NT + t;
  const bool mine = lane < RW * NT && rho < R && q < n;
  const int j = rho / r, k = rho % r;
  const SlotDev& S = p.slot[G.slot[mine ? j : 0]];
  const int pos = seg0 + q;
  if (n_kc == 1) {
    if (mine) {
      const int64_t row = S.t_by_token ? (int64_t)__ldg(p.sc.perm + pos) : (int64_t)pos;
      S.tfin[row * S.ldt + k] = v;
    }
    return;
  }
  if (mine) S.tpart[((int64_t)kc * p.max_tokens + pos) * P.max_rank + k] = v;
  __threadfence();
  __syncwarp();
  int old = 0;
  if (lane == 0) old = atomicAdd(p.sc.ctr + ci, 1);
  old = __shfl_sync(FULL_MASK, old, 0);
  if (old != n_kc - 1) return;
  __threadfence();
  if (mine) {  // last of the n_kc chunk tasks: sum the partials in chunk order
    float s = 0.f;
    for (int c = 0; c < n_kc; ++c) s += __ldcg(S.tpart + ((int64_t)c * p.max_tokens + pos) * P.max_rank + k);
    const int64_t row = S.t_by_token ? (int64_t)__ldg(p.sc.perm + pos) : (int64_t)pos;
    S.tfin[row * S.ldt + k] = s;
  }
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 2) k_shrink(const __grid_constant__ BgmvParams p) {
  const int lane = threadIdx.x & 31;
  const ScratchDev& sc = p.sc;
  const int S = sc.meta[kMetaS];
  const int total = sc.meta[kMetaShrinkTotal];
  for (;;) {
    int task = 0;
    if (lane == 0) task = atomicAdd(sc.meta + kMetaShrinkWork, 1);
    task = __shfl_sync(FULL_MASK, task, 0);
    if (task >= total) return;
    int g = 0, base = 0;
    for (; g < p.n_groups; ++g) {
      const int tg_tot = sc.shrink_prefix[g * (sc.MS + 1) + S];
      if (task < base + tg_tot) break;
      base += tg_tot;
    }
    const GroupDev& G = p.group[g];
    const int32_t* pre = sc.shrink_prefix + g * (sc.MS + 1);
    const int s = find_seg(pre, S, task - base);
    int q = task - base - pre[s];
    const int a = sc.seg_adapter[s];
    const int seg0 = sc.seg_start[s], n = sc.seg_start[s + 1] - seg0;
    const int r = p.pool.rank[a];
    const int nt = nt_class(n);
    const int n_tg = cdiv_i(n, nt), n_kc = cdiv_i(G.d_in, kShrinkKC);
    const int tg = q % n_tg;
    q /= n_tg;
    const int kc = q % n_kc, rg = q / n_kc;
    const int ci = sc.ctr_prefix[g * (sc.MS + 1) + s] + rg * n_tg + tg;
    switch (nt) {
      case 1: shrink_task<DT, 1, 8>(p, G, a, r, seg0, n, rg, tg, kc, n_kc, ci); break;
      case 2: shrink_task<DT, 2, 4>(p, G, a, r, seg0, n, rg, tg, kc, n_kc, ci); break;
      case 4: shrink_task<DT, 4, 4>(p, G, a, r, seg0, n, rg, tg, kc, n_kc, ci); break;
      default: shrink_task<DT, 8, 4>(p, G, a, r, seg0, n, rg, tg, kc, n_kc, ci); break;
    }
  }
}

// ---------------------------------------------------------------------------
// Expand task: NT tokens x LC outputs of one projection.
template <int DT, int NT>
__device__ __forceinline__ void expand_task(const BgmvParams& p, const SlotDev& L, int a, int r,
                                            int seg0, int n, int tg, int lc) {
  const int lane = threadIdx.x & 31;
  const PoolDev& P = p.pool;
  const float s_a = P.scale[a];
  const int LC = lc_of(r);
  int token[NT];
  bool tok_ok[NT];
  const float* trow[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int q = tg * NT + t;
    tok_ok[t] = q < n;
    const int pos = seg0 + (tok_ok[t] ? q : 0);
    token[t] = __ldg(p.sc.perm + pos);
    trow[t] = L.tfin + (L.t_by_token ? (int64_t)token[t] : (int64_t)pos) * L.ldt;
  }
  const int l_end = min(L.d_out, (lc + 1) * LC);
  for (int l = lc * LC + lane * 8; l - lane * 8 < l_end; l += 256) {
    const bool act = l < l_end;
    float acc[NT][8];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[t][e] = 0.f;
#pragma unroll 1
    for (int k0 = 0; k0 < r; k0 += 4) {
      uint4 bv[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        bv[kk] = (act && k0 + kk < r) ? ldg_nc(page_addr(P, a, L.listB, (int64_t)(k0 + kk) * L.d_out + l))
                                      : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        float bf[8];
        unpack8<DT>(bv[kk], bf);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float tv = (k0 + kk < r) ? __ldg(trow[t] + k0 + kk) : 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[t][e] = fmaf(tv, bf[e], acc[t][e]);
        }
      }
    }
    if (!act) continue;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (!tok_ok[t]) continue;
      float yf[8];
      unpack8<DT>(*reinterpret_cast<const uint4*>(L.y + (int64_t)token[t] * L.ldy + l), yf);
      uint4 o;
      o.x = pack2<DT>(fmaf(s_a, acc[t][0], yf[0]), fmaf(s_a, acc[t][1], yf[1]));
      o.y = pack2<DT>(fmaf(s_a, acc[t][2], yf[2]), fmaf(s_a, acc[t][3], yf[3]));
      o.z = pack2<DT>(fmaf(s_a, acc[t][4], yf[4]), fmaf(s_a, acc[t][5], yf[5]));
      o.w = pack2<DT>(fmaf(s_a, acc[t][6], yf[6]), fmaf(s_a, acc[t][7], yf[7]));
      *reinterpret_cast<uint4*>(L.y + (int64_t)token[t] * L.ldy + l) = o;
    }
  }
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 2) k_expand(const __grid_constant__ BgmvParams p) {
  const int lane = threadIdx.x & 31;
  const ScratchDev& sc = p.sc;
  const int S = sc.meta[kMetaS];
  const int total = sc.meta[kMetaExpandTotal];
  for (;;) {
    int task = 0;
    if (lane == 0) task = atomicAdd(sc.meta + kMetaExpandWork, 1);
    task = __shfl_sync(FULL_MASK, task, 0);
    if (task >= total) return;
    int k = 0, base = 0;
    for (; k < p.n_slots; ++k) {
      const int tk = sc.expand_prefix[k * (sc.MS + 1) + S];
      if (task < base + tk) break;
      base += tk;
    }
    const SlotDev& L = p.slot[k];
    const int32_t* pre = sc.expand_prefix + k * (sc.MS + 1);
    const int s = find_seg(pre, S, task - base);
    const int q = task - base - pre[s];
    const int a = sc.seg_adapter[s];
    const int seg0 = sc.seg_start[s], n = sc.seg_start[s + 1] - seg0;
    const int r = p.pool.rank[a];
    const int nt = nte_class(n);
    const int n_tg = cdiv_i(n, nt);
    const int tg = q % n_tg, lc = q / n_tg;
    switch (nt) {
      case 1: expand_task<DT, 1>(p, L, a, r, seg0, n, tg, lc); break;
      case 2: expand_task<DT, 2>(p, L, a, r, seg0, n, tg, lc); break;
      default: expand_task<DT, 4>(p, L, a, r, seg0, n, tg, lc); break;
    }
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
cudaError_t launch_segments(const BgmvParams& p, const int32_t* idx, int T, cudaStream_t s) {
  const size_t smem = sizeof(int) * (size_t)p.pool.max_adapters;
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(k_segments, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024 + 1024);
    attr_done = true;
  }
  k_segments<<<1, 1024, smem, s>>>(p, idx, T);
  return cudaGetLastError();
}

cudaError_t launch_shrink(const BgmvParams& p, int dtype, int grid, cudaStream_t s) {
  if (dtype == SLORA_BF16) k_shrink<SLORA_BF16><<<grid, kThreads, 0, s>>>(p);
  else k_shrink<SLORA_F16><<<grid, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_expand(const BgmvParams& p, int dtype, int grid, cudaStream_t s) {
  if (dtype == SLORA_BF16) k_expand<SLORA_BF16><<<grid, kThreads, 0, s>>>(p);
  else k_expand<SLORA_F16><<<grid, kThreads, 0, s>>>(p);
  return cudaGetLastError();
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

int occupancy_blocks(int which) {
  int n = 0;
  if (which == 0) cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_shrink<SLORA_F16>, kThreads, 0);
  else cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_expand<SLORA_F16>, kThreads, 0);
  return n > 0 ? n : 1;
}

}  // namespace slora
