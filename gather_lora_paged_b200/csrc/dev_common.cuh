// dev_common.cuh -- device helpers shared by the decode kernels (bgmv.cu,
// fused.cu): bounded mbarrier and counter waits, bulk copies, 16-bit
// arithmetic with fp32 accumulation, page-table addressing and block scans.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "slora_internal.h"

namespace slora {

#define FULL_MASK 0xffffffffu

constexpr long long kWaitLimit = 2000000000ll;  // clock cycles before a wait gives up

__host__ __device__ __forceinline__ int cdiv_i(int a, int b) { return (a + b - 1) / b; }

// Token classes of a task (template NT of the consumers): shrink and expand
// tasks take up to 4 tokens of a segment.  (Shrink consumers read every x row
// of the task once per rank row, so larger token groups are bound by shared-
// memory bandwidth rather than by the adapter stream.)
__host__ __device__ __forceinline__ int nt_class(int n) { return n <= 1 ? 1 : (n == 2 ? 2 : 4); }
__host__ __device__ __forceinline__ int nte_class(int n) { return n <= 1 ? 1 : (n == 2 ? 2 : 4); }
constexpr int kMaxPieces = 5;                 // pieces of a 2048-element row over >= 512-element pages

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
// try_wait blocks for a system-dependent time; the clock is read only every
// 64 attempts.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* err) {
  const uint32_t a = smem_u32(bar);
  long long t0 = -1;
  for (uint32_t it = 0;; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if ((it & 63) == 0) {
      const long long now = clock64();
      if (t0 < 0) t0 = now;
      else if (now - t0 > kWaitLimit) {
        record_error(err, 4, (int)blockIdx.x);
        return false;
      }
    }
  }
}

// Bounded wait until the shared counter *c reaches `target` (a count only ever
// grows, so unlike an mbarrier phase parity it cannot be misread however far
// behind the waiter is); false (and a recorded error) if it gives up.
__device__ __forceinline__ bool counter_wait(const int* c, int target, int32_t* err) {
  long long t0 = -1;
  for (uint32_t it = 0;; ++it) {
    int v;
    asm volatile("ld.volatile.shared.s32 %0, [%1];" : "=r"(v) : "r"(smem_u32(c)) : "memory");
    if (v >= target) return true;
    if ((it & 63) == 0) {
      const long long now = clock64();
      if (t0 < 0) t0 = now;
      else if (now - t0 > kWaitLimit) {
        record_error(err, 4, (int)blockIdx.x);
        return false;
      }
    }
    __nanosleep(32);
  }
}


__device__ __forceinline__ int ld_volatile_s32(const int* a) {
  int v;
  asm volatile("ld.volatile.shared.s32 %0, [%1];" : "=r"(v) : "r"(smem_u32(a)) : "memory");
  return v;
}
__device__ __forceinline__ void st_volatile_s32(int* a, int v) {
  asm volatile("st.volatile.shared.s32 [%0], %1;" ::"r"(smem_u32(a)), "r"(v) : "memory");
}


// Bulk async copy global -> shared, completion counted on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(const unsigned char* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// 16-bit -> fp32 for 8 packed elements, exact.  fp16 is widened by the
// mixed-precision FMA x * 1 + (-0) on the FMA pipe (the conversion unit is the
// scarce one on this part); bf16 is the upper half of an fp32.
__device__ __forceinline__ void h2x2f(uint32_t w, float& lo, float& hi) {
  asm("{.reg .f16 l, h, one;\n\t"
      "mov.b32 {l, h}, %2;\n\tmov.b16 one, 0x3C00;\n\t"
      "fma.rn.f32.f16 %0, l, one, 0f80000000;\n\tfma.rn.f32.f16 %1, h, one, 0f80000000;}"
      : "=f"(lo), "=f"(hi) : "r"(w));
}
template <int DT>
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (DT == SLORA_BF16) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    } else {
      h2x2f(w[i], f[2 * i], f[2 * i + 1]);
    }
  }
}

// acc + a.lo * b.lo + a.hi * b.hi for two packed 16-bit pairs, with the
// mixed-precision FMA (16-bit sources, fp32 accumulator, one rounding each):
// the same result as converting exactly and using fp32 FMAs, in order.
template <int DT>
__device__ __forceinline__ float fma2_16(uint32_t a, uint32_t b, float acc) {
  if (DT == SLORA_BF16)
    asm("{.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\tfma.rn.f32.bf16 %0, ah, bh, %0;}"
        : "+f"(acc) : "r"(a), "r"(b));
  else
    asm("{.reg .f16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.f16 %0, al, bl, %0;\n\tfma.rn.f32.f16 %0, ah, bh, %0;}"
        : "+f"(acc) : "r"(a), "r"(b));
  return acc;
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
__device__ __forceinline__ int block_exscan(int v, int* total, int* sh) {
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

// Exclusive block-wide prefix sums of four independent values at once; *tot
// gets the four totals.  sh: 32 int4 of shared memory.
__device__ __forceinline__ int4 block_exscan4(int4 v, int4* tot, int4* sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int4 x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y0 = __shfl_up_sync(FULL_MASK, x.x, o), y1 = __shfl_up_sync(FULL_MASK, x.y, o);
    const int y2 = __shfl_up_sync(FULL_MASK, x.z, o), y3 = __shfl_up_sync(FULL_MASK, x.w, o);
    if (lane >= o) x = make_int4(x.x + y0, x.y + y1, x.z + y2, x.w + y3);
  }
  int4 ex = make_int4(__shfl_up_sync(FULL_MASK, x.x, 1), __shfl_up_sync(FULL_MASK, x.y, 1),
                      __shfl_up_sync(FULL_MASK, x.z, 1), __shfl_up_sync(FULL_MASK, x.w, 1));
  if (lane == 0) ex = make_int4(0, 0, 0, 0);
  if (lane == 31) sh[w] = x;
  __syncthreads();
  if (w == 0) {
    int4 s = lane < nw ? sh[lane] : make_int4(0, 0, 0, 0);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y0 = __shfl_up_sync(FULL_MASK, s.x, o), y1 = __shfl_up_sync(FULL_MASK, s.y, o);
      const int y2 = __shfl_up_sync(FULL_MASK, s.z, o), y3 = __shfl_up_sync(FULL_MASK, s.w, o);
      if (lane >= o) s = make_int4(s.x + y0, s.y + y1, s.z + y2, s.w + y3);
    }
    sh[lane] = s;
  }
  __syncthreads();
  const int4 wp = w ? sh[w - 1] : make_int4(0, 0, 0, 0);
  *tot = sh[nw - 1];
  __syncthreads();
  return make_int4(wp.x + ex.x, wp.y + ex.y, wp.z + ex.z, wp.w + ex.w);
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


// Page id of flat element f of tensor (adapter a, page-list offset lo).
__device__ __forceinline__ int32_t page_id(const PoolDev& P, int a, int lo, int64_t f) {
  return __ldg(P.page_list + (int64_t)a * P.list_stride + lo + (f >> P.page_shift));
}
__device__ __forceinline__ const uint16_t* page_ptr(const PoolDev& P, int32_t pg, int64_t f) {
  return P.pool + ((int64_t)pg << P.page_shift) + (f & ((1ll << P.page_shift) - 1));
}


// A paged range [f0, f1) cut at page boundaries: piece q starts at f0 (q = 0)
// or at the q-th boundary after f0.
__device__ __forceinline__ bool piece_range(const PoolDev& P, int64_t f0, int64_t f1, int q, int64_t& b,
                                            int64_t& e) {
  const int64_t PE = 1ll << P.page_shift;
  const int64_t pb0 = ((f0 >> P.page_shift) + 1) << P.page_shift;
  b = q == 0 ? f0 : pb0 + (int64_t)(q - 1) * PE;
  e = pb0 + (int64_t)q * PE;
  if (e > f1) e = f1;
  return b < f1;
}

}  // namespace slora
