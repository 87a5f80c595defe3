// token.cu -- the decode delta for small batches: one CTA per token (sm_100a).
//
// For a batch of a few tokens the delta is bound by latency, not by bytes: a
// segment build, a copy ring and a hand-over between phases cost more than the
// few hundred kilobytes of weights.  Here CTA i computes, for token i and
// every projection of the call,
//     t_k = sum_j x[i, j] * A_a[j, k]            (shrink, fp32)
//     y[i, l] <- RN(y[i, l] + (alpha_a / r_a) * sum_k t_k * B_a[k, l])
// with plain coalesced 16-byte loads straight from the pages ("Paper
// explainer: S-LoRA", BGMV kernel section: the per-token loop with weights
// fetched from paged memory by adapter id; -1 = no adapter).  Tokens that
// share an adapter each read it (L2 serves the repeats); no scratch is used.
#include "dev_common.cuh"

namespace slora {

namespace {

constexpr int kTThreads = 512;  // 16 warps
constexpr int kTMaxR = 128;
constexpr int kTMaxList = 4096; // page-list entries staged in shared memory

template <int DT>
__global__ void __launch_bounds__(kTThreads) k_token(const __grid_constant__ BgmvParams p) {
  __shared__ float t_s[kMaxSlots][kTMaxR];
  __shared__ int32_t plist[kTMaxList];
  const int i = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a = p.idx[i];
  if (a == -1) return;
  if (a < -1 || a >= p.pool.max_adapters) {
    if (tid == 0) record_error(p.pool.err, 1, i);
    return;
  }
  // the rank, the scale and the adapter's page-list row in one round trip
  const int64_t row0 = (int64_t)a * p.pool.list_stride;
  const bool staged = p.pool.list_stride <= kTMaxList;
  if (staged)
    for (int e = tid; e < p.pool.list_stride; e += kTThreads) plist[e] = __ldg(p.pool.page_list + row0 + e);
  const int r = p.pool.rank[a];
  const float s_a = p.pool.scale[a];
  __syncthreads();
  if (r < 0) {
    if (tid == 0) record_error(p.pool.err, 2, i);
    return;
  }
  if (r == 0) return;
  const int32_t* list = staged ? plist : p.pool.page_list + row0;
  // every 128-byte line of B goes to L2 now, while the shrink runs (a line never
  // straddles a page: pages are a power of two of at least 512 elements)
  for (int k = 0; k < p.n_slots; ++k) {
    const SlotDev& L = p.slot[k];
    const int64_t n = (int64_t)r * L.d_out;
    for (int64_t f = (int64_t)tid * 64; f < n; f += kTThreads * 64)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(page_ptr(p.pool, list[L.listB + (f >> p.pool.page_shift)], f)));
  }
  // shrink: warp w takes the (slot, rank row) pairs w, w + 16, ...; lane l the
  // 8-element pieces l, l + 32, ... of the row; four chains per lane
  const int pairs = p.n_slots * r;
  for (int q = warp; q < pairs; q += kTThreads / 32) {
    const int k = q / r, kk = q % r;
    const SlotDev& L = p.slot[k];
    const uint16_t* x = L.x + (int64_t)i * L.ldx;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int c = 0;
#pragma unroll 4
    for (int j = lane * 8; j < L.d_in; j += 256, ++c) {
      const int64_t f = (int64_t)kk * L.d_in + j;
      const int32_t pg = list[L.listA + (f >> p.pool.page_shift)];
      const uint4 av = *reinterpret_cast<const uint4*>(page_ptr(p.pool, pg, f));
      const uint4 xv = *reinterpret_cast<const uint4*>(x + j);
      float s0 = acc[c & 3];
      s0 = fma2_16<DT>(av.x, xv.x, s0);
      s0 = fma2_16<DT>(av.y, xv.y, s0);
      s0 = fma2_16<DT>(av.z, xv.z, s0);
      s0 = fma2_16<DT>(av.w, xv.w, s0);
      acc[c & 3] = s0;
    }
    float v = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
    if (lane == 0) t_s[k][kk] = v;
  }
  __syncthreads();
  // expand: thread tid takes 8 consecutive outputs l = 8 tid + 2048 m of each slot
  for (int k = 0; k < p.n_slots; ++k) {
    const SlotDev& L = p.slot[k];
    uint16_t* y = L.y + (int64_t)i * L.ldy;
    for (int l = tid * 8; l < L.d_out; l += kTThreads * 8) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const uint4 yv = *reinterpret_cast<const uint4*>(y + l);
#pragma unroll 8
      for (int kk = 0; kk < r; ++kk) {
        const int64_t f = (int64_t)kk * L.d_out + l;
        const int32_t pg = list[L.listB + (f >> p.pool.page_shift)];
        float bf[8];
        unpack8<DT>(*reinterpret_cast<const uint4*>(page_ptr(p.pool, pg, f)), bf);
        const float tk = t_s[k][kk];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(tk, bf[e], acc[e]);
      }
      float yf[8];
      unpack8<DT>(yv, yf);
      uint4 o;
      o.x = pack2<DT>(fmaf(s_a, acc[0], yf[0]), fmaf(s_a, acc[1], yf[1]));
      o.y = pack2<DT>(fmaf(s_a, acc[2], yf[2]), fmaf(s_a, acc[3], yf[3]));
      o.z = pack2<DT>(fmaf(s_a, acc[4], yf[4]), fmaf(s_a, acc[5], yf[5]));
      o.w = pack2<DT>(fmaf(s_a, acc[6], yf[6]), fmaf(s_a, acc[7], yf[7]));
      *reinterpret_cast<uint4*>(y + l) = o;
    }
  }
}

}  // namespace

cudaError_t launch_token(const BgmvParams& p, int dtype, const int32_t* idx, int T, cudaStream_t s) {
  BgmvParams q = p;
  q.idx = idx;
  q.T = T;
  if (dtype == SLORA_BF16) k_token<SLORA_BF16><<<T, kTThreads, 0, s>>>(q);
  else k_token<SLORA_F16><<<T, kTThreads, 0, s>>>(q);
  return cudaGetLastError();
}

}  // namespace slora
