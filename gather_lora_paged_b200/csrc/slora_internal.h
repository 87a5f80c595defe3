// slora_internal.h -- parameter blocks shared by the host runtime (runtime.cpp)
// and the CUDA kernels.  Not part of the public ABI (include/slora.h is).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/slora.h"

namespace slora {

// Shrink work split (decode path).  A shrink task covers a block of rank
// rows x NT tokens x kShrinkKT elements of d_in; it leaves one fp32 partial
// per kPartK (= kShrinkKT) slice of d_in, which the expand sums in index order.
constexpr int kShrinkKT = 2048;
constexpr int kPartK = 2048;
constexpr int kMaxSlots = SLORA_MAX_PROJ;   // projections per call
constexpr int kThreads = 256;               // threads per CTA of the decode kernels
constexpr int kEventRing = 64;

// One-kernel decode path (fused.cu): every CTA keeps the batch's token order
// and segment table in shared memory, which bounds the tokens per call; larger
// calls take the three-kernel path (bgmv.cu).
constexpr int kFMaxT = 1024;                // tokens per call
constexpr int kFSegCap = kFMaxT;            // segments per call (<= tokens)
// Ready counters of the fused path, one per (segment, x group), then a count
// of finished CTAs; all zero between calls (the last CTA of a call clears
// them).  They sit at the start of every scratch layout.
constexpr int kFReadyCap = kFSegCap * kMaxSlots;
constexpr size_t kFReadyBytes = 4 * (kFReadyCap + 64);

// Device view of the pool and its tables.
struct PoolDev {
  uint16_t* pool;          // page storage
  int page_shift;          // log2(page_elems)
  int max_adapters;
  int max_rank;
  int64_t list_stride;     // page-list entries per adapter
  int32_t* rank;           // [max_adapters], -1 = not resident
  float* scale;            // [max_adapters], alpha / rank
  int32_t* page_list;      // [max_adapters * list_stride]
  int32_t* err;            // [2]: first error code, its token
  float* qscale;           // e4m3 weights: [max_adapters][n_proj][A_t, B][max_rank] row scales
  int wfmt;                // slora_weight_format_t
  int n_proj;              // projections per adapter
};

// One projection entry of a compute call.
struct SlotDev {
  const uint16_t* x;
  int64_t ldx;
  uint16_t* y;
  int64_t ldy;
  int d_in, d_out;
  int listA, listB;        // offsets of this projection's A_t / B page lists in an adapter row
  int proj;                // the pool's projection index
  int nsplit;              // shrink partials = ceil(d_in / kPartK)
  int group;               // index of the x-sharing group
  int gpos;                // rank-row block of this slot inside its group
  // t (rank-r intermediate): element (row, k, c) at t[row * t_rs + k * t_ns + c],
  // summed over c < t_ns.  row = position in perm order, or the token id when
  // t_by_token (a caller's dense t, t_ns = 1).
  float* t;
  int64_t t_rs;
  int t_ns;
  int t_by_token;
  float* tout;             // slora_bgmv_shrink: reduced t per token (ldt_out), else NULL
  int64_t ldt_out;
};

struct GroupDev {
  int n;                   // slots in the group (share x and d_in)
  int slot[kMaxSlots];
  int d_in;
  const uint16_t* x;
  int64_t ldx;
};

// Scratch arrays of one compute call (all in the caller's dev_scratch).
struct ScratchDev {
  int32_t* perm;           // [max_tokens]
  int32_t* seg_start;      // [MS + 1]
  int32_t* seg_adapter;    // [MS]
  int32_t* meta;           // [16]: S, n_valid, shrink total, expand total
  int32_t* shrink_prefix;  // [MS + 1] shrink tasks before each segment (segment-major)
  int32_t* expand_prefix;  // [MS + 1] expand tasks before each segment
  int32_t* seg_rank;       // [MS] rank of each segment's adapter
  int32_t* ready;          // [kFReadyCap + 1] fused path: ready counters, then finished CTAs
  int MS;                  // max segments = min(max_tokens, max_adapters)
};

enum MetaIdx { kMetaS = 0, kMetaValid = 1, kMetaShrinkTotal = 2, kMetaExpandTotal = 3,
               kMetaShrinkClaim = 4, kMetaExpandClaim = 5,  // dynamic task counters
               kMetaCount = 16 };

struct BgmvParams {
  PoolDev pool;
  ScratchDev sc;
  int n_slots;
  SlotDev slot[kMaxSlots];
  int n_groups;
  GroupDev group[kMaxSlots];
  int max_tokens;
  const int32_t* idx;       // the call's adapter per token (set by launch_segments)
  int T;
  int do_shrink, do_expand; // which phases this call plans
};

// Page-in descriptor, written by the host into pinned staging memory and read
// by the page-in kernel through its device-mapped address.
struct PageInHeader {
  int32_t n_new;           // adapters to copy in
  int32_t n_evict;         // adapters whose table entries are cleared
  int32_t n_proj;
  int32_t copy_data;       // 0: tables only (the copy engine moves the data)
  int64_t list_stride;
  int64_t total_units;     // (adapter, tensor, page) copy units
  int64_t off_evict;       // byte offsets inside the descriptor
  int64_t off_new;
};
struct PageInNew {
  int32_t id;
  int32_t rank;
  float scale;
  int32_t n_units;         // pages of this adapter
  int64_t unit_base;       // prefix of units over previous adapters
  int64_t list_off;        // byte offset of its page-list row in the descriptor
  int64_t qs_off;          // byte offset of its e4m3 row scales ([proj][A_t, B][rank]), -1: none
  const uint16_t* host[kMaxSlots][2];   // device-usable pointers to pinned host weights
};

// Launchers (kernels.cu).  All return cudaGetLastError() of the launch.
// Also records idx and T in p, for the kernels launched after it.
cudaError_t launch_segments(BgmvParams& p, const int32_t* idx, int T, cudaStream_t s);
cudaError_t launch_shrink(const BgmvParams& p, int dtype, int grid, cudaStream_t s);
cudaError_t launch_expand(const BgmvParams& p, int dtype, int grid, cudaStream_t s);
cudaError_t launch_reduce_t(const BgmvParams& p, int T, cudaStream_t s);
// The one-kernel decode delta (fused.cu): T <= kFMaxT, both phases.
cudaError_t launch_fused(BgmvParams& p, int dtype, const int32_t* idx, int T, int grid, cudaStream_t s);
int fused_grid_bound(const BgmvParams& p, int T);  // CTAs worth launching for T tokens
// The decode delta as one kernel of streaming tasks (stream.cu): T <= kFMaxT,
// both phases; grid = SMs x stream_blocks_per_sm (any size works).
cudaError_t launch_stream(BgmvParams& p, int dtype, const int32_t* idx, int T, int grid, cudaStream_t s);
int stream_blocks_per_sm(int max_adapters);
// The small-batch decode delta (token.cu): one CTA per token, no scratch.
constexpr int kTokenMaxT = 16;
cudaError_t launch_token(const BgmvParams& p, int dtype, const int32_t* idx, int T, cudaStream_t s);
cudaError_t launch_merge_requests(const int32_t* req_start, const int32_t* req_adapter, int n,
                                  int32_t* seg_start, int32_t* seg_adapter, int32_t* S_out,
                                  cudaStream_t s);
cudaError_t launch_page_in(const PoolDev& pool, const int* d_in, const int* d_out,
                           const int* listA, const int* listB, const void* desc_dev,
                           int64_t total_units, int grid, cudaStream_t s);
cudaError_t launch_gather_debug(const PoolDev& pool, int id, int d, int list_off, int rank,
                                uint16_t* out_dev, cudaStream_t s);
int occupancy_blocks(int which);   // resident CTAs per SM of the decode kernels

}  // namespace slora
