// slora_internal.h -- parameter blocks shared by the host runtime (runtime.cpp)
// and the CUDA kernels.  Not part of the public ABI (include/slora.h is).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/slora.h"

namespace slora {

// Shrink work split (decode path).  A task covers RW rank rows x NT tokens x
// KC elements of d_in; KC is fixed so every projection has a fixed number of
// fp32 partial slices (ceil(d_in / KC)).
constexpr int kShrinkKC = 512;
constexpr int kMaxSlots = SLORA_MAX_PROJ;   // projections per call
constexpr int kThreads = 256;               // threads per CTA of the decode kernels
constexpr int kEventRing = 64;

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
};

// One projection entry of a compute call.
struct SlotDev {
  const uint16_t* x;
  int64_t ldx;
  uint16_t* y;
  int64_t ldy;
  int d_in, d_out;
  int listA, listB;        // offsets of this projection's A_t / B page lists in an adapter row
  int nck;                 // shrink partial slices = ceil(d_in / kShrinkKC)
  int group;               // index of the x-sharing group
  int gpos;                // rank-row block of this slot inside its group
  float* tpart;            // [nck][max_tokens][max_rank], position-ordered
  float* tfin;             // final t: position-ordered [max_tokens][ldt] or token-ordered
  int64_t ldt;
  int t_by_token;          // 1: tfin row = token id; 0: row = position in perm order
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
  int32_t* meta;           // [16]: S, n_valid, shrink total, expand total, ctr total, work counters
  int32_t* shrink_prefix;  // [MS + 1] shrink tasks before each segment (segment-major)
  int32_t* expand_prefix;  // [MS + 1] expand tasks before each segment
  int32_t* ctr_prefix;     // [MS + 1] reduction counters before each segment
  int32_t* seg_rank;       // [MS] rank of each segment's adapter
  int32_t* ctr;            // reduction counters
  int64_t ctr_cap;
  int MS;                  // max segments = min(max_tokens, max_adapters)
};

enum MetaIdx { kMetaS = 0, kMetaValid = 1, kMetaShrinkTotal = 2, kMetaExpandTotal = 3,
               kMetaCtrTotal = 4, kMetaShrinkWork = 5, kMetaExpandWork = 6, kMetaCount = 16 };

struct BgmvParams {
  PoolDev pool;
  ScratchDev sc;
  int n_slots;
  SlotDev slot[kMaxSlots];
  int n_groups;
  GroupDev group[kMaxSlots];
  int max_tokens;
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
  const uint16_t* host[kMaxSlots][2];   // device-usable pointers to pinned host weights
};

// Launchers (kernels.cu).  All return cudaGetLastError() of the launch.
cudaError_t launch_segments(const BgmvParams& p, const int32_t* idx, int T, cudaStream_t s);
cudaError_t launch_shrink(const BgmvParams& p, int dtype, int grid, cudaStream_t s);
cudaError_t launch_expand(const BgmvParams& p, int dtype, int grid, cudaStream_t s);
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
