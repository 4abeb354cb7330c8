// Shared device helpers of the GQLA decode library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gqla.h"

namespace gqla {

// Kernel-side copy of gqla_kv_layout (passed by value).
struct KvLayout {
  const int32_t* seq_lens;
  const int32_t* block_table;
  int32_t batch;
  int32_t max_seq_len;
  int32_t page_size;   // 0 = contiguous
  int32_t capacity;
  int32_t mbps;        // max blocks per sequence
  int32_t num_pages;
};

// Split plan: split s of a sequence covers tokens [s*chunk, (s+1)*chunk).
struct SplitPlan {
  int32_t num_splits;
  int32_t chunk;
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ void flag_status(int32_t* st, int32_t bits) {
  if (st) atomicOr(st, bits);
}

// Checks sequence b against the layout and s_q.  Returns its length, or -1
// (after flagging) when its rows must be skipped.
__device__ __forceinline__ int seq_len_checked(const KvLayout& ly, int b, int s_q, int32_t* st) {
  int L = ly.seq_lens[b];
  if (L < s_q || L < 1) { flag_status(st, GQLA_DEV_SHORT_SEQ); return -1; }
  bool over = L > ly.max_seq_len;
  if (ly.page_size == 0) over |= L > ly.capacity;
  else over |= (L + ly.page_size - 1) / ly.page_size > ly.mbps;
  if (over) { flag_status(st, GQLA_DEV_OVERFLOW); return -1; }
  return L;
}

// Row layout of the expanded K pool (gqla_k_layout): elements per token row,
// and where group g's parts start in it: d_nope part at g * gs, RoPE part at
// rope + g * rope_gs (rope_gs = 0 when the RoPE key is stored once).
struct KRow {
  int pitch, gs, rope, rope_gs;
  __host__ __device__ int nope_at(int g) const { return g * gs; }
  __host__ __device__ int rope_at(int g) const { return rope + g * rope_gs; }
};

// Pool row of token (b, t); -1 (flagged) for a page id outside the pool.
__device__ __forceinline__ long long token_row(const KvLayout& ly, int b, int t, int32_t* st) {
  if (ly.page_size == 0) return (long long)b * ly.capacity + t;
  int page = ly.block_table[(long long)b * ly.mbps + t / ly.page_size];
  if (page < 0 || page >= ly.num_pages) { flag_status(st, GQLA_DEV_BAD_PAGE); return -1; }
  return (long long)page * ly.page_size + (t % ly.page_size);
}

// Block-wide check that every page of sequence b (length L) is inside the
// pool; all threads of the block must call it.  Flags GQLA_DEV_BAD_PAGE.
__device__ __forceinline__ bool seq_pages_ok(const KvLayout& ly, int b, int L, int32_t* st) {
  int bad = 0;
  if (ly.page_size > 0 && L > 0) {
    const int nb = (L + ly.page_size - 1) / ly.page_size;
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
      int page = ly.block_table[(long long)b * ly.mbps + i];
      bad |= (page < 0 || page >= ly.num_pages);
    }
  }
  bad = __syncthreads_or(bad);
  if (bad && threadIdx.x == 0) flag_status(st, GQLA_DEV_BAD_PAGE);
  return !bad;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace gqla
