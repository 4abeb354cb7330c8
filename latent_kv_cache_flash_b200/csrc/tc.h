// Tensor-core (bf16) kernels of the GQLA decode library.
#pragma once

#include "launch.h"

#include <cuda.h>

namespace gqla {

// Row-major [rows, cols] bf16 tensor map, 64-column x box_rows boxes, 128-byte
// swizzle (tmap.cu).  cols * 2 and row_pitch_elems * 2 must be multiples of 16.
bool tmap_bf16_sw128(CUtensorMap* map, const void* base, long long cols, long long rows, long long row_pitch_elems,
                     int box_rows);
// The expanded K and V pools as [pool row, row width] maps with 64 x 64 boxes;
// a group's d_nope / RoPE / V chunks sit at column offsets given by p.kr.
bool gqa_pool_maps(const Problem& p, const void* k_pool, const void* v_pool, CUtensorMap* kmap, CUtensorMap* vmap);

// GQA decode over the expanded cache: mma.sync bf16 tiles, cp.async.bulk
// staged K/V pages, online softmax per 16-row block.
bool tc_gqa_supports(const Problem& p);
// With split partials (o_part), a counter array of B * G * ceil(m s_q / 16)
// ints and few rows per group, the mma.sync kernel merges the splits itself
// into out_final / lse_final and sets *merged; otherwise the caller runs the
// combine.
cudaError_t tc_gqa_decode(const Problem& p, const void* q, const void* k_pool, const void* v_pool, void* out,
                          float* o_part, float* lse_dst, int32_t* st, cudaStream_t s, int* counters = nullptr,
                          void* out_final = nullptr, float* lse_final = nullptr, bool* merged = nullptr);

// GQA decode for m * s_q >= 64 rows per group: tcgen05/TMEM (tc_gqa_wide.cu);
// tc_gqa_decode hands such problems to it.
bool tc_gqa_wide_supports(const Problem& p);
cudaError_t tc_gqa_wide_decode(const Problem& p, const void* q, const void* k_pool, const void* v_pool, void* out,
                               float* o_part, float* lse_dst, int32_t* st, cudaStream_t s);

// MQA-absorb decode: absorbed query, latent attention on tcgen05/TMEM, combine,
// up-projection.
bool tc_absorb_supports(const Problem& p);
cudaError_t tc_absorb_decode(const Problem& p, const void* q, const void* latent, const void* W_uk,
                             const void* W_uv, void* out, float* lse, const Workspace& w, int32_t* st,
                             cudaStream_t s);

// Small GEMMs on mma.sync (tc_gemm.cu): absorbed queries (bf16 out), the
// fused split combine + up-projection of the absorb path.
bool gemm_absorb_q_supports(const Problem& p);
cudaError_t absorb_q_mma(const Problem& p, const void* q, const void* W_uk, __nv_bfloat16* qt, cudaStream_t s);
bool gemm_combine_up_supports(const Problem& p);
// The split merge of the latent output and the up-projection, one launch.
cudaError_t combine_up_mma(const Problem& p, int S, const float* o_part, const float* lse_part, const void* W_uv,
                           void* out, float* lse_out, cudaStream_t s);

// Cache expansion GEMM on tcgen05 (tc_expand.cu).
bool tc_expand_supports(const Problem& p);
// Expansion of a dense matrix of the B * s_q new token rows (row b * s_q + i
// is token seq_lens[b] - s_q + i), written to those tokens' pool rows.
cudaError_t tc_expand_dense(const Problem& p, const void* rows, void* k_pool, void* v_pool, const void* W_uk,
                            const void* W_uv, int32_t* st, cudaStream_t s);
cudaError_t tc_expand(const Problem& p, const void* latent, const void* W_uk, const void* W_uv, void* k_pool,
                      void* v_pool, int tail, int32_t* st, cudaStream_t s);

}  // namespace gqla
