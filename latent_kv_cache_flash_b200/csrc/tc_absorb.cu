// MQA-absorb decode on the 5th-generation tensor cores (tcgen05 + TMEM), bf16.
//
// The absorb path ("GQLA" chatpaper.ai Abstract: an MQA-absorb path identical
// to MLA's; "GQLA: Group-Query Latent Attention for Hardware-Adaptive
// Decoding", scholarbro.com, Abstract) lets every (query, head) row attend
// over the shared latent cache rows [c_KV ; k_rope] (576 elements) with the
// absorbed query [W_uk^g q_nope ; q_rope], and produces the latent output
// sum_t p_t c_t (512 elements), which the up-projection lifts by W_uv^g.
// All heads read the same cache row, so a tile of tokens serves up to 64
// (query, head) rows at once: a dense contraction for the tensor cores.
//
// One CTA per (key-range split, sequence, block of 64 rows):
//  * the absorbed-query tile (64 x 576) lives in TMEM and is the A operand of
//    the score MMAs, so shared memory holds a 3-stage ring of 64-token latent
//    tiles (72 KB each, TMA) next to the P tile;
//  * TMEM: with M = 64 an accumulator occupies 16 of every 32 lanes.  Lanes
//    0-15 of each quarter hold Q~ (columns 0..287, bf16 pairs) and the two S
//    buffers (288..415); lanes 16-31 hold the two 256-column halves of O;
//  * warp 1 owns the TMEM columns and issues S = Q~ C^T as 36 tcgen05.mma
//    (M=64, N=64, K=16, A from TMEM); warp 6 issues O += P C[:, :512] as 8
//    tcgen05.mma (M=64, N=256, A = P from shared memory, B = the same latent
//    tile as an MN-major operand), so a stage is released as soon as its PV
//    completes;
//  * warps 2-5 load Q~ into TMEM, then per tile read S with tcgen05.ld in the
//    16-lane shape (two threads per row, 32 tokens each, so all 128 threads
//    work), run the online softmax in the log2 domain with lazy rescaling (O
//    is rescaled only when a row maximum grows by more than 2^8, through the
//    same shape so the Q~/S lanes are never touched), write P (bf16) to shared
//    memory, and at the end stage O through shared memory to write the fp32
//    latent output and the log-sum-exp of the split;
//  * warps 0 and 7 load the latent tiles, five and four of a tile's nine
//    128-byte column chunks, onto the stage's barrier.
#include <math.h>

#include "ptx.cuh"
#include "tc.h"

namespace gqla {

cudaError_t absorb_q_bf16(const Problem& p, const void* q, const void* W_uk, __nv_bfloat16* qt, cudaStream_t s);

namespace {

constexpr int kR = 512;
constexpr int kDr = 64;
constexpr int kE = kR + kDr;                 // 576 latent row elements
constexpr int kM = 64;                       // (query, head) rows per CTA
constexpr int kTk = 64;                      // tokens per tile
constexpr int kStages = 3;
constexpr int kChunks = kE / 64;             // 128-byte column chunks of a row
constexpr int kKVChunk = kTk * 128;
constexpr int kStageBytes = kChunks * kKVChunk;      // 73728
constexpr int kPBytes = kM * 128;                    // 64 rows x 64 tokens (bf16)
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + kPBytes + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kQCols = kE / 2;                  // 288 columns of bf16 pairs
constexpr uint32_t kSCol = kQCols;                   // S buffers at 288 and 352
constexpr uint32_t kOLane = 16u << 16;               // O in lanes 16-31 of each quarter
constexpr int kOStride = kR + 4;                     // staging pitch (floats) for the output
constexpr int kThreads = 8 * 32;
constexpr float kRescaleLog2 = 8.f;

static_assert(kSCol + 2 * kTk <= kTmemCols, "Q~ and the S buffers must fit the low half-lanes");
static_assert((size_t)kM * kOStride * 4 <= (size_t)kStages * kStageBytes, "output staging fits the ring");

struct AbsorbParams {
  KvLayout ly;
  SplitPlan plan;
  const __nv_bfloat16* qt;  // absorbed queries [rows, 512]
  const __nv_bfloat16* q;   // queries [rows, d_nope + 64] (for q_rope)
  int d_nope;
  float* o_part;   // [S, rows, 512] normalised latent outputs of each split
  float* lse;      // [S, rows] their log-sum-exp
  int s_q;
  int rows_unit;   // n_h * s_q rows of one sequence
  int hblocks;     // ceil(rows_unit / 64)
  float scale_log2;
  long long rows;
  int32_t* st;
};

__global__ void __launch_bounds__(kThreads, 1)
    absorb_decode_kernel(const __grid_constant__ CUtensorMap kv_map, const AbsorbParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sKV = smem;
  uint8_t* sP = sKV + kStages * kStageBytes;
  __shared__ __align__(8) uint64_t q_full, p_full, pv_done, qk_drain, pv_drain;
  __shared__ __align__(8) uint64_t kv_full[kStages], kv_empty[kStages], s_full[2], s_free[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int b = blockIdx.y / p.hblocks, hb = blockIdx.y % p.hblocks;
  ptx::pdl_trigger();   // the merge may launch once every CTA of this grid has started

  if (threadIdx.x == 0) {
    ptx::mbar_init(&q_full, 4);
    ptx::mbar_init(&p_full, 4);
    ptx::mbar_init(&pv_done, 1);
    ptx::mbar_init(&qk_drain, 1);
    ptx::mbar_init(&pv_drain, 1);
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&kv_full[s], 2);
      ptx::mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&s_full[s], 1);
      ptx::mbar_init(&s_free[s], 4);
    }
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&tmem_base_sh, kTmemCols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  int L = seq_len_checked(p.ly, b, p.s_q, (split == 0 && hb == 0) ? p.st : nullptr);
  if (!seq_pages_ok(p.ly, b, L, p.st)) L = -1;   // includes a __syncthreads
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int t_begin = split * p.plan.chunk;
  const int t_stop = L < 0 ? t_begin : min(t_begin + p.plan.chunk, L);
  const int n_tiles = t_stop > t_begin ? (t_stop - t_begin + kTk - 1) / kTk : 0;
  const long long grow0 = (long long)b * p.rows_unit + (long long)hb * kM;

  if (warp == 0 || warp == 7) {
    // ------------------------------------------------------- TMA producers
    // One issuing thread brings at most about 27 bytes per cycle into the SM,
    // so a 72 KB tile took about 2.7k cycles to land, inside the loop through
    // the 3-stage ring; two threads (chunks 0-4 and 5-8) halve that.
    const int c_lo = warp == 0 ? 0 : 5, c_hi = warp == 0 ? 5 : kChunks;
    if (lane == 0 && n_tiles > 0) {
      ptx::prefetch_tmap(&kv_map);
      int issued = 0;
      // a tile's pool row (a page-table read when paged) is looked up one
      // tile ahead, so its latency overlaps the wait for the slot
      int row_next = (int)token_row(p.ly, b, t_begin, nullptr);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kStages, k = j / kStages;
        const int row0 = row_next;
        if (j + 1 < n_tiles) row_next = (int)token_row(p.ly, b, t_begin + (j + 1) * kTk, nullptr);
        if (k > 0 && !ptx::mbar_wait(&kv_empty[s], (k - 1) & 1)) {
          flag_status(p.st, GQLA_DEV_TIMEOUT);
          atomicExch(&abort_flag, 1);
          break;
        }
        if (*(volatile int*)&abort_flag) break;
        uint8_t* dst = sKV + s * kStageBytes;
        ptx::mbar_arrive_expect_tx(&kv_full[s], (c_hi - c_lo) * kKVChunk);
        for (int c = c_lo; c < c_hi; ++c) ptx::tma_load_2d(dst + c * kKVChunk, &kv_map, &kv_full[s], 64 * c, row0);
        issued = j + 1;
      }
      // no copy may still be landing in shared memory when the CTA retires
      for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
        ptx::mbar_wait(&kv_full[j % kStages], (j / kStages) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------- QK issuer, TMEM owner
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_qk = ptx::idesc_bf16(kM, kTk, false, false);
      const uint32_t kv_addr = ptx::smem_u32(sKV);
      bool ok = ptx::mbar_wait(&q_full, 0);
      ptx::tc_fence_after();
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kStages, sb = j & 1;
        ok = ptx::mbar_wait(&kv_full[s], (j / kStages) & 1);
        if (ok && j >= 2) ok = ptx::mbar_wait(&s_free[sb], ((j >> 1) - 1) & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + kSCol + (uint32_t)kTk * sb;
        const uint64_t bd0 = ptx::umma_desc_sw128(kv_addr + s * kStageBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kE / 16; ++kk)
          ptx::umma_bf16_ts(d, tmem + 8u * kk, ptx::umma_desc_add(bd0, (kk >> 2) * kKVChunk + (kk & 3) * 32),
                            idesc_qk, kk > 0);
        ptx::umma_commit(&s_full[sb]);
      }
      if (!ok) {
        flag_status(p.st, GQLA_DEV_TIMEOUT);
        atomicExch(&abort_flag, 1);
      }
      // every issued MMA has finished before TMEM is released
      ptx::umma_commit(&qk_drain);
      ptx::mbar_wait(&qk_drain, 0);
    }
  } else if (warp == 6) {
    // ---------------------------------------------------------- PV issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_pv = ptx::idesc_bf16(kM, 256, false, true);
      const uint32_t kv_addr = ptx::smem_u32(sKV);
      const uint64_t ad0 = ptx::umma_desc_sw128(ptx::smem_u32(sP), 16, 1024);
      bool ok = true;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kStages;
        ok = ptx::mbar_wait(&p_full, j & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint64_t bd0 = ptx::umma_desc_sw128(kv_addr + s * kStageBytes, kKVChunk, 1024);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int kk = 0; kk < kTk / 16; ++kk)
            ptx::umma_bf16(tmem + kOLane + 256u * h, ptx::umma_desc_add(ad0, kk * 32),
                           ptx::umma_desc_add(bd0, (4 * h) * kKVChunk + kk * 16 * 128), idesc_pv,
                           (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::umma_commit(&pv_done);
        ptx::umma_commit(&kv_empty[s]);
      }
      if (!ok) {
        flag_status(p.st, GQLA_DEV_TIMEOUT);
        atomicExch(&abort_flag, 1);
      }
      ptx::umma_commit(&pv_drain);
      ptx::mbar_wait(&pv_drain, 0);
    }
  } else {
    // ------------------------------------------- softmax + epilogue warps
    const int qd = warp & 3;                    // TMEM lane quarter of this warp
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    // S and O are read through the 16-lane TMEM shape: thread t holds row
    // 8 (t % 2) + t / 4 of the quarter and the columns of parity (t / 2) % 2,
    // so every row is shared by two threads (t and t ^ 2), 32 tokens each.
    const int o_dp = 8 * (lane & 1) + (lane >> 2);
    const int half = (lane >> 1) & 1;
    const int row = 16 * qd + o_dp;
    const int r_local = hb * kM + row;
    const bool in_range = r_local < p.rows_unit;   // rows past the sequence's heads are padding
    const bool valid = in_range && L >= 0;
    const int vis = valid ? L - p.s_q + r_local / (p.rows_unit / p.s_q) + 1 : 0;

    // Q~ = [q~ (512) ; q_rope (64)] of each row into TMEM (lanes 0-15, one
    // row per lane), as bf16 pairs; lanes 16-31 store zeros into the O
    // half-lanes, which the first PV overwrites.  q~ comes from the launch
    // ahead of this one, which may still be running (the latent loads above
    // do not depend on it).
    ptx::pdl_wait();
    {
      const int row_q = 16 * qd + (lane & 15);
      const bool load = lane < 16 && hb * kM + row_q < p.rows_unit && grow0 + row_q < p.rows;
      const long long grow = grow0 + row_q;
      for (int c = 0; c < (int)kQCols / 32; ++c) {
        uint32_t v[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int col = 32 * c + e;            // bf16-pair column = element pair
          uint4 w = make_uint4(0, 0, 0, 0);
          if (load) {
            if (col < kR / 2) w = *reinterpret_cast<const uint4*>(p.qt + grow * kR + 2 * col);
            else w = *reinterpret_cast<const uint4*>(p.q + grow * (p.d_nope + kDr) + p.d_nope + 2 * (col - kR / 2));
          }
          v[e] = w.x;
          v[e + 1] = w.y;
          v[e + 2] = w.z;
          v[e + 3] = w.w;
        }
        ptx::tmem_st32(tl + 32u * c, v);
      }
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&q_full);
    }

    float m_used = -INFINITY, l_sum = 0.f;
    bool ok = true;
    // After a failed (bounded) wait the warp stops waiting and only keeps the
    // per-tile barrier arrivals in step with the other three warps.
    for (int j = 0; j < n_tiles; ++j) {
      const int sb = j & 1, s = j % kStages;
      const int t0 = t_begin + j * kTk;
      if (ok) ok = ptx::mbar_wait(&s_full[sb], (j >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      uint32_t sv[kTk / 2];                      // tokens 2 v + half, v = 0..31
      if (ok) {
        ptx::tc_fence_after();
        ptx::tmem_ld16x64(tl + kSCol + (uint32_t)kTk * sb, sv);
        ptx::tmem_ld_wait();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s_free[sb]);
      float factor = 1.f;
      int need = 0;
      if (ok) {
        // A tile every row of the warp sees whole needs no mask; the scale is
        // applied once, to the extreme raw score (the largest for a positive
        // scale, the smallest for a negative one), and the exponent is one
        // fused multiply-add.
        const bool whole = __all_sync(0xffffffffu, !valid || t0 + kTk <= vis);
        const float sgn = p.scale_log2 < 0.f ? -1.f : 1.f;
        float raw = -INFINITY;                   // max of sgn * s over the visible tokens
        if (whole) {
#pragma unroll
          for (int v = 0; v < kTk / 2; ++v) raw = fmaxf(raw, sgn * __uint_as_float(sv[v]));
        } else {
#pragma unroll
          for (int v = 0; v < kTk / 2; ++v)
            if (t0 + 2 * v + half < vis) raw = fmaxf(raw, sgn * __uint_as_float(sv[v]));
        }
        raw = fmaxf(raw, __shfl_xor_sync(0xffffffffu, raw, 2));   // the row's other half
        const float mx = (valid && raw != -INFINITY) ? raw * (sgn * p.scale_log2) : -INFINITY;
        if (m_used == -INFINITY) {
          m_used = mx;                            // O holds only zeros so far
        } else if (mx > m_used + kRescaleLog2) {
          factor = ptx::fast_exp2(m_used - mx);
          need = 1;
          l_sum *= factor;
          m_used = mx;
        }
        const float neg_m = -m_used;
        float acc = 0.f;
#pragma unroll
        for (int v = 0; v < kTk / 2; ++v) {
          const bool seen = m_used != -INFINITY && (whole || t0 + 2 * v + half < vis);
          const float e = seen ? ptx::fast_exp2(fmaf(__uint_as_float(sv[v]), p.scale_log2, neg_m)) : 0.f;
          sv[v] = __float_as_uint(e);
          acc += e;
        }
        l_sum += acc;                            // this thread's half of the row sum
      } else {
#pragma unroll
        for (int v = 0; v < kTk / 2; ++v) sv[v] = 0u;
      }
      const float f_row = factor;                // O rows use the same thread mapping
      const bool any_rescale = __any_sync(0xffffffffu, need) != 0;
      // PV(j-1) must be done before O is rescaled and before P is overwritten
      if (ok && j >= 1) ok = ptx::mbar_wait(&pv_done, (j - 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (ok && any_rescale) {
        ptx::tc_fence_after();
        for (int c = 0; c < kR / 64; ++c) {
          uint32_t ov[32];
          ptx::tmem_ld16x64(tl + kOLane + 64u * c, ov);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f_row);
          ptx::tmem_st16x64(tl + kOLane + 64u * c, ov);
        }
        ptx::tmem_st_wait();
      }
      if (t0 + kTk > L) {
        // latent rows past the sequence may hold anything: zero them for PV
        const int tid = threadIdx.x - 64;
        for (int idx = tid; idx < kTk * 8 * 8; idx += 128) {
          const int tok = idx >> 6, rem = idx & 63;
          if (t0 + tok >= L)
            *reinterpret_cast<uint4*>(sKV + s * kStageBytes + (rem >> 3) * kKVChunk + ptx::swz128(tok, rem & 7)) =
                make_uint4(0, 0, 0, 0);
        }
      }
      {
        // P row: the half == 0 thread writes tokens 0..31, its partner 32..63;
        // each trades the 16 values the other one needs (one shuffle each)
        uint32_t pk[kTk / 4];                    // bf16 pairs of tokens 32 half + 2 i, + 1
#pragma unroll
        for (int i = 0; i < kTk / 4; ++i) {
          const uint32_t send = half ? sv[i] : sv[kTk / 4 + i];
          const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 2);
          pk[i] = half ? ptx::pack_bf16(__uint_as_float(recv), __uint_as_float(sv[kTk / 4 + i]))
                       : ptx::pack_bf16(__uint_as_float(sv[i]), __uint_as_float(recv));
        }
#pragma unroll
        for (int g = 0; g < kTk / 16; ++g)
          *reinterpret_cast<uint4*>(sP + ptx::swz128(row, 4 * half + g)) =
              make_uint4(pk[4 * g], pk[4 * g + 1], pk[4 * g + 2], pk[4 * g + 3]);
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      asm volatile("bar.sync 1, 128;" ::: "memory");   // tail zeroing is shared by the four warps
      if (lane == 0) ptx::mbar_arrive(&p_full);
    }
    if (!ok && lane == 0) {
      flag_status(p.st, GQLA_DEV_TIMEOUT);
      atomicExch(&abort_flag, 1);
    }
    // ----------------------------------------------------------- epilogue
    bool have_o = ok && n_tiles > 0 && ptx::mbar_wait(&pv_done, (n_tiles - 1) & 1);
    have_o = __all_sync(0xffffffffu, have_o);
    // the whole ring is idle now (every load was consumed): stage O there
    asm volatile("bar.sync 1, 128;" ::: "memory");
    float* stage = reinterpret_cast<float*>(sKV);
    const float l_row = l_sum + __shfl_xor_sync(0xffffffffu, l_sum, 2);
    const float inv_o = (l_row > 0.f && have_o) ? 1.f / l_row : 0.f;
    if (have_o) {
      ptx::tc_fence_after();
      const int orow = row, par = half;
      for (int c = 0; c < kR / 64; ++c) {
        uint32_t ov[32];
        ptx::tmem_ld16x64(tl + kOLane + 64u * c, ov);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) stage[orow * kOStride + 64 * c + par + 2 * e] = __uint_as_float(ov[e]) * inv_o;
      }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int tid = threadIdx.x - 64;
    for (int idx = tid; idx < kM * (kR / 4); idx += 128) {
      const int rr = idx / (kR / 4), c4 = (idx % (kR / 4)) * 4;
      if (hb * kM + rr >= p.rows_unit || !ok) continue;
      const long long grow = grow0 + rr;
      float4 v = have_o ? *reinterpret_cast<const float4*>(stage + rr * kOStride + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(p.o_part + ((long long)split * p.rows + grow) * kR + c4) = v;
    }
    if (in_range && ok && half == 0) {
      const bool empty = !(l_row > 0.f) || !have_o;
      const float lse = empty ? -INFINITY : (m_used + log2f(l_row)) * 0.69314718055994531f;
      p.lse[(long long)split * p.rows + grow0 + row] = lse;
    }
  }
  // ------------------------------------------------------------ teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool tc_absorb_supports(const Problem& p) {
  const auto& d = p.d;
  if (d.dtype != GQLA_BF16) return false;
  if (d.r != kR || d.d_rope != kDr || d.d_nope % 8 != 0) return false;
  if (p.ly.page_size != 0 && p.ly.page_size % kTk != 0) return false;
  const long long hblocks = ((long long)d.n_h * d.s_q + kM - 1) / kM;
  if ((long long)p.ly.batch * hblocks > 65535) return false;
  if (p.rows + kM > (1LL << 31)) return false;
  return true;
}

cudaError_t tc_absorb_decode(const Problem& p, const void* q, const void* latent, const void* W_uk,
                             const void* W_uv, void* out, float* lse, const Workspace& w, int32_t* st,
                             cudaStream_t s) {
  const auto& d = p.d;
  const int S = p.plan.num_splits;
  cudaError_t e = gemm_absorb_q_supports(p) ? absorb_q_mma(p, q, W_uk, (__nv_bfloat16*)w.qt, s)
                                            : absorb_q_bf16(p, q, W_uk, (__nv_bfloat16*)w.qt, s);
  if (e != cudaSuccess) return e;
  long long nrows = p.ly.page_size == 0 ? (long long)p.ly.batch * p.ly.capacity
                                        : (long long)p.ly.num_pages * p.ly.page_size;
  CUtensorMap kv_map;
  if (!tmap_bf16_sw128(&kv_map, latent, kE, nrows, kE, kTk)) return cudaErrorInvalidValue;
  AbsorbParams prm;
  prm.ly = p.ly;
  prm.plan = p.plan;
  prm.qt = (const __nv_bfloat16*)w.qt;
  prm.q = (const __nv_bfloat16*)q;
  prm.d_nope = d.d_nope;
  prm.o_part = w.o_part;
  prm.lse = w.lse_part;
  prm.s_q = d.s_q;
  prm.rows_unit = d.n_h * d.s_q;
  prm.hblocks = (prm.rows_unit + kM - 1) / kM;
  prm.scale_log2 = d.scale * 1.4426950408889634f;
  prm.rows = p.rows;
  prm.st = st;
  e = ensure_smem_limit((const void*)absorb_decode_kernel, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(S, p.ly.batch * prm.hblocks);
  e = launch_pdl(absorb_decode_kernel, grid, dim3(kThreads), kSmemBytes, s, kv_map, prm);
  count_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (gemm_combine_up_supports(p))
    return combine_up_mma(p, S, w.o_part, w.lse_part, W_uv, out, lse, s);
  e = combine(S, p.rows, kR, w.o_part, w.lse_part, w.o_lat, GQLA_F32, lse, s);
  if (e != cudaSuccess) return e;
  return simt_up_proj(p, w.o_lat, W_uv, out, s);
}

}  // namespace gqla
