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
//  * warp 0 loads the absorbed-query tile once (64 x 576, 72 KB) and streams
//    64-token latent tiles (72 KB) with TMA into a 2-stage mbarrier ring;
//  * warps 1 and 7 issue S = Q~ C^T as 36 tcgen05.mma (M=64, N=64, K=16),
//    split along K into two double-buffered S halves in TMEM (one issuing
//    thread cannot keep up with such small MMAs); warp 1 owns the 512 TMEM
//    columns; warp 6 issues
//    O += P C[:, :512] as 8 tcgen05.mma (M=64, N=256, K=16), reading the same
//    latent tile as an MN-major B operand.  Two issuing threads keep the
//    stage release (after PV) independent of the next tile's QK issue;
//  * the M=64 accumulator uses 16 of every 32 TMEM lanes, so the two 256-wide
//    halves of O sit interleaved at lane offsets 0 and 16 of the same 256
//    columns; the S halves and buffers take columns 256..511;
//  * warps 2-5 read S rows from TMEM, run the online softmax in the log2
//    domain with lazy rescaling (O is only rescaled when a row max grows by
//    more than 2^8), write P (bf16) to shared memory, and in the end scale O
//    by 1/l and store the fp32 latent output and the log-sum-exp.
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
constexpr int kStages = 2;
constexpr int kChunks = kE / 64;             // 128-byte column chunks of a row
constexpr int kQChunk = kM * 128;
constexpr int kKVChunk = kTk * 128;
constexpr int kQBytes = kChunks * kQChunk;           // 73728
constexpr int kStageBytes = kChunks * kKVChunk;      // 36864
constexpr int kPBytes = kM * 128;                    // 64 rows x 64 tokens (bf16)
constexpr size_t kSmemBytes = (size_t)kQBytes + (size_t)kStages * kStageBytes + kPBytes + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 256;                  // S buffers: [half a|b][buffer 0|1] x kTk columns
constexpr int kQkSplit = 18;                     // k-steps (of 36) issued by the first QK warp
constexpr int kThreads = 8 * 32;
constexpr float kRescaleLog2 = 8.f;

struct AbsorbParams {
  KvLayout ly;
  SplitPlan plan;
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
    absorb_decode_kernel(const __grid_constant__ CUtensorMap qt_map, const __grid_constant__ CUtensorMap qr_map,
                         const __grid_constant__ CUtensorMap kv_map, const AbsorbParams p, int d_nope) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kQBytes;
  uint8_t* sP = sKV + kStages * kStageBytes;
  __shared__ __align__(8) uint64_t q_full, p_full, pv_done, qk_drain[2], pv_drain;
  __shared__ __align__(8) uint64_t kv_full[kStages], kv_empty[kStages], s_full[2], s_free[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int b = blockIdx.y / p.hblocks, hb = blockIdx.y % p.hblocks;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&q_full, 1);
    ptx::mbar_init(&p_full, 4);
    ptx::mbar_init(&pv_done, 1);
    ptx::mbar_init(&qk_drain[0], 1);
    ptx::mbar_init(&qk_drain[1], 1);
    ptx::mbar_init(&pv_drain, 1);
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&kv_full[s], 1);
      ptx::mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&s_full[s], 2);   // one commit from each QK issuer
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

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0 && n_tiles > 0) {
      ptx::prefetch_tmap(&qt_map);
      ptx::prefetch_tmap(&qr_map);
      ptx::prefetch_tmap(&kv_map);
      ptx::mbar_arrive_expect_tx(&q_full, kQBytes);
      for (int c = 0; c < kR / 64; ++c) ptx::tma_load_2d(sQ + c * kQChunk, &qt_map, &q_full, 64 * c, (int)grow0);
      ptx::tma_load_2d(sQ + (kR / 64) * kQChunk, &qr_map, &q_full, d_nope, (int)grow0);
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kStages, k = j / kStages;
        if (k > 0 && !ptx::mbar_wait(&kv_empty[s], (k - 1) & 1)) {
          flag_status(p.st, GQLA_DEV_TIMEOUT);
          atomicExch(&abort_flag, 1);
          break;
        }
        if (*(volatile int*)&abort_flag) break;
        const int row0 = (int)token_row(p.ly, b, t_begin + j * kTk, nullptr);
        uint8_t* dst = sKV + s * kStageBytes;
        ptx::mbar_arrive_expect_tx(&kv_full[s], kStageBytes);
        for (int c = 0; c < kChunks; ++c) ptx::tma_load_2d(dst + c * kKVChunk, &kv_map, &kv_full[s], 64 * c, row0);
        issued = j + 1;
      }
      // no copy may still be landing in shared memory when the CTA retires
      ptx::mbar_wait(&q_full, 0);
      for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
        ptx::mbar_wait(&kv_full[j % kStages], (j / kStages) & 1);
    }
  } else if (warp == 1 || warp == 7) {
    // ------------------------------------------------------- QK issuers
    // One tcgen05.mma costs its issuing thread about as much time as a small
    // (N=64) MMA takes to run, so two warps issue the 36 QK k-steps: warp 1
    // k-steps [0, kQkSplit) into S half a, warp 7 the rest into S half b; the
    // softmax adds the halves.  Warp 1 also owns the TMEM allocation.
    const int half_q = warp == 7 ? 1 : 0;
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_qk = ptx::idesc_bf16(kM, kTk, false, false);
      const uint32_t q_addr = ptx::smem_u32(sQ), kv_addr = ptx::smem_u32(sKV);
      const int k_lo = half_q ? kQkSplit : 0, k_hi = half_q ? kE / 16 : kQkSplit;
      bool ok = ptx::mbar_wait(&q_full, 0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kStages, sb = j & 1;
        ok = ptx::mbar_wait(&kv_full[s], (j / kStages) & 1);
        if (ok && j >= 2) ok = ptx::mbar_wait(&s_free[sb], ((j >> 1) - 1) & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + kSCol + (uint32_t)kTk * (2 * half_q + sb);
        const uint32_t st_addr = kv_addr + s * kStageBytes;
        for (int kk = k_lo; kk < k_hi; ++kk) {
          const uint32_t koff = (kk >> 2), kin = (kk & 3) * 32;
          const uint64_t a = ptx::umma_desc_sw128(q_addr + koff * kQChunk + kin, 16, 1024);
          const uint64_t bd = ptx::umma_desc_sw128(st_addr + koff * kKVChunk + kin, 16, 1024);
          ptx::umma_bf16(d, a, bd, idesc_qk, kk > k_lo);
        }
        ptx::umma_commit(&s_full[sb]);
      }
      if (!ok) {
        flag_status(p.st, GQLA_DEV_TIMEOUT);
        atomicExch(&abort_flag, 1);
      }
      // every issued MMA has finished before TMEM is released
      ptx::umma_commit(&qk_drain[half_q]);
      ptx::mbar_wait(&qk_drain[half_q], 0);
    }
  } else if (warp == 6) {
    // ---------------------------------------------------------- PV issuer
    // A second issuing thread: PV(j) goes out as soon as P(j) is ready, so
    // the stage it releases is not held behind the next tile's QK.
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_pv = ptx::idesc_bf16(kM, 256, false, true);
      const uint32_t kv_addr = ptx::smem_u32(sKV), p_addr = ptx::smem_u32(sP);
      bool ok = true;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kStages;
        ok = ptx::mbar_wait(&p_full, j & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t st_addr = kv_addr + s * kStageBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int kk = 0; kk < kTk / 16; ++kk) {
            const uint64_t a = ptx::umma_desc_sw128(p_addr + kk * 32, 16, 1024);
            const uint64_t bd = ptx::umma_desc_sw128(st_addr + (4 * h) * kKVChunk + kk * 16 * 128, kKVChunk, 1024);
            ptx::umma_bf16(tmem + (h ? (16u << 16) : 0u), a, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
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
    const int row = 16 * qd + (lane & 15);      // M-row (query, head) index
    const int half = lane >> 4;                 // 0: O columns 0..255, 1: 256..511
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    const int r_local = hb * kM + row;
    const bool in_range = r_local < p.rows_unit;   // rows past the sequence's heads are padding
    const bool valid = in_range && L >= 0;
    const int vis = valid ? L - p.s_q + r_local / (p.rows_unit / p.s_q) + 1 : 0;
    float m_used = -INFINITY, l_sum = 0.f;
    bool ok = true;
    // After a failed (bounded) wait the warp stops waiting and only keeps the
    // per-tile barrier arrivals in step with the other three warps.
    for (int j = 0; j < n_tiles; ++j) {
      const int sb = j & 1, s = j % kStages;
      const int t0 = t_begin + j * kTk;
      if (ok) ok = ptx::mbar_wait(&s_full[sb], (j >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      uint32_t sv[kTk];
      if (ok) {
        ptx::tc_fence_after();
        uint32_t sb2[32];
        ptx::tmem_ld32(tl + kSCol + (uint32_t)kTk * sb, sv);
        ptx::tmem_ld32(tl + kSCol + (uint32_t)kTk * sb + 32u, sv + 32);
        ptx::tmem_ld32(tl + kSCol + (uint32_t)kTk * (2 + sb), sb2);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t) sv[t] = __float_as_uint(__uint_as_float(sv[t]) + __uint_as_float(sb2[t]));
        ptx::tmem_ld32(tl + kSCol + (uint32_t)kTk * (2 + sb) + 32u, sb2);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t)
          sv[32 + t] = __float_as_uint(__uint_as_float(sv[32 + t]) + __uint_as_float(sb2[t]));
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s_free[sb]);
      float pv[kTk];
      float factor = 1.f;
      int need = 0;
      if (half == 0 && ok) {
        float mx = -INFINITY;
#pragma unroll
        for (int t = 0; t < kTk; ++t) {
          const float x = (t0 + t < vis) ? __uint_as_float(sv[t]) * p.scale_log2 : -INFINITY;
          pv[t] = x;
          mx = fmaxf(mx, x);
        }
        if (m_used == -INFINITY) {
          m_used = mx;                            // O holds only zeros so far
        } else if (mx > m_used + kRescaleLog2) {
          factor = ptx::fast_exp2(m_used - mx);
          need = 1;
          l_sum *= factor;
          m_used = mx;
        }
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < kTk; ++t) {
          const float e = m_used == -INFINITY ? 0.f : ptx::fast_exp2(pv[t] - m_used);
          pv[t] = e;
          acc += e;
        }
        l_sum += acc;
      } else {
#pragma unroll
        for (int t = 0; t < kTk; ++t) pv[t] = 0.f;
      }
      const float f_row = __shfl_sync(0xffffffffu, factor, lane & 15);
      const bool any_rescale = __any_sync(0xffffffffu, need) != 0;
      // PV(j-1) must be done before O is rescaled and before P is overwritten
      if (ok && j >= 1) ok = ptx::mbar_wait(&pv_done, (j - 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (ok && any_rescale) {
        ptx::tc_fence_after();
        for (int c = 0; c < 8; ++c) {
          uint32_t ov[32];
          ptx::tmem_ld32(tl + 32u * c, ov);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f_row);
          ptx::tmem_st32(tl + 32u * c, ov);
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
      if (half == 0) {
#pragma unroll
        for (int g8 = 0; g8 < kTk / 8; ++g8) {
          uint4 v;
          v.x = ptx::pack_bf16(pv[8 * g8 + 0], pv[8 * g8 + 1]);
          v.y = ptx::pack_bf16(pv[8 * g8 + 2], pv[8 * g8 + 3]);
          v.z = ptx::pack_bf16(pv[8 * g8 + 4], pv[8 * g8 + 5]);
          v.w = ptx::pack_bf16(pv[8 * g8 + 6], pv[8 * g8 + 7]);
          *reinterpret_cast<uint4*>(sP + ptx::swz128(row, g8)) = v;
        }
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
    ptx::tc_fence_after();
    const float l_tot = __shfl_sync(0xffffffffu, l_sum, lane & 15);
    const float m_tot = __shfl_sync(0xffffffffu, m_used, lane & 15);
    const bool empty = !(l_tot > 0.f) || !have_o;
    const float inv = empty ? 0.f : 1.f / l_tot;
    const long long grow = grow0 + row;
    float* dst = nullptr;
    if (in_range && ok) dst = p.o_part + ((long long)split * p.rows + grow) * kR + half * 256;
    for (int c = 0; c < 8; ++c) {
      uint32_t ov[32];
      if (have_o) {
        ptx::tmem_ld32(tl + 32u * c, ov);
        ptx::tmem_ld_wait();
      }
      if (dst) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float4 v = empty ? make_float4(0.f, 0.f, 0.f, 0.f)
                           : make_float4(__uint_as_float(ov[e]) * inv, __uint_as_float(ov[e + 1]) * inv,
                                         __uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
          *reinterpret_cast<float4*>(dst + 32 * c + e) = v;
        }
      }
    }
    if (in_range && ok && half == 0) {
      const float lse = empty ? -INFINITY : (m_tot + log2f(l_tot)) * 0.69314718055994531f;
      p.lse[(long long)split * p.rows + grow] = lse;
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)f;
  }
  return fn;
}

// Row-major [rows, cols] bf16 matrix, boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool make_2d_map(CUtensorMap* map, const void* base, long long cols, long long rows, long long row_pitch_elems,
                 int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)row_pitch_elems * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
  CUtensorMap qt_map, qr_map, kv_map;
  if (!make_2d_map(&qt_map, w.qt, kR, p.rows, kR, kM) || !make_2d_map(&qr_map, q, p.d_qk, p.rows, p.d_qk, kM) ||
      !make_2d_map(&kv_map, latent, kE, nrows, kE, kTk))
    return cudaErrorInvalidValue;
  AbsorbParams prm;
  prm.ly = p.ly;
  prm.plan = p.plan;
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
  absorb_decode_kernel<<<grid, kThreads, kSmemBytes, s>>>(qt_map, qr_map, kv_map, prm, d.d_nope);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (gemm_combine_up_supports(p))
    return combine_up_mma(p, S, w.o_part, w.lse_part, W_uv, out, lse, (__nv_bfloat16*)w.o_lat, s);
  e = combine(S, p.rows, kR, w.o_part, w.lse_part, w.o_lat, GQLA_F32, lse, s);
  if (e != cudaSuccess) return e;
  return simt_up_proj(p, w.o_lat, W_uv, out, s);
}

}  // namespace gqla
