// GQA-path decode for many rows per group (m * s_q >= 64), bf16, on tcgen05.
//
// Grouped-query decode over the per-group expanded cache ("GQLA" chatpaper.ai
// Abstract: a GQA path with a per-group expanded cache; "Grouped Query
// Attention (GQA)" glossary, "Fonctionnement de la GQA").  With few groups
// and several new tokens per sequence a group serves hundreds of (query,
// head) rows, and the contraction becomes tensor-bound: this kernel runs it
// on the 5th-generation tensor cores with the rows as the MMA's M.
//
// One CTA per (key-range split, sequence, group, block of 128 rows):
//  * the 128 x 192 query tile is stored into TMEM once (the A operand of
//    the score MMAs), which leaves shared memory to two mbarrier rings of
//    64-token tiles (TMA, 2-D maps over the pools' token rows; a group's
//    chunks are column offsets) and two P tiles: K tiles (64 x 192) in 3
//    slots, each freed as soon as its score MMAs complete, and V tiles
//    (64 x 128) in 7 slots, each held until its PV MMAs complete.  A tile's
//    V lives about twice as long as its K (through the softmax), and with
//    one ring for both the slots' lifetime bounded the tile rate;
//  * warp 1 issues S = Q K^T (12 tcgen05.mma, M=128, N=64, K=16) into S[j % 2]
//    in TMEM; warp 6 issues O[j % 2] += P[j % 2] V (4 tcgen05.mma, M=128,
//    N=128, K=16, V as an MN-major operand);
//  * two softmax warpgroups take alternate tiles (warps 2-5 the even ones,
//    8-11 the odd ones), each with its own running maximum, sum and O
//    accumulator: the softmax of 128 rows x 64 tokens takes about twice the
//    tensor pipe's time for the tile, so one warpgroup would leave the pipe
//    idle half the time.  Within a group a thread owns one row: online
//    softmax in the log2 domain with lazy rescaling of its O (only when the
//    row maximum grows by more than 2^8), P to shared memory;
//  * at the end the even group merges the two states (the odd group's
//    maximum and sum through shared memory, both O halves straight from
//    TMEM) and writes the normalised output and the log-sum-exp.
#include <math.h>

#include "ptx.cuh"
#include "tc.h"

namespace gqla {

namespace {

constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr int kM = 128;                       // (query, head) rows per CTA
constexpr int kT = 64;                        // tokens per tile
constexpr int kKStages = 3, kVStages = 7;
constexpr int kKChunks = kDqk / 64;           // 3 K chunks of 64 dims
constexpr int kVChunks = kDv / 64;            // 2 V chunks
constexpr int kChunkBytes = kT * 128;         // 8 KB
constexpr int kKSlotBytes = kKChunks * kChunkBytes;   // 24 KB
constexpr int kVSlotBytes = kVChunks * kChunkBytes;   // 16 KB
constexpr int kPBytes = kM * 128;             // 128 rows x 64 tokens (bf16)
constexpr size_t kSmemBytes =
    (size_t)kKStages * kKSlotBytes + (size_t)kVStages * kVSlotBytes + 2 * kPBytes + 2 * kM * 4 + 1024;
constexpr uint32_t kTmemCols = 512;           // S: 2 x 64 at 0, O: 2 x 128 at 128, Q: 96 at 384
constexpr uint32_t kSCol = 0, kOCol = 128, kQCol = 384;
constexpr int kThreads = 12 * 32;
constexpr float kRescaleLog2 = 8.f;

struct WideParams {
  KvLayout ly;
  SplitPlan plan;
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  float* o_part;
  float* lse;
  int n_h, G, m, s_q;
  int rows_unit;      // m * s_q
  int rblocks;        // ceil(rows_unit / 128)
  KRow kr;            // K pool row layout
  float scale_log2;
  long long rows;     // B * s_q * n_h
  int32_t* st;
};

__global__ void __launch_bounds__(kThreads, 1)
    gqa_wide_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                    const WideParams p) {
  // launched while the kernel ahead of it may still run: wait for it before
  // any memory access, then let the next kernel launch
  ptx::pdl_wait();
  ptx::pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sK = smem;
  uint8_t* sV = sK + kKStages * kKSlotBytes;
  uint8_t* sP = sV + kVStages * kVSlotBytes;           // P[2]: one per softmax group
  float* sML = reinterpret_cast<float*>(sP + 2 * kPBytes);   // the odd group's row max and sum
  __shared__ __align__(8) uint64_t q_full, qk_drain, pv_drain;
  __shared__ __align__(8) uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages],
      s_full[2], s_free[2], p_full[2], pv_done[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the row blocks of one (sequence, group, split) are neighbours in the grid,
  // so they run together and read each K/V tile from HBM once, through L2
  const int split = blockIdx.x / p.rblocks, rb = blockIdx.x % p.rblocks;
  const int b = blockIdx.y / p.G, g = blockIdx.y % p.G;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&q_full, 4);
    ptx::mbar_init(&qk_drain, 1);
    ptx::mbar_init(&pv_drain, 1);
    for (int s = 0; s < kKStages; ++s) {
      ptx::mbar_init(&k_full[s], 1);
      ptx::mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      ptx::mbar_init(&v_full[s], 1);
      ptx::mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&s_full[s], 1);
      ptx::mbar_init(&s_free[s], 4);
      ptx::mbar_init(&p_full[s], 4);
      ptx::mbar_init(&pv_done[s], 1);
    }
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&tmem_base_sh, kTmemCols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  int L = seq_len_checked(p.ly, b, p.s_q, (split == 0 && g == 0 && rb == 0) ? p.st : nullptr);
  if (!seq_pages_ok(p.ly, b, L, p.st)) L = -1;   // includes a __syncthreads
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int t_begin = split * p.plan.chunk;
  const int t_stop = L < 0 ? t_begin : min(t_begin + p.plan.chunk, L);
  const int n_tiles = t_stop > t_begin ? (t_stop - t_begin + kT - 1) / kT : 0;

  if (warp == 0 || warp == 7) {
    // ---------------------------------------------------- TMA producers
    // One issuing thread brings about 27 bytes per cycle into an SM; the
    // tile needs more at the tensor pipe's pace, so warp 0 loads the K ring
    // and warp 7 the V ring.
    const bool kside = warp == 0;
    const int nst = kside ? kKStages : kVStages;
    uint64_t* full = kside ? k_full : v_full;
    uint64_t* empty = kside ? k_empty : v_empty;
    if (lane == 0 && n_tiles > 0) {
      ptx::prefetch_tmap(kside ? &kmap : &vmap);
      int issued = 0;
      // a tile's pool row (a page-table read when paged) is looked up one
      // tile ahead, so its latency overlaps the wait for the slot
      int row_next = (int)token_row(p.ly, b, t_begin, nullptr);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % nst, k = j / nst;
        const int row0 = row_next;
        if (j + 1 < n_tiles) row_next = (int)token_row(p.ly, b, t_begin + (j + 1) * kT, nullptr);
        if (k > 0 && !ptx::mbar_wait(&empty[s], (k - 1) & 1)) {
          flag_status(p.st, GQLA_DEV_TIMEOUT);
          atomicExch(&abort_flag, 1);
          break;
        }
        if (*(volatile int*)&abort_flag) break;
        if (kside) {
          uint8_t* dst = sK + s * kKSlotBytes;
          ptx::mbar_arrive_expect_tx(&full[s], kKSlotBytes);
          ptx::tma_load_2d(dst, &kmap, &full[s], p.kr.nope_at(g), row0);
          ptx::tma_load_2d(dst + kChunkBytes, &kmap, &full[s], p.kr.nope_at(g) + 64, row0);
          ptx::tma_load_2d(dst + 2 * kChunkBytes, &kmap, &full[s], p.kr.rope_at(g), row0);
        } else {
          uint8_t* dst = sV + s * kVSlotBytes;
          ptx::mbar_arrive_expect_tx(&full[s], kVSlotBytes);
          for (int c = 0; c < kVChunks; ++c)
            ptx::tma_load_2d(dst + c * kChunkBytes, &vmap, &full[s], g * kDv + 64 * c, row0);
        }
        issued = j + 1;
      }
      // no copy may be in flight when the CTA exits
      for (int j = issued > nst ? issued - nst : 0; j < issued; ++j) ptx::mbar_wait(&full[j % nst], (j / nst) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------- QK issuer, TMEM owner
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_qk = ptx::idesc_bf16(kM, kT, false, false);
      const uint32_t k_addr = ptx::smem_u32(sK);
      bool ok = ptx::mbar_wait(&q_full, 0);
      ptx::tc_fence_after();
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kKStages, sb = j & 1;
        ok = ptx::mbar_wait(&k_full[s], (j / kKStages) & 1);
        if (ok && j >= 2) ok = ptx::mbar_wait(&s_free[sb], ((j >> 1) - 1) & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint64_t bd0 = ptx::umma_desc_sw128(k_addr + s * kKSlotBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kDqk / 16; ++kk)
          ptx::umma_bf16_ts(tmem + kSCol + (uint32_t)kT * sb, tmem + kQCol + 8u * kk,
                            ptx::umma_desc_add(bd0, (kk >> 2) * kChunkBytes + (kk & 3) * 32), idesc_qk, kk > 0);
        ptx::umma_commit(&s_full[sb]);
        ptx::umma_commit(&k_empty[s]);            // the K slot is free once these MMAs complete
      }
      if (!ok) {
        flag_status(p.st, GQLA_DEV_TIMEOUT);
        atomicExch(&abort_flag, 1);
      }
      ptx::umma_commit(&qk_drain);
      ptx::mbar_wait(&qk_drain, 0);
    }
  } else if (warp == 6) {
    // ---------------------------------------------------------- PV issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_pv = ptx::idesc_bf16(kM, kDv, false, true);
      const uint32_t v_addr = ptx::smem_u32(sV);
      const uint64_t ad0 = ptx::umma_desc_sw128(ptx::smem_u32(sP), 16, 1024);
      bool ok = true;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kVStages, sb = j & 1;
        ok = ptx::mbar_wait(&p_full[sb], (j >> 1) & 1);
        if (ok) ok = ptx::mbar_wait(&v_full[s], (j / kVStages) & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint64_t bd0 = ptx::umma_desc_sw128(v_addr + s * kVSlotBytes, kChunkBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk)
          ptx::umma_bf16(tmem + kOCol + (uint32_t)kDv * sb, ptx::umma_desc_add(ad0, sb * kPBytes + kk * 32),
                         ptx::umma_desc_add(bd0, kk * 16 * 128), idesc_pv, (j >= 2 || kk > 0) ? 1u : 0u);
        ptx::umma_commit(&pv_done[sb]);
        ptx::umma_commit(&v_empty[s]);
      }
      if (!ok) {
        flag_status(p.st, GQLA_DEV_TIMEOUT);
        atomicExch(&abort_flag, 1);
      }
      ptx::umma_commit(&pv_drain);
      ptx::mbar_wait(&pv_drain, 0);
    }
  } else if (warp >= 2 && warp != 6 && warp != 7) {
    // ----------------------------------- softmax warpgroups and epilogue
    const int gp = warp >= 8 ? 1 : 0;           // this group's tiles: j % 2 == gp
    const int qd = warp & 3;
    const int row = 32 * qd + lane;             // M row = TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    const uint32_t o_col = kOCol + (uint32_t)kDv * gp;
    uint8_t* sPg = sP + gp * kPBytes;
    const int r_local = rb * kM + row;
    const bool in_range = r_local < p.rows_unit;
    const bool valid = in_range && L >= 0;
    const int i_q = in_range ? r_local / p.m : 0;
    const long long grow = in_range ? ((long long)b * p.s_q + i_q) * p.n_h + g * p.m + r_local % p.m : 0;
    const int vis = valid ? L - p.s_q + i_q + 1 : 0;
    if (gp == 0) {
      // this row's query into TMEM (lane = row, bf16 pairs; zeros for padding rows)
      for (int c = 0; c < kKChunks; ++c) {
        uint32_t v[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          uint4 w = make_uint4(0, 0, 0, 0);
          if (in_range) w = *reinterpret_cast<const uint4*>(p.q + grow * kDqk + 64 * c + 2 * e);
          v[e] = w.x;
          v[e + 1] = w.y;
          v[e + 2] = w.z;
          v[e + 3] = w.w;
        }
        ptx::tmem_st32(tl + kQCol + 32u * c, v);
      }
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&q_full);
    }

    float m_used = -INFINITY, l_sum = 0.f;
    bool ok = true;
    int last = -1;                               // this group's last tile
    for (int j = gp; j < n_tiles; j += 2) {
      const int t0 = t_begin + j * kT;
      last = j;
      if (ok) ok = ptx::mbar_wait(&s_full[gp], (j >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      // the row maximum over the tile's 64 scores, read in two halves; S[gp]
      // is next written for tile j + 2, this group's own next tile.  A tile
      // that every row of the CTA sees whole needs no mask, and the scale is
      // applied once to the extreme score (the largest for a positive scale,
      // the smallest for a negative one).
      const bool whole = __all_sync(0xffffffffu, !valid || t0 + kT <= vis);
      const float sgn = p.scale_log2 < 0.f ? -1.f : 1.f;
      float mx = -INFINITY;
      if (ok) {
        ptx::tc_fence_after();
        float raw = -INFINITY;                    // max of sgn * s over the visible tokens
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sv[32];
          ptx::tmem_ld32(tl + kSCol + (uint32_t)kT * gp + 32u * h, sv);
          ptx::tmem_ld_wait();
          if (whole && sgn > 0.f) {
#pragma unroll
            for (int t = 0; t < 32; ++t) raw = fmaxf(raw, __uint_as_float(sv[t]));
          } else if (whole) {
#pragma unroll
            for (int t = 0; t < 32; ++t) raw = fmaxf(raw, -__uint_as_float(sv[t]));
          } else {
#pragma unroll
            for (int t = 0; t < 32; ++t)
              if (t0 + 32 * h + t < vis) raw = fmaxf(raw, sgn * __uint_as_float(sv[t]));
          }
        }
        mx = (valid && raw != -INFINITY) ? raw * (sgn * p.scale_log2) : -INFINITY;
      }
      float factor = 1.f;
      int need = 0;
      if (m_used == -INFINITY) {
        m_used = mx;                              // this group's O holds only zeros so far
      } else if (mx > m_used + kRescaleLog2) {
        factor = ptx::fast_exp2(m_used - mx);
        need = 1;
        l_sum *= factor;
        m_used = mx;
      }
      const bool any_rescale = __any_sync(0xffffffffu, need) != 0;
      // this group's previous PV (tile j - 2) must be done before its O is
      // rescaled and its P overwritten
      if (ok && j >= 2) ok = ptx::mbar_wait(&pv_done[gp], ((j >> 1) - 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (ok && any_rescale) {
        ptx::tc_fence_after();
        for (int c = 0; c < kDv / 32; ++c) {
          uint32_t ov[32];
          ptx::tmem_ld32(tl + o_col + 32u * c, ov);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * factor);
          ptx::tmem_st32(tl + o_col + 32u * c, ov);
        }
        ptx::tmem_st_wait();
      }
      // P = 2^(s - m) in bf16, the two halves read again from TMEM
      float acc = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t sv[32];
        if (ok) {
          ptx::tmem_ld32(tl + kSCol + (uint32_t)kT * gp + 32u * h, sv);
          ptx::tmem_ld_wait();
        }
        if (h == 1) {
          // S[gp] is read for the last time: the next score MMAs may overwrite it
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&s_free[gp]);
        }
        // 2^(s * scale - m): one fused multiply-add per score; a whole tile
        // needs no per-score mask
        const float neg_m = -m_used;
        if (ok && whole && m_used != -INFINITY) {
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const float e = ptx::fast_exp2(fmaf(__uint_as_float(sv[t]), p.scale_log2, neg_m));
            sv[t] = __float_as_uint(e);
            acc += e;
          }
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const bool seen = ok && m_used != -INFINITY && t0 + 32 * h + t < vis;
            const float e = seen ? ptx::fast_exp2(fmaf(__uint_as_float(sv[t]), p.scale_log2, neg_m)) : 0.f;
            sv[t] = __float_as_uint(e);
            acc += e;
          }
        }
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          uint4 v;
          v.x = ptx::pack_bf16(__uint_as_float(sv[8 * g8 + 0]), __uint_as_float(sv[8 * g8 + 1]));
          v.y = ptx::pack_bf16(__uint_as_float(sv[8 * g8 + 2]), __uint_as_float(sv[8 * g8 + 3]));
          v.z = ptx::pack_bf16(__uint_as_float(sv[8 * g8 + 4]), __uint_as_float(sv[8 * g8 + 5]));
          v.w = ptx::pack_bf16(__uint_as_float(sv[8 * g8 + 6]), __uint_as_float(sv[8 * g8 + 7]));
          *reinterpret_cast<uint4*>(sPg + ptx::swz128(row, 4 * h + g8)) = v;
        }
      }
      l_sum += acc;
      if (t0 + kT > L) {
        // value rows past the sequence may hold anything: zero them for PV,
        // once the tile's V has landed (its slot cannot be refilled before
        // this group's P is delivered)
        const int sv = j % kVStages;
        bool vok = ok && ptx::mbar_wait(&v_full[sv], (j / kVStages) & 1);
        vok = __all_sync(0xffffffffu, vok);
        const int tid = 32 * qd + lane;
        for (int idx = tid; vok && idx < kT * kVChunks * 8; idx += 128) {
          const int tok = idx / (kVChunks * 8), rem = idx % (kVChunks * 8);
          if (t0 + tok >= L)
            *reinterpret_cast<uint4*>(sV + sv * kVSlotBytes + (rem / 8) * kChunkBytes + ptx::swz128(tok, rem % 8)) =
                make_uint4(0, 0, 0, 0);
        }
        ok = vok;
      }
      ptx::fence_proxy_async_smem();
      asm volatile("bar.sync %0, 128;" ::"r"(1 + gp) : "memory");   // the tail zeroing is shared by the group
      if (lane == 0) ptx::mbar_arrive(&p_full[gp]);
    }
    if (!ok && lane == 0) {
      flag_status(p.st, GQLA_DEV_TIMEOUT);
      atomicExch(&abort_flag, 1);
    }
    // ----------------------------------------------------------- epilogue
    bool have_o = ok && last >= 0 && ptx::mbar_wait(&pv_done[gp], (last >> 1) & 1);
    have_o = __all_sync(0xffffffffu, have_o);
    if (gp == 1) {
      sML[row] = have_o ? m_used : -INFINITY;
      sML[kM + row] = have_o ? l_sum : 0.f;
    }
    // both groups meet: the odd group's state is in shared memory and its O final
    asm volatile("bar.sync 3, 256;" ::: "memory");
    const bool ok1 = ok && *(volatile int*)&abort_flag == 0;   // a failed wait anywhere: write nothing
    if (gp == 0) {
      const float m1 = sML[row], l1 = sML[kM + row];
      const bool have1 = m1 != -INFINITY;
      const float m0 = have_o ? m_used : -INFINITY;
      const float mt = fmaxf(m0, m1);
      const float w0 = (m0 == -INFINITY) ? 0.f : ptx::fast_exp2(m0 - mt);
      const float w1 = have1 ? ptx::fast_exp2(m1 - mt) : 0.f;
      const float l = (have_o ? l_sum * w0 : 0.f) + (have1 ? l1 * w1 : 0.f);
      const bool empty = !(l > 0.f) || !ok1;
      const float inv = empty ? 0.f : 1.f / l;
      const float a0 = w0 * inv, a1 = w1 * inv;
      ptx::tc_fence_after();
      for (int c = 0; c < kDv / 32; ++c) {
        uint32_t o0[32], o1[32];
        if (have_o) {
          ptx::tmem_ld32(tl + kOCol + 32u * c, o0);
          ptx::tmem_ld_wait();
        }
        if (__any_sync(0xffffffffu, have1)) {
          ptx::tmem_ld32(tl + kOCol + (uint32_t)kDv + 32u * c, o1);
          ptx::tmem_ld_wait();
        }
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float x = have_o ? __uint_as_float(o0[e]) * a0 : 0.f;
          if (have1) x += __uint_as_float(o1[e]) * a1;   // select: an unused O half may hold anything
          v[e] = empty ? 0.f : x;
        }
        if (in_range && ok1) {
          if (p.o_part) {
            float* dst = p.o_part + ((long long)split * p.rows + grow) * kDv + 32 * c;
#pragma unroll
            for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
          } else {
            __nv_bfloat16* dst = p.out + grow * kDv + 32 * c;
#pragma unroll
            for (int e = 0; e < 32; e += 8)
              *reinterpret_cast<uint4*>(dst + e) =
                  make_uint4(ptx::pack_bf16(v[e], v[e + 1]), ptx::pack_bf16(v[e + 2], v[e + 3]),
                             ptx::pack_bf16(v[e + 4], v[e + 5]), ptx::pack_bf16(v[e + 6], v[e + 7]));
          }
        }
      }
      if (in_range && ok1 && p.lse) {
        const float lse = empty ? -INFINITY : (mt + log2f(l)) * 0.69314718055994531f;
        p.lse[p.o_part ? (long long)split * p.rows + grow : grow] = lse;
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool tc_gqa_wide_supports(const Problem& p) {
  const auto& d = p.d;
  if (d.dtype != GQLA_BF16 || p.d_qk != kDqk || d.d_v != kDv) return false;
  if (p.m * d.s_q < 64) return false;
  if (p.ly.page_size != 0 && p.ly.page_size % kT != 0) return false;
  if ((long long)p.ly.batch * d.G > 65535) return false;
  return true;
}

cudaError_t tc_gqa_wide_decode(const Problem& p, const void* q, const void* k_pool, const void* v_pool, void* out,
                               float* o_part, float* lse_dst, int32_t* st, cudaStream_t s) {
  const auto& d = p.d;
  CUtensorMap kmap, vmap;
  if (!gqa_pool_maps(p, k_pool, v_pool, &kmap, &vmap)) return cudaErrorInvalidValue;
  WideParams prm;
  prm.ly = p.ly;
  prm.plan = p.plan;
  prm.q = (const __nv_bfloat16*)q;
  prm.out = (__nv_bfloat16*)out;
  prm.o_part = o_part;
  prm.lse = lse_dst;
  prm.n_h = d.n_h;
  prm.G = d.G;
  prm.m = p.m;
  prm.s_q = d.s_q;
  prm.rows_unit = p.m * d.s_q;
  prm.rblocks = (prm.rows_unit + kM - 1) / kM;
  prm.scale_log2 = d.scale * 1.4426950408889634f;
  prm.rows = p.rows;
  prm.st = st;
  prm.kr = p.kr;
  cudaError_t e = ensure_smem_limit((const void*)gqa_wide_kernel, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.plan.num_splits * prm.rblocks, p.ly.batch * d.G);
  e = launch_pdl(gqa_wide_kernel, grid, dim3(kThreads), kSmemBytes, s, kmap, vmap, prm);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace gqla
