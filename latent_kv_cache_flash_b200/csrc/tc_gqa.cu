// GQA-path decode over the per-group expanded cache, bf16, on sm_100a.
//
// Grouped-query decode ("GQLA" chatpaper.ai Abstract: a GQA path with a
// per-group expanded cache; "Grouped Query Attention (GQA)" glossary,
// "Fonctionnement de la GQA": every query head of group g attends over the
// group's single K/V head).  Decode at m*s_q <= 16 rows per group is a
// bandwidth-bound stream of the K/V pages (640 bytes per group-token at
// d_qk = 192, d_v = 128), so the kernel is built around moving those bytes:
//
//  * one CTA per (key-range split, sequence, group[, 64-row block]);
//  * a producer warp streams 64-token K and V tiles with TMA (2-D tensor maps
//    over the pools' token rows, 128-byte swizzle; the group's chunks are
//    column offsets, so a RoPE key stored once per row is read from there)
//    into a 2-stage mbarrier ring; two CTAs fit on an SM;
//  * four consumer warps each take 16 tokens of a tile (or, for more than 16
//    rows, one 16-row block each), compute S = Q K^T and O += P V with
//    mma.sync m16n8k16 bf16 (fp32 accumulate) from ldmatrix'd fragments, and
//    keep an online softmax (running max in the log2 domain) per row;
//  * the warps' partial states are merged through shared memory at the end;
//    the result goes to `out` (one split) or to fp32 split partials.  With
//    split partials and few rows per group (m * s_q * splits <= 64), the last
//    CTA of a (sequence, group, row block) to finish (an atomic count per
//    block) merges all splits' partials by their log-sum-exp and writes the
//    final output, so no separate combine pass re-reads them.
#include <math.h>

#include "ptx.cuh"
#include "tc.h"

namespace gqla {

namespace {

constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr int kT = 64;                       // tokens per tile
constexpr int kStages = 2;
constexpr int kKChunks = kDqk / 64;          // 64-column (128-byte) chunks
constexpr int kVChunks = kDv / 64;
constexpr int kChunkBytes = kT * 128;
constexpr int kStageBytes = (kKChunks + kVChunks) * kChunkBytes;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kOStride = kDv + 4;            // merge buffer row pitch (floats)
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + 1024;

struct GqaParams {
  KvLayout ly;
  SplitPlan plan;
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  float* o_part;
  float* lse;
  int n_h, G, m, s_q;
  int rows_unit;   // m * s_q rows of one (sequence, group)
  int rbc;         // 16-row blocks per CTA: 1, 2 or 4
  KRow kr;         // K pool row layout
  float scale_log2;
  long long rows;  // B * s_q * n_h
  int32_t* st;
  // split merge in the kernel (o_part != nullptr): counters zeroed before
  // the launch, one per (sequence, group, CTA row block); final outputs
  int* counters;
  __nv_bfloat16* out_final;
  float* lse_final;
};

static_assert(kConsumerWarps * 16 * kOStride * 4 + 2 * kConsumerWarps * 16 * 4 <= kStages * kStageBytes,
              "merge buffer must fit in the stage ring");

__global__ void __launch_bounds__(kThreads, 2)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const GqaParams p) {
  // launched while the kernel ahead of it may still run: wait for it before
  // any memory access, then let the next kernel launch
  ptx::pdl_wait();
  ptx::pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int b = blockIdx.y / p.G, g = blockIdx.y % p.G;
  const int rb0 = blockIdx.z * p.rbc;            // first global 16-row block of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full_bar[s], 1);
      ptx::mbar_init(&empty_bar[s], kConsumerWarps);
    }
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  int L = seq_len_checked(p.ly, b, p.s_q, (split == 0 && g == 0 && blockIdx.z == 0) ? p.st : nullptr);
  if (!seq_pages_ok(p.ly, b, L, p.st)) L = -1;   // includes a __syncthreads
  const int t_begin = split * p.plan.chunk;
  const int t_stop = L < 0 ? t_begin : min(t_begin + p.plan.chunk, L);
  const int n_tiles = t_stop > t_begin ? (t_stop - t_begin + kT - 1) / kT : 0;

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      ptx::prefetch_tmap(&kmap);
      ptx::prefetch_tmap(&vmap);
      const int kx = p.kr.nope_at(g), kxr = p.kr.rope_at(g), vx = g * kDv;
      // a tile's pool row (a page-table read when paged) is looked up one
      // tile ahead, so its latency overlaps the wait for the slot
      int row_next = n_tiles > 0 ? (int)token_row(p.ly, b, t_begin, nullptr) : 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kStages, k = j / kStages;
        const int row0 = row_next;
        if (j + 1 < n_tiles) row_next = (int)token_row(p.ly, b, t_begin + (j + 1) * kT, nullptr);
        if (k > 0 && !ptx::mbar_wait(&empty_bar[s], (k - 1) & 1)) {
          flag_status(p.st, GQLA_DEV_TIMEOUT);
          atomicExch(&abort_flag, 1);
          break;
        }
        if (*(volatile int*)&abort_flag) break;
        uint8_t* st = smem + s * kStageBytes;
        ptx::mbar_arrive_expect_tx(&full_bar[s], kStageBytes);
        // K: the group's two d_nope chunks, then its RoPE chunk; V: two chunks
        ptx::tma_load_2d(st, &kmap, &full_bar[s], kx, row0);
        ptx::tma_load_2d(st + kChunkBytes, &kmap, &full_bar[s], kx + 64, row0);
        ptx::tma_load_2d(st + 2 * kChunkBytes, &kmap, &full_bar[s], kxr, row0);
#pragma unroll
        for (int c = 0; c < kVChunks; ++c)
          ptx::tma_load_2d(st + (kKChunks + c) * kChunkBytes, &vmap, &full_bar[s], vx + 64 * c, row0);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int ts = kConsumerWarps / p.rbc;         // token slices per tile
  const int rbl = warp / ts, slice = warp % ts;
  const int sub_steps = (kT / ts) / 16;
  const int gid = lane >> 2, tig = lane & 3;
  const int rbg = rb0 + rbl;                      // this warp's global row block
  int vis[2];
  long long grow[2];
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int r = rbg * 16 + gid + 8 * h2;
    if (r < p.rows_unit && L >= 0) {
      const int i = r / p.m, h = g * p.m + r % p.m;
      vis[h2] = L - p.s_q + i + 1;
      grow[h2] = ((long long)b * p.s_q + i) * p.n_h + h;
    } else {
      vis[h2] = 0;
      grow[h2] = -1;
    }
  }
  // Q fragments (A operand, 16 rows x 192) straight from global memory.
  uint32_t qa[kDqk / 16][4];
#pragma unroll
  for (int kk = 0; kk < kDqk / 16; ++kk) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int h2 = e & 1, hi = e >> 1;
      uint32_t v = 0;
      if (grow[h2] >= 0)
        v = *reinterpret_cast<const uint32_t*>(p.q + grow[h2] * kDqk + kk * 16 + hi * 8 + 2 * tig);
      qa[kk][e] = v;
    }
  }
  float o[kDv / 8][4];
#pragma unroll
  for (int n = 0; n < kDv / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  bool aborted = false;

  for (int j = 0; j < n_tiles; ++j) {
    const int s = j % kStages;
    if (!ptx::mbar_wait(&full_bar[s], (j / kStages) & 1)) {
      flag_status(p.st, GQLA_DEV_TIMEOUT);
      atomicExch(&abort_flag, 1);
      aborted = true;
      break;
    }
    const int t0 = t_begin + j * kT;
    const uint8_t* st = smem + s * kStageBytes;
    const uint32_t kbase = ptx::smem_u32(st);
    const uint32_t vbase = kbase + kKChunks * kChunkBytes;
    if (t0 + kT > L) {
      // rows past the sequence may hold anything: zero this warp's V rows there
      for (int idx = lane; idx < (kT / ts) * kVChunks * 8; idx += 32) {
        const int tok = slice * (kT / ts) + idx / (kVChunks * 8);
        const int rem = idx % (kVChunks * 8);
        if (t0 + tok >= L)
          *reinterpret_cast<uint4*>(const_cast<uint8_t*>(st) + kKChunks * kChunkBytes + (rem / 8) * kChunkBytes +
                                    ptx::swz128(tok, rem % 8)) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    for (int u = 0; u < sub_steps; ++u) {
      const int tt0 = slice * (kT / ts) + u * 16;
      float sc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) sc[e] = 0.f;
      const int mat = lane >> 3, mr = lane & 7;
#pragma unroll
      for (int kk = 0; kk < kDqk / 16; ++kk) {
        const int tok = tt0 + (mat >> 1) * 8 + mr;
        const int gi = (kk & 3) * 2 + (mat & 1);
        uint32_t r0, r1, r2, r3;
        ptx::ldsm_x4(kbase + (kk >> 2) * kChunkBytes + ptx::swz128(tok, gi), r0, r1, r2, r3);
        ptx::mma_bf16_16816(&sc[0], qa[kk], r0, r1);
        ptx::mma_bf16_16816(&sc[4], qa[kk], r2, r3);
      }
      // scale into the log2 domain and mask invisible tokens (select, so a
      // non-finite key past the end cannot leak in)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int h2 = (e >> 1) & 1;
        const int tok = t0 + tt0 + (e >> 2) * 8 + 2 * tig + (e & 1);
        sc[e] = tok < vis[h2] ? sc[e] * p.scale_log2 : -INFINITY;
        mx[h2] = fmaxf(mx[h2], sc[e]);
      }
      float corr[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 1));
        mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 2));
        const float mn = fmaxf(mrow[h2], mx[h2]);
        corr[h2] = mn == -INFINITY ? 1.f : ptx::fast_exp2(mrow[h2] - mn);
        mrow[h2] = mn;
      }
      float ps[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int h2 = (e >> 1) & 1;
        ps[e] = mrow[h2] == -INFINITY ? 0.f : ptx::fast_exp2(sc[e] - mrow[h2]);
      }
      lrow[0] = lrow[0] * corr[0] + (ps[0] + ps[1] + ps[4] + ps[5]);
      lrow[1] = lrow[1] * corr[1] + (ps[2] + ps[3] + ps[6] + ps[7]);
      if (corr[0] != 1.f || corr[1] != 1.f) {
#pragma unroll
        for (int n = 0; n < kDv / 8; ++n) {
          o[n][0] *= corr[0];
          o[n][1] *= corr[0];
          o[n][2] *= corr[1];
          o[n][3] *= corr[1];
        }
      }
      uint32_t pa[4];
      pa[0] = ptx::pack_bf16(ps[0], ps[1]);
      pa[1] = ptx::pack_bf16(ps[2], ps[3]);
      pa[2] = ptx::pack_bf16(ps[4], ps[5]);
      pa[3] = ptx::pack_bf16(ps[6], ps[7]);
#pragma unroll
      for (int np = 0; np < kDv / 16; ++np) {
        const int tok = tt0 + (mat & 1) * 8 + mr;
        const int gi = (np & 3) * 2 + (mat >> 1);
        uint32_t r0, r1, r2, r3;
        ptx::ldsm_x4_t(vbase + (np >> 2) * kChunkBytes + ptx::swz128(tok, gi), r0, r1, r2, r3);
        ptx::mma_bf16_16816(o[2 * np], pa, r0, r1);
        ptx::mma_bf16_16816(o[2 * np + 1], pa, r2, r3);
      }
    }
    if (t0 + kT > L) ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty_bar[s]);
  }

  // ------------------------------------------------ merge the token slices
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    lrow[h2] += __shfl_xor_sync(0xffffffffu, lrow[h2], 1);
    lrow[h2] += __shfl_xor_sync(0xffffffffu, lrow[h2], 2);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
  if (aborted || *(volatile int*)&abort_flag) return;
  float* ob = reinterpret_cast<float*>(smem);                       // [warp][16][kOStride]
  float* ml = ob + kConsumerWarps * 16 * kOStride;                  // [warp][16] max, then [warp][16] sum
#pragma unroll
  for (int n = 0; n < kDv / 8; ++n) {
    *reinterpret_cast<float2*>(&ob[(warp * 16 + gid) * kOStride + n * 8 + 2 * tig]) = make_float2(o[n][0], o[n][1]);
    *reinterpret_cast<float2*>(&ob[(warp * 16 + gid + 8) * kOStride + n * 8 + 2 * tig]) =
        make_float2(o[n][2], o[n][3]);
  }
  if (tig == 0) {
    ml[warp * 16 + gid] = mrow[0];
    ml[warp * 16 + gid + 8] = mrow[1];
    ml[kConsumerWarps * 16 + warp * 16 + gid] = lrow[0];
    ml[kConsumerWarps * 16 + warp * 16 + gid + 8] = lrow[1];
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
  // Merge: every consumer thread takes (row, 4 columns) pieces of the
  // CTA's rows; the ts partial states of a row are combined with per-row
  // weights held in registers.
  const int tid = threadIdx.x;
  for (int idx = tid; idx < p.rbc * 16 * (kDv / 4); idx += kConsumerWarps * 32) {
    const int rl = idx / (kDv / 4), d4 = (idx % (kDv / 4)) * 4;
    const int rbl2 = rl >> 4, rr = rl & 15;
    const int r = (rb0 + rbl2) * 16 + rr;
    if (r >= p.rows_unit) continue;
    const int i = r / p.m, h = g * p.m + r % p.m;
    const long long gr = ((long long)b * p.s_q + i) * p.n_h + h;
    float mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w)
      if (w < ts) mt = fmaxf(mt, ml[(rbl2 * ts + w) * 16 + rr]);
    float wsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      if (w < ts) {
        const float mwv = ml[(rbl2 * ts + w) * 16 + rr];
        const float wv = mwv == -INFINITY ? 0.f : ptx::fast_exp2(mwv - mt);
        wsum += wv * ml[kConsumerWarps * 16 + (rbl2 * ts + w) * 16 + rr];
        const float4 o4 = *reinterpret_cast<const float4*>(&ob[((rbl2 * ts + w) * 16 + rr) * kOStride + d4]);
        acc.x = fmaf(wv, o4.x, acc.x);
        acc.y = fmaf(wv, o4.y, acc.y);
        acc.z = fmaf(wv, o4.z, acc.z);
        acc.w = fmaf(wv, o4.w, acc.w);
      }
    }
    const bool empty = !(wsum > 0.f);
    const float inv = empty ? 0.f : 1.f / wsum;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    if (p.o_part) {
      *reinterpret_cast<float4*>(p.o_part + ((long long)split * p.rows + gr) * kDv + d4) = acc;
    } else {
      *reinterpret_cast<uint2*>(p.out + gr * kDv + d4) =
          make_uint2(ptx::pack_bf16(acc.x, acc.y), ptx::pack_bf16(acc.z, acc.w));
    }
    if (d4 == 0 && p.lse) {
      const float lse = empty ? -INFINITY : (mt + log2f(wsum)) * 0.69314718055994531f;
      p.lse[p.o_part ? (long long)split * p.rows + gr : gr] = lse;
    }
  }
  if (p.o_part && p.counters) {
    // ------------------------------------ merge the splits (last CTA only)
    __shared__ int last_cta;
    __threadfence();                              // this CTA's partials are visible before the count
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
    const int S = p.plan.num_splits;
    int* counter = p.counters + ((long long)blockIdx.y * gridDim.z + blockIdx.z);
    if (tid == 0) last_cta = atomicAdd(counter, 1) == S - 1;
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
    if (last_cta) {
      __threadfence();
      // the ring is idle now: per row of this CTA, the splits' weights
      const int nrow = min(p.rbc * 16, p.rows_unit - rb0 * 16);
      float* wtab = reinterpret_cast<float*>(smem);   // [nrow][S]
      float* rmax = wtab + nrow * S;                  // [nrow]
      float* rsum = rmax + nrow;                      // [nrow]
      for (int rl = warp; rl < nrow; rl += kConsumerWarps) {
        const int r = rb0 * 16 + rl;
        const int i = r / p.m, h = g * p.m + r % p.m;
        const long long gr = ((long long)b * p.s_q + i) * p.n_h + h;
        float mx = -INFINITY;
        for (int sp = lane; sp < S; sp += 32) mx = fmaxf(mx, __ldcg(p.lse + (long long)sp * p.rows + gr));
        mx = warp_max(mx);
        float z = 0.f;
        for (int sp = lane; sp < S; sp += 32) {
          const float ls = __ldcg(p.lse + (long long)sp * p.rows + gr);
          const float w = (ls == -INFINITY) ? 0.f : expf(ls - mx);
          wtab[rl * S + sp] = w;
          z += w;
        }
        z = warp_sum(z);
        if (lane == 0) {
          rmax[rl] = mx;
          rsum[rl] = z;
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
      // weighted sums: the splits' loads are independent (an empty split holds zeros)
      for (int idx = tid; idx < nrow * (kDv / 4); idx += kConsumerWarps * 32) {
        const int rl = idx / (kDv / 4), d4 = (idx % (kDv / 4)) * 4;
        const int r = rb0 * 16 + rl;
        const int i = r / p.m, h = g * p.m + r % p.m;
        const long long gr = ((long long)b * p.s_q + i) * p.n_h + h;
        const float* src = p.o_part + gr * kDv + d4;
        const long long sstride = p.rows * kDv;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int sp = 0; sp < S; ++sp) {
          const float w = wtab[rl * S + sp];
          const float4 o = __ldcg(reinterpret_cast<const float4*>(src + sp * sstride));
          acc.x = fmaf(w, o.x, acc.x);
          acc.y = fmaf(w, o.y, acc.y);
          acc.z = fmaf(w, o.z, acc.z);
          acc.w = fmaf(w, o.w, acc.w);
        }
        const float z = rsum[rl];
        const float inv = z > 0.f ? 1.f / z : 0.f;
        *reinterpret_cast<uint2*>(p.out_final + gr * kDv + d4) =
            make_uint2(ptx::pack_bf16(acc.x * inv, acc.y * inv), ptx::pack_bf16(acc.z * inv, acc.w * inv));
        if (d4 == 0 && p.lse_final) p.lse_final[gr] = rmax[rl] == -INFINITY ? -INFINITY : rmax[rl] + logf(z);
      }
      if (tid == 0) *counter = 0;                 // back to zero for the next call
    }
  }
}

}  // namespace

bool tc_gqa_supports(const Problem& p) {
  const auto& d = p.d;
  if (d.dtype != GQLA_BF16) return false;
  if (p.d_qk != kDqk || d.d_v != kDv) return false;
  if (p.ly.page_size != 0 && p.ly.page_size % kT != 0) return false;
  if ((long long)p.ly.batch * d.G > 65535) return false;
  return true;
}

cudaError_t tc_gqa_decode(const Problem& p, const void* q, const void* k_pool, const void* v_pool, void* out,
                          float* o_part, float* lse_dst, int32_t* st, cudaStream_t s, int* counters,
                          void* out_final, float* lse_final, bool* merged) {
  if (merged) *merged = false;
  if (tc_gqa_wide_supports(p)) return tc_gqa_wide_decode(p, q, k_pool, v_pool, out, o_part, lse_dst, st, s);
  const auto& d = p.d;
  CUtensorMap kmap, vmap;
  if (!gqa_pool_maps(p, k_pool, v_pool, &kmap, &vmap)) return cudaErrorInvalidValue;
  GqaParams prm;
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
  const int rb = (prm.rows_unit + 15) / 16;
  prm.rbc = rb >= 4 ? 4 : (rb == 3 ? 4 : rb);
  prm.scale_log2 = d.scale * 1.4426950408889634f;
  prm.rows = p.rows;
  prm.st = st;
  prm.kr = p.kr;
  dim3 grid(p.plan.num_splits, p.ly.batch * d.G, (rb + prm.rbc - 1) / prm.rbc);
  // Merging in the last CTA pays when a block's merge is small (measured: it
  // wins at 4 rows x 8 splits, loses at 16-32 rows x 8-16 splits, where the
  // combine pass spreads the same work over the whole GPU).
  const bool merge = o_part && counters && out_final && (long long)p.m * d.s_q * p.plan.num_splits <= 64;
  prm.counters = merge ? counters : nullptr;
  prm.out_final = (__nv_bfloat16*)out_final;
  prm.lse_final = lse_final;
  if (merge) {
    cudaError_t e0 = cudaMemsetAsync(counters, 0, sizeof(int) * (size_t)grid.y * grid.z, s);
    if (e0 != cudaSuccess) return e0;
  }
  cudaError_t e = ensure_smem_limit((const void*)gqa_decode_kernel, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(gqa_decode_kernel, grid, dim3(kThreads), kSmemBytes, s, kmap, vmap, prm);
  count_launch();
  if (e != cudaSuccess) return e;
  if (merge && merged) *merged = true;
  return cudaGetLastError();
}

}  // namespace gqla
