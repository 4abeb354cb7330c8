// Per-group cache expansion on the 5th-generation tensor cores (tcgen05).
//
// The GQA path runs over a per-group expanded cache ("GQLA" chatpaper.ai
// Abstract): for every token t and group g,
//     K[t, g] = [ c_t W_uk^g ; k_rope_t ],   V[t, g] = c_t W_uv^g.
// Per group this is one dense GEMM  C = X [T x 512] * [W_uk^g | W_uv^g]
// [512 x 256], so it runs as a persistent tcgen05 GEMM:
//  * work item = (128-token tile, group), group index fastest, so the G items
//    that share a latent tile run at the same time and L2 serves the re-reads;
//  * warp 0 streams K-chunks of 64 (A: 128 tokens x 64, two 64-row TMA boxes
//    so that a tile may span two pages; B: 64 rows x 256 columns of the two
//    weight matrices) into a 4-stage mbarrier ring;
//  * warp 1 issues 4 tcgen05.mma (M=128, N=256, K=16; A K-major, B MN-major)
//    per chunk into one of two TMEM accumulators (2 x 256 columns);
//  * warps 2-5 drain an accumulator (tcgen05.ld, one token row per thread)
//    and round to bf16.  Each warp works alone, without block barriers: when
//    all 32 of its rows are written it stages 64 columns at a time in its own
//    ring of 128-byte-swizzled 32 x 64 boxes and sends each with a TMA store
//    (each row from one thread would make every warp store touch 32 rows
//    G * 640 bytes apart), waiting only until the store that last used a box
//    has read it; other rows are stored by their thread.  The RoPE key needs
//    no accumulator: the warp loads it (eight lanes per row, 16 bytes each)
//    before it waits for the MMAs and stores it after its columns.  (Eight
//    epilogue warps, two per lane quarter, measured slower: the ring, the
//    operand reads and the staging share the SM's shared-memory bandwidth.)
// Tiles start on a 64-token boundary; rows outside [first token, L) of the
// sequence are computed but not written.  This single-CTA kernel serves the
// newest-tokens form and the dense form below; the whole cache goes to the
// two-SM kernel further down (same tiles, same epilogue, M = 256 over a
// cluster pair) when the device can hold such pairs.
//
// A second form takes a dense matrix of token rows instead of the pool (the
// s_q new rows of every sequence, B * s_q of them, at decode time): its
// tiles are 128 consecutive rows of that matrix, so the new tokens of many
// sequences share one tile, and each output row goes to its token's pool
// row.  A dense item may also cover only the K or only the V half of the
// outputs (N = 128), so that a small batch of new tokens spreads over twice
// as many CTAs, each loading half the weights.  Every output element is
// still the same K-ordered sum of bf16 products, so a token's expansion is
// the same numbers whichever form produced it.
#include <mutex>

#include "ptx.cuh"
#include "tc.h"

namespace gqla {

namespace {

using bf16 = __nv_bfloat16;

constexpr int kR = 512, kDn = 128, kDv = 128, kDr = 64, kE = kR + kDr;
constexpr int kTM = 128;                          // tokens per tile
constexpr int kN = kDn + kDv;                     // 256 outputs per group
constexpr int kKC = 64;                           // K per stage
constexpr int kStages = 4;
constexpr int kABytes = kTM * 128;                // 16 KB
constexpr int kBBox = kKC * 128;                  // 8 KB: 64 K-rows x 64 columns
constexpr int kBBytes = 4 * kBBox;                // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;    // 48 KB
constexpr int kEpiWarps = 4;                      // one per TMEM lane quarter
constexpr int kSlots = 2;                         // staging boxes per epilogue warp
constexpr int kBoxBytes = 32 * 128;              // a 32-row x 64-column bf16 box (one warp's rows)
constexpr int kOutBytes = kEpiWarps * kSlots * kBoxBytes;   // a ring of kSlots boxes for each epilogue warp
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + kOutBytes + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = (2 + kEpiWarps) * 32;
static_assert(kSmemBytes <= 227 * 1024, "ring and staging must fit the shared memory of one CTA");

// This thread's bulk-copy groups, all but the newest n, have read their
// shared-memory sources.
template <int n>
__device__ __forceinline__ void bulk_wait_read_allbut() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}

struct ExpandParams {
  KvLayout ly;
  bf16* kp;
  KRow kr;
  bf16* vp;
  const bf16* latent;
  int G;
  int tail;          // > 0: only the newest `tail` tokens of each sequence
  int tps;           // tiles per sequence
  long long n_items; // batch * tps * G  (dense form: ceil(dense_rows / 128) * G)
  const bf16* dense; // dense form: [dense_rows, 576] new rows, row b * s_q + i = token L_b - s_q + i
  int dense_rows;    // 0: pool form
  int halves;        // 2: an item covers the K or the V outputs only (item % 2), else both
  int s_q;
  int32_t* st;
};

// Dense form: pool row of dense row dr (= b * s_q + i), or -1 when the
// sequence is invalid or the page is outside the pool (flagged).
__device__ __forceinline__ long long dense_row_target(const ExpandParams& p, int dr) {
  const KvLayout& ly = p.ly;
  const int b = dr / p.s_q, i = dr % p.s_q;
  const int L = ly.seq_lens[b];
  const bool bad = L < p.s_q || L > ly.max_seq_len ||
                   (ly.page_size == 0 ? L > ly.capacity : (L + ly.page_size - 1) / ly.page_size > ly.mbps);
  if (bad) return -1;
  return token_row(ly, b, L - p.s_q + i, p.st);
}

// Tile j of sequence b: first token t0 (64-aligned) and the token range
// [t_lo, t_hi) that is written.  Returns false when the item is empty.  In
// the dense form "sequence" 0 has tiles of 128 dense rows: t0 is the first.
__device__ __forceinline__ bool item_tile(const ExpandParams& p, int b, int j, int* t0, int* t_lo, int* t_hi,
                                          bool report = false) {
  if (p.dense_rows > 0) {
    *t0 = j * kTM;
    *t_lo = 0;
    *t_hi = p.dense_rows;
    return *t0 < p.dense_rows;
  }
  const KvLayout& ly = p.ly;
  const int L = ly.seq_lens[b];
  const bool bad = L < 1 || L > ly.max_seq_len ||
                   (ly.page_size == 0 ? L > ly.capacity : (L + ly.page_size - 1) / ly.page_size > ly.mbps);
  if (bad) {
    if (report && j == 0) flag_status(p.st, L < 1 ? GQLA_DEV_SHORT_SEQ : GQLA_DEV_OVERFLOW);
    return false;
  }
  const int start = p.tail > 0 ? max(0, L - p.tail) : 0;
  *t0 = (start / 64) * 64 + j * kTM;
  *t_lo = start;
  *t_hi = L;
  return *t0 < L;
}

// Pool row of the first token of a 64-token half tile: 0 for a half past
// the sequence (read, never written), -1 for a page outside the pool.
__device__ __forceinline__ int half_row(const KvLayout& ly, int b, int t, int L) {
  if (ly.page_size == 0) return (int)((long long)b * ly.capacity + t);
  const int nb = (L + ly.page_size - 1) / ly.page_size;
  const int blk = t / ly.page_size;
  if (blk >= nb) return 0;
  const int page = ly.block_table[(long long)b * ly.mbps + blk];
  if (page < 0 || page >= ly.num_pages) return -1;
  return page * ly.page_size + (t % ly.page_size);
}

__global__ void __launch_bounds__(kThreads, 1)
    expand_tc_kernel(const __grid_constant__ CUtensorMap lat_map, const __grid_constant__ CUtensorMap uk_map,
                     const __grid_constant__ CUtensorMap uv_map, const __grid_constant__ CUtensorMap k_store,
                     const __grid_constant__ CUtensorMap v_store, const ExpandParams p) {
  // launched while the kernel ahead of it may still run: wait for it before
  // any memory access, then let the next kernel launch
  ptx::pdl_wait();
  ptx::pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_base_sh;
  uint8_t* s_out = smem + kStages * kStageBytes;   // 1024-aligned staging boxes
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full_bar[s], 1);
      ptx::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&acc_full[a], 1);
      ptx::mbar_init(&acc_empty[a], kEpiWarps);
    }
    ptx::mbar_init(&drain, 1);
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&tmem_base_sh, kTmemCols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int G = p.G;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&lat_map);
      ptx::prefetch_tmap(&uk_map);
      ptx::prefetch_tmap(&uv_map);
      long long it = 0;
      bool ok = true;
      for (long long item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const int hf = p.halves == 2 ? (int)(item & 1) : -1;
        const long long it2 = p.halves == 2 ? item >> 1 : item;
        const int g = (int)(it2 % G);
        const long long bt = it2 / G;
        const int b = (int)(bt / p.tps), j = (int)(bt % p.tps);
        int t0, tlo, thi;
        if (!item_tile(p, b, j, &t0, &tlo, &thi, g == 0)) continue;
        // dense form: rows of the dense matrix (a box past its end reads zeros)
        const int row0 = p.dense_rows > 0 ? t0 : max(0, half_row(p.ly, b, t0, thi));
        const int row1 = p.dense_rows > 0 ? t0 + 64 : max(0, half_row(p.ly, b, t0 + 64, thi));
        for (int kc = 0; kc < kR / kKC; ++kc, ++it) {
          const int s = (int)(it % kStages);
          const long long k = it / kStages;
          if (k > 0 && !ptx::mbar_wait(&empty_bar[s], (uint32_t)((k - 1) & 1))) {
            flag_status(p.st, GQLA_DEV_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          ptx::mbar_arrive_expect_tx(&full_bar[s], hf < 0 ? kStageBytes : kABytes + 2 * kBBox);
          ptx::tma_load_2d(st, &lat_map, &full_bar[s], kKC * kc, row0);
          ptx::tma_load_2d(st + kABytes / 2, &lat_map, &full_bar[s], kKC * kc, row1);
          uint8_t* bs = st + kABytes;
          const int wrow = g * kR + kKC * kc;
          if (hf != 1) {
            ptx::tma_load_2d(bs + 0 * kBBox, &uk_map, &full_bar[s], 0, wrow);
            ptx::tma_load_2d(bs + 1 * kBBox, &uk_map, &full_bar[s], 64, wrow);
          }
          if (hf != 0) {
            const int vb = hf < 0 ? 2 : 0;       // V boxes after the K boxes, or alone
            ptx::tma_load_2d(bs + (vb + 0) * kBBox, &uv_map, &full_bar[s], 0, wrow);
            ptx::tma_load_2d(bs + (vb + 1) * kBBox, &uv_map, &full_bar[s], 64, wrow);
          }
        }
      }
      // no copy may still be landing when the CTA retires
      for (long long i = it > kStages ? it - kStages : 0; i < it; ++i)
        ptx::mbar_wait(&full_bar[i % kStages], (uint32_t)((i / kStages) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_full = ptx::idesc_bf16(kTM, kN, false, true);
      constexpr uint32_t idesc_half = ptx::idesc_bf16(kTM, kN / 2, false, true);
      const uint32_t base = ptx::smem_u32(smem);
      long long it = 0, li = 0;
      bool ok = true;
      for (long long item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const int hf = p.halves == 2 ? (int)(item & 1) : -1;
        const long long it2 = p.halves == 2 ? item >> 1 : item;
        const int g = (int)(it2 % G);
        const long long bt = it2 / G;
        const int b = (int)(bt / p.tps), j = (int)(bt % p.tps);
        int t0, tlo, thi;
        (void)g;
        const uint32_t idesc = hf < 0 ? idesc_full : idesc_half;
        if (!item_tile(p, b, j, &t0, &tlo, &thi)) continue;
        const int ab = (int)(li & 1);
        if (li >= 2 && !ptx::mbar_wait(&acc_empty[ab], (uint32_t)(((li >> 1) - 1) & 1))) {
          ok = false;
          break;
        }
        const uint32_t d = tmem + (uint32_t)(ab * kN);
        for (int kc = 0; kc < kR / kKC; ++kc, ++it) {
          const int s = (int)(it % kStages);
          if (!ptx::mbar_wait(&full_bar[s], (uint32_t)((it / kStages) & 1))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_addr = base + s * kStageBytes;
          const uint64_t ad0 = ptx::umma_desc_sw128(a_addr, 16, 1024);
          const uint64_t bd0 = ptx::umma_desc_sw128(a_addr + kABytes, kBBox, 1024);
#pragma unroll
          for (int kk = 0; kk < kKC / 16; ++kk)
            ptx::umma_bf16(d, ptx::umma_desc_add(ad0, kk * 32), ptx::umma_desc_add(bd0, kk * 16 * 128), idesc,
                           (kc | kk) != 0);
          ptx::umma_commit(&empty_bar[s]);
        }
        if (!ok) break;
        ptx::umma_commit(&acc_full[ab]);
        ++li;
      }
      if (!ok) flag_status(p.st, GQLA_DEV_TIMEOUT);
      ptx::umma_commit(&drain);
      ptx::mbar_wait(&drain, 0);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int qd = warp & 3;                   // TMEM lane quarter
    const int r = 32 * qd + lane;              // tile row = token offset
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    uint8_t* ring = s_out + (warp - 2) * kSlots * kBoxBytes;
    long long li = 0, stores = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      const int hf = p.halves == 2 ? (int)(item & 1) : -1;
      const long long it2 = p.halves == 2 ? item >> 1 : item;
      const int g = (int)(it2 % G);
      const long long bt = it2 / G;
      const int b = (int)(bt / p.tps), j = (int)(bt % p.tps);
      int t0, tlo, thi;
      if (!item_tile(p, b, j, &t0, &tlo, &thi)) continue;
      const int ab = (int)(li & 1);
      const int t = t0 + r;
      bool write = t >= tlo && t < thi;
      long long row = 0;
      if (write) {
        if (p.dense_rows > 0) {
          row = dense_row_target(p, t);
          write = row >= 0;
        } else {
          const int hr = half_row(p.ly, b, t0 + (r & ~63), thi);
          if (hr < 0) {
            flag_status(p.st, GQLA_DEV_BAD_PAGE);
            write = false;
          }
          row = (long long)hr + (r & 63);
        }
      }
      // RoPE key rows of this warp (a shared key: by group 0): lanes 8i..8i+7
      // take 16 bytes each of row 4k + i; loaded now, stored after the columns
      const bool rope = ok && hf != 1 && (p.kr.rope_gs != 0 || g == 0);
      uint4 rv[8];
      bool rw[8];
      long long rrow[8];
      if (rope) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = 4 * k + (lane >> 3);
          rw[k] = __shfl_sync(0xffffffffu, write, rr);
          rrow[k] = __shfl_sync(0xffffffffu, row, rr);
          if (rw[k]) {
            const long long src_row = p.dense_rows > 0 ? (long long)(t0 + 32 * qd + rr) : rrow[k];
            const bf16* base = p.dense_rows > 0 ? p.dense : p.latent;
            rv[k] = *reinterpret_cast<const uint4*>(base + src_row * kE + kR + 8 * (lane & 7));
          }
        }
      }
      if (ok) ok = ptx::mbar_wait(&acc_full[ab], (uint32_t)((li >> 1) & 1));
      ok = __all_sync(0xffffffffu, ok);
      write = write && ok;
      // all 32 rows of this warp written, consecutive in the pool: TMA stores
      const int w_lo = t0 + 32 * qd;
      const int hr0 = p.dense_rows == 0 ? half_row(p.ly, b, t0 + 64 * (qd >> 1), thi) : -1;
      const bool tma_rows = ok && p.dense_rows == 0 && w_lo >= tlo && w_lo + 32 <= thi && hr0 >= 0;
      const int y0 = hr0 + 32 * (qd & 1);
      if (ok) {
        ptx::tc_fence_after();
        const int ncg = (hf < 0 ? kN : kN / 2) / 64;   // 64-column groups in the accumulator
#pragma unroll 1
        for (int c = 0; c < ncg; ++c) {
          uint32_t v[64];
          ptx::tmem_ld32(tl + (uint32_t)(ab * kN + 64 * c), v);
          ptx::tmem_ld32(tl + (uint32_t)(ab * kN + 64 * c + 32), v + 32);
          ptx::tmem_ld_wait();
          uint4 w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            w[e].x = ptx::pack_bf16(__uint_as_float(v[8 * e + 0]), __uint_as_float(v[8 * e + 1]));
            w[e].y = ptx::pack_bf16(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3]));
            w[e].z = ptx::pack_bf16(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5]));
            w[e].w = ptx::pack_bf16(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7]));
          }
          const int oc = hf == 1 ? c + kDn / 64 : c;    // 64-column group of [K nope | V]
          if (tma_rows) {
            uint8_t* box = ring + (int)(stores % kSlots) * kBoxBytes;
            if (lane == 0) bulk_wait_read_allbut<kSlots - 1>();   // the box's last store has read it
            __syncwarp();
#pragma unroll
            for (int e = 0; e < 8; ++e) *reinterpret_cast<uint4*>(box + ptx::swz128(lane, e)) = w[e];
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (oc < kDn / 64)
                ptx::tma_store_2d(&k_store, box, p.kr.nope_at(g) + 64 * oc, y0);
              else
                ptx::tma_store_2d(&v_store, box, g * kDv + 64 * (oc - kDn / 64), y0);
              ptx::bulk_commit_group();
            }
            ++stores;
          } else if (write) {
            bf16* dst = oc < kDn / 64 ? p.kp + row * p.kr.pitch + p.kr.nope_at(g) + 64 * oc
                                      : p.vp + (row * G + g) * kDv + 64 * (oc - kDn / 64);
#pragma unroll
            for (int e = 0; e < 8; ++e) *reinterpret_cast<uint4*>(dst + 8 * e) = w[e];
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&acc_empty[ab]);
      if (rope && ok) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (rw[k]) *reinterpret_cast<uint4*>(p.kp + rrow[k] * p.kr.pitch + p.kr.rope_at(g) + 8 * (lane & 7)) = rv[k];
      }
      ++li;
    }
    if (!ok && lane == 0) flag_status(p.st, GQLA_DEV_TIMEOUT);
    if (lane == 0) ptx::bulk_wait_group();   // every store has landed before the CTA ends
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------ CTA pairs
// The whole-cache form on pairs of SMs (tcgen05 cta_group::2): one MMA of
// M = 256 rows, N = 256, K = 16 covers the 128-token tiles of both CTAs of a
// cluster pair, and each CTA stages only its half of B (CTA 0 the W_uk^g
// columns, CTA 1 the W_uv^g columns), so per SM a K-chunk moves 32 KB through
// shared memory instead of 48 KB, and six stages fit.  Each CTA's TMEM gets the
// full 256 output columns of its own 128 rows.  CTA 0 issues the MMAs; both
// CTAs' copies complete on CTA 0's stage barriers; the commits arrive on the
// stage and accumulator barriers of both CTAs; the epilogue warps of CTA 1
// free an accumulator by arriving on CTA 0's barrier.
namespace pairx {

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address, in the cluster's shared window, of the same variable in CTA `rank`.
__device__ __forceinline__ uint32_t at_rank(const void* v, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(ptx::smem_u32(v)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA tile load into this CTA's shared memory, completing on a barrier of
// either CTA of the pair (`bar` in the cluster window).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(ptx::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(ptx::smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The pair's MMAs issued so far arrive, when complete, on the barrier at this
// offset in both CTAs.
__device__ __forceinline__ void umma_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          ptx::smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
// Arrive on CTA 0's barrier; the values read from TMEM are already in
// registers, so nothing else needs ordering.
__device__ __forceinline__ void arrive_remote(uint32_t bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

}  // namespace pairx

constexpr int kPStages = 6;
constexpr int kPStageBytes = kABytes + 2 * kBBox;   // 16 KB of A + this CTA's 16 KB half of B
constexpr int kPSlots = 2;
constexpr int kPOutBytes = 4 * kPSlots * kBoxBytes;
constexpr size_t kPSmemBytes = (size_t)kPStages * kPStageBytes + kPOutBytes + 1024;
constexpr int kPThreads = 6 * 32;
static_assert(kPSmemBytes <= 227 * 1024, "pair ring and staging must fit the shared memory of one CTA");

// Tile `id` of the flattened (sequence, tile) list of the pool form.
__device__ __forceinline__ bool pool_tile(const ExpandParams& p, long long id, int* b, int* t0, int* tlo, int* thi,
                                          bool report) {
  if (id >= (long long)p.ly.batch * p.tps) return false;
  *b = (int)(id / p.tps);
  return item_tile(p, *b, (int)(id % p.tps), t0, tlo, thi, report);
}

// Work item i (pair level) = (tile pair i / G, group i % G); CTA r of the pair
// takes tile 2 (i / G) + r.  An item is skipped when both tiles are empty; a
// CTA whose own tile is empty still stages rows (row 0) for the shared MMA
// and writes nothing.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
    expand_pair_kernel(const __grid_constant__ CUtensorMap lat_map, const __grid_constant__ CUtensorMap uk_map,
                       const __grid_constant__ CUtensorMap uv_map, const __grid_constant__ CUtensorMap k_store,
                       const __grid_constant__ CUtensorMap v_store, const ExpandParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kPStages], empty_bar[kPStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_base_sh;
  uint8_t* s_out = smem + kPStages * kPStageBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = pairx::cta_rank();
  const long long pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      ptx::mbar_init(&full_bar[s], 1);
      ptx::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&acc_full[a], 1);
      ptx::mbar_init(&acc_empty[a], 8);           // the epilogue warps of both CTAs
    }
    ptx::mbar_init(&drain, 1);
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    pairx::tmem_alloc(&tmem_base_sh, kTmemCols);
    pairx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  pairx::cluster_sync();                          // both CTAs' barriers and TMEM are ready
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int G = p.G;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&lat_map);
      ptx::prefetch_tmap(rank == 0 ? &uk_map : &uv_map);
      const CUtensorMap* wmap = rank == 0 ? &uk_map : &uv_map;
      long long it = 0;
      bool ok = true;
      for (long long item = pair_id; ok && item < p.n_items; item += n_pairs) {
        const int g = (int)(item % G);
        const long long tp = item / G;
        int b0, t00, lo0, hi0, b1, t01, lo1, hi1;
        const bool v0 = pool_tile(p, 2 * tp, &b0, &t00, &lo0, &hi0, rank == 0 && g == 0);
        const bool v1 = pool_tile(p, 2 * tp + 1, &b1, &t01, &lo1, &hi1, rank == 1 && g == 0);
        if (!v0 && !v1) continue;
        const bool mine = rank == 0 ? v0 : v1;
        const int b = rank == 0 ? b0 : b1, t0 = rank == 0 ? t00 : t01, thi = rank == 0 ? hi0 : hi1;
        const int row0 = mine ? max(0, half_row(p.ly, b, t0, thi)) : 0;
        const int row1 = mine ? max(0, half_row(p.ly, b, t0 + 64, thi)) : 0;
        for (int kc = 0; kc < kR / kKC; ++kc, ++it) {
          const int s = (int)(it % kPStages);
          const long long k = it / kPStages;
          if (k > 0 && !ptx::mbar_wait(&empty_bar[s], (uint32_t)((k - 1) & 1))) {
            flag_status(p.st, GQLA_DEV_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kPStageBytes;
          if (rank == 0) ptx::mbar_arrive_expect_tx(&full_bar[s], 2 * kPStageBytes);
          const uint32_t fb = pairx::at_rank(&full_bar[s], 0);
          pairx::tma_load_2d(st, &lat_map, fb, kKC * kc, row0);
          pairx::tma_load_2d(st + kABytes / 2, &lat_map, fb, kKC * kc, row1);
          const int wrow = g * kR + kKC * kc;
          pairx::tma_load_2d(st + kABytes, wmap, fb, 0, wrow);
          pairx::tma_load_2d(st + kABytes + kBBox, wmap, fb, 64, wrow);
        }
      }
      // every copy of this CTA has landed and been read by the MMAs
      for (long long i = it > kPStages ? it - kPStages : 0; i < it; ++i)
        ptx::mbar_wait(&empty_bar[i % kPStages], (uint32_t)((i / kPStages) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (CTA 0)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16(2 * kTM, kN, false, true);
      const uint32_t base = ptx::smem_u32(smem);
      long long it = 0, li = 0;
      bool ok = true;
      for (long long item = pair_id; ok && item < p.n_items; item += n_pairs) {
        const long long tp = item / G;
        int b0, t00, lo0, hi0, b1, t01, lo1, hi1;
        const bool v0 = pool_tile(p, 2 * tp, &b0, &t00, &lo0, &hi0, false);
        const bool v1 = pool_tile(p, 2 * tp + 1, &b1, &t01, &lo1, &hi1, false);
        if (!v0 && !v1) continue;
        const int ab = (int)(li & 1);
        if (li >= 2 && !ptx::mbar_wait(&acc_empty[ab], (uint32_t)(((li >> 1) - 1) & 1))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(ab * kN);
        for (int kc = 0; kc < kR / kKC; ++kc, ++it) {
          const int s = (int)(it % kPStages);
          if (!ptx::mbar_wait(&full_bar[s], (uint32_t)((it / kPStages) & 1))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_addr = base + s * kPStageBytes;
          const uint64_t ad0 = ptx::umma_desc_sw128(a_addr, 16, 1024);
          const uint64_t bd0 = ptx::umma_desc_sw128(a_addr + kABytes, kBBox, 1024);
#pragma unroll
          for (int kk = 0; kk < kKC / 16; ++kk)
            pairx::umma_bf16(d, ptx::umma_desc_add(ad0, kk * 32), ptx::umma_desc_add(bd0, kk * 16 * 128), idesc,
                             (kc | kk) != 0);
          pairx::umma_commit_both(&empty_bar[s]);
        }
        if (!ok) break;
        pairx::umma_commit_both(&acc_full[ab]);
        ++li;
      }
      if (!ok) flag_status(p.st, GQLA_DEV_TIMEOUT);
      pairx::umma_commit_both(&drain);
      ptx::mbar_wait(&drain, 0);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int qd = warp & 3;                   // TMEM lane quarter
    const int r = 32 * qd + lane;              // tile row = token offset
    const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
    uint8_t* ring = s_out + (warp - 2) * kPSlots * kBoxBytes;
    const uint32_t free0 = pairx::at_rank(&acc_empty[0], 0), free1 = pairx::at_rank(&acc_empty[1], 0);
    long long li = 0, stores = 0;
    bool ok = true;
    for (long long item = pair_id; item < p.n_items; item += n_pairs) {
      const int g = (int)(item % G);
      const long long tp = item / G;
      int b0, t00, lo0, hi0, b1, t01, lo1, hi1;
      const bool v0 = pool_tile(p, 2 * tp, &b0, &t00, &lo0, &hi0, false);
      const bool v1 = pool_tile(p, 2 * tp + 1, &b1, &t01, &lo1, &hi1, false);
      if (!v0 && !v1) continue;
      const bool mine = rank == 0 ? v0 : v1;
      const int b = rank == 0 ? b0 : b1, t0 = rank == 0 ? t00 : t01;
      const int tlo = rank == 0 ? lo0 : lo1, thi = rank == 0 ? hi0 : hi1;
      const int ab = (int)(li & 1);
      const int t = t0 + r;
      bool write = mine && t >= tlo && t < thi;
      long long row = 0;
      if (write) {
        const int hr = half_row(p.ly, b, t0 + (r & ~63), thi);
        if (hr < 0) {
          flag_status(p.st, GQLA_DEV_BAD_PAGE);
          write = false;
        }
        row = (long long)hr + (r & 63);
      }
      // RoPE key rows of this warp (a shared key: by group 0): lanes 8i..8i+7
      // take 16 bytes each of row 4k + i; loaded now, stored after the columns
      const bool rope = ok && mine && (p.kr.rope_gs != 0 || g == 0);
      uint4 rv[8];
      bool rw[8];
      long long rrow[8];
      if (rope) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = 4 * k + (lane >> 3);
          rw[k] = __shfl_sync(0xffffffffu, write, rr);
          rrow[k] = __shfl_sync(0xffffffffu, row, rr);
          if (rw[k]) rv[k] = *reinterpret_cast<const uint4*>(p.latent + rrow[k] * kE + kR + 8 * (lane & 7));
        }
      }
      if (ok) ok = ptx::mbar_wait(&acc_full[ab], (uint32_t)((li >> 1) & 1));
      ok = __all_sync(0xffffffffu, ok);
      write = write && ok;
      const int w_lo = t0 + 32 * qd;
      const int hr0 = mine ? half_row(p.ly, b, t0 + 64 * (qd >> 1), thi) : -1;
      const bool tma_rows = ok && mine && w_lo >= tlo && w_lo + 32 <= thi && hr0 >= 0;
      const int y0 = hr0 + 32 * (qd & 1);
      if (ok && mine) {
        ptx::tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kN / 64; ++c) {
          uint32_t v[64];
          ptx::tmem_ld32(tl + (uint32_t)(ab * kN + 64 * c), v);
          ptx::tmem_ld32(tl + (uint32_t)(ab * kN + 64 * c + 32), v + 32);
          ptx::tmem_ld_wait();
          uint4 w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            w[e].x = ptx::pack_bf16(__uint_as_float(v[8 * e + 0]), __uint_as_float(v[8 * e + 1]));
            w[e].y = ptx::pack_bf16(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3]));
            w[e].z = ptx::pack_bf16(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5]));
            w[e].w = ptx::pack_bf16(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7]));
          }
          if (tma_rows) {
            uint8_t* box = ring + (int)(stores % kPSlots) * kBoxBytes;
            if (lane == 0) bulk_wait_read_allbut<kPSlots - 1>();   // the box's last store has read it
            __syncwarp();
#pragma unroll
            for (int e = 0; e < 8; ++e) *reinterpret_cast<uint4*>(box + ptx::swz128(lane, e)) = w[e];
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (c < kDn / 64)
                ptx::tma_store_2d(&k_store, box, p.kr.nope_at(g) + 64 * c, y0);
              else
                ptx::tma_store_2d(&v_store, box, g * kDv + 64 * (c - kDn / 64), y0);
              ptx::bulk_commit_group();
            }
            ++stores;
          } else if (write) {
            bf16* dst = c < kDn / 64 ? p.kp + row * p.kr.pitch + p.kr.nope_at(g) + 64 * c
                                     : p.vp + (row * G + g) * kDv + 64 * (c - kDn / 64);
#pragma unroll
            for (int e = 0; e < 8; ++e) *reinterpret_cast<uint4*>(dst + 8 * e) = w[e];
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          ptx::mbar_arrive(&acc_empty[ab]);
        else
          pairx::arrive_remote(ab ? free1 : free0);
      }
      if (rope && ok) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (rw[k]) *reinterpret_cast<uint4*>(p.kp + rrow[k] * p.kr.pitch + p.kr.rope_at(g) + 8 * (lane & 7)) = rv[k];
      }
      ++li;
    }
    if (!ok && lane == 0) flag_status(p.st, GQLA_DEV_TIMEOUT);
    if (lane == 0) ptx::bulk_wait_group();   // every store has landed before the CTA ends
  }
  ptx::tc_fence_before();
  __syncthreads();
  pairx::cluster_sync();                      // the pair's MMAs, copies and arrivals are over
  if (warp == 1) {
    ptx::tc_fence_after();
    pairx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Store maps of the expanded pools with one epilogue warp's 32 rows per box.
bool store_maps(const Problem& p, const void* k_pool, const void* v_pool, CUtensorMap* kmap, CUtensorMap* vmap) {
  const long long nrows = p.ly.page_size == 0 ? (long long)p.ly.batch * p.ly.capacity
                                              : (long long)p.ly.num_pages * p.ly.page_size;
  const long long vpitch = (long long)p.d.G * p.d.d_v;
  return tmap_bf16_sw128(kmap, k_pool, p.kr.pitch, nrows, p.kr.pitch, 32) &&
         tmap_bf16_sw128(vmap, v_pool, vpitch, nrows, vpitch, 32);
}

// Cluster pairs of the pair kernel that can be resident at once on the
// current device (0: it cannot run, the single-CTA kernel takes the work).
int pair_slots() {
  static std::mutex mu;
  static int cached[64];
  static bool known[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (known[dev]) return cached[dev];
  int n = 0;
  if (ensure_smem_limit((const void*)expand_pair_kernel, (int)kPSmemBytes) != cudaSuccess) {
    cudaGetLastError();   // clear only the error of this failed query
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    cfg.blockDim = dim3(kPThreads, 1, 1);
    cfg.dynamicSmemBytes = kPSmemBytes;
    if (cudaOccupancyMaxActiveClusters(&n, (const void*)expand_pair_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
  }
  cached[dev] = n;
  known[dev] = true;
  return n;
}

}  // namespace

bool tc_expand_supports(const Problem& p) {
  const auto& d = p.d;
  if (d.dtype != GQLA_BF16 || d.r != kR || d.d_nope != kDn || d.d_v != kDv || d.d_rope != kDr) return false;
  if (p.ly.page_size != 0 && p.ly.page_size % 64 != 0) return false;
  const long long nrows = p.ly.page_size == 0 ? (long long)p.ly.batch * p.ly.capacity
                                              : (long long)p.ly.num_pages * p.ly.page_size;
  if (nrows + 128 >= (1LL << 31)) return false;
  return true;
}

cudaError_t tc_expand(const Problem& p, const void* latent, const void* W_uk, const void* W_uv, void* k_pool,
                      void* v_pool, int tail, int32_t* st, cudaStream_t s) {
  const auto& d = p.d;
  const long long nrows = p.ly.page_size == 0 ? (long long)p.ly.batch * p.ly.capacity
                                              : (long long)p.ly.num_pages * p.ly.page_size;
  CUtensorMap lat_map, uk_map, uv_map;
  if (!tmap_bf16_sw128(&lat_map, latent, kE, nrows, kE, 64) ||
      !tmap_bf16_sw128(&uk_map, W_uk, kDn, (long long)d.G * kR, kDn, kKC) ||
      !tmap_bf16_sw128(&uv_map, W_uv, kDv, (long long)d.G * kR, kDv, kKC))
    return cudaErrorInvalidValue;
  CUtensorMap k_store, v_store;
  if (!store_maps(p, k_pool, v_pool, &k_store, &v_store)) return cudaErrorInvalidValue;
  ExpandParams prm;
  prm.ly = p.ly;
  prm.kp = (bf16*)k_pool;
  prm.kr = p.kr;
  prm.vp = (bf16*)v_pool;
  prm.latent = (const bf16*)latent;
  prm.G = d.G;
  const int span = tail > 0 ? (tail < p.ly.max_seq_len ? tail : p.ly.max_seq_len) : p.ly.max_seq_len;
  prm.tail = tail > 0 ? span : 0;
  prm.tps = (span + 63 + kTM - 1) / kTM;
  prm.n_items = (long long)p.ly.batch * prm.tps * d.G;
  prm.dense = nullptr;
  prm.dense_rows = 0;
  prm.halves = 1;
  prm.s_q = d.s_q;
  prm.st = st;
  // the whole cache goes to the pair kernel when pairs can be resident
  const int slots = tail == 0 ? pair_slots() : 0;
  if (slots > 0) {
    ExpandParams pp = prm;
    pp.n_items = ((long long)p.ly.batch * prm.tps + 1) / 2 * d.G;
    const long long pairs = pp.n_items < slots ? pp.n_items : slots;
    if (pairs < 1) return cudaSuccess;
    expand_pair_kernel<<<(unsigned)(2 * pairs), kPThreads, kPSmemBytes, s>>>(lat_map, uk_map, uv_map, k_store,
                                                                               v_store, pp);
    count_launch();
    return cudaGetLastError();
  }
  cudaError_t e = ensure_smem_limit((const void*)expand_tc_kernel, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long grid = prm.n_items < num_sms() ? prm.n_items : num_sms();
  if (grid < 1) return cudaSuccess;
  e = launch_pdl(expand_tc_kernel, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, s, lat_map, uk_map, uv_map,
                 k_store, v_store, prm);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t tc_expand_dense(const Problem& p, const void* rows, void* k_pool, void* v_pool, const void* W_uk,
                            const void* W_uv, int32_t* st, cudaStream_t s) {
  const auto& d = p.d;
  const long long n = (long long)p.ly.batch * d.s_q;
  if (n > (1LL << 30)) return cudaErrorInvalidValue;
  CUtensorMap lat_map, uk_map, uv_map;
  if (!tmap_bf16_sw128(&lat_map, rows, kE, n, kE, 64) ||
      !tmap_bf16_sw128(&uk_map, W_uk, kDn, (long long)d.G * kR, kDn, kKC) ||
      !tmap_bf16_sw128(&uv_map, W_uv, kDv, (long long)d.G * kR, kDv, kKC))
    return cudaErrorInvalidValue;
  CUtensorMap k_store, v_store;   // unused by the dense form (its rows are scattered)
  if (!store_maps(p, k_pool, v_pool, &k_store, &v_store)) return cudaErrorInvalidValue;
  ExpandParams prm;
  prm.ly = p.ly;
  prm.kp = (bf16*)k_pool;
  prm.kr = p.kr;
  prm.vp = (bf16*)v_pool;
  prm.latent = nullptr;
  prm.G = d.G;
  prm.tail = 0;
  prm.tps = (int)((n + kTM - 1) / kTM);
  prm.halves = 2;
  prm.n_items = (long long)prm.tps * d.G * prm.halves;
  prm.dense = (const bf16*)rows;
  prm.dense_rows = (int)n;
  prm.s_q = d.s_q;
  prm.st = st;
  cudaError_t e = ensure_smem_limit((const void*)expand_tc_kernel, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long grid = prm.n_items < num_sms() ? prm.n_items : num_sms();
  e = launch_pdl(expand_tc_kernel, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, s, lat_map, uk_map, uv_map,
                 k_store, v_store, prm);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace gqla
