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
//    and round to bf16.  A 64-token half tile whose rows are all written
//    goes through a 128-byte-swizzled staging tile to TMA stores of 64 x 64
//    boxes (each row from one thread would make every warp store touch 32
//    rows G * 640 bytes apart); other rows are stored by their thread.  The
//    shared RoPE key is copied by the threads.
// Tiles start on a 64-token boundary; rows outside [first token, L) of the
// sequence are computed but not written.
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
#include "ptx.cuh"
#include "tc.h"

namespace gqla {

namespace {

using bf16 = __nv_bfloat16;

constexpr int kR = 512, kDn = 128, kDv = 128, kDr = 64, kE = kR + kDr;
constexpr int kTM = 128;                          // tokens per tile
constexpr int kN = kDn + kDv;                     // 256 outputs per group
constexpr int kKC = 64;                           // K per stage
constexpr int kStages = 3;
constexpr int kABytes = kTM * 128;                // 16 KB
constexpr int kBBox = kKC * 128;                  // 8 KB: 64 K-rows x 64 columns
constexpr int kBBytes = 4 * kBBox;                // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;    // 48 KB
constexpr int kBoxBytes = 64 * 128;              // a 64-row x 64-column bf16 box
constexpr int kOutBytes = 8 * kBoxBytes;          // staging: 2 half tiles x (K nope, V) x 2 column boxes
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + kOutBytes + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 6 * 32;

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
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int s_bad;                            // an epilogue warp's wait failed: no more TMA stores
  uint8_t* s_out = smem + kStages * kStageBytes;   // 1024-aligned staging tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full_bar[s], 1);
      ptx::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&acc_full[a], 1);
      ptx::mbar_init(&acc_empty[a], 4);
    }
    ptx::mbar_init(&drain, 1);
    s_bad = 0;
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
    long long li = 0;
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
      if (ok) ok = ptx::mbar_wait(&acc_full[ab], (uint32_t)((li >> 1) & 1));
      ok = __all_sync(0xffffffffu, ok);
      const int t = t0 + r;
      bool write = ok && t >= tlo && t < thi;
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
      // this warp's 32 rows lie in half tile hh; it goes out by TMA stores when
      // every one of its 64 rows is written (pool form, both output halves)
      const int hh = r >> 6;
      const int h_lo = t0 + 64 * hh;
      const bool tma_half = ok && p.dense_rows == 0 && hf < 0 && h_lo >= tlo && h_lo + 64 <= thi &&
                            half_row(p.ly, b, h_lo, thi) >= 0;
      if (ok) {
        ptx::tc_fence_after();
        const int ncol = hf < 0 ? kN / 32 : kN / 64;   // 32-column groups in the accumulator
#pragma unroll 1
        for (int c = 0; c < ncol; ++c) {
          uint32_t v[32];
          ptx::tmem_ld32(tl + (uint32_t)(ab * kN + 32 * c), v);
          ptx::tmem_ld_wait();
          uint4 w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            w[e].x = ptx::pack_bf16(__uint_as_float(v[8 * e + 0]), __uint_as_float(v[8 * e + 1]));
            w[e].y = ptx::pack_bf16(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3]));
            w[e].z = ptx::pack_bf16(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5]));
            w[e].w = ptx::pack_bf16(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7]));
          }
          if (tma_half) {
            // box (half, c / 2) of the staging tile, columns 32 (c % 2) .. of it
            uint8_t* box = s_out + (hh * 4 + c / 2) * kBoxBytes;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              *reinterpret_cast<uint4*>(box + ptx::swz128(r & 63, 4 * (c & 1) + e)) = w[e];
          } else if (write) {
            const int oc = hf == 1 ? c + kDn / 32 : c;   // column group of [K nope | V]
            bf16* dst = oc < kDn / 32 ? p.kp + row * p.kr.pitch + p.kr.nope_at(g) + 32 * oc
                                      : p.vp + (row * G + g) * kDv + 32 * (oc - kDn / 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) *reinterpret_cast<uint4*>(dst + 8 * e) = w[e];
          }
        }
        if (write && hf != 1 && (p.kr.rope_gs != 0 || g == 0)) {   // a shared RoPE key: by group 0
          const uint4* src = reinterpret_cast<const uint4*>(p.dense_rows > 0 ? p.dense + (long long)t * kE + kR
                                                                             : p.latent + row * kE + kR);
          uint4* dst = reinterpret_cast<uint4*>(p.kp + row * p.kr.pitch + p.kr.rope_at(g));
#pragma unroll
          for (int e = 0; e < kDr / 8; ++e) dst[e] = src[e];
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&acc_empty[ab]);
      // staged half tiles out with TMA stores, then the staging is free again
      if (!ok && lane == 0) atomicExch(&s_bad, 1);
      ptx::fence_proxy_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (threadIdx.x == 2 * 32 && !s_bad) {
        for (int h = 0; h < 2; ++h) {
          const int lo = t0 + 64 * h;
          if (!(p.dense_rows == 0 && hf < 0 && lo >= tlo && lo + 64 <= thi)) continue;
          const int y = half_row(p.ly, b, lo, thi);
          if (y < 0) continue;                    // a page outside the pool (flagged by its rows)
          ptx::tma_store_2d(&k_store, s_out + (h * 4 + 0) * kBoxBytes, p.kr.nope_at(g), y);
          ptx::tma_store_2d(&k_store, s_out + (h * 4 + 1) * kBoxBytes, p.kr.nope_at(g) + 64, y);
          ptx::tma_store_2d(&v_store, s_out + (h * 4 + 2) * kBoxBytes, g * kDv, y);
          ptx::tma_store_2d(&v_store, s_out + (h * 4 + 3) * kBoxBytes, g * kDv + 64, y);
        }
        ptx::bulk_commit_group();
        ptx::bulk_wait_group_read();              // the next item may overwrite the staging
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      ++li;
    }
    if (!ok && lane == 0) flag_status(p.st, GQLA_DEV_TIMEOUT);
    if (threadIdx.x == 2 * 32) ptx::bulk_wait_group();   // every store has landed before the CTA ends
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
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
  if (!gqa_pool_maps(p, k_pool, v_pool, &k_store, &v_store)) return cudaErrorInvalidValue;
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
  cudaError_t e = ensure_smem_limit((const void*)expand_tc_kernel, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long grid = prm.n_items < num_sms() ? prm.n_items : num_sms();
  if (grid < 1) return cudaSuccess;
  expand_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, s>>>(lat_map, uk_map, uv_map, k_store, v_store, prm);
  count_launch();
  return cudaGetLastError();
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
  if (!gqa_pool_maps(p, k_pool, v_pool, &k_store, &v_store)) return cudaErrorInvalidValue;
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
  expand_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, s>>>(lat_map, uk_map, uv_map, k_store, v_store, prm);
  count_launch();
  return cudaGetLastError();
}

}  // namespace gqla
