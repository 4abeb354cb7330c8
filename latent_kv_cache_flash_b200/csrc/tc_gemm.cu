// Small bf16 GEMMs around the decode kernels, on mma.sync m16n8k16 tiles
// (fp32 accumulate):
//  * absorb_q:      q~[row] = W_uk^g q_nope[row]          (per group, r outputs)
//  * combine_lat + up_proj: LSE merge of the split partials of the latent
//                   output (bf16), then out[row] = o_lat[row] W_uv^g
//  * expand:        K[t,g] = [c_t W_uk^g ; k_rope_t], V[t,g] = c_t W_uv^g
//                   (the GQA path's per-group expanded cache, for all tokens
//                   or for the newest `tail` tokens of every sequence)
// All three read their row-major operands through ldmatrix from padded shared
// memory; the weight operand is shared by every row of a group.
#include <math.h>

#include "ptx.cuh"
#include "tc.h"

namespace gqla {

namespace {

using bf16 = __nv_bfloat16;

__device__ __forceinline__ void ldsm_a(uint32_t base, int pitch_bytes, int row0, int k0, uint32_t* a) {
  const int lane = threadIdx.x & 31;
  const int row = row0 + (lane & 7) + ((lane >> 3) & 1) * 8;
  const int col = k0 + (lane >> 4) * 8;
  ptx::ldsm_x4(base + row * pitch_bytes + col * 2, a[0], a[1], a[2], a[3]);
}
// B stored [n][k] (K contiguous): fragments of n-tiles n0 and n0+8 at k-step k0.
__device__ __forceinline__ void ldsm_b_nk(uint32_t base, int pitch_bytes, int n0, int k0, uint32_t* b) {
  const int lane = threadIdx.x & 31;
  const int n = n0 + (lane & 7) + (lane >> 4) * 8;
  const int k = k0 + ((lane >> 3) & 1) * 8;
  ptx::ldsm_x4(base + n * pitch_bytes + k * 2, b[0], b[1], b[2], b[3]);
}
// B stored [k][n] (N contiguous): same fragments through the transposing load.
__device__ __forceinline__ void ldsm_b_kn(uint32_t base, int pitch_bytes, int n0, int k0, uint32_t* b) {
  const int lane = threadIdx.x & 31;
  const int k = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
  const int n = n0 + (lane >> 4) * 8;
  ptx::ldsm_x4_t(base + k * pitch_bytes + n * 2, b[0], b[1], b[2], b[3]);
}

// ------------------------------------------------------------- absorb_q
// CTA: 32 rows of group g x 128 outputs; 4 warps = 2 row blocks x 2 output
// halves.  K = d_nope.
constexpr int kAqRows = 32, kAqN = 128, kAqMaxK = 256;

__global__ void __launch_bounds__(128) absorb_q_mma_kernel(const bf16* __restrict__ q, const bf16* __restrict__ W_uk,
                                                           bf16* __restrict__ qt, int rows_g, int n_h, int m,
                                                           int d_n, int d_qk, int r) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int g = blockIdx.z, n0 = blockIdx.y * kAqN;
  const int pitch = (d_n + 8) * 2;
  uint8_t* sA = sm;
  uint8_t* sB = sm + kAqRows * pitch;
  const int gran = d_n / 8;
  for (int i = threadIdx.x; i < kAqRows * gran; i += blockDim.x) {
    const int rr = i / gran, c = i % gran;
    const int lr = blockIdx.x * kAqRows + rr;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (lr < rows_g) {
      const long long grow = (long long)(lr / m) * n_h + g * m + lr % m;
      v = *reinterpret_cast<const uint4*>(q + grow * d_qk + c * 8);
    }
    *reinterpret_cast<uint4*>(sA + rr * pitch + c * 16) = v;
  }
  for (int i = threadIdx.x; i < kAqN * gran; i += blockDim.x) {
    const int nn = i / gran, c = i % gran;
    *reinterpret_cast<uint4*>(sB + nn * pitch + c * 16) =
        *reinterpret_cast<const uint4*>(W_uk + ((size_t)g * r + n0 + nn) * d_n + c * 8);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wr = warp & 1, wn = warp >> 1;
  float acc[kAqN / 16][4];
#pragma unroll
  for (int n = 0; n < kAqN / 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const uint32_t a_base = ptx::smem_u32(sA), b_base = ptx::smem_u32(sB);
  for (int k0 = 0; k0 < d_n; k0 += 16) {
    uint32_t a[4];
    ldsm_a(a_base, pitch, wr * 16, k0, a);
#pragma unroll
    for (int np = 0; np < kAqN / 32; ++np) {
      uint32_t b[4];
      ldsm_b_nk(b_base, pitch, wn * (kAqN / 2) + np * 16, k0, b);
      ptx::mma_bf16_16816(acc[2 * np], a, b[0], b[1]);
      ptx::mma_bf16_16816(acc[2 * np + 1], a, b[2], b[3]);
    }
  }
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int lr = blockIdx.x * kAqRows + wr * 16 + gid + 8 * h2;
    if (lr >= rows_g) continue;
    const long long grow = (long long)(lr / m) * n_h + g * m + lr % m;
#pragma unroll
    for (int n = 0; n < kAqN / 16; ++n)
      *reinterpret_cast<uint32_t*>(qt + grow * r + n0 + wn * (kAqN / 2) + n * 8 + 2 * tig) =
          ptx::pack_bf16(acc[n][2 * h2], acc[n][2 * h2 + 1]);
  }
}

// --------------------------------------------------------- combine_lat
// LSE merge of the split partials of the absorb path's latent output, one
// warp per (row, 128-column quarter); output rounded to bf16 for the
// up-projection's A operand.
constexpr int kLat = 512;

__global__ void __launch_bounds__(256) combine_lat_kernel(int S, const float* __restrict__ o_part,
                                                          const float* __restrict__ lse_part,
                                                          bf16* __restrict__ o_lat, float* __restrict__ lse_out,
                                                          long long rows) {
  const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long row = wid >> 2;
  const int q4 = (int)(wid & 3);
  if (row >= rows) return;
  float mx = -INFINITY;
  for (int s = lane; s < S; s += 32) mx = fmaxf(mx, lse_part[(long long)s * rows + row]);
  mx = warp_max(mx);
  float Z = 0.f;
  if (mx != -INFINITY)
    for (int s = lane; s < S; s += 32) Z += expf(lse_part[(long long)s * rows + row] - mx);
  Z = warp_sum(Z);
  const float inv = mx == -INFINITY ? 0.f : 1.f / Z;
  const int col = q4 * 128 + lane * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx != -INFINITY) {
    int s = 0;
    for (; s + 4 <= S; s += 4) {
      float4 v[4];
      float w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float ls = lse_part[(long long)(s + u) * rows + row];
        w[u] = ls == -INFINITY ? 0.f : expf(ls - mx) * inv;
        v[u] = *reinterpret_cast<const float4*>(o_part + ((long long)(s + u) * rows + row) * kLat + col);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc.x = fmaf(w[u], v[u].x, acc.x);
        acc.y = fmaf(w[u], v[u].y, acc.y);
        acc.z = fmaf(w[u], v[u].z, acc.z);
        acc.w = fmaf(w[u], v[u].w, acc.w);
      }
    }
    for (; s < S; ++s) {
      const float ls = lse_part[(long long)s * rows + row];
      const float w = ls == -INFINITY ? 0.f : expf(ls - mx) * inv;
      const float4 v = *reinterpret_cast<const float4*>(o_part + ((long long)s * rows + row) * kLat + col);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
  }
  *reinterpret_cast<uint2*>(o_lat + row * kLat + col) =
      make_uint2(ptx::pack_bf16(acc.x, acc.y), ptx::pack_bf16(acc.z, acc.w));
  if (q4 == 0 && lane == 0 && lse_out) lse_out[row] = mx == -INFINITY ? -INFINITY : mx + logf(Z);
}

// ------------------------------------------------------------- up_proj
// out[row] = o_lat[row] W_uv^g.  CTA: 16 rows of group g x 128 outputs,
// 4 warps of 32 outputs; K = 512 in 64-wide chunks, double-buffered cp.async.
constexpr int kUpRows = 16, kUpN = 128, kUpKC = 64;
constexpr int kUpApitch = (kUpKC + 8) * 2;     // 144 B
constexpr int kUpBpitch = (kUpN + 8) * 2;      // 272 B
constexpr int kUpAbytes = kUpRows * kUpApitch;
constexpr int kUpBbytes = kUpKC * kUpBpitch;
constexpr size_t kUpSmem = 2 * (size_t)(kUpAbytes + kUpBbytes);

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool pred) {
  const int sz = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(128) up_proj_mma_kernel(const bf16* __restrict__ o_lat,
                                                          const bf16* __restrict__ W_uv, bf16* __restrict__ out,
                                                          int rows_g, int n_h, int m) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = ptx::smem_u32(sm);
  auto grow_of = [&](int rr) -> long long {
    const int lr = blockIdx.x * kUpRows + rr;
    return lr < rows_g ? (long long)(lr / m) * n_h + g * m + lr % m : -1;
  };
  const bf16* Wg = W_uv + (size_t)g * kLat * kUpN;
  auto load_chunk = [&](int kc, int buf) {
    const uint32_t a = base + buf * (kUpAbytes + kUpBbytes);
    const uint32_t b = a + kUpAbytes;
    for (int i = threadIdx.x; i < kUpRows * (kUpKC / 8); i += blockDim.x) {
      const int rr = i / (kUpKC / 8), c = i % (kUpKC / 8);
      const long long grow = grow_of(rr);
      cp_async16(a + rr * kUpApitch + c * 16, o_lat + (grow < 0 ? 0 : grow) * kLat + kc + c * 8, grow >= 0);
    }
    for (int i = threadIdx.x; i < kUpKC * (kUpN / 8); i += blockDim.x) {
      const int kk = i / (kUpN / 8), c = i % (kUpN / 8);
      cp_async16(b + kk * kUpBpitch + c * 16, Wg + (size_t)(kc + kk) * kUpN + c * 8, true);
    }
    cp_async_commit();
  };
  float acc[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  load_chunk(0, 0);
  for (int c = 0; c < kLat / kUpKC; ++c) {
    if (c + 1 < kLat / kUpKC) {
      load_chunk((c + 1) * kUpKC, (c + 1) & 1);
      cp_async_wait1();
    } else {
      cp_async_wait0();
    }
    __syncthreads();
    const uint32_t a = base + (c & 1) * (kUpAbytes + kUpBbytes);
    const uint32_t b = a + kUpAbytes;
#pragma unroll
    for (int k0 = 0; k0 < kUpKC; k0 += 16) {
      uint32_t af[4];
      ldsm_a(a, kUpApitch, 0, k0, af);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t bf[4];
        ldsm_b_kn(b, kUpBpitch, warp * 32 + np * 16, k0, bf);
        ptx::mma_bf16_16816(acc[2 * np], af, bf[0], bf[1]);
        ptx::mma_bf16_16816(acc[2 * np + 1], af, bf[2], bf[3]);
      }
    }
    __syncthreads();
  }
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const long long grow = grow_of(gid + 8 * h2);
    if (grow < 0) continue;
#pragma unroll
    for (int n = 0; n < 4; ++n)
      *reinterpret_cast<uint32_t*>(out + grow * kUpN + warp * 32 + n * 8 + 2 * tig) =
          ptx::pack_bf16(acc[n][2 * h2], acc[n][2 * h2 + 1]);
  }
}

// --------------------------------------------------------------- expand
// CTA: 64 tokens x 64 outputs of group g (quarter q of its 256 outputs: q = 0,1
// key-nope through W_uk^g, q = 2,3 values through W_uv^g); 4 warps of 16 rows.
// K = 512 in 64-wide chunks, double-buffered with cp.async.  Quarter 0 also
// copies the shared RoPE key into the group's key.
constexpr int kExR = 512, kExDn = 128, kExDv = 128, kExDr = 64, kExE = kExR + kExDr;
constexpr int kExT = 64, kExKC = 64, kExN = 64;
constexpr int kExApitch = (kExKC + 8) * 2;                 // 144 B
constexpr int kExBpitch = (kExN + 8) * 2;                  // 144 B
constexpr int kExAbytes = kExT * kExApitch;
constexpr int kExBbytes = kExKC * kExBpitch;
constexpr size_t kExSmem = 2 * (size_t)(kExAbytes + kExBbytes);

__global__ void __launch_bounds__(128) expand_mma_kernel(KvLayout ly, const bf16* __restrict__ latent,
                                                         const bf16* __restrict__ W_uk,
                                                         const bf16* __restrict__ W_uv, bf16* __restrict__ kp,
                                                         bf16* __restrict__ vp, int G, int tail, int blocks_per_seq,
                                                         long long n_tiles, int32_t* st) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ long long srow[kExT];
  // blockIdx.x = (group, quarter) fastest so that the 4*G CTAs sharing a
  // token tile run together and its latent rows are read from DRAM once;
  // token tiles stride over blockIdx.y
  const int g = blockIdx.x >> 2, quarter = blockIdx.x & 3;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool is_k = quarter < 2;
  const bf16* Wsrc = is_k ? W_uk + (size_t)g * kExR * kExDn + quarter * kExN
                          : W_uv + (size_t)g * kExR * kExDv + (quarter - 2) * kExN;
  const int wld = is_k ? kExDn : kExDv;
  const uint32_t base = ptx::smem_u32(sm);
  for (long long tile = blockIdx.y; tile < n_tiles; tile += gridDim.y) {
    // which token each tile row holds (pool row, or -1)
    __syncthreads();
    if (threadIdx.x < kExT) {
      long long row = -1;
      int b, t;
      if (tail > 0) {
        const long long idx = tile * kExT + threadIdx.x;
        b = (int)(idx / tail);
        t = b < ly.batch ? ly.seq_lens[b] - tail + (int)(idx % tail) : -1;
      } else {
        b = (int)(tile / blocks_per_seq);
        t = (int)(tile % blocks_per_seq) * kExT + threadIdx.x;
      }
      if (b < ly.batch) {
        const int L = ly.seq_lens[b];
        const bool bad = L < 1 || L > ly.max_seq_len ||
                         (ly.page_size == 0 ? L > ly.capacity : (L + ly.page_size - 1) / ly.page_size > ly.mbps);
        const bool reporter = g == 0 && quarter == 0 &&
                              (tail > 0 ? (int)((tile * kExT + threadIdx.x) % tail) == 0 : t == 0);
        if (bad) {
          if (reporter) flag_status(st, L < 1 ? GQLA_DEV_SHORT_SEQ : GQLA_DEV_OVERFLOW);
        } else if (t >= 0 && t < L) {
          row = token_row(ly, b, t, (g == 0 && quarter == 0) ? st : nullptr);
        }
      }
      srow[threadIdx.x] = row;
    }
    __syncthreads();
    auto load_chunk = [&](int kc, int buf) {
      const uint32_t a = base + buf * (kExAbytes + kExBbytes);
      const uint32_t bb = a + kExAbytes;
      for (int i = threadIdx.x; i < kExT * (kExKC / 8); i += blockDim.x) {
        const int tt = i / (kExKC / 8), c = i % (kExKC / 8);
        const long long row = srow[tt];
        cp_async16(a + tt * kExApitch + c * 16, latent + (row < 0 ? 0 : row) * kExE + kc + c * 8, row >= 0);
      }
      for (int i = threadIdx.x; i < kExKC * (kExN / 8); i += blockDim.x) {
        const int kk = i / (kExN / 8), c = i % (kExN / 8);
        cp_async16(bb + kk * kExBpitch + c * 16, Wsrc + (size_t)(kc + kk) * wld + c * 8, true);
      }
      cp_async_commit();
    };
    float acc[kExN / 8][4];
#pragma unroll
    for (int n = 0; n < kExN / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    load_chunk(0, 0);
    for (int c = 0; c < kExR / kExKC; ++c) {
      if (c + 1 < kExR / kExKC) {
        load_chunk((c + 1) * kExKC, (c + 1) & 1);
        cp_async_wait1();
      } else {
        cp_async_wait0();
      }
      __syncthreads();
      const uint32_t a = base + (c & 1) * (kExAbytes + kExBbytes);
      const uint32_t bb = a + kExAbytes;
#pragma unroll
      for (int k0 = 0; k0 < kExKC; k0 += 16) {
        uint32_t af[4];
        ldsm_a(a, kExApitch, warp * 16, k0, af);
#pragma unroll
        for (int np = 0; np < kExN / 16; ++np) {
          uint32_t b[4];
          ldsm_b_kn(bb, kExBpitch, np * 16, k0, b);
          ptx::mma_bf16_16816(acc[2 * np], af, b[0], b[1]);
          ptx::mma_bf16_16816(acc[2 * np + 1], af, b[2], b[3]);
        }
      }
      __syncthreads();
    }
    const int gid = lane >> 2, tig = lane & 3;
    constexpr int kDqk = kExDn + kExDr;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const long long row = srow[warp * 16 + gid + 8 * h2];
      if (row < 0) continue;
      bf16* dst = is_k ? kp + (row * G + g) * kDqk + quarter * kExN : vp + (row * G + g) * kExDv + (quarter - 2) * kExN;
#pragma unroll
      for (int n = 0; n < kExN / 8; ++n)
        *reinterpret_cast<uint32_t*>(dst + n * 8 + 2 * tig) = ptx::pack_bf16(acc[n][2 * h2], acc[n][2 * h2 + 1]);
    }
    if (quarter == 0) {
      // the shared RoPE key is copied into every group's key
      for (int i = threadIdx.x; i < kExT * (kExDr / 8); i += blockDim.x) {
        const int tt = i / (kExDr / 8), c = i % (kExDr / 8);
        const long long row = srow[tt];
        if (row < 0) continue;
        *reinterpret_cast<uint4*>(kp + (row * G + g) * kDqk + kExDn + c * 8) =
            *reinterpret_cast<const uint4*>(latent + row * kExE + kExR + c * 8);
      }
    }
  }
}

}  // namespace

bool gemm_absorb_q_supports(const Problem& p) {
  return p.d.d_nope % 16 == 0 && p.d.d_nope <= kAqMaxK && p.d.r % kAqN == 0;
}

cudaError_t absorb_q_mma(const Problem& p, const void* q, const void* W_uk, bf16* qt, cudaStream_t s) {
  const auto& d = p.d;
  const int rows_g = p.ly.batch * d.s_q * p.m;
  const int pitch = (d.d_nope + 8) * 2;
  const size_t smem = (size_t)(kAqRows + kAqN) * pitch;
  cudaError_t e = ensure_smem_limit((const void*)absorb_q_mma_kernel, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((rows_g + kAqRows - 1) / kAqRows, d.r / kAqN, d.G);
  absorb_q_mma_kernel<<<grid, 128, smem, s>>>((const bf16*)q, (const bf16*)W_uk, qt, rows_g, d.n_h, p.m, d.d_nope,
                                              p.d_qk, d.r);
  count_launch();
  return cudaGetLastError();
}

bool gemm_combine_up_supports(const Problem& p) {
  return p.d.r == kLat && p.d.d_v == kUpN;
}

cudaError_t combine_up_mma(const Problem& p, int S, const float* o_part, const float* lse_part, const void* W_uv,
                           void* out, float* lse_out, bf16* o_lat, cudaStream_t s) {
  const auto& d = p.d;
  const long long warps = p.rows * 4;
  combine_lat_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(S, o_part, lse_part, o_lat, lse_out, p.rows);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int rows_g = p.ly.batch * d.s_q * p.m;
  e = ensure_smem_limit((const void*)up_proj_mma_kernel, (int)kUpSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((rows_g + kUpRows - 1) / kUpRows, d.G);
  up_proj_mma_kernel<<<grid, 128, kUpSmem, s>>>(o_lat, (const bf16*)W_uv, (bf16*)out, rows_g, d.n_h, p.m);
  count_launch();
  return cudaGetLastError();
}

bool tc_expand_supports(const Problem& p) {
  const auto& d = p.d;
  return d.dtype == GQLA_BF16 && d.r == kExR && d.d_nope == kExDn && d.d_v == kExDv && d.d_rope == kExDr;
}

cudaError_t tc_expand(const Problem& p, const void* latent, const void* W_uk, const void* W_uv, void* k_pool,
                      void* v_pool, int tail, int32_t* st, cudaStream_t s) {
  const int span = tail > 0 ? (tail < p.ly.max_seq_len ? tail : p.ly.max_seq_len) : p.ly.max_seq_len;
  const int bps = (span + kExT - 1) / kExT;
  long long gx = tail > 0 ? ((long long)p.ly.batch * span + kExT - 1) / kExT : (long long)p.ly.batch * bps;

  cudaError_t e = ensure_smem_limit((const void*)expand_mma_kernel, (int)kExSmem);
  if (e != cudaSuccess) return e;
  if (gx < 1) return cudaSuccess;
  dim3 grid(p.d.G * 4, (unsigned)(gx < 65535 ? gx : 65535));
  expand_mma_kernel<<<grid, 128, kExSmem, s>>>(p.ly, (const bf16*)latent, (const bf16*)W_uk, (const bf16*)W_uv,
                                               (bf16*)k_pool, (bf16*)v_pool, p.d.G, tail > 0 ? span : 0, bps, gx, st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace gqla
