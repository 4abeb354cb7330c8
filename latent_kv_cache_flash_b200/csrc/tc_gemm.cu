// Small bf16 GEMMs around the decode kernels, on mma.sync m16n8k16 tiles
// (fp32 accumulate):
//  * absorb_q:      q~[row] = W_uk^g q_nope[row]          (per group, r outputs)
//  * combine_lat + up_proj: LSE merge of the split partials of the latent
//                   output (bf16), then out[row] = o_lat[row] W_uv^g
// They read their row-major operands through ldmatrix from padded shared
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
// 4 warps of 32 outputs; the whole K = 512 of both operands is fetched with
// cp.async in one go (A 16 KB, B 128 KB), so the GEMM pays one load latency.
constexpr int kUpRows = 16, kUpN = 128;
constexpr int kUpApitch = (kLat + 8) * 2;      // 1040 B
constexpr int kUpBpitch = (kUpN + 8) * 2;      // 272 B
constexpr int kUpAbytes = kUpRows * kUpApitch;
constexpr int kUpBbytes = kLat * kUpBpitch;
constexpr size_t kUpSmem = (size_t)kUpAbytes + kUpBbytes;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool pred) {
  const int sz = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(128) up_proj_mma_kernel(const bf16* __restrict__ o_lat,
                                                          const bf16* __restrict__ W_uv, bf16* __restrict__ out,
                                                          int rows_g, int n_h, int m) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t a = ptx::smem_u32(sm), b = a + kUpAbytes;
  auto grow_of = [&](int rr) -> long long {
    const int lr = blockIdx.x * kUpRows + rr;
    return lr < rows_g ? (long long)(lr / m) * n_h + g * m + lr % m : -1;
  };
  const bf16* Wg = W_uv + (size_t)g * kLat * kUpN;
  for (int i = threadIdx.x; i < kUpRows * (kLat / 8); i += blockDim.x) {
    const int rr = i / (kLat / 8), c = i % (kLat / 8);
    const long long grow = grow_of(rr);
    cp_async16(a + rr * kUpApitch + c * 16, o_lat + (grow < 0 ? 0 : grow) * kLat + c * 8, grow >= 0);
  }
  for (int i = threadIdx.x; i < kLat * (kUpN / 8); i += blockDim.x) {
    const int kk = i / (kUpN / 8), c = i % (kUpN / 8);
    cp_async16(b + kk * kUpBpitch + c * 16, Wg + (size_t)kk * kUpN + c * 8, true);
  }
  cp_async_commit();
  cp_async_wait0();
  __syncthreads();
  float acc[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll 4
  for (int k0 = 0; k0 < kLat; k0 += 16) {
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

}  // namespace gqla
