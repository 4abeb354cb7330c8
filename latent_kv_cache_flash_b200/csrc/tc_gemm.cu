// Small bf16 GEMMs around the decode kernels, on mma.sync m16n8k16 tiles
// (fp32 accumulate):
//  * absorb_q:  q~[row] = W_uk^g q_nope[row]              (per group, r outputs)
//  * merge_up:  LSE merge of the split partials of the latent output (rounded
//               to bf16 in shared memory), then out[row] = o_lat[row] W_uv^g,
//               in one launch
// They read their row-major operands through ldmatrix from padded shared
// memory; the weight operand is shared by every row of a group, so a CTA
// takes 64 rows of one group to load each weight slice once per 64 rows.
#include <math.h>

#include "ptx.cuh"
#include "tc.h"

namespace gqla {

namespace {

using bf16 = __nv_bfloat16;

// 16-byte global -> shared copies that do not hold the issuing thread; a
// false predicate fills the destination with zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool pred) {
  const int sz = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

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
// CTA: 64 rows of group g x 128 outputs; 8 warps = 4 row blocks x 2 output
// halves.  K = d_nope.  Both operands come in through cp.async, all in
// flight at once.
constexpr int kAqRows = 64, kAqN = 128, kAqMaxK = 256, kAqThreads = 256;

__global__ void __launch_bounds__(kAqThreads) absorb_q_mma_kernel(const bf16* __restrict__ q, const bf16* __restrict__ W_uk,
                                                           bf16* __restrict__ qt, int rows_g, int n_h, int m,
                                                           int d_n, int d_qk, int r) {
  // launched while the kernel ahead of it may still run: wait for it before
  // any memory access, then let the decode launch and start its loads
  ptx::pdl_wait();
  ptx::pdl_trigger();
  extern __shared__ __align__(16) uint8_t sm[];
  const int g = blockIdx.z, n0 = blockIdx.y * kAqN;
  const int pitch = (d_n + 8) * 2;
  uint8_t* sA = sm;
  uint8_t* sB = sm + kAqRows * pitch;
  const int gran = d_n / 8;
  const uint32_t a_base = ptx::smem_u32(sA), b_base = ptx::smem_u32(sB);
  for (int i = threadIdx.x; i < kAqRows * gran; i += blockDim.x) {
    const int rr = i / gran, c = i % gran;
    const int lr = blockIdx.x * kAqRows + rr;
    const long long grow = lr < rows_g ? (long long)(lr / m) * n_h + g * m + lr % m : 0;
    cp_async16(a_base + rr * pitch + c * 16, q + grow * d_qk + c * 8, lr < rows_g);
  }
  for (int i = threadIdx.x; i < kAqN * gran; i += blockDim.x) {
    const int nn = i / gran, c = i % gran;
    cp_async16(b_base + nn * pitch + c * 16, W_uk + ((size_t)g * r + n0 + nn) * d_n + c * 8, true);
  }
  cp_async_commit();
  cp_async_wait0();
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wr = warp & 3, wn = warp >> 2;
  float acc[kAqN / 16][4];
#pragma unroll
  for (int n = 0; n < kAqN / 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
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

// ------------------------------------------------------------ merge_up
// out[row] = (sum_s w_s o_part[s][row]) W_uv^g with w_s = exp(lse_s - lse),
// lse = log sum_s exp(lse_s): the split-KV merge of the latent output and the
// group's up-projection in one launch.  CTA: R rows of group g (64, or 32
// or 16 when fewer CTAs would leave SMs idle) x the 128 outputs, 16 warps.
// W_uv^g (128 KB) streams in through cp.async while the warps merge the
// partials, R/16 rows each with the loads of 4 splits in flight, into a bf16
// A tile in shared memory (the up-projection's operand is the merged latent
// rounded to bf16); then R/16 row blocks x 4 output quarters of mma.sync
// tiles, one warp each.
constexpr int kLat = 512;
constexpr int kUpN = 128, kUpThreads = 512;
constexpr int kUpApitch = (kLat + 8) * 2;      // 1040 B
constexpr int kUpBpitch = (kUpN + 8) * 2;      // 272 B
constexpr int kUpBbytes = kLat * kUpBpitch;
constexpr size_t up_smem(int rows) { return (size_t)rows * kUpApitch + kUpBbytes; }

template <int kUpRows>
__global__ void __launch_bounds__(kUpThreads) merge_up_kernel(int S, const float* __restrict__ o_part,
                                                              const float* __restrict__ lse_part,
                                                              const bf16* __restrict__ W_uv, bf16* __restrict__ out,
                                                              float* __restrict__ lse_out, long long rows,
                                                              int rows_g, int n_h, int m) {
  extern __shared__ __align__(16) uint8_t sm[];
  ptx::pdl_trigger();   // the next call's first kernel may launch (it waits for this one)
  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t a = ptx::smem_u32(sm), b = a + kUpRows * kUpApitch;
  auto grow_of = [&](int rr) -> long long {
    const int lr = blockIdx.x * kUpRows + rr;
    return lr < rows_g ? (long long)(lr / m) * n_h + g * m + lr % m : -1;
  };
  const bf16* Wg = W_uv + (size_t)g * kLat * kUpN;
  for (int i = threadIdx.x; i < kLat * (kUpN / 8); i += blockDim.x) {
    const int kk = i / (kUpN / 8), c = i % (kUpN / 8);
    cp_async16(b + kk * kUpBpitch + c * 16, Wg + (size_t)kk * kUpN + c * 8, true);
  }
  cp_async_commit();
  // the decode's partials are read from here on (W_uv^g is already on its way)
  ptx::pdl_wait();

  // merge: a warp per row, a lane on 4 columns of each 128-column quarter
  for (int rr = warp; rr < kUpRows; rr += kUpThreads / 32) {
    const long long row = grow_of(rr);
    float4 acc[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) acc[q4] = make_float4(0.f, 0.f, 0.f, 0.f);
    float mx = -INFINITY, Z = 0.f;
    if (row >= 0) {
      for (int s = lane; s < S; s += 32) mx = fmaxf(mx, lse_part[(long long)s * rows + row]);
      mx = warp_max(mx);
      if (mx != -INFINITY)
        for (int s = lane; s < S; s += 32) Z += expf(lse_part[(long long)s * rows + row] - mx);
      Z = warp_sum(Z);
    }
    if (mx != -INFINITY) {
      const float inv = 1.f / Z;
      for (int s0 = 0; s0 < S; s0 += 4) {
        float w[4];
        float4 v[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (s0 + u < S) {
            const float ls = lse_part[(long long)(s0 + u) * rows + row];
            w[u] = ls == -INFINITY ? 0.f : expf(ls - mx) * inv;
            const float* src = o_part + ((long long)(s0 + u) * rows + row) * kLat + lane * 4;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) v[u][q4] = *reinterpret_cast<const float4*>(src + q4 * 128);
          }
        }
        // the splits in order, as a sequential sum
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (s0 + u < S) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              acc[q4].x = fmaf(w[u], v[u][q4].x, acc[q4].x);
              acc[q4].y = fmaf(w[u], v[u][q4].y, acc[q4].y);
              acc[q4].z = fmaf(w[u], v[u][q4].z, acc[q4].z);
              acc[q4].w = fmaf(w[u], v[u][q4].w, acc[q4].w);
            }
          }
        }
      }
    }
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
      *reinterpret_cast<uint2*>(sm + rr * kUpApitch + (q4 * 128 + lane * 4) * 2) =
          make_uint2(ptx::pack_bf16(acc[q4].x, acc[q4].y), ptx::pack_bf16(acc[q4].z, acc[q4].w));
    if (row >= 0 && lane == 0 && lse_out) lse_out[row] = mx == -INFINITY ? -INFINITY : mx + logf(Z);
  }
  cp_async_wait0();
  __syncthreads();

  // up-projection: warp = (16-row block, 32-output quarter)
  constexpr int kRb = kUpRows / 16;
  if (warp >= 4 * kRb) return;
  const int wr = warp % kRb, wn = warp / kRb;
  float acc[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll 4
  for (int k0 = 0; k0 < kLat; k0 += 16) {
    uint32_t af[4];
    ldsm_a(a, kUpApitch, wr * 16, k0, af);
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      uint32_t bf[4];
      ldsm_b_kn(b, kUpBpitch, wn * 32 + np * 16, k0, bf);
      ptx::mma_bf16_16816(acc[2 * np], af, bf[0], bf[1]);
      ptx::mma_bf16_16816(acc[2 * np + 1], af, bf[2], bf[3]);
    }
  }
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const long long grow = grow_of(wr * 16 + gid + 8 * h2);
    if (grow < 0) continue;
#pragma unroll
    for (int n = 0; n < 4; ++n)
      *reinterpret_cast<uint32_t*>(out + grow * kUpN + wn * 32 + n * 8 + 2 * tig) =
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
  e = launch_pdl(absorb_q_mma_kernel, grid, dim3(kAqThreads), smem, s, (const bf16*)q, (const bf16*)W_uk, qt, rows_g,
                 d.n_h, p.m, d.d_nope, p.d_qk, d.r);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

bool gemm_combine_up_supports(const Problem& p) {
  return p.d.r == kLat && p.d.d_v == kUpN;
}

cudaError_t combine_up_mma(const Problem& p, int S, const float* o_part, const float* lse_part, const void* W_uv,
                           void* out, float* lse_out, cudaStream_t s) {
  const auto& d = p.d;
  const int rows_g = p.ly.batch * d.s_q * p.m;
  // the largest row tile that still gives about a CTA per SM: the merge of a
  // CTA's rows is bound by its loads in flight, so small batches take more
  // CTAs of fewer rows (each loads W_uv^g from L2)
  auto ctas = [&](int rows) { return (long long)((rows_g + rows - 1) / rows) * d.G; };
  const int want = num_sms() * 4 / 5;
  const int R = ctas(64) >= want ? 64 : ctas(32) >= want ? 32 : 16;
  const void* fn = R == 64 ? (const void*)merge_up_kernel<64>
                 : R == 32 ? (const void*)merge_up_kernel<32> : (const void*)merge_up_kernel<16>;
  cudaError_t e = ensure_smem_limit(fn, (int)up_smem(R));
  if (e != cudaSuccess) return e;
  dim3 grid((rows_g + R - 1) / R, d.G);
  const bf16* w = (const bf16*)W_uv;
  bf16* o = (bf16*)out;
  if (R == 64)
    e = launch_pdl(merge_up_kernel<64>, grid, dim3(kUpThreads), up_smem(64), s, S, o_part, lse_part, w, o, lse_out, p.rows,
                   rows_g, d.n_h, p.m);
  else if (R == 32)
    e = launch_pdl(merge_up_kernel<32>, grid, dim3(kUpThreads), up_smem(32), s, S, o_part, lse_part, w, o, lse_out, p.rows,
                   rows_g, d.n_h, p.m);
  else
    e = launch_pdl(merge_up_kernel<16>, grid, dim3(kUpThreads), up_smem(16), s, S, o_part, lse_part, w, o, lse_out, p.rows,
                   rows_g, d.n_h, p.m);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace gqla
