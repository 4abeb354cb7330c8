// Generic CUDA-core kernels of the GQLA decode library: cache expansion,
// query absorption, split-KV decode with an online softmax, latent
// up-projection and the log-sum-exp combine.  They accumulate in fp32 and are
// the path for fp32 problems (true fp32 arithmetic, no TF32) and for bf16 dims
// the tensor-core kernels do not take.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace gqla {

namespace {

constexpr int kMaxKeyPerLane = 20;   // key/query dims up to 640
constexpr int kMaxValPerLane = 16;   // value dims up to 512
constexpr int kExpandTokens = 16;

// ---------------------------------------------------------------------------
// Cache expansion: K[b,t,g] = [c W_uk^g ; k_rope], V[b,t,g] = c W_uv^g
// ("GQLA" chatpaper.ai Abstract: GQA path over a per-group expanded cache).
// Block = (16-token block, sequence, group); threads stride the output columns.
template <typename T>
__global__ void expand_kernel(KvLayout ly, const T* __restrict__ latent, const T* __restrict__ W_uk,
                              const T* __restrict__ W_uv, T* __restrict__ kp, T* __restrict__ vp, KRow kr,
                              int G, int d_n, int d_r, int d_v, int r, int tail, int32_t* st) {
  extern __shared__ float sc[];  // [kExpandTokens][r]
  __shared__ long long srow[kExpandTokens];
  const int b = blockIdx.y, g = blockIdx.z;
  const int L = ly.seq_lens[b];
  if (L < 1 || L > ly.max_seq_len ||
      (ly.page_size == 0 ? L > ly.capacity : (L + ly.page_size - 1) / ly.page_size > ly.mbps)) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && g == 0) flag_status(st, L < 1 ? GQLA_DEV_SHORT_SEQ : GQLA_DEV_OVERFLOW);
    return;
  }
  const int t_start = tail > 0 ? max(0, L - tail) : 0;
  const int t0 = t_start + blockIdx.x * kExpandTokens;
  if (t0 >= L) return;
  const int nt = min(kExpandTokens, L - t0);
  const int E = r + d_r;
  if (threadIdx.x < nt) srow[threadIdx.x] = token_row(ly, b, t0 + threadIdx.x, st);
  __syncthreads();
  for (int i = threadIdx.x; i < nt * r; i += blockDim.x) {
    int tt = i / r, k = i % r;
    long long row = srow[tt];
    sc[tt * r + k] = row < 0 ? 0.f : to_f32(latent[row * E + k]);
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d_n + d_v; j += blockDim.x) {
    const bool isk = j < d_n;
    const T* W = isk ? (W_uk + (size_t)g * r * d_n + j) : (W_uv + (size_t)g * r * d_v + (j - d_n));
    const int ld = isk ? d_n : d_v;
    float acc[kExpandTokens];
#pragma unroll
    for (int tt = 0; tt < kExpandTokens; ++tt) acc[tt] = 0.f;
    for (int k = 0; k < r; ++k) {
      float w = to_f32(W[(size_t)k * ld]);
#pragma unroll
      for (int tt = 0; tt < kExpandTokens; ++tt) acc[tt] = fmaf(sc[tt * r + k], w, acc[tt]);
    }
    for (int tt = 0; tt < nt; ++tt) {
      long long row = srow[tt];
      if (row < 0) continue;
      if (isk) kp[row * kr.pitch + kr.nope_at(g) + j] = from_f32<T>(acc[tt]);
      else vp[(row * G + g) * d_v + (j - d_n)] = from_f32<T>(acc[tt]);
    }
  }
  // the RoPE key: in every group's part, or once per row (written by group 0)
  if (kr.rope_gs != 0 || g == 0) {
    for (int i = threadIdx.x; i < nt * d_r; i += blockDim.x) {
      int tt = i / d_r, a = i % d_r;
      long long row = srow[tt];
      if (row >= 0) kp[row * kr.pitch + kr.rope_at(g) + a] = latent[row * E + r + a];
    }
  }
}

// q~[row, k] = sum_j W_uk[g, k, j] q_nope[row, j]  (absorbed query, fp32
// accumulation, stored as OutT).
template <typename T, typename OutT>
__global__ void absorb_q_kernel(const T* __restrict__ q, const T* __restrict__ W_uk, OutT* __restrict__ qt,
                                int n_h, int m, int d_n, int d_qk, int r) {
  extern __shared__ float sq[];  // [d_n]
  const long long row = blockIdx.x;
  const int h = (int)(row % n_h), g = h / m;
  for (int j = threadIdx.x; j < d_n; j += blockDim.x) sq[j] = to_f32(q[row * d_qk + j]);
  __syncthreads();
  for (int k = threadIdx.x; k < r; k += blockDim.x) {
    const T* w = W_uk + ((size_t)g * r + k) * d_n;
    float acc = 0.f;
    for (int j = 0; j < d_n; ++j) acc = fmaf(to_f32(w[j]), sq[j], acc);
    qt[row * r + k] = from_f32<OutT>(acc);
  }
}

// Split-KV decode, one warp per output row at a time, online softmax over the
// split's tokens.  Block = (split, sequence * G + group).
template <typename T, bool ABSORB>
__global__ void decode_kernel(KvLayout ly, SplitPlan plan, const T* __restrict__ q, const float* __restrict__ qt,
                              const T* __restrict__ kpool, const T* __restrict__ vpool, KRow kr,
                              int n_h, int G, int s_q, int d_n, int d_r, int d_v, int r, float scale,
                              T* __restrict__ out_T, float* __restrict__ o_f32, float* __restrict__ lse_dst,
                              long long rows, int32_t* st) {
  const int split = blockIdx.x;
  const int b = blockIdx.y / G, g = blockIdx.y % G;
  const int m = n_h / G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int d_qk = d_n + d_r;
  const int Dk = ABSORB ? (r + d_r) : d_qk;           // key width
  const int Dv = ABSORB ? r : d_v;                    // value width
  // key element j of a token row: j < ksplit at koff + j, else at kro + (j - ksplit)
  const long long krs = ABSORB ? (long long)(r + d_r) : (long long)kr.pitch;  // key row stride
  const long long vrs = ABSORB ? (long long)(r + d_r) : (long long)G * d_v;
  const int ksplit = ABSORB ? r : d_n;
  const int koff = ABSORB ? 0 : kr.nope_at(g);
  const int kro = ABSORB ? r : kr.rope_at(g);
  const int voff = ABSORB ? 0 : g * d_v;
  int L = seq_len_checked(ly, b, s_q, (split == 0 && g == 0) ? st : nullptr);
  if (!seq_pages_ok(ly, b, L, st)) L = -1;
  const int t_begin = split * plan.chunk;

  for (int wr = warp; wr < m * s_q; wr += nwarps) {
    const int i = wr / m, h = g * m + wr % m;
    const long long row = ((long long)b * s_q + i) * n_h + h;
    float qv[kMaxKeyPerLane];
#pragma unroll
    for (int u = 0; u < kMaxKeyPerLane; ++u) {
      int j = lane + 32 * u;
      float x = 0.f;
      if (j < Dk) {
        if (ABSORB) x = j < r ? qt[row * r + j] : to_f32(q[row * d_qk + d_n + (j - r)]);
        else x = to_f32(q[row * d_qk + j]);
      }
      qv[u] = x;
    }
    float acc[kMaxValPerLane];
#pragma unroll
    for (int u = 0; u < kMaxValPerLane; ++u) acc[u] = 0.f;
    float mx = -INFINITY, l = 0.f;
    bool bad = L < 0;
    int t_end = 0;
    if (!bad) t_end = min(t_begin + plan.chunk, L - s_q + i + 1);
    for (int t = t_begin; !bad && t < t_end; ++t) {
      long long tr = token_row(ly, b, t, st);
      if (tr < 0) { bad = true; break; }
      const T* krow = kpool + tr * krs;
      float part = 0.f;
#pragma unroll
      for (int u = 0; u < kMaxKeyPerLane; ++u) {
        int j = lane + 32 * u;
        if (j < Dk) part = fmaf(qv[u], to_f32(krow[j < ksplit ? koff + j : kro + (j - ksplit)]), part);
      }
      const float s = warp_sum(part) * scale;
      const float mn = fmaxf(mx, s);
      const float corr = expf(mx - mn);
      const float p = expf(s - mn);
      l = l * corr + p;
      mx = mn;
      const T* vr = vpool + tr * vrs + voff;
#pragma unroll
      for (int u = 0; u < kMaxValPerLane; ++u) {
        int j = lane + 32 * u;
        if (j < Dv) acc[u] = fmaf(p, to_f32(vr[j]), acc[u] * corr);
      }
    }
    const bool empty = bad || l == 0.f;
    const float inv = empty ? 0.f : 1.f / l;
    const float lse = empty ? -INFINITY : mx + logf(l);
    const long long orow = (long long)split * rows + row;
#pragma unroll
    for (int u = 0; u < kMaxValPerLane; ++u) {
      int j = lane + 32 * u;
      if (j < Dv) {
        float o = acc[u] * inv;
        if (o_f32) o_f32[orow * Dv + j] = o;
        else out_T[row * Dv + j] = from_f32<T>(o);
      }
    }
    if (lane == 0 && lse_dst) lse_dst[orow] = lse;
  }
}

// out[row, :] = o_lat[row, :] W_uv^g   (absorb path's up-projection).
template <typename T>
__global__ void up_proj_kernel(const float* __restrict__ o_lat, const T* __restrict__ W_uv, T* __restrict__ out,
                               int n_h, int m, int r, int d_v) {
  extern __shared__ float so[];  // [r]
  const long long row = blockIdx.x;
  const int g = (int)(row % n_h) / m;
  for (int k = threadIdx.x; k < r; k += blockDim.x) so[k] = o_lat[row * r + k];
  __syncthreads();
  const T* W = W_uv + (size_t)g * r * d_v;
  for (int j = threadIdx.x; j < d_v; j += blockDim.x) {
    float acc = 0.f;
    for (int k = 0; k < r; ++k) acc = fmaf(so[k], to_f32(W[(size_t)k * d_v + j]), acc);
    out[row * d_v + j] = from_f32<T>(acc);
  }
}

// Log-sum-exp merge, one warp per row.
template <typename T>
__global__ void combine_kernel(int S, long long rows, int D, const float* __restrict__ o_part,
                               const float* __restrict__ lse_part, T* __restrict__ out, float* __restrict__ lse_out) {
  // launched while the kernel ahead of it may still run: wait for it before
  // any memory access, then let the next kernel launch
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float mx = -INFINITY;
  for (int s = 0; s < S; ++s) mx = fmaxf(mx, lse_part[(long long)s * rows + row]);
  float Z = 0.f;
  if (mx != -INFINITY)
    for (int s = 0; s < S; ++s) Z += expf(lse_part[(long long)s * rows + row] - mx);
  const float inv = mx == -INFINITY ? 0.f : 1.f / Z;
  for (int j = lane; j < D; j += 32) {
    float acc = 0.f;
    if (mx != -INFINITY)
      for (int s = 0; s < S; ++s) {
        float ls = lse_part[(long long)s * rows + row];
        if (ls != -INFINITY) acc = fmaf(expf(ls - mx) * inv, o_part[((long long)s * rows + row) * D + j], acc);
      }
    out[row * D + j] = from_f32<T>(acc);
  }
  if (lane == 0 && lse_out) lse_out[row] = mx == -INFINITY ? -INFINITY : mx + logf(Z);
}

}  // namespace

cudaError_t simt_expand(const Problem& p, const void* latent, const void* W_uk, const void* W_uv,
                        void* k_pool, void* v_pool, int tail, int32_t* st, cudaStream_t s) {
  const auto& d = p.d;
  int span = tail > 0 ? (tail < p.ly.max_seq_len ? tail : p.ly.max_seq_len) : p.ly.max_seq_len;
  dim3 grid((span + kExpandTokens - 1) / kExpandTokens, p.ly.batch, d.G);
  size_t smem = (size_t)kExpandTokens * d.r * sizeof(float);
  if (d.dtype == GQLA_F32) {
    auto k = expand_kernel<float>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, 256, smem, s>>>(p.ly, (const float*)latent, (const float*)W_uk, (const float*)W_uv,
                              (float*)k_pool, (float*)v_pool, p.kr, d.G, d.d_nope, d.d_rope, d.d_v, d.r, tail,
                              st);
  } else {
    auto k = expand_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, 256, smem, s>>>(p.ly, (const __nv_bfloat16*)latent, (const __nv_bfloat16*)W_uk,
                              (const __nv_bfloat16*)W_uv, (__nv_bfloat16*)k_pool, (__nv_bfloat16*)v_pool, p.kr,
                              d.G, d.d_nope, d.d_rope, d.d_v, d.r, tail, st);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t simt_absorb_q(const Problem& p, const void* q, const void* W_uk, float* qt, cudaStream_t s) {
  const auto& d = p.d;
  size_t smem = (size_t)d.d_nope * sizeof(float);
  if (d.dtype == GQLA_F32)
    absorb_q_kernel<float, float><<<(unsigned)p.rows, 256, smem, s>>>((const float*)q, (const float*)W_uk, qt,
                                                                      d.n_h, p.m, d.d_nope, p.d_qk, d.r);
  else
    absorb_q_kernel<__nv_bfloat16, float><<<(unsigned)p.rows, 256, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)W_uk, qt, d.n_h, p.m, d.d_nope, p.d_qk, d.r);
  count_launch();
  return cudaGetLastError();
}

cudaError_t absorb_q_bf16(const Problem& p, const void* q, const void* W_uk, __nv_bfloat16* qt, cudaStream_t s) {
  const auto& d = p.d;
  size_t smem = (size_t)d.d_nope * sizeof(float);
  absorb_q_kernel<__nv_bfloat16, __nv_bfloat16><<<(unsigned)p.rows, 256, smem, s>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)W_uk, qt, d.n_h, p.m, d.d_nope, p.d_qk, d.r);
  count_launch();
  return cudaGetLastError();
}

cudaError_t simt_decode(const Problem& p, gqla_path path, const void* q, const float* qt, const void* kpool,
                        const void* vpool, void* out_T, float* o_f32, float* lse, int32_t* st, cudaStream_t s) {
  const auto& d = p.d;
  dim3 grid(p.plan.num_splits, p.ly.batch * d.G);
  const int threads = 128;
#define GQLA_DEC(T, AB)                                                                                   \
  decode_kernel<T, AB><<<grid, threads, 0, s>>>(p.ly, p.plan, (const T*)q, qt, (const T*)kpool,           \
                                                (const T*)vpool, p.kr, d.n_h, d.G, d.s_q, d.d_nope,       \
                                                d.d_rope, d.d_v, d.r, d.scale, (T*)out_T, o_f32, lse,     \
                                                p.rows, st)
  if (d.dtype == GQLA_F32) {
    if (path == GQLA_PATH_ABSORB) GQLA_DEC(float, true); else GQLA_DEC(float, false);
  } else {
    if (path == GQLA_PATH_ABSORB) GQLA_DEC(__nv_bfloat16, true); else GQLA_DEC(__nv_bfloat16, false);
  }
#undef GQLA_DEC
  count_launch();
  return cudaGetLastError();
}

cudaError_t simt_up_proj(const Problem& p, const float* o_lat, const void* W_uv, void* out, cudaStream_t s) {
  const auto& d = p.d;
  size_t smem = (size_t)d.r * sizeof(float);
  if (d.dtype == GQLA_F32)
    up_proj_kernel<float><<<(unsigned)p.rows, 128, smem, s>>>(o_lat, (const float*)W_uv, (float*)out, d.n_h, p.m,
                                                              d.r, d.d_v);
  else
    up_proj_kernel<__nv_bfloat16><<<(unsigned)p.rows, 128, smem, s>>>(
        o_lat, (const __nv_bfloat16*)W_uv, (__nv_bfloat16*)out, d.n_h, p.m, d.r, d.d_v);
  count_launch();
  return cudaGetLastError();
}

cudaError_t combine(int S, long long rows, int D, const float* o_part, const float* lse_part, void* out,
                    gqla_dtype out_dtype, float* lse_out, cudaStream_t s) {
  const int wpb = 8;
  unsigned blocks = (unsigned)((rows + wpb - 1) / wpb);
  cudaError_t e;
  if (out_dtype == GQLA_F32)
    e = launch_pdl(combine_kernel<float>, dim3(blocks), dim3(32 * wpb), 0, s, S, rows, D, o_part, lse_part,
                   (float*)out, lse_out);
  else
    e = launch_pdl(combine_kernel<__nv_bfloat16>, dim3(blocks), dim3(32 * wpb), 0, s, S, rows, D, o_part, lse_part,
                   (__nv_bfloat16*)out, lse_out);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace gqla
