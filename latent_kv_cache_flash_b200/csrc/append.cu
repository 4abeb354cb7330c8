// Decode-time cache append: scatter the step's new latent rows into the
// (paged) latent pool; the entry point then expands just those tokens into
// the per-group pools.
#include "common.cuh"
#include "launch.h"
#include "tc.h"

namespace gqla {

namespace {

// One CTA per (sequence, new token): copies one latent row (16-byte vectors
// when the row pitch allows, elements otherwise).
template <typename T>
__global__ void append_rows_kernel(KvLayout ly, const T* __restrict__ new_rows, T* __restrict__ latent, int s_q,
                                   int E, int32_t* st) {
  // launched while the kernel ahead of it may still run: wait for it before
  // any memory access, then let the next kernel launch
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const int b = blockIdx.x / s_q, i = blockIdx.x % s_q;
  const int L = seq_len_checked(ly, b, s_q, i == 0 ? st : nullptr);
  if (L < 0) return;
  const long long row = token_row(ly, b, L - s_q + i, st);
  if (row < 0) return;
  const T* src = new_rows + ((long long)b * s_q + i) * E;
  T* dst = latent + row * E;
  if ((E * sizeof(T)) % 16 == 0) {
    const int nv = (int)(E * sizeof(T) / 16);
    for (int v = threadIdx.x; v < nv; v += blockDim.x)
      reinterpret_cast<uint4*>(dst)[v] = reinterpret_cast<const uint4*>(src)[v];
  } else {
    for (int e = threadIdx.x; e < E; e += blockDim.x) dst[e] = src[e];
  }
}

}  // namespace

cudaError_t append_rows(const Problem& p, const void* new_rows, void* latent, int32_t* st, cudaStream_t s) {
  const int blocks = p.ly.batch * p.d.s_q;
  cudaError_t e;
  if (p.d.dtype == GQLA_F32)
    e = launch_pdl(append_rows_kernel<float>, dim3(blocks), dim3(64), 0, s, p.ly, (const float*)new_rows,
                   (float*)latent, p.d.s_q, p.E, st);
  else
    e = launch_pdl(append_rows_kernel<__nv_bfloat16>, dim3(blocks), dim3(64), 0, s, p.ly,
                   (const __nv_bfloat16*)new_rows, (__nv_bfloat16*)latent, p.d.s_q, p.E, st);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace gqla
