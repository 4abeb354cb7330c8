// Host-side launchers shared between the API translation unit and the kernel
// translation units of the GQLA library.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "gqla.h"

namespace gqla {

// A validated decode problem with the derived sizes.
struct Problem {
  gqla_dims d;
  KvLayout ly;
  int m;        // heads per group
  int d_qk;     // d_nope + d_rope
  int E;        // latent row width r + d_rope
  long long rows;  // B * s_q * n_h output rows
  KRow kr;         // expanded K pool row layout
  SplitPlan plan;
};

// Workspace carve-up of one decode call (all fp32 except qt, which is fp32 for
// the SIMT path and bf16 for the tensor-core path).
struct Workspace {
  void* qt;        // absorbed queries [rows, r]
  float* o_part;   // [S, rows, D] when S > 1
  float* lse_part; // [S, rows] when S > 1
  float* o_lat;    // absorb: combined latent outputs [rows, r]
  int* counters;   // GQA with S > 1: split counts per (sequence, group, row block)
};

// The GQA call from its workspace: decode (and the split merge, in the
// kernel or as a combine pass).  Shared by the workspace and no-alloc entries.
cudaError_t gqa_decode_call(const Problem& p, bool tc, const void* q, const void* k_pool, const void* v_pool,
                            void* out, float* lse, const Workspace& w, int32_t* st, cudaStream_t s);

// Validates dims/layout and builds the problem with its split plan.
gqla_status make_problem(const gqla_dims* dims, const gqla_kv_layout* layout, int num_splits, gqla_path path,
                         Problem* p);
// The generic kernels keep a row's query and accumulator in registers.
bool simt_supports(const Problem& p, gqla_path path);

size_t ws_layout(const Problem& p, gqla_path path, bool tc, Workspace* ws, char* base);

// ---- generic CUDA-core kernels (fp32 math; any supported dims) ----
cudaError_t simt_expand(const Problem& p, const void* latent, const void* W_uk, const void* W_uv,
                        void* k_pool, void* v_pool, int tail, int32_t* st, cudaStream_t s);
cudaError_t simt_absorb_q(const Problem& p, const void* q, const void* W_uk, float* qt,
                          cudaStream_t s);
// path GQA: keys/values are the expanded pools; path ABSORB: the latent pool.
// Writes o (normalised) + lse per (split, row): to o_part/lse_part when S > 1,
// else to out_T (GQA) or o_lat (absorb) and lse.
cudaError_t simt_decode(const Problem& p, gqla_path path, const void* q, const float* qt,
                        const void* kpool, const void* vpool, void* out_T, float* o_f32,
                        float* lse, int32_t* st, cudaStream_t s);
cudaError_t simt_up_proj(const Problem& p, const float* o_lat, const void* W_uv, void* out,
                         cudaStream_t s);
// Scatter of the step's new latent rows into the pool (append.cu).
cudaError_t append_rows(const Problem& p, const void* new_rows, void* latent, int32_t* st, cudaStream_t s);
cudaError_t combine(int S, long long rows, int D, const float* o_part, const float* lse_part,
                    void* out, gqla_dtype out_dtype, float* lse_out, cudaStream_t s);

int num_sms();

// Counts one kernel launch (reported by gqla_launch_counter).
void count_launch(int n = 1);

// Raises a kernel's dynamic shared-memory limit once per device.
cudaError_t ensure_smem_limit(const void* func, int bytes);

namespace ptx {
// A kernel launched by launch_pdl may begin while the kernel ahead of it on the
// stream is still running.  pdl_wait() returns once that kernel has completed
// and its memory writes are visible (at once when the launch had no such
// dependency); pdl_trigger() lets the next such kernel begin launching once
// every CTA of this grid has called it or exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
}  // namespace ptx

// Launches a kernel that may begin before the kernel ahead of it on the stream
// has finished (programmatic stream serialisation): the kernel reads that
// kernel's results only after ptx::pdl_wait().
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace gqla
