// gqla_decode_gqa_noalloc: the GQA decode entry point without a caller-supplied
// workspace.  Its split-KV scratch (per-split partial outputs and their
// log-sum-exp) lives in one file-scope device array of fixed size, so the call
// needs no allocation at all: for hosts that own every byte of device memory
// and hand a plug-in none of it, and for decode loops that may not call an
// allocator on the hot path (cudaMalloc/cudaFree synchronise the device).
#include <cuda.h>

#include <mutex>

#include "gqla.h"
#include "launch.h"
#include "tc.h"

namespace {

// 32 MiB of split scratch per device that loads the library, held until the
// process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array for the current device.  In host code
// g_noalloc_scratch names a host-side stand-in, not device memory, so the
// address is looked up with that device current.  It is cached per device
// together with the context it was looked up in: a device reset or a new
// primary context loads the module afresh, so a changed context triggers a
// new lookup instead of reusing a stale address.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// A driver entry point, looked up through the runtime (the library does not
// link libcuda); nullptr when the driver lacks it.
void* driver_fn(const char* name) {
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return f;
}

// An identity of the context current on this thread, 0 when there is none:
// the driver's unique context id (never reused within the process), else the
// context handle.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = (CtxGetCurrentFn)driver_fn("cuCtxGetCurrent");
  static CtxGetIdFn get_id = (CtxGetIdFn)driver_fn("cuCtxGetId");
  CUcontext ctx = nullptr;
  if (!get_current || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id && get_id(ctx, &id) == CUDA_SUCCESS && id != 0) return id;
  return (unsigned long long)(uintptr_t)ctx;
}

void* scratch_for_current_device(gqla_status* status) {
  static std::mutex mu;
  static void* cached[64] = {nullptr};
  static unsigned long long cached_ctx[64] = {0};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    *status = GQLA_ERR_CUDA;
    return nullptr;
  }
  // the context current on this thread (none before the runtime's first call
  // here; the symbol lookup below creates the device's primary context then)
  unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (ctx != 0 && cached[dev] != nullptr && cached_ctx[dev] == ctx) return cached[dev];
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e == cudaSuccess) ctx = current_context_id();
  if (e != cudaSuccess || ptr == nullptr || ctx == 0) {
    cudaGetLastError();
    cached[dev] = nullptr;
    *status = GQLA_ERR_CUDA;
    return nullptr;
  }
  cached[dev] = ptr;
  cached_ctx[dev] = ctx;
  return ptr;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

using namespace gqla;

extern "C" gqla_status gqla_decode_gqa_noalloc(const gqla_dims* dims, const gqla_kv_layout* layout,
                                               const void* q, const void* k_pool, const void* v_pool, void* out,
                                               float* lse, int32_t num_splits, int32_t* dev_status,
                                               void* stream) {
  Problem p;
  gqla_status s = make_problem(dims, layout, num_splits, GQLA_PATH_GQA, &p);
  if (s != GQLA_OK) return s;
  if (!q || !k_pool || !v_pool || !out) return GQLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out)) return GQLA_ERR_ALIGNMENT;
  const bool tc = tc_gqa_supports(p);
  if (!tc && !simt_supports(p, GQLA_PATH_GQA)) return GQLA_ERR_UNSUPPORTED;
  const size_t need = ws_layout(p, GQLA_PATH_GQA, false, nullptr, nullptr);
  if (need > kNoAllocScratchBytes) return GQLA_ERR_WORKSPACE;   // ask for fewer splits
  void* scratch = nullptr;
  if (need > 0) {
    s = GQLA_OK;
    scratch = scratch_for_current_device(&s);
    if (!scratch) return s;
  }
  Workspace w;
  ws_layout(p, GQLA_PATH_GQA, false, &w, (char*)scratch);
  // Every split writes its whole partial (an empty split writes zeros and
  // lse = -inf) and the split counters are zeroed before the launch, so
  // nothing left in the scratch by an earlier call is read.
  cudaError_t e = gqa_decode_call(p, tc, q, k_pool, v_pool, out, lse, w, dev_status, (cudaStream_t)stream);
  return e == cudaSuccess ? GQLA_OK : GQLA_ERR_CUDA;
}
