// C-ABI entry points of the GQLA decode library: host-side validation, the
// split-KV plan, workspace carve-up and kernel dispatch.
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "gqla.h"
#include "launch.h"
#include "tc.h"

namespace gqla {

namespace {

constexpr int kSplitGranule = 128;   // token granule of split boundaries
constexpr int kMaxSplits = 256;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

gqla_status check_dims(const gqla_dims* d) {
  if (!d) return GQLA_ERR_INVALID_ARG;
  if (d->n_h < 1 || d->G < 1 || d->n_h % d->G != 0) return GQLA_ERR_INVALID_ARG;
  if (d->d_nope < 1 || d->d_rope < 0 || d->d_v < 1 || d->r < 1) return GQLA_ERR_INVALID_ARG;
  if (d->s_q < 1 || d->s_q > 4) return GQLA_ERR_INVALID_ARG;
  if (!(d->scale == d->scale) || isinf(d->scale)) return GQLA_ERR_INVALID_ARG;
  if (d->dtype != GQLA_F32 && d->dtype != GQLA_BF16) return GQLA_ERR_INVALID_ARG;
  if (d->k_layout != GQLA_K_PER_GROUP && d->k_layout != GQLA_K_SHARED_ROPE) return GQLA_ERR_INVALID_ARG;
  return GQLA_OK;
}

gqla_status check_layout(const gqla_kv_layout* l) {
  if (!l || !l->seq_lens) return GQLA_ERR_INVALID_ARG;
  if (l->batch < 1 || l->max_seq_len < 1 || l->page_size < 0) return GQLA_ERR_INVALID_ARG;
  if (l->batch > 65535) return GQLA_ERR_UNSUPPORTED;
  if (l->page_size == 0) {
    if (l->capacity < 1) return GQLA_ERR_INVALID_ARG;
  } else {
    if (!l->block_table || l->max_blocks_per_seq < 1 || l->num_pages < 1) return GQLA_ERR_INVALID_ARG;
  }
  return GQLA_OK;
}

KvLayout to_kernel_layout(const gqla_kv_layout* l) {
  KvLayout k;
  k.seq_lens = l->seq_lens;
  k.block_table = l->block_table;
  k.batch = l->batch;
  k.max_seq_len = l->max_seq_len;
  k.page_size = l->page_size;
  k.capacity = l->page_size == 0 ? l->capacity : l->max_blocks_per_seq * l->page_size;
  k.mbps = l->max_blocks_per_seq;
  k.num_pages = l->num_pages;
  return k;
}

size_t esize(gqla_dtype t) { return t == GQLA_F32 ? 4 : 2; }

// Split-KV plan.  A requested count is honoured up to rounding the chunk to
// the kernel's tile.  The automatic choice:
//  * the streaming GQA kernel (two CTAs per SM, HBM-bound): a wave of n CTAs
//    streams its chunks in the time HBM takes for max(n, busy) of them, since
//    fewer CTAs do not keep HBM busy (busy: about 1.35 CTAs per SM up to 16
//    rows a group, every slot beyond); the plan minimises that
//    over the waves plus the split partials (B200, LLaMA-shaped layer, B32
//    L8K: 256 CTAs, one split 0.193 ms, eight 0.218 ms; n_h 128, G 16, B64
//    L32K: one split leaves a last wave of 136 CTAs, 3.26 ms, two 3.08 ms);
//  * the tensor-core kernels (one CTA per SM) minimise (waves of CTAs) x
//    (chunk tokens + the CTA's fixed cost in tokens) x (bytes a CTA streams
//    per token), the busiest SM's time, plus the split partials written and
//    read back.  The absorb CTA's prologue and epilogue cost about as much as
//    300 tokens of its stream (B32 L8K: four splits 0.100 ms, nine 0.112 ms;
//    B64 L32K, n_h 128: eight splits best).
SplitPlan make_plan(const gqla_dims& d, const gqla_kv_layout& l, int requested, gqla_path path, bool tc) {
  const long long L = l.max_seq_len;
  const int granule = !tc ? kSplitGranule : 64;
  auto chunk_for = [&](long long S) {
    long long c = (L + S - 1) / S;
    return ((c + granule - 1) / granule) * granule;
  };
  if (requested > 0) {
    long long S = requested > kMaxSplits ? kMaxSplits : requested;
    long long c = chunk_for(S);
    return SplitPlan{(int)((L + c - 1) / c), (int)c};
  }
  const long long rows = (long long)l.batch * d.s_q * d.n_h;
  long long max_s = (L + granule - 1) / granule;
  if (max_s > kMaxSplits) max_s = kMaxSplits;
  auto plan_of = [&](long long S) {
    const long long c = chunk_for(S);
    return SplitPlan{(int)((L + c - 1) / c), (int)c};
  };
  const bool wide = (d.n_h / d.G) * d.s_q >= 64 && tc;
  if (path == GQLA_PATH_GQA && !wide) {
    const long long units = (long long)l.batch * d.G * (((d.n_h / d.G) * d.s_q + 63) / 64);
    const long long slots = (long long)num_sms() * 2;
    // CTAs that keep HBM busy: beyond 16 rows a group a CTA's MMAs slow its
    // stream (n_h 128, B32 L32K: G 16, s_q 4 takes 1.63 ms with every slot
    // filled, 1.73 ms with one split)
    const long long busy = (d.n_h / d.G) * d.s_q <= 16 ? (long long)num_sms() * 27 / 20 : slots;
    const double unit_bytes = 2.0 * (d.d_nope + d.d_rope + d.d_v);
    const double part_bytes = (double)rows * (d.d_v + 1) * 4 * 2;
    long long best_s = 1;
    double best = -1.0;
    for (long long S = 1; S <= max_s; ++S) {
      const long long c = chunk_for(S);
      const long long Se = (L + c - 1) / c;
      if (Se != S) continue;
      const long long n = units * Se, rem = n % slots;
      const double width = (double)(n - rem) + (rem ? (double)(rem > busy ? rem : busy) : 0.0);
      const double cost = width * c * unit_bytes + (Se > 1 ? Se * part_bytes : 0.0);
      if (best < 0 || cost < best * 0.999) {
        best = cost;
        best_s = Se;
      }
    }
    return plan_of(best_s);
  }
  long long units, slots, rb = 1;
  double unit_bytes, part_bytes, cta_tokens;
  if (path == GQLA_PATH_ABSORB) {
    units = (long long)l.batch * ((d.n_h * d.s_q + 63) / 64);
    slots = (long long)num_sms() * 1;
    unit_bytes = 2.0 * (d.r + d.d_rope);
    part_bytes = (double)rows * (d.r + 1) * 4 * 2;
    cta_tokens = 300.0;
  } else {
    // the tcgen05 GQA kernel: 128-row blocks, one CTA per SM.  Its CTA costs
    // about 900 tokens of stream up front (the first tile's latency, the
    // query into TMEM, the merge of the two softmax states).  Only the first
    // row block of a (sequence, group, split) reads a K/V tile from HBM (the
    // others hit L2), and about 95% of the SMs' worth of such readers keep
    // HBM busy: a wave with more of them streams each tile proportionally
    // slower.  (Measured on B200, n_h 128, B32 L32K: one wave of 128 CTAs,
    // 1-4 splits, beats two to seven waves of 8-9 splits by 4-15% at every
    // shape with 64-512 rows a group.)
    rb = ((d.n_h / d.G) * d.s_q + 127) / 128;
    units = (long long)l.batch * d.G * rb;
    slots = (long long)num_sms();
    unit_bytes = 2.0 * (d.d_nope + d.d_rope + d.d_v);
    part_bytes = (double)rows * (d.d_v + 1) * 4 * 2;
    cta_tokens = 900.0;
  }
  const double busy = 0.95 * (double)slots;
  long long best_s = 1;
  double best = -1.0;
  for (long long S = 1; S <= max_s; ++S) {
    const long long c = chunk_for(S);
    const long long Se = (L + c - 1) / c;
    if (Se != S) continue;
    double cost = Se > 1 ? Se * part_bytes : 0.0;
    if (path == GQLA_PATH_ABSORB) {
      const long long waves = (units * Se + slots - 1) / slots;
      cost += (double)waves * (c + cta_tokens) * unit_bytes * slots;
    } else {
      for (long long left = units * Se; left > 0; left -= slots) {
        const double w = (double)(left < slots ? left : slots);
        const double share = w / (double)rb / busy;
        cost += (c + cta_tokens) * unit_bytes * slots * (share > 1.0 ? share : 1.0);
      }
    }
    if (best < 0 || cost < best * 0.999) {
      best = cost;
      best_s = Se;
    }
  }
  return plan_of(best_s);
}

}  // namespace

gqla_status make_problem(const gqla_dims* dims, const gqla_kv_layout* layout, int num_splits, gqla_path path,
                         Problem* p) {
  gqla_status s = check_dims(dims);
  if (s != GQLA_OK) return s;
  s = check_layout(layout);
  if (s != GQLA_OK) return s;
  p->d = *dims;
  p->ly = to_kernel_layout(layout);
  p->m = dims->n_h / dims->G;
  p->d_qk = dims->d_nope + dims->d_rope;
  p->E = dims->r + dims->d_rope;
  p->rows = (long long)layout->batch * dims->s_q * dims->n_h;
  if (dims->k_layout == GQLA_K_SHARED_ROPE)
    p->kr = KRow{dims->G * dims->d_nope + dims->d_rope, dims->d_nope, dims->G * dims->d_nope, 0};
  else
    p->kr = KRow{dims->G * p->d_qk, p->d_qk, dims->d_nope, p->d_qk};
  p->plan = SplitPlan{1, layout->max_seq_len};
  const bool tc = path == GQLA_PATH_ABSORB ? tc_absorb_supports(*p) : tc_gqa_supports(*p);
  p->plan = make_plan(*dims, *layout, num_splits, path, tc);
  return GQLA_OK;
}

// The generic kernels keep a row's query and accumulator in registers.
bool simt_supports(const Problem& p, gqla_path path) {
  int dk = path == GQLA_PATH_ABSORB ? p.E : p.d_qk;
  int dv = path == GQLA_PATH_ABSORB ? p.d.r : p.d.d_v;
  return dk <= 640 && dv <= 512;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t ws_layout(const Problem& p, gqla_path path, bool tc, Workspace* ws, char* base) {
  size_t off = 0;
  const int S = p.plan.num_splits;
  const int D = path == GQLA_PATH_ABSORB ? p.d.r : p.d.d_v;
  Workspace w{nullptr, nullptr, nullptr, nullptr, nullptr};
  auto take = [&](size_t bytes) {
    void* ptr = base ? base + off : nullptr;
    off = align256(off + bytes);
    return ptr;
  };
  if (path == GQLA_PATH_ABSORB) {
    w.qt = take((size_t)p.rows * p.d.r * (tc ? 2 : 4));
    w.o_lat = (float*)take((size_t)p.rows * p.d.r * 4);
  }
  // the tensor-core absorb kernel always writes per-split partials
  if (S > 1 || (tc && path == GQLA_PATH_ABSORB)) {
    w.o_part = (float*)take((size_t)S * p.rows * D * 4);
    w.lse_part = (float*)take((size_t)S * p.rows * 4);
  }
  if (S > 1 && path == GQLA_PATH_GQA) {
    const long long blocks = (long long)p.ly.batch * p.d.G * ((p.m * p.d.s_q + 15) / 16);
    w.counters = (int*)take((size_t)blocks * 4);
  }
  if (ws) *ws = w;
  return off;
}

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

cudaError_t ensure_smem_limit(const void* func, int bytes) {
  static std::mutex mu;
  struct Entry { const void* f; int dev; int bytes; };
  static Entry done[256];
  static int n_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].f == func && done[i].dev == dev && done[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && n_done < 256) done[n_done++] = Entry{func, dev, bytes};
  return e;
}

int num_sms() {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  std::lock_guard<std::mutex> g(mu);
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 148;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

cudaError_t gqa_decode_call(const Problem& p, bool tc, const void* q, const void* k_pool, const void* v_pool,
                            void* out, float* lse, const Workspace& w, int32_t* st, cudaStream_t s) {
  const int S = p.plan.num_splits;
  cudaError_t e;
  bool merged = false;
  if (tc) e = tc_gqa_decode(p, q, k_pool, v_pool, S > 1 ? nullptr : out, S > 1 ? w.o_part : nullptr,
                            S > 1 ? w.lse_part : lse, st, s, w.counters, out, lse, &merged);
  else e = simt_decode(p, GQLA_PATH_GQA, q, nullptr, k_pool, v_pool, S > 1 ? nullptr : out,
                       S > 1 ? w.o_part : nullptr, S > 1 ? w.lse_part : lse, st, s);
  if (e == cudaSuccess && S > 1 && !merged)
    e = combine(S, p.rows, p.d.d_v, w.o_part, w.lse_part, out, p.d.dtype, lse, s);
  return e;
}

}  // namespace gqla

using namespace gqla;

extern "C" {

const char* gqla_version(void) { return "gqla-b200 0.1"; }

uint64_t gqla_launch_counter(void) { return g_launches.load(std::memory_order_relaxed); }

const char* gqla_status_string(gqla_status s) {
  switch (s) {
    case GQLA_OK: return "GQLA_OK";
    case GQLA_ERR_INVALID_ARG: return "GQLA_ERR_INVALID_ARG: invalid argument";
    case GQLA_ERR_UNSUPPORTED: return "GQLA_ERR_UNSUPPORTED: dims not handled by this library";
    case GQLA_ERR_ALIGNMENT: return "GQLA_ERR_ALIGNMENT: pointer or pitch not 16-byte aligned";
    case GQLA_ERR_WORKSPACE: return "GQLA_ERR_WORKSPACE: workspace missing or too small";
    case GQLA_ERR_CUDA: return "GQLA_ERR_CUDA: CUDA launch failed";
  }
  return "unknown gqla_status";
}

size_t gqla_cache_bytes_per_token(const gqla_dims* dims, gqla_path path) {
  if (check_dims(dims) != GQLA_OK) return 0;
  size_t e = esize(dims->dtype);
  if (path == GQLA_PATH_ABSORB) return (size_t)(dims->r + dims->d_rope) * e;
  if (path == GQLA_PATH_GQA) {
    const size_t k = dims->k_layout == GQLA_K_SHARED_ROPE ? (size_t)dims->G * dims->d_nope + dims->d_rope
                                                          : (size_t)dims->G * (dims->d_nope + dims->d_rope);
    return (k + (size_t)dims->G * dims->d_v) * e;
  }
  return 0;
}

int32_t gqla_num_splits(const gqla_dims* dims, const gqla_kv_layout* layout, int32_t num_splits, gqla_path path) {
  Problem p;
  if (make_problem(dims, layout, num_splits, path, &p) != GQLA_OK) return 0;
  return p.plan.num_splits;
}

size_t gqla_workspace_bytes(const gqla_dims* dims, const gqla_kv_layout* layout, int32_t num_splits,
                            gqla_path path) {
  Problem p;
  if (make_problem(dims, layout, num_splits, path, &p) != GQLA_OK) return 0;
  bool tc = path == GQLA_PATH_ABSORB ? tc_absorb_supports(p) : false;
  return ws_layout(p, path, tc, nullptr, nullptr);
}

gqla_status gqla_expand_cache(const gqla_dims* dims, const gqla_kv_layout* layout, const void* latent,
                              const void* W_uk, const void* W_uv, void* k_pool, void* v_pool,
                              int32_t tail_tokens, int32_t* dev_status, void* stream) {
  Problem p;
  gqla_status s = make_problem(dims, layout, 1, GQLA_PATH_GQA, &p);
  if (s != GQLA_OK) return s;
  if (!latent || !W_uk || !W_uv || !k_pool || !v_pool) return GQLA_ERR_INVALID_ARG;
  if (!aligned16(latent) || !aligned16(W_uk) || !aligned16(W_uv) || !aligned16(k_pool) || !aligned16(v_pool))
    return GQLA_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (tc_expand_supports(p)) e = tc_expand(p, latent, W_uk, W_uv, k_pool, v_pool, tail_tokens, dev_status, st);
  else e = simt_expand(p, latent, W_uk, W_uv, k_pool, v_pool, tail_tokens, dev_status, st);
  return e == cudaSuccess ? GQLA_OK : GQLA_ERR_CUDA;
}

gqla_status gqla_append_tokens(const gqla_dims* dims, const gqla_kv_layout* layout, const void* new_rows,
                               void* latent, const void* W_uk, const void* W_uv, void* k_pool, void* v_pool,
                               int32_t* dev_status, void* stream) {
  Problem p;
  gqla_status s = make_problem(dims, layout, 1, GQLA_PATH_GQA, &p);
  if (s != GQLA_OK) return s;
  if (!new_rows) return GQLA_ERR_INVALID_ARG;
  const bool expand = k_pool || v_pool;
  if (!latent && !expand) return GQLA_ERR_INVALID_ARG;
  if (expand && (!k_pool || !v_pool || !W_uk || !W_uv)) return GQLA_ERR_INVALID_ARG;
  if (!aligned16(new_rows) || (latent && !aligned16(latent))) return GQLA_ERR_ALIGNMENT;
  if (expand && (!aligned16(W_uk) || !aligned16(W_uv) || !aligned16(k_pool) || !aligned16(v_pool)))
    return GQLA_ERR_ALIGNMENT;
  // without a latent pool the expansion must read the dense new rows
  if (!latent && !tc_expand_supports(p)) return GQLA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = latent ? append_rows(p, new_rows, latent, dev_status, st) : cudaSuccess;
  if (e == cudaSuccess && expand) {
    // the new rows are dense: the tensor-core form packs many sequences' new
    // tokens into each 128-row tile
    if (tc_expand_supports(p)) e = tc_expand_dense(p, new_rows, k_pool, v_pool, W_uk, W_uv, dev_status, st);
    else e = simt_expand(p, latent, W_uk, W_uv, k_pool, v_pool, p.d.s_q, dev_status, st);
  }
  return e == cudaSuccess ? GQLA_OK : GQLA_ERR_CUDA;
}

gqla_status gqla_splitkv_combine(int32_t num_splits, int32_t rows, int32_t D, const float* o_part,
                                 const float* lse_part, void* out, gqla_dtype out_dtype, float* lse_out,
                                 void* stream) {
  if (num_splits < 1 || rows < 1 || D < 1 || !o_part || !lse_part || !out) return GQLA_ERR_INVALID_ARG;
  if (out_dtype != GQLA_F32 && out_dtype != GQLA_BF16) return GQLA_ERR_INVALID_ARG;
  cudaError_t e = combine(num_splits, rows, D, o_part, lse_part, out, out_dtype, lse_out, (cudaStream_t)stream);
  return e == cudaSuccess ? GQLA_OK : GQLA_ERR_CUDA;
}

gqla_status gqla_decode_gqa(const gqla_dims* dims, const gqla_kv_layout* layout, const void* q,
                            const void* k_pool, const void* v_pool, void* out, float* lse, int32_t num_splits,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  Problem p;
  gqla_status s = make_problem(dims, layout, num_splits, GQLA_PATH_GQA, &p);
  if (s != GQLA_OK) return s;
  if (!q || !k_pool || !v_pool || !out) return GQLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out)) return GQLA_ERR_ALIGNMENT;
  const bool tc = tc_gqa_supports(p);
  if (!tc && !simt_supports(p, GQLA_PATH_GQA)) return GQLA_ERR_UNSUPPORTED;
  Workspace w;
  size_t need = ws_layout(p, GQLA_PATH_GQA, false, &w, (char*)workspace);
  if (need > 0 && (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u))) return GQLA_ERR_WORKSPACE;
  cudaError_t e = gqa_decode_call(p, tc, q, k_pool, v_pool, out, lse, w, dev_status, (cudaStream_t)stream);
  return e == cudaSuccess ? GQLA_OK : GQLA_ERR_CUDA;
}


gqla_status gqla_decode_absorb(const gqla_dims* dims, const gqla_kv_layout* layout, const void* q,
                               const void* latent, const void* W_uk, const void* W_uv, void* out, float* lse,
                               int32_t num_splits, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                               void* stream) {
  Problem p;
  gqla_status s = make_problem(dims, layout, num_splits, GQLA_PATH_ABSORB, &p);
  if (s != GQLA_OK) return s;
  if (!q || !latent || !W_uk || !W_uv || !out) return GQLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(latent) || !aligned16(W_uk) || !aligned16(W_uv) || !aligned16(out))
    return GQLA_ERR_ALIGNMENT;
  const bool tc = tc_absorb_supports(p);
  if (!tc && !simt_supports(p, GQLA_PATH_ABSORB)) return GQLA_ERR_UNSUPPORTED;
  Workspace w;
  size_t need = ws_layout(p, GQLA_PATH_ABSORB, tc, &w, (char*)workspace);
  if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)) return GQLA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  const int S = p.plan.num_splits;
  cudaError_t e;
  if (tc) {
    e = tc_absorb_decode(p, q, latent, W_uk, W_uv, out, lse, w, dev_status, st);
  } else {
    e = simt_absorb_q(p, q, W_uk, (float*)w.qt, st);
    if (e == cudaSuccess)
      e = simt_decode(p, GQLA_PATH_ABSORB, q, (const float*)w.qt, latent, latent, nullptr,
                      S > 1 ? w.o_part : w.o_lat, S > 1 ? w.lse_part : lse, dev_status, st);
    if (e == cudaSuccess && S > 1) e = combine(S, p.rows, p.d.r, w.o_part, w.lse_part, w.o_lat, GQLA_F32, lse, st);
    if (e == cudaSuccess) e = simt_up_proj(p, w.o_lat, W_uv, out, st);
  }
  return e == cudaSuccess ? GQLA_OK : GQLA_ERR_CUDA;
}

}  // extern "C"
