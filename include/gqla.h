/*
 * gqla.h -- C ABI of the GQLA decode-attention library (libgqla.so, sm_100a).
 *
 * Group-Query Latent Attention keeps one joint latent c_KV (rank r) and one
 * decoupled RoPE key k_rope per cached token, and group-shared up-projections
 * W_uk^g, W_uv^g (one pair per group of m = n_h / G query heads).  The same
 * weights decode two ways ("GQLA: Group-Query Latent Attention for
 * Hardware-Adaptive Decoding", scholarbro.com, Abstract; "GQLA" on
 * chatpaper.ai, Abstract): the MQA-absorb path attends every head over the
 * latent cache with the query carried through W_uk^g, and the GQA path expands
 * the latent into a per-group K/V cache and runs grouped-query decode over it.
 * Both give, for batch b, new token i in [0, s_q) and head h in group g:
 *
 *     k_{g,t} = [ c_t W_uk^g ; k_rope_t ]      v_{g,t} = c_t W_uv^g
 *     s_t = scale * <q_{b,i,h}, k_{g,t}>        for t = 0 .. L_b - s_q + i
 *     out_{b,i,h} = sum_t softmax(s)_t v_{g,t}  lse_{b,i,h} = ln sum_t exp(s_t)
 *
 * Conventions shared by every entry point:
 *  - All pointers named *device* are CUDA device pointers owned by the caller;
 *    the library never allocates device memory (split-KV scratch is passed in
 *    as a workspace) and never frees anything.  The one exception is
 *    gqla_decode_gqa_noalloc, whose split scratch is a fixed 32 MiB
 *    library-owned __device__ array (described at that call).  Host structs
 *    are read during the call only.
 *  - Work is queued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *    and runs asynchronously; no call synchronises.  The tensor-core kernels
 *    are launched with programmatic stream serialisation: each call's first
 *    kernel waits for all earlier work on the stream before touching memory,
 *    and later kernels of the call may begin while their predecessor ends.
 *    Work the caller queues afterwards sees the call's results in stream
 *    order, except a kernel the caller itself launches with that attribute,
 *    which (as any such kernel) must execute griddepcontrol.wait first.
 *  - Arguments are validated on the host before any launch; a failed check
 *    returns a status and launches nothing.  A kernel launch failure returns
 *    GQLA_ERR_CUDA.
 *  - Problems only the device can see (a sequence shorter than s_q or longer
 *    than its slots, a page id outside the pool) set bits in *dev_status
 *    (device int32, may be NULL) and the affected rows are written as zeros with
 *    lse = -inf; the kernel never traps.
 *  - Element type of q, caches, weights and out is dims.dtype (fp32 or bf16);
 *    lse and all accumulation are fp32.  The fp32 kernels compute in true fp32
 *    (no TF32); the bf16 kernels use tensor cores with fp32 accumulation.
 *  - Row-major layouts:
 *      q       [B, s_q, n_h, d_nope + d_rope]       nope part first
 *      latent  token rows [c_KV (r) ; k_rope (d_rope)]
 *      K pool  token rows [G, d_nope + d_rope]      (per-group key with its own
 *                                                     copy of k_rope), or
 *              [G * d_nope + d_rope] with dims.k_layout = GQLA_K_SHARED_ROPE
 *      V pool  token rows [G, d_v]
 *      W_uk    [G, r, d_nope]      W_uv [G, r, d_v]
 *      out     [B, s_q, n_h, d_v]  lse [B, s_q, n_h]
 *    Head h belongs to group h / m.  Rotary embedding is applied before these
 *    calls (q_rope and k_rope arrive rotated).
 */
#ifndef GQLA_H
#define GQLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gqla_status {
  GQLA_OK = 0,
  GQLA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, n_h % G != 0, s_q out of [1,4] */
  GQLA_ERR_UNSUPPORTED = 2,  /* valid GQLA dims no kernel of this library handles */
  GQLA_ERR_ALIGNMENT = 3,    /* a pointer or row pitch below the 16-byte rule */
  GQLA_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than gqla_workspace_bytes */
  GQLA_ERR_CUDA = 5          /* a CUDA call or kernel launch failed */
} gqla_status;

typedef enum gqla_dtype { GQLA_F32 = 0, GQLA_BF16 = 1 } gqla_dtype;

typedef enum gqla_path { GQLA_PATH_ABSORB = 0, GQLA_PATH_GQA = 1 } gqla_path;

/* Row layout of the expanded K pool of the GQA path.  The decoupled RoPE key
 * is one vector per token shared by every head ("GQLA" scholarbro.com
 * Abstract: a shared decoupled-RoPE key beside the joint latent), so a K row
 * may either repeat it in every group or hold it once:
 *   GQLA_K_PER_GROUP    row = G x [k_nope (d_nope) ; k_rope (d_rope)]
 *                       (every group is a plain GQA key head of d_nope+d_rope)
 *   GQLA_K_SHARED_ROPE  row = [G x k_nope (d_nope) ; k_rope (d_rope)]
 *                       (G*d_nope + d_rope elements: at G = 16, 2112 instead
 *                       of 3072 per token, 4160 instead of 5120 with V)
 * Both give the same scores; the second streams fewer bytes. */
typedef enum gqla_k_layout { GQLA_K_PER_GROUP = 0, GQLA_K_SHARED_ROPE = 1 } gqla_k_layout;

/* Device status bits written to *dev_status (OR-ed). */
#define GQLA_DEV_SHORT_SEQ 1   /* seq_lens[b] < s_q (or < 0): rows of b zeroed  */
#define GQLA_DEV_OVERFLOW 2    /* seq_lens[b] above the sequence's token slots  */
#define GQLA_DEV_BAD_PAGE 4    /* block_table entry outside [0, num_pages)      */
#define GQLA_DEV_TIMEOUT 8     /* a bounded pipeline wait gave up               */

/* Model dimensions of one attention layer.  The group count must divide n_h
 * ("gqla_attn" module page, frankenstein-transformer docs: GQLAAttention
 * raises when gqla_num_groups does not divide num_heads).  scale multiplies
 * <q, k> (commonly 1/sqrt(d_nope + d_rope)); s_q is the number of new tokens
 * per sequence decoded in one step (multi-token prediction, 1..4). */
typedef struct gqla_dims {
  int32_t n_h;      /* query heads                                   */
  int32_t G;        /* groups (KV heads of the expanded path)        */
  int32_t d_nope;   /* per-head query/key dims without RoPE          */
  int32_t d_rope;   /* shared decoupled-RoPE key dims                */
  int32_t d_v;      /* value dims per head                           */
  int32_t r;        /* latent rank of c_KV                           */
  int32_t s_q;      /* new tokens per sequence, 1..4                 */
  float scale;      /* softmax scale                                 */
  gqla_dtype dtype; /* element type of q, caches, weights and out    */
  int32_t k_layout; /* gqla_k_layout of the expanded K pool (GQA path
                       and expansion; 0 = GQLA_K_PER_GROUP)            */
} gqla_dims;

/* Where token t of sequence b lives in a token pool (the same geometry serves
 * the latent pool and the expanded K and V pools).  A pool is an array of
 * token rows; `row` below is that pool's row width in elements.
 *   contiguous (page_size == 0): pool [batch, capacity, row]; token (b, t) is
 *     row b * capacity + t.
 *   paged (page_size > 0): pool [num_pages, page_size, row]; token (b, t) is
 *     row block_table[b * max_blocks_per_seq + t / page_size] * page_size
 *     + t % page_size (fixed-size blocks as in PagedAttention, "Grouped Query
 *     Attention (GQA)" glossary, section "GQA et techniques connexes").
 * seq_lens[b] counts all tokens of sequence b, its s_q new tokens included;
 * slots past it may hold any finite values. */
typedef struct gqla_kv_layout {
  int32_t batch;                /* B > 0                                      */
  const int32_t* seq_lens;      /* device [batch]                              */
  int32_t max_seq_len;          /* host upper bound on seq_lens (plans splits) */
  int32_t page_size;            /* 0 = contiguous; else tokens per page        */
  int32_t capacity;             /* contiguous: token slots per sequence        */
  const int32_t* block_table;   /* paged: device [batch, max_blocks_per_seq]   */
  int32_t max_blocks_per_seq;   /* paged: columns of block_table               */
  int32_t num_pages;            /* paged: pages in the pool                    */
} gqla_kv_layout;

/* Per-group cache expansion, the GQA path's precondition ("GQLA" chatpaper.ai
 * Abstract: a GQA path with a per-group expanded cache):
 *   K[b,t,g,:] = [ c_{b,t} W_uk^g ; k_rope_{b,t} ],  V[b,t,g,:] = c_{b,t} W_uv^g
 * (with GQLA_K_SHARED_ROPE the k_rope part is stored once per token row)
 * for tokens t in [max(0, seq_lens[b] - tail_tokens), seq_lens[b]) of every
 * sequence (tail_tokens <= 0: all tokens).  tail_tokens = s_q expands just the
 * tokens appended by one decode step.
 *   latent  device, pool with rows of r + d_rope elements
 *   W_uk    device [G, r, d_nope];  W_uv device [G, r, d_v]
 *   k_pool  device, pool with rows of G*(d_nope+d_rope) elements, or
 *           G*d_nope + d_rope with GQLA_K_SHARED_ROPE (written)
 *   v_pool  device, pool with rows of G*d_v elements (written)
 * All three pools use `layout`.  Rows outside the expanded range are not
 * touched.  With the bf16 tensor-core kernels the whole-cache form
 * (tail_tokens <= 0) launches clusters of two CTAs (one MMA tile over both);
 * on a device where such pairs cannot be resident it uses one CTA per tile.
 * Every output element is the same K-ordered sum of bf16 products either
 * way. */
gqla_status gqla_expand_cache(const gqla_dims* dims, const gqla_kv_layout* layout,
                              const void* latent, const void* W_uk, const void* W_uv,
                              void* k_pool, void* v_pool, int32_t tail_tokens,
                              int32_t* dev_status, void* stream);

/* Decode-time cache append: the per-step write of the new tokens before the
 * attention ("GQLA" chatpaper.ai Abstract: the absorb path caches the joint
 * latent, the GQA path a per-group expanded cache).  For every sequence b the
 * s_q rows new_rows[b, i, :] = [c_KV (r) ; k_rope (d_rope)] are written to
 * token positions seq_lens[b] - s_q + i of the latent pool (seq_lens already
 * count the new tokens), and, when k_pool and v_pool are given, those tokens
 * are expanded into the per-group pools as gqla_expand_cache does.
 *   new_rows  device [B, s_q, r + d_rope]
 *   latent    device pool (written at the new positions only), or NULL for
 *             a GQA-only cache: then only the expansion happens (bf16 dims
 *             of the tensor-core kernels only; else GQLA_ERR_UNSUPPORTED)
 *   W_uk, W_uv, k_pool, v_pool  as for gqla_expand_cache; k_pool/v_pool may
 *             both be NULL (absorb-only cache), then W_uk/W_uv are unused.
 *             latent and k_pool may not both be NULL.
 * With the tensor-core kernels the expansion reads the dense new_rows, many
 * sequences' tokens to an MMA tile; each token's K/V rows are the same
 * numbers gqla_expand_cache produces for it.
 * A sequence shorter than s_q, longer than its slots or with a page outside
 * the pool is skipped and flagged in *dev_status. */
gqla_status gqla_append_tokens(const gqla_dims* dims, const gqla_kv_layout* layout, const void* new_rows,
                               void* latent, const void* W_uk, const void* W_uv, void* k_pool,
                               void* v_pool, int32_t* dev_status, void* stream);

/* MQA-absorb decode ("GQLA" chatpaper.ai Abstract: an MQA-absorb path
 * identical to MLA's).  Per head: q~ = W_uk^g q_nope, scores
 * scale*(<q~, c_t> + <q_rope, k_rope_t>), latent output sum_t p_t c_t, then
 * out = that latent output times W_uv^g.
 *   q        device [B, s_q, n_h, d_nope + d_rope]
 *   latent   device pool, rows of r + d_rope
 *   out      device [B, s_q, n_h, d_v] (written)
 *   lse      device fp32 [B, s_q, n_h] or NULL
 *   num_splits  key-range splits per sequence, 0 = chosen by the library
 *   workspace   device, >= gqla_workspace_bytes(dims, layout, num_splits,
 *               GQLA_PATH_ABSORB) bytes, 256-byte aligned; contents clobbered */
gqla_status gqla_decode_absorb(const gqla_dims* dims, const gqla_kv_layout* layout,
                               const void* q, const void* latent,
                               const void* W_uk, const void* W_uv,
                               void* out, float* lse, int32_t num_splits,
                               void* workspace, size_t workspace_bytes,
                               int32_t* dev_status, void* stream);

/* GQA decode over the expanded per-group cache ("GQLA" chatpaper.ai Abstract;
 * grouped-query attention as in the "Grouped Query Attention (GQA)" glossary,
 * section "Fonctionnement de la GQA": every head of group g attends over the
 * group's K/V).
 *   q       device [B, s_q, n_h, d_nope + d_rope]
 *   k_pool  device pool, rows of G*(d_nope+d_rope) (G*d_nope + d_rope with
 *           GQLA_K_SHARED_ROPE);  v_pool rows of G*d_v
 *   out, lse, num_splits, workspace as for gqla_decode_absorb (path GQA). */
gqla_status gqla_decode_gqa(const gqla_dims* dims, const gqla_kv_layout* layout,
                            const void* q, const void* k_pool, const void* v_pool,
                            void* out, float* lse, int32_t num_splits,
                            void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, void* stream);

/* gqla_decode_gqa without a workspace argument, for callers that cannot
 * allocate device memory: a plug-in whose host framework owns every byte of
 * device memory and gives it no allocator, or a decode loop that must not call
 * cudaMalloc/cudaFree (they synchronise the device) on its hot path.  The
 * pages have no counterpart to this call; it is a deployment convenience.
 *   Same arguments, layouts, results and errors as gqla_decode_gqa, minus the
 *   workspace.  The split scratch is a library-owned device array of 32 MiB,
 *   reserved on every GPU that loads the library and held until the process
 *   exits.  A problem whose split scratch would exceed 32 MiB (about
 *   num_splits * B * s_q * n_h * (d_v + 1) * 4 bytes) is refused with
 *   GQLA_ERR_WORKSPACE before any launch: pass a smaller num_splits.
 *   The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   The address is kept with the CUDA context it belongs to: after a device
 *   reset, or when that context is replaced, the next call looks it up again
 *   (so that call, too, belongs outside a stream capture).
 *   All calls share the one array, so calls whose kernels may overlap on the
 *   GPU (different streams, or other threads) race: serialise them. */
gqla_status gqla_decode_gqa_noalloc(const gqla_dims* dims, const gqla_kv_layout* layout,
                                    const void* q, const void* k_pool, const void* v_pool,
                                    void* out, float* lse, int32_t num_splits,
                                    int32_t* dev_status, void* stream);

/* Log-sum-exp merge of attention results over disjoint key ranges:
 *   lse[row] = ln sum_j exp(lse_part[j,row]);
 *   out[row] = sum_j exp(lse_part[j,row] - lse[row]) * o_part[j,row,:]
 * A part with lse = -inf has weight 0; a row whose parts are all -inf gets
 * out = 0, lse = -inf.  (The pages name FlashAttention-style kernels --
 * "Grouped Query Attention (GQA)" glossary, "GQA et techniques connexes" --
 * but print no merge rule; this is the identity softmax obeys.)
 *   o_part   device fp32 [num_splits, rows, D];  lse_part device fp32 [num_splits, rows]
 *   out      device [rows, D] of out_dtype;      lse_out device fp32 [rows] or NULL */
gqla_status gqla_splitkv_combine(int32_t num_splits, int32_t rows, int32_t D,
                                 const float* o_part, const float* lse_part,
                                 void* out, gqla_dtype out_dtype, float* lse_out,
                                 void* stream);

/* Workspace bytes a decode call needs (0 when none), for the given split count
 * (0 = the library's choice, the same one the decode call will make). */
size_t gqla_workspace_bytes(const gqla_dims* dims, const gqla_kv_layout* layout,
                            int32_t num_splits, gqla_path path);

/* Split count a decode call with this num_splits argument will use. */
int32_t gqla_num_splits(const gqla_dims* dims, const gqla_kv_layout* layout,
                        int32_t num_splits, gqla_path path);

/* Hardware figures for gqla_select_path.  NULL selects the library's
 * defaults: the current device's SM count with the copy bandwidth and dense
 * bf16 tensor rate measured on a B200. */
typedef struct gqla_hw {
  int32_t sms;        /* streaming multiprocessors                      */
  double hbm_gbs;     /* device-memory copy bandwidth, GB/s              */
  double tc_tflops;   /* dense bf16 tensor-core rate, TFLOP/s            */
} gqla_hw;

typedef struct gqla_path_estimate {
  double absorb_us;   /* predicted device time of gqla_decode_absorb     */
  double gqa_us;      /* predicted device time of gqla_decode_gqa        */
  gqla_path path;     /* the faster of the two                           */
} gqla_path_estimate;

/* Runtime path choice ("GQLA" chatpaper.ai Abstract: the same weights run
 * either path and the runtime picks the one that suits the hardware).  From
 * the dims (k_layout included), the layout's batch and max_seq_len, and the
 * batch's total cached tokens (sum of seq_lens, known to the caller; the
 * device array is not read), predicts both calls' device times with a model
 * of this library's kernels (bound resource, tile shape, split plan and
 * measured efficiency) on the given hardware, and names the faster path.
 * Host only: launches nothing.  Errors: INVALID_ARG for bad dims or layout,
 * total_tokens outside [batch * s_q, batch * max_seq_len], or non-positive
 * hardware figures. */
gqla_status gqla_select_path(const gqla_dims* dims, const gqla_kv_layout* layout, int64_t total_tokens,
                             const gqla_hw* hw, gqla_path_estimate* est);

/* Cached bytes per token per layer: absorb path (r + d_rope) elements, GQA
 * path G*(d_nope + d_rope + d_v) elements (G*(d_nope + d_v) + d_rope with
 * GQLA_K_SHARED_ROPE), times the element size.  At
 * LLaMA-3-8B shapes the absorb cache is (512+64)/(2*8*128) = 28.125 % of a
 * GQA baseline with 8 KV heads of 128 ("GQLA" chatpaper.ai Abstract). */
size_t gqla_cache_bytes_per_token(const gqla_dims* dims, gqla_path path);

/* Static text for a status code. */
const char* gqla_status_string(gqla_status status);

/* Library version, e.g. "gqla-b200 0.1". */
const char* gqla_version(void);

/* Number of CUDA kernels this library has launched in this process so far
 * (all devices, all streams; a diagnostic counter, thread-safe). */
uint64_t gqla_launch_counter(void);

#ifdef __cplusplus
}
#endif

#endif /* GQLA_H */
