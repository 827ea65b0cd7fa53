/*
 * palu.h — C ABI of libpalu.so: Palu's decode step read straight from a
 * low-rank latent KV cache, on NVIDIA B200 (sm_100a).
 *
 * The method (cited by page title and section):
 *   "PALU 论文低秩投影分解：从数学结构到工程落地，一次讲透" (palu-low-rank explainer)
 *     §低秩投影分解: K = x W_k ≈ x A_k B_k, V ≈ x A_v B_v with A ∈ R^{d_model×r},
 *       B ∈ R^{r×d}; the cache holds z_k = x A_k and z_v = x A_v instead of K, V.
 *     §把它放进一次真实推理流程里看 (Prefill 阶段 / Decode 阶段): prefill computes and
 *       caches z; decode reads z and rebuilds K/V through B, or fuses that into the
 *       attention kernel without materialising K/V.
 *   "Palu: Compressing KV-Cache with Low-Rank Projection" (arXiv 2407.21118 v2
 *     abstract): medium-grained (group-head) decomposition, RoPE-based attention,
 *     quantisation compatibility, fused GPU kernels.
 *
 * Conventions shared by every entry point
 *   - Heads are grouped consecutively: head h belongs to group h / group_size
 *     and uses columns [(h % group_size)·head_dim, +head_dim) of its group's B.
 *     G = num_heads / group_size groups, group width W = group_size·head_dim.
 *   - All tensors are dense, row-major, in DEVICE memory owned by the caller.
 *     The library allocates nothing, keeps no per-call state, and never frees
 *     what it is given.  Tensor-map descriptors are encoded on the host for
 *     each launch and passed by value; no state survives a call.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument checks are synchronous and return a status
 *     before anything is launched.  Faults found by the kernels themselves
 *     (a page index past the pool, a bounded wait that ran out) are recorded
 *     in a status word at the start of the workspace, read back with
 *     palu_get_device_status(); the kernels skip the bad access instead of
 *     faulting.
 *   - No exception, abort or trap crosses this ABI.
 *
 * Latent-cache layout (the "cache manager" side; paged by sequence):
 *   K pool  [num_pages][G] blocks of page_size tokens × row_k bytes
 *   V pool  [num_pages][G] blocks of page_size tokens × row_v bytes
 *           row_k = rank_k elements of the latent dtype (int4: rank_k/2 bytes);
 *           row_k and row_v must be multiples of 128 bytes.
 *   Inside one (page, group) block the bytes are column-blocked and swizzled:
 *   byte o of token t's latent row lives at
 *       (o / 128)·(page_size·128) + t·128 + (((o % 128) / 16) XOR (t % 8))·16 + o % 16
 *   i.e. 128-byte column blocks of all page_size tokens, the 16-byte units of
 *   each token's 128 bytes permuted by t mod 8.  That is the 128-byte-swizzled
 *   shared-memory image the tensor-core MMAs consume, so every 128-byte column
 *   block of a page reaches shared memory as one contiguous bulk copy.
 *   int4 scale pools [num_pages][G][page_size][srow]   srow = 16-byte padded
 *           rank/32 fp16 scales (one per 32 consecutive latent entries), token-major
 *   pos pool [num_pages][page_size] int32 (optional)
 *   A token lives at slot = page·page_size + offset; page_size is a multiple of 8.
 */
#ifndef PALU_H_
#define PALU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* palu_stream_t; /* same handle as cudaStream_t */

typedef enum palu_status {
  PALU_OK = 0,
  PALU_ERR_INVALID_ARG = 1,    /* NULL pointer, negative size, inconsistent shape */
  PALU_ERR_UNSUPPORTED = 2,    /* a valid shape/dtype this build has no kernel for */
  PALU_ERR_ALIGNMENT = 3,      /* a pointer or row stride not 16-byte aligned */
  PALU_ERR_WORKSPACE = 4,      /* workspace NULL or smaller than the size query */
  PALU_ERR_CUDA = 5,           /* a CUDA runtime/launch error (see palu_last_cuda_error) */
  PALU_ERR_DEVICE_TIMEOUT = 6, /* a kernel's bounded wait ran out (device status) */
  PALU_ERR_DEVICE_BOUNDS = 7   /* a kernel found a page/slot index out of range */
} palu_status;

typedef enum palu_dtype {
  PALU_F32 = 0,
  PALU_F16 = 1,
  PALU_BF16 = 2,
  PALU_INT4 = 3 /* latent dtype only */
} palu_dtype;

typedef struct palu_config {
  int32_t num_heads;    /* H query heads (= KV heads) */
  int32_t head_dim;     /* d_h, even */
  int32_t group_size;   /* g heads share one latent (medium-grained decomposition);
                           num_heads / group_size <= 64 groups */
  int32_t rank_k;       /* r_k latent width per group for keys */
  int32_t rank_v;       /* r_v latent width per group for values */
  int32_t page_size;    /* tokens per cache page */
  float rope_base;      /* RoPE base (10000); 0 turns RoPE off */
  int32_t act_dtype;    /* palu_dtype of q, x, A, B and out: F32 | F16 | BF16 */
  int32_t latent_dtype; /* palu_dtype of the cache: act_dtype, or INT4 with F16/BF16 act */
} palu_config;

/* Bytes of one page of each pool for `cfg` (scale pages are 0 unless INT4).
 * Returns PALU_ERR_INVALID_ARG / PALU_ERR_UNSUPPORTED for a bad config. */
palu_status palu_cache_strides(const palu_config* cfg, size_t* k_page_bytes, size_t* v_page_bytes,
                               size_t* k_scale_page_bytes, size_t* v_scale_page_bytes);

/* Workspace bytes palu_compress_append needs for n_tokens rows (status word +
 * per-split partial sums and counters when the K range is split across CTAs).
 * Always >= 256.  Zero-fill a workspace once before its first use; every call
 * leaves its counters back at zero (after a call whose kernels reported
 * PALU_ERR_DEVICE_TIMEOUT, zero-fill it again). */
palu_status palu_compress_workspace_size(const palu_config* cfg, int n_tokens, int d_model,
                                         size_t* bytes);

/* Compress / append — the prefill (and per-step append) projection.
 * "PALU 论文低秩投影分解" §低秩投影分解 (z_k = x A_k, z_v = x A_v) and
 * §把它放进一次真实推理流程里看, Prefill 阶段 (compute z and cache it).
 *
 *   x        [n_tokens][d_model]        act dtype
 *   A_k      [d_model][G·rank_k]        act dtype (group g = columns [g·r_k, +r_k))
 *   A_v      [d_model][G·rank_v]        act dtype
 *   slot_mapping [n_tokens] int32       destination slot page·page_size + offset;
 *                                       a negative slot skips that row
 *   positions [n_tokens] int32 or NULL  written to pos_pool[slot] when both are
 *                                       non-NULL
 *   zk_pool, zv_pool, zk_scales, zv_scales, pos_pool: the cache (layout above);
 *            scales are used only for INT4 latents (else may be NULL)
 *   num_pages  pool capacity in pages (slots >= num_pages·page_size are
 *            skipped and reported as PALU_ERR_DEVICE_BOUNDS)
 *
 * Each latent row is z = x·A accumulated in float32 and rounded to nearest even
 * into the latent dtype; INT4 rows are quantised per 32 entries with a
 * symmetric fp16 scale s = fp16(max|z|/7) and codes clamp(rint(z/s), -7, 7),
 * two's-complement nibbles, even entry in the low nibble.
 * d_model must be a multiple of 64; every pointer 16-byte aligned.
 */
palu_status palu_compress_append(const palu_config* cfg, int n_tokens, int d_model,
                                 const void* x, const void* A_k, const void* A_v,
                                 const int32_t* slot_mapping, const int32_t* positions,
                                 void* zk_pool, void* zv_pool, void* zk_scales, void* zv_scales,
                                 int32_t* pos_pool, int num_pages,
                                 void* workspace, size_t workspace_bytes, palu_stream_t stream);

/* The split count palu_decode_attn uses when asked for num_splits = 0. */
palu_status palu_decode_num_splits(const palu_config* cfg, int batch, int max_pages,
                                   int* num_splits);

/* Workspace bytes palu_decode_attn needs (status word + per-split partials
 * (m, l, a[rank_v]) in float32 for every (sequence, head, split)). */
palu_status palu_decode_workspace_size(const palu_config* cfg, int batch, int max_pages,
                                       int num_splits, size_t* bytes);

/* One decode step of attention over the latent cache.
 * "PALU 论文低秩投影分解" §把它放进一次真实推理流程里看, Decode 阶段: read z, rebuild
 * keys through B_k on the fly (K = z_k B_k, rotated by RoPE at each token's
 * position), softmax(q'K'^T/sqrt(d_h)) over the cached tokens, and reduce values
 * in latent space, out_h = (p · z_v) · B_v — V is never materialised.  The
 * context is split into num_splits page ranges per sequence whose partials are
 * merged by a log-sum-exp combine.
 *
 *   q          [batch][H][head_dim]   act dtype, before RoPE
 *   q_pos      [batch] int32          the query's position
 *   zk_pool ... pos_pool              the cache; pos_pool NULL => a token's
 *                                     position is its index in the sequence
 *   page_table [batch][max_pages] int32 physical page of each logical page
 *   seq_lens   [batch] int32          cached tokens per sequence (0 allowed)
 *   num_pages  pool capacity in pages (checked on the device)
 *   B_k        [G][rank_k][W]         act dtype
 *   B_v        [G][rank_v][W]         act dtype
 *   out        [batch][H][head_dim]   act dtype (written)
 *   lse        [batch][H] float32 or NULL: m + ln(sum), -inf for an empty sequence
 *   workspace  >= palu_decode_workspace_size bytes, 256-byte aligned
 *   num_splits 0 = automatic
 * Attends over all seq_lens[b] tokens (the caller appends the current token
 * first); an empty sequence gives out = 0.
 */
palu_status palu_decode_attn(const palu_config* cfg, int batch, const void* q, const int32_t* q_pos,
                             const void* zk_pool, const void* zv_pool, const void* zk_scales,
                             const void* zv_scales, const int32_t* pos_pool,
                             const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                             int num_pages, const void* B_k, const void* B_v, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, int num_splits,
                             palu_stream_t stream);

/* Multi-token decode step: num_queries (1..PALU_MAX_QUERIES) new tokens of
 * every sequence query the cache at once, as when a step scores several
 * appended tokens together (a chunk of a prompt, or drafted tokens to verify).
 * "PALU 论文低秩投影分解" §把它放进一次真实推理流程里看: prefill and decode consume
 * the same latent cache; each query is the decode step above, restricted to
 * the cached tokens whose position is at most its own (causal among the new
 * tokens, which the caller appends to the cache first).
 *   q      [batch][num_queries][H][head_dim]   act dtype, before RoPE
 *   q_pos  [batch][num_queries] int32          each query's position
 *   out    [batch][num_queries][H][head_dim]   act dtype (written)
 *   lse    [batch][num_queries][H] float32 or NULL
 *   workspace >= palu_decode_multi_workspace_size bytes, 256-byte aligned
 * Every other argument is as in palu_decode_attn.  A query that sees no token
 * gives out = 0 and lse = -inf.  H·head_dim·(element size) must be a multiple of
 * 16 bytes when num_queries > 1 (PALU_ERR_ALIGNMENT otherwise). */
#define PALU_MAX_QUERIES 16
palu_status palu_decode_multi_workspace_size(const palu_config* cfg, int batch, int num_queries,
                                             int max_pages, int num_splits, size_t* bytes);
palu_status palu_decode_attn_multi(const palu_config* cfg, int batch, int num_queries, const void* q,
                                   const int32_t* q_pos, const void* zk_pool, const void* zv_pool,
                                   const void* zk_scales, const void* zv_scales, const int32_t* pos_pool,
                                   const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                                   int num_pages, const void* B_k, const void* B_v, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, int num_splits,
                                   palu_stream_t stream);

/* Layers whose head groups carry different ranks: the output of Palu's rank
 * search.  "PALU 论文低秩投影分解" §为什么还能保精度 (the rank is searched rather
 * than cut uniformly everywhere), §怎么落地 路线 B (ranks found offline per layer
 * and per group of heads, then served from the compressed cache) and
 * §风险、边界和别踩的坑 风险 1 (one rank for every layer loses accuracy or gain).
 * A per-layer rank needs nothing new: each layer has its own config.  These
 * calls take a rank pair per group instead of cfg->rank_k / cfg->rank_v:
 *   ranks_k, ranks_v  [G] int32, HOST memory, read during the call only.  Each
 *            pair must be valid in a config of its own (the rank rules of
 *            palu_config).  NULL for both = every group uses cfg's ranks, and
 *            the call is exactly its uniform counterpart.
 * Layout, with r_k,g the key rank of group g (V and the int4 scale pools the
 * same way, with their own row sizes):
 *   K pool  page p holds every group's block back to back: group g's block of
 *           page_size rows of row_k,g bytes starts at
 *           p·k_page_bytes + Σ_{g'<g} page_size·row_k,g'
 *           (palu_cache_strides_ranked gives k_page_bytes and those offsets);
 *           inside the block the swizzled layout above applies unchanged.
 *   A_k     [d_model][Σ_g r_k,g]: group g's columns start at Σ_{g'<g} r_k,g'
 *   B_k     [Σ_g r_k,g][W]: group g's rows start at Σ_{g'<g} r_k,g'
 * With equal ranks this is byte for byte the uniform layout.  Compress runs one
 * launch for every group; decode runs one split launch and one combine per set
 * of groups sharing a value rank and kernel family (key ranks may differ within
 * a set), the sets one after another on `stream`.  Every other argument, rule
 * and status is that of the uniform call named in each comment. */
/* as palu_cache_strides; k_group_offsets / v_group_offsets [G] (optional)
 * receive the byte offset of each group's block within a K / V page.  In an
 * int4 scale page, group g's block starts at Σ_{g'<g} page_size·srow_g'. */
palu_status palu_cache_strides_ranked(const palu_config* cfg, const int32_t* ranks_k, const int32_t* ranks_v,
                                      size_t* k_page_bytes, size_t* v_page_bytes, size_t* k_scale_page_bytes,
                                      size_t* v_scale_page_bytes, size_t* k_group_offsets,
                                      size_t* v_group_offsets);
/* as palu_compress_workspace_size / palu_compress_append */
palu_status palu_compress_ranked_workspace_size(const palu_config* cfg, const int32_t* ranks_k,
                                                const int32_t* ranks_v, int n_tokens, int d_model, size_t* bytes);
palu_status palu_compress_append_ranked(const palu_config* cfg, const int32_t* ranks_k, const int32_t* ranks_v,
                                        int n_tokens, int d_model, const void* x, const void* A_k, const void* A_v,
                                        const int32_t* slot_mapping, const int32_t* positions, void* zk_pool,
                                        void* zv_pool, void* zk_scales, void* zv_scales, int32_t* pos_pool,
                                        int num_pages, void* workspace, size_t workspace_bytes,
                                        palu_stream_t stream);
/* as palu_decode_multi_workspace_size / palu_decode_attn_multi (num_queries = 1
 * is palu_decode_attn) */
palu_status palu_decode_ranked_workspace_size(const palu_config* cfg, const int32_t* ranks_k,
                                              const int32_t* ranks_v, int batch, int num_queries, int max_pages,
                                              int num_splits, size_t* bytes);
palu_status palu_decode_attn_ranked(const palu_config* cfg, const int32_t* ranks_k, const int32_t* ranks_v,
                                    int batch, int num_queries, const void* q, const int32_t* q_pos,
                                    const void* zk_pool, const void* zv_pool, const void* zk_scales,
                                    const void* zv_scales, const int32_t* pos_pool, const int32_t* page_table,
                                    int max_pages, const int32_t* seq_lens, int num_pages, const void* B_k,
                                    const void* B_v, void* out, float* lse, void* workspace,
                                    size_t workspace_bytes, int num_splits, palu_stream_t stream);

/* Allocation-free decode step (the paper has no counterpart: this is a
 * deployment convenience of this library).
 * Some callers cannot call cudaMalloc at all: plug-ins whose host framework
 * owns all device memory and forbids further allocations, processes held to a
 * fixed device-memory budget, or latency-critical paths that must not pay for
 * an allocation (cudaMalloc can synchronise the device).  This entry point runs
 * exactly palu_decode_attn, but keeps the workspace in a fixed array of device
 * memory owned by the library: PALU_NOALLOC_SCRATCH_BYTES on every GPU that
 * loads the library, held until the process exits.  The caller still passes
 * every input and output.
 *   - Calls whose workspace (palu_decode_workspace_size) exceeds the array
 *     return PALU_ERR_WORKSPACE before launching anything.
 *   - The first call on a device looks up the array's device address for that
 *     device (cudaGetSymbolAddress, with that device current); make that first
 *     call before any stream capture.  Only a successful lookup is kept: a
 *     call whose lookup failed returns PALU_ERR_CUDA and the next call on that
 *     device tries again.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; each call clears the status word (an asynchronous memset on
 *     `stream`) and rewrites all partials.  Calls that overlap on the GPU (on
 *     different streams, or from different threads) race on the array: the
 *     caller must order them.
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   - status_out NULL: asynchronous like palu_decode_attn; faults the kernels
 *     detect are still skipped, but not reported.  status_out non-NULL: the
 *     call waits for `stream`, returns the device status (PALU_OK,
 *     PALU_ERR_DEVICE_TIMEOUT or PALU_ERR_DEVICE_BOUNDS) and stores the
 *     kernel's detail code in *status_out (host memory). */
#define PALU_NOALLOC_SCRATCH_BYTES (8u << 20)
palu_status palu_decode_attn_noalloc(const palu_config* cfg, int batch, const void* q,
                                     const int32_t* q_pos, const void* zk_pool, const void* zv_pool,
                                     const void* zk_scales, const void* zv_scales,
                                     const int32_t* pos_pool, const int32_t* page_table, int max_pages,
                                     const int32_t* seq_lens, int num_pages, const void* B_k,
                                     const void* B_v, void* out, float* lse, int num_splits,
                                     palu_stream_t stream, int32_t* status_out);

/* Synchronises `stream`, then reads and clears the device status word at the
 * start of `workspace`.  Returns PALU_OK, PALU_ERR_DEVICE_TIMEOUT or
 * PALU_ERR_DEVICE_BOUNDS; *detail (optional) receives the kernel's detail code. */
palu_status palu_get_device_status(void* workspace, palu_stream_t stream, int32_t* detail);

/* Static description of a status code. */
const char* palu_status_string(palu_status status);

/* The last CUDA error string seen by this thread's calls ("" if none). */
const char* palu_last_cuda_error(void);

/* Which kernel family a decode call with this config would launch:
 * 0 = none (unsupported), 1 = CUDA-core kernels, 2 = tcgen05/TMA kernels,
 * 3 = the fused no-RoPE kernel (query folded through B_k, scores straight
 * from z_k). */
int palu_decode_kernel_kind(const palu_config* cfg);

/* Phase tracing of the tensor-core decode kernel, for performance analysis.
 * After this call every palu_decode_attn launch of the tensor-core kernel
 * records, per CTA and per tile (up to `tiles_per_cta`), the SM clock
 * (clock64, relative to the CTA's start) at kPaluTraceEvents points:
 *   0 MMA: slot free, key MMAs of the tile start   1 MMA: key MMAs issued
 *   2 MMA: the tile's value MMAs issued            3 epilogue: tile keys ready
 *   4 epilogue: scores done (both warpgroups)      5 epilogue: P written
 *   6 value latents of the tile: first copy issued (int4: codes staged)
 *   7 MMA thread: the tile's first value-latent block seen in shared memory
 * into `buffer` (device memory, int64 [cta][event][tile], CTA = linear block
 * index); entries never reached stay as they were.  Pass NULL to stop.
 * `bytes` must cover grid CTAs × 8 × tiles_per_cta × 8 bytes of the launches
 * traced; launches whose grid does not fit are not traced.  Process-wide
 * setting, not thread-safe with concurrent decode calls. */
#define PALU_TRACE_EVENTS 8
palu_status palu_debug_trace(void* buffer, size_t bytes, int tiles_per_cta);

/* Test hook for the kernels' timeout path: every wait inside the tensor-core
 * kernels (compress and decode) is bounded, and on expiry the kernel records
 * PALU_ERR_DEVICE_TIMEOUT in the workspace status word, waits (with a bound of
 * its own) for the copies and MMAs it has already issued, frees its tensor
 * memory and returns, leaving the context usable.  The call's outputs are then
 * void; a compress workspace must be zero-filled again before its next use.
 *   wait_cycles  bound of each wait in SM clock cycles for launches after this
 *                call; 0 = the default (2^31 cycles, about a second at 2 GHz)
 *   stall        non-zero: the MMA thread of every tensor-core launch first
 *                waits on a barrier phase that nothing completes before its
 *                own teardown, so every such launch runs out that bound
 * palu_debug_timeout_test(0, 0) restores normal operation.  Process-wide, not
 * thread-safe with concurrent calls; meant for tests only.  Returns
 * PALU_ERR_INVALID_ARG for a negative wait_cycles. */
palu_status palu_debug_timeout_test(int64_t wait_cycles, int stall);

/* Number of CUDA kernels this library has launched in this process (all
 * entry points, all devices).  A monotone counter for instrumentation. */
uint64_t palu_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* PALU_H_ */
