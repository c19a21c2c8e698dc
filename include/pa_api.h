/*
 * pa_api.h -- C ABI of the B200 (sm_100a) paged-attention decode library
 * (libpagedattn.so).
 *
 * Three operations make up one decode step of one attention layer:
 *
 *   pa_append_kv    store each new token's K and V in its cache slot;
 *   pa_decode       one query token per sequence attends to that sequence's
 *                   whole cached history, gathered through its block table;
 *   pa_copy_blocks  duplicate whole blocks (copy-on-write at a fork).
 *
 * Variants: pa_append_decode (append fused into the decode launch),
 * pa_decode_sliding_window, pa_decode_shared_prefix (a shared prefix attended
 * once for the whole batch), pa_copy_blocks_layers (every layer's caches in
 * one call), pa_decode_static_workspace (no caller workspace), and
 * pa_decode_partial + pa_merge_partials (a sequence's history split across
 * calls or GPUs, merged after an exchange of the partial results).
 *
 * Sources of the definitions (page titles and sections):
 *  - "AI 陪读顶会论文（三）：KV Cache 显存占用计算与 PagedAttention 原理拆解",
 *    section "为什么自回归解码必须使用 KV Cache？": the attention equation
 *    o = softmax(q_t K_{1:t}^T / sqrt(d)) V_{1:t}, and the rule that each
 *    step computes only the new token's k_t, v_t and appends them;
 *    section "PagedAttention 的破局哲学": fixed-size blocks (16 tokens by
 *    default) in arbitrary physical places, a block table per sequence,
 *    copy-on-write for branches that share prompt blocks.
 *  - KV cache article (ainews.alishangtian.com), section
 *    "PagedAttention：把操作系统的老智慧搬进推理引擎": block table, shared
 *    prefix blocks stored once and reference-counted, copy-on-write at the
 *    fork point; section "显存账本：长上下文时代，KV cache 反超权重": grouped-
 *    query attention (several query heads share one KV head); section
 *    "再往后：压 KV 的三条路线": FP8 K/V with per-channel scaling factors.
 *
 * Conventions shared by every entry point
 *  - Every tensor argument is a DEVICE pointer to caller-owned memory (for
 *    example a torch tensor's data_ptr()), dense and row-major in the layout
 *    stated, and 16-byte aligned. The library allocates no device memory;
 *    pa_decode's split-K workspace is supplied by the caller.
 *  - KV cache layout: [num_blocks][block_size][num_kv_heads][head_dim]. The
 *    token at logical position j of sequence b lives in physical block
 *    block_tables[b * max_blocks_per_seq + j / block_size], row
 *    j % block_size; slot s names block s / block_size, row s % block_size.
 *  - Query head i reads KV head i / (num_q_heads / num_kv_heads).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream); every
 *    call is asynchronous on it and returns after enqueueing its kernels.
 *  - Arguments are checked on the host before anything is enqueued; a
 *    failed check returns PA_ERR_INVALID_ARG or PA_ERR_UNSUPPORTED and leaves
 *    all memory untouched. Values that live in device memory (slots, block
 *    ids, context lengths) are checked by the kernels: an out-of-range value
 *    sets a bit in a per-device error word and the access it would have made
 *    is skipped (reads yield zeros, writes are dropped); pa_get_device_error
 *    reports and clears that word.
 *  - Supported: block_size a power of two in [1, 256]; head_dim 64 or 128;
 *    16-bit caches (PA_F16, PA_BF16) whose dtype equals the input's, or an
 *    E4M3 cache with fp16 or bf16 inputs; num_q_heads a multiple of
 *    num_kv_heads.
 */
#ifndef PA_API_H
#define PA_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* a host-side argument check failed */
  PA_ERR_UNSUPPORTED = 2,   /* valid, but a dtype/shape the library has no kernel for */
  PA_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
  PA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
  PA_ERR_DEVICE_BOUNDS = 5  /* pa_get_device_error: a kernel saw an out-of-range value */
} pa_status;

typedef enum pa_dtype { PA_F16 = 0, PA_BF16 = 1, PA_E4M3 = 2 } pa_dtype;

/* Bits of the device error word (pa_get_device_error). */
#define PA_DEVERR_BLOCK_ID 0x1u    /* a block-table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 0x2u /* context_len < 0, > max_context, or beyond the table */
#define PA_DEVERR_SLOT 0x4u        /* append slot >= num_blocks * block_size, or (fused
                                      append) not the slot of position context_len - 1 */
#define PA_DEVERR_PREFIX 0x8u      /* pa_decode_shared_prefix: a sequence does not start
                                      with the shared prefix blocks, or is shorter */
#define PA_DEVERR_TIMEOUT 0x10u    /* a kernel's bounded wait for its own tensor-core
                                      work gave up (1 s); its results are not written */

/* Describes one paged KV cache (one layer's K cache and V cache). */
typedef struct pa_cache_desc {
  int64_t num_blocks;    /* physical blocks in each of the K and V caches */
  int32_t block_size;    /* tokens per block: power of two in [1, 256] */
  int32_t num_kv_heads;
  int32_t head_dim;      /* 64 or 128 */
  int32_t cache_dtype;   /* pa_dtype */
  /* E4M3 caches only (NULL otherwise): device fp32 arrays [num_kv_heads *
   * head_dim], 16-byte aligned (checked). A stored code c of head h, channel d stands for
   * e4m3(c) * scale[h*head_dim + d]; append stores
   * e4m3_rn_satfinite(fp32(x) * inv_scale[h*head_dim + d]). */
  const float* k_scale;
  const float* v_scale;
  const float* k_inv_scale;
  const float* v_inv_scale;
} pa_cache_desc;

/* Store new tokens' K and V into their cache slots.
 *   k, v          [num_tokens][num_kv_heads][head_dim] in in_dtype (PA_F16
 *                 or PA_BF16).
 *   slot_mapping  [num_tokens] int64; slot < 0 skips the token (padding).
 *   k_cache, v_cache  caches described by `cache`; a 16-bit cache receives
 *                 the input bits unchanged (its dtype must equal in_dtype);
 *                 an E4M3 cache receives the quantised codes.
 * Slots of one call must be distinct (two tokens written to one slot race).
 * num_tokens == 0 is a no-op. */
pa_status pa_append_kv(const void* k, const void* v, int32_t in_dtype, int64_t num_tokens,
                       const int64_t* slot_mapping, void* k_cache, void* v_cache,
                       const pa_cache_desc* cache, void* stream);

/* Bytes of workspace pa_decode needs for these sizes and this partition
 * choice (0 when one partition covers max_context). Pure host function.
 * The workspace holds the split-K partials (head_dim + 2 floats per query
 * head and partition) and the call's work list (one 8-byte entry per
 * partition a sequence can have, plus 256 bytes): a split decode of more than
 * one sequence first lists its (sequence, partition) items, longest first,
 * in one small kernel, then runs them on as many decode CTAs as the GPU holds
 * at once. Nothing in the workspace needs a starting value.
 * Sizes whose workspace would pass 2^60 bytes are refused: this returns 0
 * and every decode entry point returns PA_ERR_UNSUPPORTED for them (the same
 * rule holds for the sliding-window and shared-prefix sizes below). */
size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t max_context,
                                int32_t partition_tokens, const pa_cache_desc* cache);

/* Tokens per split-K partition that pa_decode uses for these sizes when
 * called with partition_tokens == 0. Pure host function. */
int32_t pa_decode_partition_tokens(int32_t batch, int32_t max_context,
                                   const pa_cache_desc* cache);

/* Single-query paged attention for a batch of sequences:
 *   out[b][i][:] = softmax_j(scale * q[b][i] . K_j) V_j over the
 *   context_lens[b] cached tokens of sequence b, KV head i / group.
 *   q             [batch][num_q_heads][head_dim], q_dtype PA_F16 or PA_BF16
 *                 (for a 16-bit cache q_dtype must equal the cache dtype).
 *   block_tables  [batch][max_blocks_per_seq] int32 physical block ids;
 *                 entries past ceil(context_lens[b] / block_size) are not read.
 *   context_lens  [batch] int32, each in [0, max_context]; 0 gives a zero row.
 *   max_context   host-side upper bound of context_lens (sizes the launch).
 *   scale         multiplies q.K before the softmax (1/sqrt(head_dim)).
 *   out           [batch][num_q_heads][head_dim] in q_dtype.
 *   partition_tokens  0 lets the library split long contexts; otherwise a
 *                 multiple of 16 in [16, 1 << 20] fixes the split-K partition
 *                 length (results agree up to rounding for any choice).
 *   workspace     device scratch of at least pa_decode_workspace_size(...)
 *                 bytes (may be NULL when that size is 0), 256-byte aligned.
 * Blocks may be shared between sequences (shared prefixes, beams); the
 * caches are only read. */
pa_status pa_decode(const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads,
                    const void* k_cache, const void* v_cache, const pa_cache_desc* cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t max_context, float scale, void* out,
                    int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                    void* stream);

/* pa_append_kv followed by pa_decode in one launch, for a batch with one new
 * token per sequence ("AI 陪读顶会论文（三）：...", section "为什么自回归解码必须
 * 使用 KV Cache？": each step computes the new token's k_t, v_t, appends them and
 * attends over the whole cache). The new token of sequence b is the token at
 * position context_lens[b] - 1: the decode reads its K/V from k / v directly
 * (quantised exactly as pa_append_kv would for an E4M3 cache) and the CTA of
 * the sequence's last partition stores it at slot_mapping[b]. Caches and
 * output equal those of the two separate calls.
 *   q             [batch][num_q_heads][head_dim] in dtype.
 *   k, v          [batch][num_kv_heads][head_dim] in dtype (PA_F16 / PA_BF16;
 *                 for a 16-bit cache, the cache dtype).
 *   slot_mapping  [batch] int64; slot_mapping[b] must be the slot of position
 *                 context_lens[b] - 1 in sequence b's table (else the device
 *                 error word gets PA_DEVERR_SLOT, nothing is stored and that
 *                 sequence's result is not meaningful); < 0: no new token for
 *                 b (plain decode). The slot must not lie in another
 *                 sequence's context in this batch (copy-on-write has run).
 *   k_cache, v_cache  written at the new slots (the same as pa_decode's
 *                 caches otherwise).
 * Other arguments as for pa_decode (same workspace size). */
pa_status pa_append_decode(const void* q, const void* k, const void* v, int32_t dtype,
                           int32_t batch, int32_t num_q_heads, const int64_t* slot_mapping,
                           void* k_cache, void* v_cache, const pa_cache_desc* cache,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, int32_t max_context, float scale,
                           void* out, int32_t partition_tokens, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Workspace bytes for pa_decode_sliding_window. Pure host function. */
size_t pa_decode_sliding_window_workspace_size(int32_t batch, int32_t num_q_heads,
                                               int32_t max_context, int32_t window,
                                               int32_t partition_tokens,
                                               const pa_cache_desc* cache);

/* pa_decode with sliding-window attention (KV cache article, section
 * "再往后：压 KV 的三条路线": each token attends only to the most recent window
 * of tokens, so the cache a sequence needs is bounded by the window): the
 * query of sequence b attends to its tokens [max(0, L - window), L), L =
 * context_lens[b], the new token included.
 *   window  >= 1 tokens.
 * Table entries for blocks that hold only tokens before the window are never
 * read, so a caller may have freed those blocks (their entries may hold any
 * value). Other arguments as for pa_decode; the workspace comes from
 * pa_decode_sliding_window_workspace_size. */
pa_status pa_decode_sliding_window(const void* q, int32_t q_dtype, int32_t batch,
                                   int32_t num_q_heads, const void* k_cache, const void* v_cache,
                                   const pa_cache_desc* cache, const int32_t* block_tables,
                                   int32_t max_blocks_per_seq, const int32_t* context_lens,
                                   int32_t max_context, int32_t window, float scale, void* out,
                                   int32_t partition_tokens, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Tokens per suffix partition that pa_decode_shared_prefix uses for these
 * sizes when called with partition_tokens == 0 (for 16-bit caches up to
 * four times pa_decode's choice while that still gives two CTAs per SM:
 * every row already merges the prefix partials). 0 for invalid sizes. Pure
 * host function. */
int32_t pa_decode_shared_prefix_partition_tokens(int32_t batch, int32_t num_q_heads,
                                                 int32_t max_context, int32_t prefix_blocks,
                                                 const pa_cache_desc* cache);

/* Workspace bytes for pa_decode_shared_prefix (equals
 * pa_decode_workspace_size when prefix_blocks == 0). Pure host function. */
size_t pa_decode_shared_prefix_workspace_size(int32_t batch, int32_t num_q_heads,
                                              int32_t max_context, int32_t prefix_blocks,
                                              int32_t partition_tokens,
                                              const pa_cache_desc* cache);

/* pa_decode for a batch whose sequences all begin with the same physical
 * blocks -- a shared system prompt stored once and referenced by every
 * sequence (KV cache article, section "PagedAttention：把操作系统的老智慧搬进
 * 推理引擎": prefix sharing).
 * Precondition: block_tables[b][0 .. prefix_blocks) are the same for every b,
 * and every context_lens[b] >= prefix_blocks * block_size. Then the result
 * equals pa_decode's (up to rounding): the attention over the shared prefix
 * is computed once per KV head for all batch x group query columns (a dense
 * tensor-core contraction that reads each prefix block a few times instead
 * of once per sequence), each sequence's own tokens after the prefix are
 * handled as in pa_decode, and the two are merged as split-K partials.
 * A sequence whose table or length breaks the precondition sets
 * PA_DEVERR_PREFIX (its output is then not meaningful).
 * 16-bit caches with blocks of at least 8 tokens, at most 128 query heads
 * per KV head and fewer than 2^31 slots: the prefix part runs on tcgen05
 * tensor cores. The call enqueues three kernels on `stream`: the prefix
 * kernel, the suffix decode launched as its programmatic dependent (it runs
 * beside the prefix kernel and completes only after it), and the split-K
 * merge as the suffix decode's dependent. Work enqueued on `stream` after
 * the call therefore sees the complete result, and the call can be captured
 * into a CUDA graph from `stream`. A tensor-core wait that gives up (1 s)
 * sets PA_DEVERR_TIMEOUT. Other caches (E4M3, smaller blocks, larger groups)
 * run the prefix on mma.sync in the same launch as the suffixes.
 *   prefix_blocks  number of shared leading blocks (0: plain pa_decode);
 *                  prefix_blocks * block_size must not exceed max_context.
 *   workspace      at least pa_decode_shared_prefix_workspace_size(...) bytes,
 *                  256-byte aligned; always needed when prefix_blocks > 0.
 * Other arguments as for pa_decode; partition_tokens applies to the suffixes. */
pa_status pa_decode_shared_prefix(const void* q, int32_t q_dtype, int32_t batch,
                                  int32_t num_q_heads, const void* k_cache, const void* v_cache,
                                  const pa_cache_desc* cache, const int32_t* block_tables,
                                  int32_t max_blocks_per_seq, const int32_t* context_lens,
                                  int32_t max_context, int32_t prefix_blocks, float scale,
                                  void* out, int32_t partition_tokens, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Copy whole blocks: for p in [0, num_pairs), K block pairs_host[2p] ->
 * K block pairs_host[2p+1], and the same for V.
 *   pairs_host    HOST array of num_pairs (src, dst) int32 pairs, read before
 *                 the call returns (passed to the kernel by value).
 * Every id must be in [0, num_blocks), destinations distinct, and no
 * destination may also be a source (then the order of copies cannot
 * matter); otherwise PA_ERR_INVALID_ARG. num_pairs == 0 is a no-op. */
pa_status pa_copy_blocks(const int32_t* pairs_host, int32_t num_pairs, void* k_cache,
                         void* v_cache, const pa_cache_desc* cache, void* stream);

/* pa_copy_blocks applied to every layer of a model in one call (one launch
 * per 32 layers and 256 pairs). Copy-on-write is decided per sequence, not
 * per layer, so a step's block copies are the same for all layers and can
 * run before any layer does; a layer's append and decode cannot be batched
 * this way, since they need that layer's input.
 *   k_caches, v_caches  HOST arrays of num_layers DEVICE pointers, one K and
 *                 one V cache per layer, all described by `cache`; every
 *                 pointer non-null and 16-byte aligned.
 * Pair rules as for pa_copy_blocks; num_pairs == 0 or num_layers == 0 is a
 * no-op. */
pa_status pa_copy_blocks_layers(const int32_t* pairs_host, int32_t num_pairs,
                                void* const* k_caches, void* const* v_caches, int32_t num_layers,
                                const pa_cache_desc* cache, void* stream);

/* Test hook for the failure path of pa_decode_shared_prefix's tensor-core
 * prefix kernel (16-bit caches). While on (process-wide), that kernel's MMA
 * warp issues nothing: its softmax warps' waits run out after their 1 s
 * limit, every role of the CTA drains, no partial is written and the device
 * error word gets PA_DEVERR_TIMEOUT; the context stays usable. Off by
 * default; not for production calls. */
void pa_testing_withhold_prefix_scores(int32_t on);

/* Test hook for the failure path of a steal-mode decode that merges its rows
 * inside the launch (see pa_set_deterministic: a single long sequence whose
 * CTAs all fit on the GPU at once). While on (process-wide), the first CTA
 * of each row does not count its partial, so every CTA's wait for the row
 * runs out after its 1 s limit: no row is merged, the output is left as it
 * was, the device error word gets PA_DEVERR_TIMEOUT and the context stays
 * usable. Off by default; not for production calls. */
void pa_testing_withhold_steal_counts(int32_t on);

/* Synchronise `stream`, then read and clear the current device's error
 * word into *flags (PA_DEVERR_* bits). Returns PA_ERR_DEVICE_BOUNDS when
 * any bit was set, PA_OK when none, PA_ERR_CUDA on a runtime failure.
 * The word is one per device, shared by every stream: only `stream` is
 * synchronised, so a bit set by a kernel on another stream is reported by
 * whichever call reads the word next (and a kernel on another stream still
 * running may set one after the read). To attribute errors to calls, read
 * the word with no other stream of the library's calls in flight. */
pa_status pa_get_device_error(void* stream, uint32_t* flags);

/* pa_decode without a caller-supplied workspace and without allocating any.
 * (The pages have no counterpart: this is an integration convenience.)
 *
 * For callers that cannot call cudaMalloc or take memory from an allocator
 * on this path -- for example a plug-in inside an engine that owns all device
 * memory through its own pool, or code on a latency-critical path where an
 * allocation's implicit synchronisation is not acceptable. The split-K
 * workspace is a fixed 32 MiB array in the library's own device memory
 * (reserved on every GPU that loads the library, until the process exits),
 * so the call allocates nothing; inputs and outputs are still the caller's.
 * Arguments and results are those of pa_decode (same partition choice, same
 * argument checks and status codes, bitwise the same output), minus the
 * workspace. If a valid call's plan needs more than 32 MiB of workspace
 * (pa_decode_workspace_size(...) > 32 MiB) the call returns
 * PA_ERR_WORKSPACE and enqueues nothing; use pa_decode with a larger buffer
 * or a longer partition.
 * The array's device address belongs to a CUDA context: the first call in
 * each context (a device's primary context, or a context the caller made
 * current, or one created after a device reset) looks it up with
 * cudaGetSymbolAddress while that context is current; make that first call
 * before any stream capture. Every call on a device shares the one array,
 * which keeps the previous call's contents (nothing in it needs a starting
 * value); calls whose kernels overlap on the GPU -- concurrent streams, or
 * several host threads -- race on it and must be serialised by the caller. */
pa_status pa_decode_static_workspace(const void* q, int32_t q_dtype, int32_t batch,
                                     int32_t num_q_heads, const void* k_cache,
                                     const void* v_cache, const pa_cache_desc* cache,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, int32_t max_context,
                                     float scale, void* out, int32_t partition_tokens,
                                     void* stream);

/* Context parallelism, part 1: pa_decode over the tokens each sequence's
 * table lists, stopping short of the final normalisation across calls, so
 * that several calls over disjoint parts of every sequence's history (for
 * example the block-aligned context slices that several GPUs hold) can be
 * merged by pa_merge_partials into exactly what one pa_decode over the whole
 * history gives, up to rounding. It is the decode's own split-K merge
 * (softmax of the scores over partitions) carried across calls; the pages
 * have no counterpart beyond that merge.
 *   part_o   [batch][num_q_heads][head_dim] fp32: each row's attention
 *            output over this call's tokens (normalised as pa_decode's);
 *            16-byte aligned.
 *   part_ml  [batch][num_q_heads][2] fp32: each row's (m, l) over the
 *            same tokens, with s_j = scale * q.k_j * log2(e), m a reference
 *            value at or below max_j s_j and within 8 of it (the decode moves
 *            its running maximum only by steps of at least 8), and
 *            l = sum_j 2^(s_j - m): the pair encodes the softmax
 *            denominator, m + log2(l) = log2(sum_j 2^(s_j)). A row with no
 *            tokens (context_lens[b] == 0) gives output 0, m = -inf, l = 0.
 *            16-byte aligned.
 * Other arguments, checks, statuses and the workspace (the
 * pa_decode_workspace_size formula) as for pa_decode; `out` is not used.
 * The call keeps the plain grid of partitions (no work list, no steal mode)
 * and is reproducible. */
pa_status pa_decode_partial(const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads,
                            const void* k_cache, const void* v_cache, const pa_cache_desc* cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* context_lens, int32_t max_context, float scale,
                            float* part_o, float* part_ml, int32_t partition_tokens,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Context parallelism, part 2: merge num_parts results of pa_decode_partial
 * stacked part-major, part_o [num_parts][rows][head_dim] and part_ml
 * [num_parts][rows][2] (rows = batch * num_q_heads; the layout an all-gather
 * of each GPU's part_o / part_ml produces), into out [rows][head_dim] in
 * out_dtype (PA_F16 or PA_BF16): out = sum_n w_n o_n / sum_n w_n with
 * w_n = l_n * 2^(m_n - max over the parts of m). Parts with l = 0 weigh
 * nothing; a row whose parts all have l = 0 gives 0. head_dim 64 or 128;
 * every pointer 16-byte aligned device memory. Returns PA_ERR_INVALID_ARG /
 * PA_ERR_UNSUPPORTED on bad sizes or pointers (nothing enqueued). */
pa_status pa_merge_partials(const float* part_o, const float* part_ml, int32_t num_parts,
                            int64_t rows, int32_t head_dim, void* out, int32_t out_dtype,
                            void* stream);

/* Reproducible results (process-wide, any thread; 0 at load). With 0, a
 * pa_decode, pa_decode_static_workspace or pa_decode_sliding_window call on
 * one sequence (batch == 1) over a 16-bit cache with blocks of 16 tokens or
 * more, whose plan splits it into partitions of 1024 tokens or more, runs in
 * steal mode: the CTAs of each KV head group take the sequence's tiles in
 * chunks from a counter in the workspace instead of each reading a fixed
 * partition, so that no CTA on a slower SM holds up the call. Which CTA
 * combines which tiles then varies from call to call, and so may the last
 * bits of the output (every result is within the same rounding of the
 * split-K merge). With 1, no call uses steal mode, and a call repeated with
 * the same inputs, sizes and partition length gives the same bits; every
 * other decode is reproducible in either setting. The switch is read when a
 * call is made (a captured launch keeps its mode). Returns the previous
 * setting. */
int32_t pa_set_deterministic(int32_t on);

/* Static text for a status code. */
const char* pa_status_string(int32_t status);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_API_H */
