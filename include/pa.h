/*
 * libpa -- paged KV-cache decode attention for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every pointer argument is DEVICE memory owned by the caller unless the
 * comment says otherwise; the library allocates nothing on these paths.  Device
 * pointers are not queried on the launch paths (only pa_swap_blocks, which accepts
 * host pools, asks the runtime what each pool is): a host pointer, or memory of
 * another device than the current one, where device memory is required is
 * undefined behaviour.  The Python binding checks device, dtype, contiguity and
 * shapes of its tensors before it calls in.  Every call is asynchronous on
 * `stream` (a cudaStream_t passed as void*, NULL = the legacy default stream) and
 * never synchronises the device, except pa_get_device_error, which says so.  The
 * launch entry points may be called from several host threads at once: they keep no
 * host state besides a once-initialised driver entry point and per-device caches, and
 * on the device they share only the sticky error word (and the scratch array of
 * pa_decode_static_scratch, which says so).
 *
 * Data layout (both caches, the same for every call):
 *   k_cache, v_cache : [num_blocks][num_kv_heads][block_size][head_dim], 16-bit
 *                      elements (pa_dtype); one (block, kv head) is one contiguous run.
 *   block_tables     : int32 [num_seqs][max_blocks_per_seq]; entry j of row s is the
 *                      physical block that holds logical tokens [j*bs, (j+1)*bs) of
 *                      sequence s.  Entries at or past ceil(context_lens[s] / bs) never
 *                      select a page: the decode kernels may load them (a
 *                      partition's whole table range is fetched before its length
 *                      is known) but never use their values, so they may hold any
 *                      value, -1 and out-of-range ids included.  Every load stays
 *                      inside row s (max_blocks_per_seq entries).
 *   slot             : block * block_size + offset inside the block.
 *
 * Errors.  A problem the host can see (null or misaligned pointer, unsupported
 * shape, too small a workspace) returns a status before anything is launched.  A
 * problem in device data (a block id or slot outside the pool, a context longer
 * than its table or than the partition grid, a bounded wait that expired) sets a
 * bit in a sticky per-device error word (PA_DEVERR_*) and the offending item is
 * skipped; its output is then unspecified.  No call traps, aborts or throws.
 *
 * Source of each operation: the vLLM paged-attention pages -- "IO-5 vLLM Paged
 * Attention" note (sections 2-4: page table, K = concat of pages, attention
 * unchanged) and the "PagedAttention and dynamic memory management" blog (KV of
 * every generated token is stored in the cache; pages are shared between requests).
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, workspace too small */
    PA_ERR_UNSUPPORTED = 2, /* head_dim, block size or group size not built, or a size
                               past a launch limit the entry point states (split the call) */
    PA_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch, attribute, ...) */
    PA_ERR_OUT_OF_RANGE = 4,
    PA_ERR_TIMEOUT = 5,
    PA_ERR_NO_FREE_BLOCK = 6, /* host block manager: the pool cannot satisfy the request */
    PA_ERR_HOST_ALLOC = 7     /* host block manager: a host allocation failed; nothing changed */
} pa_status;

typedef enum { PA_FP16 = 0, PA_BF16 = 1 } pa_dtype;

/* Bits of the sticky per-device error word. */
#define PA_DEVERR_BLOCK_ID 0x1u /* a block table entry outside [0, num_blocks) */
#define PA_DEVERR_SLOT 0x2u     /* a slot >= num_blocks * block_size */
#define PA_DEVERR_PAIR 0x4u     /* a copy pair id outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT 0x8u  /* context longer than its table or the partition grid */
#define PA_DEVERR_TIMEOUT 0x10u /* a bounded wait on a copy expired */
#define PA_DEVERR_WORKSPACE 0x20u /* dynamic split: the workspace's counters were not zero */

/*
 * Cache write ("PagedAttention and dynamic memory management" blog, first section:
 * each generated token's K and V are stored in the KV cache; in a paged cache the
 * store goes to the token's slot).
 *
 * For each token t < num_tokens with slot = slot_mapping[t] >= 0 and every kv head h:
 *   k_cache[slot / block_size][h][slot % block_size][:] = key[t*key_token_stride + h*head_dim + :]
 *   v_cache[...] likewise from value.   A negative slot is skipped.
 * key, value      : [num_tokens][...] rows of num_kv_heads*head_dim elements, heads
 *                   contiguous; token strides in ELEMENTS (multiple of 8).
 * slot_mapping    : int64 [num_tokens].
 * Alignment       : key, value, k_cache, v_cache 16-byte aligned.
 * Duplicate slots within one call give an unspecified winner.
 * Bit-exact copy of the 16-bit patterns.  head_dim multiple of 8, block_size >= 1.
 * One call moves at most 2^31 - 1 16-byte chunks (num_tokens * num_kv_heads *
 * head_dim / 8); larger calls return PA_ERR_UNSUPPORTED (split them).
 */
pa_status pa_kv_write(const void *key, const void *value, const int64_t *slot_mapping,
                      int num_tokens, int num_kv_heads, int head_dim, int64_t key_token_stride,
                      int64_t value_token_stride, void *k_cache, void *v_cache, int num_blocks,
                      int block_size, pa_dtype dtype, void *stream);

/*
 * Block copy for copy-on-write of shared blocks (the pages let several requests
 * share KV blocks -- "PagedAttention" summary, features 2; a sequence that appends
 * into a shared, partially filled block first needs a private copy).
 *
 * For each pair p < num_pairs: block pairs[2p+1] := block pairs[2p] in both caches
 * (all kv heads, all block_size slots).  src_dst_pairs: int64 [num_pairs][2], device.
 * Destinations must be distinct and no destination may be a source of the same call.
 * Bit-exact.  Caches 16-byte aligned; num_kv_heads*block_size*head_dim multiple of 8.
 * A pair id outside [0, num_blocks) sets PA_DEVERR_PAIR and that pair is skipped.
 * At most 65535 pairs per call, and a block of at most 65535 x 2048 16-byte chunks;
 * larger calls return PA_ERR_UNSUPPORTED (split them).
 */
pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *src_dst_pairs,
                         int num_pairs, int num_kv_heads, int block_size, int head_dim,
                         int num_blocks, pa_dtype dtype, void *stream);

/*
 * Block swap between two pools -- the GPU cache and a host pool in pinned memory --
 * for preemption ("PagedAttention" summary, section 5 and conclusion: block-level
 * memory management with preemptive request scheduling; "PagedAttention and dynamic
 * memory management" blog, BlockSpaceManager(num_cpu_blocks=...)): a preempted
 * sequence's blocks are copied out to host blocks and later back in.
 *
 * For each pair p < num_pairs: dst block pairs[2p+1] := src block pairs[2p] in both
 * caches (all kv heads and slots).  src/dst caches have the cache layout with
 * src_num_blocks / dst_num_blocks blocks; each may be device memory or pinned host
 * memory mapped for the device (cudaHostAlloc / cudaHostRegister, reached through
 * unified addressing).  src_dst_pairs: int64 [num_pairs][2] in device memory (or
 * mapped pinned memory).  Destination blocks must be distinct and the two pools must
 * not overlap.  One launch; bit-exact.  A pair id outside its pool sets
 * PA_DEVERR_PAIR and that pair is skipped.  Pointers 16-byte aligned.  Every pointer
 * is checked with the runtime before the launch: pageable host memory returns
 * PA_ERR_INVALID_ARG.  A block of at most 65535 x 2048 16-byte chunks (else
 * PA_ERR_UNSUPPORTED).
 */
pa_status pa_swap_blocks(void *dst_k_cache, void *dst_v_cache, const void *src_k_cache,
                         const void *src_v_cache, const int64_t *src_dst_pairs, int num_pairs,
                         int num_kv_heads, int block_size, int head_dim, int src_num_blocks,
                         int dst_num_blocks, pa_dtype dtype, void *stream);

/*
 * Decode attention over the paged cache ("IO-5 vLLM Paged Attention" note, section 4:
 * Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V with K, V loaded page by page,
 * K = concat(K_page_a, K_page_b, ...) in table order; section 3: Sequence -> [page
 * indices]).  For every sequence s and query head h, with G = num_q_heads /
 * num_kv_heads and g = h / G:
 *   out[s][h][:] = sum_{t < L} softmax_t(scale * <q[s][h], K_s[t]>) V_s[t]
 *   K_s[t] = k_cache[block_tables[s][t / bs]][g][t % bs][:],   L = context_lens[s].
 * L == 0 gives zeros.  Math in fp32 (online softmax), output rounded to nearest even.
 *
 * q, out          : [num_seqs][num_q_heads][head_dim], contiguous, 16-byte aligned.
 * context_lens    : int32 [num_seqs].
 * head_dim        : 64 or 128.  block_size: power of two in [8, 512].
 * G               : 1, 2, 4 or 8.
 * max_context_len : host-side upper bound of context_lens (0 = unknown: the table
 *                   width max_blocks_per_seq * block_size is used).  A context longer
 *                   than the bound sets PA_DEVERR_CONTEXT.
 * sliding_window  : 0 = attend to the whole context.  W > 0 = attend to the last W
 *                   tokens only, t in [max(0, L - W), L) (the block manager's
 *                   sliding_window setting, "PagedAttention and dynamic memory
 *                   management" blog, BlockSpaceManager example).  Table entries of
 *                   pages wholly before that range are never read, so their blocks
 *                   may have been returned to the pool (entry -1).  Negative:
 *                   PA_ERR_INVALID_ARG.
 * partition_size  : how contexts are split (split-K); partial results of the pieces
 *                   of one context -- fp32 running max, sum and normalised output --
 *                   are merged by log-sum-exp in a second kernel.
 *                     > 0 (a multiple of 64): fixed partitions of that many tokens, one
 *                         CTA each (a context of at most one partition is done in a
 *                         single pass and needs no merge);
 *                     PA_PARTITION_BALANCED (-1): balanced split -- persistent warps each
 *                         take an equal share of all (sequence, kv head, 16-token tile)
 *                         work, cutting contexts wherever the shares end (needs
 *                         num_seqs <= 16383 for head_dim 128, 8191 for 64; otherwise
 *                         fixed partitions are used);
 *                     PA_PARTITION_DYNAMIC (-2): dynamic split for a few long contexts
 *                         -- persistent CTAs (3 per SM), each (sequence, kv head) unit
 *                         served by CTAs in proportion to its length, whose warps claim
 *                         32-token chunks of it from a counter while they run, so warps
 *                         on faster SMs take more.  Needs num_seqs * num_kv_heads <=
 *                         min(3 * SMs, 1024) (otherwise the library's fixed split is
 *                         used) and the workspace rule below.  The split of each sum
 *                         varies between calls, so results may differ in the last bits
 *                         from call to call;
 *                     0: the library chooses (a fixed split: the same inputs always
 *                         give the same bits).
 * workspace       : fp32 scratch for those partial results, at least
 *                   pa_decode_workspace_bytes(...) bytes, 256-byte aligned; may be
 *                   NULL when no context needs more than one partition.  Its contents
 *                   are overwritten, except that with PA_PARTITION_DYNAMIC its first
 *                   PA_WORKSPACE_ZERO_BYTES bytes hold counters: they must be
 *                   zero before the workspace's first such call (one cudaMemset after
 *                   allocating it), and every call leaves them zero (a call that finds
 *                   them otherwise sets PA_DEVERR_WORKSPACE).  No split writes those
 *                   bytes otherwise, so one workspace can serve calls with different
 *                   splits, and no other split needs any initialisation.  Calls that
 *                   share a workspace must not overlap on the GPU.
 * Launches 1 kernel (one partition per sequence) or 2 (partition pass + merge).
 */
pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, int max_blocks_per_seq, float scale, int max_context_len,
                    int sliding_window, int partition_size, void *workspace,
                    size_t workspace_bytes, pa_dtype dtype, void *stream);

#define PA_PARTITION_BALANCED (-1)
#define PA_PARTITION_DYNAMIC (-2)
#define PA_WORKSPACE_ZERO_BYTES 8192

/*
 * One decode step with its cache write fused in: the cache write of each sequence's
 * new token followed by pa_decode, in one launch (plus the merge when contexts are
 * split).  For every sequence s with L = context_lens[s] > 0 and every kv head h:
 *   k_cache[block_tables[s][(L-1) / bs]][h][(L-1) % bs][:] = key[s*key_token_stride + h*head_dim + :]
 *   v_cache[...] likewise from value,
 * then the attention of pa_decode over [0, L) (or the last sliding_window tokens of
 * it) -- which therefore includes the new token.
 * The write is done by the CTA (the warp, under PA_PARTITION_DYNAMIC) that reads the
 * last tile of (s, h), before it reads that position, so the result equals pa_kv_write
 * (with slot = the slot of position L-1) followed by pa_decode -- bit for bit under a
 * fixed split.
 * key, value : [num_seqs][...] rows, heads contiguous, token strides in elements
 *              (multiples of 8), 16-byte aligned.
 * Sequences must not share the block that holds their position L-1 (copy a shared
 * block first with pa_copy_blocks).  partition_size as pa_decode; the balanced split
 * (PA_PARTITION_BALANCED) is not supported here (PA_ERR_UNSUPPORTED).  Other
 * arguments, errors and the workspace as pa_decode.
 */
pa_status pa_decode_append(void *out, const void *q, const void *key, const void *value,
                           int64_t key_token_stride, int64_t value_token_stride, void *k_cache,
                           void *v_cache, const int32_t *block_tables,
                           const int32_t *context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           int max_blocks_per_seq, float scale, int max_context_len,
                           int sliding_window, int partition_size, void *workspace,
                           size_t workspace_bytes, pa_dtype dtype, void *stream);

/*
 * pa_decode (with key and value: pa_decode_append) for a caller that also holds the
 * context lengths on the host, as a serving engine's scheduler does.  The launch is
 * planned from them: only the (sequence, partition) units that exist are launched --
 * under the fixed split a context of L tokens has ceil(L / partition) of them, where the
 * full grid holds the longest context's count for every sequence.  When that leaves out
 * at least 30% of the grid's rows they are taken longest first (every full partition,
 * then the shorter last partitions by decreasing length); otherwise in the full grid's
 * own order without its empty rows (partition 0 of every sequence, then each later
 * partition index longest first).  The results are bit-identical to pa_decode /
 * pa_decode_append.
 *
 * host_context_lens : int32 [num_seqs], host memory, read during the call only; it must
 *                     hold the values of context_lens.  A context whose device length
 *                     needs another partition count than the plan sets
 *                     PA_DEVERR_CONTEXT (a partition the plan left out is not computed).
 * key, value        : both NULL (no cache write) or both given, as pa_decode_append.
 * The plan applies to the fixed split without a sliding window, with at most
 * 4096 units and 255 partitions per context, when the full grid has an empty row; other
 * calls run as pa_decode / pa_decode_append.  Other arguments, errors and the workspace
 * as pa_decode.
 */
pa_status pa_decode_planned(void *out, const void *q, const void *key, const void *value,
                            int64_t key_token_stride, int64_t value_token_stride,
                            void *k_cache, void *v_cache, const int32_t *block_tables,
                            const int32_t *context_lens, const int32_t *host_context_lens,
                            int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                            int block_size, int num_blocks, int max_blocks_per_seq, float scale,
                            int max_context_len, int sliding_window, int partition_size,
                            void *workspace, size_t workspace_bytes, pa_dtype dtype,
                            void *stream);

/*
 * The launch pa_decode_planned would make for these arguments, host-side (no device
 * work; the SM count is read as pa_decode_workspace_bytes reads it): returns the number
 * of (sequence, partition) units it launches -- 0 when it launches the full grid -- and
 * writes the first min(that, max_units) of them to units in launch order, each
 * sequence << 16 | partition << 8 | the sequence's partition count.  -1 for invalid
 * arguments (those pa_decode rejects, a NULL host_context_lens with num_seqs > 0, or
 * units NULL with max_units > 0).
 */
int pa_decode_planned_units(const int32_t *host_context_lens, int num_seqs, int num_q_heads,
                            int num_kv_heads, int head_dim, int block_size,
                            int max_blocks_per_seq, int max_context_len, int sliding_window,
                            int partition_size, uint32_t *units, int max_units);

/*
 * One decode step with the copy-on-write of a shared block folded into the attention
 * pass (the pages let several requests share KV blocks -- "PagedAttention" summary,
 * features 2 -- so a sequence that appends into a shared, partially filled block
 * first needs a private copy of it).  Instead of a pa_copy_blocks launch before the
 * step, each sequence names the block it copies, and the rows are copied by the CTAs
 * that read them, just before they read them.
 *
 * cow : int32 [num_seqs][3] in device memory, 4-byte aligned.  For sequence s the
 *       triple (src, lb, rows): src < 0 means no copy; otherwise, for every kv head
 *       h and every r < rows,
 *         k_cache[block_tables[s][lb]][h][r][:] = k_cache[src][h][r][:]
 *       and likewise in v_cache, done before any of those rows is read.  Rows >= rows
 *       of the destination are left as they are: they hold this sequence's own tokens
 *       (written before the call, e.g. by pa_kv_write) or are unused.  With rows =
 *       block_size this is pa_copy_blocks of the pair (src, block_tables[s][lb]).
 *       Every row is copied whether or not the attention reads it (rows outside the
 *       context or before the sliding window too).  src outside [0, num_blocks), lb
 *       outside [0, max_blocks_per_seq) or rows outside [0, block_size] sets
 *       PA_DEVERR_PAIR, and an entry block_tables[s][lb] outside [0, num_blocks) sets
 *       PA_DEVERR_BLOCK_ID; that sequence's copy is skipped.  A destination must be
 *       private to its sequence, must not be the source of any copy of the call, and
 *       no other sequence of the call may read it; no row a copy reads may be one that
 *       the call's fused cache write stores.
 * key, value : both NULL (no cache write), or both given: the fused write of
 *       pa_decode_append, done after the copy (so a written row wins over a copied
 *       one).  Strides and alignment as pa_decode_append.
 * The result equals pa_copy_blocks of the rows, then (with key) pa_kv_write of the
 * new tokens, then pa_decode -- bit for bit.  partition_size as pa_decode, except
 * that a call that would take the balanced or the dynamic split returns
 * PA_ERR_UNSUPPORTED (the fixed split only).  Other arguments, errors and the
 * workspace as pa_decode.  Launches as pa_decode.
 */
pa_status pa_decode_cow(void *out, const void *q, const void *key, const void *value,
                        int64_t key_token_stride, int64_t value_token_stride, void *k_cache,
                        void *v_cache, const int32_t *block_tables, const int32_t *context_lens,
                        const int32_t *cow, int num_seqs, int num_q_heads, int num_kv_heads,
                        int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                        float scale, int max_context_len, int sliding_window,
                        int partition_size, void *workspace, size_t workspace_bytes,
                        pa_dtype dtype, void *stream);

/*
 * Bytes of workspace pa_decode needs for these sizes and this partition_size.
 * Host-side; it reads the current device's SM count (cudaDeviceGetAttribute, no
 * synchronisation; 148 when no device is visible), because the balanced and dynamic
 * splits keep partial records per resident warp or CTA.  Returns 0 when no merge is
 * needed.
 */
size_t pa_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int block_size, int max_blocks_per_seq, int max_context_len,
                                 int sliding_window, int partition_size);

/*
 * The partition size (tokens) pa_decode uses for these arguments when its
 * partition_size argument is `partition_size`: 0 means the balanced or the dynamic
 * split is used;
 * a value >= the longest context means one pass per sequence.  Host-side, as
 * pa_decode_workspace_bytes.
 */
int pa_decode_partition_tokens(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int max_blocks_per_seq, int max_context_len,
                               int sliding_window, int partition_size);

/*
 * pa_decode for callers that cannot allocate device memory.  The paged-attention
 * pages have no counterpart to this call; it exists for users of this library.
 *
 * Some callers have no way to hand pa_decode a workspace: an engine that gave all
 * free HBM to its KV-cache pool and offers its plugins no allocator, or a caller
 * that must not run cudaMalloc (and its device-wide synchronisation) inside its
 * decode loop.  This entry point takes the same arguments as pa_decode without the
 * workspace and keeps the split-K partial results in a scratch array that the
 * library itself holds in device memory: a fixed PA_STATIC_SCRATCH_BYTES per GPU,
 * reserved on every GPU that loads the library until the process exits.  Nothing
 * is allocated by the call.
 *
 *  - Sizes whose partial results need more than PA_STATIC_SCRATCH_BYTES (see
 *    pa_decode_workspace_bytes) are rejected with PA_ERR_INVALID_ARG before any
 *    launch; use pa_decode with a caller workspace for those.
 *  - The first call on a device looks up the array's device address on that device
 *    (cudaGetSymbolAddress, with the device current); make that first call before
 *    any stream capture.  Later calls reuse the address, which the library keeps
 *    for the life of the process: after cudaDeviceReset on a device the module
 *    may be loaded at another address, so this entry point must not be called on
 *    that device again in the same process (pa_decode with a workspace is not
 *    affected).
 *  - Every call on a device shares the one array, and it keeps the last call's
 *    contents.  Its partial results need no clearing (each call writes every one it
 *    reads); its first PA_WORKSPACE_ZERO_BYTES, the counters of PA_PARTITION_DYNAMIC,
 *    are zero when the library loads and every call leaves them zero.  Calls that
 *    overlap on the GPU race on the array: serialise them (one stream, or events
 *    between streams).
 */
#define PA_STATIC_SCRATCH_BYTES ((size_t)16 << 20) /* 16 MiB per GPU */

pa_status pa_decode_static_scratch(void *out, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *block_tables,
                                   const int32_t *context_lens, int num_seqs, int num_q_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int num_blocks, int max_blocks_per_seq, float scale,
                                   int max_context_len, int sliding_window,
                                   int partition_size, pa_dtype dtype, void *stream);

/*
 * Multi-query attention over the paged cache: prefill and chunked prefill ("IO-5 vLLM
 * Paged Attention" note, section 4, Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V
 * with a matrix Q: the new tokens of requests that continuous batching -- section 6 --
 * adds to the batch).  The tokens of sequence s are rows query_start_loc[s] ..
 * query_start_loc[s+1]-1 of q (n_s of them); their K and V are already in the cache
 * (pa_kv_write), which holds L_s = context_lens[s] >= n_s tokens of the sequence, so
 * token i of the chunk is at position p = L_s - n_s + i.  It attends causally:
 *   out[t][h][:] = sum_{u <= p} softmax_u(scale * <q[t][h], K_s[u]>) V_s[u],  g = h / G,
 * over u in [max(0, p - W + 1), p] under a sliding window W > 0 (the table must then
 * hold the pages from position L_s - n_s - W + 1 on; earlier entries are never read).
 * Causality is the reading taken where the pages are silent (autoregressive models).
 * A chunk of one token is a decode step; pa_decode is the faster call for those.
 *
 * q, out          : [num_tokens][num_q_heads][head_dim], contiguous, 16-byte aligned.
 * query_start_loc : int32 [num_seqs + 1], non-decreasing, [0] = 0, [num_seqs] = num_tokens.
 * scale           : > 0 (1/sqrt(d_k)); other values are PA_ERR_INVALID_ARG.
 * Other arguments : as pa_decode (head_dim 64 or 128, G in {1, 2, 4, 8}, block_size a
 *                   power of two in [8, 512]).
 * Math: S = Q K^T and O = P V on the tcgen05 tensor cores (fp32 accumulation in tensor
 * memory), softmax in fp32; P enters the P V product as two values of the input type, a
 * high part and the rounded remainder, so it keeps about twice the input type's
 * precision (the accuracy bar of the output, not the tensor rate, sets this).
 * One launch, no workspace.  Errors: host-checkable problems as pa_decode; n_s > L_s
 * or L_s beyond the table sets PA_DEVERR_CONTEXT (that sequence's rows are not
 * written); an out-of-range table entry sets PA_DEVERR_BLOCK_ID.
 */
pa_status pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *block_tables, const int32_t *context_lens,
                     const int32_t *query_start_loc, int num_seqs, int num_tokens,
                     int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                     int num_blocks, int max_blocks_per_seq, float scale, int sliding_window,
                     pa_dtype dtype, void *stream);

/*
 * Reads (and with clear != 0 resets) the sticky error word of `device`.
 * SYNCHRONISES that device first.  *bits_out receives PA_DEVERR_* bits (0 = none).
 */
pa_status pa_get_device_error(int device, uint32_t *bits_out, int clear);

/* Static description of a status code.  Never NULL. */
const char *pa_status_str(pa_status status);

/* Library ABI version (major * 100 + minor): 201. */
int pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
