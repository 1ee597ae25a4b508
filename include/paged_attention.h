/*
 * paged_attention.h -- C ABI of libpa.so: PagedAttention decode for NVIDIA
 * B200 (sm_100a), with the two cache-maintenance operations that feed it.
 *
 * The key/value cache of every sequence is cut into fixed-size blocks of
 * block_size token slots (16, the size the pages give as the usual one), and
 * a per-sequence block table maps the sequence's logical block j to a
 * physical block id in one shared pool (skandtandon.pages.dev day-9 post,
 * section "Idea 1: PagedAttention"; "What vLLM Is and Why It Exists",
 * section "The idea vLLM started from: pages").  The decode kernel finds
 * each of a sequence's cached keys and values through the block table,
 * wherever in the pool its block lies (same section), so its result is
 * ordinary attention over the sequence's tokens.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument except the function's own scalars is a DEVICE
 *    pointer, owned by the caller; the library allocates nothing, keeps no
 *    state between calls (apart from the fixed scratch array used by
 *    pa_decode_noalloc), and frees nothing.
 *  - Element type (pa_dtype) is the same for q, out, key, value and both
 *    caches: IEEE fp32 or bf16.  Arithmetic is fp32 in every case.
 *  - Cache layout, for K and for V alike:
 *        cache[num_blocks][num_kv_heads][block_size][head_dim]   (contiguous)
 *    so one (block, kv head) tile of block_size * head_dim elements is
 *    contiguous in memory.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  A returned PA_OK means "validated and launched".
 *  - Host-checkable problems return a non-OK status BEFORE anything is
 *    launched, and leave every buffer untouched.  These checks need no GPU.
 *  - Problems only the device can see (an index read from device memory that
 *    is out of range) never fault, trap or hang: the offending item is
 *    skipped and a bit is OR-ed into *err_flag (a device int32 the caller
 *    zeroes; may be NULL).  The bits are PA_ERRBIT_*.
 *  - Every device-side wait is bounded (about one second); a wait that runs
 *    out sets PA_ERRBIT_TIMEOUT and the kernel returns.
 */
#ifndef PAGED_ATTENTION_H
#define PAGED_ATTENTION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,  /* a null pointer, a negative size, a misaligned buffer ... */
    PA_ERR_UNSUPPORTED = 2,  /* a valid shape the library has no kernel for            */
    PA_ERR_WORKSPACE = 3,    /* the decode workspace is missing or too small            */
    PA_ERR_CUDA = 4          /* the CUDA runtime refused a query or a launch            */
} pa_status;

typedef enum pa_dtype {
    PA_F32 = 0,
    PA_BF16 = 1
} pa_dtype;

/* bits OR-ed into *err_flag by the device */
#define PA_ERRBIT_BLOCK_ID    1   /* a live block-table entry outside [0, num_blocks): that
                                     sequence's output rows are written as zeros            */
#define PA_ERRBIT_CONTEXT_LEN 2   /* context_lens[s] outside [0, min(max_context_len,
                                     max_blocks_per_seq * block_size)]: rows written as 0   */
#define PA_ERRBIT_SLOT        4   /* slot_mapping[t] >= num_blocks * block_size: skipped    */
#define PA_ERRBIT_PAIR        8   /* a copy pair with an id outside [0, num_blocks) or
                                     src == dst: skipped                                  */
#define PA_ERRBIT_TIMEOUT     16  /* a bounded device wait ran out; results are invalid and
                                     the decode workspace must be re-initialised           */
#define PA_ERRBIT_QUERY       32  /* pa_prefill: a sequence's query_start pair out of order
                                     or more query rows than tokens: its rows written as 0 */
#define PA_ERRBIT_GROUP       64  /* pa_decode_shared_prefix: a group entry that does not
                                     match the block tables (or a sequence two groups list)
                                     was ignored; those sequences were attended in full, so
                                     the output is still exact                            */

/* Human-readable name of a status code (static storage). */
const char *pa_status_str(pa_status status);

/* ------------------------------------------------------------------------
 * Decode attention
 * ------------------------------------------------------------------------
 * For each sequence s (one new query token per head) and query head h:
 *
 *     n      = context_lens[s]                      (tokens in the cache)
 *     token i (0 <= i < n) lives in physical block block_tables[s][i / 16],
 *            slot i % 16, of KV head g = h / (num_q_heads / num_kv_heads)
 *     x_i    = scale * dot(q[s][h][:], K_i[g][:])
 *     out[s][h][:] = sum_i exp(x_i - max x) V_i[g][:] / sum_i exp(x_i - max x)
 *
 * Only tokens 0..n-1 are read; unused slots of a partial last block and
 * table entries past ceil(n/16) may hold anything (NaN, -1).  n == 0 gives a
 * zero row.  out is rounded once (nearest-even) to the element type.
 * Arithmetic is fp32.  For bf16 caches with 8 query heads per KV head the
 * dot products and the weighted sum of V run on the tensor cores (bf16
 * operands, fp32 accumulation), the softmax weights being rounded to bf16
 * for that sum (and for its normaliser alike).
 *
 * Arguments:
 *   out            [num_seqs][num_q_heads][head_dim]            written
 *   q              [num_seqs][num_q_heads][head_dim]            read
 *   k_cache,
 *   v_cache        [num_blocks][num_kv_heads][16][head_dim]     read
 *   block_tables   int32 [num_seqs][max_blocks_per_seq]         read
 *   context_lens   int32 [num_seqs]                             read
 *   max_context_len  host-side upper bound of context_lens (sizes the launch
 *                  and the workspace without a device-to-host copy)
 *   scale          logit scale, usually 1/sqrt(head_dim)
 *   partition_size the most tokens one partial result may cover before the
 *                  log-sum-exp merge (a multiple of 16); 0 lets the library
 *                  cut each sequence only where it balances the work across
 *                  the GPU.  Every split is merged exactly (up to rounding):
 *                  M = max m_j, out = sum_j e^(m_j-M) o_j / sum_j e^(m_j-M) l_j.
 *   workspace      device scratch of at least pa_decode_workspace_size()
 *                  bytes, zero-filled once before its first use (for
 *                  instance with pa_decode_workspace_init); every call leaves
 *                  it zero-filled again where it must be.  Two calls that
 *                  may run at the same time must not share a workspace.
 *
 * Supported: block_size == 16; head_dim 64 or 128; num_q_heads /
 * num_kv_heads in {1, 2, 4, 8}; q, out, k_cache, v_cache 16-byte aligned.
 * Shapes outside that return PA_ERR_UNSUPPORTED.
 */
pa_status pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                   int head_dim, int max_context_len, int partition_size,
                                   pa_dtype dtype, size_t *bytes);

/* cudaMemsetAsync(workspace, 0, bytes, stream): makes a fresh workspace usable. */
pa_status pa_decode_workspace_init(void *workspace, size_t bytes, void *stream);

/* The launch pa_decode would make for these arguments on the current device:
 * CTAs in the grid, warps per CTA, pipeline depth (tiles in flight per warp)
 * and dynamic shared memory per CTA.  Any output pointer may be NULL. */
pa_status pa_decode_launch_config(int num_seqs, int num_q_heads, int num_kv_heads,
                                  int head_dim, int max_context_len, int partition_size,
                                  pa_dtype dtype, int *grid, int *warps_per_cta,
                                  int *pipeline_depth, int *smem_bytes);

pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, const int32_t *context_lens,
                    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                    int block_size, int max_blocks_per_seq, int num_blocks,
                    int max_context_len, float scale, int partition_size, pa_dtype dtype,
                    void *workspace, size_t workspace_bytes, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Decode attention without a caller-provided workspace
 * ------------------------------------------------------------------------
 * The pages describe no counterpart of this entry point; it exists for
 * callers that cannot allocate device memory while they run -- an engine
 * whose memory pool already owns the device, a step loop that cannot take
 * the device synchronisation cudaMalloc/cudaFree may cause, or a caller with
 * no allocator at all.
 *
 * Same arguments and results as pa_decode, minus the workspace: the scratch
 * it needs comes from one array of PA_NOALLOC_SCRATCH_BYTES inside the
 * library (every GPU that loads libpa.so holds it until the process exits).
 * It allocates nothing and frees nothing.
 *  - A call whose pa_decode_workspace_size exceeds PA_NOALLOC_SCRATCH_BYTES
 *    returns PA_ERR_WORKSPACE and launches nothing.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture begins.  The address is kept for the life of
 *    the process: after a cudaDeviceReset of that device (which destroys the
 *    context the address belongs to), later calls on it are invalid.
 *  - All calls share the one array.  Each call first clears, on `stream`,
 *    the part that must start at zero; calls that can run at the same time
 *    on the GPU (different streams without ordering) race on the array.
 */
#define PA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

pa_status pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_tables, const int32_t *context_lens,
                            int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                            int block_size, int max_blocks_per_seq, int num_blocks,
                            int max_context_len, float scale, int partition_size,
                            pa_dtype dtype, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Slot write (reshape_and_cache)
 * ------------------------------------------------------------------------
 * Writes each step's new key/value rows into the cache: the cache gets
 * longer with every generated token ("vLLM Solved the Wrong Bottleneck...",
 * section "Paged Attention"), and every request gains one token per step
 * ("What vLLM Is and Why It Exists", section "A picture").  For every token t and KV
 * head h:
 *     slot = slot_mapping[t];  if slot < 0: skip (padding)
 *     k_cache[slot / block_size][h][slot % block_size][:] = key[t][h][:]
 *     v_cache[...same...]                                 = value[t][h][:]
 * A bit-exact copy.  key, value: [num_tokens][num_kv_heads][head_dim];
 * slot_mapping: int64 [num_tokens].  Slots must be distinct within a call.
 * head_dim * element size must be a multiple of 16 bytes; buffers 16-byte
 * aligned; any block_size >= 1.
 */
pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_cache,
                               void *v_cache, const int64_t *slot_mapping, int num_tokens,
                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               pa_dtype dtype, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Fused slot write + decode attention
 * ------------------------------------------------------------------------
 * One decode step in one call: each sequence's newest key/value row (one new
 * token per request per step, "What vLLM Is and Why It Exists", section "A
 * picture"; the cache grows by that token, "vLLM Solved the Wrong
 * Bottleneck...", section "Paged Attention") is written to its slot AND used
 * by the attention of the same step.  For every sequence s with
 * n = context_lens[s] >= 1 (n counts the new token) and KV head h, with
 * slot = block_tables[s][(n-1) / block_size] * block_size + (n-1) % block_size:
 *     k_cache[slot / block_size][h][slot % block_size][:] = key[s][h][:]
 *     v_cache[...same...]                                 = value[s][h][:]
 *     out[s] = pa_decode's result over positions 0..n-1
 * The result is that of pa_reshape_and_cache with those slots followed by
 * pa_decode, bit for bit: the kernel takes the newest row from key/value
 * (not from the cache) and writes it back from shared memory, so the step
 * costs one launch pair instead of two and never re-reads the row it wrote.
 *
 *   key, value  device, [num_seqs][num_kv_heads][head_dim], 16-byte aligned.
 *   Every other argument, the workspace rule and the supported shapes are
 *   pa_decode's.
 * A sequence with n == 0 writes nothing and gets out = 0.  A sequence whose
 * n is out of range (PA_ERRBIT_CONTEXT_LEN) or whose last block-table entry
 * is out of range (PA_ERRBIT_BLOCK_ID) writes nothing.  The block receiving
 * the new row must belong to that sequence alone (copy-on-write done
 * beforehand, as pa_copy_blocks does): a block another sequence of the same
 * call also reads races with the write.
 */
pa_status pa_decode_append(void *out, const void *q, const void *key, const void *value,
                           void *k_cache, void *v_cache, const int32_t *block_tables,
                           const int32_t *context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size,
                           int max_blocks_per_seq, int num_blocks, int max_context_len,
                           float scale, int partition_size, pa_dtype dtype, void *workspace,
                           size_t workspace_bytes, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Several query tokens per sequence (chunked prefill, checked drafts)
 * ------------------------------------------------------------------------
 * A chunk of a prompt is attended to like decode tokens, each seeing the
 * cache up to its own position.  The chunk's K/V must already be in the
 * cache (pa_reshape_and_cache), since the cache grows by every token before
 * it attends ("vLLM Solved the Wrong Bottleneck...", section "Paged
 * Attention").  For sequence s with n = context_lens[s] cached tokens and
 * Q = query_start[s+1] - query_start[s] query rows, query row j (global row
 * r = query_start[s] + j) is the token at position p = n - Q + j:
 *     out[r][h][:] = softmax_i(scale * q[r][h] . K_i) . V_i  over i = 0..p
 * with K_i, V_i of KV head h / (num_q_heads / num_kv_heads), found through
 * block_tables[s] as in pa_decode.
 *
 *   q, out          device, [num_query_tokens][num_q_heads][head_dim].
 *   query_start     device int32 [num_seqs + 1], non-decreasing, from 0 to
 *                   num_query_tokens; Q <= n for every sequence.  A
 *                   sequence with Q > n gets zero rows and PA_ERRBIT_QUERY;
 *                   query_start values out of order or outside
 *                   [0, num_query_tokens] set PA_ERRBIT_QUERY, and rows no
 *                   valid sequence covers may be left unwritten.
 *   workspace       pa_prefill_workspace_size() bytes, zero-filled before
 *                   first use (pa_decode_workspace_init), as for pa_decode.
 *   Everything else is as in pa_decode.
 *
 *   bf16 caches with head_dim 64 or 128, 1, 2, 4 or 8 query heads per KV
 *   head and fewer than 2^24 (query row, head) columns per KV head run on
 *   the tcgen05 tensor cores: a column is one (query row, query
 *   head) of a KV head, 128 columns form a tile, and a CTA takes two tiles
 *   of one sequence, which share each 64-key K/V tile of their causal
 *   prefix (the weights are rounded to bf16 for the P.V product, the sum
 *   takes them as rounded).  A one-CTA plan kernel first checks every block
 *   each sequence attends to (a bad block id zeroes that sequence's rows
 *   and sets PA_ERRBIT_BLOCK_ID) and lists the work longest first.  This
 *   path needs no zeroed workspace and uses about 225 KiB of shared memory
 *   per CTA at head_dim 128 (PA_ERR_UNSUPPORTED if the device has less).
 *   fp32 caches, and other shapes, take the decode kernel with each query
 *   row (or, for bf16 with 8 query heads per KV head, each pair of rows)
 *   as a work item over its own prefix; there, launch-time shared memory
 *   grows with num_query_tokens (12 to 20 bytes per row) and too many rows
 *   for one SM's shared memory returns PA_ERR_UNSUPPORTED.
 */
pa_status pa_prefill_workspace_size(int num_seqs, int num_query_tokens, int num_q_heads,
                                    int num_kv_heads, int head_dim, int max_context_len,
                                    int partition_size, pa_dtype dtype, size_t *bytes);

/* The launch pa_prefill would make (as pa_decode_launch_config). */
pa_status pa_prefill_launch_config(int num_seqs, int num_query_tokens, int num_q_heads,
                                   int num_kv_heads, int head_dim, int max_context_len,
                                   int partition_size, pa_dtype dtype, int *grid,
                                   int *warps_per_cta, int *pipeline_depth, int *smem_bytes);

pa_status pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *block_tables, const int32_t *context_lens,
                     const int32_t *query_start, int num_seqs, int num_query_tokens,
                     int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                     int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                     int partition_size, pa_dtype dtype, void *workspace,
                     size_t workspace_bytes, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Prefix-deduplicated decode
 * ------------------------------------------------------------------------
 * Requests with a common prefix hold the same physical blocks for it
 * (day-9 post, section "Idea 1: PagedAttention", sharing).  pa_decode reads
 * such a block once per sequence; pa_decode_shared_prefix reads it once per
 * group: a tensor-core pass computes, for every (member, query head) of a
 * group and the group's shared blocks, the online-softmax state (running
 * max, sum of weights, unnormalised output), and the decode kernel goes on
 * from that state over each sequence's remaining blocks.  Attention over the
 * union of two token sets is the log-sum-exp combination of the two, so the
 * result is that of pa_decode (or, with key/value, pa_decode_append) up to
 * rounding: the shared part's weights are rounded to bf16 for the product,
 * as on the tensor-core decode path.  bf16 only (fp32 returns
 * PA_ERR_UNSUPPORTED).
 *
 * The groups: group g lists its member sequences in
 *   group_seqs[group_start[g] .. group_start[g+1])   (device int32)
 * and shares its first group_blocks[g] logical blocks (device int32): every
 * member's block table holds the same physical ids there, and every member
 * has at least one token after them (16 * group_blocks[g] < n).  Both are
 * checked on the device (by the kernel that folds the pass's ranges into
 * each member's state); a member that fails, or a sequence that two groups
 * list, is attended in full by the decode kernel and PA_ERRBIT_GROUP is
 * set.  A sequence in no group is attended as by pa_decode.
 * num_listed = group_start[num_groups]; num_groups <= 16384
 * (PA_ERR_UNSUPPORTED above) and num_groups <= num_listed (PA_ERR_INVALID_ARG).
 *
 * pa_shared_prefix_plan finds such groups on the HOST (its pointers are
 * host pointers, unlike every other entry point's): sequences whose first
 * physical block is the same form a candidate group, which shares the
 * longest run of leading blocks all its members hold, capped so that each
 * keeps one token of its own.  Groups of one member, or sharing fewer than
 * min_shared_blocks blocks, are dropped.  Output arrays: group_seqs and
 * group_blocks of num_seqs entries, group_start of num_seqs + 1.  Groups are
 * ordered by their first member, members by sequence index.
 *
 * Workspace: pa_shared_prefix_workspace_size() bytes, zero-filled before
 * first use (pa_decode_workspace_init); the calls leave it ready for the
 * next one.  Everything else is as in pa_decode / pa_decode_append.
 */
pa_status pa_shared_prefix_plan(const int32_t *block_tables, const int32_t *context_lens,
                                int num_seqs, int max_blocks_per_seq, int block_size,
                                int min_shared_blocks, int32_t *group_seqs,
                                int32_t *group_start, int32_t *group_blocks, int *num_groups,
                                int *num_listed);

/* The same output for sharing that forms a tree (forks of forks): the groups
 * are chosen on the trie of the sequences' block paths (each path: the
 * table up to the block before the one holding the last token).  Bottom-up,
 * the k sequences left ungrouped below a trie node of depth d are grouped
 * there, sharing d blocks, when (k - 1) * d >= k * d_parent; otherwise they
 * go up to the parent node.  It never saves fewer block reads than
 * pa_shared_prefix_plan and saves more when a sub-group shares a longer run
 * than its whole family.  Host pointers, as pa_shared_prefix_plan. */
pa_status pa_shared_prefix_plan_tree(const int32_t *block_tables, const int32_t *context_lens,
                                     int num_seqs, int max_blocks_per_seq, int block_size,
                                     int min_shared_blocks, int32_t *group_seqs,
                                     int32_t *group_start, int32_t *group_blocks,
                                     int *num_groups, int *num_listed);

pa_status pa_shared_prefix_workspace_size(int num_seqs, int num_listed, int num_q_heads,
                                          int num_kv_heads, int head_dim,
                                          int max_blocks_per_seq, int max_context_len,
                                          int partition_size, pa_dtype dtype, size_t *bytes);

/* key, value: NULL for plain decode, or both given for the fused slot write
 * of pa_decode_append. */
pa_status pa_decode_shared_prefix(void *out, const void *q, const void *key, const void *value,
                                  void *k_cache, void *v_cache, const int32_t *block_tables,
                                  const int32_t *context_lens, const int32_t *group_seqs,
                                  const int32_t *group_start, const int32_t *group_blocks,
                                  int num_groups, int num_listed, int num_seqs, int num_q_heads,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int max_blocks_per_seq, int num_blocks, int max_context_len,
                                  float scale, int partition_size, pa_dtype dtype,
                                  void *workspace, size_t workspace_bytes, int32_t *err_flag,
                                  void *stream);

/* ------------------------------------------------------------------------
 * Block copy-on-write (copy_blocks)
 * ------------------------------------------------------------------------
 * A block shared by several sequences is duplicated, alone, at the moment
 * one of them must change it (day-9 post, section "Idea 1: PagedAttention",
 * copy-on-write).  For each pair p of
 * block_mapping (int32 [num_pairs][2] = {src, dst}), the whole physical
 * block src -- all KV heads, all block_size slots -- is copied to dst, in
 * k_cache and in v_cache.  A bit-exact copy.  The dst ids must be distinct
 * and disjoint from the src ids (otherwise the result is undefined).
 */
pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int32_t *block_mapping,
                         int num_pairs, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype dtype, int32_t *err_flag, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_ATTENTION_H */
