/*
 * pagedkv.h: C ABI of libpagedkv.so, decode-step attention over a block-paged
 * KV cache on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages on paged attention; cited by title and section):
 *   [Explained] "Paged Attention Explained: How LLMs Manage GPU Memory for
 *               Faster AI Inference"
 *   [Wiki]      "PagedAttention: paging the KV cache like an OS pages memory"
 *   [Index]     "PagedAttention and KV Cache Compression: Optimizing LLM
 *               Inference"
 *
 * Data layout (row-major, element type bf16 or fp32, identical for K and V):
 *   k_cache, v_cache  [num_blocks][block_size][Hkv][D]   the block pool
 *   block_tables      [B][max_blocks] int32               physical id of each
 *                                                         logical block
 *   seq_lens          [B] int32                           cached tokens per sequence
 *   q, out            [B][Hq][D]                          one query per sequence
 *   k, v (new tokens) [N][Hkv][D]
 *   slot_mapping      [N] int64, slot = block * block_size + offset; < 0 skips
 *   block_mapping     [P][2] int64, (src, dst) physical block ids
 *
 * Conventions shared by every call:
 *   - Ownership: every pointer is caller-owned device memory (pointers that are
 *     passed to a kernel must be device-accessible).  The library keeps no
 *     pointer after the call returns.  Apart from the decode workspace, which
 *     the caller provides, it allocates no device memory.
 *   - Streams: every call enqueues its work on `stream` (NULL = the legacy
 *     default stream) and returns without synchronising.  Kernels are
 *     launched with programmatic stream serialization: a launch's CTAs may be
 *     placed while the kernel before it in the stream finishes, but each waits
 *     for that kernel to complete before it reads or writes global memory, so
 *     every access keeps the stream order.
 *   - Alignment: every data pointer must be 16-byte aligned.
 *   - Errors: a call returns PKV_OK or a negative status.  It validates
 *     arguments on the host before enqueueing anything, and on a validation
 *     error nothing is enqueued.  Values that only the device sees (slots,
 *     block ids, lengths) are range-checked in the kernels: an offending entry
 *     is skipped or clamped, never dereferenced out of bounds, and its bit
 *     is OR-ed into a device error word that pkv_device_errors() reads.
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *pkv_stream_t;

/* Element type of q, k, v, out and both caches. */
typedef enum { PKV_BF16 = 0, PKV_F32 = 1 } pkv_dtype;

/* Status codes. */
enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, bad dimension or dtype */
    PKV_ERR_OUT_OF_RANGE = -2, /* a host-checkable size or bound is out of range */
    PKV_ERR_WORKSPACE = -3,    /* decode workspace missing or too small */
    PKV_ERR_CUDA = -4,         /* a CUDA call failed; see pkv_last_cuda_error() */
    PKV_ERR_UNSUPPORTED = -5,  /* valid but unsupported shape (head dim, block size, G) */
    PKV_ERR_SCRATCH_LIMIT = -6 /* paged_attention_decode_noalloc: sizes need more than
                                  PKV_NOALLOC_SCRATCH_BYTES of scratch */
};

/* Device error bits (pkv_device_errors). */
#define PKV_DEVERR_SLOT 0x1u     /* paged_kv_write skipped a slot >= num_blocks*block_size */
#define PKV_DEVERR_SEQLEN 0x2u   /* a seq_len < 0, > max_blocks*block_size or > max_seq_len was clamped */
#define PKV_DEVERR_BLOCK_ID 0x4u /* a block-table id outside [0, num_blocks) was read as zeros */
#define PKV_DEVERR_COPY 0x8u     /* copy_blocks skipped a pair with an id outside [0, num_blocks) */
#define PKV_DEVERR_TIMEOUT 0x10u /* a pipeline wait gave up after its time limit */
#define PKV_DEVERR_PREFIX 0x20u  /* shared-prefix decode: a member's table entries differ from
                                    the group's first member, or a sequence is in no group */

/*
 * paged_kv_write: the cache update.  [Explained] "Step 2: Allocate Blocks
 * Dynamically" and the list of duties of a production implementation ("cache
 * updates") in "Practical Example"; [Index] "5. Real-World Consequences" (a
 * new token fills the current block; a new block only when it is full).
 *
 * For every n < N with s = slot_mapping[n] >= 0, row n of k and v
 * (Hkv*D elements each) is copied bit for bit to k_cache and v_cache at
 * block s / block_size, offset s % block_size.  Slots < 0 are skipped.
 * Slots >= num_blocks*block_size are skipped and flag PKV_DEVERR_SLOT.
 * Two tokens with the same slot race (one of them wins).
 *   k, v            device [N][Hkv][D]
 *   k_cache,v_cache device [num_blocks][block_size][Hkv][D], updated in place
 *   slot_mapping    device [N] int64
 * Requires Hkv*D*element size to be a multiple of 16 bytes.  N == 0 is a no-op.
 */
int paged_kv_write(const void *k, const void *v, void *k_cache, void *v_cache,
                   const int64_t *slot_mapping, int64_t N, int Hkv, int D, int block_size,
                   int64_t num_blocks, pkv_dtype dtype, pkv_stream_t stream);

/*
 * Partition length (tokens) that paged_attention_decode uses for these sizes:
 * `partition_size` itself when it is > 0, otherwise the library's choice, a
 * multiple of 16 that depends only on the arguments (0 when the process runs
 * the work-balanced split, see pkv_set_decode_split).  Returns a negative
 * status for invalid arguments.
 */
int paged_attention_decode_partition_size(int B, int Hkv, int max_seq_len, int block_size,
                                          int partition_size);

/*
 * Workspace bytes paged_attention_decode needs for these sizes, in either
 * split mode (0 when no partial results can arise).  It is a pure host function
 * with no CUDA calls.  Returns 0 for invalid arguments (the call then reports
 * the error).
 */
size_t paged_attention_decode_workspace_size(int B, int Hq, int Hkv, int D, int max_seq_len,
                                             int block_size, int partition_size);

/*
 * paged_attention_decode: single-query attention over the paged cache.
 * The attention is ordinary softmax attention; only the storage layout
 * differs ([Wiki] "How it works").  The kernel follows the block table to
 * find each token's keys and values ([Explained] "Step 3: Maintain a Block
 * Table", "Step 4: Retrieve Cached Data During Attention"; [Index] "4.
 * Technical Depth").  Scores are accumulated with a running maximum and sum
 * (online softmax, the tiling idea named in [Explained] "What Is the
 * Difference Between PagedAttention and FlashAttention?").
 *
 * For b < B and h < Hq, with G = Hq / Hkv, kvh = h / G, L = seq_lens[b]:
 *   K_t = k_cache[block_tables[b][t / block_size]][t % block_size][kvh]
 *   V_t likewise, for t < L
 *   out[b][h] = sum_t softmax_t(scale * q[b][h] . K_t) * V_t
 * out[b][h] = 0 when L == 0.  Arithmetic is fp32; bf16 inputs are widened
 * exactly and the result is rounded to nearest even.  Slots past L in the
 * last block, and table entries past ceil(L / block_size), are never read.
 *
 * Work split.  Each sequence is cut into partitions of P tokens (P =
 * partition_size, or the library's choice when it is 0), one CTA per (KV
 * head, partition, sequence).  pkv_set_decode_split selects a work-balanced
 * persistent split instead.  A (sequence, KV head) cut in several pieces yields
 * one partial (max, sum, weighted V) per piece.  The partials are merged with a
 * log-sum-exp rescale in the same launch.
 *
 *   out             device [B][Hq][D], written
 *   q               device [B][Hq][D]
 *   k_cache,v_cache device [num_blocks][block_size][Hkv][D]
 *   block_tables    device [B][max_blocks] int32
 *   seq_lens        device [B] int32
 *   max_seq_len     host upper bound of seq_lens (sets the partition grid
 *                   without a device-to-host copy); a larger seq_len is
 *                   clamped to it and flags PKV_DEVERR_SEQLEN
 *   partition_size  0 = library choice, else a positive multiple of 16
 *   workspace       device, >= paged_attention_decode_workspace_size(...)
 *                   bytes, 256-byte aligned, ZERO-FILLED before its first
 *                   use.  Each completed call leaves it ready for the next
 *                   one (its counters are back at zero).  Two calls that
 *                   share a workspace must not overlap on the GPU.  It may be
 *                   NULL when the size is 0.  After a call that raised
 *                   PKV_DEVERR_TIMEOUT the counters may be left non-zero (the
 *                   CTAs that stopped early took no ticket): zero-fill the
 *                   workspace again before its next use.
 * Supported: bf16 with D in {64, 128, 256}; fp32 with D in {64, 128};
 * block_size 8, or a multiple of 16 up to 256 (the kernels stream 16-token
 * stages; with 8-token blocks a stage is gathered from two blocks); G = Hq / Hkv
 * <= 16 (bf16) or <= 8 (fp32); num_blocks * block_size < 2^31.  The
 * work-balanced split (pkv_set_decode_split) needs block_size a multiple of 16;
 * with 8-token blocks the fixed split runs.
 */
int paged_attention_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *block_tables, int max_blocks, const int32_t *seq_lens,
                           int max_seq_len, int B, int Hq, int Hkv, int D, int block_size,
                           int64_t num_blocks, float scale, pkv_dtype dtype,
                           int partition_size, void *workspace, size_t workspace_bytes,
                           pkv_stream_t stream);

/*
 * paged_attention_decode_contiguous: the same decode over an UNPAGED cache, as a
 * measurement control for the cost of paging.  [Index] "Limitations" says that
 * following the block table may make a request slightly slower than a perfectly
 * contiguous allocation; this call runs paged_attention_decode's own kernel with
 * the block-table walk removed, so that the two can be timed on the same K/V.
 *   k_cache, v_cache  device [B][row_stride][Hkv][D]: sequence b's token t is row
 *                     b * row_stride + t (row_stride >= max_seq_len)
 *   workspace         as paged_attention_decode's, sized by
 *                     paged_attention_decode_workspace_size(B, Hq, Hkv, D,
 *                     max_seq_len, 16, partition_size)
 * Every other argument is paged_attention_decode's.  bf16 only (the tensor-core
 * kernel); fixed-length partitions whatever pkv_set_decode_split says; B *
 * row_stride < 2^31.
 */
int paged_attention_decode_contiguous(void *out, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *seq_lens,
                                      int max_seq_len, int row_stride, int B, int Hq, int Hkv,
                                      int D, float scale, pkv_dtype dtype, int partition_size,
                                      void *workspace, size_t workspace_bytes,
                                      pkv_stream_t stream);

/*
 * paged_attention_prefill: multi-query attention over the paged cache, for
 * prefill or a chunked append.  Sequence b holds L = seq_lens[b] cached tokens,
 * whose last Q = cu_q[b+1] - cu_q[b] are this call's queries (their K/V already
 * written, e.g. by paged_kv_write).  Query i (row cu_q[b] + i of q) sits at
 * position L - Q + i and attends causally to tokens 0 .. L - Q + i: each row is
 * paged_attention_decode's softmax attention over its visible prefix ([Wiki]
 * "How it works": standard causal attention, only the layout changes).
 *   out, q        device [total_q][Hq][D]
 *   cu_q          device [B + 1] int32, non-decreasing, cu_q[B] = total_q
 *   max_q_len     host upper bound of Q; max_seq_len host upper bound of L
 * It runs on the tcgen05 tensor cores: a query tile is 128 rows (128/G tokens x
 * the G query heads of one KV head); S = Q K^T and O += P V accumulate in tensor
 * memory.  For D <= 128 a CTA takes two query tiles of one KV head and streams
 * the sequence's K/V in 128-token tiles (the two tiles' softmaxes alternate
 * with the other tile's MMAs); for D = 256 one tile and 64-token K/V tiles.
 * bf16 only; G in {1, 2, 4, 8, 16}; D in {64, 128, 256}; block_size a multiple
 * of 16 up to 256.  A sequence with Q > L flags PKV_DEVERR_SEQLEN and its rows
 * are not written.
 *   workspace     device scratch of paged_attention_prefill_workspace_size()
 *                 bytes (4-byte aligned, no initialisation needed) or NULL.
 *                 With it (D <= 128), a first small kernel orders the work
 *                 items (pairs of query tiles) longest first and one CTA per
 *                 SM takes them in that order; without it, one CTA per item.
 *                 A workspace serves one call at a time (stream order).
 */
size_t paged_attention_prefill_workspace_size(int B, int Hq, int Hkv, int max_q_len);
int paged_attention_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_tables, int max_blocks, const int32_t *seq_lens,
                            const int32_t *cu_q, int total_q, int max_q_len, int max_seq_len,
                            int B, int Hq, int Hkv, int D, int block_size, int64_t num_blocks,
                            float scale, pkv_dtype dtype, void *workspace,
                            size_t workspace_bytes, pkv_stream_t stream);

/*
 * paged_decode_step: one whole decode step in one launch.  For every sequence b
 * with L = seq_lens[b] > 0, in this order:
 *   1. if cow_src != NULL and cow_src[b] >= 0: copy physical block cow_src[b] into
 *      the block that holds token L - 1 (block_tables[b][(L-1) / block_size]),
 *      as copy_blocks does;
 *   2. store k_new[b], v_new[b] as token L - 1, as paged_kv_write does with
 *      slot = block_tables[b][(L-1) / block_size] * block_size + (L-1) % block_size;
 *   3. decode as paged_attention_decode over tokens 0 .. L-1.
 * This is the per-step loop of the pages: cache the new token, copying a shared
 * block before modifying it ([Explained] "Step 2" and "Step 4"; [Wiki] "How it
 * works").  The copy and the write are done, per KV head, by the decode CTA of
 * the sequence's last partition, which is the only CTA that reads that block.
 * So one launch replaces three.
 *   seq_lens  lengths after the step (they include the new token)
 *   k_new, v_new  device [B][Hkv][D]
 *   cow_src   device [B] int32 or NULL; -1 = no copy
 * Contract: the copy targets only blocks that receive this step's new tokens
 * (copy-on-write of a shared block about to be written).  The other arguments,
 * the workspace rules and the supported shapes are those of
 * paged_attention_decode, with fixed-length partitions whatever
 * pkv_set_decode_split says, and the partition length (partition_size, or the
 * library's choice) rounded up to a multiple of block_size: the block that
 * receives a sequence's new token then lies in its last partition only.  The
 * size from paged_attention_decode_workspace_size for the same arguments
 * suffices (longer partitions leave fewer partials).
 */
int paged_decode_step(void *out, const void *q, const void *k_new, const void *v_new,
                      void *k_cache, void *v_cache, const int32_t *block_tables, int max_blocks,
                      const int32_t *seq_lens, const int32_t *cow_src, int max_seq_len, int B,
                      int Hq, int Hkv, int D, int block_size, int64_t num_blocks, float scale,
                      pkv_dtype dtype, int partition_size, void *workspace, size_t workspace_bytes,
                      pkv_stream_t stream);

/*
 * paged_attention_decode_shared_prefix: paged_attention_decode for batches in
 * which consecutive sequences share the physical blocks of a prefix: decode
 * branches of one request, parallel samples, a common prompt.  Physical blocks
 * are shared through identical table entries ([Wiki] "How it works";
 * [Index] "Complex Decoding (Beam Search & Parallel Sampling)").  The result
 * is the same; each shared block is read once per group instead of once per
 * member.  Prefix pieces score one read of the shared K/V against the queries
 * of up to 16 / G members at once, stacked in the tensor-core N dimension.
 * Pieces over each sequence's own tokens follow, as in paged_attention_decode.
 * The pieces' partials are merged in the same launch.  When partition_size is
 * 0 and max_group_size <= 16 / G, each (group, KV head) is instead one CTA that
 * reads the prefix once and every member's own tokens, with no partials (the
 * workspace is then left untouched, but must still be passed).
 *   group_offsets  device [n_groups + 1] int32: group g is sequences
 *                  group_offsets[g] .. group_offsets[g+1]-1.  The offsets start
 *                  at 0, end at B and never decrease (a group may have one member).
 *   prefix_lens    device [n_groups] int32: leading tokens whose blocks are
 *                  the same physical blocks in every member (equal table
 *                  entries).  The decode uses min(prefix_len, shortest member's
 *                  length - 1), rounded down to whole blocks.  0 means nothing shared.
 *   max_group_size host upper bound of the group sizes.
 * The other arguments are as for paged_attention_decode.  bf16 only, G <= 16.
 * The workspace (paged_attention_decode_shared_prefix_workspace_size) follows the
 * same rules as paged_attention_decode's: zero-filled before first use, left
 * ready for the next call, not shared by overlapping calls.  A prefix piece checks the
 * members' table entries against the first member's; a mismatch, or a sequence
 * that no group covers, flags PKV_DEVERR_PREFIX.
 */
int paged_attention_decode_shared_prefix(void *out, const void *q, const void *k_cache,
                                         const void *v_cache, const int32_t *block_tables,
                                         int max_blocks, const int32_t *seq_lens, int max_seq_len,
                                         const int32_t *group_offsets, const int32_t *prefix_lens,
                                         int n_groups, int max_group_size, int B, int Hq, int Hkv,
                                         int D, int block_size, int64_t num_blocks, float scale,
                                         pkv_dtype dtype, int partition_size, void *workspace,
                                         size_t workspace_bytes, pkv_stream_t stream);

/*
 * paged_decode_step_shared_prefix: paged_decode_step for grouped batches.  It
 * does the copy-on-write copy and the new token's write, then
 * paged_attention_decode_shared_prefix, all in one launch.  The new token
 * (position seq_lens[b] - 1) must lie after the group's shared prefix; the decode
 * caps the prefix one token short of the shortest member and rounds it down to
 * whole blocks, so that holds for any prefix_lens value, and the block a step
 * rewrites is never one a prefix piece reads.  With partitions (partition_size
 * > 0, or groups larger than 16 / G), the partition length is rounded up to a
 * multiple of block_size, as in paged_decode_step.  Arguments are those of the
 * two calls.
 */
int paged_decode_step_shared_prefix(void *out, const void *q, const void *k_new,
                                    const void *v_new, void *k_cache, void *v_cache,
                                    const int32_t *block_tables, int max_blocks,
                                    const int32_t *seq_lens, const int32_t *cow_src,
                                    int max_seq_len, const int32_t *group_offsets,
                                    const int32_t *prefix_lens, int n_groups, int max_group_size,
                                    int B, int Hq, int Hkv, int D, int block_size,
                                    int64_t num_blocks, float scale, pkv_dtype dtype,
                                    int partition_size, void *workspace, size_t workspace_bytes,
                                    pkv_stream_t stream);

/* Workspace bytes of paged_attention_decode_shared_prefix (pure host function;
 * 0 for invalid arguments). */
size_t paged_attention_decode_shared_prefix_workspace_size(int B, int Hq, int Hkv, int D,
                                                           int max_seq_len, int block_size,
                                                           int partition_size);

/*
 * paged_attention_decode_noalloc: the same decode as paged_attention_decode
 * for callers that cannot allocate device memory and have no workspace of
 * their own to lend.  Examples are a host program whose device memory is
 * entirely owned by its own pool allocator, and a serving loop that must not
 * call cudaMalloc mid-step because the call may synchronise the device.  The
 * pages describe no such entry point; it has no counterpart there.
 *
 * Arguments and results are those of paged_attention_decode without the
 * workspace.  The split-partition scratch lives in one array of
 * PKV_NOALLOC_SCRATCH_BYTES in the library's device memory.  Every GPU that
 * loads the library holds that array until the process exits.  The call
 * allocates and frees nothing.
 *   - Sizes whose scratch (paged_attention_decode_workspace_size) exceeds
 *     PKV_NOALLOC_SCRATCH_BYTES are rejected with PKV_ERR_SCRATCH_LIMIT before
 *     anything is enqueued.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and keeps it for the
 *     process.  Make that first call before any stream capture.  A
 *     cudaDeviceReset after it is not supported: the kept address would be
 *     stale.
 *   - All calls share the one array, and it keeps what the last call left.
 *     Each call therefore clears the part that must start at zero (the
 *     partition counters) on `stream` before the decode.  Calls that overlap
 *     on the GPU (other streams, other host threads) race on the array and
 *     give wrong results; serialise them.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (16u << 20)
int paged_attention_decode_noalloc(void *out, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *block_tables,
                                   int max_blocks, const int32_t *seq_lens, int max_seq_len, int B,
                                   int Hq, int Hkv, int D, int block_size, int64_t num_blocks,
                                   float scale, pkv_dtype dtype, int partition_size,
                                   pkv_stream_t stream);

/*
 * copy_blocks: block-granularity copy-on-write copies.  Physical blocks are
 * reference-counted and shared between requests or decode branches, and a
 * shared block that must be modified is first copied ([Wiki] "How it works";
 * [Index] "Complex Decoding (Beam Search & Parallel Sampling)", glossary
 * "Copy-on-Write").  Deciding which blocks to copy is the caller's job.
 *
 * For each pair i < P: k_cache[dst] = k_cache[src] and v_cache[dst] =
 * v_cache[src], whole blocks of block_bytes bytes, bit for bit.  The dst ids
 * must be distinct and no dst may also be a src (otherwise the result
 * depends on order).  Pairs with an id outside [0, num_blocks) are skipped
 * and flag PKV_DEVERR_COPY.
 *   k_cache,v_cache device pools of num_blocks blocks of block_bytes each
 *   block_mapping   device [P][2] int64 (src, dst)
 *   block_bytes     block_size*Hkv*D*element size, a multiple of 16
 */
int copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping, int64_t P,
                int64_t block_bytes, int64_t num_blocks, pkv_stream_t stream);

/* Short English text for a status code (static storage). */
const char *pkv_status_string(int status);

/* The cudaError_t of the last PKV_ERR_CUDA returned on this host thread
 * (100000 + CUresult when encoding a TMA tensor map failed). */
int pkv_last_cuda_error(void);

/*
 * Reads the device error word of the current device into *bits, and clears it
 * when `clear` is non-zero.  This synchronises with the device.  When
 * PKV_DEVERR_TIMEOUT is set, the outputs of the launches that saw it are
 * undefined, and every decode workspace they used must be zero-filled again
 * before its next use (their partition counters may be left non-zero).
 */
int pkv_device_errors(uint32_t *bits, int clear);

/*
 * Self-test of the pipelines' time limit.  Launches (on `stream`) one kernel
 * whose single thread waits, with the bounded wait that every TMA / MMA
 * pipeline of this library uses, on a barrier that nothing completes.  After
 * 2^30 SM cycles (about 0.55 s at 1.965 GHz) the wait gives up and sets
 * PKV_DEVERR_TIMEOUT; the device stays usable.  While that bit is set, every
 * CTA of every attention launch (decode, shared-prefix decode, prefill) returns
 * at once, whole, without reading or writing anything, so that one stall does
 * not become a wait per CTA; pkv_device_errors(&bits, 1) clears it.  Such a
 * CTA takes no partition ticket, so a workspace used while the bit was set must
 * be zero-filled again before its next use.  Returns PKV_OK or PKV_ERR_CUDA
 * (launch failure).
 */
int pkv_debug_stalled_wait(pkv_stream_t stream);

/*
 * Arithmetic units used by paged_attention_decode, set for the whole process
 * (for testing and measuring both kernels):
 *   PKV_PATH_AUTO          every bf16 call on tensor cores, fp32 on CUDA cores;
 *   PKV_PATH_CUDA_CORES    fp32 FMAs whenever G <= 8;
 *   PKV_PATH_TENSOR_CORES  warp-level bf16 MMA for every bf16 call.
 * fp32 always runs on CUDA cores.  Returns the previous mode, or
 * PKV_ERR_INVALID_ARG.  The results of both kernels satisfy the same bounds.
 */
enum { PKV_PATH_AUTO = 0, PKV_PATH_CUDA_CORES = 1, PKV_PATH_TENSOR_CORES = 2 };
int pkv_set_decode_path(int mode);

/*
 * Launch overlap, set for the whole process: 1 (default) launches every kernel
 * with programmatic stream serialization (a launch's CTAs may be placed while the
 * kernel before it in the stream finishes; each waits for that kernel before it
 * touches global memory); 0 launches them in plain stream order, each grid
 * starting once the previous kernel has completed.  Results are the same bits
 * either way.  Returns the previous setting, or PKV_ERR_INVALID_ARG.
 */
int pkv_set_launch_overlap(int enabled);

/*
 * Kernel used by paged_attention_prefill, set for the whole process (for
 * testing and measuring both):
 *   PKV_PREFILL_AUTO         D <= 128: the warp-specialised kernel with two
 *                            query tiles per CTA; D = 256: one tile per CTA;
 *   PKV_PREFILL_SINGLE_TILE  one query tile per CTA for every D.
 * Both give results within the same bounds.  Returns the previous mode, or
 * PKV_ERR_INVALID_ARG.
 */
enum { PKV_PREFILL_AUTO = 0, PKV_PREFILL_SINGLE_TILE = 1 };
int pkv_set_prefill_path(int mode);

/*
 * How paged_attention_decode with partition_size == 0 cuts the work, set for
 * the whole process:
 *   PKV_SPLIT_FIXED (default)  partitions of a library-chosen length, one CTA
 *                              each (grid over KV heads, partitions, sequences);
 *   PKV_SPLIT_BALANCED         a persistent grid in which every warp takes an
 *                              equal contiguous range of one KV head's stream of
 *                              16-token stages (B <= 2048; otherwise FIXED).
 * Both give results within the same bounds.  paged_attention_decode_workspace_size
 * covers either mode.  Returns the previous mode, or PKV_ERR_INVALID_ARG.
 */
enum { PKV_SPLIT_FIXED = 0, PKV_SPLIT_BALANCED = 1 };
int pkv_set_decode_split(int mode);

/*
 * Number of CTAs of the work-balanced decode kernel, set for the whole process
 * (for tests and measurements): 0 (default) launches as many as are resident
 * at once, at most 2 per SM; n > 0 launches min(n, 296).  Results satisfy the
 * same bounds for every value.  Returns the previous value, or
 * PKV_ERR_INVALID_ARG for n < 0.
 */
int pkv_set_decode_ctas(int ctas);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */
