/*
 * pa.h - C ABI of the B200 (sm_100a) paged KV-cache decode library (libpa.so).
 *
 * The operation is PagedAttention's data path as three web pages describe it:
 *   [GLOSS] "PagedAttention", inferensys.com LLM-operations glossary;
 *   [BLOG]  "How PagedAttention Powers vLLM's KV Cache", hassanahmed.net;
 *   [LAB]   "PagedAttention", divagr.pages.dev attention-lab explainer.
 * Keys and values of each sequence live in fixed-size physical blocks of one shared
 * pool; a per-sequence block table maps logical block j to a physical block ([BLOG]
 * "PagedAttention: paging, borrowed from the operating system"; [LAB] "Keep pages in
 * order").  The attention kernel walks that table and gathers K/V block by block
 * ([BLOG] "The attention kernel has to read scattered blocks"); blocks are shared
 * between sequences with reference counts and copied before a shared block is
 * written ([BLOG] "The bonus contiguous storage can't give you: sharing"; [LAB]
 * "Share matching prefixes").
 *
 * Conventions shared by every entry point
 *   - Return value: a pa_status.  PA_OK is 0; anything else means the call did
 *     nothing (argument errors are found before any launch) or, for PA_ERR_CUDA,
 *     that a launch failed.
 *   - Tensor arguments of the GPU entry points are DEVICE pointers owned by the
 *     caller, contiguous, 16-byte aligned, in the layouts stated below.  The kernel
 *     entry points never allocate, free or keep device memory; scratch space is
 *     passed in by the caller (see pa_decode_workspace_bytes).  The decode-step
 *     runtime (pa_decoder_*) is the exception: it owns the staging and scratch
 *     buffers it allocates when a batch is bound, and frees them when destroyed.
 *   - GPU work is enqueued on the caller's stream (a cudaStream_t passed as
 *     pa_stream_t; NULL = legacy default stream) and is asynchronous: no entry
 *     point synchronises, except pa_device_error_read.
 *   - Element types: PA_F32, PA_BF16, PA_F16.  q, out and both caches share one,
 *     except in the _fp8 entry points, whose caches hold PA_FP8_E4M3 codes.
 *   - Cache layout (K and V alike): [num_blocks, num_kv_heads, block_size, head_dim];
 *     so each (block, kv head) pair is one contiguous block_size*head_dim run.
 *     Slot s means block s / block_size, offset s % block_size.
 *   - Kernels check every block id and slot they dereference against num_blocks.
 *     An out-of-range index is skipped (never dereferenced) and recorded in a
 *     device error word; pa_device_error_read returns and clears it.
 *   - Allocator handles are host objects owned by the library; not thread-safe.
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
  PA_ERR_INVALID_ARG = 1,    /* bad pointer, size, dtype, alignment or workspace   */
  PA_ERR_NO_FREE_BLOCKS = 2, /* the pool cannot supply the blocks this call needs  */
  PA_ERR_UNKNOWN_SEQ = 3,    /* sequence id not present in the allocator            */
  PA_ERR_SEQ_EXISTS = 4,     /* sequence id already present                         */
  PA_ERR_BAD_INDEX = 5,      /* a kernel met an out-of-range block id / slot / len  */
  PA_ERR_CUDA = 6,           /* a CUDA runtime call or launch failed                */
  PA_ERR_UNSUPPORTED = 7,    /* valid but not built: head_dim / block_size / dtype  */
  PA_ERR_TOO_LARGE = 8       /* request exceeds a fixed built-in capacity           */
} pa_status;

typedef enum { PA_F32 = 0, PA_BF16 = 1, PA_F16 = 2, PA_FP8_E4M3 = 3 } pa_dtype;

typedef void* pa_stream_t; /* a cudaStream_t */

/* Bits of the device error word (pa_device_error_read). */
#define PA_DEVERR_SLOT 1u        /* reshape_and_cache: slot >= num_blocks*block_size */
#define PA_DEVERR_COPY_BLOCK 2u  /* copy_blocks: src or dst outside [0, num_blocks)  */
#define PA_DEVERR_TABLE 4u       /* decode: block-table entry outside [0, num_blocks)*/
#define PA_DEVERR_SEQ_LEN 8u     /* decode: seq_len < 0, > max_seq_len or > table    */
#define PA_DEVERR_TIMEOUT 16u    /* a bounded wait on an async copy gave up          */
#define PA_DEVERR_GROUP 32u      /* grouped decode: a sequence's own partitions start
                                    below first_part (those partitions were skipped)  */
#define PA_DEVERR_ORDER 64u      /* pa_decode: a seq_order entry outside [0, num_seqs)
                                    (that grid row was skipped)                       */
#define PA_DEVERR_SMEM 128u      /* grouped decode: a CTA's dynamic shared memory did
                                    not start 1024-byte aligned (the CTA did nothing) */

/* ------------------------------------------------------------------------- */
/* GPU entry points                                                           */
/* ------------------------------------------------------------------------- */

/*
 * pa_reshape_and_cache - write each new token's K and V into its slot.
 * ([BLOG] "Quick recap: the KV cache is per token, and it grows": each generated
 * token adds one key and one value; the slot comes from the block manager.)
 *
 *   key, value    [num_tokens, num_kv_heads, head_dim]           (read)
 *   k_cache, v_cache  cache layout above                          (written)
 *   slot_mapping  int64 [num_tokens]; slot of token t, or -1 = skip (read)
 * For every t with slot_mapping[t] >= 0: k_cache[slot/bs, h, slot%bs, :] =
 * key[t, h, :] for all h, and the same for V.  Bits are copied unchanged.
 * Slots must be distinct (two tokens with one slot race).  A slot >=
 * num_blocks*block_size is skipped and sets PA_DEVERR_SLOT.
 * head_dim*element size must be a multiple of 16 bytes.  num_tokens == 0 is a no-op.
 */
int pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int64_t num_blocks, int dtype,
                         pa_stream_t stream);

/*
 * pa_reshape_and_cache_fp8 - pa_reshape_and_cache into an fp8 (e4m3) cache ([BLOG]
 * "Where it bites": a quantized cache stacks with paging; the pages give no format,
 * so the reading here is one float32 scale per cache tensor).  key/value are
 * input_dtype (PA_F32, PA_BF16, PA_F16) [num_tokens, num_kv_heads, head_dim]; each
 * element x is stored as e4m3(float32(x) * (1.0f / scale)), rounded to nearest even,
 * saturated to +-448.  head_dim must be a multiple of 16.  Slots as in
 * pa_reshape_and_cache.  Scales must be positive and finite.
 */
int pa_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int64_t num_blocks, int input_dtype,
                             float k_scale, float v_scale, pa_stream_t stream);

/*
 * pa_copy_blocks - make the private copies of copy-on-write.
 * ([BLOG] "The bonus contiguous storage can't give you: sharing": a sequence that
 * writes into a shared block first copies it; [LAB] "Share matching prefixes".)
 *
 *   block_mapping_dev   int32 [num_pairs, 2] (src, dst) pairs on the device (read)
 *   block_mapping_host  the same pairs in host memory, used only to validate;
 *                       may be NULL to skip validation
 * Every dst block (all kv heads, all slots) of K and V becomes a copy of its src.
 * With block_mapping_host given, the call returns PA_ERR_INVALID_ARG unless every
 * id is in [0, num_blocks), no dst repeats and no dst is also a src (so the result
 * does not depend on the order the pairs run in).  A src may repeat.  The kernel
 * re-checks ids and skips (PA_DEVERR_COPY_BLOCK) any outside the pool.
 * num_pairs == 0 is a no-op.
 */
int pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* block_mapping_dev,
                   const int32_t* block_mapping_host, int num_pairs, int num_kv_heads,
                   int head_dim, int block_size, int64_t num_blocks, int dtype,
                   pa_stream_t stream);

/*
 * pa_swap_blocks - copy whole blocks between two caches, e.g. the device pool and a
 * host swap pool when a sequence is preempted and later resumed ([GLOSS] "pages can
 * be efficiently swapped or evicted ... spilling to CPU RAM"; [BLOG] "Where it bites":
 * a full pool swaps blocks out to CPU memory).
 *   dst_k, dst_v   destination cache [dst_num_blocks, num_kv_heads, block_size, head_dim]
 *   src_k, src_v   source cache      [src_num_blocks, ...]
 *   block_mapping  int32 [num_pairs, 2] (src block, dst block), device-reachable
 *   block_mapping_host  same pairs on the host for validation (nullable)
 * Each side may be device memory of the current device or page-locked host memory
 * (cudaHostAlloc / cudaMallocHost / cudaHostRegister; the kernel reaches it through
 * unified addressing).  Every pointer is checked with cudaPointerGetAttributes before
 * the launch; pageable or foreign memory gives PA_ERR_INVALID_ARG.  With the host
 * mapping given, ids must be in range and destinations distinct.  One kernel launch
 * copies all pairs (K and V); ids outside the pools are skipped (PA_DEVERR_COPY_BLOCK).
 */
int pa_swap_blocks(void* dst_k, void* dst_v, int64_t dst_num_blocks, const void* src_k,
                   const void* src_v, int64_t src_num_blocks, const int32_t* block_mapping,
                   const int32_t* block_mapping_host, int num_pairs, int num_kv_heads,
                   int head_dim, int block_size, int dtype, pa_stream_t stream);

/*
 * pa_decode_workspace_bytes - scratch bytes pa_decode_attention needs.
 * P = ceil(max_seq_len / partition_size) partitions per sequence; when P > 1 the
 * workspace holds float32 partial outputs [P, num_seqs, num_heads, head_dim] and
 * float32 maxima and exp-sums [P, num_seqs, num_heads] (the max is the one the
 * partition's weights were taken against; it may trail the true maximum logit by up
 * to 8 in base 2, and the merge uses each pair as a whole).  A kernel that computes
 * several consecutive partitions of a row may combine them itself and leave one
 * partial in the first one's slot, the others with exp-sum 0.  After the partials, one
 * int32 arrival counter per (sequence, head) row [num_seqs, num_heads], which the
 * grouped call clears itself before use.  The contents need no initialisation and
 * are not kept between calls.  Returns 0 when P <= 1 (no merge needed) and 0 for
 * invalid sizes.
 */
size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim, int max_seq_len,
                                 int partition_size);

/*
 * pa_decode_partition_size - a partition size for pa_decode_attention chosen from the
 * shape of its grid.  Host only; no GPU work.  (The pages fix no partitioning; the
 * split of long sequences and its size are this library's.)
 *   cache_dtype   PA_F32 / PA_BF16 / PA_F16, or PA_FP8_E4M3 for the fp8 entry point
 *   num_seqs, num_heads, num_kv_heads, head_dim, block_size   as for the decode call
 *   max_seq_len   the max_seq_len the decode call will be given
 *   num_sms       SMs of the GPU; 0 = ask the current device
 * Starting at 512 tokens, the size doubles while the partition grid keeps at least
 * 12 CTAs per SM (four waves of the three ~64 KiB CTAs an SM holds) that have tokens
 * to read, counting a sequence's partitions as if its length were spread uniformly
 * up to max_seq_len ((P + 1) / 2 of P partitions working) and stopping once one
 * partition covers max_seq_len.  Fewer, longer partitions write and merge less
 * partial state; enough CTAs keep every SM streaming.  The result is a power of two
 * times 512 (a multiple of every supported block size) and >= 512.  It does not
 * consider prefix groups, whose shared partitions want partitions shorter than the
 * shared prefix (pa_decode_attention_grouped).  Returns 0 for invalid arguments or
 * when num_sms is 0 and no device can be queried.
 */
int pa_decode_partition_size(int cache_dtype, int num_seqs, int num_heads, int num_kv_heads,
                             int head_dim, int block_size, int max_seq_len, int num_sms);

/*
 * pa_decode_attention - single-query (decode) attention over the paged cache.
 * ([BLOG] "The attention kernel has to read scattered blocks"; [LAB] "Keep pages in
 * order" and "Measure memory use across requests": the attention equation is
 * unchanged, only the K/V addressing goes through the block table; [BLOG] "Where it
 * bites": grouped-query attention, several query heads sharing one kv head.)
 *
 *   out           [num_seqs, num_heads, head_dim]                 (written)
 *   q             [num_seqs, num_heads, head_dim]                 (read)
 *   k_cache, v_cache  cache layout above                          (read)
 *   block_tables  int32 [num_seqs, max_blocks_per_seq]; row s lists the physical
 *                 blocks of sequence s in logical order; entries past
 *                 ceil(seq_lens[s]/block_size) are never read   (read)
 *   seq_lens      int32 [num_seqs]: cached tokens of each sequence, including the
 *                 token written this step                          (read)
 *   scale         logit scale (typically 1/sqrt(head_dim))
 *   block_size, num_kv_heads   as in the cache; num_heads % num_kv_heads == 0
 *   max_seq_len   host-side upper bound of seq_lens (sizes the grid and workspace
 *                 without a device-to-host read); a longer seq_len is skipped and
 *                 sets PA_DEVERR_SEQ_LEN
 *   partition_size  tokens per partition (multiple of block_size; 0 = 512).  A
 *                 sequence longer than one partition is split; the partitions are
 *                 merged by log-sum-exp weights in a second kernel.
 *   workspace     device scratch of at least pa_decode_workspace_bytes(...) bytes
 *                 (may be NULL when that is 0); contents need no initialisation.
 * For each sequence s and query head h (kv head g = h / (num_heads/num_kv_heads)):
 *   out[s,h,:] = sum_t softmax_t(scale * q[s,h,:] . K_t) V_t over the seq_lens[s]
 * cached tokens t, K_t/V_t read from block block_tables[s, t / block_size], offset
 * t % block_size, kv head g.  Accumulation is float32 and the softmax weights come
 * from the hardware base-2 exponential (relative error about 2^-22); out is rounded to
 * the cache dtype (round-to-nearest-even).  seq_lens[s] == 0 gives zeros.
 * Supported: head_dim in {64, 128, 256}; block_size in {4, 8, 16, 32}; tensor-core
 * path for num_heads/num_kv_heads a multiple of 8 with bf16/f16, head_dim 64/128/256
 * and block_size 16/32; other shapes use the CUDA-core path.
 */
int pa_decode_attention(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, const int32_t* seq_lens, float scale,
                        int block_size, int num_kv_heads, int num_seqs, int num_heads,
                        int head_dim, int max_blocks_per_seq, int64_t num_blocks,
                        int max_seq_len, int partition_size, int dtype, void* workspace,
                        size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_decode_attention_static_ws - pa_decode_attention without a caller-provided
 * workspace, for callers that are not allowed to allocate device memory: code running
 * inside a host program that owns and budgets every byte of the GPU's memory (a
 * serving runtime that reserves the card at start-up, a plug-in loaded into someone
 * else's process), loops that cannot afford the synchronisation and unbounded latency
 * of cudaMalloc, and deployments that forbid any allocation after initialisation.
 * (The pages have no counterpart: this entry point is an interface convenience.)
 *
 * Arguments, layouts and results are those of pa_decode_attention minus workspace and
 * workspace_bytes.  The partition scratch is a library-owned device array of
 * PA_STATIC_WORKSPACE_BYTES (16 MiB) that every GPU which loads the library holds until
 * the process exits.  A call whose pa_decode_workspace_bytes(...) exceeds that returns
 * PA_ERR_TOO_LARGE and does nothing; use pa_decode_attention with your own workspace
 * for such sizes.  The call allocates nothing (no cudaMalloc / cudaFree).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it; make that first
 *     call before any stream capture.
 *   - With CUDA's default lazy module loading, the array's 16 MiB are reserved on a
 *     device when the library's device code is first loaded there: at that first
 *     call at the latest (at context creation under CUDA_MODULE_LOADING=EAGER).  A
 *     caller that budgets device memory once at start-up should make one call per
 *     device during its initialisation, so that nothing is reserved later.
 *   - Every call on a device shares the one array.  The scratch needs no clearing (each
 *     call writes every entry it reads), but calls that overlap on the GPU - on
 *     different streams, or from different threads - race on it and must be ordered
 *     by the caller.
 */
#define PA_STATIC_WORKSPACE_BYTES (16u << 20)
int pa_decode_attention_static_ws(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables,
                                  const int32_t* seq_lens, float scale, int block_size,
                                  int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                                  int max_blocks_per_seq, int64_t num_blocks, int max_seq_len,
                                  int partition_size, int dtype, pa_stream_t stream);

/*
 * pa_decode_uses_tensor_cores - 1 if pa_decode_attention serves this shape with the
 * tensor-core (mma.sync) partition kernel, 0 if with the CUDA-core kernel.  Host
 * only; no GPU work.
 */
int pa_decode_uses_tensor_cores(int dtype, int num_heads, int num_kv_heads, int head_dim,
                                int block_size);

/*
 * pa_decode_attention_fp8 - pa_decode_attention over an fp8 (e4m3) cache written by
 * pa_reshape_and_cache_fp8: K_t = e4m3(k codes) * k_scale, V_t = e4m3(v codes) *
 * v_scale.  q and out are dtype (PA_BF16 or PA_F16); head_dim 128 or 256.  Groups of
 * 8 or 16 query heads per kv head with block_size 16/32 run on tensor cores (the codes
 * are loaded as MMA fragments and converted exactly to f16 in registers, q to f16, P
 * is f16); other shapes on CUDA cores, where the codes become f16 exactly and the
 * products are mixed-precision f16 x f16 -> float32 FMAs: q is carried as f16 (a bf16 q
 * times a power of two per head, exact apart from parts below 2^-24 of the head's
 * largest element) and the softmax weights of p.V are rounded to f16.  The cache is
 * half the bytes of a 16-bit one.  Codes 0x7F / 0xFF (NaN; written only for NaN
 * inputs) give unspecified outputs.
 */
int pa_decode_attention_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* seq_lens, float scale,
                            int block_size, int num_kv_heads, int num_seqs, int num_heads,
                            int head_dim, int max_blocks_per_seq, int64_t num_blocks,
                            int max_seq_len, int partition_size, int dtype, float k_scale,
                            float v_scale, void* workspace, size_t workspace_bytes,
                            pa_stream_t stream);

/*
 * pa_decode_attention_grouped - pa_decode_attention for a batch in which groups of
 * sequences share their leading blocks (prompt sharing / parallel samples forked
 * from one prefix: [GLOSS] prompt sharing and sampling algorithms; [BLOG] "The bonus
 * contiguous storage can't give you: sharing").  Same result as pa_decode_attention;
 * the whole partitions a group shares are read once for the group instead of once
 * per member: a tensor-core tile whose columns are the members' (query, head) pairs.
 *
 * Extra arguments (device int32 arrays, as filled by pa_build_prefix_groups and copied
 * to the device):
 *   prefix_parts   [num_seqs]  shared partitions of each sequence (0 = not grouped)
 *   chunk_members  [num_chunks, max_members]  batch positions of a chunk, -1 padded
 *   chunk_parts    [num_chunks]  shared partitions of the chunk
 *   max_members    1..16; max_chunk_parts = max(chunk_parts) (sizes the grid).
 * Contract: all members of a chunk map the chunk's first chunk_parts *
 * partition_size / block_size logical blocks to the same physical blocks (what
 * pa_build_prefix_groups guarantees); prefix_parts[i] equals its chunk's parts.
 * A sequence never has its last token's partition computed by the group, so every
 * grouped sequence is finished by a log-sum-exp merge of its partitions.  The call is
 * one grid: the groups' shared partitions first, then every sequence's own
 * partitions; the CTA that stores the last partial of a (sequence, kv head) merges
 * that sequence's heads itself (arrival counters in the workspace, cleared by a small
 * kernel launched just before the grid), so no merge kernel follows.
 * first_part: the lowest partition any sequence computes itself, min over s of
 * min(prefix_parts[s], (seq_lens[s]-1) / partition_size) (0 when any sequence has no
 * group); the sequences' own part of the grid starts there, so the partitions every
 * group covers launch no CTAs at all.  A sequence whose own partitions start lower is
 * reported (PA_DEVERR_GROUP) and those partitions are left out.  When the shape does not qualify
 * (f32 cache, block_size not 16/32, max_members * num_heads/num_kv_heads > 16, or a
 * single partition) the groups are ignored and the plain path runs.
 */
int pa_decode_attention_grouped(void* out, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* block_tables,
                                const int32_t* seq_lens, float scale, int block_size,
                                int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                                int max_blocks_per_seq, int64_t num_blocks, int max_seq_len,
                                int partition_size, int dtype, const int32_t* prefix_parts,
                                const int32_t* chunk_members, const int32_t* chunk_parts,
                                int num_chunks, int max_members, int max_chunk_parts,
                                int first_part, void* workspace, size_t workspace_bytes,
                                pa_stream_t stream);

/*
 * pa_decode - the decode call with every option in one argument block: the plain,
 * fp8 and grouped forms above, and the order in which the partition grid takes the
 * sequences.  Same results as those entry points.
 *   struct_size      sizeof(pa_decode_args_t)
 *   out ... workspace_bytes, stream   as for pa_decode_attention
 *   cache_dtype      dtype, or PA_FP8_E4M3 (then k_scale / v_scale as for
 *                    pa_decode_attention_fp8; ignored otherwise)
 *   seq_order        NULL, or device int32 [num_seqs], a permutation of the batch
 *                    positions: grid row y of the partition kernels serves sequence
 *                    seq_order[y].  Giving the longest sequences first lets their
 *                    long rows start early and the short ones fill the end (the
 *                    results do not depend on it).  An entry outside [0, num_seqs)
 *                    skips that row and sets PA_DEVERR_ORDER.
 *   prefix_parts ... first_part   the prefix-group arguments of
 *                    pa_decode_attention_grouped; num_chunks = 0 for none (not with an
 *                    fp8 cache).
 */
typedef struct {
  size_t struct_size;
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  float scale;
  int block_size, num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq;
  int64_t num_blocks;
  int max_seq_len, partition_size, dtype, cache_dtype;
  float k_scale, v_scale;
  const int32_t* seq_order;
  const int32_t* prefix_parts;
  const int32_t* chunk_members;
  const int32_t* chunk_parts;
  int num_chunks, max_members, max_chunk_parts, first_part;
  void* workspace;
  size_t workspace_bytes;
  pa_stream_t stream;
} pa_decode_args_t;
int pa_decode(const pa_decode_args_t* args);

/*
 * pa_device_error_read - synchronise the current device, then return (in *bits) and
 * clear the device error word that the kernels set on out-of-range indices or on
 * a bounded wait that gave up (PA_DEVERR_* bits; 0 = none).
 */
int pa_device_error_read(uint32_t* bits);

/*
 * pa_last_cuda_error - text of the last CUDA error an entry point met on this
 * thread (the reason behind a PA_ERR_CUDA), or "" if none.  Owned by the library.
 */
const char* pa_last_cuda_error(void);

/*
 * pa_selftest_bounded_wait - failure-detection check of the bounded waits.  Launches
 * one thread that waits, with the same bounded mbarrier wait as the decode kernels, on
 * an mbarrier that nothing ever completes.  After the bound (about one second of
 * %globaltimer, or 2^26 polls) the wait gives up, the kernel sets PA_DEVERR_TIMEOUT in
 * the device error word and returns, and the context stays usable.  Read the result
 * with pa_device_error_read.  (Not part of the pages' method: a diagnostic.)
 */
int pa_selftest_bounded_wait(pa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Host block allocator                                                       */
/* ------------------------------------------------------------------------- */
/*
 * The block manager of [BLOG] "PagedAttention: paging, borrowed from the operating
 * system" and "The bonus contiguous storage can't give you: sharing", and [LAB]
 * "Add pages as the request grows" / "Share matching prefixes":
 *   - one pool of num_blocks physical blocks of block_size token slots;
 *   - a sequence takes a new block only when its last block is full, so only its
 *     last block can have unused slots;
 *   - fork shares every block of a parent with a child (reference counts + 1);
 *   - copy-on-write: when the block the next token goes into is shared (count > 1)
 *     the writer gets a fresh block and a (src, dst) pair to copy with
 *     pa_copy_blocks before writing; after a full shared block only a new block is
 *     taken;
 *   - a freed sequence drops its counts; blocks that reach zero return to the pool.
 * Pool order: a LIFO stack whose successive pops return free_order[0],
 * free_order[1], ... (identity order when free_order is NULL); a block returned to
 * the pool goes on top; a freed sequence returns its blocks in logical order.
 * Every failing call leaves the allocator state unchanged.
 */
typedef struct pa_alloc pa_alloc_t;

typedef struct {
  int64_t num_blocks;        /* pool size                                        */
  int64_t block_size;        /* token slots per block                            */
  int64_t free_blocks;       /* blocks in the free pool                          */
  int64_t used_blocks;       /* blocks with reference count > 0                  */
  int64_t shared_blocks;     /* blocks with reference count > 1                  */
  int64_t total_refs;        /* sum of reference counts = block-table entries    */
  int64_t num_seqs;          /* live sequences                                   */
  int64_t logical_tokens;    /* sum of sequence lengths                          */
  int64_t allocated_slots;   /* used_blocks * block_size                         */
  int64_t tail_waste_slots;  /* sum over sequences of blocks*block_size - length */
  int64_t cow_copies;        /* copy-on-write pairs issued so far                */
  int64_t blocks_allocated;  /* blocks taken from the pool so far                */
  int64_t cached_blocks;     /* blocks registered in the prefix cache            */
  int64_t evictable_blocks;  /* cached blocks nobody references (reusable)       */
  int64_t cache_hits;        /* prompt blocks served from the prefix cache       */
  int64_t cache_evictions;   /* cached blocks evicted to serve a pop             */
} pa_stats_t;

/* Create a pool; free_order (host int32 [num_blocks], a permutation) or NULL. */
int pa_alloc_create(int64_t num_blocks, int block_size, const int32_t* free_order,
                    pa_alloc_t** out);
int pa_alloc_destroy(pa_alloc_t* a);

/* Admit seq_id with num_tokens cached tokens: ceil(num_tokens/block_size) blocks. */
int pa_seq_add(pa_alloc_t* a, int64_t seq_id, int64_t num_tokens);
/* Admit seq_id by its prompt's n token ids with automatic prefix caching: every
 * leading full block whose tokens - and whole prefix - match a cached block reuses
 * that block (count + 1); the remaining full blocks are fresh and registered in the
 * cache (the caller must write their K/V before anyone attends over them); a partial
 * last block is fresh and not registered.  *cached_tokens = tokens covered by reused
 * blocks (their K/V need not be computed again).  A cached block that nobody
 * references stays cached but evictable: pops take a free block first, else evict
 * the least recently released cached block.  A write into a cached block copies it
 * when shared and uncaches it otherwise. */
int pa_seq_add_prompt(pa_alloc_t* a, int64_t seq_id, const int32_t* token_ids, int64_t n,
                      int64_t* cached_tokens);
/* child shares all of parent's blocks and its length. */
int pa_seq_fork(pa_alloc_t* a, int64_t parent, int64_t child);
/* Room for one more token of seq_id: *slot receives its slot; *cow_src and *cow_dst the
 * copy to make first, or -1/-1.  Length grows by one. */
int pa_seq_append_slot(pa_alloc_t* a, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                       int32_t* cow_dst);
/* One append for each of seq_ids[0..n) in order, all or nothing.  slots[i] gets the
 * slot of seq_ids[i]; the copy pairs go to cow_pairs (int32 [n, 2] capacity) in
 * order, their count to *num_cow. */
int pa_seq_append_slots(pa_alloc_t* a, const int64_t* seq_ids, int n, int64_t* slots,
                        int32_t* cow_pairs, int* num_cow);
/* Shorten each seq_ids[i] to new_lens[i] (<= its length), e.g. to drop a rejected
 * draft token; blocks past ceil(new_len/block_size) drop a reference (released in
 * logical order).  No copy is ever needed.  Ids must be distinct.  All or nothing. */
int pa_seq_truncate(pa_alloc_t* a, const int64_t* seq_ids, const int64_t* new_lens, int n);
/* Move sequences from one pool to another (swap-out to a host pool, swap-in back):
 * each distinct block the moved sequences reference gets one fresh block in `to`
 * (first-appearance order: sequence order, then logical order), so blocks shared
 * inside the moved set stay shared; a block also used by sequences staying in `from`
 * becomes a private copy.  Lengths and logical order are kept; each moved reference in
 * `from` is dropped in the same order.  pairs_out (capacity cap pairs) receives the
 * (from_block, to_block) copies to make with pa_swap_blocks, *num_pairs their count.
 * Ids must be distinct, present in `from`, absent from `to`; block sizes must match.
 * All or nothing (PA_ERR_NO_FREE_BLOCKS when `to` is short). */
int pa_seqs_move(pa_alloc_t* from, pa_alloc_t* to, const int64_t* seq_ids, int n,
                 int32_t* pairs_out, int64_t cap, int64_t* num_pairs);
/* Release seq_id. */
int pa_seq_free(pa_alloc_t* a, int64_t seq_id);
int pa_seq_len(const pa_alloc_t* a, int64_t seq_id, int64_t* len);
/* Copy seq_id's block table (logical order) into out[0..cap); *n = its length. */
int pa_seq_blocks(const pa_alloc_t* a, int64_t seq_id, int32_t* out, int64_t cap,
                  int64_t* n);
/* Host int32 tables [num_seqs, max_blocks_per_seq] (rows padded with -1) and int32
 * seq_lens [num_seqs] for the listed sequences, ready to copy to the device. */
int pa_build_block_tables(const pa_alloc_t* a, const int64_t* seq_ids, int num_seqs,
                          int32_t* tables, int max_blocks_per_seq, int32_t* seq_lens);
/* Prefix groups for pa_decode_attention_grouped.  Among the listed sequences (batch
 * positions 0..num_seqs-1), those whose block tables begin with the same physical
 * block form a group (order of first appearance; at least two members).  Its common
 * table prefix, in blocks, gives parts = floor(common * block_size / partition_size)
 * whole partitions that every member shares; groups with parts == 0 are dropped.
 * Outputs (host buffers): prefix_parts[num_seqs] (the member's parts, 0 if none);
 * chunk_members[num_chunks * max_members] (each group split in order into chunks of at
 * most max_members positions, rows padded with -1; capacity num_seqs * max_members);
 * chunk_parts[num_chunks] (capacity num_seqs); *num_chunks; *max_chunk_parts. */
int pa_build_prefix_groups(const pa_alloc_t* a, const int64_t* seq_ids, int num_seqs,
                           int partition_size, int max_members, int32_t* prefix_parts,
                           int32_t* chunk_members, int32_t* chunk_parts, int* num_chunks,
                           int* max_chunk_parts);
int pa_block_refcount(const pa_alloc_t* a, int32_t block, int32_t* refcount);
/* Free blocks in the order the next pops return them; *n = how many. */
int pa_alloc_free_list(const pa_alloc_t* a, int32_t* out, int64_t cap, int64_t* n);
int pa_alloc_stats(const pa_alloc_t* a, pa_stats_t* stats);

/* ------------------------------------------------------------------------- */
/* Decode-step runtime                                                        */
/* ------------------------------------------------------------------------- */
/*
 * A pa_decoder runs decode steps of a bound batch of sequences, host side included,
 * in native code.  One step, in the order of [BLOG] "PagedAttention: paging, borrowed
 * from the operating system" and "The bonus contiguous storage can't give you:
 * sharing":
 *   1. (rolling batches) every sequence is truncated back to its length at bind time,
 *      so that a long run keeps decoding the same lengths;
 *   2. pa_seq_append_slots gives every sequence room for one more token: its slot,
 *      and a copy-on-write pair where that token's block is shared;
 *   3. slots, pairs, lengths and block tables (pa_build_block_tables) and, for
 *      batches that share prefixes, the prefix groups (pa_build_prefix_groups) are
 *      written into one of two page-locked staging sets and sent to the device with
 *      one copy on the decoder's copy stream; the caller's stream waits for it;
 *   4. pa_copy_blocks makes the copies (before the write: the token lands in the copy);
 *   5. pa_reshape_and_cache (or _fp8) writes the new tokens' K/V into their slots;
 *   6. pa_decode (the plain, fp8 or grouped form) attends over every cached token, the
 *      new one included; without prefix groups the grid takes the sequences longest
 *      first (an order sorted on the host each step and staged with the rest).
 * Steps 4-6 are enqueued on the caller's stream; the call returns without waiting
 * for the GPU.  Step k fills staging set k % 2 while the kernels of step k - 1 may
 * still read the other set; the host waits only before rewriting a set whose copy
 * has not finished.
 *
 * The decoder borrows the allocator (which must outlive it and must not be used
 * from another thread during a call) and the caches.  It owns its streams, events and
 * the page-locked host halves of the staging sets.  It allocates no device memory:
 * the caller passes one device buffer to pa_decoder_bind (its size from
 * pa_decoder_device_bytes), which holds the device halves of the two staging sets,
 * the decode workspace for the bound batch at full table capacity and the two device
 * sets of q / new K / new V / out for host-fed steps.  That buffer must stay
 * allocated, and be used by nothing else, until the decoder is destroyed or bound
 * again (both wait for the decoder's work in flight first).  Nothing is allocated
 * inside a step.  Not thread-safe.  Every call makes the decoder's device (current at
 * create) current for its duration.
 * Failures: every check that can refuse a step (a sequence at the table's capacity,
 * an unknown sequence, the pool out of blocks) runs before the block manager commits
 * the step, and leaves the state unchanged.  A CUDA call that fails after that commit
 * leaves the sequences one token longer than the device cache; the decoder then
 * refuses every further step with PA_ERR_CUDA until it is bound again.
 */
typedef struct pa_decoder pa_decoder_t;

typedef struct {
  size_t struct_size;      /* sizeof(pa_decoder_config_t)                          */
  void* k_cache;           /* device caches, layout above, caller-owned            */
  void* v_cache;
  int64_t num_blocks;      /* >= the allocator's pool                              */
  int num_kv_heads;
  int block_size;          /* the allocator's block size                           */
  int head_dim;
  int num_heads;           /* query heads, a multiple of num_kv_heads              */
  int dtype;               /* q, new K/V rows, out: PA_F32 / PA_BF16 / PA_F16      */
  int cache_dtype;         /* dtype, or PA_FP8_E4M3 with dtype PA_BF16 / PA_F16    */
  float scale;             /* logit scale                                          */
  float k_scale, v_scale;  /* fp8 per-tensor scales (ignored for 16/32-bit caches) */
  int max_blocks_per_seq;  /* block-table width: capacity per sequence in blocks   */
  int partition_size;      /* 0 = pa_decode_partition_size for the bound batch at
                              full table capacity; else a multiple of block_size   */
  int group_members;       /* prefix-group chunk size 0..16 (0 = no groups;
                              always 0 for fp8 caches)                              */
} pa_decoder_config_t;

typedef struct {
  size_t struct_size;      /* set by the caller: sizeof(pa_step_info_t)            */
  int num_cow;             /* copy-on-write pairs of the step                      */
  int max_seq_len;         /* longest sequence after the append                    */
  int partition_size;
  int num_chunks;          /* prefix-group chunks (0 = plain decode)               */
  int max_chunk_parts;
  int first_part;
  int kernels;             /* library kernels the step launched                    */
  /* Host views of the step's staging set (page-locked; valid until the step after
   * next): slots int64 [S], cow_pairs int32 [num_cow, 2], block_tables int32
   * [S, max_blocks_per_seq], seq_lens int32 [S]; S = the bound batch size. */
  const int64_t* slots;
  const int32_t* cow_pairs;
  const int32_t* block_tables;
  const int32_t* seq_lens;
} pa_step_info_t;

/* Checks the configuration (struct_size, pointers, sizes, dtypes) before any CUDA
 * call; then creates the decoder's streams and events on the current device. */
int pa_decoder_create(const pa_decoder_config_t* cfg, pa_alloc_t* alloc,
                      pa_decoder_t** out);
/* Waits for the decoder's work in flight, then frees everything it owns. */
int pa_decoder_destroy(pa_decoder_t* d);
/* Device bytes pa_decoder_bind needs for a batch of num_seqs sequences (staging sets,
 * workspace and host-I/O sets, each piece 256-byte aligned).  Host only, except that
 * the automatic partition size reads the device's SM count. */
int pa_decoder_device_bytes(const pa_decoder_t* d, int num_seqs, size_t* bytes);
/* Fix the batch (distinct ids present in the allocator, each shorter than the table
 * capacity) and lay its buffers out in the caller's device_buffer (256-byte aligned,
 * at least pa_decoder_device_bytes(num_seqs) bytes: else PA_ERR_INVALID_ARG and
 * nothing changes); rolling != 0 makes every step first roll the sequences back to
 * their current lengths.  Waits for the decoder's work in flight, then drops the
 * previous batch's buffers. */
int pa_decoder_bind(pa_decoder_t* d, const int64_t* seq_ids, int num_seqs, int rolling,
                    void* device_buffer, size_t device_bytes);
/* One step with DEVICE inputs: q [S, num_heads, head_dim], new_k / new_v
 * [S, num_kv_heads, head_dim] (row i is seq_ids[i]'s new token), out [S, num_heads,
 * head_dim], all dtype.  ev_begin / ev_end (cudaEvent_t or NULL) are recorded on the
 * stream around the attention call.  info (or NULL) receives the step's facts. */
int pa_decoder_step(pa_decoder_t* d, const void* q, const void* new_k, const void* new_v,
                    void* out, pa_stream_t stream, void* ev_begin, void* ev_end,
                    pa_step_info_t* info);
/* One step with HOST inputs and output (page-locked for the copies to overlap):
 * q, new_k, new_v are copied to the device on the decoder's input stream, the step
 * runs on `stream`, and out is copied back on its output stream.  Two device I/O
 * sets alternate, so a step's copies overlap the neighbouring steps' kernels.  The
 * call returns at once; *ticket (or NULL) names the step for pa_decoder_wait.  The
 * caller must not rewrite q / new_k / new_v or read out before that wait. */
int pa_decoder_step_host(pa_decoder_t* d, const void* q, const void* new_k,
                         const void* new_v, void* out, pa_stream_t stream, int64_t* ticket,
                         pa_step_info_t* info);
/* Block until the host-fed step `ticket` has written its output (and finished reading
 * its inputs). */
int pa_decoder_wait(pa_decoder_t* d, int64_t ticket);
/* Make `stream` wait for every outstanding read-back of host-fed steps. */
int pa_decoder_drain(pa_decoder_t* d, pa_stream_t stream);
/* Facts of the bound batch: the partition size in use, the workspace bytes and the
 * bytes of one staging set (the host-to-device copy of a step).  NULL outputs are
 * skipped. */
int pa_decoder_query(const pa_decoder_t* d, int* partition_size, size_t* workspace_bytes,
                     size_t* staging_bytes);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
