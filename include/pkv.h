/*
 * pkv.h - C ABI of libpkv.so: paged-KV decode attention for NVIDIA B200 (sm_100a).
 *
 * The problem these calls solve is the one stated on three pages about KV-cache
 * memory management:
 *   [mlqm]   "LLM推理显存优化KV Cache管理3大策略实测节省60%显存开销" (mlqm.cn/news/267625)
 *   [gpuyard]"生产级 LLM 推理的 KV 缓存优化" (GPUYard repost on feinterview.poetries.top)
 *   [yunthe] "大模型推理加速实战：KV Cache内存优化与PagedAttention分页管理方案" (yunthe.com)
 *
 * Memory layout (all device buffers, row-major, densely packed):
 *   cache  k_cache, v_cache : [num_blocks][block_size][num_kv_heads][head_dim]
 *          One physical block holds block_size token rows of all KV heads
 *          ([mlqm] §2, the Block class: k_data/v_data of block_size x hidden).
 *   scales k_scale, v_scale : fp32 [num_blocks][num_kv_heads][block_size]
 *          (INT8 and FP8 caches only; one scale per token per head, [mlqm] §4).
 *   slot   physical_block * block_size + offset_in_block.
 *   table  block_tables     : int32 [num_seqs][max_blocks_per_seq]; entry j is
 *          the physical block of logical block j ([yunthe], PagedAttention
 *          section, the block_table example; [mlqm] §2 BlockTable).
 *
 * Calls:
 *   append           pkv_kv_cache_append (bf16/fp32 copy, INT8/FP8 quantising)
 *   decode           pkv_paged_attention_decode, pkv_decode_num_splits,
 *                    pkv_workspace_size, pkv_paged_attention_decode_noalloc
 *   one-launch step  pkv_paged_attention_decode_append (append inside decode)
 *   shared prefix    pkv_paged_attention_decode_shared_prefix[_append],
 *                    pkv_shared_prefix_workspace_size, pkv_shared_prefix_plan
 *   block manager    pkv_bm_* (host bookkeeping: blocks, ref counts, fork,
 *                    copy-on-write, swap), pkv_copy_blocks (block copies)
 *   misc             pkv_copy, pkv_read, pkv_strerror, pkv_version
 *
 * Conventions shared by every call:
 *   - The caller allocates and owns every device buffer; the GPU calls keep no
 *     state between calls, allocate nothing and never synchronise.  (Two
 *     exceptions, each described at its call: the host block manager objects
 *     of pkv_bm_create, and the fixed device scratch behind
 *     pkv_paged_attention_decode_noalloc.)
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and targets the current CUDA device.
 *   - Argument errors return a negative pkv_status before anything is launched.
 *   - Data errors found on the device (bad block id, bad slot, context length
 *     out of range) are OR-ed as PKV_FLAG_* bits into *err_flag (a device int,
 *     may be NULL); the offending token/row is skipped, the kernel never traps.
 *   - Device pointers must be 16-byte aligned unless a call states otherwise;
 *     int32 arrays (block tables, context lengths) and err_flag need 4 bytes,
 *     int64 slot arrays 8.  A misaligned pointer returns PKV_ERR_ALIGN.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* pkv_stream_t; /* identical to cudaStream_t */

/* PKV_FP8: E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * largest finite value 448) with one fp32 scale per token per head, like PKV_I8. */
typedef enum { PKV_F32 = 0, PKV_BF16 = 1, PKV_I8 = 2, PKV_FP8 = 3 } pkv_dtype;

typedef enum {
  PKV_OK = 0,
  PKV_ERR_ARG = -1,         /* null pointer, negative size, n_q % n_kv != 0 */
  PKV_ERR_DTYPE = -2,       /* unsupported dtype combination */
  PKV_ERR_SHAPE = -3,       /* head_dim / block_size / group outside the supported set */
  PKV_ERR_UNSUPPORTED = -4, /* no kernel for this configuration */
  PKV_ERR_WORKSPACE = -5,   /* split-K needs a workspace of pkv_workspace_size() bytes */
  PKV_ERR_CUDA = -6,        /* a CUDA runtime call or launch failed */
  PKV_ERR_ALIGN = -7,       /* a device pointer is not aligned as its call requires */
  PKV_ERR_SCRATCH_LIMIT = -8, /* split-K scratch would exceed PKV_NOALLOC_SCRATCH_BYTES */
  PKV_ERR_NO_BLOCKS = -9      /* the block pool cannot supply the blocks an operation needs */
} pkv_status;

/* Bits written into *err_flag by the kernels. */
#define PKV_FLAG_BAD_BLOCK 1   /* block table entry outside [0, num_blocks): block skipped */
#define PKV_FLAG_BAD_SLOT 2    /* slot >= num_blocks * block_size: token not written */
#define PKV_FLAG_CTX_RANGE 4   /* context_len > max_blocks_per_seq * block_size or
                                  > max_context_len: clamped */
#define PKV_FLAG_NEG_CTX 8     /* negative context_len: treated as 0 */
#define PKV_FLAG_TIMEOUT 16    /* a kernel's bounded wait on its own tensor-core work gave up:
                                  its outputs are not valid (should never be seen) */

/* Supported sets: head_dim in {64, 128}; block_size a power of two in [8, 256];
 * group = num_q_heads / num_kv_heads in [1, 16]. */

/*
 * pkv_kv_cache_append - write each new token's K and V into its cache slot.
 *
 * Defined by [yunthe] (KV-cache overhead section: every generated token's
 * key/value is written into the KV cache) and [mlqm] §2 (block rows).  Token t
 * with slot s = slot_mapping[t] goes to block s / block_size, row
 * s % block_size; s < 0 skips the token (padding).  With cache_dt == PKV_I8 each
 * (token, head) row of head_dim values is quantised as in [mlqm] §4
 * (quantize_tensor): scale = 127 / max|x| over head_dim and code =
 * clamp(rint(x * scale), -128, 127), all in fp32, round-half-to-even, no fused
 * multiply-add; an all-zero row stores codes 0 and scale 1.  The scale goes to
 * k_scale/v_scale[block][head][row].  With cache_dt == PKV_FP8 (the pages'
 * --kv-cache-dtype fp8: [gpuyard] serving flags, [yunthe] KV quantisation) the
 * same per-row rule uses scale = 448 / max|x| and code = E4M3(x * scale),
 * rounded to nearest even and saturated to +-448, in fp32.
 *
 *   k, v          device, [num_tokens][num_kv_heads][head_dim], dtype in_dt
 *                 (PKV_F32 or PKV_BF16), contiguous.  Read only.
 *   slot_mapping  device int64 [num_tokens], 8-byte aligned.
 *   k_cache, v_cache  device, cache layout above, dtype cache_dt (== in_dt, PKV_I8
 *                 or PKV_FP8).
 *   k_scale, v_scale  device fp32 scale arrays; required iff cache_dt is PKV_I8 or
 *                 PKV_FP8 (4-byte alignment suffices for this call).
 *   err_flag      device int or NULL (PKV_FLAG_BAD_SLOT).
 * Two tokens with the same slot race (last writer wins, unspecified).
 */
int pkv_kv_cache_append(const void* k, const void* v, const int64_t* slot_mapping,
                        int num_tokens, int num_kv_heads, int head_dim, pkv_dtype in_dt,
                        void* k_cache, void* v_cache, pkv_dtype cache_dt, int num_blocks,
                        int block_size, float* k_scale, float* v_scale, int* err_flag,
                        pkv_stream_t stream);

/*
 * pkv_decode_num_splits - the number of context splits (split-K partitions)
 * pkv_paged_attention_decode picks when given num_splits = 0, for the current
 * device.  Always >= 1.  Returns a negative pkv_status on bad arguments.
 */
int pkv_decode_num_splits(int num_seqs, int num_kv_heads, int head_dim, int max_context_len,
                          pkv_dtype cache_dt);

/*
 * pkv_workspace_size - bytes of device workspace pkv_paged_attention_decode
 * needs for this shape with `num_splits` splits (0 = the automatic choice).
 * 0 when one split suffices (no workspace needed).
 */
size_t pkv_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                          int max_context_len, pkv_dtype cache_dt, int num_splits);

/*
 * pkv_paged_attention_decode - one decode step of attention over a paged cache.
 *
 * Defined by [yunthe], PagedAttention section: look up each token's physical
 * block through the block table, stitch the scattered K/V together and run
 * standard attention; GQA grouping from [mlqm] §3 (q head h uses KV head
 * h / (num_q_heads / num_kv_heads)).  For sequence s with c = context_lens[s]:
 *     out[s][h] = sum_t softmax_t(softmax_scale * <q[s][h], K_s[t]>) V_s[t],
 *     K_s[t] = k_cache[block_tables[s][t / block_size]][t % block_size][h / group]
 * over 0 <= t < c (c = 0 gives zeros).  INT8 and FP8 caches are dequantised as
 * value(code) / scale on load.  Long contexts are cut into num_splits splits whose
 * partial results are merged exactly through their log-sum-exp.
 *
 *   out           device [num_seqs][num_q_heads][head_dim], dtype q_dt.  Written.
 *   q             device [num_seqs][num_q_heads][head_dim], dtype q_dt:
 *                 PKV_BF16 for BF16/I8/FP8 caches; PKV_F32 or PKV_BF16 for F32 caches.
 *   k_cache, v_cache, k_scale, v_scale  as above (scales only for PKV_I8 and
 *                 PKV_FP8; the scale arrays must be 16-byte aligned here).
 *   block_tables  device int32 [num_seqs][max_blocks_per_seq]; entries past the
 *                 sequence's last block are never read.
 *   context_lens  device int32 [num_seqs].
 *   max_context_len  host-side upper bound of context_lens (sizes the splits).
 *   softmax_scale usually 1/sqrt(head_dim).
 *   workspace     device scratch of >= pkv_workspace_size(...) bytes (may be NULL
 *                 when that size is 0).  Overwritten; not read before written.
 *   num_splits    0 = automatic, else the number of splits to use.
 *   err_flag      device int or NULL (PKV_FLAG_BAD_BLOCK, _CTX_RANGE, _NEG_CTX).
 * Output for a sequence with a bad block id covers its remaining tokens only.
 */
int pkv_paged_attention_decode(void* out, const void* q, pkv_dtype q_dt, const void* k_cache,
                               const void* v_cache, pkv_dtype cache_dt, const float* k_scale,
                               const float* v_scale, const int32_t* block_tables,
                               int max_blocks_per_seq, const int32_t* context_lens,
                               int max_context_len, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               float softmax_scale, void* workspace, size_t workspace_bytes,
                               int num_splits, int* err_flag, pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_append - one decode step in one call: each
 * sequence's new token is appended ([yunthe], KV-cache overhead section: every
 * generated token's K/V goes into the cache; §4 of [mlqm] for the quantised
 * rows) and the sequence then attends over its context_lens tokens, new token
 * included.  The result, cache contents included, is that of
 * pkv_kv_cache_append(k, v, slot_mapping, num_seqs tokens) followed by
 * pkv_paged_attention_decode, provided slot_mapping[s] is the slot the block
 * table gives position context_lens[s] - 1 of sequence s.  The CTA that
 * attends that position writes the token's rows of its KV head first, so no
 * separate append launch is needed.
 *
 * Arguments as for pkv_paged_attention_decode, plus:
 *   k, v          device bf16 [num_seqs][num_kv_heads][head_dim], contiguous,
 *                 16-byte aligned: the new token of each sequence.
 *   slot_mapping  device int64 [num_seqs], 8-byte aligned.  A negative slot
 *                 writes nothing.  A slot that is not the one of position
 *                 context_lens[s] - 1 (or outside the pool) writes nothing and
 *                 sets PKV_FLAG_BAD_SLOT.
 *   in_dt         PKV_BF16 (k, v and q).
 *   k_cache, v_cache, k_scale, v_scale  written (the new rows and scales).
 * Supported: cache_dt PKV_BF16, PKV_I8 or PKV_FP8 (PKV_F32:
 * PKV_ERR_UNSUPPORTED; use the two calls).
 */
int pkv_paged_attention_decode_append(void* out, const void* q, const void* k, const void* v,
                                      const int64_t* slot_mapping, pkv_dtype in_dt,
                                      void* k_cache, void* v_cache, pkv_dtype cache_dt,
                                      float* k_scale, float* v_scale,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* context_lens, int max_context_len,
                                      int num_seqs, int num_q_heads, int num_kv_heads,
                                      int head_dim, int block_size, int num_blocks,
                                      float softmax_scale, void* workspace,
                                      size_t workspace_bytes, int num_splits, int* err_flag,
                                      pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_shared_prefix - pkv_paged_attention_decode for a
 * batch whose sequences all begin with the same `prefix_len` tokens stored in
 * the same physical blocks (prefix caching: "生产级 LLM 推理的 KV 缓存优化"
 * (GPUYard), serving flags, --enable-prefix-caching; shared blocks with a
 * ref_count: [mlqm] §2).  The result is the same attention as
 * pkv_paged_attention_decode; only the order of the work differs: the shared
 * blocks are read once per KV head for all sequences (a dense q-rows x tokens
 * contraction), each sequence's remaining tokens are attended separately, and
 * the partials are merged through their log-sum-exp.
 *
 * Arguments as for pkv_paged_attention_decode, plus:
 *   prefix_len    host int, a multiple of block_size, <= max_blocks_per_seq *
 *                 block_size.  The prefix blocks are read from sequence 0's
 *                 block table; every sequence's table must hold the same
 *                 entries there (sequences shorter than prefix_len attend to
 *                 their first context_lens tokens only).  0 = plain decode.
 *   workspace     >= pkv_shared_prefix_workspace_size(...) bytes (always needed
 *                 when prefix_len > 0).
 * Supported: cache_dt == PKV_BF16 (others: PKV_ERR_UNSUPPORTED), q_dt == PKV_BF16.
 */
size_t pkv_shared_prefix_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                        int head_dim, int max_context_len, int prefix_len,
                                        pkv_dtype cache_dt, int num_splits);

/*
 * pkv_shared_prefix_plan - how a shared-prefix call with these sizes divides
 * its work (host only, launches nothing).  *prefix_slices receives the number
 * of slices of the shared tokens (one prefix-pass partial each), and
 * *suffix_splits the number of splits of each sequence's remaining tokens:
 * num_splits itself, or the automatic choice when num_splits == 0.  That
 * choice differs from pkv_decode_num_splits of the suffix length: the prefix
 * pass runs beside the suffix decode and fills its last wave, so the suffix is
 * not split to fill it.  Either output may be NULL.  Returns PKV_OK, or
 * PKV_ERR_ARG (a size out of range, prefix_len <= 0, num_q_heads not a
 * multiple of num_kv_heads).
 */
int pkv_shared_prefix_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                           int max_context_len, int prefix_len, pkv_dtype cache_dt,
                           int num_splits, int* prefix_slices, int* suffix_splits);
int pkv_paged_attention_decode_shared_prefix(
    void* out, const void* q, pkv_dtype q_dt, const void* k_cache, const void* v_cache,
    pkv_dtype cache_dt, const float* k_scale, const float* v_scale, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* context_lens, int max_context_len, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
    float softmax_scale, int prefix_len, void* workspace, size_t workspace_bytes, int num_splits,
    int* err_flag, pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_shared_prefix_append - the shared-prefix decode
 * with each sequence's new token appended in the same call, by the suffix
 * decode kernel (as in pkv_paged_attention_decode_append).  The result, cache
 * included, is that of pkv_kv_cache_append followed by
 * pkv_paged_attention_decode_shared_prefix, provided slot_mapping[s] is the
 * slot of position context_lens[s] - 1 and that position lies past the shared
 * prefix (>= prefix_len); a token inside the shared blocks is not written and
 * sets PKV_FLAG_BAD_SLOT (shared blocks are not written through this call).
 * Arguments as for pkv_paged_attention_decode_shared_prefix, plus k, v
 * (device bf16 [num_seqs][num_kv_heads][head_dim], 16-byte aligned) and
 * slot_mapping (device int64 [num_seqs], 8-byte aligned; negative: nothing
 * written).  Supported: cache_dt PKV_BF16, in_dt PKV_BF16.
 */
int pkv_paged_attention_decode_shared_prefix_append(
    void* out, const void* q, const void* k, const void* v, const int64_t* slot_mapping,
    pkv_dtype in_dt, void* k_cache, void* v_cache, pkv_dtype cache_dt,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
    int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int num_blocks, float softmax_scale, int prefix_len, void* workspace,
    size_t workspace_bytes, int num_splits, int* err_flag, pkv_stream_t stream);

/*
 * pkv_copy - device-to-device copy of `bytes` bytes (a multiple of 16) with a
 * streaming kernel; used to measure the attainable HBM bandwidth in the same
 * process as the attention kernels.  Not part of the attention path.
 */
int pkv_copy(void* dst, const void* src, size_t bytes, pkv_stream_t stream);

/*
 * pkv_read - streaming read of `bytes` bytes (a multiple of 16) at `src`
 * (device, 16-byte aligned), folded by XOR into the device word *sink (4-byte
 * aligned; the call XORs into it, so its value only keeps the loads alive).
 * Used to measure the attainable HBM read bandwidth in the same process as the
 * attention kernels, and, over a buffer larger than the L2, to flush the L2
 * between timed calls: its loads allocate in L2 and write nothing, so no dirty
 * line is left for the next call to write back.  Not part of the attention
 * path.  Returns PKV_ERR_ARG for a null pointer or a size not a multiple of 16.
 */
int pkv_read(const void* src, size_t bytes, unsigned int* sink, pkv_stream_t stream);

/* Bytes of the fixed device scratch behind pkv_paged_attention_decode_noalloc. */
#define PKV_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * pkv_paged_attention_decode_noalloc - pkv_paged_attention_decode for callers
 * that cannot allocate device memory.  The pages have no counterpart for this
 * call; it exists for callers such as code embedded in a host runtime that owns
 * every device allocation and gives its plugins no allocator or workspace.
 *
 * Arguments, layouts and results are those of pkv_paged_attention_decode minus
 * `workspace` and `workspace_bytes`: the split-K scratch lives in one fixed
 * device array of PKV_NOALLOC_SCRATCH_BYTES (16 MiB) inside the library, held
 * on every GPU that loads the library until the process exits.
 *   - Returns PKV_ERR_SCRATCH_LIMIT, before any launch, when the scratch the
 *     call needs (pkv_workspace_size for the same shape and num_splits) is
 *     larger than that array.
 *   - Every call shares the array: calls whose kernels overlap on the GPU
 *     (e.g. on different streams) race and must be serialised by the caller.
 *     Nothing in the array has to start at zero.
 *   - The first call in each CUDA context (normally once per device) looks
 *     up the array's device address with that device current and caches it
 *     with the context's unique id; a call in a new context (for example after
 *     cudaDeviceReset) looks it up again rather than reuse a stale address.
 *   - The driver reserves the array's 16 MiB when it loads the module that
 *     holds it; with lazy module loading (the CUDA default) that is this
 *     first call, which can then fail with PKV_ERR_CUDA if the device has no
 *     16 MiB left.  Make the first call at start-up, before any stream capture.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
int pkv_paged_attention_decode_noalloc(void* out, const void* q, pkv_dtype q_dt,
                                       const void* k_cache, const void* v_cache,
                                       pkv_dtype cache_dt, const float* k_scale,
                                       const float* v_scale, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* context_lens,
                                       int max_context_len, int num_seqs, int num_q_heads,
                                       int num_kv_heads, int head_dim, int block_size,
                                       int num_blocks, float softmax_scale, int num_splits,
                                       int* err_flag, pkv_stream_t stream);

/*
 * Block manager (host) - the pages' block bookkeeping ([mlqm] §2: fixed-size
 * blocks, a block table from logical to physical blocks, Block.ref_count;
 * [yunthe], PagedAttention section: blocks allocated on demand, reclaimed when
 * a sequence ends; its deployment parameters: swap_space moves inactive KV to
 * CPU memory).  A manager owns the ids of one pool of num_blocks blocks
 * (device or host); the caller owns the memory and moves data with
 * pkv_copy_blocks.  Blocks come off a free list (block 0 first, freed blocks
 * reused last-in first-out).  Every call is atomic (PKV_ERR_NO_BLOCKS leaves
 * the manager unchanged) and calls on one manager are serialised by a mutex.
 * Sequence ids are caller-chosen 64-bit keys.
 */
typedef struct pkv_block_manager pkv_block_manager;
int pkv_bm_create(int num_blocks, int block_size, pkv_block_manager** out);
void pkv_bm_destroy(pkv_block_manager* m);
/* free blocks; references of a block (0 = free) */
int pkv_bm_num_free(pkv_block_manager* m);
int pkv_bm_ref_count(pkv_block_manager* m, int32_t block);
/* a new empty sequence */
int pkv_bm_add_sequence(pkv_block_manager* m, int64_t seq_id);
/* child shares every block of parent (references + 1) and its length */
int pkv_bm_fork(pkv_block_manager* m, int64_t parent, int64_t child);
/* blocks pkv_bm_reserve would take for num_tokens more tokens (>= 0) */
int pkv_bm_blocks_needed(pkv_block_manager* m, int64_t seq_id, int num_tokens);
/*
 * Reserves the slots of the sequence's next num_tokens tokens (slots_out[i] =
 * block * block_size + offset, ready for pkv_kv_cache_append), allocating a
 * block at each block boundary.  If the sequence's last block is shared and
 * partially filled it is first replaced by a private block (copy-on-write):
 * *num_cow = 1 and cow_pair_out[0..1] = (shared block, new block) - copy it
 * with pkv_copy_blocks before appending.  Otherwise *num_cow = 0.
 */
int pkv_bm_reserve(pkv_block_manager* m, int64_t seq_id, int num_tokens, int64_t* slots_out,
                   int32_t* cow_pair_out, int* num_cow);
/* drops the sequence; blocks whose references reach 0 return to the free list */
int pkv_bm_free(pkv_block_manager* m, int64_t seq_id);
int pkv_bm_seq_len(pkv_block_manager* m, int64_t seq_id, int64_t* len_out, int* num_blocks_out);
/* dense block tables [num_seqs][max_blocks_per_seq] (padding -1) and lengths */
int pkv_bm_block_tables(pkv_block_manager* m, const int64_t* seq_ids, int num_seqs,
                        int max_blocks_per_seq, int32_t* tables_out, int32_t* lens_out);
/*
 * Moves a sequence between a device-pool manager and a host-pool manager (same
 * block_size): fresh blocks are taken in the destination, the source blocks
 * are released, and pairs_out[2i], pairs_out[2i+1] = (source block, destination
 * block) for each of its *num_pairs blocks, in table order - pass them to
 * pkv_copy_blocks.  A block the sequence shared with others stays with them.
 */
int pkv_bm_swap_out(pkv_block_manager* device, pkv_block_manager* host, int64_t seq_id,
                    int32_t* pairs_out, int capacity, int* num_pairs);
int pkv_bm_swap_in(pkv_block_manager* host, pkv_block_manager* device, int64_t seq_id,
                   int32_t* pairs_out, int capacity, int* num_pairs);

/*
 * pkv_copy_blocks - copies whole blocks: for each pair i, block pairs[2i] of the
 * source pool goes to block pairs[2i+1] of the destination pool, K and V (and
 * the per-token scales when scale_bytes_per_block > 0).  Pools are laid out as
 * the cache ([num_blocks][block_bytes]) and may be device memory or
 * page-locked host memory the device can address (swap).  `pairs` must be
 * device-accessible (int32 [num_pairs][2]).  Out-of-range ids set
 * PKV_FLAG_BAD_BLOCK and skip the pair.  block_bytes and scale_bytes_per_block
 * are multiples of 16; pointers 16-byte aligned.  Source and destination
 * blocks must not overlap.
 */
int pkv_copy_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                    size_t block_bytes, int dst_num_blocks, int src_num_blocks, float* dst_k_scale,
                    float* dst_v_scale, const float* src_k_scale, const float* src_v_scale,
                    size_t scale_bytes_per_block, const int32_t* pairs, int num_pairs,
                    int* err_flag, pkv_stream_t stream);

/* Human-readable text for a pkv_status. */
const char* pkv_strerror(int status);

/* ABI version: (major << 16) | minor. */
int pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
