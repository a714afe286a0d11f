// Launch parameters and host entry points of the decode kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv.h"

namespace pkv {

struct DecodeParams {
  void* out;                    // [num_seqs][num_q_heads][head_dim], bf16 or fp32
  const void* q;                // same shape, bf16 or fp32
  const void* k_cache;          // [num_blocks][block_size][num_kv_heads][head_dim]
  const void* v_cache;
  const float* k_scale;         // [num_blocks][num_kv_heads][block_size] (INT8 only)
  const float* v_scale;
  const int32_t* block_tables;  // [num_seqs][max_blocks_per_seq]
  const int32_t* context_lens;  // [num_seqs]
  float* ws_o;                  // [num_seqs][num_q_heads][num_splits][head_dim]
  float* ws_lse;                // [num_seqs][num_q_heads][num_splits] (log2 domain)
  int* err_flag;                // may be null
  int max_blocks_per_seq;
  int num_seqs, num_q_heads, num_kv_heads, group;
  int block_size, log2_bs, num_blocks;
  int max_context_len;
  int chunk;       // tokens per split (multiple of 16)
  int num_splits;
  int t_start;     // first token the split kernels cover (0, or a shared prefix length)
  int ws_slots;    // partial results per (sequence, q head) in the workspace
  int ws_base;     // workspace slot of split 0 (lower slots: shared-prefix partials)
  int direct;      // 1: a single split writes `out` itself (no merge kernel)
  int phys_bytes;  // shared-memory bytes reserved for the block-table slice
  float scale_log2;  // softmax_scale * log2(e)
  int q_f32;
  int out_f32;
  // Fused append (pkv_paged_attention_decode_append): sequence s's new token,
  // written into its slot by the CTA that attends position context_lens[s] - 1
  // before that CTA reads the cache.  Null for a plain decode.
  const void* new_k = nullptr;             // [num_seqs][num_kv_heads][head_dim] bf16
  const void* new_v = nullptr;
  const int64_t* slot_mapping = nullptr;   // [num_seqs]
};

// Shared-prefix pass (prefix.cu): slices of the common prefix, all rows at once.
struct PrefixParams {
  int prefix_len;     // tokens at the start of every sequence held in shared blocks
  int pchunk;         // prefix tokens per slice (a multiple of kPrefixTokens)
  int prefix_splits;  // slices; slice i writes workspace slot i
  int rows;           // q rows per KV head: num_seqs * group
  int phys_bytes;     // shared-memory bytes for one slice's block-table entries
};
constexpr int kPrefixTokens = 64;  // tokens per shared-memory stage
// Partial rows the merge kernel loads per lane before it knows their weights
// (one memory round trip for up to this many partials per row).
constexpr int kMergeBatch = 16;
constexpr int kMaxPrefixChunk = 8192;  // prefix tokens per slice at most

cudaError_t launch_decode(const DecodeParams& p, pkv_dtype cache_dt, int head_dim,
                          cudaStream_t st);
// One-byte caches (INT8, FP8): the engine of decode_q8.cu, and how many of its
// CTAs fit one SM.
cudaError_t launch_decode_q8(const DecodeParams& p, pkv_dtype cache_dt, int head_dim,
                             cudaStream_t st);
int decode_q8_ctas_per_sm(pkv_dtype cache_dt, int head_dim);
// behind_decode: the pass is launched right after the suffix decode of the
// same call, with programmatic stream serialization (it may start while that
// decode's last CTAs run, and completes only after that decode).
cudaError_t launch_prefix(const DecodeParams& p, const PrefixParams& pp, int head_dim,
                          bool behind_decode, cudaStream_t st);
// CTAs of rows per KV head in the shared-prefix pass (128 / group sequences each).
int prefix_row_groups(int num_seqs, int group);
cudaError_t launch_merge(const DecodeParams& p, int head_dim, cudaStream_t st);
int decode_ctas_per_sm_hint(pkv_dtype cache_dt, int head_dim);

cudaError_t launch_append(const void* k, const void* v, const int64_t* slot_mapping,
                          int num_tokens, int num_kv_heads, int head_dim, pkv_dtype in_dt,
                          void* k_cache, void* v_cache, pkv_dtype cache_dt, int num_blocks,
                          int block_size, float* k_scale, float* v_scale, int* err_flag,
                          cudaStream_t st);

cudaError_t launch_copy(void* dst, const void* src, size_t bytes, int num_sms, cudaStream_t st);
cudaError_t launch_read(const void* src, size_t bytes, unsigned int* sink, int num_sms,
                        cudaStream_t st);

}  // namespace pkv
