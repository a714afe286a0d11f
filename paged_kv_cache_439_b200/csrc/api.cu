// C ABI of libpkv.so: argument validation, split planning, launches.
// The declarations and their contracts are in include/pkv.h.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "decode.cuh"
#include "pkv.h"

namespace {

// Prefix slices are planned for about this many CTAs of the shared-prefix
// pass per 100 SMs (over KV heads and row groups).
#ifndef PKV_PREFIX_CTAS_PER_100_SMS
#define PKV_PREFIX_CTAS_PER_100_SMS 200
#endif

constexpr int kMaxChunk = 8192;   // tokens per split (bounds the block-table slice in smem)
constexpr int kMinChunk = 256;    // below this a split costs more than it balances
constexpr int kTile = 16;         // tokens per tile of the decode kernels
constexpr int kCtasPerSlot = 4;   // target CTAs per resident-CTA slot of the device

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

int log2i(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// Smallest number of splits allowed and the automatic choice.
int min_splits(int max_ctx) { return max_ctx <= 0 ? 1 : (max_ctx + kMaxChunk - 1) / kMaxChunk; }

// Automatic split count.  With U = num_seqs * num_kv_heads (sequence, head)
// units and R CTAs resident on the device at once:
//  * U >= R / 2: every unit already has a CTA in the first wave, so splitting
//    only adds partial results to merge.  Keep S = 1 unless the last wave would
//    run under half full with fewer than two waves in total, then take the
//    smallest S that fixes that.
//  * U < R / 2 (few, long sequences): cut the context so that about
//    kCtasPerSlot CTAs per resident slot exist, which also evens out unequal
//    context lengths; no split shorter than kMinChunk tokens.  Among the
//    counts from half to twice that target, take the smallest whose U * S
//    CTAs fill their last wave at least 90% (equal-length contexts), else the
//    best-filled one: 128 units on 444 slots take S = 10 (2.9 waves) rather
//    than 14 (4.04 waves, the fifth nearly empty).
//  * beside_prefix (the suffix of a shared-prefix call): the prefix pass is
//    launched behind the suffix decode and its CTAs take the slots that the
//    decode's last wave leaves free, so with U >= R / 2 the suffix keeps S at
//    its minimum instead of splitting to fill that wave.
int auto_splits(int num_seqs, int num_kv_heads, int head_dim, int max_ctx, pkv_dtype cache_dt,
                bool beside_prefix = false) {
  if (max_ctx <= 0 || num_seqs <= 0) return 1;
  const long long units = (long long)num_seqs * num_kv_heads;
  const long long slots = (long long)sm_count() * pkv::decode_ctas_per_sm_hint(cache_dt, head_dim);
  const int lo = min_splits(max_ctx);
  const int hi = (max_ctx + kMinChunk - 1) / kMinChunk;
  long long want;
  if (2 * units >= slots && beside_prefix) {
    want = lo;
  } else if (2 * units >= slots) {
    want = 1;
    for (int s = 1; s <= 8; ++s) {
      const long long ctas = units * s;
      const long long full_waves = ctas / slots, rest = ctas % slots;
      want = s;
      if (full_waves >= 2 || rest == 0 || 2 * rest >= slots) break;
    }
  } else {
    const long long target = (kCtasPerSlot * slots + units - 1) / units;
    long long best = target;
    double best_fill = -1.0;
    for (long long s = (target + 1) / 2; s <= 2 * target; ++s) {
      if (s < lo || s > hi) continue;
      const long long ctas = units * s;
      const long long waves = (ctas + slots - 1) / slots;
      const double fill = (double)ctas / (double)(waves * slots);
      if (fill >= 0.9) {
        best = s;
        break;
      }
      if (fill > best_fill) {
        best_fill = fill;
        best = s;
      }
    }
    want = best;
  }
  if (want > hi) want = hi;
  if (want < lo) want = lo;
  return (int)want;
}

// Normalises a split count: chunk = 16-aligned ceil(max_ctx / s), s = ceil(max_ctx / chunk).
void plan(int max_ctx, int s_req, int* s_out, int* chunk_out) {
  if (max_ctx <= 0) {
    *s_out = 1;
    *chunk_out = kTile;
    return;
  }
  int chunk = round_up((max_ctx + s_req - 1) / s_req, kTile);
  *chunk_out = chunk;
  *s_out = (max_ctx + chunk - 1) / chunk;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

size_t ws_bytes(int num_seqs, int num_q_heads, int head_dim, int splits) {
  if (splits <= 1) return 0;
  const size_t rows = (size_t)num_seqs * num_q_heads * splits;
  return align256(rows * head_dim * sizeof(float)) + align256(rows * sizeof(float));
}

int map_cuda(cudaError_t e) { return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA; }

// Shared-prefix plan: the suffix splits of the remaining context, then the
// prefix slices: about PKV_PREFIX_CTAS_PER_100_SMS CTAs per 100 SMs over KV
// heads and row groups, and no more than leave the slices and splits of a row
// within the merge kernel's one-round-trip batch.
struct PrefixPlan {
  int ps, pchunk;      // prefix slices and their length
  int splits, chunk;   // suffix splits
  int slots;           // workspace partials per (sequence, q head)
  size_t ws;           // workspace bytes
};

PrefixPlan plan_prefix(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                       int max_ctx, int prefix_len, pkv_dtype cache_dt, int num_splits) {
  PrefixPlan pl;
  const long long rg = pkv::prefix_row_groups(num_seqs, num_q_heads / num_kv_heads);
  const long long target = ((long long)PKV_PREFIX_CTAS_PER_100_SMS * sm_count() + 99) / 100;
  long long ps = (target + num_kv_heads * rg - 1) / (num_kv_heads * rg);
  const int max_ps = (prefix_len + pkv::kPrefixTokens - 1) / pkv::kPrefixTokens;
  const int min_ps = (prefix_len + pkv::kMaxPrefixChunk - 1) / pkv::kMaxPrefixChunk;
  const int suffix = max_ctx > prefix_len ? max_ctx - prefix_len : 0;
  int req = num_splits;
  if (req == 0) req = auto_splits(num_seqs, num_kv_heads, head_dim, suffix, cache_dt, true);
  plan(suffix, req, &pl.splits, &pl.chunk);
  // with every partial of a row in one batch, the merge reads them in one
  // memory round trip
  if (ps > pkv::kMergeBatch - pl.splits) ps = pkv::kMergeBatch - pl.splits;
  if (ps > max_ps) ps = max_ps;
  if (ps < min_ps) ps = min_ps;  // bounds the block-table slice in shared memory
  if (ps < 1) ps = 1;
  pl.pchunk = round_up((int)((prefix_len + ps - 1) / ps), pkv::kPrefixTokens);
  pl.ps = (prefix_len + pl.pchunk - 1) / pl.pchunk;
  pl.slots = pl.ps + pl.splits;
  const size_t r = (size_t)num_seqs * num_q_heads * pl.slots;
  pl.ws = align256(r * head_dim * sizeof(float)) + align256(r * sizeof(float));
  return pl;
}

}  // namespace

extern "C" {

int pkv_version(void) { return (1 << 16) | 0; }

const char* pkv_strerror(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_ARG: return "invalid argument (null pointer, negative size or n_q % n_kv != 0)";
    case PKV_ERR_DTYPE: return "unsupported dtype combination";
    case PKV_ERR_SHAPE:
      return "unsupported shape (head_dim must be 64 or 128, block_size a power of two in "
             "[8, 256], group in [1, 16])";
    case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case PKV_ERR_WORKSPACE: return "workspace missing or smaller than pkv_workspace_size()";
    case PKV_ERR_CUDA: return "CUDA runtime error";
    case PKV_ERR_ALIGN: return "device pointer not aligned as the call requires";
    case PKV_ERR_NO_BLOCKS: return "the block pool has too few free blocks";
    case PKV_ERR_SCRATCH_LIMIT:
      return "split-K scratch for this shape exceeds the fixed no-allocation scratch "
             "(PKV_NOALLOC_SCRATCH_BYTES); use pkv_paged_attention_decode with a workspace";
    default: return "unknown pkv status";
  }
}

int pkv_kv_cache_append(const void* k, const void* v, const int64_t* slot_mapping,
                        int num_tokens, int num_kv_heads, int head_dim, pkv_dtype in_dt,
                        void* k_cache, void* v_cache, pkv_dtype cache_dt, int num_blocks,
                        int block_size, float* k_scale, float* v_scale, int* err_flag,
                        pkv_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PKV_ERR_ARG;
  if (!k_cache || !v_cache) return PKV_ERR_ARG;
  if (num_tokens > 0 && (!k || !v || !slot_mapping)) return PKV_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_SHAPE;
  if (!pow2_in(block_size, 8, 256)) return PKV_ERR_SHAPE;
  if (in_dt != PKV_F32 && in_dt != PKV_BF16) return PKV_ERR_DTYPE;
  const bool coded = cache_dt == PKV_I8 || cache_dt == PKV_FP8;
  if (cache_dt != in_dt && !coded) return PKV_ERR_DTYPE;
  if (coded && (!k_scale || !v_scale)) return PKV_ERR_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8) || !aligned(k_scale, 4) || !aligned(v_scale, 4) ||
      !aligned(err_flag, 4))
    return PKV_ERR_ALIGN;
  if (num_tokens == 0) return PKV_OK;
  return map_cuda(pkv::launch_append(k, v, slot_mapping, num_tokens, num_kv_heads, head_dim,
                                     in_dt, k_cache, v_cache, cache_dt, num_blocks, block_size,
                                     k_scale, v_scale, err_flag, (cudaStream_t)stream));
}

int pkv_decode_num_splits(int num_seqs, int num_kv_heads, int head_dim, int max_context_len,
                          pkv_dtype cache_dt) {
  if (num_seqs < 0 || num_kv_heads <= 0 || max_context_len < 0) return PKV_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_SHAPE;
  if (cache_dt != PKV_F32 && cache_dt != PKV_BF16 && cache_dt != PKV_I8 && cache_dt != PKV_FP8)
    return PKV_ERR_DTYPE;
  int s, chunk;
  plan(max_context_len, auto_splits(num_seqs, num_kv_heads, head_dim, max_context_len, cache_dt),
       &s, &chunk);
  return s;
}

size_t pkv_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                          int max_context_len, pkv_dtype cache_dt, int num_splits) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0 ||
      num_splits < 0)
    return 0;
  int req = num_splits;
  if (req == 0) req = auto_splits(num_seqs, num_kv_heads, head_dim, max_context_len, cache_dt);
  int s, chunk;
  plan(max_context_len, req, &s, &chunk);
  return ws_bytes(num_seqs, num_q_heads, head_dim, s);
}

}  // extern "C"

namespace {

// Plain decode, or decode with the fused append of each sequence's new token
// (new_k, new_v, slot_mapping non-null).
int decode_impl(void* out, const void* q, pkv_dtype q_dt, const void* k_cache,
                const void* v_cache, pkv_dtype cache_dt, const float* k_scale,
                const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq,
                const int32_t* context_lens, int max_context_len, int num_seqs,
                int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                float softmax_scale, void* workspace, size_t workspace_bytes, int num_splits,
                int* err_flag, pkv_stream_t stream, const void* new_k, const void* new_v,
                const int64_t* slot_mapping) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0 || max_context_len < 0 || num_splits < 0)
    return PKV_ERR_ARG;
  if (num_q_heads % num_kv_heads != 0) return PKV_ERR_ARG;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_ERR_ARG;
  if (!isfinite(softmax_scale)) return PKV_ERR_ARG;
  const int group = num_q_heads / num_kv_heads;
  if (group > 16) return PKV_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_SHAPE;
  if (!pow2_in(block_size, 8, 256)) return PKV_ERR_SHAPE;
  if (cache_dt == PKV_BF16 || cache_dt == PKV_I8 || cache_dt == PKV_FP8) {
    if (q_dt != PKV_BF16) return PKV_ERR_DTYPE;
  } else if (cache_dt == PKV_F32) {
    if (q_dt != PKV_F32 && q_dt != PKV_BF16) return PKV_ERR_DTYPE;
  } else {
    return PKV_ERR_DTYPE;
  }
  if ((cache_dt == PKV_I8 || cache_dt == PKV_FP8) && (!k_scale || !v_scale)) return PKV_ERR_ARG;
  // the header's convention: 16-byte device pointers (the kernels load q, the
  // cache rows and the workspace 16 bytes at a time), 4-byte int32 arrays
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(k_scale, 16) || !aligned(v_scale, 16) || !aligned(block_tables, 4) ||
      !aligned(context_lens, 4) || !aligned(err_flag, 4) || !aligned(workspace, 16))
    return PKV_ERR_ALIGN;
  if (num_seqs == 0) return PKV_OK;
  if (num_seqs > 65535) return PKV_ERR_UNSUPPORTED;  // grid y dimension

  long long cap = (long long)max_blocks_per_seq * block_size;
  const int max_ctx = (int)(max_context_len < cap ? max_context_len : cap);
  int req = num_splits;
  if (req == 0) req = auto_splits(num_seqs, num_kv_heads, head_dim, max_ctx, cache_dt);
  if (req < min_splits(max_ctx)) return PKV_ERR_UNSUPPORTED;
  int splits, chunk;
  plan(max_ctx, req, &splits, &chunk);
  const size_t need = ws_bytes(num_seqs, num_q_heads, head_dim, splits);
  if (need > 0 && (!workspace || workspace_bytes < need)) return PKV_ERR_WORKSPACE;

  pkv::DecodeParams p;
  p.out = out;
  p.q = q;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.err_flag = err_flag;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.block_size = block_size;
  p.log2_bs = log2i(block_size);
  p.num_blocks = num_blocks;
  p.max_context_len = max_context_len;
  p.chunk = chunk;
  p.num_splits = splits;
  p.t_start = 0;
  p.ws_slots = splits;
  p.ws_base = 0;
  p.direct = splits == 1;
  p.phys_bytes = round_up((chunk / block_size + 2) * 4, 128);
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.q_f32 = q_dt == PKV_F32;
  p.out_f32 = q_dt == PKV_F32;
  if (splits > 1) {
    const size_t rows = (size_t)num_seqs * num_q_heads * splits;
    p.ws_o = static_cast<float*>(workspace);
    p.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                        align256(rows * head_dim * sizeof(float)));
  } else {
    p.ws_o = nullptr;
    p.ws_lse = nullptr;
  }
  p.new_k = new_k;
  p.new_v = new_v;
  p.slot_mapping = slot_mapping;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = pkv::launch_decode(p, cache_dt, head_dim, st);
  if (e != cudaSuccess) return PKV_ERR_CUDA;
  if (splits > 1) {
    e = pkv::launch_merge(p, head_dim, st);
    if (e != cudaSuccess) return PKV_ERR_CUDA;
  }
  return PKV_OK;
}

}  // namespace

extern "C" {

int pkv_paged_attention_decode(void* out, const void* q, pkv_dtype q_dt, const void* k_cache,
                               const void* v_cache, pkv_dtype cache_dt, const float* k_scale,
                               const float* v_scale, const int32_t* block_tables,
                               int max_blocks_per_seq, const int32_t* context_lens,
                               int max_context_len, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               float softmax_scale, void* workspace, size_t workspace_bytes,
                               int num_splits, int* err_flag, pkv_stream_t stream) {
  return decode_impl(out, q, q_dt, k_cache, v_cache, cache_dt, k_scale, v_scale, block_tables,
                     max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_q_heads,
                     num_kv_heads, head_dim, block_size, num_blocks, softmax_scale, workspace,
                     workspace_bytes, num_splits, err_flag, stream, nullptr, nullptr, nullptr);
}

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
                                      pkv_stream_t stream) {
  if (!k || !v || !slot_mapping) return PKV_ERR_ARG;
  if (cache_dt != PKV_BF16 && cache_dt != PKV_I8 && cache_dt != PKV_FP8)
    return PKV_ERR_UNSUPPORTED;  // fp32 caches: pkv_kv_cache_append, then decode
  if (in_dt != PKV_BF16) return PKV_ERR_DTYPE;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(slot_mapping, 8)) return PKV_ERR_ALIGN;
  return decode_impl(out, q, in_dt, k_cache, v_cache, cache_dt, k_scale, v_scale, block_tables,
                     max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_q_heads,
                     num_kv_heads, head_dim, block_size, num_blocks, softmax_scale, workspace,
                     workspace_bytes, num_splits, err_flag, stream, k, v, slot_mapping);
}

size_t pkv_shared_prefix_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                        int head_dim, int max_context_len, int prefix_len,
                                        pkv_dtype cache_dt, int num_splits) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0 ||
      num_splits < 0 || prefix_len < 0 || num_q_heads % num_kv_heads != 0)
    return 0;
  if (prefix_len == 0)
    return pkv_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                              cache_dt, num_splits);
  return plan_prefix(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, prefix_len,
                     cache_dt, num_splits)
      .ws;
}

int pkv_shared_prefix_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                           int max_context_len, int prefix_len, pkv_dtype cache_dt,
                           int num_splits, int* prefix_slices, int* suffix_splits) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0 ||
      num_splits < 0 || prefix_len <= 0 || num_q_heads % num_kv_heads != 0)
    return PKV_ERR_ARG;
  const PrefixPlan pl = plan_prefix(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                    max_context_len, prefix_len, cache_dt, num_splits);
  if (prefix_slices) *prefix_slices = pl.ps;
  if (suffix_splits) *suffix_splits = pl.splits;
  return PKV_OK;
}

}  // extern "C"

namespace {

// Shared-prefix decode, optionally with the fused append of each sequence's new
// token (new_k, new_v, slot_mapping non-null; done by the suffix decode kernel).
int shared_prefix_impl(
    void* out, const void* q, pkv_dtype q_dt, const void* k_cache, const void* v_cache,
    pkv_dtype cache_dt, const float* k_scale, const float* v_scale, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* context_lens, int max_context_len, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
    float softmax_scale, int prefix_len, void* workspace, size_t workspace_bytes, int num_splits,
    int* err_flag, pkv_stream_t stream, const void* new_k, const void* new_v,
    const int64_t* slot_mapping) {
  if (prefix_len < 0) return PKV_ERR_ARG;
  if (prefix_len == 0)
    return decode_impl(out, q, q_dt, k_cache, v_cache, cache_dt, k_scale, v_scale, block_tables,
                       max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, softmax_scale, workspace,
                       workspace_bytes, num_splits, err_flag, stream, new_k, new_v,
                       slot_mapping);
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0 || max_context_len < 0 || num_splits < 0)
    return PKV_ERR_ARG;
  if (num_q_heads % num_kv_heads != 0) return PKV_ERR_ARG;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_ERR_ARG;
  if (!isfinite(softmax_scale)) return PKV_ERR_ARG;
  const int group = num_q_heads / num_kv_heads;
  if (group > 16) return PKV_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_SHAPE;
  if (!pow2_in(block_size, 8, 256)) return PKV_ERR_SHAPE;
  if (cache_dt != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  if (q_dt != PKV_BF16) return PKV_ERR_DTYPE;
  if (prefix_len % block_size != 0 || (long long)prefix_len > (long long)max_blocks_per_seq * block_size)
    return PKV_ERR_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(err_flag, 4) ||
      !aligned(workspace, 16))
    return PKV_ERR_ALIGN;
  if (num_seqs == 0) return PKV_OK;
  if (num_seqs > 65535) return PKV_ERR_UNSUPPORTED;

  const long long cap = (long long)max_blocks_per_seq * block_size;
  const int max_ctx = (int)(max_context_len < cap ? max_context_len : cap);
  const int suffix = max_ctx > prefix_len ? max_ctx - prefix_len : 0;
  if (num_splits != 0 && num_splits < min_splits(suffix)) return PKV_ERR_UNSUPPORTED;
  const PrefixPlan pl = plan_prefix(num_seqs, num_q_heads, num_kv_heads, head_dim, max_ctx,
                                    prefix_len, cache_dt, num_splits);
  if (pl.splits < min_splits(suffix)) return PKV_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < pl.ws) return PKV_ERR_WORKSPACE;

  pkv::DecodeParams p;
  p.out = out;
  p.q = q;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.err_flag = err_flag;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.block_size = block_size;
  p.log2_bs = log2i(block_size);
  p.num_blocks = num_blocks;
  p.max_context_len = max_context_len;
  p.chunk = pl.chunk;
  p.num_splits = pl.splits;
  p.t_start = prefix_len;
  p.ws_slots = pl.slots;
  p.ws_base = pl.ps;
  p.direct = 0;
  p.phys_bytes = round_up((pl.chunk / block_size + 2) * 4, 128);
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.q_f32 = 0;
  p.out_f32 = 0;
  const size_t rows = (size_t)num_seqs * num_q_heads * pl.slots;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                      align256(rows * head_dim * sizeof(float)));
  pkv::PrefixParams pp;
  pp.prefix_len = prefix_len;
  pp.pchunk = pl.pchunk;
  pp.prefix_splits = pl.ps;
  pp.rows = num_seqs * group;
  pp.phys_bytes = round_up((pl.pchunk / block_size + 2) * 4, 128);

  p.new_k = new_k;
  p.new_v = new_v;
  p.slot_mapping = slot_mapping;

  cudaStream_t st = (cudaStream_t)stream;
  // The suffix decode first; the prefix pass (independent of it: disjoint
  // workspace slots, and the fused append never writes a shared block) is
  // launched behind it and fills the SMs its last wave leaves idle; then the
  // merge, behind both.
  if (pkv::launch_decode(p, cache_dt, head_dim, st) != cudaSuccess) return PKV_ERR_CUDA;
  if (pkv::launch_prefix(p, pp, head_dim, true, st) != cudaSuccess) return PKV_ERR_CUDA;
  if (pkv::launch_merge(p, head_dim, st) != cudaSuccess) return PKV_ERR_CUDA;
  return PKV_OK;
}

}  // namespace

extern "C" {

int pkv_paged_attention_decode_shared_prefix(
    void* out, const void* q, pkv_dtype q_dt, const void* k_cache, const void* v_cache,
    pkv_dtype cache_dt, const float* k_scale, const float* v_scale, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* context_lens, int max_context_len, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
    float softmax_scale, int prefix_len, void* workspace, size_t workspace_bytes, int num_splits,
    int* err_flag, pkv_stream_t stream) {
  return shared_prefix_impl(out, q, q_dt, k_cache, v_cache, cache_dt, k_scale, v_scale,
                            block_tables, max_blocks_per_seq, context_lens, max_context_len,
                            num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                            num_blocks, softmax_scale, prefix_len, workspace, workspace_bytes,
                            num_splits, err_flag, stream, nullptr, nullptr, nullptr);
}

int pkv_paged_attention_decode_shared_prefix_append(
    void* out, const void* q, const void* k, const void* v, const int64_t* slot_mapping,
    pkv_dtype in_dt, void* k_cache, void* v_cache, pkv_dtype cache_dt,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
    int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int num_blocks, float softmax_scale, int prefix_len, void* workspace,
    size_t workspace_bytes, int num_splits, int* err_flag, pkv_stream_t stream) {
  if (!k || !v || !slot_mapping) return PKV_ERR_ARG;
  if (cache_dt != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  if (in_dt != PKV_BF16) return PKV_ERR_DTYPE;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(slot_mapping, 8)) return PKV_ERR_ALIGN;
  return shared_prefix_impl(out, q, in_dt, k_cache, v_cache, cache_dt, nullptr, nullptr,
                            block_tables, max_blocks_per_seq, context_lens, max_context_len,
                            num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                            num_blocks, softmax_scale, prefix_len, workspace, workspace_bytes,
                            num_splits, err_flag, stream, k, v, slot_mapping);
}

int pkv_read(const void* src, size_t bytes, unsigned int* sink, pkv_stream_t stream) {
  if (!src || !sink) return PKV_ERR_ARG;
  if (bytes % 16) return PKV_ERR_ARG;
  if (!aligned(src, 16) || !aligned(sink, 4)) return PKV_ERR_ALIGN;
  return map_cuda(pkv::launch_read(src, bytes, sink, sm_count(), (cudaStream_t)stream));
}

int pkv_copy(void* dst, const void* src, size_t bytes, pkv_stream_t stream) {
  if (!dst || !src) return PKV_ERR_ARG;
  if (bytes % 16) return PKV_ERR_ARG;
  if (!aligned(dst, 16) || !aligned(src, 16)) return PKV_ERR_ALIGN;
  return map_cuda(pkv::launch_copy(dst, src, bytes, sm_count(), (cudaStream_t)stream));
}

}  // extern "C"
