// Whole-block copies between two block pools (C ABI in include/pkv.h).
//
// Serves the block manager: copy-on-write of a shared, partially filled block
// inside the device pool, and swapping a sequence's blocks out to a pinned host
// pool and back in ("大模型推理加速实战：KV Cache内存优化与PagedAttention分页管理方案",
// deployment parameters: swap_space lets inactive KV caches move to CPU memory
// so that more requests fit than HBM holds).  Either pool may be device memory
// or page-locked host memory that the device reaches through unified
// addressing; one kernel launch moves every listed block, 16 bytes per access,
// all loads of a thread in flight before its stores.
#include "common.cuh"

namespace pkv {

namespace {

struct CopyParams {
  uint8_t* dst_k;
  uint8_t* dst_v;
  const uint8_t* src_k;
  const uint8_t* src_v;
  float* dst_ks;
  float* dst_vs;
  const float* src_ks;
  const float* src_vs;
  const int32_t* pairs;  // [num_pairs][2]: source block, destination block
  long long block_vecs;  // 16-byte vectors per block of K (or V)
  int scale_vecs;        // 16-byte vectors of scales per block (0: none)
  int src_blocks, dst_blocks;
  int* err_flag;
};

constexpr int kCopyThreads = 256;
constexpr int kCopyVecs = 4;  // vectors per thread per tensor

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(const CopyParams cp) {
  const int pair = blockIdx.x;
  const int src = cp.pairs[2 * pair], dst = cp.pairs[2 * pair + 1];
  if (src < 0 || src >= cp.src_blocks || dst < 0 || dst >= cp.dst_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_flag(cp.err_flag, PKV_FLAG_BAD_BLOCK);
    return;
  }
  const uint4* sk = reinterpret_cast<const uint4*>(cp.src_k) + (size_t)src * cp.block_vecs;
  const uint4* sv = reinterpret_cast<const uint4*>(cp.src_v) + (size_t)src * cp.block_vecs;
  uint4* dk = reinterpret_cast<uint4*>(cp.dst_k) + (size_t)dst * cp.block_vecs;
  uint4* dv = reinterpret_cast<uint4*>(cp.dst_v) + (size_t)dst * cp.block_vecs;
  const long long first = (long long)blockIdx.y * kCopyThreads * kCopyVecs + threadIdx.x;
  uint4 a[kCopyVecs], b[kCopyVecs];
#pragma unroll
  for (int i = 0; i < kCopyVecs; ++i) {
    const long long idx = first + (long long)i * kCopyThreads;
    if (idx < cp.block_vecs) {
      a[i] = sk[idx];
      b[i] = sv[idx];
    }
  }
#pragma unroll
  for (int i = 0; i < kCopyVecs; ++i) {
    const long long idx = first + (long long)i * kCopyThreads;
    if (idx < cp.block_vecs) {
      dk[idx] = a[i];
      dv[idx] = b[i];
    }
  }
  if (blockIdx.y == 0 && cp.scale_vecs > 0) {
    for (int i = threadIdx.x; i < cp.scale_vecs; i += kCopyThreads) {
      reinterpret_cast<uint4*>(cp.dst_ks)[(size_t)dst * cp.scale_vecs + i] =
          reinterpret_cast<const uint4*>(cp.src_ks)[(size_t)src * cp.scale_vecs + i];
      reinterpret_cast<uint4*>(cp.dst_vs)[(size_t)dst * cp.scale_vecs + i] =
          reinterpret_cast<const uint4*>(cp.src_vs)[(size_t)src * cp.scale_vecs + i];
    }
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace pkv

extern "C" int pkv_copy_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               size_t block_bytes, int dst_num_blocks, int src_num_blocks,
                               float* dst_k_scale, float* dst_v_scale, const float* src_k_scale,
                               const float* src_v_scale, size_t scale_bytes_per_block,
                               const int32_t* pairs, int num_pairs, int* err_flag,
                               pkv_stream_t stream) {
  using namespace pkv;
  if (num_pairs < 0 || dst_num_blocks <= 0 || src_num_blocks <= 0) return PKV_ERR_ARG;
  if (num_pairs == 0) return PKV_OK;
  if (!dst_k || !dst_v || !src_k || !src_v || !pairs) return PKV_ERR_ARG;
  if (block_bytes == 0 || block_bytes % 16 != 0 || scale_bytes_per_block % 16 != 0)
    return PKV_ERR_SHAPE;
  const bool scales = scale_bytes_per_block > 0;
  if (scales && (!dst_k_scale || !dst_v_scale || !src_k_scale || !src_v_scale)) return PKV_ERR_ARG;
  if (!aligned16(dst_k) || !aligned16(dst_v) || !aligned16(src_k) || !aligned16(src_v) ||
      (scales && (!aligned16(dst_k_scale) || !aligned16(dst_v_scale) ||
                  !aligned16(src_k_scale) || !aligned16(src_v_scale))) ||
      (reinterpret_cast<uintptr_t>(pairs) & 3u) || (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return PKV_ERR_ALIGN;
  CopyParams cp;
  cp.dst_k = static_cast<uint8_t*>(dst_k);
  cp.dst_v = static_cast<uint8_t*>(dst_v);
  cp.src_k = static_cast<const uint8_t*>(src_k);
  cp.src_v = static_cast<const uint8_t*>(src_v);
  cp.dst_ks = dst_k_scale;
  cp.dst_vs = dst_v_scale;
  cp.src_ks = src_k_scale;
  cp.src_vs = src_v_scale;
  cp.pairs = pairs;
  cp.block_vecs = (long long)(block_bytes / 16);
  cp.scale_vecs = (int)(scale_bytes_per_block / 16);
  cp.src_blocks = src_num_blocks;
  cp.dst_blocks = dst_num_blocks;
  cp.err_flag = err_flag;
  const long long per_cta = (long long)kCopyThreads * kCopyVecs;
  const dim3 grid((unsigned)num_pairs, (unsigned)((cp.block_vecs + per_cta - 1) / per_cta));
  copy_blocks_kernel<<<grid, kCopyThreads, 0, (cudaStream_t)stream>>>(cp);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
