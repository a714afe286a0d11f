// KV-cache append for sm_100a.
//
// Each new token's K and V rows are written into their slots
// ("大模型推理加速实战…", KV-cache overhead section: every generated token's
// key/value goes into the cache; "LLM推理显存优化KV Cache管理3大策略" §2: a block
// holds block_size token rows).  Slot s -> block s / block_size, row
// s % block_size.  Because a cache row holds all KV heads of one token
// contiguously, the source row and the destination row have the same shape
// and the copy is a straight 16-byte vector copy.
//
// The INT8 variant quantises each (token, head) row as in §4 of the same
// mlqm.cn page (quantize_tensor): scale = 127 / max|x| over head_dim,
// code = clamp(rint(x * scale), -128, 127) in fp32 with round-half-to-even;
// __fdiv_rn / __fmul_rn keep the division and the product correctly rounded
// and unfused.  An all-zero row stores codes 0 and scale 1.  The FP8 variant
// uses scale = 448 / max|x| and E4M3 codes (see append_fp8_kernel).
#include "common.cuh"
#include "decode.cuh"

namespace pkv {

namespace {

constexpr int kAppendThreads = 128;

// Grid (token, K|V, row piece): each CTA copies kAppendThreads * kVecs 16-byte
// vectors of one token's row (all KV heads).  Every thread issues all of its
// loads before any store, so a launch costs one memory round trip.
constexpr int kVecs = 4;

__global__ void __launch_bounds__(kAppendThreads)
    append_copy_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                       const int64_t* __restrict__ slot_mapping, int row_vecs,
                       uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                       long long num_slots, int* err_flag) {
  const int t = blockIdx.x;
  const long long slot = slot_mapping[t];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) set_flag(err_flag, PKV_FLAG_BAD_SLOT);
    return;
  }
  const uint4* src = (blockIdx.y ? v : k) + (size_t)t * row_vecs;
  uint4* dst = (blockIdx.y ? v_cache : k_cache) + (size_t)slot * row_vecs;
  const int first = blockIdx.z * (kAppendThreads * kVecs) + threadIdx.x;
  uint4 buf[kVecs];
#pragma unroll
  for (int i = 0; i < kVecs; ++i) {
    const int idx = first + i * kAppendThreads;
    if (idx < row_vecs) buf[i] = __ldg(src + idx);
  }
#pragma unroll
  for (int i = 0; i < kVecs; ++i) {
    const int idx = first + i * kAppendThreads;
    if (idx < row_vecs) dst[idx] = buf[i];
  }
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// One warp per (token, tensor K|V, head) row.  Lane l holds head_dim/32
// consecutive elements.
template <typename T, int HD>
__global__ void __launch_bounds__(kAppendThreads)
    append_int8_kernel(const T* __restrict__ k, const T* __restrict__ v,
                       const int64_t* __restrict__ slot_mapping, int num_tokens,
                       int num_kv_heads, int8_t* __restrict__ k_cache,
                       int8_t* __restrict__ v_cache, float* __restrict__ k_scale,
                       float* __restrict__ v_scale, int block_size, long long num_slots,
                       int* err_flag) {
  constexpr int E = HD / kWarp;  // elements per lane (2 or 4)
  const int lane = threadIdx.x % kWarp;
  const long long row = (long long)blockIdx.x * (kAppendThreads / kWarp) + threadIdx.x / kWarp;
  const long long rows = (long long)num_tokens * 2 * num_kv_heads;
  if (row >= rows) return;
  const int t = (int)(row / (2 * num_kv_heads));
  const int rem = (int)(row % (2 * num_kv_heads));
  const bool is_v = rem >= num_kv_heads;
  const int h = is_v ? rem - num_kv_heads : rem;
  const long long slot = slot_mapping[t];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (lane == 0 && h == 0 && !is_v) set_flag(err_flag, PKV_FLAG_BAD_SLOT);
    return;
  }
  const T* src = (is_v ? v : k) + ((size_t)t * num_kv_heads + h) * HD + lane * E;
  float x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = to_f32(src[e]);
  float scale;
  const uint32_t packed = quant_row_int8<E>(x, &scale);
  const long long blk = slot / block_size;
  const int off = (int)(slot % block_size);
  int8_t* dst = (is_v ? v_cache : k_cache) + ((size_t)slot * num_kv_heads + h) * HD + lane * E;
  if constexpr (E == 4)
    *reinterpret_cast<uint32_t*>(dst) = packed;
  else
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
  if (lane == 0) {
    float* sc = is_v ? v_scale : k_scale;
    sc[((size_t)blk * num_kv_heads + h) * block_size + off] = scale;
  }
}

// FP8 (E4M3) variant of the same row rule: scale = 448 / max|x|, codes
// E4M3(x * scale) with round-to-nearest-even and saturation (hardware cvt);
// an all-zero row stores codes 0 and scale 1.
template <typename T, int HD>
__global__ void __launch_bounds__(kAppendThreads)
    append_fp8_kernel(const T* __restrict__ k, const T* __restrict__ v,
                      const int64_t* __restrict__ slot_mapping, int num_tokens, int num_kv_heads,
                      uint8_t* __restrict__ k_cache, uint8_t* __restrict__ v_cache,
                      float* __restrict__ k_scale, float* __restrict__ v_scale, int block_size,
                      long long num_slots, int* err_flag) {
  constexpr int E = HD / kWarp;  // elements per lane (2 or 4)
  const int lane = threadIdx.x % kWarp;
  const long long row = (long long)blockIdx.x * (kAppendThreads / kWarp) + threadIdx.x / kWarp;
  const long long rows = (long long)num_tokens * 2 * num_kv_heads;
  if (row >= rows) return;
  const int t = (int)(row / (2 * num_kv_heads));
  const int rem = (int)(row % (2 * num_kv_heads));
  const bool is_v = rem >= num_kv_heads;
  const int h = is_v ? rem - num_kv_heads : rem;
  const long long slot = slot_mapping[t];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (lane == 0 && h == 0 && !is_v) set_flag(err_flag, PKV_FLAG_BAD_SLOT);
    return;
  }
  const T* src = (is_v ? v : k) + ((size_t)t * num_kv_heads + h) * HD + lane * E;
  float x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = to_f32(src[e]);
  float scale;
  const uint32_t packed = quant_row_fp8<E>(x, &scale);
  const long long blk = slot / block_size;
  const int off = (int)(slot % block_size);
  uint8_t* dst = (is_v ? v_cache : k_cache) + ((size_t)slot * num_kv_heads + h) * HD + lane * E;
  if constexpr (E == 4)
    *reinterpret_cast<uint32_t*>(dst) = packed;
  else
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
  if (lane == 0) {
    float* sc = is_v ? v_scale : k_scale;
    sc[((size_t)blk * num_kv_heads + h) * block_size + off] = scale;
  }
}

template <typename T>
cudaError_t launch_fp8(const void* k, const void* v, const int64_t* slot_mapping, int num_tokens,
                       int num_kv_heads, int head_dim, void* k_cache, void* v_cache,
                       float* k_scale, float* v_scale, int block_size, long long num_slots,
                       int* err_flag, cudaStream_t st) {
  const long long rows = (long long)num_tokens * 2 * num_kv_heads;
  const long long per = kAppendThreads / kWarp;
  const unsigned grid = (unsigned)((rows + per - 1) / per);
  if (head_dim == 128)
    append_fp8_kernel<T, 128><<<grid, kAppendThreads, 0, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), slot_mapping, num_tokens,
        num_kv_heads, static_cast<uint8_t*>(k_cache), static_cast<uint8_t*>(v_cache), k_scale,
        v_scale, block_size, num_slots, err_flag);
  else
    append_fp8_kernel<T, 64><<<grid, kAppendThreads, 0, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), slot_mapping, num_tokens,
        num_kv_heads, static_cast<uint8_t*>(k_cache), static_cast<uint8_t*>(v_cache), k_scale,
        v_scale, block_size, num_slots, err_flag);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_i8(const void* k, const void* v, const int64_t* slot_mapping, int num_tokens,
                      int num_kv_heads, int head_dim, void* k_cache, void* v_cache,
                      float* k_scale, float* v_scale, int block_size, long long num_slots,
                      int* err_flag, cudaStream_t st) {
  const long long rows = (long long)num_tokens * 2 * num_kv_heads;
  const long long per = kAppendThreads / kWarp;
  const unsigned grid = (unsigned)((rows + per - 1) / per);
  if (head_dim == 128)
    append_int8_kernel<T, 128><<<grid, kAppendThreads, 0, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), slot_mapping, num_tokens,
        num_kv_heads, static_cast<int8_t*>(k_cache), static_cast<int8_t*>(v_cache), k_scale,
        v_scale, block_size, num_slots, err_flag);
  else
    append_int8_kernel<T, 64><<<grid, kAppendThreads, 0, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), slot_mapping, num_tokens,
        num_kv_heads, static_cast<int8_t*>(k_cache), static_cast<int8_t*>(v_cache), k_scale,
        v_scale, block_size, num_slots, err_flag);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append(const void* k, const void* v, const int64_t* slot_mapping,
                          int num_tokens, int num_kv_heads, int head_dim, pkv_dtype in_dt,
                          void* k_cache, void* v_cache, pkv_dtype cache_dt, int num_blocks,
                          int block_size, float* k_scale, float* v_scale, int* err_flag,
                          cudaStream_t st) {
  if (num_tokens == 0) return cudaSuccess;
  const long long num_slots = (long long)num_blocks * block_size;
  if (cache_dt == PKV_FP8) {
    if (in_dt == PKV_BF16)
      return launch_fp8<__nv_bfloat16>(k, v, slot_mapping, num_tokens, num_kv_heads, head_dim,
                                       k_cache, v_cache, k_scale, v_scale, block_size,
                                       num_slots, err_flag, st);
    return launch_fp8<float>(k, v, slot_mapping, num_tokens, num_kv_heads, head_dim, k_cache,
                             v_cache, k_scale, v_scale, block_size, num_slots, err_flag, st);
  }
  if (cache_dt == PKV_I8) {
    if (in_dt == PKV_BF16)
      return launch_i8<__nv_bfloat16>(k, v, slot_mapping, num_tokens, num_kv_heads, head_dim,
                                      k_cache, v_cache, k_scale, v_scale, block_size, num_slots,
                                      err_flag, st);
    return launch_i8<float>(k, v, slot_mapping, num_tokens, num_kv_heads, head_dim, k_cache,
                            v_cache, k_scale, v_scale, block_size, num_slots, err_flag, st);
  }
  const int elem = (in_dt == PKV_F32) ? 4 : 2;
  const int row_vecs = num_kv_heads * head_dim * elem / 16;
  const dim3 grid(num_tokens, 2, (row_vecs + kAppendThreads * kVecs - 1) / (kAppendThreads * kVecs));
  append_copy_kernel<<<grid, kAppendThreads, 0, st>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, row_vecs,
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), num_slots, err_flag);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Streaming copy (HBM bandwidth probe): grid-stride 16-byte vectors, four in
// flight per thread.
__global__ void __launch_bounds__(256) copy_kernel(uint4* __restrict__ dst,
                                                   const uint4* __restrict__ src, size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n; i += 4 * stride) {
    const uint4 a = __ldcs(src + i);
    const uint4 b = __ldcs(src + i + stride);
    const uint4 c = __ldcs(src + i + 2 * stride);
    const uint4 d = __ldcs(src + i + 3 * stride);
    __stcs(dst + i, a);
    __stcs(dst + i + stride, b);
    __stcs(dst + i + 2 * stride, c);
    __stcs(dst + i + 3 * stride, d);
  }
  for (; i < n; i += stride) __stcs(dst + i, __ldcs(src + i));
}

// Streaming read (HBM read-bandwidth probe, and an L2 flush that leaves only
// clean lines behind): grid-stride 16-byte loads that allocate in L2, eight in
// flight per thread, folded by XOR into one word per CTA so that no load is
// dead.
__global__ void __launch_bounds__(256) read_kernel(const uint4* __restrict__ src, size_t n,
                                                   unsigned int* __restrict__ sink) {
  constexpr int kIn = 8;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  unsigned int x = 0;
  for (; i + (kIn - 1) * stride < n; i += kIn * stride) {
    uint4 v[kIn];
#pragma unroll
    for (int j = 0; j < kIn; ++j) v[j] = __ldcg(src + i + j * stride);
#pragma unroll
    for (int j = 0; j < kIn; ++j) x ^= v[j].x ^ v[j].y ^ v[j].z ^ v[j].w;
  }
  for (; i < n; i += stride) {
    const uint4 v = __ldcg(src + i);
    x ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x ^= __shfl_xor_sync(0xffffffffu, x, off);
  __shared__ unsigned int s_x[8];
  if (threadIdx.x % kWarp == 0) s_x[threadIdx.x / kWarp] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned int r = 0;
    for (int w = 0; w < (int)(blockDim.x / kWarp); ++w) r ^= s_x[w];
    atomicXor(sink, r);
  }
}

cudaError_t launch_read(const void* src, size_t bytes, unsigned int* sink, int num_sms,
                        cudaStream_t st) {
  const size_t n = bytes / 16;
  if (n == 0) return cudaSuccess;
  read_kernel<<<num_sms * 8, 256, 0, st>>>(static_cast<const uint4*>(src), n, sink);
  return cudaGetLastError();
}

cudaError_t launch_copy(void* dst, const void* src, size_t bytes, int num_sms, cudaStream_t st) {
  const size_t n = bytes / 16;
  if (n == 0) return cudaSuccess;
  copy_kernel<<<num_sms * 8, 256, 0, st>>>(static_cast<uint4*>(dst),
                                           static_cast<const uint4*>(src), n);
  return cudaGetLastError();
}

}  // namespace pkv
