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
// uses scale = 448 / max|x| and E4M3 codes (append_quant_kernel).
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

// Quantising append (INT8 or FP8 cache).  One CTA of kQuantThreads threads
// per token; a (tensor K|V, head) row of head_dim elements is held by a group
// of kLanesPerRow lanes, lane j of the group holding elements EPL*j ..
// EPL*j + EPL - 1 (EPL = head_dim / 8) with 16-byte vector loads, so one warp
// works on four rows at once and the per-row steps (absmax reduction, the
// scale division) are shared by those four.  The token's 2 * num_kv_heads
// rows (K rows of every head, then V rows) are dealt to the groups; each lane
// loads the rows of kQuantBatch passes before quantising any, so that many
// row loads stay in flight.  The row rule is the one of quant_row_int8 /
// quant_row_fp8 (common.cuh), written for the group layout: scale =
// 127 / max|x| (448 / max|x| for FP8), correctly rounded; each code is the
// correctly rounded fp32 product x * scale converted with round-to-nearest-
// even and saturation (cvt.rni.sat.s8.f32, i.e. clamp(rint(.), -128, 127); for
// FP8 cvt.rn.satfinite.e4m3x2); an all-zero row stores codes 0 and scale 1.
constexpr int kQuantThreads = 256;
constexpr int kLanesPerRow = 8;
constexpr int kRowsPerPass = kQuantThreads / kLanesPerRow;  // 32 rows per CTA pass
constexpr int kQuantBatch = 2;

// One code of the INT8 rule from the fp32 product p: round half to even, then
// saturate to [-128, 127].
__device__ __forceinline__ uint32_t s8_code(float p) {
  short q;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=h"(q) : "f"(p));
  return (uint32_t)q & 0xFFu;
}

// Four codes of the INT8 rule, packed, for products |p| < 127.5 (every
// product of a row whose scale 127 / max|x| is finite): adding 1.5 * 2^23 in
// round-to-nearest-even leaves rint(p) in the low mantissa bits (the sum's
// unit in the last place is 1), and its low byte is the two's-complement
// code; no saturation can occur.  An FMA-pipe add and two byte permutes
// instead of four conversions.
__device__ __forceinline__ uint32_t s8_codes4(float p0, float p1, float p2, float p3) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const uint32_t b0 = __float_as_uint(__fadd_rn(p0, kRound));
  const uint32_t b1 = __float_as_uint(__fadd_rn(p1, kRound));
  const uint32_t b2 = __float_as_uint(__fadd_rn(p2, kRound));
  const uint32_t b3 = __float_as_uint(__fadd_rn(p3, kRound));
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

template <typename T, int EPL>
__device__ __forceinline__ void widen_vecs(const uint4 (&v)[EPL * sizeof(T) / 16], float (&x)[EPL]) {
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < EPL / 8; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        x[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
        x[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < EPL / 4; ++i) {
      x[4 * i] = __uint_as_float(v[i].x);
      x[4 * i + 1] = __uint_as_float(v[i].y);
      x[4 * i + 2] = __uint_as_float(v[i].z);
      x[4 * i + 3] = __uint_as_float(v[i].w);
    }
  }
}

template <typename T, int HD, bool FP8>
__global__ void __launch_bounds__(kQuantThreads)
    append_quant_kernel(const T* __restrict__ k, const T* __restrict__ v,
                        const int64_t* __restrict__ slot_mapping, int num_kv_heads,
                        uint8_t* __restrict__ k_cache, uint8_t* __restrict__ v_cache,
                        float* __restrict__ k_scale, float* __restrict__ v_scale, int log2_bs,
                        long long num_slots, int* err_flag) {
  constexpr int EPL = HD / kLanesPerRow;         // elements per lane: 16 or 8
  constexpr int VECS = EPL * (int)sizeof(T) / 16;  // 16-byte loads per lane per row
  constexpr int WORDS = EPL / 4;                 // 4-byte code words per lane per row
  const int t = blockIdx.x;
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int j = lane % kLanesPerRow;
  const long long slot = slot_mapping[t];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (threadIdx.x == 0) set_flag(err_flag, PKV_FLAG_BAD_SLOT);
    return;
  }
  const int bs = 1 << log2_bs;
  const long long blk = slot >> log2_bs;
  const int off = (int)(slot & (bs - 1));
  const int rows = 2 * num_kv_heads;
  const size_t src_row0 = (size_t)t * num_kv_heads;
  const size_t dst_row0 = (size_t)slot * num_kv_heads;
  // every lane of a warp runs the same passes (the group shuffles need all 32)
  for (int base = warp * (kWarp / kLanesPerRow); base < rows;
       base += kRowsPerPass * kQuantBatch) {
    uint4 buf[kQuantBatch][VECS];
#pragma unroll
    for (int b = 0; b < kQuantBatch; ++b) {
      const int r = base + lane / kLanesPerRow + b * kRowsPerPass;
      if (r < rows) {
        const bool is_v = r >= num_kv_heads;
        const int h = is_v ? r - num_kv_heads : r;
        const uint4* src =
            reinterpret_cast<const uint4*>((is_v ? v : k) + (src_row0 + h) * HD) + j * VECS;
#pragma unroll
        for (int i = 0; i < VECS; ++i) buf[b][i] = __ldg(src + i);
      } else {
#pragma unroll
        for (int i = 0; i < VECS; ++i) buf[b][i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int b = 0; b < kQuantBatch; ++b) {
      const int r = base + lane / kLanesPerRow + b * kRowsPerPass;
      float x[EPL];
      widen_vecs<T, EPL>(buf[b], x);
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
      for (int o = 1; o < kLanesPerRow; o <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float scale = amax > 0.f ? __fdiv_rn(FP8 ? 448.0f : 127.0f, amax) : 1.0f;
      // finite max and scale: |x * scale| < 127.5 (the row's common branch)
      const bool fast = amax <= 3.4e38f && scale <= 3.4e38f;
      uint32_t w[WORDS];
      if (FP8 || fast) {
#pragma unroll
        for (int q = 0; q < WORDS; ++q) {
          const float p0 = __fmul_rn(x[4 * q], scale), p1 = __fmul_rn(x[4 * q + 1], scale);
          const float p2 = __fmul_rn(x[4 * q + 2], scale), p3 = __fmul_rn(x[4 * q + 3], scale);
          if constexpr (FP8)
            w[q] = amax > 0.f ? (f32x2_to_e4m3x2(p0, p1) | (f32x2_to_e4m3x2(p2, p3) << 16)) : 0u;
          else
            w[q] = s8_codes4(p0, p1, p2, p3);
        }
      } else {  // INT8 row whose scale is not finite (max |x| infinite, NaN or below 2^-126 * 127)
#pragma unroll
        for (int q = 0; q < WORDS; ++q) {
          const float p0 = __fmul_rn(x[4 * q], scale), p1 = __fmul_rn(x[4 * q + 1], scale);
          const float p2 = __fmul_rn(x[4 * q + 2], scale), p3 = __fmul_rn(x[4 * q + 3], scale);
          w[q] = s8_code(p0) | (s8_code(p1) << 8) | (s8_code(p2) << 16) | (s8_code(p3) << 24);
        }
      }
      if (r < rows) {
        const bool is_v = r >= num_kv_heads;
        const int h = is_v ? r - num_kv_heads : r;
        uint8_t* dst = (is_v ? v_cache : k_cache) + (dst_row0 + h) * HD + j * EPL;
        if constexpr (WORDS == 4)
          *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        else
          *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
        if (j == 0) (is_v ? v_scale : k_scale)[((size_t)blk * num_kv_heads + h) * bs + off] = scale;
      }
    }
  }
}

template <typename T, bool FP8>
cudaError_t launch_quant(const void* k, const void* v, const int64_t* slot_mapping,
                         int num_tokens, int num_kv_heads, int head_dim, void* k_cache,
                         void* v_cache, float* k_scale, float* v_scale, int block_size,
                         long long num_slots, int* err_flag, cudaStream_t st) {
  int log2_bs = 0;
  while ((1 << log2_bs) < block_size) ++log2_bs;
  const dim3 grid((unsigned)num_tokens);
  constexpr int threads = kQuantThreads;
  if (head_dim == 128)
    append_quant_kernel<T, 128, FP8><<<grid, threads, 0, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), slot_mapping, num_kv_heads,
        static_cast<uint8_t*>(k_cache), static_cast<uint8_t*>(v_cache), k_scale, v_scale,
        log2_bs, num_slots, err_flag);
  else
    append_quant_kernel<T, 64, FP8><<<grid, threads, 0, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), slot_mapping, num_kv_heads,
        static_cast<uint8_t*>(k_cache), static_cast<uint8_t*>(v_cache), k_scale, v_scale,
        log2_bs, num_slots, err_flag);
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
      return launch_quant<__nv_bfloat16, true>(k, v, slot_mapping, num_tokens, num_kv_heads,
                                               head_dim, k_cache, v_cache, k_scale, v_scale,
                                               block_size, num_slots, err_flag, st);
    return launch_quant<float, true>(k, v, slot_mapping, num_tokens, num_kv_heads, head_dim,
                                     k_cache, v_cache, k_scale, v_scale, block_size, num_slots,
                                     err_flag, st);
  }
  if (cache_dt == PKV_I8) {
    if (in_dt == PKV_BF16)
      return launch_quant<__nv_bfloat16, false>(k, v, slot_mapping, num_tokens, num_kv_heads,
                                                head_dim, k_cache, v_cache, k_scale, v_scale,
                                                block_size, num_slots, err_flag, st);
    return launch_quant<float, false>(k, v, slot_mapping, num_tokens, num_kv_heads, head_dim,
                                      k_cache, v_cache, k_scale, v_scale, block_size, num_slots,
                                      err_flag, st);
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
