// Device and host helpers shared by the decode engines (decode.cu: bf16 and
// fp32 caches, split merge; decode_q8.cu: one-byte INT8 and FP8 caches).
#pragma once

#include <math_constants.h>

#include <atomic>

#include "common.cuh"
#include "decode.cuh"

namespace pkv {

struct CtaSetup {
  int seq, kvh, split;
  int ctx;             // the sequence's (clamped) context length
  int t_begin, t_end;  // token range of this CTA
  int blk0;            // first logical block in s_phys
  bool active;
  bool clean;          // every block of the CTA's slice is in range
};

// Clamped context length: identical in decode and merge kernels.
__device__ __forceinline__ int effective_ctx(const DecodeParams& p, int seq, bool report) {
  int ctx = p.context_lens[seq];
  if (ctx < 0) {
    if (report) set_flag(p.err_flag, PKV_FLAG_NEG_CTX);
    ctx = 0;
  }
  const long long cap_tab = (long long)p.max_blocks_per_seq * p.block_size;
  const long long cap_split = (long long)p.t_start + (long long)p.num_splits * p.chunk;
  if (ctx > p.max_context_len || ctx > cap_tab) {
    if (report) set_flag(p.err_flag, PKV_FLAG_CTX_RANGE);
  }
  long long c = ctx;
  if (c > cap_tab) c = cap_tab;
  if (c > cap_split) c = cap_split;
  return (int)c;
}

// Loads and validates this CTA's slice of the block table into smem.
__device__ __forceinline__ CtaSetup cta_setup(const DecodeParams& p, int* s_phys) {
  CtaSetup c;
  c.kvh = blockIdx.x;
  c.seq = blockIdx.y;
  c.split = blockIdx.z;
  const bool report = (c.kvh == 0 && c.split == 0 && threadIdx.x == 0);
  const int ctx = effective_ctx(p, c.seq, report);
  c.t_begin = p.t_start + c.split * p.chunk;
  c.ctx = ctx;
  c.t_end = min(ctx, c.t_begin + p.chunk);
  c.active = c.t_begin < c.t_end;
  c.blk0 = c.t_begin >> p.log2_bs;
  int bad = 0;
  if (c.active) {
    const int nphys = ((c.t_end - 1) >> p.log2_bs) - c.blk0 + 1;
    const int32_t* row = p.block_tables + (size_t)c.seq * p.max_blocks_per_seq;
    for (int i = threadIdx.x; i < nphys; i += blockDim.x) {
      int b = row[c.blk0 + i];
      if (b < 0 || b >= p.num_blocks) {
        set_flag(p.err_flag, PKV_FLAG_BAD_BLOCK);
        b = -1;
        bad = 1;
      }
      s_phys[i] = b;
    }
  }
  c.clean = !__syncthreads_or(bad);
  return c;
}

// Cache formats of the mma engine.
constexpr int kQuantNone = 0;  // bf16 values
constexpr int kQuantI8 = 1;    // int8 codes, fp32 scale per token per head
constexpr int kQuantFp8 = 2;   // E4M3 codes, fp32 scale per token per head

// Fused append (pkv_paged_attention_decode_append), in two parts.
//
// Prefetch, in every warp before the CTA's first barrier: each lane loads its
// share of the sequence's new K and V rows of this KV head (bf16 rows: lane l
// holds 16-byte chunk l of K, then of V; one-byte caches: lane l holds
// elements E*l .. E*l+E-1 of K in .x/.y and of V in .z/.w, E = head_dim / 32)
// and the token's slot, so their latency overlaps the CTA set-up.
template <int HD, int QM>
__device__ __forceinline__ uint4 fused_prefetch(const DecodeParams& p, long long* slot) {
  uint4 r = make_uint4(0u, 0u, 0u, 0u);
  *slot = -1;
  if (p.new_k == nullptr) return r;
  const int lane = threadIdx.x % kWarp;
  const size_t base = ((size_t)blockIdx.y * p.num_kv_heads + blockIdx.x) * HD;
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(p.new_k) + base;
  const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(p.new_v) + base;
  *slot = p.slot_mapping[blockIdx.y];
  if constexpr (QM == kQuantNone) {
    constexpr int V = HD / 8;  // 16-byte chunks of a bf16 row
    if (lane < 2 * V) r = reinterpret_cast<const uint4*>(lane < V ? k : v)[lane % V];
  } else if constexpr (HD / kWarp == 4) {
    const uint2 a = reinterpret_cast<const uint2*>(k)[lane];
    const uint2 b = reinterpret_cast<const uint2*>(v)[lane];
    r = make_uint4(a.x, a.y, b.x, b.y);
  } else {
    r.x = reinterpret_cast<const uint32_t*>(k)[lane];
    r.z = reinterpret_cast<const uint32_t*>(v)[lane];
  }
  return r;
}

// Commit, after the set-up: the warp that will read the 16-token tile holding
// position ctx - 1 (tile i of the CTA belongs to warp i % NWARPS) writes the
// token's K and V rows into slot_mapping[seq], quantised for one-byte caches
// with the append kernels' own row rule, then syncs the warp, so that its
// later cp.async reads of that position see the rows.  No other CTA reads the
// position.  The slot must be the one the block table gives position ctx - 1;
// otherwise nothing is written and PKV_FLAG_BAD_SLOT is set.  A negative slot
// writes nothing.
template <int HD, int QM, int NWARPS>
__device__ __forceinline__ void fused_commit(const DecodeParams& p, const CtaSetup& c,
                                             const int* s_phys, uint4 r, long long slot) {
  if (p.new_k == nullptr || !c.active || c.t_end != c.ctx) return;
  const int pos = c.ctx - 1;
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  if (warp != ((pos - c.t_begin) >> 4) % NWARPS || slot < 0) return;
  const int bs = p.block_size;
  const int b = s_phys[(pos >> p.log2_bs) - c.blk0];
  if (b < 0 || slot != (long long)b * bs + (pos & (bs - 1))) {
    if (lane == 0) set_flag(p.err_flag, PKV_FLAG_BAD_SLOT);
    return;
  }
  const size_t row = (size_t)slot * p.num_kv_heads + c.kvh;  // in head_dim units
  if constexpr (QM == kQuantNone) {
    constexpr int V = HD / 8;
    if (lane < 2 * V) {
      void* cache = const_cast<void*>(lane < V ? p.k_cache : p.v_cache);
      reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(cache) + row * HD)[lane % V] = r;
    }
  } else {
    constexpr int E = HD / kWarp;  // elements per lane
#pragma unroll
    for (int t = 0; t < 2; ++t) {  // K, then V
      const uint32_t w0 = t ? r.z : r.x, w1 = t ? r.w : r.y;
      float x[E];
      x[0] = __uint_as_float(w0 << 16);
      x[1] = __uint_as_float(w0 & 0xFFFF0000u);
      if constexpr (E == 4) {
        x[2] = __uint_as_float(w1 << 16);
        x[3] = __uint_as_float(w1 & 0xFFFF0000u);
      }
      float scale;
      const uint32_t packed =
          QM == kQuantI8 ? quant_row_int8<E>(x, &scale) : quant_row_fp8<E>(x, &scale);
      uint8_t* dst = static_cast<uint8_t*>(const_cast<void*>(t ? p.v_cache : p.k_cache)) +
                     row * HD + lane * E;
      if constexpr (E == 4)
        *reinterpret_cast<uint32_t*>(dst) = packed;
      else
        *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
      if (lane == 0) {
        float* sc = const_cast<float*>(t ? p.v_scale : p.k_scale);
        sc[((size_t)b * p.num_kv_heads + c.kvh) * bs + (pos & (bs - 1))] = scale;
      }
    }
  }
  __syncwarp();
}

// Physical block of token t (-1 when masked: past the range or bad block).
__device__ __forceinline__ int phys_of(const DecodeParams& p, const CtaSetup& c,
                                       const int* s_phys, int t) {
  return t < c.t_end ? s_phys[(t >> p.log2_bs) - c.blk0] : -1;
}

// Epilogue shared by both engines: merges the warps' (m, l, o) and writes the
// output (one split) or the split's normalised partial + log2-sum-exp.
// s_m/s_l: [NWARPS][GP]; s_o: [NWARPS][GP][HD]; s_w: [NWARPS][GP]; s_L: [GP].
template <int HD, int NWARPS, int GP>
__device__ __forceinline__ void combine_and_store(const DecodeParams& p, const CtaSetup& c,
                                                  float* s_m, float* s_l, float* s_o,
                                                  float* s_w, float* s_L) {
  const int G = p.group;
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) M = fmaxf(M, s_m[w * GP + h]);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) {
      const float mw = s_m[w * GP + h];
      const float wt = (mw == -CUDART_INF_F) ? 0.f : exp2f(mw - M);
      s_w[w * GP + h] = wt;
      L += wt * s_l[w * GP + h];
    }
    s_L[h] = L;
    if (!p.direct && threadIdx.x < G) {
      const size_t r = ((size_t)c.seq * p.num_q_heads + (size_t)c.kvh * G + h) * p.ws_slots +
                       p.ws_base + c.split;
      p.ws_lse[r] = (L > 0.f) ? M + log2f(L) : -CUDART_INF_F;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * HD; idx += NWARPS * kWarp) {
    const int h = idx / HD, d = idx % HD;
    const float L = s_L[h];
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) O += s_w[w * GP + h] * s_o[(w * GP + h) * HD + d];
    const float val = (L > 0.f) ? O / L : 0.f;
    const size_t qh = (size_t)c.kvh * G + h;
    if (p.direct) {
      const size_t o = ((size_t)c.seq * p.num_q_heads + qh) * HD + d;
      if (p.out_f32)
        static_cast<float*>(p.out)[o] = val;
      else
        static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(val);
    } else {
      const size_t o =
          (((size_t)c.seq * p.num_q_heads + qh) * p.ws_slots + p.ws_base + c.split) * HD + d;
      p.ws_o[o] = val;
    }
  }
}

// Writes zeros for a sequence with nothing to attend (only the split-0 CTA of
// a direct launch; the merge kernel covers the other cases).
template <int HD>
__device__ __forceinline__ void store_zero(const DecodeParams& p, const CtaSetup& c) {
  if (!p.direct || c.split != 0) return;
  const int G = p.group;
  for (int idx = threadIdx.x; idx < G * HD; idx += blockDim.x) {
    const int h = idx / HD, d = idx % HD;
    const size_t o = ((size_t)c.seq * p.num_q_heads + (size_t)c.kvh * G + h) * HD + d;
    if (p.out_f32)
      static_cast<float*>(p.out)[o] = 0.f;
    else
      static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(0.f);
  }
}


namespace {

// Raises a kernel's dynamic shared-memory limit once per (device, kernel) to
// the device's opt-in maximum; later launches skip the runtime call.  The
// cached limit is per kernel (the kernel is the template argument).  Racing
// first calls from several host threads set the same value.
constexpr int kMaxDevices = 64;

template <auto Kernel>
cudaError_t prepare(int smem) {
  static std::atomic<int> limit[kMaxDevices];  // raised limit per device, 0 = not yet
  if (smem <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (cached) {
    const int l = limit[dev].load(std::memory_order_acquire);
    if (l > 0) return smem <= l ? cudaSuccess : cudaErrorInvalidValue;
  }
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  if (smem > optin) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess && cached) limit[dev].store(optin, std::memory_order_release);
  return e;
}

// Shared memory of one sm_100 SM, and the part the hardware reserves per CTA.
constexpr int kSmemPerSm = 228 * 1024, kSmemPerCta = 1024;
// A dynamic shared-memory request above which at most three CTAs fit an SM.
constexpr int kThreeCtaSmem = kSmemPerSm / 4 - kSmemPerCta + 16;

}  // namespace

}  // namespace pkv
