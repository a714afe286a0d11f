// Paged decode attention for sm_100a.
//
// Operation ("大模型推理加速实战：KV Cache内存优化与PagedAttention分页管理方案",
// PagedAttention section; GQA grouping from "LLM推理显存优化KV Cache管理3大策略"
// §3): for every sequence and query head, attend over the sequence's tokens,
// fetching each token's K/V row through the block table.
//
// Work decomposition: one CTA per (kv_head, sequence, context split).  All
// `group` query heads that share a KV head live in the same CTA, so each K/V
// byte is read from HBM once.  Tiles are 16 tokens.  Each warp keeps an fp32
// online-softmax state in registers; the warps' states are merged through
// shared memory at the end.  With one split the CTA writes the output;
// otherwise it writes a normalised partial (o, log2-sum-exp) to the workspace
// and `merge_kernel` combines the splits.
//
// Two engines:
//  * mma (bf16, INT8 and FP8 caches): per-warp cp.async stage rings; each stage is
//    read into registers as soon as it lands and refilled at once; scores and
//    the PV update run on mma.sync m16n8k16 with fp32 accumulation.
//  * simt (fp32 caches): per-warp cp.async rings, fp32 FMA dot products, two
//    lanes per token.
#include <math_constants.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "decode.cuh"

namespace pkv {

struct CtaSetup {
  int seq, kvh, split;
  int ctx;             // the sequence's (clamped) context length
  int t_begin, t_end;  // token range of this CTA
  int blk0;            // first logical block in s_phys
  bool active;
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
  if (c.active) {
    const int nphys = ((c.t_end - 1) >> p.log2_bs) - c.blk0 + 1;
    const int32_t* row = p.block_tables + (size_t)c.seq * p.max_blocks_per_seq;
    for (int i = threadIdx.x; i < nphys; i += blockDim.x) {
      int b = row[c.blk0 + i];
      if (b < 0 || b >= p.num_blocks) {
        set_flag(p.err_flag, PKV_FLAG_BAD_BLOCK);
        b = -1;
      }
      s_phys[i] = b;
    }
  }
  __syncthreads();
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

// Issues the cp.async copies of one 16-token tile of the fp32 engine (K and V)
// into a stage of the calling warp's ring; one commit group per call.
template <int HD, int ELEM>
__device__ __forceinline__ void load_tile(const DecodeParams& p, const CtaSetup& c,
                                          const int* s_phys, int tile_t0, uint8_t* k_st,
                                          uint8_t* v_st, int lane) {
  constexpr int ROWB = HD * ELEM;
  constexpr int CH = ROWB / 16;
  constexpr int PER_LANE = 16 * CH / kWarp;
  const uint8_t* kb = static_cast<const uint8_t*>(p.k_cache);
  const uint8_t* vb = static_cast<const uint8_t*>(p.v_cache);
  const size_t head_off = (size_t)c.kvh * ROWB;
  const size_t tok_stride = (size_t)p.num_kv_heads * ROWB;
  const uint32_t ks = smem_u32(k_st), vs = smem_u32(v_st);
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int cid = lane + kWarp * i;
    const int row = cid / CH, ch = cid % CH;
    const int t = tile_t0 + row;
    const int phys = phys_of(p, c, s_phys, t);
    size_t off = 0;
    int n = 0;
    if (phys >= 0) {
      off = ((size_t)phys * p.block_size + (t & (p.block_size - 1))) * tok_stride + head_off +
            (size_t)ch * 16;
      n = 16;
    }
    const uint32_t so = (uint32_t)swz<CH>(row, ch) * 16;
    cp_async_16(ks + so, kb + off, n);
    cp_async_16(vs + so, vb + off, n);
  }
  cp_async_commit();
}

// ---------------------------------------------------------------------------
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


// ---------------------------------------------------------------------------
// mma engine: bf16, INT8 or FP8 caches, q in bf16.
//
// Each warp streams its own interleaved 16-token tiles (the warp's tile i is
// CTA tile warp + i * NWARPS) through a ring of NSTAGES cp.async stages.  As
// soon as a stage lands it is read into registers with ldmatrix and refilled
// with the warp's tile i + NSTAGES, so NSTAGES tiles per warp stay in flight
// while the math runs from registers.  The refill is issued through an asm
// block that depends on every loaded register, so it cannot overtake the
// reads of the stage it overwrites.
//
// Tile math: scores S^T = K * Q^T and the update O^T += V^T * P^T on
// mma.sync m16n8k16 with fp32 accumulation (16 tokens x 8 q heads per
// instruction).  For bf16 caches P is split into bf16 hi + lo halves so the
// probabilities keep ~16 significant bits.  One-byte caches feed V as fp16, so
// P goes in as one fp16 value (11 significant bits; its rounding error, below
// 2^-11 of each term, is under the bf16 rounding of the output).  INT8 codes
// become exact fp16 values in registers; the per-token scales multiply the
// fp32 scores (K) and P (V).  FP8 (E4M3) codes convert to exact fp16 with
// cvt.rn.f16x2.e4m3x2.  INT8 codes reach the tensor core as the exact fp16
// values code + 1152 (one byte permute per pair, no subtraction); the constant
// is removed from the fp32 results: 1152 * sum_d q[h][d] from every score, and
// 1152 * sum_t P[t][h] from the output, summed over the fp16 P the tensor core
// used so that it cancels exactly.

#ifndef PKV_MMA_WARPS
#define PKV_MMA_WARPS 4
#endif
#ifndef PKV_BF16_STAGES
#define PKV_BF16_STAGES 2
#endif
#ifndef PKV_I8_STAGES
#define PKV_I8_STAGES 3
#endif


template <int HD, int QM, int NT, int NWARPS, int NSTAGES>
struct MmaCfg {
  static constexpr int ELEM = QM != kQuantNone ? 1 : 2;
  static constexpr int ROWB = HD * ELEM;        // bytes of one token row of one head
  static constexpr int CH = ROWB / 16;          // 16-byte chunks per row: 4, 8 or 16
  static constexpr int RSTEP = kWarp / CH;      // rows one warp-wide copy covers
  static constexpr int PER_LANE = 16 / RSTEP;   // copies per lane per K (or V) tile
  static constexpr int TILE = 16 * ROWB;
  static constexpr int STAGE = 2 * TILE + (ELEM == 1 ? 128 : 0);
  static constexpr int RING = NWARPS * NSTAGES * STAGE;
  static constexpr int GP = NT * 8;
  static constexpr int COMB = (3 * NWARPS * GP + GP + NWARPS * GP * HD) * 4;
  static constexpr int BODY = RING > COMB ? RING : COMB;
  static_assert(CH == 4 || CH == 8 || CH == 16, "rows of 64, 128 or 256 bytes");
};

// Issues the copies of one 16-token tile (K, V and, for one-byte caches, the
// 16 per-token scales of each) into a stage, as one commit group.  Full tiles
// inside one block take the fast path: one block-table lookup, one 64-bit base
// per lane and fixed per-lane offsets.  Rows outside the sequence or in a bad
// block are zero-filled.  With AFTER, the stage address is derived from `dep`
// (see after_dep), so no copy overtakes the reads of the stage it overwrites.
template <class Cfg, bool AFTER>
__device__ __forceinline__ void issue_tile(const DecodeParams& p, const CtaSetup& c,
                                           const int* s_phys, int tile_t0, uint32_t k_st,
                                           uint32_t v_st, uint32_t sc_st, int lane,
                                           const uint32_t (&soff)[Cfg::PER_LANE],
                                           size_t lane_goff, int lane_row, uint32_t dep) {
  const uint8_t* kb = static_cast<const uint8_t*>(p.k_cache);
  const uint8_t* vb = static_cast<const uint8_t*>(p.v_cache);
  const size_t tok_stride = (size_t)p.num_kv_heads * Cfg::ROWB;
  const int bs = p.block_size;
  if constexpr (AFTER) {
    k_st = after_dep(k_st, dep);
    v_st = after_dep(v_st, dep);
    if constexpr (Cfg::ELEM == 1) sc_st = after_dep(sc_st, dep);
  }
  // scale row of this lane: lanes 0-15 copy K scales, 16-31 V scales
  const int srow = lane & 15;
  const float* ssrc = (lane < 16) ? p.k_scale : p.v_scale;
  if (bs >= 16 && tile_t0 + 16 <= c.t_end) {
    const int phys = s_phys[(tile_t0 >> p.log2_bs) - c.blk0];
    const int n = phys >= 0 ? 16 : 0;
    const int in_blk = tile_t0 & (bs - 1);
    // a bad block reads nothing (n = 0); its addresses stay inside the cache
    const size_t base = phys >= 0 ? ((size_t)phys * bs + in_blk) * tok_stride + lane_goff : 0;
    const size_t step = (size_t)Cfg::RSTEP * tok_stride;
    const uint8_t* kp = kb + base;
    const uint8_t* vp = vb + base;
#pragma unroll
    for (int i = 0; i < Cfg::PER_LANE; ++i) {
      cp_async_16(k_st + soff[i], kp + (size_t)i * step, n);
      cp_async_16(v_st + soff[i], vp + (size_t)i * step, n);
    }
    if constexpr (Cfg::ELEM == 1) {
      const size_t soff_g =
          phys >= 0 ? ((size_t)phys * p.num_kv_heads + c.kvh) * bs + in_blk + srow : 0;
      cp_async_4(sc_st + 4 * lane, ssrc + soff_g, phys >= 0 ? 4 : 0);
    }
  } else {
    const size_t lane_col = lane_goff - (size_t)lane_row * tok_stride;  // head + chunk offset
#pragma unroll
    for (int i = 0; i < Cfg::PER_LANE; ++i) {
      const int row = lane_row + i * Cfg::RSTEP;
      const int t = tile_t0 + row;
      const int phys = phys_of(p, c, s_phys, t);
      size_t off = 0;
      int n = 0;
      if (phys >= 0) {
        off = ((size_t)phys * bs + (t & (bs - 1))) * tok_stride + lane_col;
        n = 16;
      }
      cp_async_16(k_st + soff[i], kb + off, n);
      cp_async_16(v_st + soff[i], vb + off, n);
    }
    if constexpr (Cfg::ELEM == 1) {
      const int t = tile_t0 + srow;
      const int phys = phys_of(p, c, s_phys, t);
      size_t off = 0;
      int n = 0;
      if (phys >= 0) {
        off = ((size_t)phys * p.num_kv_heads + c.kvh) * bs + (t & (bs - 1));
        n = 4;
      }
      cp_async_4(sc_st + 4 * lane, ssrc + off, n);
    }
  }
  cp_async_commit();
}

template <int HD, int QM, int NT, int NWARPS, int NSTAGES, bool MHA>
__global__ void __launch_bounds__(NWARPS * kWarp)
    decode_mma_kernel(const DecodeParams p) {
  using Cfg = MmaCfg<HD, QM, NT, NWARPS, NSTAGES>;
  static_assert(!MHA || NT == 1, "MHA: one q head per kv head");
  constexpr bool I8 = QM == kQuantI8;
  constexpr bool F8 = QM == kQuantFp8;
  constexpr bool Q8 = I8 || F8;         // one-byte codes with per-token scales
  constexpr int KS = HD / 16;           // k-steps of the score mma
  constexpr int MT = HD / 16;           // m-tiles (16 head-dim rows) of the PV mma
  constexpr int KA = Q8 ? KS / 2 : KS;  // ldmatrix.x4 per K tile
  constexpr int VA = Q8 ? MT / 2 : MT;  // ldmatrix.x4 per V tile
  constexpr int GP = Cfg::GP;
  constexpr int CH = Cfg::CH;

  extern __shared__ __align__(128) uint8_t smem[];
  int* s_phys = reinterpret_cast<int*>(smem);
  uint8_t* ring = smem + p.phys_bytes;

  long long new_slot;
  const uint4 new_rows = fused_prefetch<HD, QM>(p, &new_slot);
  const CtaSetup c = cta_setup(p, s_phys);
  if (!c.active) {
    if (c.split == 0) {
      // a new token inside a shared prefix (positions below t_start) has no
      // CTA of this kernel to write it: report it instead
      if (p.new_k != nullptr && new_slot >= 0 && c.ctx >= 1 && c.ctx - 1 < p.t_start &&
          threadIdx.x == 0)
        set_flag(p.err_flag, PKV_FLAG_BAD_SLOT);
      store_zero<HD>(p, c);
    }
    return;
  }
  fused_commit<HD, QM, NWARPS>(p, c, s_phys, new_rows, new_slot);  // before any cache read
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int g = lane >> 2, t4 = lane & 3;
  const int G = p.group;

  // q as the B operand (n = head, k = head_dim), loaded once.
  uint32_t qf[KS][NT][2];
  {
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q) +
                              ((size_t)c.seq * p.num_q_heads + (size_t)c.kvh * G) * HD;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = nt * 8 + g;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t b0 = 0, b1 = 0;
        if (h < G) {
          const __nv_bfloat16* qr = qb + (size_t)h * HD;
          if constexpr (!Q8) {
            b0 = *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * t4);
            b1 = *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * t4 + 8);
          } else {
            // k-slot order of a one-byte-code chunk: slots 2t,2t+1 <- d 16c+4t+{0,1},
            // slots 2t+8,2t+9 <- d 16c+4t+{2,3}
            const uint2 raw = *reinterpret_cast<const uint2*>(qr + 16 * ks + 4 * t4);
            const float2 lo = unpack_bf16(raw.x), hi = unpack_bf16(raw.y);
            b0 = pack_f16(lo.x, lo.y);
            b1 = pack_f16(hi.x, hi.y);
          }
        }
        qf[ks][nt][0] = b0;
        qf[ks][nt][1] = b1;
      }
    }
  }

  // INT8: the tensor core sees code + 1152 instead of code (see
  // i8pair_to_f16x2_biased), so every score carries 1152 * sum_d q[h][d]; qbias
  // holds that term for this thread's two head columns 2*t4 and 2*t4 + 1.
  float qbias[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float mine = 0.f;  // partial sum over this lane's k-slots of head nt*8 + g
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const float2 a = unpack_f16(qf[ks][nt][0]), b = unpack_f16(qf[ks][nt][1]);
      mine += (a.x + a.y) + (b.x + b.y);
    }
    mine += __shfl_xor_sync(0xffffffffu, mine, 1);
    mine += __shfl_xor_sync(0xffffffffu, mine, 2);
#pragma unroll
    for (int j = 0; j < 2; ++j)
      qbias[nt][j] = I8 ? 1152.f * __shfl_sync(0xffffffffu, mine, (2 * t4 + j) * 4) : 0.f;
  }

  float o[MT][NT][4];
  float m_run[NT][2], l_run[NT][2], p_run[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      m_run[nt][j] = -CUDART_INF_F;
      l_run[nt][j] = 0.f;
      p_run[nt][j] = 0.f;  // INT8: sum of the P fed to the PV mma (for its 1152 bias)
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[mt][nt][j] = 0.f;
  }

  // Per-lane copy geometry: lane copies chunk lane % CH of rows
  // lane / CH + i * RSTEP; its shared-memory offsets are fixed.
  const int lane_row = lane / CH, lane_ch = lane % CH;
  uint32_t soff[Cfg::PER_LANE];
#pragma unroll
  for (int i = 0; i < Cfg::PER_LANE; ++i)
    soff[i] = (uint32_t)swz<CH>(lane_row + i * Cfg::RSTEP, lane_ch) * 16;
  const size_t tok_stride = (size_t)p.num_kv_heads * Cfg::ROWB;
  const size_t lane_goff =
      (size_t)lane_row * tok_stride + (size_t)c.kvh * Cfg::ROWB + (size_t)lane_ch * 16;

  // ldmatrix lane addressing: matrix j = lane/8 supplies its row lane%8.
  const int lm_row_a = (lane & 7) + ((lane >> 3) & 1) * 8;  // j: rows 0-7, 8-15, 0-7, 8-15
  const int lm_ch_a = lane >> 4;                            //    chunk +0, +0, +1, +1
  const int lm_row_v = (lane & 7) + ((lane >> 4) & 1) * 8;  // j: rows 0-7, 0-7, 8-15, 8-15
  const int lm_ch_v = (lane >> 3) & 1;                      //    chunk +0, +1, +0, +1
  uint32_t koff[KA], voff[VA];
#pragma unroll
  for (int i = 0; i < KA; ++i) koff[i] = (uint32_t)swz<CH>(lm_row_a, 2 * i + lm_ch_a) * 16;
#pragma unroll
  for (int i = 0; i < VA; ++i)
    voff[i] = Q8 ? (uint32_t)swz<CH>(lm_row_a, 2 * i + lm_ch_a) * 16
                 : (uint32_t)swz<CH>(lm_row_v, 2 * i + lm_ch_v) * 16;

  const uint32_t my_ring = smem_u32(ring) + (uint32_t)(warp * NSTAGES * Cfg::STAGE);
  const int ntiles = (c.t_end - c.t_begin + 15) >> 4;
  const int my_n = (warp < ntiles) ? (ntiles - warp + NWARPS - 1) / NWARPS : 0;

#pragma unroll
  for (int i = 0; i < NSTAGES; ++i) {
    const uint32_t st = my_ring + (uint32_t)(i * Cfg::STAGE);
    if (i < my_n)
      issue_tile<Cfg, false>(p, c, s_phys, c.t_begin + (warp + i * NWARPS) * 16, st,
                             st + Cfg::TILE, st + 2 * Cfg::TILE, lane, soff, lane_goff, lane_row,
                             0u);
    else
      cp_async_commit();
  }

  const uint32_t ring_last = my_ring + (uint32_t)((NSTAGES - 1) * Cfg::STAGE);
  uint32_t kS = my_ring;  // stage of tile i
  int tile_t0 = c.t_begin + warp * 16;
  for (int i = 0; i < my_n;
       ++i, tile_t0 += NWARPS * 16, kS = (kS == ring_last) ? my_ring : kS + Cfg::STAGE) {
    cp_async_wait<NSTAGES - 1>();
    __syncwarp();
    const uint32_t vS = kS + Cfg::TILE;

    // ---- read the stage into registers
    uint32_t kf[KA][4], vf[VA][4];
#pragma unroll
    for (int a = 0; a < KA; ++a) ldmatrix_x4(kS + koff[a], kf[a][0], kf[a][1], kf[a][2], kf[a][3]);
#pragma unroll
    for (int a = 0; a < VA; ++a)
      ldmatrix_x4_trans(vS + voff[a], vf[a][0], vf[a][1], vf[a][2], vf[a][3]);
    float ska = 0.f, skb = 0.f, sva = 0.f, svb = 0.f;
    uint32_t dep = 0;
    if constexpr (Q8) {
      float mine;
      asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(mine) : "r"(vS + Cfg::TILE + 4 * lane));
      ska = __shfl_sync(0xffffffffu, mine, g);
      skb = __shfl_sync(0xffffffffu, mine, g + 8);
      sva = __shfl_sync(0xffffffffu, mine, 16 + g);
      svb = __shfl_sync(0xffffffffu, mine, 24 + g);
      dep = __float_as_uint(mine);
    }
    // one register of each ldmatrix: an ldmatrix completes all of its registers at once
#pragma unroll
    for (int a = 0; a < KA; ++a) dep ^= kf[a][0];
#pragma unroll
    for (int a = 0; a < VA; ++a) dep ^= vf[a][0];
    const uint32_t mask =
        __ballot_sync(0xffffffffu, phys_of(p, c, s_phys, tile_t0 + (lane & 15)) >= 0) & 0xFFFFu;

    // ---- refill the stage with this warp's tile i + NSTAGES
    {
      const int ii = i + NSTAGES;
      if (ii < my_n)
        issue_tile<Cfg, true>(p, c, s_phys, tile_t0 + NSTAGES * NWARPS * 16, kS, vS,
                              vS + Cfg::TILE, lane, soff, lane_goff, lane_row, dep);
      else
        cp_async_commit();
    }
    if (mask == 0u) continue;

    // ---- scores S^T[token][head] = K * Q^T (two accumulator chains)
    float acc[NT][4], acc2[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[nt][q] = acc2[nt][q] = 0.f;
    if constexpr (!Q8) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (ks & 1)
            mma_bf16(acc2[nt], kf[ks][0], kf[ks][1], kf[ks][2], kf[ks][3], qf[ks][nt][0],
                     qf[ks][nt][1]);
          else
            mma_bf16(acc[nt], kf[ks][0], kf[ks][1], kf[ks][2], kf[ks][3], qf[ks][nt][0],
                     qf[ks][nt][1]);
        }
      }
    } else if constexpr (F8) {
#pragma unroll
      for (int kp = 0; kp < KS / 2; ++kp) {
        // kf[kp]: (rows 0-7, c) (rows 8-15, c) (0-7, c+1) (8-15, c+1); bytes of a
        // register are d 4t..4t+3 -> slots (2t, 2t+1) (its low half) and
        // (2t+8, 2t+9) (its high half), so each half converts as it is
        const uint32_t top[2] = {kf[kp][0], kf[kp][2]};
        const uint32_t bot[2] = {kf[kp][1], kf[kp][3]};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a0 = e4m3half_to_f16x2<true>(top[h]);
          const uint32_t a2 = e4m3half_to_f16x2<false>(top[h]);
          const uint32_t a1 = e4m3half_to_f16x2<true>(bot[h]);
          const uint32_t a3 = e4m3half_to_f16x2<false>(bot[h]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (h)
              mma_f16(acc2[nt], a0, a1, a2, a3, qf[2 * kp + h][nt][0], qf[2 * kp + h][nt][1]);
            else
              mma_f16(acc[nt], a0, a1, a2, a3, qf[2 * kp + h][nt][0], qf[2 * kp + h][nt][1]);
          }
        }
      }
    } else {
#pragma unroll
      for (int kp = 0; kp < KS / 2; ++kp) {
        // kf[kp]: (rows 0-7, c) (rows 8-15, c) (0-7, c+1) (8-15, c+1)
        const uint32_t top[2] = {kf[kp][0] ^ 0x80808080u, kf[kp][2] ^ 0x80808080u};
        const uint32_t bot[2] = {kf[kp][1] ^ 0x80808080u, kf[kp][3] ^ 0x80808080u};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a0 = i8pair_to_f16x2_biased<0x4140>(top[h]);
          const uint32_t a2 = i8pair_to_f16x2_biased<0x4342>(top[h]);
          const uint32_t a1 = i8pair_to_f16x2_biased<0x4140>(bot[h]);
          const uint32_t a3 = i8pair_to_f16x2_biased<0x4342>(bot[h]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (h)
              mma_f16(acc2[nt], a0, a1, a2, a3, qf[2 * kp + h][nt][0], qf[2 * kp + h][nt][1]);
            else
              mma_f16(acc[nt], a0, a1, a2, a3, qf[2 * kp + h][nt][0], qf[2 * kp + h][nt][1]);
          }
        }
      }
    }

    // ---- mask, scale, online softmax (tokens g, g+8; heads 2t4, 2t4+1)
    const bool va = (mask >> g) & 1u, vb = (mask >> (g + 8)) & 1u;
    float fa = p.scale_log2, fb = p.scale_log2;
    float pva = 1.f, pvb = 1.f;
    if constexpr (Q8) {
      fa = va ? fa * fast_rcp(ska) : 0.f;
      fb = vb ? fb * fast_rcp(skb) : 0.f;
      pva = va ? fast_rcp(sva) : 0.f;
      pvb = vb ? fast_rcp(svb) : 0.f;
    }
    uint32_t bh[NT][2], bl[NT][2];
    float alpha[NT][2];
    bool rescale = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pr[4];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        if (MHA && jj == 1) {  // one q head per kv head: column 2*t4 + 1 holds none
          pr[1] = pr[3] = 0.f;
          alpha[nt][1] = 1.f;
          continue;
        }
        // scores of head 2*t4 + jj for tokens g (sa) and g + 8 (sb)
        const float sa =
            va ? ((acc[nt][jj] + acc2[nt][jj]) - qbias[nt][jj]) * fa : -CUDART_INF_F;
        const float sb =
            vb ? ((acc[nt][jj + 2] + acc2[nt][jj + 2]) - qbias[nt][jj]) * fb : -CUDART_INF_F;
        float mx = fmaxf(sa, sb);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[nt][jj], mx);
        const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
        const float a = fast_exp2(m_run[nt][jj] - m_use);
        pr[jj] = fast_exp2(sa - m_use);
        pr[jj + 2] = fast_exp2(sb - m_use);
        l_run[nt][jj] = l_run[nt][jj] * a + pr[jj] + pr[jj + 2];
        m_run[nt][jj] = m_new;
        alpha[nt][jj] = a;
        rescale |= (a != 1.f);
      }
      const float q0 = pr[0] * pva, q1 = pr[1] * pva, q2 = pr[2] * pvb, q3 = pr[3] * pvb;
      if constexpr (!Q8) {
        const uint32_t h01 = pack_bf16(q0, q1), h23 = pack_bf16(q2, q3);
        const float2 f01 = unpack_bf16(h01), f23 = unpack_bf16(h23);
        bh[nt][0] = movmatrix_trans(h01);
        bh[nt][1] = movmatrix_trans(h23);
        bl[nt][0] = movmatrix_trans(pack_bf16(q0 - f01.x, q1 - f01.y));
        bl[nt][1] = movmatrix_trans(pack_bf16(q2 - f23.x, q3 - f23.y));
      } else {
        const uint32_t h01 = pack_f16(q0, q1), h23 = pack_f16(q2, q3);
        if constexpr (I8) {  // the P the tensor core sees, for the 1152 bias
          const float2 f01 = unpack_f16(h01), f23 = unpack_f16(h23);
          p_run[nt][0] = p_run[nt][0] * alpha[nt][0] + (f01.x + f23.x);
          p_run[nt][1] = p_run[nt][1] * alpha[nt][1] + (f01.y + f23.y);
        }
        bh[nt][0] = movmatrix_trans(h01);
        bh[nt][1] = movmatrix_trans(h23);
      }
    }
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[mt][nt][0] *= alpha[nt][0];
          o[mt][nt][2] *= alpha[nt][0];
          o[mt][nt][1] *= alpha[nt][1];
          o[mt][nt][3] *= alpha[nt][1];
        }
    }

    // ---- O^T[d][head] += V^T * P^T
    if constexpr (!Q8) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_bf16(o[mt][nt], vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3], bh[nt][0], bh[nt][1]);
          mma_bf16(o[mt][nt], vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3], bl[nt][0], bl[nt][1]);
        }
      }
    } else if constexpr (F8) {
#pragma unroll
      for (int mp = 0; mp < MT / 2; ++mp) {
        // vf[mp] transposed: a register holds bytes (t 2t, d 2g) (2t, 2g+1)
        // (2t+1, 2g) (2t+1, 2g+1); rows m <-> d as in the INT8 case
        const uint32_t top[2] = {vf[mp][0], vf[mp][2]};
        const uint32_t bot[2] = {vf[mp][1], vf[mp][3]};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a0 = e4m3pair_to_f16x2<0x0020>(top[h]);
          const uint32_t a1 = e4m3pair_to_f16x2<0x0031>(top[h]);
          const uint32_t a2 = e4m3pair_to_f16x2<0x0020>(bot[h]);
          const uint32_t a3 = e4m3pair_to_f16x2<0x0031>(bot[h]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_f16(o[2 * mp + h][nt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
          }
        }
      }
    } else {
#pragma unroll
      for (int mp = 0; mp < MT / 2; ++mp) {
        // vf[mp]: (rows 0-7, c) (rows 8-15, c) (0-7, c+1) (8-15, c+1), transposed
        const uint32_t top[2] = {vf[mp][0] ^ 0x80808080u, vf[mp][2] ^ 0x80808080u};
        const uint32_t bot[2] = {vf[mp][1] ^ 0x80808080u, vf[mp][3] ^ 0x80808080u};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // rows m <-> d: m = g -> 16c + 2g, m = g + 8 -> 16c + 2g + 1
          const uint32_t a0 = i8pair_to_f16x2_biased<0x4240>(top[h]);
          const uint32_t a1 = i8pair_to_f16x2_biased<0x4341>(top[h]);
          const uint32_t a2 = i8pair_to_f16x2_biased<0x4240>(bot[h]);
          const uint32_t a3 = i8pair_to_f16x2_biased<0x4341>(bot[h]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_f16(o[2 * mp + h][nt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
          }
        }
      }
    }
  }
  cp_async_wait<0>();

  if constexpr (I8) {
    // O carries 1152 * sum_t P[t][h] from the biased V codes: remove it.
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float ps = p_run[nt][j];
        ps += __shfl_xor_sync(0xffffffffu, ps, 4);
        ps += __shfl_xor_sync(0xffffffffu, ps, 8);
        ps += __shfl_xor_sync(0xffffffffu, ps, 16);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          o[mt][nt][j] -= 1152.f * ps;
          o[mt][nt][j + 2] -= 1152.f * ps;
        }
      }
  }

  // ---- per-warp final state -> smem (the ring is reused: wait for every warp)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float l = l_run[nt][j];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      l_run[nt][j] = l;
    }
  __syncthreads();
  float* s_m = reinterpret_cast<float*>(ring);
  float* s_l = s_m + NWARPS * GP;
  float* s_w = s_l + NWARPS * GP;
  float* s_L = s_w + NWARPS * GP;
  float* s_o = s_L + GP;
  if (g == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        s_m[warp * GP + nt * 8 + 2 * t4 + j] = m_run[nt][j];
        s_l[warp * GP + nt * 8 + 2 * t4 + j] = l_run[nt][j];
      }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int m = g + (j >> 1) * 8;  // fragment row
        const int h = nt * 8 + 2 * t4 + (j & 1);
        const int d = Q8 ? 16 * mt + (m < 8 ? 2 * m : 2 * (m - 8) + 1) : 16 * mt + m;
        s_o[(warp * GP + h) * HD + d] = o[mt][nt][j];
      }
  combine_and_store<HD, NWARPS, GP>(p, c, s_m, s_l, s_o, s_w, s_L);
}

// ---------------------------------------------------------------------------
// simt engine: fp32 caches, q in fp32 or bf16.  Lanes l and l+16 share token
// l%16, each summing half of head_dim; the PV update gives lane l the head_dim
// columns l, l+32, ...
template <int HD, int NWARPS, int NSTAGES>
__global__ void __launch_bounds__(NWARPS * kWarp)
    decode_simt_kernel(const DecodeParams p) {
  constexpr int ELEM = 4;
  constexpr int ROWB = HD * ELEM;
  constexpr int CH = ROWB / 16;
  constexpr int TILE_B = 16 * ROWB;
  constexpr int STAGE_B = 2 * TILE_B;
  constexpr int GP = 16;
  constexpr int DJ = HD / kWarp;

  extern __shared__ __align__(128) uint8_t smem[];
  int* s_phys = reinterpret_cast<int*>(smem);
  float* s_q = reinterpret_cast<float*>(smem + p.phys_bytes);  // [GP][HD]
  uint8_t* ring = smem + p.phys_bytes + GP * HD * 4;

  const CtaSetup c = cta_setup(p, s_phys);
  if (!c.active) {
    if (c.split == 0) store_zero<HD>(p, c);
    return;
  }
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int G = p.group;
  {
    const size_t qbase = ((size_t)c.seq * p.num_q_heads + (size_t)c.kvh * G) * HD;
    for (int idx = threadIdx.x; idx < G * HD; idx += blockDim.x) {
      float v;
      if (p.q_f32)
        v = static_cast<const float*>(p.q)[qbase + idx];
      else
        v = __bfloat162float(static_cast<const __nv_bfloat16*>(p.q)[qbase + idx]);
      s_q[idx] = v;
    }
  }
  __syncthreads();

  float o[GP][DJ];
  float m_run[GP], l_run[GP];
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    m_run[h] = -CUDART_INF_F;
    l_run[h] = 0.f;
#pragma unroll
    for (int j = 0; j < DJ; ++j) o[h][j] = 0.f;
  }

  uint8_t* my_ring = ring + (size_t)warp * NSTAGES * STAGE_B;
  const int ntiles = (c.t_end - c.t_begin + 15) >> 4;
  const int my_n = (warp < ntiles) ? (ntiles - warp + NWARPS - 1) / NWARPS : 0;
#pragma unroll
  for (int i = 0; i < NSTAGES - 1; ++i) {
    if (i < my_n)
      load_tile<HD, ELEM>(p, c, s_phys, c.t_begin + (warp + i * NWARPS) * 16,
                          my_ring + (size_t)i * STAGE_B, my_ring + (size_t)i * STAGE_B + TILE_B,
                          lane);
    else
      cp_async_commit();
  }
  const int tr = lane & 15, hf = lane >> 4;
  for (int i = 0; i < my_n; ++i) {
    {
      const int ii = i + NSTAGES - 1;
      if (ii < my_n) {
        uint8_t* st = my_ring + (size_t)(ii % NSTAGES) * STAGE_B;
        load_tile<HD, ELEM>(p, c, s_phys, c.t_begin + (warp + ii * NWARPS) * 16, st,
                            st + TILE_B, lane);
      } else {
        cp_async_commit();
      }
    }
    cp_async_wait<NSTAGES - 1>();
    __syncwarp();
    const uint8_t* kt = my_ring + (size_t)(i % NSTAGES) * STAGE_B;
    const uint8_t* vt = kt + TILE_B;
    const int tile_t0 = c.t_begin + (warp + i * NWARPS) * 16;
    const bool valid = phys_of(p, c, s_phys, tile_t0 + tr) >= 0;

    float s[GP];
#pragma unroll
    for (int h = 0; h < GP; ++h) s[h] = 0.f;
#pragma unroll
    for (int cc = 0; cc < CH / 2; ++cc) {
      const int ch = hf * (CH / 2) + cc;
      const float4 kv = *reinterpret_cast<const float4*>(kt + swz<CH>(tr, ch) * 16);
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        if (h < G) {
          const float4 qv = *reinterpret_cast<const float4*>(s_q + h * HD + ch * 4);
          s[h] = fmaf(qv.x, kv.x, s[h]);
          s[h] = fmaf(qv.y, kv.y, s[h]);
          s[h] = fmaf(qv.z, kv.z, s[h]);
          s[h] = fmaf(qv.w, kv.w, s[h]);
        }
      }
    }
    float pr[GP];
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      if (h < G) {
        float sv = s[h] + __shfl_xor_sync(0xffffffffu, s[h], 16);
        sv = valid ? sv * p.scale_log2 : -CUDART_INF_F;
        float mx = sv;
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        const float m_new = fmaxf(m_run[h], mx);
        const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
        const float alpha = exp2f(m_run[h] - m_use);
        pr[h] = exp2f(sv - m_use);
        l_run[h] = l_run[h] * alpha + (hf == 0 ? pr[h] : 0.f);
        m_run[h] = m_new;
#pragma unroll
        for (int j = 0; j < DJ; ++j) o[h][j] *= alpha;
      }
    }
#pragma unroll 4
    for (int t = 0; t < 16; ++t) {
      float vv[DJ];
#pragma unroll
      for (int j = 0; j < DJ; ++j) {
        const int e = lane + kWarp * j;
        vv[j] = *reinterpret_cast<const float*>(vt + swz<CH>(t, e >> 2) * 16 + (e & 3) * 4);
      }
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        if (h < G) {
          const float pt = __shfl_sync(0xffffffffu, pr[h], t);
#pragma unroll
          for (int j = 0; j < DJ; ++j) o[h][j] = fmaf(pt, vv[j], o[h][j]);
        }
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    float l = l_run[h];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    l_run[h] = l;
  }
  __syncthreads();
  float* s_m = reinterpret_cast<float*>(ring);
  float* s_l = s_m + NWARPS * GP;
  float* s_w = s_l + NWARPS * GP;
  float* s_L = s_w + NWARPS * GP;
  float* s_o = s_L + GP;
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      s_m[warp * GP + h] = m_run[h];
      s_l[warp * GP + h] = l_run[h];
    }
  }
#pragma unroll
  for (int h = 0; h < GP; ++h)
    if (h < G)
#pragma unroll
      for (int j = 0; j < DJ; ++j) s_o[(warp * GP + h) * HD + lane + kWarp * j] = o[h][j];
  combine_and_store<HD, NWARPS, GP>(p, c, s_m, s_l, s_o, s_w, s_L);
}

// ---------------------------------------------------------------------------
// Split merge: out = sum_k 2^{lse_k} o_k / sum_k 2^{lse_k} over the partials
// of one (sequence, q head): the shared-prefix slots [0, ws_base) and the
// splits that hold tokens (every one of them was written, so all are finite).
// One warp per (q head, sequence); lane l sums head_dim columns 4l..4l+3 of the
// weighted partials with 16-byte loads.  The first kMergeBatch partial rows are
// loaded before the weights are known, so their latency overlaps the
// log-sum-exp reads; the weights are held one per lane and broadcast with
// shuffles, 32 slots per round.
constexpr int kMergeWarps = 4;
constexpr int kMergeBatch = 8;  // partial rows in flight per lane

template <int HD>
__global__ void __launch_bounds__(kMergeWarps* kWarp) merge_kernel(const DecodeParams p) {
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int qh = blockIdx.x * kMergeWarps + warp, seq = blockIdx.y;
  if (qh >= p.num_q_heads) return;
  const int ctx = effective_ctx(p, seq, false);
  const int rest = ctx > p.t_start ? ctx - p.t_start : 0;
  const int n = p.ws_base + (rest + p.chunk - 1) / p.chunk;
  const size_t r = ((size_t)seq * p.num_q_heads + qh) * p.ws_slots;
  const bool cols = lane * 4 < HD;
  const float4* src = reinterpret_cast<const float4*>(p.ws_o + r * HD) + lane;
  constexpr int kRow = HD / 4;  // float4 per partial row

  float4 v[kMergeBatch];
#pragma unroll
  for (int i = 0; i < kMergeBatch; ++i)
    if (cols && i < n) v[i] = src[(size_t)i * kRow];
  float M = -CUDART_INF_F;
  for (int k = lane; k < n; k += kWarp) M = fmaxf(M, p.ws_lse[r + k]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float L = 0.f;
  if (M != -CUDART_INF_F) {
    for (int base = 0; base < n; base += kWarp) {
      const int cnt = min(n - base, kWarp);
      const float lse = lane < cnt ? p.ws_lse[r + base + lane] : -CUDART_INF_F;
      const float w = lse == -CUDART_INF_F ? 0.f : exp2f(lse - M);
      float ws = w;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, off);
      L += ws;
      for (int k0 = 0; k0 < cnt; k0 += kMergeBatch) {
        if (base + k0 >= kMergeBatch) {  // the first batch is already in registers
#pragma unroll
          for (int i = 0; i < kMergeBatch; ++i)
            if (cols && k0 + i < cnt) v[i] = src[(size_t)(base + k0 + i) * kRow];
        }
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
          const float wk = __shfl_sync(0xffffffffu, w, (k0 + i) & (kWarp - 1));
          if (k0 + i < cnt) {
            acc[0] += wk * v[i].x;
            acc[1] += wk * v[i].y;
            acc[2] += wk * v[i].z;
            acc[3] += wk * v[i].w;
          }
        }
      }
    }
  }
  if (!cols) return;
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const size_t o = ((size_t)seq * p.num_q_heads + qh) * HD + lane * 4;
  if (p.out_f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(p.out) + o) =
        make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  } else {
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(p.out) + o;
    *reinterpret_cast<uint2*>(ob) =
        make_uint2(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv));
  }
}

// ---------------------------------------------------------------------------
// Host side: kernel selection and launch.

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

template <int HD, int QM, int NT, int NWARPS, int NSTAGES, bool MHA>
cudaError_t launch_mma(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  using Cfg = MmaCfg<HD, QM, NT, NWARPS, NSTAGES>;
  int smem = p.phys_bytes + Cfg::BODY;
  // The one-byte MHA kernels at head_dim 128 fit four CTAs per SM by
  // registers, the other one-byte kernels three.  Held to three as well, the
  // FP8 13B workload ran 3% faster (INT8 within 1%), and the split planner's
  // occupancy figure (taken from the general kernel) stays exact.
  if constexpr (MHA && QM != kQuantNone && HD == 128)
    smem = smem > kThreeCtaSmem ? smem : kThreeCtaSmem;
  constexpr auto k = decode_mma_kernel<HD, QM, NT, NWARPS, NSTAGES, MHA>;
  cudaError_t e = prepare<k>(smem);
  if (e != cudaSuccess) return e;
  k<<<grid, NWARPS * kWarp, smem, st>>>(p);
  return cudaGetLastError();
}

template <int HD, int NWARPS, int NSTAGES>
cudaError_t launch_simt(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  constexpr int STAGE_B = 2 * 16 * HD * 4;
  constexpr int RING = NWARPS * NSTAGES * STAGE_B;
  constexpr int GP = 16;
  constexpr int COMB = (3 * NWARPS * GP + GP + NWARPS * GP * HD) * 4;
  const int smem = p.phys_bytes + GP * HD * 4 + (RING > COMB ? RING : COMB);
  constexpr auto k = decode_simt_kernel<HD, NWARPS, NSTAGES>;
  cudaError_t e = prepare<k>(smem);
  if (e != cudaSuccess) return e;
  k<<<grid, NWARPS * kWarp, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

constexpr int kF32Warps = 4, kF32Stages = 2;
constexpr int kMW = PKV_MMA_WARPS;

namespace {

template <auto Kernel>
int occupancy(int threads, int smem) {
  static std::atomic<int> cached[kMaxDevices];  // resident CTAs per SM, 0 = not yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
  int n = cached[dev].load(std::memory_order_acquire);
  if (n > 0) return n;
  if (prepare<Kernel>(smem) != cudaSuccess) return 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, threads, smem) != cudaSuccess ||
      n < 1)
    n = 1;
  cached[dev].store(n, std::memory_order_release);
  return n;
}

constexpr int kTypicalPhysBytes = 1024;  // block-table slice of a typical split

template <int HD, int QM>
int mma_occupancy() {
  constexpr int NS = QM != kQuantNone ? PKV_I8_STAGES : PKV_BF16_STAGES;
  using Cfg = MmaCfg<HD, QM, 1, kMW, NS>;
  return occupancy<decode_mma_kernel<HD, QM, 1, kMW, NS, false>>(kMW * kWarp,
                                                          kTypicalPhysBytes + Cfg::BODY);
}

}  // namespace

int decode_ctas_per_sm_hint(pkv_dtype cache_dt, int head_dim) {
  if (cache_dt == PKV_BF16) return head_dim == 128 ? mma_occupancy<128, kQuantNone>()
                                                   : mma_occupancy<64, kQuantNone>();
  if (cache_dt == PKV_I8) return head_dim == 128 ? mma_occupancy<128, kQuantI8>()
                                                 : mma_occupancy<64, kQuantI8>();
  if (cache_dt == PKV_FP8) return head_dim == 128 ? mma_occupancy<128, kQuantFp8>()
                                                  : mma_occupancy<64, kQuantFp8>();
  const int smem = kF32Warps * kF32Stages * 2 * 16 * head_dim * 4 + 16 * head_dim * 4 + 1024;
  const int n = kSmemPerSm / (smem + kSmemPerCta);
  return n < 1 ? 1 : n;
}

namespace {

// Picks the q-head tiling: two n-tiles for groups above 8, the MHA form for a
// group of one, else one n-tile.
template <int HD, int QM, int NS>
cudaError_t launch_mma_group(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  if (p.group > 8) return launch_mma<HD, QM, 2, kMW, NS, false>(p, grid, st);
  if (p.group == 1) return launch_mma<HD, QM, 1, kMW, NS, true>(p, grid, st);
  return launch_mma<HD, QM, 1, kMW, NS, false>(p, grid, st);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, pkv_dtype cache_dt, int head_dim,
                          cudaStream_t st) {
  dim3 grid(p.num_kv_heads, p.num_seqs, p.num_splits);
  if (cache_dt == PKV_BF16)
    return head_dim == 128 ? launch_mma_group<128, kQuantNone, PKV_BF16_STAGES>(p, grid, st)
                           : launch_mma_group<64, kQuantNone, PKV_BF16_STAGES>(p, grid, st);
  if (cache_dt == PKV_I8)
    return head_dim == 128 ? launch_mma_group<128, kQuantI8, PKV_I8_STAGES>(p, grid, st)
                           : launch_mma_group<64, kQuantI8, PKV_I8_STAGES>(p, grid, st);
  if (cache_dt == PKV_FP8)
    return head_dim == 128 ? launch_mma_group<128, kQuantFp8, PKV_I8_STAGES>(p, grid, st)
                           : launch_mma_group<64, kQuantFp8, PKV_I8_STAGES>(p, grid, st);
  if (head_dim == 128) return launch_simt<128, kF32Warps, kF32Stages>(p, grid, st);
  return launch_simt<64, kF32Warps, kF32Stages>(p, grid, st);
}

cudaError_t launch_merge(const DecodeParams& p, int head_dim, cudaStream_t st) {
  dim3 grid((p.num_q_heads + kMergeWarps - 1) / kMergeWarps, p.num_seqs);
  if (head_dim == 128)
    merge_kernel<128><<<grid, kMergeWarps * kWarp, 0, st>>>(p);
  else
    merge_kernel<64><<<grid, kMergeWarps * kWarp, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
