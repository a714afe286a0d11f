// Paged decode attention for sm_100a.
//
// Operation ("大模型推理加速实战：KV Cache内存优化与PagedAttention分页管理方案",
// PagedAttention section; GQA grouping from "LLM推理显存优化KV Cache管理3大策略"
// §3): for every sequence and query head, attend over the sequence's tokens,
// fetching each token's K/V row through the block table.
//
// Work decomposition: one CTA per (kv_head, sequence, context split).  All
// `group` query heads that share a KV head live in the same CTA, so each K/V
// byte is read from HBM once.  Inside a CTA every warp owns an interleaved
// subset of 16-token tiles and streams them through its own cp.async ring in
// shared memory (16-byte coalesced row segments, zero-fill for masked rows),
// keeps an fp32 online-softmax state in registers, and the warps' states are
// merged through shared memory at the end.  With one split the CTA writes the
// output; otherwise it writes a normalised partial (o, log2-sum-exp) to the
// workspace and `merge_kernel` combines the splits.
//
// Two tile engines:
//  * mma (bf16 and int8 caches): scores S^T = K * Q^T and the update
//    O^T += V^T * P^T run on mma.sync m16n8k16 with fp32 accumulation, 16
//    tokens x 8 heads per instruction.  P is split into hi + lo halves so the
//    probabilities keep ~16 significant bits.  INT8 codes are converted to
//    exact fp16 values in registers and the per-token scales are applied to the
//    fp32 scores (K) and to P (V).
//  * simt (fp32 caches): fp32 FMA dot products, 2 lanes per token.
#include <math_constants.h>

#include <atomic>

#include "common.cuh"
#include "decode.cuh"

namespace pkv {

// Smem index of the 16-byte chunk `ch` of tile row `row` (rows of CH chunks).
// XOR-swizzle so that the 8 rows an ldmatrix phase reads hit 8 distinct bank
// groups.
template <int CH>
__device__ __forceinline__ int swz(int row, int ch) {
  if constexpr (CH >= 8) {
    return row * CH + (ch ^ (row & 7));
  } else {
    static_assert(CH == 4, "rows of 4 or a multiple of 8 chunks");
    return row * CH + (ch ^ ((row >> 1) & 3));
  }
}

struct CtaSetup {
  int seq, kvh, split;
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
  const long long cap_split = (long long)p.num_splits * p.chunk;
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
  c.t_begin = c.split * p.chunk;
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

// Physical block of token t (-1 when masked: past the range or bad block).
__device__ __forceinline__ int phys_of(const DecodeParams& p, const CtaSetup& c,
                                       const int* s_phys, int t) {
  return t < c.t_end ? s_phys[(t >> p.log2_bs) - c.blk0] : -1;
}

// Issues the cp.async copies of one 16-token tile (K and V, plus INT8 scales)
// into a stage of the calling warp's ring; one commit group per call.
template <int HD, int ELEM, bool I8>
__device__ __forceinline__ void load_tile(const DecodeParams& p, const CtaSetup& c,
                                          const int* s_phys, int tile_t0, uint8_t* k_st,
                                          uint8_t* v_st, float* sc_st, int lane) {
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
  if constexpr (I8) {
    const int row = lane & 15;
    const int t = tile_t0 + row;
    const int phys = phys_of(p, c, s_phys, t);
    const float* src = (lane < 16) ? p.k_scale : p.v_scale;
    size_t off = 0;
    int n = 0;
    if (phys >= 0) {
      off = ((size_t)phys * p.num_kv_heads + c.kvh) * p.block_size + (t & (p.block_size - 1));
      n = 4;
    }
    cp_async_4(smem_u32(sc_st + lane), src + off, n);
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
    if (p.num_splits > 1 && threadIdx.x < G) {
      const size_t r = ((size_t)c.seq * p.num_q_heads + (size_t)c.kvh * G + h) * p.num_splits +
                       c.split;
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
    if (p.num_splits == 1) {
      const size_t o = ((size_t)c.seq * p.num_q_heads + qh) * HD + d;
      if (p.out_f32)
        static_cast<float*>(p.out)[o] = val;
      else
        static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(val);
    } else {
      const size_t o =
          (((size_t)c.seq * p.num_q_heads + qh) * p.num_splits + c.split) * HD + d;
      p.ws_o[o] = val;
    }
  }
}

// Writes zeros for a sequence with nothing to attend (only the split-0 CTA of
// a single-split launch; the merge kernel covers the multi-split case).
template <int HD>
__device__ __forceinline__ void store_zero(const DecodeParams& p, const CtaSetup& c) {
  if (p.num_splits != 1 || c.split != 0) return;
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
// mma engine: bf16 or int8 caches, q in bf16.
template <int HD, bool I8, int NT, int NWARPS, int NSTAGES>
__global__ void __launch_bounds__(NWARPS * kWarp)
    decode_mma_kernel(const DecodeParams p) {
  constexpr int ELEM = I8 ? 1 : 2;
  constexpr int ROWB = HD * ELEM;
  constexpr int CH = ROWB / 16;
  constexpr int TILE_B = 16 * ROWB;
  constexpr int STAGE_B = 2 * TILE_B + (I8 ? 128 : 0);
  constexpr int KS = HD / 16;  // k-steps of the score mma
  constexpr int MT = HD / 16;  // m-tiles (16 head-dim rows) of the PV mma
  constexpr int GP = NT * 8;

  extern __shared__ __align__(128) uint8_t smem[];
  int* s_phys = reinterpret_cast<int*>(smem);
  uint8_t* ring = smem + p.phys_bytes;

  const CtaSetup c = cta_setup(p, s_phys);
  if (!c.active) {
    if (c.split == 0) store_zero<HD>(p, c);
    return;
  }
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
          if constexpr (!I8) {
            b0 = *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * t4);
            b1 = *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * t4 + 8);
          } else {
            // k-slot order of an int8 chunk: slots 2t,2t+1 <- d 16c+4t+{0,1},
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

  float o[MT][NT][4];
  float m_run[NT][2], l_run[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      m_run[nt][j] = -CUDART_INF_F;
      l_run[nt][j] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[mt][nt][j] = 0.f;
  }

  uint8_t* my_ring = ring + (size_t)warp * NSTAGES * STAGE_B;
  const int ntiles = (c.t_end - c.t_begin + 15) >> 4;
  const int my_n = (warp < ntiles) ? (ntiles - warp + NWARPS - 1) / NWARPS : 0;

  auto stage_k = [&](int s) { return my_ring + (size_t)s * STAGE_B; };
  auto stage_v = [&](int s) { return my_ring + (size_t)s * STAGE_B + TILE_B; };
  auto stage_sc = [&](int s) {
    return reinterpret_cast<float*>(my_ring + (size_t)s * STAGE_B + 2 * TILE_B);
  };

#pragma unroll
  for (int i = 0; i < NSTAGES - 1; ++i) {
    if (i < my_n)
      load_tile<HD, ELEM, I8>(p, c, s_phys, c.t_begin + (warp + i * NWARPS) * 16, stage_k(i),
                              stage_v(i), stage_sc(i), lane);
    else
      cp_async_commit();
  }

  // ldmatrix lane addressing: matrix j = lane/8 supplies its row lane%8.
  const int lm_row_a = (lane & 7) + ((lane >> 3) & 1) * 8;  // j: rows 0-7, 8-15, 0-7, 8-15
  const int lm_ch_a = lane >> 4;                            //    chunk +0, +0, +1, +1
  const int lm_row_v = (lane & 7) + ((lane >> 4) & 1) * 8;  // j: rows 0-7, 0-7, 8-15, 8-15
  const int lm_ch_v = (lane >> 3) & 1;                      //    chunk +0, +1, +0, +1

  for (int i = 0; i < my_n; ++i) {
    {
      const int ii = i + NSTAGES - 1;
      if (ii < my_n)
        load_tile<HD, ELEM, I8>(p, c, s_phys, c.t_begin + (warp + ii * NWARPS) * 16,
                                stage_k(ii % NSTAGES), stage_v(ii % NSTAGES),
                                stage_sc(ii % NSTAGES), lane);
      else
        cp_async_commit();
    }
    cp_async_wait<NSTAGES - 1>();
    __syncwarp();

    const int st = i % NSTAGES;
    const uint32_t kS = smem_u32(stage_k(st));
    const uint32_t vS = smem_u32(stage_v(st));
    const float* sc = stage_sc(st);
    const int tile_t0 = c.t_begin + (warp + i * NWARPS) * 16;

    // ---- scores S^T[token][head] = K * Q^T
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[nt][j] = 0.f;
    if constexpr (!I8) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(kS + swz<CH>(lm_row_a, 2 * ks + lm_ch_a) * 16, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_bf16(acc[nt], a0, a1, a2, a3, qf[ks][nt][0], qf[ks][nt][1]);
      }
    } else {
#pragma unroll
      for (int kp = 0; kp < KS / 2; ++kp) {
        uint32_t r0, r1, r2, r3;  // (rows 0-7, c) (rows 8-15, c) (0-7, c+1) (8-15, c+1)
        ldmatrix_x4(kS + swz<CH>(lm_row_a, 2 * kp + lm_ch_a) * 16, r0, r1, r2, r3);
        const uint32_t top[2] = {r0 ^ 0x80808080u, r2 ^ 0x80808080u};
        const uint32_t bot[2] = {r1 ^ 0x80808080u, r3 ^ 0x80808080u};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a0 = i8pair_to_f16x2<0x4140>(top[h]);
          const uint32_t a2 = i8pair_to_f16x2<0x4342>(top[h]);
          const uint32_t a1 = i8pair_to_f16x2<0x4140>(bot[h]);
          const uint32_t a3 = i8pair_to_f16x2<0x4342>(bot[h]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_f16(acc[nt], a0, a1, a2, a3, qf[2 * kp + h][nt][0], qf[2 * kp + h][nt][1]);
        }
      }
    }

    // ---- mask, scale, online softmax (this thread: tokens g, g+8; heads 2t4, 2t4+1)
    const int ta = tile_t0 + g, tb = tile_t0 + g + 8;
    const bool va = phys_of(p, c, s_phys, ta) >= 0;
    const bool vb = phys_of(p, c, s_phys, tb) >= 0;
    float fa = p.scale_log2, fb = p.scale_log2;
    float pva = 1.f, pvb = 1.f;
    if constexpr (I8) {
      fa = va ? fa / sc[g] : 0.f;
      fb = vb ? fb / sc[g + 8] : 0.f;
      pva = va ? 1.f / sc[16 + g] : 0.f;
      pvb = vb ? 1.f / sc[16 + g + 8] : 0.f;
    }
    uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float s[4];
      s[0] = va ? acc[nt][0] * fa : -CUDART_INF_F;
      s[1] = va ? acc[nt][1] * fa : -CUDART_INF_F;
      s[2] = vb ? acc[nt][2] * fb : -CUDART_INF_F;
      s[3] = vb ? acc[nt][3] * fb : -CUDART_INF_F;
      float pr[4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float mx = fmaxf(s[j], s[j + 2]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[nt][j], mx);
        const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
        const float alpha = exp2f(m_run[nt][j] - m_use);
        pr[j] = exp2f(s[j] - m_use);
        pr[j + 2] = exp2f(s[j + 2] - m_use);
        l_run[nt][j] = l_run[nt][j] * alpha + pr[j] + pr[j + 2];
        m_run[nt][j] = m_new;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          o[mt][nt][j] *= alpha;
          o[mt][nt][j + 2] *= alpha;
        }
      }
      // P (token-major fragment) -> P^T B operand; hi/lo split keeps precision
      const float q0 = pr[0] * pva, q1 = pr[1] * pva, q2 = pr[2] * pvb, q3 = pr[3] * pvb;
      uint32_t h01, h23, l01, l23;
      if constexpr (!I8) {
        h01 = pack_bf16(q0, q1);
        h23 = pack_bf16(q2, q3);
        const float2 f01 = unpack_bf16(h01), f23 = unpack_bf16(h23);
        l01 = pack_bf16(q0 - f01.x, q1 - f01.y);
        l23 = pack_bf16(q2 - f23.x, q3 - f23.y);
      } else {
        h01 = pack_f16(q0, q1);
        h23 = pack_f16(q2, q3);
        const float2 f01 = unpack_f16(h01), f23 = unpack_f16(h23);
        l01 = pack_f16(q0 - f01.x, q1 - f01.y);
        l23 = pack_f16(q2 - f23.x, q3 - f23.y);
      }
      bh[nt][0] = movmatrix_trans(h01);
      bh[nt][1] = movmatrix_trans(h23);
      bl[nt][0] = movmatrix_trans(l01);
      bl[nt][1] = movmatrix_trans(l23);
    }

    // ---- O^T[d][head] += V^T * P^T
    if constexpr (!I8) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(vS + swz<CH>(lm_row_v, 2 * mt + lm_ch_v) * 16, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_bf16(o[mt][nt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
          mma_bf16(o[mt][nt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
        }
      }
    } else {
#pragma unroll
      for (int mp = 0; mp < MT / 2; ++mp) {
        uint32_t r0, r1, r2, r3;  // (rows 0-7, c) (rows 8-15, c) (0-7, c+1) (8-15, c+1)
        ldmatrix_x4_trans(vS + swz<CH>(lm_row_a, 2 * mp + lm_ch_a) * 16, r0, r1, r2, r3);
        const uint32_t top[2] = {r0 ^ 0x80808080u, r2 ^ 0x80808080u};
        const uint32_t bot[2] = {r1 ^ 0x80808080u, r3 ^ 0x80808080u};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // rows m <-> d: m = g -> 16c + 2g, m = g + 8 -> 16c + 2g + 1
          const uint32_t a0 = i8pair_to_f16x2<0x4240>(top[h]);
          const uint32_t a1 = i8pair_to_f16x2<0x4341>(top[h]);
          const uint32_t a2 = i8pair_to_f16x2<0x4240>(bot[h]);
          const uint32_t a3 = i8pair_to_f16x2<0x4341>(bot[h]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_f16(o[2 * mp + h][nt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
            mma_f16(o[2 * mp + h][nt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
          }
        }
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();

  // ---- per-warp final state -> smem (ring is reused: wait for every warp)
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
        const int d = I8 ? 16 * mt + (m < 8 ? 2 * m : 2 * (m - 8) + 1) : 16 * mt + m;
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
      load_tile<HD, ELEM, false>(p, c, s_phys, c.t_begin + (warp + i * NWARPS) * 16,
                                 my_ring + (size_t)i * STAGE_B,
                                 my_ring + (size_t)i * STAGE_B + TILE_B, nullptr, lane);
    else
      cp_async_commit();
  }
  const int tr = lane & 15, hf = lane >> 4;
  for (int i = 0; i < my_n; ++i) {
    {
      const int ii = i + NSTAGES - 1;
      if (ii < my_n) {
        uint8_t* st = my_ring + (size_t)(ii % NSTAGES) * STAGE_B;
        load_tile<HD, ELEM, false>(p, c, s_phys, c.t_begin + (warp + ii * NWARPS) * 16, st,
                                   st + TILE_B, nullptr, lane);
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
// Split merge: out = sum_k 2^{lse_k} o_k / sum_k 2^{lse_k} over the splits that
// hold tokens.  One CTA per (q head, sequence), one thread per head_dim column.
template <int HD>
__global__ void __launch_bounds__(HD) merge_kernel(const DecodeParams p) {
  const int qh = blockIdx.x, seq = blockIdx.y, d = threadIdx.x;
  const int ctx = effective_ctx(p, seq, false);
  const int n_valid = (ctx + p.chunk - 1) / p.chunk;
  const size_t r = ((size_t)seq * p.num_q_heads + qh) * p.num_splits;
  float M = -CUDART_INF_F;
  for (int k = 0; k < n_valid; ++k) M = fmaxf(M, p.ws_lse[r + k]);
  float val = 0.f;
  if (M != -CUDART_INF_F) {
    float L = 0.f, O = 0.f;
    for (int k = 0; k < n_valid; ++k) {
      const float lse = p.ws_lse[r + k];
      if (lse == -CUDART_INF_F) continue;
      const float w = exp2f(lse - M);
      L += w;
      O += w * p.ws_o[(r + k) * HD + d];
    }
    val = O / L;
  }
  const size_t o = ((size_t)seq * p.num_q_heads + qh) * HD + d;
  if (p.out_f32)
    static_cast<float*>(p.out)[o] = val;
  else
    static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(val);
}

// ---------------------------------------------------------------------------
// Host side: kernel selection and launch.

namespace {

// Raises a kernel's dynamic shared-memory limit once per (device, kernel) to
// the largest size any launch can ask for; later launches skip the runtime
// call.  The flag array is per kernel (the kernel is the template argument).
// Racing first calls from several host threads both set the same value.
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

template <int HD, bool I8, int NT, int NWARPS, int NSTAGES>
int mma_smem(const DecodeParams& p) {
  constexpr int ELEM = I8 ? 1 : 2;
  constexpr int STAGE_B = 2 * 16 * HD * ELEM + (I8 ? 128 : 0);
  constexpr int RING = NWARPS * NSTAGES * STAGE_B;
  constexpr int GP = NT * 8;
  constexpr int COMB = (3 * NWARPS * GP + GP + NWARPS * GP * HD) * 4;
  return p.phys_bytes + (RING > COMB ? RING : COMB);
}

template <int HD, bool I8, int NT, int NWARPS, int NSTAGES>
cudaError_t launch_mma(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  constexpr auto k = decode_mma_kernel<HD, I8, NT, NWARPS, NSTAGES>;
  const int smem = mma_smem<HD, I8, NT, NWARPS, NSTAGES>(p);
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

// Tile-engine configuration per cache type (warps per CTA, ring depth).
constexpr int kBf16Warps = 4, kBf16Stages = 3;
constexpr int kI8Warps = 4, kI8Stages = 4;
constexpr int kF32Warps = 4, kF32Stages = 2;

int decode_ctas_per_sm_hint(pkv_dtype cache_dt, int head_dim) {
  // resident CTAs per SM implied by the shared-memory ring (228 KB per SM)
  int ring;
  if (cache_dt == PKV_BF16)
    ring = kBf16Warps * kBf16Stages * 2 * 16 * head_dim * 2;
  else if (cache_dt == PKV_I8)
    ring = kI8Warps * kI8Stages * (2 * 16 * head_dim + 128);
  else
    ring = kF32Warps * kF32Stages * 2 * 16 * head_dim * 4 + 16 * head_dim * 4;
  int n = (228 * 1024) / (ring + 4096);
  return n < 1 ? 1 : (n > 8 ? 8 : n);
}

cudaError_t launch_decode(const DecodeParams& p, pkv_dtype cache_dt, int head_dim,
                          cudaStream_t st) {
  dim3 grid(p.num_kv_heads, p.num_seqs, p.num_splits);
  const bool two = p.group > 8;
  if (cache_dt == PKV_BF16) {
    if (head_dim == 128)
      return two ? launch_mma<128, false, 2, kBf16Warps, kBf16Stages>(p, grid, st)
                 : launch_mma<128, false, 1, kBf16Warps, kBf16Stages>(p, grid, st);
    return two ? launch_mma<64, false, 2, kBf16Warps, kBf16Stages>(p, grid, st)
               : launch_mma<64, false, 1, kBf16Warps, kBf16Stages>(p, grid, st);
  }
  if (cache_dt == PKV_I8) {
    if (head_dim == 128)
      return two ? launch_mma<128, true, 2, kI8Warps, kI8Stages>(p, grid, st)
                 : launch_mma<128, true, 1, kI8Warps, kI8Stages>(p, grid, st);
    return two ? launch_mma<64, true, 2, kI8Warps, kI8Stages>(p, grid, st)
               : launch_mma<64, true, 1, kI8Warps, kI8Stages>(p, grid, st);
  }
  if (head_dim == 128) return launch_simt<128, kF32Warps, kF32Stages>(p, grid, st);
  return launch_simt<64, kF32Warps, kF32Stages>(p, grid, st);
}

cudaError_t launch_merge(const DecodeParams& p, int head_dim, cudaStream_t st) {
  dim3 grid(p.num_q_heads, p.num_seqs);
  if (head_dim == 128)
    merge_kernel<128><<<grid, 128, 0, st>>>(p);
  else
    merge_kernel<64><<<grid, 64, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
