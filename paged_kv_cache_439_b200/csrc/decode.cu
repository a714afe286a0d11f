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
#include "decode_common.cuh"

namespace pkv {

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

template <int HD, int NT, int NWARPS, int NSTAGES>
struct MmaCfg {
  static constexpr int ROWB = HD * 2;           // bytes of one token row of one head
  static constexpr int CH = ROWB / 16;          // 16-byte chunks per row: 8 or 16
  static constexpr int RSTEP = kWarp / CH;      // rows one warp-wide copy covers
  static constexpr int PER_LANE = 16 / RSTEP;   // copies per lane per K (or V) tile
  static constexpr int TILE = 16 * ROWB;
  static constexpr int STAGE = 2 * TILE;
  static constexpr int RING = NWARPS * NSTAGES * STAGE;
  static constexpr int GP = NT * 8;
  static constexpr int COMB = (3 * NWARPS * GP + GP + NWARPS * GP * HD) * 4;
  static constexpr int BODY = RING > COMB ? RING : COMB;
  static_assert(CH == 8 || CH == 16, "rows of 128 or 256 bytes");
};

// Issues the copies of one 16-token tile (K and V) into a stage, as one
// commit group.  Full tiles
// inside one block take the fast path: one block-table lookup, one 64-bit base
// per lane and fixed per-lane offsets.  Rows outside the sequence or in a bad
// block are zero-filled.  With AFTER, the stage address is derived from `dep`
// (see after_dep), so no copy overtakes the reads of the stage it overwrites.
template <class Cfg, bool AFTER>
__device__ __forceinline__ void issue_tile(const DecodeParams& p, const CtaSetup& c,
                                           const int* s_phys, int tile_t0, uint32_t k_st,
                                           uint32_t v_st,
                                           const uint32_t (&soff)[Cfg::PER_LANE],
                                           size_t lane_goff, int lane_row, uint32_t dep) {
  const uint8_t* kb = static_cast<const uint8_t*>(p.k_cache);
  const uint8_t* vb = static_cast<const uint8_t*>(p.v_cache);
  const size_t tok_stride = (size_t)p.num_kv_heads * Cfg::ROWB;
  const int bs = p.block_size;
  if constexpr (AFTER) {
    k_st = after_dep(k_st, dep);
    v_st = after_dep(v_st, dep);
  }
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
  }
  cp_async_commit();
}

template <int HD, int NT, int NWARPS, int NSTAGES, bool MHA>
__global__ void __launch_bounds__(NWARPS * kWarp)
    decode_mma_kernel(const DecodeParams p) {
  pdl_trigger();  // the split merge may be scheduled once every CTA has started
  using Cfg = MmaCfg<HD, NT, NWARPS, NSTAGES>;
  static_assert(!MHA || NT == 1, "MHA: one q head per kv head");
  constexpr int KS = HD / 16;           // k-steps of the score mma
  constexpr int MT = HD / 16;           // m-tiles (16 head-dim rows) of the PV mma
  constexpr int KA = KS;                // ldmatrix.x4 per K tile
  constexpr int VA = MT;                // ldmatrix.x4 per V tile
  constexpr int GP = Cfg::GP;
  constexpr int CH = Cfg::CH;

  extern __shared__ __align__(128) uint8_t smem[];
  int* s_phys = reinterpret_cast<int*>(smem);
  uint8_t* ring = smem + p.phys_bytes;

  long long new_slot;
  const uint4 new_rows = fused_prefetch<HD, kQuantNone>(p, &new_slot);
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
  fused_commit<HD, kQuantNone, NWARPS>(p, c, s_phys, new_rows, new_slot);  // before any cache read
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
          b0 = *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * t4);
          b1 = *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * t4 + 8);
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
    voff[i] = (uint32_t)swz<CH>(lm_row_v, 2 * i + lm_ch_v) * 16;

  const uint32_t my_ring = smem_u32(ring) + (uint32_t)(warp * NSTAGES * Cfg::STAGE);
  const int ntiles = (c.t_end - c.t_begin + 15) >> 4;
  const int my_n = (warp < ntiles) ? (ntiles - warp + NWARPS - 1) / NWARPS : 0;

#pragma unroll
  for (int i = 0; i < NSTAGES; ++i) {
    const uint32_t st = my_ring + (uint32_t)(i * Cfg::STAGE);
    if (i < my_n)
      issue_tile<Cfg, false>(p, c, s_phys, c.t_begin + (warp + i * NWARPS) * 16, st,
                             st + Cfg::TILE, soff, lane_goff, lane_row, 0u);
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
    uint32_t dep = 0;
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
        issue_tile<Cfg, true>(p, c, s_phys, tile_t0 + NSTAGES * NWARPS * 16, kS, vS, soff,
                              lane_goff, lane_row, dep);
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

    // ---- mask, scale, online softmax (tokens g, g+8; heads 2t4, 2t4+1)
    const bool va = (mask >> g) & 1u, vb = (mask >> (g + 8)) & 1u;
    const float fa = p.scale_log2, fb = p.scale_log2;
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
        const float sa = va ? (acc[nt][jj] + acc2[nt][jj]) * fa : -CUDART_INF_F;
        const float sb = vb ? (acc[nt][jj + 2] + acc2[nt][jj + 2]) * fb : -CUDART_INF_F;
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
      const float q0 = pr[0], q1 = pr[1], q2 = pr[2], q3 = pr[3];
      const uint32_t h01 = pack_bf16(q0, q1), h23 = pack_bf16(q2, q3);
      const float2 f01 = unpack_bf16(h01), f23 = unpack_bf16(h23);
      bh[nt][0] = movmatrix_trans(h01);
      bh[nt][1] = movmatrix_trans(h23);
      bl[nt][0] = movmatrix_trans(pack_bf16(q0 - f01.x, q1 - f01.y));
      bl[nt][1] = movmatrix_trans(pack_bf16(q2 - f23.x, q3 - f23.y));
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

    // ---- O^T[d][head] += V^T * P^T (P as bf16 hi + lo)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_bf16(o[mt][nt], vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3], bh[nt][0], bh[nt][1]);
        mma_bf16(o[mt][nt], vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3], bl[nt][0], bl[nt][1]);
      }
    }
  }
  cp_async_wait<0>();

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
        const int d = 16 * mt + m;
        s_o[(warp * GP + h) * HD + d] = o[mt][nt][j];
      }
  combine_and_store<HD, NWARPS, GP>(p, c, s_m, s_l, s_o, s_w, s_L);
}

// ---------------------------------------------------------------------------
// simt engine: fp32 caches (ELEM 4; q in fp32 or bf16), or bf16 caches
// (ELEM 2) where the tensor cores are not used.  Lanes l and l+16 share token
// l%16, each summing half of head_dim; the PV update gives lane l the head_dim
// columns l, l+32, ... (fp32) or the pairs 2l, 2l+1, 2l+64, 2l+65 (bf16).  GP
// (a power of two, at least the group) bounds the q heads held per thread.
template <int HD, int NWARPS, int NSTAGES, int ELEM, int GP>
__global__ void __launch_bounds__(NWARPS * kWarp)
    decode_simt_kernel(const DecodeParams p) {
  pdl_trigger();
  static_assert(ELEM == 4 || ELEM == 2, "fp32 or bf16 cache rows");
  constexpr int ROWB = HD * ELEM;
  constexpr int CH = ROWB / 16;
  constexpr int TILE_B = 16 * ROWB;
  constexpr int STAGE_B = 2 * TILE_B;
  constexpr int DJ = HD / kWarp;
  constexpr int EPC = 16 / ELEM;  // elements per 16-byte chunk

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
      const uint4 raw = *reinterpret_cast<const uint4*>(kt + swz<CH>(tr, ch) * 16);
      float kv[EPC];
      if constexpr (ELEM == 4) {
        kv[0] = __uint_as_float(raw.x);
        kv[1] = __uint_as_float(raw.y);
        kv[2] = __uint_as_float(raw.z);
        kv[3] = __uint_as_float(raw.w);
      } else {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = unpack_bf16(w[k]);
          kv[2 * k] = f.x;
          kv[2 * k + 1] = f.y;
        }
      }
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        if (h < G) {
#pragma unroll
          for (int e4 = 0; e4 < EPC; e4 += 4) {
            const float4 qv = *reinterpret_cast<const float4*>(s_q + h * HD + ch * EPC + e4);
            s[h] = fmaf(qv.x, kv[e4], s[h]);
            s[h] = fmaf(qv.y, kv[e4 + 1], s[h]);
            s[h] = fmaf(qv.z, kv[e4 + 2], s[h]);
            s[h] = fmaf(qv.w, kv[e4 + 3], s[h]);
          }
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
      if constexpr (ELEM == 4) {
#pragma unroll
        for (int j = 0; j < DJ; ++j) {
          const int e = lane + kWarp * j;
          vv[j] = *reinterpret_cast<const float*>(vt + swz<CH>(t, e >> 2) * 16 + (e & 3) * 4);
        }
      } else {
#pragma unroll
        for (int j = 0; j < DJ / 2; ++j) {
          const int e = 2 * lane + 2 * kWarp * j;  // column pair e, e + 1
          const float2 f = unpack_bf16(*reinterpret_cast<const uint32_t*>(
              vt + swz<CH>(t, e >> 3) * 16 + (e & 7) * 2));
          vv[2 * j] = f.x;
          vv[2 * j + 1] = f.y;
        }
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
      for (int j = 0; j < DJ; ++j) {
        const int d = ELEM == 4 ? lane + kWarp * j : 2 * lane + 2 * kWarp * (j >> 1) + (j & 1);
        s_o[(warp * GP + h) * HD + d] = o[h][j];
      }
  combine_and_store<HD, NWARPS, GP>(p, c, s_m, s_l, s_o, s_w, s_L);
}

// ---------------------------------------------------------------------------
// Host side: kernel selection and launch.

namespace {

template <int HD, int NT, int NWARPS, int NSTAGES, bool MHA>
cudaError_t launch_mma(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  using Cfg = MmaCfg<HD, NT, NWARPS, NSTAGES>;
  const int smem = p.phys_bytes + Cfg::BODY;
  constexpr auto k = decode_mma_kernel<HD, NT, NWARPS, NSTAGES, MHA>;
  cudaError_t e = prepare<k>(smem);
  if (e != cudaSuccess) return e;
  k<<<grid, NWARPS * kWarp, smem, st>>>(p);
  return cudaGetLastError();
}

template <int HD, int NWARPS, int NSTAGES, int ELEM = 4, int GP = 16>
cudaError_t launch_simt(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  constexpr int STAGE_B = 2 * 16 * HD * ELEM;
  constexpr int RING = NWARPS * NSTAGES * STAGE_B;
  constexpr int COMB = (3 * NWARPS * GP + GP + NWARPS * GP * HD) * 4;
  const int smem = p.phys_bytes + GP * HD * 4 + (RING > COMB ? RING : COMB);
  constexpr auto k = decode_simt_kernel<HD, NWARPS, NSTAGES, ELEM, GP>;
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

template <int HD>
int mma_occupancy() {
  constexpr int NS = PKV_BF16_STAGES;
  using Cfg = MmaCfg<HD, 1, kMW, NS>;
  return occupancy<decode_mma_kernel<HD, 1, kMW, NS, false>>(kMW * kWarp,
                                                       kTypicalPhysBytes + Cfg::BODY);
}

}  // namespace

int decode_ctas_per_sm_hint(pkv_dtype cache_dt, int head_dim) {
  if (cache_dt == PKV_BF16) return head_dim == 128 ? mma_occupancy<128>() : mma_occupancy<64>();
  if (cache_dt == PKV_I8 || cache_dt == PKV_FP8) return decode_q8_ctas_per_sm(cache_dt, head_dim);
  const int smem = kF32Warps * kF32Stages * 2 * 16 * head_dim * 4 + 16 * head_dim * 4 + 1024;
  const int n = kSmemPerSm / (smem + kSmemPerCta);
  return n < 1 ? 1 : n;
}

namespace {

// Picks the q-head tiling: two n-tiles for groups above 8, the MHA form for a
// group of one, else one n-tile.
template <int HD, int NS>
cudaError_t launch_mma_group(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  if (p.group > 8) return launch_mma<HD, 2, kMW, NS, false>(p, grid, st);
  if (p.group == 1) return launch_mma<HD, 1, kMW, NS, true>(p, grid, st);
  return launch_mma<HD, 1, kMW, NS, false>(p, grid, st);
}

}  // namespace

// bf16 caches on the SIMT engine instead of the tensor cores, for groups below
// this value (0: never).  The tensor-core engine is the default at every group
// size: measured against this SIMT form at groups 1 and 4 it was faster (the
// figures are in the project's design notes); the switch exists to repeat that
// comparison.
#ifndef PKV_SIMT_BELOW_GROUP
#define PKV_SIMT_BELOW_GROUP 0
#endif

template <int HD>
cudaError_t launch_simt_bf16(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  if (p.group <= 1) return launch_simt<HD, kF32Warps, kF32Stages, 2, 1>(p, grid, st);
  if (p.group <= 2) return launch_simt<HD, kF32Warps, kF32Stages, 2, 2>(p, grid, st);
  if (p.group <= 4) return launch_simt<HD, kF32Warps, kF32Stages, 2, 4>(p, grid, st);
  if (p.group <= 8) return launch_simt<HD, kF32Warps, kF32Stages, 2, 8>(p, grid, st);
  return launch_simt<HD, kF32Warps, kF32Stages, 2, 16>(p, grid, st);
}

cudaError_t launch_decode(const DecodeParams& p, pkv_dtype cache_dt, int head_dim,
                          cudaStream_t st) {
  dim3 grid(p.num_kv_heads, p.num_seqs, p.num_splits);
  if (cache_dt == PKV_BF16 && p.group < PKV_SIMT_BELOW_GROUP && p.new_k == nullptr)
    return head_dim == 128 ? launch_simt_bf16<128>(p, grid, st) : launch_simt_bf16<64>(p, grid, st);
  if (cache_dt == PKV_BF16)
    return head_dim == 128 ? launch_mma_group<128, PKV_BF16_STAGES>(p, grid, st)
                           : launch_mma_group<64, PKV_BF16_STAGES>(p, grid, st);
  if (cache_dt == PKV_I8 || cache_dt == PKV_FP8) return launch_decode_q8(p, cache_dt, head_dim, st);
  if (head_dim == 128) return launch_simt<128, kF32Warps, kF32Stages>(p, grid, st);
  return launch_simt<64, kF32Warps, kF32Stages>(p, grid, st);
}

}  // namespace pkv
