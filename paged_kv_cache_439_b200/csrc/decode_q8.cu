// Paged decode attention over one-byte KV caches (INT8 or FP8 E4M3 codes with
// one fp32 scale per token per head), sm_100a.
//
// Operation ("大模型推理加速实战：KV Cache内存优化与PagedAttention分页管理方案",
// PagedAttention section; GQA grouping from "LLM推理显存优化KV Cache管理3大策略"
// §3; INT8 codes and their per-token scale from the same page's §4
// quantize_tensor, dequantised as code / scale): for every sequence and query
// head, attend over the sequence's tokens, fetching each token's K/V row
// through the block table.
//
// Work decomposition as in the bf16 engine (decode.cu): one CTA per
// (kv_head, sequence, context split), all `group` query heads of a KV head in
// the CTA, 16-token tiles streamed by each warp through its own ring of
// cp.async stages, each stage read into registers and refilled as soon as it
// lands, scores and P V on mma.sync m16n8k16 with fp32 accumulation.  A
// one-byte tile carries half the bytes of a bf16 tile for the same per-tile
// work, so this engine is built to spend as few instructions per tile as it
// can:
//  * copies: one warp-wide cp.async covers whole 128-byte rows (lane l copies
//    16-byte chunk l % CH of rows l / CH + i * (32 / CH)), into XOR-swizzled
//    rows so that the ldmatrix phases are conflict-free.  Measured on the
//    13B-shaped cache without the math, this mapping streamed 6.6 TB/s, where
//    giving each lane pair one row (32-byte pieces of 16 rows per
//    instruction) reached 4.8 TB/s and per-row bulk copies 4.2 TB/s.  A full
//    tile inside one block costs one block-table lookup; a row past the CTA's
//    range or in a bad block is zero-filled, never read.  Lanes 0-15 copy the
//    16 K scales, lanes 16-31 the V scales.
//  * masking: a CTA whose block-table slice is clean takes the unmasked path
//    for every full tile (no per-tile ballot, no selects).
//  * scales: each lane takes the reciprocal of the one scale it loaded before
//    the shuffles that hand the scales to the accumulator layout.
//  * INT8: codes reach the tensor core as the exact fp16 values code + 1152
//    (one XOR per 4 bytes, one byte permute per 2).  The constant is removed
//    in fp32: the scores start from -1152 * sum_d q[h][d] (the accumulator's
//    initial value), and 1152 * sum_t P[t][h] is taken off the output at the
//    end, with sum_t P accumulated by one extra mma against a tile of ones on
//    the same fp16 P the tensor core used, so the constant cancels exactly.
//  * FP8: codes become exact fp16 values with cvt.rn.f16x2.e4m3x2 (every E4M3
//    value is an fp16 value); no constant to remove.
// P goes to the tensor core as one fp16 value (11 significant bits; its
// rounding error, below 2^-11 of each term, is under the bf16 rounding of the
// output).  The online softmax runs in fp32 with ex2.approx; its reference
// maximum moves only when a score exceeds it by more than 2^8, so most tiles
// need no warp-wide maximum and no rescale.
#include "common.cuh"
#include "decode.cuh"
#include "decode_common.cuh"

namespace pkv {

namespace {

#ifndef PKV_Q8_STAGES
#define PKV_Q8_STAGES 2
#endif
#ifndef PKV_Q8_WARPS
#define PKV_Q8_WARPS 4
#endif
#ifndef PKV_Q8_IMMA
#define PKV_Q8_IMMA 1
#endif
#ifndef PKV_Q8_MINBLOCKS
#define PKV_Q8_MINBLOCKS 3
#endif
#ifndef PKV_Q8_HOLD3
#define PKV_Q8_HOLD3 1
#endif
constexpr int kQ8Warps = PKV_Q8_WARPS;
// The softmax reference maximum moves only when a score exceeds it by more
// than this (log2 units): P stays below 2^8, far inside fp16, and most tiles
// skip the warp-wide max reduction and the rescale.
#ifndef PKV_Q8_LAZY_LOG2
#define PKV_Q8_LAZY_LOG2 8.0f
#endif
constexpr float kLazyLog2 = PKV_Q8_LAZY_LOG2;
constexpr int kQ8Stages = PKV_Q8_STAGES;

template <int HD, int NT, int NWARPS, int NSTAGES>
struct Q8Cfg {
  static constexpr int ROWB = HD;              // bytes of one token row of one head
  static constexpr int CH = ROWB / 16;         // 16-byte chunks per row: 4 or 8
  static constexpr int RSTEP = kWarp / CH;     // rows one warp-wide copy covers
  static constexpr int PER_LANE = 16 / RSTEP;  // copies per lane per K (or V) tile
  static constexpr int TILE = 16 * ROWB;       // one K (or V) tile
  static constexpr int SCB = 32 * 4;           // 16 K scales, then 16 V scales
  static constexpr int STAGE = 2 * TILE + SCB;
  static constexpr int RING = NWARPS * NSTAGES * STAGE;
  static constexpr int GP = NT * 8;
  static constexpr int COMB = (3 * NWARPS * GP + GP + NWARPS * GP * HD) * 4;
  static constexpr int BODY = RING > COMB ? RING : COMB;
  static_assert(HD == 64 || HD == 128, "head_dim 64 or 128");
  static_assert(STAGE % 16 == 0, "16-byte aligned stages");
};

// Per-lane copy geometry, fixed for the kernel.
struct Q8Lane {
  int row;              // first tile row this lane copies (then + RSTEP, + 2 RSTEP, ...)
  size_t goff;          // its row, head and chunk offset inside a block's rows
  size_t col;           // its head and chunk offset inside a cache row
  const float* sbase;   // k_scale (lanes 0-15) or v_scale (lanes 16-31)
};

// Issues the copies of one 16-token tile (K rows, V rows and the scales of
// both) into a stage, as one commit group.  A full tile inside one block takes
// the fast path: one block-table lookup, one 64-bit base per lane.  With
// AFTER, the stage address is derived from `dep` (see after_dep), so no copy
// overtakes the reads of the stage it overwrites.
template <class Cfg, bool AFTER>
__device__ __forceinline__ void q8_issue(const DecodeParams& p, const CtaSetup& c,
                                         const int* s_phys, int tile_t0, uint32_t st,
                                         const uint32_t (&soff)[Cfg::PER_LANE], const Q8Lane& L,
                                         size_t tok_stride, int lane, uint32_t dep) {
  if constexpr (AFTER) st = after_dep(st, dep);
  const uint8_t* kb = static_cast<const uint8_t*>(p.k_cache);
  const uint8_t* vb = static_cast<const uint8_t*>(p.v_cache);
  const int bs = p.block_size;
  const int srow = lane & 15;
  if (bs >= 16 && tile_t0 + 16 <= c.t_end) {
    const int phys = s_phys[(tile_t0 >> p.log2_bs) - c.blk0];
    const int n = phys >= 0 ? 16 : 0;
    const int in_blk = tile_t0 & (bs - 1);
    // a bad block reads nothing (n = 0); its addresses stay inside the caches
    const size_t base = phys >= 0 ? ((size_t)phys * bs + in_blk) * tok_stride + L.goff : 0;
    const size_t step = (size_t)Cfg::RSTEP * tok_stride;
#pragma unroll
    for (int i = 0; i < Cfg::PER_LANE; ++i) {
      cp_async_16(st + soff[i], kb + base + i * step, n);
      cp_async_16(st + Cfg::TILE + soff[i], vb + base + i * step, n);
    }
    const size_t so = phys >= 0 ? ((size_t)phys * p.num_kv_heads + c.kvh) * bs + in_blk + srow : 0;
    cp_async_4(st + 2 * Cfg::TILE + 4 * lane, L.sbase + so, phys >= 0 ? 4 : 0);
  } else {
#pragma unroll
    for (int i = 0; i < Cfg::PER_LANE; ++i) {
      const int t = tile_t0 + L.row + i * Cfg::RSTEP;
      const int phys = phys_of(p, c, s_phys, t);
      size_t off = 0;
      int n = 0;
      if (phys >= 0) {
        off = ((size_t)phys * bs + (t & (bs - 1))) * tok_stride + L.col;
        n = 16;
      }
      cp_async_16(st + soff[i], kb + off, n);
      cp_async_16(st + Cfg::TILE + soff[i], vb + off, n);
    }
    const int t = tile_t0 + srow;
    const int phys = phys_of(p, c, s_phys, t);
    const size_t so = phys >= 0 ? ((size_t)phys * p.num_kv_heads + c.kvh) * bs + (t & (bs - 1)) : 0;
    cp_async_4(st + 2 * Cfg::TILE + 4 * lane, L.sbase + so, phys >= 0 ? 4 : 0);
  }
  cp_async_commit();
}

template <int HD, int QM, int NT, int NWARPS, int NSTAGES, bool MHA>
#if PKV_Q8_MINBLOCKS > 0
#define PKV_Q8_BOUNDS(threads) __launch_bounds__(threads, PKV_Q8_MINBLOCKS)
#else
#define PKV_Q8_BOUNDS(threads) __launch_bounds__(threads)
#endif
__global__ void PKV_Q8_BOUNDS(NWARPS * kWarp) decode_q8_kernel(const DecodeParams p) {
  pdl_trigger();  // the split merge may be scheduled once every CTA has started
  using Cfg = Q8Cfg<HD, NT, NWARPS, NSTAGES>;
  static_assert(!MHA || NT == 1, "MHA: one q head per kv head");
  static_assert(QM == kQuantI8 || QM == kQuantFp8, "one-byte caches");
  constexpr bool I8 = QM == kQuantI8;
  constexpr bool IK = I8 && PKV_Q8_IMMA;  // INT8 scores on the integer tensor core
  constexpr int KS = HD / 16;   // k-steps of the score mma
  constexpr int MT = HD / 16;   // m-tiles (16 head-dim rows) of the PV mma
  constexpr int KA = KS / 2;    // ldmatrix.x4 per K tile
  constexpr int VA = MT / 2;    // ldmatrix.x4 per V tile
  constexpr int GP = Cfg::GP;
  constexpr uint32_t kOnes = 0x3C003C00u;  // fp16 1.0, 1.0

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

  // q as the B operand (n = head, k = head_dim) in fp16, loaded once.  k-slot
  // order of a one-byte-code chunk: slots 2t, 2t+1 <- d 16c+4t+{0,1}; slots
  // 2t+8, 2t+9 <- d 16c+4t+{2,3} (the order the K codes arrive in).
  uint32_t qf[IK ? 1 : KS][NT][2];
  // INT8 on the integer tensor core (IK): q of head h as the integer
  // Q = rint(q * 2^E_h), E_h chosen so that max_d |q[h][d]| * 2^E_h lies in
  // [2^21, 2^22), split into three signed bytes Q = p2 * 2^16 + p1 * 2^8 + p0
  // (|Q| < 2^22 keeps |p2| <= 65; at 2^23 a largest element with a full bf16
  // mantissa would need p2 = 128).  Each score is
  // sum_d code * q = 2^-E (2^16 D2 + 2^8 D1 + D0) with Dk the exact int32 dot
  // products of the codes with the pieces.  Q is exact for every element
  // within 14 binades of its head's largest (bf16 carries 8 significant
  // bits); smaller elements are rounded at 2^-21 of that largest.
  uint32_t qp[IK ? KA : 1][3][NT][2];
  float qc[IK ? NT : 1][2][3];  // per head column: 2^16 2^-E, 2^8 2^-E, 2^-E
  if constexpr (IK) {
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q) +
                              ((size_t)c.seq * p.num_q_heads + (size_t)c.kvh * G) * HD;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = nt * 8 + g;
      float x[KA][8];  // d = 32a + 4t4 + {0..3}, then 32a + 16 + 4t4 + {0..3}
      float amax = 0.f;
#pragma unroll
      for (int a = 0; a < KA; ++a) {
        uint2 r0 = make_uint2(0u, 0u), r1 = make_uint2(0u, 0u);
        if (h < G) {
          r0 = *reinterpret_cast<const uint2*>(qb + (size_t)h * HD + 32 * a + 4 * t4);
          r1 = *reinterpret_cast<const uint2*>(qb + (size_t)h * HD + 32 * a + 16 + 4 * t4);
        }
        const uint32_t w[4] = {r0.x, r0.y, r1.x, r1.y};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[a][2 * k] = __uint_as_float(w[k] << 16);
          x[a][2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
          amax = fmaxf(amax, fmaxf(fabsf(x[a][2 * k]), fabsf(x[a][2 * k + 1])));
        }
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // E = 21 - floor(log2 amax), kept within [0, 120] so that 2^E and 2^-E
      // stay normal fp32 (a head whose largest |q| is below 2^-99 scores ~0)
      int e_max = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
      int E = amax > 0.f ? 21 - e_max : 0;
      E = E < 0 ? 0 : (E > 120 ? 120 : E);
      const float up = __uint_as_float((uint32_t)(E + 127) << 23);  // 2^E
#pragma unroll
      for (int a = 0; a < KA; ++a) {
        uint32_t pk[3][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int Q = __float2int_rn(x[a][e] * up);
          const int p0 = ((Q + 128) & 255) - 128;
          const int q1 = (Q - p0) >> 8;
          const int p1 = ((q1 + 128) & 255) - 128;
          const int p2 = (q1 - p1) >> 8;
          const int reg = e >> 2, sh = 8 * (e & 3);
          pk[0][reg] |= (uint32_t)(p0 & 255) << sh;
          pk[1][reg] |= (uint32_t)(p1 & 255) << sh;
          pk[2][reg] |= (uint32_t)(p2 & 255) << sh;
        }
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          qp[a][k][nt][0] = pk[k][0];
          qp[a][k][nt][1] = pk[k][1];
        }
      }
      // the scale factors of this thread's head columns 2*t4 and 2*t4 + 1
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int Ej = __shfl_sync(0xffffffffu, E, (2 * t4 + j) * 4);
        const float down = __uint_as_float((uint32_t)(127 - Ej) << 23);  // 2^-E
        qc[nt][j][0] = 65536.f * down;
        qc[nt][j][1] = 256.f * down;
        qc[nt][j][2] = down;
      }
    }
  } else {
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q) +
                              ((size_t)c.seq * p.num_q_heads + (size_t)c.kvh * G) * HD;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = nt * 8 + g;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t b0 = 0, b1 = 0;
        if (h < G) {
          const uint2 raw =
              *reinterpret_cast<const uint2*>(qb + (size_t)h * HD + 16 * ks + 4 * t4);
          const float2 lo = unpack_bf16(raw.x), hi = unpack_bf16(raw.y);
          b0 = pack_f16(lo.x, lo.y);
          b1 = pack_f16(hi.x, hi.y);
        }
        qf[IK ? 0 : ks][nt][0] = b0;
        qf[IK ? 0 : ks][nt][1] = b1;
      }
    }
  }

  // INT8 through fp16 (not IK): every score carries 1152 * sum_d q[h][d]; the
  // score accumulators start from its negative (this thread's head columns
  // 2*t4 and 2*t4 + 1).
  float acc_init[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float mine = 0.f;  // partial sum over this lane's k-slots of head nt*8 + g
    if constexpr (I8 && !IK) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const float2 a = unpack_f16(qf[ks][nt][0]), b = unpack_f16(qf[ks][nt][1]);
        mine += (a.x + a.y) + (b.x + b.y);
      }
      mine += __shfl_xor_sync(0xffffffffu, mine, 1);
      mine += __shfl_xor_sync(0xffffffffu, mine, 2);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j)
      acc_init[nt][j] =
          (I8 && !IK) ? -1152.f * __shfl_sync(0xffffffffu, mine, (2 * t4 + j) * 4) : 0.f;
  }

  float o[MT][NT][4];
  float o1[NT][4];  // INT8: sum_t P[t][h] of the fp16 P fed to the tensor core
  float m_run[NT][2], l_run[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      m_run[nt][j] = -CUDART_INF_F;
      l_run[nt][j] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) o1[nt][j] = 0.f;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[mt][nt][j] = 0.f;
  }

  // Per-lane copy geometry: lane copies chunk lane % CH of rows
  // lane / CH + i * RSTEP; its shared-memory offsets are fixed.
  constexpr int CH = Cfg::CH;
  const size_t tok_stride = (size_t)p.num_kv_heads * Cfg::ROWB;
  Q8Lane L;
  L.row = lane / CH;
  L.col = (size_t)c.kvh * Cfg::ROWB + (size_t)(lane % CH) * 16;
  L.goff = (size_t)L.row * tok_stride + L.col;
  L.sbase = lane < 16 ? p.k_scale : p.v_scale;
  uint32_t soff[Cfg::PER_LANE];
#pragma unroll
  for (int i = 0; i < Cfg::PER_LANE; ++i)
    soff[i] = (uint32_t)swz<CH>(L.row + i * Cfg::RSTEP, lane % CH) * 16;
  // scale this lane loads: K ones get softmax_scale * log2(e) folded in
  const float sc_fold = lane < 16 ? p.scale_log2 : 1.f;

  // ldmatrix lane addressing: matrix j = lane/8 supplies its row lane%8;
  // j: rows 0-7, 8-15, 0-7, 8-15 of chunks +0, +0, +1, +1.
  const int lm_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int lm_ch = lane >> 4;
  uint32_t koff[KA];
#pragma unroll
  for (int i = 0; i < KA; ++i) koff[i] = (uint32_t)swz<CH>(lm_row, 2 * i + lm_ch) * 16;

  const uint32_t my_ring = smem_u32(ring) + (uint32_t)(warp * NSTAGES * Cfg::STAGE);
  const int ntiles = (c.t_end - c.t_begin + 15) >> 4;
  const int my_n = (warp < ntiles) ? (ntiles - warp + NWARPS - 1) / NWARPS : 0;

#pragma unroll
  for (int i = 0; i < NSTAGES; ++i) {
    if (i < my_n)
      q8_issue<Cfg, false>(p, c, s_phys, c.t_begin + (warp + i * NWARPS) * 16,
                           my_ring + (uint32_t)(i * Cfg::STAGE), soff, L, tok_stride, lane, 0u);
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

    // ---- read the stage into registers
    uint32_t kf[KA][4], vf[VA][4];
#pragma unroll
    for (int a = 0; a < KA; ++a) ldmatrix_x4(kS + koff[a], kf[a][0], kf[a][1], kf[a][2], kf[a][3]);
#pragma unroll
    for (int a = 0; a < VA; ++a)
      ldmatrix_x4_trans(kS + Cfg::TILE + koff[a], vf[a][0], vf[a][1], vf[a][2], vf[a][3]);
    float mine;
    asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(mine) : "r"(kS + 2 * Cfg::TILE + 4 * lane));
    // one register of each ldmatrix: an ldmatrix completes all of its registers at once
    uint32_t dep = __float_as_uint(mine);
#pragma unroll
    for (int a = 0; a < KA; ++a) dep ^= kf[a][0];
#pragma unroll
    for (int a = 0; a < VA; ++a) dep ^= vf[a][0];
    const bool full = c.clean && tile_t0 + 16 <= c.t_end;
    const uint32_t mask =
        full ? 0xFFFFu
             : __ballot_sync(0xffffffffu, phys_of(p, c, s_phys, tile_t0 + (lane & 15)) >= 0) &
                   0xFFFFu;

    // ---- refill the stage with this warp's tile i + NSTAGES
    if (i + NSTAGES < my_n)
      q8_issue<Cfg, true>(p, c, s_phys, tile_t0 + NSTAGES * NWARPS * 16, kS, soff, L, tok_stride,
                          lane, dep);
    else
      cp_async_commit();
    if (mask == 0u) continue;

    // reciprocal scales in the accumulator layout: tokens g (a) and g + 8 (b);
    // K ones carry softmax_scale * log2(e).  A zero-filled row's scale is 0:
    // its reciprocal is infinite, and the masked path below never uses it.
    const float rmine = fast_rcp(mine) * sc_fold;
    const float rka = __shfl_sync(0xffffffffu, rmine, g);
    const float rkb = __shfl_sync(0xffffffffu, rmine, g + 8);
    const float rva = __shfl_sync(0xffffffffu, rmine, 16 + g);
    const float rvb = __shfl_sync(0xffffffffu, rmine, 24 + g);

    // ---- scores S^T = K * Q^T (two accumulator chains; three for IK)
    float acc[NT][4], acc2[NT][4];
    if constexpr (IK) {
      int dk[3][NT][4];
#pragma unroll
      for (int k = 0; k < 3; ++k)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int q = 0; q < 4; ++q) dk[k][nt][q] = 0;
#pragma unroll
      for (int a = 0; a < KA; ++a)
#pragma unroll
        for (int k = 0; k < 3; ++k)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_s8(dk[k][nt], kf[a][0], kf[a][1], kf[a][2], kf[a][3], qp[a][k][nt][0],
                   qp[a][k][nt][1]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float* cf = qc[nt][q & 1];
          acc[nt][q] = fmaf((float)dk[2][nt][q], cf[0],
                            fmaf((float)dk[1][nt][q], cf[1], (float)dk[0][nt][q] * cf[2]));
          acc2[nt][q] = 0.f;
        }
    } else {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[nt][q] = 0.f;
        acc2[nt][q] = acc_init[nt][q & 1];
      }
#pragma unroll
    for (int kp = 0; kp < KS / 2; ++kp) {
      // kf[kp]: (rows 0-7, c) (rows 8-15, c) (0-7, c+1) (8-15, c+1); bytes of a
      // register are d 4t..4t+3 -> slots (2t, 2t+1) (its low half) and
      // (2t+8, 2t+9) (its high half)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a0, a1, a2, a3;
        if constexpr (I8) {
          const uint32_t top = kf[kp][2 * h] ^ 0x80808080u, bot = kf[kp][2 * h + 1] ^ 0x80808080u;
          a0 = i8pair_to_f16x2_biased<0x4140>(top);
          a2 = i8pair_to_f16x2_biased<0x4342>(top);
          a1 = i8pair_to_f16x2_biased<0x4140>(bot);
          a3 = i8pair_to_f16x2_biased<0x4342>(bot);
        } else {
          a0 = e4m3half_to_f16x2<true>(kf[kp][2 * h]);
          a2 = e4m3half_to_f16x2<false>(kf[kp][2 * h]);
          a1 = e4m3half_to_f16x2<true>(kf[kp][2 * h + 1]);
          a3 = e4m3half_to_f16x2<false>(kf[kp][2 * h + 1]);
        }
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

    // ---- online softmax (tokens g, g+8; heads 2t4, 2t4+1) and P in the B layout.
    // The reference maximum m_run moves lazily: only when some score of the
    // tile exceeds it by more than kLazyLog2 (a warp vote; the first tile
    // always does) is the tile maximum reduced across the warp and the state
    // rescaled.  Otherwise P = 2^(s - m_run) <= 2^kLazyLog2, and O and l keep
    // one common reference, so the result is the same softmax.
    uint32_t bh[NT][2];
    const bool va = (mask >> g) & 1u, vb = (mask >> (g + 8)) & 1u;
    const bool all = mask == 0xFFFFu;
    float sc[NT][4];
    bool need = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        if (MHA && jj == 1) {  // one q head per kv head: column 2*t4 + 1 holds none
          sc[nt][1] = sc[nt][3] = -CUDART_INF_F;
          continue;
        }
        float sa = (acc[nt][jj] + acc2[nt][jj]) * rka;
        float sb = (acc[nt][jj + 2] + acc2[nt][jj + 2]) * rkb;
        if (!all) {
          sa = va ? sa : -CUDART_INF_F;
          sb = vb ? sb : -CUDART_INF_F;
        }
        sc[nt][jj] = sa;
        sc[nt][jj + 2] = sb;
        need |= fmaxf(sa, sb) > m_run[nt][jj] + kLazyLog2;
      }
    if (__any_sync(0xffffffffu, need)) {
      float alpha[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          if (MHA && jj == 1) {
            alpha[nt][1] = 1.f;
            continue;
          }
          float mx = fmaxf(sc[nt][jj], sc[nt][jj + 2]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m_run[nt][jj], mx);
          const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
          alpha[nt][jj] = fast_exp2(m_run[nt][jj] - m_use);  // 0 while m_run = -inf
          l_run[nt][jj] *= alpha[nt][jj];
          m_run[nt][jj] = m_new;
        }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          o[mt][nt][0] *= alpha[nt][0];
          o[mt][nt][2] *= alpha[nt][0];
          o[mt][nt][1] *= alpha[nt][1];
          o[mt][nt][3] *= alpha[nt][1];
        }
        if constexpr (I8) {
          o1[nt][0] *= alpha[nt][0];
          o1[nt][2] *= alpha[nt][0];
          o1[nt][1] *= alpha[nt][1];
          o1[nt][3] *= alpha[nt][1];
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pr[4];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        if (MHA && jj == 1) {
          pr[1] = pr[3] = 0.f;
          continue;
        }
        const float m_use = (m_run[nt][jj] == -CUDART_INF_F) ? 0.f : m_run[nt][jj];
        pr[jj] = fast_exp2(sc[nt][jj] - m_use);
        pr[jj + 2] = fast_exp2(sc[nt][jj + 2] - m_use);
        l_run[nt][jj] += pr[jj] + pr[jj + 2];
      }
      // V scales fold into P (a masked token's P is 0: keep its factor finite)
      const float fva = (all || va) ? rva : 0.f, fvb = (all || vb) ? rvb : 0.f;
      bh[nt][0] = movmatrix_trans(pack_f16(pr[0] * fva, pr[1] * fva));
      bh[nt][1] = movmatrix_trans(pack_f16(pr[2] * fvb, pr[3] * fvb));
    }

    // ---- O^T[d][head] += V^T * P^T
#pragma unroll
    for (int mp = 0; mp < MT / 2; ++mp) {
      // vf[mp] transposed: a register holds bytes (t 2t, d 2g) (2t, 2g+1)
      // (2t+1, 2g) (2t+1, 2g+1); rows m <-> d: m = g -> 16c + 2g,
      // m = g + 8 -> 16c + 2g + 1
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a0, a1, a2, a3;
        if constexpr (I8) {
          const uint32_t top = vf[mp][2 * h] ^ 0x80808080u, bot = vf[mp][2 * h + 1] ^ 0x80808080u;
          a0 = i8pair_to_f16x2_biased<0x4240>(top);
          a1 = i8pair_to_f16x2_biased<0x4341>(top);
          a2 = i8pair_to_f16x2_biased<0x4240>(bot);
          a3 = i8pair_to_f16x2_biased<0x4341>(bot);
        } else {
          a0 = e4m3pair_to_f16x2<0x0020>(vf[mp][2 * h]);
          a1 = e4m3pair_to_f16x2<0x0031>(vf[mp][2 * h]);
          a2 = e4m3pair_to_f16x2<0x0020>(vf[mp][2 * h + 1]);
          a3 = e4m3pair_to_f16x2<0x0031>(vf[mp][2 * h + 1]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_f16(o[2 * mp + h][nt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
      }
    }
    if constexpr (I8) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_f16(o1[nt], kOnes, kOnes, kOnes, kOnes, bh[nt][0], bh[nt][1]);
    }
  }
  cp_async_wait<0>();

  if constexpr (I8) {
    // O carries 1152 * sum_t P[t][h] from the biased V codes: remove it (every
    // row of o1 holds the column sums, so a thread's own registers suffice).
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[mt][nt][j] -= 1152.f * o1[nt][j];
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
        const int d = 16 * mt + (m < 8 ? 2 * m : 2 * (m - 8) + 1);
        s_o[(warp * GP + h) * HD + d] = o[mt][nt][j];
      }
  combine_and_store<HD, NWARPS, GP>(p, c, s_m, s_l, s_o, s_w, s_L);
}

// Dynamic shared memory of a launch.  Kernels at head_dim 128 are held to three
// CTAs per SM: with the stage ring alone, four fit where registers allow, but
// the cache streamed faster with three CTAs' stages in flight per SM (6.6 TB/s
// against 6.1 TB/s, measured without the math), and the split planner's
// occupancy figure stays exact.
template <int HD, class Cfg>
int q8_smem(int phys_bytes) {
  const int smem = phys_bytes + Cfg::BODY;
  if constexpr (HD == 128 && PKV_Q8_HOLD3) return smem > kThreeCtaSmem ? smem : kThreeCtaSmem;
  return smem;
}

template <int HD, int QM, int NT, bool MHA>
cudaError_t launch_q8_kernel(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  using Cfg = Q8Cfg<HD, NT, kQ8Warps, kQ8Stages>;
  const int smem = q8_smem<HD, Cfg>(p.phys_bytes);
  constexpr auto k = decode_q8_kernel<HD, QM, NT, kQ8Warps, kQ8Stages, MHA>;
  cudaError_t e = prepare<k>(smem);
  if (e != cudaSuccess) return e;
  k<<<grid, kQ8Warps * kWarp, smem, st>>>(p);
  return cudaGetLastError();
}

// q-head tiling: two n-tiles for groups above 8, the MHA form for a group of
// one, else one n-tile.
template <int HD, int QM>
cudaError_t launch_q8_group(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  if (p.group > 8) return launch_q8_kernel<HD, QM, 2, false>(p, grid, st);
  if (p.group == 1) return launch_q8_kernel<HD, QM, 1, true>(p, grid, st);
  return launch_q8_kernel<HD, QM, 1, false>(p, grid, st);
}

template <int HD, int QM>
int q8_occupancy() {
  static std::atomic<int> cached[kMaxDevices];  // resident CTAs per SM, 0 = not yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
  int n = cached[dev].load(std::memory_order_acquire);
  if (n > 0) return n;
  using Cfg = Q8Cfg<HD, 1, kQ8Warps, kQ8Stages>;
  constexpr int kTypicalPhysBytes = 1024;  // block-table slice of a typical split
  constexpr auto k = decode_q8_kernel<HD, QM, 1, kQ8Warps, kQ8Stages, false>;
  const int smem = q8_smem<HD, Cfg>(kTypicalPhysBytes);
  if (prepare<k>(smem) != cudaSuccess) return 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kQ8Warps * kWarp, smem) !=
          cudaSuccess ||
      n < 1)
    n = 1;
  cached[dev].store(n, std::memory_order_release);
  return n;
}

}  // namespace

cudaError_t launch_decode_q8(const DecodeParams& p, pkv_dtype cache_dt, int head_dim,
                             cudaStream_t st) {
  dim3 grid(p.num_kv_heads, p.num_seqs, p.num_splits);
  if (cache_dt == PKV_I8)
    return head_dim == 128 ? launch_q8_group<128, kQuantI8>(p, grid, st)
                           : launch_q8_group<64, kQuantI8>(p, grid, st);
  return head_dim == 128 ? launch_q8_group<128, kQuantFp8>(p, grid, st)
                         : launch_q8_group<64, kQuantFp8>(p, grid, st);
}

int decode_q8_ctas_per_sm(pkv_dtype cache_dt, int head_dim) {
  if (cache_dt == PKV_I8)
    return head_dim == 128 ? q8_occupancy<128, kQuantI8>() : q8_occupancy<64, kQuantI8>();
  return head_dim == 128 ? q8_occupancy<128, kQuantFp8>() : q8_occupancy<64, kQuantFp8>();
}

}  // namespace pkv
