// Shared-prefix (cascade) pass of paged decode attention, bf16 caches.
//
// Prefix caching ("生产级 LLM 推理的 KV 缓存优化" (GPUYard), the serving-flags
// section: --enable-prefix-caching avoids recomputing shared prompt prefixes;
// "LLM推理显存优化KV Cache管理3大策略" §2: blocks carry a ref_count so that
// sequences can share them) lets many sequences point at the same physical
// blocks for their common first tokens.  A per-sequence decode reads those
// blocks once per sequence.  This pass reads them once per KV head for all
// sequences: for KV head h and a slice of the prefix it computes, for every
// (sequence, q head of h's group) row, the attention of that q row over the
// slice, and writes the normalised partial (o, log2-sum-exp) into the split
// workspace.  The per-sequence suffix runs through the split decode kernel
// from token prefix_len on, and the merge kernel combines both exactly.
//
// The rows of one KV head form a dense contraction: S = Q K^T with M = rows
// (num_seqs * group), N = prefix tokens, K = head_dim, then O = P V.  Each warp
// owns 16 rows; all warps share the K/V stages of the slice in shared memory
// (cp.async, swizzled).  mma.sync m16n8k16 computes S from the warp's q
// fragments, the accumulators are re-packed in place as the A operand of the
// PV product (hi + lo bf16 halves, ~16 bits of P), fp32 online softmax per
// row.
#include <math_constants.h>

#include "common.cuh"
#include "decode.cuh"

namespace pkv {

namespace {

template <int HD, int NWARPS, int PT, int NSTAGES>
struct PrefixCfg {
  static constexpr int ROWB = HD * 2;
  static constexpr int CH = ROWB / 16;
  static constexpr int TILE = PT * ROWB;  // bytes of the K (or V) rows of one stage
  static constexpr int STAGE = 2 * TILE;
  static constexpr int THREADS = NWARPS * kWarp;
  static constexpr int CHUNKS = PT * CH;  // 16-byte chunks per K (or V) stage
  static constexpr int PER_THREAD = CHUNKS / THREADS;
  static constexpr int ROWS = NWARPS * 16;  // q rows per CTA
  static_assert(CHUNKS % THREADS == 0, "stage copies must split evenly over the threads");
  static_assert(PT % 16 == 0, "stages hold whole 16-token tiles");
};

template <int HD, int NWARPS, int PT, int NSTAGES>
__global__ void __launch_bounds__(NWARPS * kWarp)
    prefix_kernel(const DecodeParams p, const PrefixParams pp) {
  using Cfg = PrefixCfg<HD, NWARPS, PT, NSTAGES>;
  constexpr int CH = Cfg::CH;
  constexpr int KS = HD / 16;   // k-steps of the score mma
  constexpr int NTD = HD / 8;   // 8-wide head_dim tiles of the output
  extern __shared__ __align__(128) uint8_t smem[];
  int* s_phys = reinterpret_cast<int*>(smem);
  const uint32_t ring = smem_u32(smem + pp.phys_bytes);

  const int kvh = blockIdx.x, split = blockIdx.y, rg = blockIdx.z;
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int g = lane >> 2, t4 = lane & 3;
  const int G = p.group;
  const int t0 = split * pp.pchunk;
  const int t1 = min(pp.prefix_len, t0 + pp.pchunk);
  const int bs = p.block_size;
  const int blk0 = t0 >> p.log2_bs;

  // prefix blocks of this slice, from sequence 0's table (shared by all)
  {
    const int nphys = ((t1 - 1) >> p.log2_bs) - blk0 + 1;
    for (int i = threadIdx.x; i < nphys; i += Cfg::THREADS) {
      int b = p.block_tables[blk0 + i];
      if (b < 0 || b >= p.num_blocks) {
        set_flag(p.err_flag, PKV_FLAG_BAD_BLOCK);
        b = -1;
      }
      s_phys[i] = b;
    }
  }

  // this thread's two q rows and how far into the prefix each may look
  int lim[2];
  size_t qrow[2];
  bool rvalid[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = rg * Cfg::ROWS + warp * 16 + g + 8 * i;
    rvalid[i] = r < pp.rows;
    const int seq = rvalid[i] ? r / G : 0;
    const int qh = kvh * G + (rvalid[i] ? r % G : 0);
    qrow[i] = (size_t)seq * p.num_q_heads + qh;
    int ctx = rvalid[i] ? p.context_lens[seq] : 0;
    ctx = ctx < 0 ? 0 : ctx;
    lim[i] = rvalid[i] ? min(ctx, pp.prefix_len) : 0;
  }
  uint32_t qa[KS][4];
  {
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        uint32_t lo = 0, hi = 0;
        if (rvalid[i]) {
          const __nv_bfloat16* qr = qb + qrow[i] * HD + 16 * ks + 2 * t4;
          lo = *reinterpret_cast<const uint32_t*>(qr);
          hi = *reinterpret_cast<const uint32_t*>(qr + 8);
        }
        qa[ks][i] = lo;      // a0 (row g), a1 (row g + 8)
        qa[ks][2 + i] = hi;  // a2, a3: head_dim + 8
      }
    }
  }
  __syncthreads();

  float o[NTD][4];
#pragma unroll
  for (int n = 0; n < NTD; ++n)
#pragma unroll
    for (int j = 0; j < 4; ++j) o[n][j] = 0.f;
  float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_run[2] = {0.f, 0.f};

  // cooperative stage copies: chunk c = tid + THREADS * i -> row c / CH, chunk c % CH
  const uint8_t* kb = static_cast<const uint8_t*>(p.k_cache);
  const uint8_t* vb = static_cast<const uint8_t*>(p.v_cache);
  const size_t tok_stride = (size_t)p.num_kv_heads * Cfg::ROWB;
  auto issue_stage = [&](int tt, uint32_t st) {
#pragma unroll
    for (int i = 0; i < Cfg::PER_THREAD; ++i) {
      const int c = threadIdx.x + Cfg::THREADS * i;
      const int row = c / CH, ch = c % CH;
      const int t = tt + row;
      const int phys = t < t1 ? s_phys[(t >> p.log2_bs) - blk0] : -1;
      size_t off = 0;
      int n = 0;
      if (phys >= 0) {
        off = ((size_t)phys * bs + (t & (bs - 1))) * tok_stride + (size_t)kvh * Cfg::ROWB +
              (size_t)ch * 16;
        n = 16;
      }
      const uint32_t so = (uint32_t)swz<CH>(row, ch) * 16;
      cp_async_16(st + so, kb + off, n);
      cp_async_16(st + Cfg::TILE + so, vb + off, n);
    }
    cp_async_commit();
  };

  const int nst = (t1 - t0 + PT - 1) / PT;
#pragma unroll
  for (int i = 0; i < NSTAGES - 1; ++i) {
    if (i < nst)
      issue_stage(t0 + i * PT, ring + (uint32_t)(i * Cfg::STAGE));
    else
      cp_async_commit();
  }

  // ldmatrix lane addressing (matrix j = lane / 8 supplies its row lane % 8).
  // A row 16 * j + r of a stage has the swizzle of row r (16 * j keeps r & 7),
  // so the per-lane offsets inside a 16-token tile are fixed.
  const int kr = (lane & 7) + ((lane >> 4) & 1) * 8, kc = (lane >> 3) & 1;  // K: b0,b1 of 2 n-tiles
  const int vr = (lane & 7) + ((lane >> 3) & 1) * 8, vc = lane >> 4;        // V^T: 2 n-tiles
  uint32_t koff[KS], voff[NTD / 2];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) koff[ks] = (uint32_t)swz<CH>(kr, 2 * ks + kc) * 16;
#pragma unroll
  for (int dp = 0; dp < NTD / 2; ++dp) voff[dp] = (uint32_t)swz<CH>(vr, 2 * dp + vc) * 16;
  constexpr uint32_t kTileBytes = 16 * Cfg::ROWB;  // one 16-token tile of K (or V)

  for (int s = 0; s < nst; ++s) {
    {
      const int nx = s + NSTAGES - 1;
      if (nx < nst)
        issue_stage(t0 + nx * PT, ring + (uint32_t)((nx % NSTAGES) * Cfg::STAGE));
      else
        cp_async_commit();
    }
    cp_async_wait<NSTAGES - 1>();
    __syncthreads();
    const uint32_t kS = ring + (uint32_t)((s % NSTAGES) * Cfg::STAGE);
    const uint32_t vS = kS + Cfg::TILE;
    const int tt = t0 + s * PT;
#pragma unroll 1
    for (int j = 0; j < PT / 16; ++j) {
      const int tj = tt + 16 * j;
      // which of the 16 tokens exist (inside the slice, in a good block)
      const int tl = tj + (lane & 15);
      const bool tv = tl < t1 && s_phys[(tl >> p.log2_bs) - blk0] >= 0;
      const uint32_t tmask = __ballot_sync(0xffffffffu, tv) & 0xFFFFu;

      // ---- S[row][token] = Q K^T, two 8-token n-tiles (even and odd k-steps in
      // separate accumulators to halve the dependent mma chains)
      float acc[2][2][4] = {};
      const uint32_t kT = kS + (uint32_t)j * kTileBytes;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t b0, b1, b2, b3;  // (tok 0-7, c) (tok 0-7, c+1) (tok 8-15, c) (tok 8-15, c+1)
        ldmatrix_x4(kT + koff[ks], b0, b1, b2, b3);
        mma_bf16(acc[ks & 1][0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
        mma_bf16(acc[ks & 1][1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
      }
      // ---- mask, online softmax per row (rows g, g + 8; tokens 8nt + 2t4 + e)
      const bool full = __all_sync(0xffffffffu, tmask == 0xFFFFu && tj + 16 <= lim[0] &&
                                                    tj + 16 <= lim[1]);
      float sv[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = (acc[0][nt][e] + acc[1][nt][e]) * p.scale_log2;
          if (full) {
            sv[nt][e] = x;
          } else {
            const int col = 8 * nt + 2 * t4 + (e & 1);
            const bool ok = ((tmask >> col) & 1u) && (tj + col < lim[e >> 1]);
            sv[nt][e] = ok ? x : -CUDART_INF_F;
          }
        }
      float alpha[2];
      bool rescale = false;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float mx = fmaxf(fmaxf(sv[0][2 * i], sv[0][2 * i + 1]), fmaxf(sv[1][2 * i], sv[1][2 * i + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run[i], mx);
        const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
        alpha[i] = fast_exp2(m_run[i] - m_use);
        rescale |= alpha[i] != 1.f;
        m_run[i] = m_new;
        float rs = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float pv = fast_exp2(sv[nt][2 * i + e] - m_use);
            sv[nt][2 * i + e] = pv;
            rs += pv;
          }
        l_run[i] = l_run[i] * alpha[i] + rs;
      }
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int n = 0; n < NTD; ++n) {
          o[n][0] *= alpha[0];
          o[n][1] *= alpha[0];
          o[n][2] *= alpha[1];
          o[n][3] *= alpha[1];
        }
      }
      // ---- P as the A operand (rows x 16 tokens), hi + lo bf16 halves
      uint32_t ph[4], pl[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float x0 = sv[nt][2 * i], x1 = sv[nt][2 * i + 1];
          const uint32_t h = pack_bf16(x0, x1);
          const float2 f = unpack_bf16(h);
          ph[2 * nt + i] = h;  // a0: (g, 0-7) a1: (g+8, 0-7) a2: (g, 8-15) a3: (g+8, 8-15)
          pl[2 * nt + i] = pack_bf16(x0 - f.x, x1 - f.y);
        }
      // ---- O[row][d] += P V
#pragma unroll
      for (int dp = 0; dp < NTD / 2; ++dp) {
        uint32_t b0, b1, b2, b3;  // (tok 0-7, c) (tok 8-15, c) (tok 0-7, c+1) (tok 8-15, c+1)
        ldmatrix_x4_trans(vS + (uint32_t)j * kTileBytes + voff[dp], b0, b1, b2, b3);
        mma_bf16(o[2 * dp], ph[0], ph[1], ph[2], ph[3], b0, b1);
        mma_bf16(o[2 * dp], pl[0], pl[1], pl[2], pl[3], b0, b1);
        mma_bf16(o[2 * dp + 1], ph[0], ph[1], ph[2], ph[3], b2, b3);
        mma_bf16(o[2 * dp + 1], pl[0], pl[1], pl[2], pl[3], b2, b3);
      }
    }
    __syncthreads();  // the stage is refilled by the next iteration's copies
  }
  cp_async_wait<0>();

  // ---- normalise and write this slice's partial for the valid rows
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float l = l_run[i];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (!rvalid[i]) continue;
    const size_t slot = qrow[i] * p.ws_slots + split;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* dst = p.ws_o + slot * HD;
#pragma unroll
    for (int n = 0; n < NTD; ++n) {
      float2 v2 = make_float2(o[n][2 * i] * inv, o[n][2 * i + 1] * inv);
      *reinterpret_cast<float2*>(dst + 8 * n + 2 * t4) = v2;
    }
    if (t4 == 0) p.ws_lse[slot] = l > 0.f ? m_run[i] + log2f(l) : -CUDART_INF_F;
  }
}

template <int HD, int NWARPS, int PT, int NSTAGES>
cudaError_t launch(const DecodeParams& p, const PrefixParams& pp, cudaStream_t st) {
  using Cfg = PrefixCfg<HD, NWARPS, PT, NSTAGES>;
  const int smem = pp.phys_bytes + NSTAGES * Cfg::STAGE;
  auto k = prefix_kernel<HD, NWARPS, PT, NSTAGES>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(p.num_kv_heads, pp.prefix_splits, (pp.rows + Cfg::ROWS - 1) / Cfg::ROWS);
  k<<<grid, Cfg::THREADS, smem, st>>>(p, pp);
  return cudaGetLastError();
}

}  // namespace

int prefix_rows_per_cta() { return PrefixCfg<128, kPrefixWarps, kPrefixTokens, 2>::ROWS; }

cudaError_t launch_prefix(const DecodeParams& p, const PrefixParams& pp, int head_dim,
                          cudaStream_t st) {
  if (head_dim == 128) return launch<128, kPrefixWarps, kPrefixTokens, 2>(p, pp, st);
  return launch<64, kPrefixWarps, kPrefixTokens, 2>(p, pp, st);
}

}  // namespace pkv
